// decode.cu -- persistent split-KV flash decoding for R-SWA and SR-SWA on sm_100a.
//
// Work is cut into items (sequence, head, split); an item is a fixed run of
// 32-row K/V tiles of one (sequence, head). R-SWA tiles are the prefix rows
// [0, m) ("百度Unlimited OCR" paper summary §二.1: the reference prefix is
// always visible) followed by the ring's valid slots (at most two contiguous
// slot ranges). SR-SWA tiles are the routed 32-token blocks, each with its
// log-probability bias (Unlimited-OCR-2 SR-SWA explainer, 稀疏路由 step 4,
// 偏置融合), followed by the ring. Tiles past a (sequence, head)'s end are
// empty.
//
// The path is HBM-bound (about 1 FLOP per byte), so the kernel spends its
// effort on bytes in flight, not on tensor cores:
//  * the grid is one wave of resident CTAs (two per SM); each walks its items
//    in turn. Every warp owns one 16 KiB shared-memory stage (8 KiB of K and
//    8 KiB of V) and streams its own tiles through it with cp.async.bulk: the
//    CTA-local tiles w, w + 6, w + 12, ... belong to warp w, and right after a
//    warp has read a tile it issues the copy of its next one into the same
//    stage, across item boundaries, so there is no producer hand-over on the
//    refill path and the six copies of a CTA's first tiles start at once;
//  * in a warp, lane (g, c) holds dims 8c..8c+7 and rows 2j+g; the 16 partial
//    dot products of a half-warp are reduce-scattered in 15 shuffles, the
//    online softmax runs in the exp2 domain, and P.V broadcasts each row's
//    weight with a shuffle; dots and accumulators use paired f32 FMAs
//    (fma.rn.f32x2), and full tiles skip the per-row bounds checks;
//  * at the end of an item the warps merge through shared memory and either
//    write the output (one split) or a (max, sum, acc) partial; the last item
//    of a (sequence, head) to finish (atomic counter) merges the partials by
//    log-sum-exp and resets the counter.
// The split count is chosen per launch to minimise the busiest CTA's tile count.
//
// The same kernel serves, as compile-time variants: an FP8 (E4M3) prefix with block
// scales (a prefix tile is 128-byte code rows); the fused decode step (this step's token
// is read as a one-row tile and written into its ring slot inside the launch, whose last
// CTA advances wp / fill); and the SR-SWA chunked prefill (items are single queries of a
// chunk, whose key sets end with their causal band of the chunk's outputs).
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include <cmath>

#include "common.cuh"
#include "internal.h"

namespace rswa {

namespace {

#ifndef RSWA_DECODE_WARPS
#define RSWA_DECODE_WARPS 6
#endif
#ifndef RSWA_DECODE_STAGES_PER_WARP
#define RSWA_DECODE_STAGES_PER_WARP 1
#endif
// CTA-local tile li goes to warp li % kWarps; the warp's k-th tile uses its stage
// warp * kStagesPerWarp + k % kStagesPerWarp. A stage has a single owner warp,
// which tracks the stage's mbarrier phase itself (empty tiles issue no copy).
constexpr int kWarps = RSWA_DECODE_WARPS;
constexpr int kStagesPerWarp = RSWA_DECODE_STAGES_PER_WARP;
constexpr int kStages = kWarps * kStagesPerWarp;
constexpr int kDecodeThreads = kWarps * 32;
static_assert(kStagesPerWarp >= 1 && kStagesPerWarp <= 4, "stages per warp");
constexpr int kTileBytes = kBlock * kRowBytes;  // 8 KiB
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

struct DecodeSmem {
  uint8_t stage[kStages][2][kTileBytes];
  uint64_t full[kStages];
  float wm[kWarps];
  float wl[kWarps];
  float wacc[kWarps][kHeadDim];
  int is_last;
  // fused router: block reductions of a finalising CTA
  float fin_red[kWarps];
  float fin_red2[kWarps];
  int fin_redi[kWarps];
  int fin_n;
  int fin_ok;
  // page2d encoding in the fused step: the 64 pair frequencies base^(-i/64), fp64
  double rope_th[kHeadDim / 2];
};

constexpr int kDecodeMinBlocks =
    (227 * 1024) / (int)sizeof(DecodeSmem) > 0 ? (227 * 1024) / (int)sizeof(DecodeSmem) : 1;

// What a launch computes besides plain decode: nothing, the fused ring append, or the
// chunked-prefill band. A compile-time mode, so each kernel carries only its own state.
constexpr int kModeDecode = 0;
constexpr int kModeAppend = 1;
constexpr int kModeBand = 2;
constexpr int kModeRing8 = 3;  // plain decode over an FP8 prefix and an FP8 ring (row scales)
constexpr int kModeRoute = 4;        // SR-SWA with the router fused into the launch (ring as given)
constexpr int kModeRouteAppend = 5;  // SR-SWA with the router and the ring append fused: one launch per step

__host__ __device__ constexpr bool mode_appends(int m) { return m == kModeAppend || m == kModeRouteAppend; }
__host__ __device__ constexpr bool mode_routes(int m) { return m == kModeRoute || m == kModeRouteAppend; }

constexpr int kSlice = 64;        // blocks per router slice (one warp scores a slice)
constexpr int kNoBlock = 0x7fffffff;

// What a warp needs to enumerate a (sequence, head)'s tiles.
struct SeqView {
  const uint8_t* pk;  // prefix rows of this (b, h): bf16 rows, or E4M3 code rows (FP8 prefix)
  const uint8_t* pv;
  const float* ks;    // FP8 prefix: this (b, h)'s block scales
  const float* vs;
  const uint16_t* rk;  // ring rows of this (b, h)
  const uint16_t* rv;
  const uint8_t* rk8;  // FP8 ring: code rows of this (b, h) and their row scales
  const uint8_t* rv8;
  const float* rks;
  const float* rvs;
  const uint16_t* bk;  // chunked prefill: the query's causal band of output rows (null for decode)
  const uint16_t* bv;
  int m;               // valid prefix rows
  int nb;              // prefix blocks
  int n_first;         // tiles before the ring (prefix tiles, or topk route entries)
  int a0, len0, len1;  // ring slot ranges [a0, a0+len0) and [0, len1)
  int n_r0, n_r1;
  int blen, n_band;    // band rows and tiles (chunked prefill)
  int n_new;           // fused append: 1 (this step's token, the last tile) or 0
  const uint16_t* nk;  // fused append: this step's K / V row of (b, h)
  const uint16_t* nv;
  uint16_t* wk;        // fused append: ring slot wp[b] of (b, h), where the row is written
  uint16_t* wv;
  int32_t* slot_out;   // fused append: &slot_out[b] for head 0, else null
  int wslot;
  int skip_slot;       // fused append on a full ring: slot wp[b], read but masked (-1: none)
  int total;
};

// The key set of query i of (b, h) (i = 0 for decode). Decode: the prefix (or routed
// blocks) and the ring's valid slots. Chunked prefill: the routed blocks, the outputs
// j with i - n < j <= i of the chunk (the band) and, for j < 0, the previous chunk's
// last outputs from the ring: the min(n - 1 - i, fill) most recently written slots.
template <bool kSparse, bool kFp8, int kMode>
__device__ __forceinline__ SeqView make_view(const DecodeArgs& a, int b, int h, int i, bool report) {
  SeqView v;
  const int64_t bh = (int64_t)b * a.H + h;
  const bool band = kMode == kModeBand;
  int m = a.prefix_len[b];
  if (m < 0 || m > a.cap) {
    if (report) set_status(a.status, RSWA_DEVICE_BAD_PREFIX_LEN);
    m = 0;
  }
  int w = 0, f = 0;
  bool ring_ok = false;
  if ((kMode == kModeRing8 ? (const void*)a.ring_k8 : (const void*)a.ring_k) != nullptr) {
    w = a.wp[b];
    f = a.fill[b];
    ring_ok = w >= 0 && w < a.n && f >= 0 && f <= a.n;
    if (!ring_ok) {
      if (report) set_status(a.status, RSWA_DEVICE_BAD_RING_STATE);
      w = 0;
      f = 0;
    }
  }
  if (kFp8) {
    v.pk = a.pk8 + bh * a.cap * kHeadDim;
    v.pv = a.pv8 + bh * a.cap * kHeadDim;
    v.ks = a.kscale + bh * a.nb_cap;
    v.vs = a.vscale + bh * a.nb_cap;
  } else {
    v.pk = reinterpret_cast<const uint8_t*>(a.pk + bh * a.cap * kHeadDim);
    v.pv = reinterpret_cast<const uint8_t*>(a.pv + bh * a.cap * kHeadDim);
    v.ks = v.vs = nullptr;
  }
  v.rk = a.ring_k ? a.ring_k + bh * a.n * kHeadDim : nullptr;
  v.rv = a.ring_v ? a.ring_v + bh * a.n * kHeadDim : nullptr;
  if (kMode == kModeRing8) {
    v.rk8 = a.ring_k8 + bh * a.n * kHeadDim;
    v.rv8 = a.ring_v8 + bh * a.n * kHeadDim;
    v.rks = a.ring_ks + bh * a.n;
    v.rvs = a.ring_vs + bh * a.n;
  } else {
    v.rk8 = v.rv8 = nullptr;
    v.rks = v.rvs = nullptr;
  }
  v.m = m;
  v.nb = (m + kBlock - 1) / kBlock;
  int cnt = f;  // ring slots read: the cnt most recently written, (w - cnt + i) mod n for i < cnt
  if (band) cnt = min(max(a.n - 1 - i, 0), f);
  // fused append: the oldest slot of a full ring (slot w) is overwritten by this step's token,
  // which is read from k_new / v_new as the item's first tile instead
  // (a sequence with a bad ring state is left untouched, as rswa_append leaves it). A full
  // ring is still read as [0, n) in aligned tiles, with the overwritten slot masked: the bulk
  // copy of the tile holding slot w may read that row while the token's warp writes it (an
  // unsynchronised cross-proxy read and write of one row), and the mask keeps whatever it
  // reads out of every score and of P.V.
  const bool app = mode_appends(kMode) && ring_ok;
  // a full ring is read as [0, n)
  int a0 = cnt == a.n ? 0 : (w - cnt) % a.n;
  if (a0 < 0) a0 += a.n;
  v.a0 = a0;
  v.len0 = min(cnt, a.n - a0);
  v.len1 = cnt - v.len0;
  v.n_r0 = (v.len0 + kBlock - 1) / kBlock;
  v.n_r1 = (v.len1 + kBlock - 1) / kBlock;
  v.n_first = kSparse ? a.topk : v.nb;
  v.bk = v.bv = nullptr;
  v.blen = v.n_band = 0;
  if (band) {
    const int start = max(0, i - a.n + 1);
    v.blen = i - start + 1;
    v.n_band = (v.blen + kBlock - 1) / kBlock;
    v.bk = a.k_out + (bh * a.T + start) * kHeadDim;
    v.bv = a.v_out + (bh * a.T + start) * kHeadDim;
  }
  v.n_new = app ? 1 : 0;
  v.wslot = w;
  v.skip_slot = (app && f == a.n) ? w : -1;
  v.nk = v.nv = nullptr;
  v.wk = v.wv = nullptr;
  v.slot_out = nullptr;
  if (app) {
    v.nk = a.k_new + bh * kHeadDim;
    v.nv = a.v_new + bh * kHeadDim;
    v.wk = a.ring_k_w + (bh * a.n + w) * kHeadDim;
    v.wv = a.ring_v_w + (bh * a.n + w) * kHeadDim;
    if (h == 0 && a.slot_out) v.slot_out = a.slot_out + b;
  }
  v.total = v.n_first + v.n_r0 + v.n_r1 + v.n_band + v.n_new;
  return v;
}

// Tile t of a (b, h): where its K and V rows start, how many rows (0 = empty tile), the
// log2 bias, and the prefix block it covers (-1 for a ring tile, -2 for the fused append's
// token). For SR-SWA, (c, lp) is the route entry of the tile. Order: [the fused append's
// token] [prefix tiles or routed blocks] [ring ranges] [chunked-prefill band]; with the router
// fused: [the fused append's token] [ring ranges] [routed blocks], route-independent tiles first.
struct TileRef {
  const uint8_t* k;
  const uint8_t* v;
  int rows;
  float bias;
  int blk;
  int skip;        // a row of the tile to leave out (-1: none)
  const float* rs_k;  // FP8 ring tile: the row scales of its first row (null otherwise)
  const float* rs_v;
};

// Prefix tile t of a (b, h) (R-SWA), or its t-th routed block with route entry (c, lp) (SR-SWA).
template <bool kSparse, bool kFp8>
__device__ __forceinline__ TileRef first_tile(const SeqView& v, int t, int c, float lp, int32_t* status, TileRef r) {
  int blk;
  if (kSparse) {
    if (c < 0 || !(lp > -INFINITY)) return r;
    if (c >= v.nb) {
      set_status(status, RSWA_DEVICE_BAD_BLOCK_IDX);
      return r;
    }
    blk = c;
    r.bias = lp * kLog2e;
  } else {
    blk = t;
  }
  const int start = blk * kBlock;
  const int64_t row_bytes = kFp8 ? kHeadDim : kRowBytes;
  r.rows = min(kBlock, v.m - start);
  r.k = v.pk + (int64_t)start * row_bytes;
  r.v = v.pv + (int64_t)start * row_bytes;
  r.blk = blk;
  return r;
}

// Ring tile t of a (b, h): the first slot range, then the second.
template <int kMode>
__device__ __forceinline__ TileRef ring_tile(const SeqView& v, int t, TileRef r) {
  int start, len;
  if (t < v.n_r0) {
    start = v.a0 + t * kBlock;
    len = v.len0 - t * kBlock;
  } else {
    t -= v.n_r0;
    start = t * kBlock;
    len = v.len1 - t * kBlock;
  }
  r.rows = min(kBlock, len);
  if (kMode == kModeRing8) {
    r.k = v.rk8 + (int64_t)start * kHeadDim;
    r.v = v.rv8 + (int64_t)start * kHeadDim;
    r.rs_k = v.rks + start;
    r.rs_v = v.rvs + start;
    return r;
  }
  r.k = reinterpret_cast<const uint8_t*>(v.rk + (int64_t)start * kHeadDim);
  r.v = reinterpret_cast<const uint8_t*>(v.rv + (int64_t)start * kHeadDim);
  if (v.skip_slot >= start && v.skip_slot < start + r.rows) r.skip = v.skip_slot - start;
  return r;
}

template <bool kSparse, bool kFp8, int kMode>
__device__ __forceinline__ TileRef tile_at(const SeqView& v, int t, int c, float lp, int32_t* status) {
  TileRef r;
  r.bias = 0.f;
  r.k = r.v = v.pk;
  r.rows = 0;
  r.blk = -1;
  r.skip = -1;
  r.rs_k = r.rs_v = nullptr;
  if (t >= v.total) return r;
  if (mode_appends(kMode) && v.n_new) {  // fused append: this step's token comes first (no bias)
    if (t == 0) {
      r.rows = 1;
      r.k = reinterpret_cast<const uint8_t*>(v.nk);
      r.v = reinterpret_cast<const uint8_t*>(v.nv);
      r.blk = -2;
      return r;
    }
    t -= 1;
  }
  const int n_ring = v.n_r0 + v.n_r1;
  if (mode_routes(kMode)) {  // fused router: the ring before the routed blocks, which wait for the route
    if (t < n_ring) return ring_tile<kMode>(v, t, r);
    return first_tile<kSparse, kFp8>(v, t - n_ring, c, lp, status, r);
  }
  if (t < v.n_first) return first_tile<kSparse, kFp8>(v, t, c, lp, status, r);
  t -= v.n_first;
  if (t >= n_ring) {  // the causal band of a chunked-prefill query
    t -= n_ring;
    r.rows = min(kBlock, v.blen - t * kBlock);
    r.k = reinterpret_cast<const uint8_t*>(v.bk + (int64_t)t * kBlock * kHeadDim);
    r.v = reinterpret_cast<const uint8_t*>(v.bv + (int64_t)t * kBlock * kHeadDim);
    return r;
  }
  return ring_tile<kMode>(v, t, r);
}

// An item (sequence, head, split) as one warp sees it while issuing its tiles:
// the (sequence, head) view, the split's first tile and this lane's route entry.
struct ItemView {
  int item;  // -1: none loaded yet
  int t0;
  int b;
  bool routed;  // (c, lp) hold the route (fused router: read once the route is published)
  int rope_tok, rope_pg;  // fused step with the page2d encoding: the sequence's positions
  SeqView v;
  int c;
  float lp;
};

// Items are (query, split) with query vq = (b * H + h) * T + i.
template <bool kSparse, bool kFp8, int kMode>
__device__ __forceinline__ void load_item(const DecodeArgs& a, int item, int lane, ItemView& iv) {
  const int vq = item / a.splits, split = item - vq * a.splits;
  const int bh = vq / a.T, i = vq - bh * a.T;
  const int b = bh / a.H, h = bh - b * a.H;
  iv.item = item;
  iv.t0 = split * a.tiles_per_item;
  iv.b = b;
  if (mode_appends(kMode) && a.rope_tok != nullptr && split == 0) {  // loaded beside the view's reads
    iv.rope_tok = a.rope_tok[b];
    iv.rope_pg = a.rope_page[b];
  }
  iv.v = make_view<kSparse, kFp8, kMode>(a, b, h, i, lane == 0 && split == 0 && h == 0 && i == 0);
  iv.c = -1;
  iv.lp = -INFINITY;
  iv.routed = !mode_routes(kMode);  // the fused router's route is read when a routed tile needs it
  if (kSparse && !mode_routes(kMode) && lane < a.topk) {
    const int64_t ri = ((int64_t)b * a.T + i) * a.topk + lane;  // the route of query i of sequence b
    iv.c = a.blk_idx[ri];
    iv.lp = a.blk_logp[ri];
  }
}

// A tile in flight: its row count (0: nothing issued), bias, and for an FP8 tile its K / V
// scales (loaded at issue time, used at consume time): a prefix tile's block scales, or, for
// an FP8 ring tile, the scales of the row whose score this lane ends up holding (2c + g).
struct InFlight {
  int rows;
  bool armed;     // a copy was issued for it (false only for the tile a wait-timeout test drops)
  bool deferred;  // fused router: a routed tile not issued yet (its route was not to be waited for)
  int skip;
  float bias;
  bool fp8;
  float ks, vs;
};

__device__ __forceinline__ int ld_acquire_gpu(const int32_t* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// A release increment: a gpu-scope fence (cumulative: it covers the writes this thread has
// observed, e.g. its warp's or CTA's writes before a barrier), then a relaxed atomic add.
__device__ __forceinline__ void red_release_gpu(int32_t* p, int v) {
  asm volatile("fence.acq_rel.gpu;\n\tred.relaxed.gpu.global.add.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// page2d rotary encoding of this step's query and key rows inside the fused step
// (Unlimited-OCR-2 SR-SWA explainer, 2D 位置编码; constants as read for rswa_rope_page2d:
// pair i couples dims i and i + 64 and turns by pos * base^(-i/64), pos = the page number
// when i mod page_mod == page_mod - 1, else the token position; th[i] = base^(-i/64) from
// the CTA's table). Warp-collective: lane l
// takes the fp64 angles and sincos of pairs 2l and 2l + 1, and every lane then gathers the
// cos / sin (rounded to f32) of the eight pairs its 16-byte chunk c = lane & 15 touches,
// pairs 8 (c & 7) + e: the same values, and the same rotation arithmetic below, as the
// stand-alone encoding kernels, so the fused step gives their results bit for bit.
__device__ __forceinline__ void rope_lane_cos_sin(const DecodeArgs& a, const double* th, int tok, int pg, int lane,
                                                  float2 (&cs)[8]) {
  float2 mine[2];
#pragma unroll
  for (int u = 0; u < 2; ++u) {
    const int i = 2 * lane + u;
    const bool on_page = a.rope_page_mod > 0 && i % a.rope_page_mod == a.rope_page_mod - 1;
    double s, c;
    sincos((double)(on_page ? pg : tok) * th[i], &s, &c);
    mine[u] = make_float2((float)c, (float)s);
  }
  const int src = 4 * (lane & 7);  // lane holding pairs 8 (c & 7) + 0, 1
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    cs[e].x = __shfl_sync(0xffffffffu, mine[e & 1].x, src + (e >> 1));
    cs[e].y = __shfl_sync(0xffffffffu, mine[e & 1].y, src + (e >> 1));
  }
}

// Rotates the 16-byte chunk w (dims 8c..8c+7, c = lane & 15, of a row spread over a half
// warp) with its partner chunk c ^ 8, rounding to bf16. Warp-collective (every lane
// shuffles); lanes with rotate == false keep w.
__device__ __forceinline__ uint4 rope_rotate_chunk(uint4 w, const float2 (&cs)[8], int lane, bool rotate) {
  uint32_t own[4] = {w.x, w.y, w.z, w.w};
  uint32_t other[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) other[k] = __shfl_xor_sync(0xffffffffu, own[k], 8);
  if (!rotate) return w;
  const bool first_half = (lane & 8) == 0;  // dims below 64: x of y_i = x_i cos - x_{i+64} sin
  uint32_t r[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const uint32_t lo = first_half ? own[k] : other[k];  // dims i (8 (c & 7) + 2k, + 1)
    const uint32_t hi = first_half ? other[k] : own[k];  // dims i + 64
    const float2 a0 = cs[2 * k], a1 = cs[2 * k + 1];
    const float x0 = bf16lo(lo), x1 = bf16hi(lo), y0 = bf16lo(hi), y1 = bf16hi(hi);
    const __nv_bfloat162 v = first_half
        ? __floats2bfloat162_rn(fmaf(x0, a0.x, -y0 * a0.y), fmaf(x1, a1.x, -y1 * a1.y))
        : __floats2bfloat162_rn(fmaf(y0, a0.x, x0 * a0.y), fmaf(y1, a1.x, x1 * a1.y));
    r[k] = *reinterpret_cast<const uint32_t*>(&v);
  }
  return make_uint4(r[0], r[1], r[2], r[3]);
}

// Fused router: waits (bounded) until the route of the item's sequence is published, then
// gives lane t < topk route entry t. Warp-collective. A wait that gives up sets
// RSWA_DEVICE_WAIT_TIMEOUT and leaves the item without routed blocks.
template <int kMode>
__device__ __forceinline__ void acquire_route(const DecodeArgs& a, ItemView& iv, int lane) {
  const int32_t* flag = a.route_ready + iv.b;
  int ok = 1;
  if (lane == 0 && ld_acquire_gpu(flag) == 0) {
    const uint64_t t0 = global_timer_ns();
    while (ld_acquire_gpu(flag) == 0) {
      if (global_timer_ns() - t0 > a.wait_limit_ns) {
        ok = 0;
        break;
      }
      __nanosleep(64);
    }
  }
  ok = __shfl_sync(0xffffffffu, ok, 0);
  iv.routed = true;
  if (!ok) {
    if (lane == 0) set_status(a.status, RSWA_DEVICE_WAIT_TIMEOUT);
    return;
  }
  (void)ld_acquire_gpu(flag);  // every lane's own acquire before it reads the route
  if (lane < a.topk) {
    iv.c = __ldcg(a.blk_idx_w + (int64_t)iv.b * a.topk + lane);
    iv.lp = __ldcg(a.blk_logp_w + (int64_t)iv.b * a.topk + lane);
  }
}

// Issues CTA-local tile li (if it exists) into stage s: one bulk copy of its K rows and
// one of its V rows on full[s]. Warp-collective. With the router fused, a routed tile whose
// route has not been read yet is deferred (returned unissued) unless can_wait.
template <bool kSparse, bool kFp8, int kMode>
__device__ __forceinline__ InFlight issue_tile(const DecodeArgs& a, DecodeSmem& sm, int li, int s, int lane,
                                               ItemView& iv, bool can_wait = true) {
  const int P = a.tiles_per_item;
  const int it = li / P;
  const int64_t item = (int64_t)blockIdx.x + (int64_t)it * gridDim.x;
  InFlight f;
  f.rows = 0;
  f.armed = false;
  f.deferred = false;
  f.skip = -1;
  f.bias = 0.f;
  f.fp8 = false;
  f.ks = f.vs = 1.f;
  if (item >= a.items) return f;
  if (iv.item != (int)item) load_item<kSparse, kFp8, kMode>(a, (int)item, lane, iv);
  const int tile = iv.t0 + (li - it * P);
  // route entry of the tile (the fused append's token tile comes before the routed blocks, and
  // with the router fused so do the ring tiles)
  int ridx = (mode_appends(kMode) && iv.v.n_new) ? tile - 1 : tile;
  if (mode_routes(kMode)) {
    ridx -= iv.v.n_r0 + iv.v.n_r1;
    if (ridx >= 0 && tile < iv.v.total && !iv.routed) {
      if (!can_wait) {
        f.deferred = true;
        return f;
      }
      acquire_route<kMode>(a, iv, lane);
    }
  }
  const int c = __shfl_sync(0xffffffffu, iv.c, ridx & 31);
  const float lp = __shfl_sync(0xffffffffu, iv.lp, ridx & 31);
  const TileRef r = tile_at<kSparse, kFp8, kMode>(iv.v, tile, c, lp, lane == 0 ? a.status : nullptr);
  const bool rope_key = mode_appends(kMode) && r.blk == -2 && a.rope_tok != nullptr;
  if (r.blk == -2) {  // fused append: the warp writes this step's row into its ring slot
    const uint4* src = reinterpret_cast<const uint4*>(lane < 16 ? iv.v.nk : iv.v.nv);
    uint4* dst = reinterpret_cast<uint4*>(lane < 16 ? iv.v.wk : iv.v.wv);
    uint4 w = src[lane & 15];
    if (rope_key) {
      // the key is encoded on its way: lanes 0-15 rotate it, write it into the ring slot and
      // into the stage themselves (its bulk copy is left out below; V is copied as usual)
      float2 cs[8];
      rope_lane_cos_sin(a, sm.rope_th, iv.rope_tok, iv.rope_pg, lane, cs);
      w = rope_rotate_chunk(w, cs, lane, lane < 16);
      if (lane < 16) {
        reinterpret_cast<uint4*>(sm.stage[s][0])[lane] = w;
        // ordered before the bulk copy that refills this stage after the tile is read
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      }
      __syncwarp();
    }
    dst[lane & 15] = w;
    if (lane == 0 && iv.v.slot_out) *iv.v.slot_out = iv.v.wslot;
  }
  f.rows = r.rows;
  f.skip = r.skip;
  f.bias = r.bias;
  f.fp8 = kFp8 && (r.blk >= 0 || (kMode == kModeRing8 && r.blk == -1));
  if (f.fp8 && r.rows > 0) {
    if (r.blk >= 0) {
      f.ks = iv.v.ks[r.blk];
      f.vs = iv.v.vs[r.blk];
    } else {  // FP8 ring tile: lane (g, c) = (lane >> 4, lane & 15) holds row 2c + g's score
      const int row = 2 * (lane & 15) + (lane >> 4);
      f.ks = row < r.rows ? r.rs_k[row] : 1.f;
      f.vs = row < r.rows ? r.rs_v[row] : 1.f;
    }
  }
  // a wait-timeout test: CTA 0 neither arms nor fills the stage of this tile, so its consumer's
  // bounded wait runs out (no copy is in flight for it)
  if (a.drop_tile >= 0 && blockIdx.x == 0 && li == a.drop_tile) return f;
  f.armed = r.rows > 0;
  if (r.rows > 0 && lane == 0) {
    const uint32_t bytes = (uint32_t)r.rows * (f.fp8 ? (uint32_t)kHeadDim : (uint32_t)kRowBytes);
    mbar_arrive_expect_tx(&sm.full[s], rope_key ? bytes : 2 * bytes);  // an encoded key is in the stage already
    if (kSparse && r.blk >= 0) {
      // routed blocks change from step to step: mark them first to leave L2, so the ring,
      // which every step reads again, stays there (measured: 32K-history attention
      // 61.9 -> 57.0 us; the dense R-SWA prefix is streamed with the default policy, which
      // measured 1% faster there and keeps small prefixes L2-resident across steps)
      const uint64_t pol = l2_policy_evict_first();
      bulk_copy_g2s_stream(sm.stage[s][0], r.k, bytes, &sm.full[s], pol);
      bulk_copy_g2s_stream(sm.stage[s][1], r.v, bytes, &sm.full[s], pol);
    } else {
      if (!rope_key) bulk_copy_g2s(sm.stage[s][0], r.k, bytes, &sm.full[s]);
      bulk_copy_g2s(sm.stage[s][1], r.v, bytes, &sm.full[s]);
    }
  }
  return f;
}

// two E4M3 codes (low byte first) -> two floats, exactly (via f16)
__device__ __forceinline__ float2 e4m3x2_f2(uint32_t pair) {
  const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(pair & 0xffffu), __NV_E4M3);
  return __half22float2(*reinterpret_cast<const __half2*>(&h));
}

__device__ __forceinline__ float2 bf16x2_f2(uint32_t w) { return make_float2(bf16lo(w), bf16hi(w)); }

// One tile for this warp: the 32 scores, the online-softmax update and P.V.
// kFull: all 32 rows valid (no bounds checks). kFp8: the tile holds E4M3 code rows
// (128 B) of one prefix block with scales (ks, vs), folded into the score and into the
// row weight of P.V; otherwise bf16 rows (256 B) and ks = vs = 1.
template <bool kFull, bool kFp8>
__device__ __forceinline__ void consume_tile(const uint8_t* kt, const uint8_t* vt, int rows, int skip, float bias,
                                             float ks, float vs, const float2 (&q2)[4], int g, int c, float& m_run,
                                             float& l_lane, float2 (&acc)[4]) {
  float pd[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    float2 d;
    if (kFp8) {
      const uint2 w = *reinterpret_cast<const uint2*>(kt + (2 * j + g) * kHeadDim + c * 8);
      d = __fmul2_rn(q2[0], e4m3x2_f2(w.x));
      d = __ffma2_rn(q2[1], e4m3x2_f2(w.x >> 16), d);
      d = __ffma2_rn(q2[2], e4m3x2_f2(w.y), d);
      d = __ffma2_rn(q2[3], e4m3x2_f2(w.y >> 16), d);
    } else {
      const uint4 w = *reinterpret_cast<const uint4*>(kt + (2 * j + g) * kRowBytes + c * 16);
      d = __fmul2_rn(q2[0], bf16x2_f2(w.x));
      d = __ffma2_rn(q2[1], bf16x2_f2(w.y), d);
      d = __ffma2_rn(q2[2], bf16x2_f2(w.z), d);
      d = __ffma2_rn(q2[3], bf16x2_f2(w.w), d);
    }
    pd[j] = d.x + d.y;
  }
  // reduce-scatter the 16 partial dots over the 16 lanes of this half-warp
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const bool up = c & 8;
    const float send = up ? pd[i] : pd[i + 8];
    const float keep = up ? pd[i + 8] : pd[i];
    pd[i] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const bool up = c & 4;
    const float send = up ? pd[i] : pd[i + 4];
    const float keep = up ? pd[i + 4] : pd[i];
    pd[i] = keep + __shfl_xor_sync(0xffffffffu, send, 4);
  }
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const bool up = c & 2;
    const float send = up ? pd[i] : pd[i + 2];
    const float keep = up ? pd[i + 2] : pd[i];
    pd[i] = keep + __shfl_xor_sync(0xffffffffu, send, 2);
  }
  {
    const bool up = c & 1;
    const float send = up ? pd[0] : pd[1];
    const float keep = up ? pd[1] : pd[0];
    pd[0] = keep + __shfl_xor_sync(0xffffffffu, send, 1);
  }
  // this lane now holds the score of tile row 2c + g
  const float sc = (kFull || (2 * c + g < rows && 2 * c + g != skip)) ? (kFp8 ? fmaf(pd[0], ks, bias) : pd[0] + bias)
                                                                    : -INFINITY;
  const float m_new = fmaxf(m_run, warp_max(sc));
  const float alpha = exp2f(m_run - m_new);
  const float p = exp2f(sc - m_new);
  l_lane = fmaf(l_lane, alpha, p);
  const float2 a2 = make_float2(alpha, alpha);
#pragma unroll
  for (int e = 0; e < 4; ++e) acc[e] = __fmul2_rn(acc[e], a2);
  m_run = m_new;
  const float pw = kFp8 ? p * vs : p;  // the V block scale rides on the row weight
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const float pj = __shfl_sync(0xffffffffu, pw, (g << 4) | j);
    if (kFull || (2 * j + g < rows && 2 * j + g != skip)) {
      const float2 p2 = make_float2(pj, pj);
      if (kFp8) {
        const uint2 w = *reinterpret_cast<const uint2*>(vt + (2 * j + g) * kHeadDim + c * 8);
        acc[0] = __ffma2_rn(p2, e4m3x2_f2(w.x), acc[0]);
        acc[1] = __ffma2_rn(p2, e4m3x2_f2(w.x >> 16), acc[1]);
        acc[2] = __ffma2_rn(p2, e4m3x2_f2(w.y), acc[2]);
        acc[3] = __ffma2_rn(p2, e4m3x2_f2(w.y >> 16), acc[3]);
      } else {
        const uint4 w = *reinterpret_cast<const uint4*>(vt + (2 * j + g) * kRowBytes + c * 16);
        acc[0] = __ffma2_rn(p2, bf16x2_f2(w.x), acc[0]);
        acc[1] = __ffma2_rn(p2, bf16x2_f2(w.y), acc[1]);
        acc[2] = __ffma2_rn(p2, bf16x2_f2(w.z), acc[2]);
        acc[3] = __ffma2_rn(p2, bf16x2_f2(w.w), acc[3]);
      }
    }
  }
}

// ---------------------------------------------------------------------------------------
// Fused router (Unlimited-OCR-2 SR-SWA explainer, 稀疏路由 steps 2-4): the same result as
// route_kernel, computed inside the decode launch. Phase 1, every warp of the grid: score
// 64-block slices z = idx_scale <q_idx, kbar_c> and publish each slice sorted (larger score
// first, ties to the smaller block). Phase 2, one CTA per sequence: merge the slices'
// candidates (z > max z - 2, the only blocks that can get p > 0), sort them, solve the exact
// 1.5-entmax threshold (sort-based rule of Peters, Niculae & Martins 2019) and publish the
// top-k blocks with bias ln p.
// ---------------------------------------------------------------------------------------

// Strict total order of route entries: larger score first, then smaller block.
__device__ __forceinline__ bool ranks_before(float za, int ia, float zb, int ib) {
  return za > zb || (za == zb && ia < ib);
}

__device__ __forceinline__ void cmp_xchg(float& z, int& i, int j, bool keep_better) {
  const float oz = __shfl_xor_sync(0xffffffffu, z, j);
  const int oi = __shfl_xor_sync(0xffffffffu, i, j);
  if (ranks_before(oz, oi, z, i) == keep_better) {
    z = oz;
    i = oi;
  }
}

// Bitonic sort of one (z, i) per lane; lane 0 ends with the best.
__device__ __forceinline__ void warp_sort32(float& z, int& i, int lane) {
#pragma unroll
  for (int k = 2; k <= 32; k <<= 1)
#pragma unroll
    for (int j = k >> 1; j > 0; j >>= 1) cmp_xchg(z, i, j, ((lane & j) == 0) == ((lane & k) == 0));
}

// A bitonic sequence over the warp, sorted best-first.
__device__ __forceinline__ void warp_bitonic_merge32(float& z, int& i, int lane) {
#pragma unroll
  for (int j = 16; j > 0; j >>= 1) cmp_xchg(z, i, j, (lane & j) == 0);
}

__device__ __forceinline__ int clamp_prefix(const DecodeArgs& a, int b) {
  const int m = a.prefix_len[b];
  return (m < 0 || m > a.cap) ? 0 : m;
}

// Phase 1: warp `warp` of this CTA scores slices warp * grid + cta, + grid * warps, ...
__device__ void score_slices(const DecodeArgs& a, int warp, int lane) {
  const int total = a.B * a.nsl_cap;
  const int o = lane >> 3, j = lane & 7;
  for (int sl = warp * (int)gridDim.x + (int)blockIdx.x; sl < total; sl += (int)gridDim.x * kWarps) {
    const int b = sl / a.nsl_cap, s = sl - b * a.nsl_cap;
    const int NB = (clamp_prefix(a, b) + kBlock - 1) / kBlock;
    const int base = s * kSlice;
    if (base < NB) {
      // a warp load covers four blocks (512 B): octet o reads block 4i + o, lane j its dims
      // 4j..4j+3; the 16 partial dots of a lane are reduce-scattered over its octet, leaving
      // lane j the dots of blocks base + 8j + o and base + 8j + 4 + o
      const float4 qv = reinterpret_cast<const float4*>(a.q_idx + (int64_t)b * kIndexDim)[j];
      const float4* k4 = reinterpret_cast<const float4*>(a.kbar + (int64_t)b * a.nb_cap * kIndexDim);
      float4 kv[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int c = base + 4 * i + o;
        kv[i] = c < a.nb_cap ? __ldg(k4 + (int64_t)c * 8 + j) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
      float v[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        float d = qv.x * kv[i].x;
        d = fmaf(qv.y, kv[i].y, d);
        d = fmaf(qv.z, kv[i].z, d);
        v[i] = fmaf(qv.w, kv[i].w, d);
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const bool up = j & 4;
        const float send = up ? v[i] : v[i + 8];
        const float keep = up ? v[i + 8] : v[i];
        v[i] = keep + __shfl_xor_sync(0xffffffffu, send, 4);
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const bool up = j & 2;
        const float send = up ? v[i] : v[i + 4];
        const float keep = up ? v[i + 4] : v[i];
        v[i] = keep + __shfl_xor_sync(0xffffffffu, send, 2);
      }
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const bool up = j & 1;
        const float send = up ? v[i] : v[i + 2];
        const float keep = up ? v[i + 2] : v[i];
        v[i] = keep + __shfl_xor_sync(0xffffffffu, send, 1);
      }
      const int c0 = base + 8 * j + o, c1 = c0 + 4;
      float za = c0 < NB ? a.idx_scale * v[0] : -INFINITY;
      int ia = c0 < NB ? c0 : kNoBlock;
      float zb = c1 < NB ? a.idx_scale * v[1] : -INFINITY;
      int ib = c1 < NB ? c1 : kNoBlock;
      // sort both columns, then split them into the better and the worse 32 (each bitonic)
      warp_sort32(za, ia, lane);
      warp_sort32(zb, ib, lane);
      const float rz = __shfl_sync(0xffffffffu, zb, 31 - lane);
      const int ri = __shfl_sync(0xffffffffu, ib, 31 - lane);
      const bool b_first = ranks_before(rz, ri, za, ia);
      float hz = b_first ? rz : za, lz = b_first ? za : rz;
      int hi = b_first ? ri : ia, li = b_first ? ia : ri;
      warp_bitonic_merge32(hz, hi, lane);
      warp_bitonic_merge32(lz, li, lane);
      const int64_t rec = (int64_t)b * a.nsl_cap + s;
      a.slice_z[rec * kSlice + lane] = hz;
      a.slice_z[rec * kSlice + 32 + lane] = lz;
      a.slice_i[rec * kSlice + lane] = hi;
      a.slice_i[rec * kSlice + 32 + lane] = li;
      if (lane == 0) a.slice_max[rec] = hz;
    }
    __syncwarp();  // the lanes' stores are ordered before lane 0's release below
    if (lane == 0) red_release_gpu(a.seq_count + b, 1);
  }
}

// Block reductions of a finalising CTA (every thread calls them; they synchronise the CTA).
__device__ __forceinline__ float fin_block_max(DecodeSmem& sm, float v, int warp, int lane) {
  v = warp_max(v);
  __syncthreads();
  if (lane == 0) sm.fin_red[warp] = v;
  __syncthreads();
  float r = sm.fin_red[0];
#pragma unroll
  for (int w = 1; w < kWarps; ++w) r = fmaxf(r, sm.fin_red[w]);
  return r;
}

// Block-wide exclusive prefix sum over the threads (every thread calls it; it synchronises).
__device__ __forceinline__ int fin_block_excl_scan(DecodeSmem& sm, int v, int warp, int lane, int& total) {
  int inc = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += t;
  }
  __syncthreads();
  if (lane == 31) sm.fin_redi[warp] = inc;
  __syncthreads();
  int before = 0;
  total = 0;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) {
    before += w < warp ? sm.fin_redi[w] : 0;
    total += sm.fin_redi[w];
  }
  return before + inc - v;
}

// Exact 1.5-entmax threshold of the x = z / 2 problem over the C candidates gz[0, C) (sorted,
// best first), values shifted by xmax: prefix sums of y and y^2 in rank order, tau_k per rank,
// support size = the largest k with delta_k >= 0 and tau_k < y_(k). Returns tau of y.
// Warp-level when C <= 32 (the other warps return 0 and must not use the result), else
// block-level with a contiguous run of ranks per thread (every thread must call it).
__device__ float fin_threshold(DecodeSmem& sm, const float* gz, float* tau_r, int C, float xmax, int tid, int warp,
                               int lane) {
  if (C <= 32) {
    if (warp != 0) return 0.f;
    const float y = lane < C ? fmaf(gz[lane], 0.5f, -xmax) : 0.f;
    float s1 = y, s2 = y * y;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const float t1 = __shfl_up_sync(0xffffffffu, s1, o), t2 = __shfl_up_sync(0xffffffffu, s2, o);
      if (lane >= o) {
        s1 += t1;
        s2 += t2;
      }
    }
    const float k = (float)(lane + 1);
    const float mean = s1 / k;
    const float delta = (1.f - (s2 - s1 * mean)) / k;
    const float t = mean - sqrtf(fmaxf(delta, 0.f));
    const unsigned ok = __ballot_sync(0xffffffffu, lane < C && delta >= 0.f && t < y);
    const int best = ok ? 32 - __clz(ok) : 0;  // the largest rank (1-based) that qualifies
    const float tb = __shfl_sync(0xffffffffu, t, best > 0 ? best - 1 : 0);
    return best > 0 ? tb : 0.f;
  }
  const int per = (C + kDecodeThreads - 1) / kDecodeThreads;
  const int r0 = min(C, tid * per), r1 = min(C, r0 + per);
  float s1 = 0.f, s2 = 0.f;
  for (int r = r0; r < r1; ++r) {
    const float y = fmaf(gz[r], 0.5f, -xmax);
    s1 += y;
    s2 = fmaf(y, y, s2);
  }
  float i1 = s1, i2 = s2;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const float t1 = __shfl_up_sync(0xffffffffu, i1, o), t2 = __shfl_up_sync(0xffffffffu, i2, o);
    if (lane >= o) {
      i1 += t1;
      i2 += t2;
    }
  }
  __syncthreads();
  if (lane == 31) {
    sm.fin_red[warp] = i1;
    sm.fin_red2[warp] = i2;
  }
  __syncthreads();
  float e1 = i1 - s1, e2 = i2 - s2;
  for (int w = 0; w < warp; ++w) {
    e1 += sm.fin_red[w];
    e2 += sm.fin_red2[w];
  }
  int best = 0;
  for (int r = r0; r < r1; ++r) {
    const float y = fmaf(gz[r], 0.5f, -xmax);
    e1 += y;
    e2 = fmaf(y, y, e2);
    const float k = (float)(r + 1);
    const float mean = e1 / k;
    const float delta = (1.f - (e2 - e1 * mean)) / k;
    const float t = mean - sqrtf(fmaxf(delta, 0.f));
    tau_r[r] = t;
    if (delta >= 0.f && t < y) best = r + 1;
  }
  best = __reduce_max_sync(0xffffffffu, (unsigned)best);
  __syncthreads();
  if (lane == 0) sm.fin_redi[warp] = best;
  __syncthreads();
#pragma unroll
  for (int w = 0; w < kWarps; ++w) best = max(best, sm.fin_redi[w]);
  return best > 0 ? tau_r[best - 1] : 0.f;
}

// Phase 2 for sequence b, by the whole CTA, with its (idle) stage buffers as scratch. Thread s
// owns slice s (at most 8192 / 64 = 128 slices) and reads, in one round, the slice's maximum
// and its first 16 entries: the maxima give max z, and only slices whose maximum clears the
// candidate cut hold candidates, as a prefix of their sorted entries (read further only when
// more than 16 of a slice's entries are candidates). The candidates are gathered at their
// scanned offsets; at most 32 of them are sorted and thresholded by warp 0 alone, more by the
// whole CTA.
__device__ void finalize_route(const DecodeArgs& a, DecodeSmem& sm, int b, int tid, int warp, int lane) {
  constexpr int kFirst = 16;  // entries of a slice read in the first round
  float* gz = reinterpret_cast<float*>(&sm.stage[0][0][0]);      // gathered scores (up to kMaxRouteBlocks)
  int* gi = reinterpret_cast<int*>(gz + kMaxRouteBlocks);         // their blocks
  float* tau_r = reinterpret_cast<float*>(gi + kMaxRouteBlocks);  // tau_k by rank k - 1
  static_assert(sizeof(DecodeSmem::stage) >= 3 * kMaxRouteBlocks * 4, "router scratch");
  static_assert(kMaxRouteBlocks / kSlice <= kDecodeThreads, "one slice per thread");
  int32_t* ready = a.route_ready + b;
  const int m_raw = a.prefix_len[b];  // an input: read before the wait
  const int NB = (m_raw < 0 || m_raw > a.cap) ? 0 : (m_raw + kBlock - 1) / kBlock;
  // every slice of the sequence published (bounded wait); the barrier then orders the other
  // threads' reads of the slices after thread 0's acquire
  if (tid == 0) {
    int ok = 1;
    if (ld_acquire_gpu(a.seq_count + b) < a.nsl_cap) {
      const uint64_t t0 = global_timer_ns();
      while (ld_acquire_gpu(a.seq_count + b) < a.nsl_cap) {
        if (global_timer_ns() - t0 > a.wait_limit_ns) {
          ok = 0;
          break;
        }
        __nanosleep(32);
      }
    }
    sm.fin_ok = ok;
    if (!ok) set_status(a.status, RSWA_DEVICE_WAIT_TIMEOUT);
    if (m_raw < 0 || m_raw > a.cap) set_status(a.status, RSWA_DEVICE_BAD_PREFIX_LEN);
  }
  __syncthreads();
  const int64_t ro = (int64_t)b * a.topk;
  if (NB == 0 || !sm.fin_ok) {  // uniform over the CTA
    if (tid < a.topk) {
      a.blk_idx_w[ro + tid] = -1;
      a.blk_logp_w[ro + tid] = -INFINITY;
    }
    if (tid == 0 && a.tau_w) a.tau_w[b] = NAN;
    __syncthreads();
    if (tid == 0) red_release_gpu(ready, 1);
    return;
  }
  const int nsl = (NB + kSlice - 1) / kSlice;
  const int64_t rec = (int64_t)b * a.nsl_cap + tid;
  const bool own = tid < nsl;
  const float* zr = a.slice_z + rec * kSlice;
  const int* ir = a.slice_i + rec * kSlice;
  float smax = -INFINITY;
  float fz[kFirst];
  int fi[kFirst];
  if (own) {
    smax = __ldcg(a.slice_max + rec);
#pragma unroll
    for (int u = 0; u < kFirst; u += 4) {
      const float4 z4 = __ldcg(reinterpret_cast<const float4*>(zr + u));
      const int4 i4 = __ldcg(reinterpret_cast<const int4*>(ir + u));
      fz[u] = z4.x, fz[u + 1] = z4.y, fz[u + 2] = z4.z, fz[u + 3] = z4.w;
      fi[u] = i4.x, fi[u + 1] = i4.y, fi[u + 2] = i4.z, fi[u + 3] = i4.w;
    }
  } else {
#pragma unroll
    for (int u = 0; u < kFirst; ++u) {
      fz[u] = -INFINITY;
      fi[u] = kNoBlock;
    }
  }
  const float zmax = fin_block_max(sm, smax, warp, lane);
  const float zcut = zmax - 2.f;  // candidates: z / 2 > max z / 2 - 1
  // this slice's candidates: a prefix of its sorted entries
  int cnt = 0;
#pragma unroll
  for (int u = 0; u < kFirst; ++u) cnt += fz[u] > zcut ? 1 : 0;
  if (cnt == kFirst)
    for (int c = kFirst; c < kSlice && __ldcg(zr + c) > zcut; ++c) ++cnt;
  int C = 0;
  int off = fin_block_excl_scan(sm, cnt, warp, lane, C);  // C >= 1 (the maximum)
  int take = cnt;
  if (C < a.topk) {
    // fewer candidates than topk: each slice's first topk valid entries join them (they hold the
    // top-k; the candidates, the largest, stay in front after the sort)
    take = 0;
    if (own) {
#pragma unroll
      for (int u = 0; u < kFirst; ++u) take += (u < a.topk && fz[u] > -INFINITY) ? 1 : 0;  // valid: a prefix
      if (take == kFirst)
        for (int c = kFirst; c < a.topk && __ldcg(zr + c) > -INFINITY; ++c) ++take;
    }
    int n_lists = 0;
    off = fin_block_excl_scan(sm, take, warp, lane, n_lists);
  }
#pragma unroll
  for (int u = 0; u < kFirst; ++u)
    if (u < take) {
      gz[off + u] = fz[u];
      gi[off + u] = fi[u];
    }
  for (int c = kFirst; c < take; ++c) {
    gz[off + c] = __ldcg(zr + c);
    gi[off + c] = __ldcg(ir + c);
  }
  int n = 0;
  if (tid == kDecodeThreads - 1) sm.fin_n = off + take;  // the last thread's end is the total
  __syncthreads();
  n = sm.fin_n;
  const float xmax = 0.5f * zmax;
  if (n <= 32) {
    // warp 0 alone: sort (best first: larger score, then smaller block), threshold, outputs
    if (warp != 0) return;
    float z = lane < n ? gz[lane] : -INFINITY;
    int i = lane < n ? gi[lane] : kNoBlock;
    warp_sort32(z, i, lane);
    const float y = lane < C ? fmaf(z, 0.5f, -xmax) : 0.f;
    float s1 = y, s2 = y * y;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const float t1 = __shfl_up_sync(0xffffffffu, s1, o), t2 = __shfl_up_sync(0xffffffffu, s2, o);
      if (lane >= o) {
        s1 += t1;
        s2 += t2;
      }
    }
    const float k = (float)(lane + 1);
    const float mean = s1 / k;
    const float delta = (1.f - (s2 - s1 * mean)) / k;
    const float t = mean - sqrtf(fmaxf(delta, 0.f));
    const unsigned okb = __ballot_sync(0xffffffffu, lane < C && delta >= 0.f && t < y);
    const int best = okb ? 32 - __clz(okb) : 0;  // the largest qualifying rank (1-based)
    const float tb = __shfl_sync(0xffffffffu, t, best > 0 ? best - 1 : 0);
    const float tau_y = best > 0 ? tb : 0.f;
    if (lane < a.topk) {
      if (i == kNoBlock) {
        a.blk_idx_w[ro + lane] = -1;
        a.blk_logp_w[ro + lane] = -INFINITY;
      } else {
        const float d = fmaf(z, 0.5f, -xmax) - tau_y;
        const float pr = d > 0.f ? d * d : 0.f;
        a.blk_idx_w[ro + lane] = i;
        a.blk_logp_w[ro + lane] = pr > 0.f ? logf(pr) : -INFINITY;
      }
    }
    if (lane == 0 && a.tau_w) a.tau_w[b] = tau_y + xmax;
    __syncwarp();
    if (lane == 0) red_release_gpu(ready, 1);
    return;
  }
  // bitonic sort of the block, padded to a power of two
  int np2 = 64;
  while (np2 < n) np2 <<= 1;
  for (int i = n + tid; i < np2; i += kDecodeThreads) {
    gz[i] = -INFINITY;
    gi[i] = kNoBlock;
  }
  for (int k2 = 2; k2 <= np2; k2 <<= 1)
    for (int j = k2 >> 1; j > 0; j >>= 1) {
      __syncthreads();
      for (int i = tid; i < np2; i += kDecodeThreads) {
        const int p = i ^ j;
        if (p > i) {
          const bool first_better = ranks_before(gz[i], gi[i], gz[p], gi[p]);
          if (first_better != ((i & k2) == 0)) {
            const float tz = gz[i];
            gz[i] = gz[p];
            gz[p] = tz;
            const int ti = gi[i];
            gi[i] = gi[p];
            gi[p] = ti;
          }
        }
      }
    }
  __syncthreads();
  const float tau_y = fin_threshold(sm, gz, tau_r, C, xmax, tid, warp, lane);
  // with C <= 32 only warp 0 holds tau; topk <= 32, so warp 0 writes the outputs either way
  if (tid < a.topk) {
    const int bi = tid < n ? gi[tid] : kNoBlock;
    if (bi == kNoBlock) {
      a.blk_idx_w[ro + tid] = -1;
      a.blk_logp_w[ro + tid] = -INFINITY;
    } else {
      const float d = fmaf(gz[tid], 0.5f, -xmax) - tau_y;
      const float pr = d > 0.f ? d * d : 0.f;
      a.blk_idx_w[ro + tid] = bi;
      a.blk_logp_w[ro + tid] = pr > 0.f ? logf(pr) : -INFINITY;
    }
  }
  if (tid == 0 && a.tau_w) a.tau_w[b] = tau_y + xmax;
  if (warp == 0) {
    __syncwarp();
    if (lane == 0) red_release_gpu(ready, 1);
  }
}

template <bool kSparse, bool kFp8, int kMode>
__global__ void __launch_bounds__(kDecodeThreads, kDecodeMinBlocks) decode_kernel(const DecodeArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  DecodeSmem& sm = *reinterpret_cast<DecodeSmem*>(smem_raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int P = a.tiles_per_item;

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) mbar_init(&sm.full[s], 1);
    fence_mbar_init();
  }
  if constexpr (mode_appends(kMode)) {
    if (a.rope_tok != nullptr && tid < kHeadDim / 2)
      sm.rope_th[tid] = exp2(-(2.0 * tid / kHeadDim) * a.rope_log2_base);
  }
  __syncthreads();
  griddep_wait();               // inputs may be written by the previous kernel in the stream
  griddep_launch_dependents();  // the next kernel may start its prologue

  // In-flight tiles of this warp, oldest first: the warp's tiles k .. k + kStagesPerWarp - 1
  // (rows 0: nothing issued).
  ItemView iv;
  iv.item = -1;
  InFlight fl[kStagesPerWarp];
  if constexpr (mode_routes(kMode)) {
    // fused router: every warp first scores its router slices (their block-key reads reach
    // HBM ahead of the ring copies, and nothing has waited yet, so no wait below can depend
    // on a warp that is itself waiting); the last n_fin CTAs then finalise routes in their
    // stage buffers before they stream, the others issue their route-independent first
    // tiles (token, ring) at once.
    const bool fin = (int)blockIdx.x >= (int)gridDim.x - a.n_fin;
    score_slices(a, warp, lane);
    if (!fin) {
#pragma unroll
      for (int j = 0; j < kStagesPerWarp; ++j)
        fl[j] = issue_tile<kSparse, kFp8, kMode>(a, sm, warp + j * kWarps, warp * kStagesPerWarp + j, lane, iv,
                                                 false);
    }
    if (fin) {
      for (int b = (int)gridDim.x - 1 - (int)blockIdx.x; b < a.B; b += (int)gridDim.x)
        finalize_route(a, sm, b, tid, warp, lane);
      // the stage buffers were written by plain stores and are refilled by bulk copies next
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      __syncthreads();
    }
#pragma unroll
    for (int j = 0; j < kStagesPerWarp; ++j)
      if (fin || fl[j].deferred)
        fl[j] = issue_tile<kSparse, kFp8, kMode>(a, sm, warp + j * kWarps, warp * kStagesPerWarp + j, lane, iv);
  } else {
#pragma unroll
    for (int j = 0; j < kStagesPerWarp; ++j)
      fl[j] = issue_tile<kSparse, kFp8, kMode>(a, sm, warp + j * kWarps, warp * kStagesPerWarp + j, lane, iv);
  }
  uint32_t phase = 0;  // bit j: parity of the next completion of this warp's stage j
  int k = 0;           // tiles of this warp consumed so far
  bool ok = true;

  const int g = lane >> 4, c = lane & 15;
  // the next item's query is loaded while the current item streams
  uint4 q_next = make_uint4(0, 0, 0, 0);
  int2 pos_next = make_int2(0, 0);  // fused step with the encoding: the next item's positions
  const bool rope_q = mode_appends(kMode) && a.rope_tok != nullptr;
  if (blockIdx.x < a.items) {
    q_next = *reinterpret_cast<const uint4*>(a.q + (int64_t)(blockIdx.x / a.splits) * kHeadDim + c * 8);
    if (rope_q) {
      const int bn = (int)blockIdx.x / a.splits / a.H;
      pos_next = make_int2(a.rope_tok[bn], a.rope_page[bn]);
    }
  }
  int li_base = 0;
  for (int item = blockIdx.x; item < a.items; item += gridDim.x, li_base += P) {
    // vq: the item's query, (b * H + h) * T + i; q, out, lse and the split partials are per query
    const int vq = item / a.splits, split = item - vq * a.splits;
    uint4 q_cur = q_next;
    const int2 pos_cur = pos_next;
    if (item + (int)gridDim.x < a.items) {
      q_next = *reinterpret_cast<const uint4*>(a.q + (int64_t)((item + gridDim.x) / a.splits) * kHeadDim + c * 8);
      if (rope_q) {
        const int bn = (item + (int)gridDim.x) / a.splits / a.H;
        pos_next = make_int2(a.rope_tok[bn], a.rope_page[bn]);
      }
    }
    if constexpr (mode_appends(kMode)) {
      if (rope_q) {  // the query encoded at its sequence's position (one query per item)
        float2 cs[8];
        rope_lane_cos_sin(a, sm.rope_th, pos_cur.x, pos_cur.y, lane, cs);
        q_cur = rope_rotate_chunk(q_cur, cs, lane, true);
      }
    }
    float2 q2[4];
    {
      const uint32_t ws[4] = {q_cur.x, q_cur.y, q_cur.z, q_cur.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) q2[e] = make_float2(bf16lo(ws[e]) * a.qscale, bf16hi(ws[e]) * a.qscale);
    }
    float m_run = -INFINITY, l_lane = 0.f;
    float2 acc[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[e] = make_float2(0.f, 0.f);

    const int first = li_base + ((warp - li_base % kWarps) + kWarps) % kWarps;
    for (int li = first; ok && li < li_base + P; li += kWarps) {
      const int j = k % kStagesPerWarp;
      const int s = warp * kStagesPerWarp + j;
      const InFlight cur = fl[0];
      const int rows = cur.rows;
      if (rows > 0) {
        // every lane waits (each needs the acquire), then the warp agrees
        if (!__all_sync(0xffffffffu, mbar_wait(&sm.full[s], (phase >> j) & 1u, a.wait_limit_ns))) {
          if (lane == 0) set_status(a.status, RSWA_DEVICE_WAIT_TIMEOUT);
          ok = false;
          break;
        }
        phase ^= 1u << j;
        const uint8_t* kt = sm.stage[s][0];
        const uint8_t* vt = sm.stage[s][1];
        const bool full = rows == kBlock && cur.skip < 0;
        if (kFp8 && cur.fp8) {
          if (full)
            consume_tile<true, true>(kt, vt, rows, -1, cur.bias, cur.ks, cur.vs, q2, g, c, m_run, l_lane, acc);
          else
            consume_tile<false, true>(kt, vt, rows, cur.skip, cur.bias, cur.ks, cur.vs, q2, g, c, m_run, l_lane,
                                      acc);
        } else {
          if (full)
            consume_tile<true, false>(kt, vt, rows, -1, cur.bias, 1.f, 1.f, q2, g, c, m_run, l_lane, acc);
          else
            consume_tile<false, false>(kt, vt, rows, cur.skip, cur.bias, 1.f, 1.f, q2, g, c, m_run, l_lane, acc);
        }
      }
      __syncwarp();  // every lane has read the stage before it is refilled
#pragma unroll
      for (int i = 0; i + 1 < kStagesPerWarp; ++i) fl[i] = fl[i + 1];
      fl[kStagesPerWarp - 1] = issue_tile<kSparse, kFp8, kMode>(a, sm, li + kWarps * kStagesPerWarp, s, lane, iv);
      ++k;
    }
    // fold the two half-warps (same dims, different rows) and the lanes' sums
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      acc[e].x += __shfl_xor_sync(0xffffffffu, acc[e].x, 16);
      acc[e].y += __shfl_xor_sync(0xffffffffu, acc[e].y, 16);
    }
    const float l = warp_sum(l_lane);
    if (g == 0) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        sm.wacc[warp][c * 8 + 2 * e] = acc[e].x;
        sm.wacc[warp][c * 8 + 2 * e + 1] = acc[e].y;
      }
    }
    if (lane == 0) {
      sm.wm[warp] = m_run;
      sm.wl[warp] = l;
    }
    __syncthreads();

    // ---------------- merge the warps ----------------
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) M = fmaxf(M, sm.wm[w]);
    float fw[kWarps];
    float L = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      fw[w] = M > -INFINITY ? exp2f(sm.wm[w] - M) : 0.f;
      L = fmaf(sm.wl[w], fw[w], L);
    }
    if (a.splits == 1) {
      for (int d = tid; d < kHeadDim; d += kDecodeThreads) {
        float A = 0.f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) A = fmaf(sm.wacc[w][d], fw[w], A);
        a.out[(int64_t)vq * kHeadDim + d] = L > 0.f ? A / L : 0.f;
      }
      if (tid == 0 && a.lse) a.lse[vq] = L > 0.f ? (M + log2f(L)) * kLn2 : -INFINITY;
    } else {
      float* rec = a.partials + ((int64_t)vq * a.splits + split) * (kHeadDim + 2);
      for (int d = tid; d < kHeadDim; d += kDecodeThreads) {
        float A = 0.f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) A = fmaf(sm.wacc[w][d], fw[w], A);
        rec[2 + d] = A;
      }
      if (tid == 0) {
        rec[0] = M;
        rec[1] = L;
      }
      __threadfence();
      __syncthreads();
      if (tid == 0) sm.is_last = (atomicAdd(&a.counters[vq], 1) == a.splits - 1);
      __syncthreads();
      if (sm.is_last) {
        __threadfence();
        const float* recs = a.partials + (int64_t)vq * a.splits * (kHeadDim + 2);
        float Mg = -INFINITY;
        for (int s = 0; s < a.splits; ++s) Mg = fmaxf(Mg, __ldcg(recs + s * (kHeadDim + 2)));
        float Lg = 0.f;
        if (Mg > -INFINITY)
          for (int s = 0; s < a.splits; ++s) {
            const float* r = recs + s * (kHeadDim + 2);
            Lg = fmaf(__ldcg(r + 1), exp2f(__ldcg(r) - Mg), Lg);
          }
        for (int d = tid; d < kHeadDim; d += kDecodeThreads) {
          float Ag = 0.f;
          if (Mg > -INFINITY)
            for (int s = 0; s < a.splits; ++s) {
              const float* r = recs + s * (kHeadDim + 2);
              Ag = fmaf(__ldcg(r + 2 + d), exp2f(__ldcg(r) - Mg), Ag);
            }
          a.out[(int64_t)vq * kHeadDim + d] = Lg > 0.f ? Ag / Lg : 0.f;
        }
        if (tid == 0) {
          if (a.lse) a.lse[vq] = Lg > 0.f ? (Mg + log2f(Lg)) * kLn2 : -INFINITY;
          a.counters[vq] = 0;
        }
      }
    }
    // the merge buffers are rewritten by the next item; a warp that gave up ends the CTA
    if (__syncthreads_or(!ok)) break;
  }
  // after a give-up, copies issued for later tiles may still be in flight: let them land
  // before the CTA's shared memory goes away (after a normal end none are left). This wait
  // is bounded too: if a copy has not landed within the limit either, the CTA exits anyway
  // (the status word already reports the give-up, and the output is not valid).
#pragma unroll
  for (int i = 0; i < kStagesPerWarp; ++i)
    if (fl[i].armed) {
      const int j = (k + i) % kStagesPerWarp;
      mbar_wait(&sm.full[warp * kStagesPerWarp + j], (phase >> j) & 1u, a.wait_limit_ns);
      phase ^= 1u << j;
    }
  if constexpr (mode_appends(kMode) || mode_routes(kMode)) {
    // fused append: every CTA has read wp / fill once it gets here; the last one to arrive
    // advances them (sequences with a bad ring state stay untouched) and rearms the counter.
    // (Advancing per sequence as its last item finishes put a fence and an atomic at every
    // item boundary and measured slower.) Fused router: no CTA waits on a route flag or a
    // slice count any more, so the last one clears them for the next launch.
    __syncthreads();
    if (tid == 0) {
      __threadfence();
      sm.is_last = atomicAdd(a.grid_counter, 1) == (int)gridDim.x - 1;
    }
    __syncthreads();
    if (sm.is_last) {
      __threadfence();
      for (int b = tid; b < a.B; b += kDecodeThreads) {
        if (mode_appends(kMode)) {
          const int w = a.wp_w[b], f = a.fill_w[b];
          if (w >= 0 && w < a.n && f >= 0 && f <= a.n) {
            a.wp_w[b] = (w + 1 == a.n) ? 0 : w + 1;
            a.fill_w[b] = min(f + 1, a.n);
          }
        }
        if (mode_routes(kMode)) {
          a.seq_count[b] = 0;
          a.route_ready[b] = 0;
        }
      }
      if (tid == 0) *a.grid_counter = 0;
    }
  }
}

}  // namespace

// Per-device "shared-memory limit raised" bits of each decode instantiation.
unsigned long long g_smem_done[11] = {};

int decode_ctas_per_sm() { return kDecodeMinBlocks; }

// The fused-router kernels wait on one another's CTAs, so their grid must be co-resident:
// the occupancy the runtime reports for them (with their shared memory) bounds it.
// (Queried once per device, after the kernels' shared-memory limit is raised.)
int routed_decode_ctas_per_sm() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  static int cached[64] = {};
  int c = __atomic_load_n(&cached[dev], __ATOMIC_ACQUIRE);
  if (c > 0) return c;
  void (*k0)(const DecodeArgs) = decode_kernel<true, false, kModeRoute>;
  void (*k1)(const DecodeArgs) = decode_kernel<true, false, kModeRouteAppend>;
  if (ensure_smem_limit(k0, sizeof(DecodeSmem), &g_smem_done[9]) != cudaSuccess ||
      ensure_smem_limit(k1, sizeof(DecodeSmem), &g_smem_done[10]) != cudaSuccess)
    return 0;
  int n0 = 0, n1 = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n0, k0, kDecodeThreads, sizeof(DecodeSmem)) != cudaSuccess ||
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n1, k1, kDecodeThreads, sizeof(DecodeSmem)) != cudaSuccess)
    return 0;
  c = n0 < n1 ? n0 : n1;
  __atomic_store_n(&cached[dev], c, __ATOMIC_RELEASE);
  return c;
}

size_t route_area_bytes(int B, int64_t cap) {
  const int64_t nb_cap = (cap + kBlock - 1) / kBlock;
  const int64_t nsl = (nb_cap + kSlice - 1) / kSlice;
  const size_t flags = ((size_t)B * 8 + 255) / 256 * 256;                  // seq_count, route_ready
  const size_t maxes = ((size_t)B * nsl * 4 + 255) / 256 * 256;            // slice_max
  const size_t recs = (size_t)B * nsl * kSlice * 8;                        // slice_z, slice_i
  return flags + maxes + recs;
}

int64_t decode_max_tiles_dense(int64_t cap, int n) {
  return (cap + kBlock - 1) / kBlock + (n + kBlock - 1) / kBlock + 1;
}

int64_t decode_max_tiles_sparse(int topk, int n) { return topk + (n + kBlock - 1) / kBlock + 1; }

WorkspacePlan plan_decode_workspace(int B, int H, int64_t max_tiles, int sm_count, size_t max_bytes) {
  WorkspacePlan p;
  const int64_t bh = (int64_t)B * H;
  const int64_t slots = (int64_t)sm_count * kDecodeMinBlocks;
  const size_t fixed = 256 + ((size_t)bh * 4 + 255) / 256 * 256;
  // pick the split count that minimises the busiest CTA's cost, counted in
  // tiles: ceil(items / grid) x (tiles per item + a fixed cost per item, about
  // two tiles for the item's query load and hand-over, two more for writing and
  // merging a split partial), preferring fewer splits on ties; with a byte
  // budget, only plans that fit
  int best_s = 1;
  int64_t best_cost = -1;
  for (int s = 1; s <= 64; ++s) {
    const int64_t per = (max_tiles + s - 1) / s;
    if (s > 1 && per < 2) break;
    if (s > 1 && max_bytes > 0 && fixed + (size_t)bh * s * (kHeadDim + 2) * 4 > max_bytes) break;
    const int64_t items = bh * s;
    const int64_t grid = items < slots ? items : slots;
    const int64_t cost = (items + grid - 1) / grid * (per + 2 + (s > 1 ? 2 : 0));
    if (best_cost < 0 || cost < best_cost) {
      best_cost = cost;
      best_s = s;
    }
  }
  p.splits = best_s;
  p.tiles_per_item = (int)((max_tiles + best_s - 1) / best_s);
  p.items = bh * best_s;
  p.grid = (int)(p.items < slots ? p.items : slots);
  p.counters_off = 256;
  p.partials_off = p.counters_off + ((size_t)bh * 4 + 255) / 256 * 256;
  p.bytes = p.partials_off + (p.splits > 1 ? (size_t)bh * p.splits * (kHeadDim + 2) * 4 : 0);
  return p;
}

cudaError_t launch_decode(const DecodeArgs& a, int grid, bool sparse, cudaStream_t stream) {
  const size_t smem = sizeof(DecodeSmem);
  // the instantiations in use: plain decode for every prefix format and over an FP8 prefix with
  // an FP8 ring; the fused append and the chunked-prefill band over a bf16 prefix
  int mode = a.k_out != nullptr ? kModeBand
             : (a.k_new != nullptr ? kModeAppend : (a.ring_k8 != nullptr ? kModeRing8 : kModeDecode));
  if (a.q_idx != nullptr) {
    if (!sparse || a.fp8 || a.k_out != nullptr || a.ring_k8 != nullptr) return cudaErrorNotSupported;
    mode = a.k_new != nullptr ? kModeRouteAppend : kModeRoute;
  }
  void (*kernel)(const DecodeArgs) = nullptr;
  int slot = 0;
  if (mode == kModeDecode) {
    kernel = sparse ? (a.fp8 ? decode_kernel<true, true, kModeDecode> : decode_kernel<true, false, kModeDecode>)
                    : (a.fp8 ? decode_kernel<false, true, kModeDecode> : decode_kernel<false, false, kModeDecode>);
    slot = (sparse ? 2 : 0) + (a.fp8 ? 1 : 0);
  } else if (mode == kModeRoute || mode == kModeRouteAppend) {
    kernel = mode == kModeRoute ? decode_kernel<true, false, kModeRoute> : decode_kernel<true, false, kModeRouteAppend>;
    slot = mode == kModeRoute ? 9 : 10;
  } else if (mode == kModeRing8) {
    if (!a.fp8) return cudaErrorNotSupported;
    kernel = sparse ? decode_kernel<true, true, kModeRing8> : decode_kernel<false, true, kModeRing8>;
    slot = sparse ? 8 : 7;
  } else if (a.fp8) {
    return cudaErrorNotSupported;
  } else if (mode == kModeAppend) {
    kernel = sparse ? decode_kernel<true, false, kModeAppend> : decode_kernel<false, false, kModeAppend>;
    slot = sparse ? 5 : 4;
  } else {
    if (!sparse) return cudaErrorNotSupported;
    kernel = decode_kernel<true, false, kModeBand>;
    slot = 6;
  }
  cudaError_t e = ensure_smem_limit(kernel, smem, &g_smem_done[slot]);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  fill_launch_config(cfg, attr, dim3(grid), dim3(kDecodeThreads), smem, stream);
  return cudaLaunchKernelEx(&cfg, kernel, a);
}

}  // namespace rswa
