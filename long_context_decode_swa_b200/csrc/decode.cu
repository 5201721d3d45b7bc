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
//    in turn and a producer warp keeps a 6-stage shared-memory ring filled
//    with cp.async.bulk copies (8 KiB of K and 8 KiB of V per stage) across
//    item boundaries, so the copy pipeline never drains between items;
//  * six consumer warps take the tiles round-robin, one stage each (a sweep of
//    2-8 consumer warps and 1-3 stages per warp put this shape first for the
//    batched, 32K-history and ragged long-horizon workloads alike); stage s
//    always belongs to warp s mod 6, so each warp meets its stages' mbarrier
//    phases in order.
//    In a warp, lane (g, c) holds dims 8c..8c+7 and rows 2j+g; the 16 partial
//    dot products of a half-warp are reduce-scattered in 15 shuffles, the
//    online softmax runs in the exp2 domain, and P.V broadcasts each row's
//    weight with a shuffle;
//  * at the end of an item the consumer warps merge (named barrier) and either
//    write the output (one split) or a (max, sum, acc) partial; the last item
//    of a (sequence, head) to finish (atomic counter) merges the partials by
//    log-sum-exp and resets the counter.
// The split count is chosen per launch to minimise the busiest CTA's tile count.
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
// Local tile li goes to consumer warp li % kConsumerWarps and to stage
// li % kStages. kStages is a multiple of kConsumerWarps, so every stage has
// exactly one consumer warp, which meets that stage's uses in order: the
// parity of each mbarrier wait then names the right phase (a warp can never
// wait on a stage two phases ahead of the copy in flight).
constexpr int kConsumerWarps = RSWA_DECODE_WARPS;
constexpr int kStages = RSWA_DECODE_WARPS * RSWA_DECODE_STAGES_PER_WARP;
constexpr int kDecodeThreads = (kConsumerWarps + 1) * 32;
constexpr int kConsumerThreads = kConsumerWarps * 32;
static_assert(kStages % kConsumerWarps == 0, "each stage needs a single consumer warp");
constexpr int kTileBytes = kBlock * kRowBytes;  // 8 KiB
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

struct DecodeSmem {
  uint8_t stage[kStages][2][kTileBytes];
  uint64_t full[kStages];
  uint64_t empty[kStages];
  int rows[kStages];
  int tile_id[kStages];  // producer's local tile index for the stage's current use
  float bias[kStages];   // log2 domain
  float wm[kConsumerWarps];
  float wl[kConsumerWarps];
  float wacc[kConsumerWarps][kHeadDim];
  int abort_flag;
  int is_last;
};

constexpr int kDecodeMinBlocks =
    (227 * 1024) / (int)sizeof(DecodeSmem) > 0 ? (227 * 1024) / (int)sizeof(DecodeSmem) : 1;

// What the producer needs to enumerate a (sequence, head)'s tiles.
struct SeqView {
  const uint16_t* pk;  // prefix rows of this (b, h)
  const uint16_t* pv;
  const uint16_t* rk;  // ring rows of this (b, h)
  const uint16_t* rv;
  int m;               // valid prefix rows
  int nb;              // prefix blocks (SR-SWA)
  int n_first;         // tiles before the ring (prefix tiles, or topk route entries)
  int a0, len0, len1;  // ring slot ranges [a0, a0+len0) and [0, len1)
  int n_r0, n_r1;
  int total;
};

template <bool kSparse>
__device__ __forceinline__ SeqView make_view(const DecodeArgs& a, int b, int h, bool report) {
  SeqView v;
  const int64_t bh = (int64_t)b * a.H + h;
  int m = a.prefix_len[b];
  if (m < 0 || m > a.cap) {
    if (report) set_status(a.status, RSWA_DEVICE_BAD_PREFIX_LEN);
    m = 0;
  }
  int w = a.wp[b], f = a.fill[b];
  if (w < 0 || w >= a.n || f < 0 || f > a.n) {
    if (report) set_status(a.status, RSWA_DEVICE_BAD_RING_STATE);
    w = 0;
    f = 0;
  }
  v.pk = a.pk + bh * a.cap * kHeadDim;
  v.pv = a.pv + bh * a.cap * kHeadDim;
  v.rk = a.ring_k + bh * a.n * kHeadDim;
  v.rv = a.ring_v + bh * a.n * kHeadDim;
  v.m = m;
  v.nb = (m + kBlock - 1) / kBlock;
  // valid slots are (w - f + i) mod n, i < f; a full ring is read as [0, n)
  int a0 = f == a.n ? 0 : (w - f) % a.n;
  if (a0 < 0) a0 += a.n;
  v.a0 = a0;
  v.len0 = min(f, a.n - a0);
  v.len1 = f - v.len0;
  v.n_r0 = (v.len0 + kBlock - 1) / kBlock;
  v.n_r1 = (v.len1 + kBlock - 1) / kBlock;
  v.n_first = kSparse ? a.topk : v.nb;
  v.total = v.n_first + v.n_r0 + v.n_r1;
  return v;
}

// Tile t of a (b, h): source rows, row count (0 = empty tile) and log2 bias.
// For SR-SWA, (c, lp) is route entry t when t < topk.
template <bool kSparse>
__device__ __forceinline__ void tile_at(const SeqView& v, int t, int c, float lp, const uint16_t*& k,
                                        const uint16_t*& val, int& rows, float& bias, int32_t* status) {
  bias = 0.f;
  k = val = v.pk;
  rows = 0;
  if (t >= v.total) return;
  if (t < v.n_first) {
    int start;
    if (kSparse) {
      if (c < 0 || !(lp > -INFINITY)) return;
      if (c >= v.nb) {
        set_status(status, RSWA_DEVICE_BAD_BLOCK_IDX);
        return;
      }
      start = c * kBlock;
      bias = lp * kLog2e;
    } else {
      start = t * kBlock;
    }
    rows = min(kBlock, v.m - start);
    k = v.pk + (int64_t)start * kHeadDim;
    val = v.pv + (int64_t)start * kHeadDim;
    return;
  }
  t -= v.n_first;
  int start, len;
  if (t < v.n_r0) {
    start = v.a0 + t * kBlock;
    len = v.len0 - t * kBlock;
  } else {
    t -= v.n_r0;
    start = t * kBlock;
    len = v.len1 - t * kBlock;
  }
  rows = min(kBlock, len);
  k = v.rk + (int64_t)start * kHeadDim;
  val = v.rv + (int64_t)start * kHeadDim;
}

__device__ __forceinline__ void consumer_sync() {
  asm volatile("bar.sync 1, %0;" ::"r"(kConsumerThreads) : "memory");
}

template <bool kSparse>
__global__ void __launch_bounds__(kDecodeThreads, kDecodeMinBlocks) decode_kernel(const DecodeArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  DecodeSmem& sm = *reinterpret_cast<DecodeSmem*>(smem_raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int P = a.tiles_per_item;

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], 1);
    }
    sm.abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  griddep_wait();               // inputs may be written by the previous kernel in the stream
  griddep_launch_dependents();  // the next kernel may start its prologue

  if (warp == kConsumerWarps) {
    // ---------------- producer warp: lane 0 issues, the warp fetches route entries ----------------
    int li = 0, issued = 0;
    bool aborted = false;
    for (int item = blockIdx.x; item < a.items && !aborted; item += gridDim.x) {
      const int bh = item / a.splits, split = item - bh * a.splits;
      const int b = bh / a.H, h = bh - b * a.H;
      const SeqView v = make_view<kSparse>(a, b, h, lane == 0 && split == 0 && h == 0);
      int my_c = -1;
      float my_lp = -INFINITY;
      if (kSparse && lane < a.topk) {
        my_c = a.blk_idx[(int64_t)b * a.topk + lane];
        my_lp = a.blk_logp[(int64_t)b * a.topk + lane];
      }
      const int t0 = split * P;
      for (int t = 0; t < P; ++t, ++li) {
        const int s = li % kStages;
        if (li >= kStages && !__all_sync(0xffffffffu, mbar_wait(&sm.empty[s], ((li / kStages) - 1) & 1))) {
          aborted = true;
          break;
        }
        if (*reinterpret_cast<volatile int*>(&sm.abort_flag)) {
          aborted = true;
          break;
        }
        const int tile = t0 + t;
        const int c = __shfl_sync(0xffffffffu, my_c, tile & 31);
        const float lp = __shfl_sync(0xffffffffu, my_lp, tile & 31);
        if (lane == 0) {
          const uint16_t *kp, *vp;
          int rows;
          float bias;
          tile_at<kSparse>(v, tile, c, lp, kp, vp, rows, bias, a.status);
          sm.rows[s] = rows;
          sm.bias[s] = bias;
          sm.tile_id[s] = li;
          if (rows > 0) {
            const uint32_t bytes = (uint32_t)rows * kRowBytes;
            mbar_arrive_expect_tx(&sm.full[s], 2 * bytes);
            bulk_copy_g2s(sm.stage[s][0], kp, bytes, &sm.full[s]);
            bulk_copy_g2s(sm.stage[s][1], vp, bytes, &sm.full[s]);
          } else {
            mbar_arrive(&sm.full[s]);
          }
        }
        __syncwarp();
        issued = li + 1;
      }
    }
    if (aborted && lane == 0) {
      sm.abort_flag = 1;
      set_status(a.status, RSWA_DEVICE_WAIT_TIMEOUT);
      // let every copy still in flight land before the CTA's shared memory goes away
      for (int j = max(0, issued - kStages); j < issued; ++j) mbar_wait(&sm.full[j % kStages], (j / kStages) & 1);
    }
    return;
  }

  // ---------------- consumer warps ----------------
  const int g = lane >> 4, c = lane & 15;
  int li_base = 0;
  bool ok = true;
  // the next item's query is loaded while the current item streams
  uint4 q_next = make_uint4(0, 0, 0, 0);
  if (blockIdx.x < a.items)
    q_next = *reinterpret_cast<const uint4*>(a.q + (int64_t)(blockIdx.x / a.splits) * kHeadDim + c * 8);
  for (int item = blockIdx.x; item < a.items; item += gridDim.x, li_base += P) {
    const int bh = item / a.splits, split = item - bh * a.splits;
    const uint4 q_cur = q_next;
    if (item + (int)gridDim.x < a.items)
      q_next = *reinterpret_cast<const uint4*>(a.q + (int64_t)((item + gridDim.x) / a.splits) * kHeadDim + c * 8);
    float qf[8];
    {
      const uint4 w = q_cur;
      const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        qf[2 * e] = bf16lo(ws[e]) * a.qscale;
        qf[2 * e + 1] = bf16hi(ws[e]) * a.qscale;
      }
    }
    float m_run = -INFINITY, l_lane = 0.f;
    float acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.f;

    const int first = li_base + ((warp - li_base % kConsumerWarps) + kConsumerWarps) % kConsumerWarps;
    for (int li = first; ok && li < li_base + P; li += kConsumerWarps) {
      const int s = li % kStages;
      // every lane waits (each needs the acquire), then the warp agrees
      if (!__all_sync(0xffffffffu, mbar_wait(&sm.full[s], (li / kStages) & 1))) {
        if (lane == 0) {
          sm.abort_flag = 1;
          set_status(a.status, RSWA_DEVICE_WAIT_TIMEOUT);
        }
        ok = false;
        break;
      }
      if (sm.tile_id[s] != li) {  // protocol check: never compute on another tile's data
        if (lane == 0) {
          sm.abort_flag = 1;
          set_status(a.status, RSWA_DEVICE_PIPELINE);
        }
        ok = false;
        break;
      }
      const int rows = sm.rows[s];
      if (rows > 0) {
        const float bias = sm.bias[s];
        const uint8_t* kt = sm.stage[s][0];
        const uint8_t* vt = sm.stage[s][1];
        float pd[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const uint4 w = *reinterpret_cast<const uint4*>(kt + (2 * j + g) * kRowBytes + c * 16);
          float d = qf[0] * bf16lo(w.x);
          d = fmaf(qf[1], bf16hi(w.x), d);
          d = fmaf(qf[2], bf16lo(w.y), d);
          d = fmaf(qf[3], bf16hi(w.y), d);
          d = fmaf(qf[4], bf16lo(w.z), d);
          d = fmaf(qf[5], bf16hi(w.z), d);
          d = fmaf(qf[6], bf16lo(w.w), d);
          d = fmaf(qf[7], bf16hi(w.w), d);
          pd[j] = d;
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
        const float sc = (2 * c + g < rows) ? pd[0] + bias : -INFINITY;
        const float m_new = fmaxf(m_run, warp_max(sc));
        const float alpha = exp2f(m_run - m_new);
        const float p = exp2f(sc - m_new);
        l_lane = fmaf(l_lane, alpha, p);
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] *= alpha;
        m_run = m_new;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const float pj = __shfl_sync(0xffffffffu, p, (g << 4) | j);
          if (2 * j + g < rows) {
            const uint4 w = *reinterpret_cast<const uint4*>(vt + (2 * j + g) * kRowBytes + c * 16);
            acc[0] = fmaf(pj, bf16lo(w.x), acc[0]);
            acc[1] = fmaf(pj, bf16hi(w.x), acc[1]);
            acc[2] = fmaf(pj, bf16lo(w.y), acc[2]);
            acc[3] = fmaf(pj, bf16hi(w.y), acc[3]);
            acc[4] = fmaf(pj, bf16lo(w.z), acc[4]);
            acc[5] = fmaf(pj, bf16hi(w.z), acc[5]);
            acc[6] = fmaf(pj, bf16lo(w.w), acc[6]);
            acc[7] = fmaf(pj, bf16hi(w.w), acc[7]);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.empty[s]);
    }
    // fold the two half-warps (same dims, different rows) and the lanes' sums
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], 16);
    const float l = warp_sum(l_lane);
    if (g == 0) {
#pragma unroll
      for (int e = 0; e < 8; ++e) sm.wacc[warp][c * 8 + e] = acc[e];
    }
    if (lane == 0) {
      sm.wm[warp] = m_run;
      sm.wl[warp] = l;
    }
    consumer_sync();

    // ---------------- merge the consumer warps ----------------
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kConsumerWarps; ++w) M = fmaxf(M, sm.wm[w]);
    float fw[kConsumerWarps];
    float L = 0.f;
#pragma unroll
    for (int w = 0; w < kConsumerWarps; ++w) {
      fw[w] = M > -INFINITY ? exp2f(sm.wm[w] - M) : 0.f;
      L = fmaf(sm.wl[w], fw[w], L);
    }
    if (a.splits == 1) {
      for (int d = tid; d < kHeadDim; d += kConsumerThreads) {
        float A = 0.f;
#pragma unroll
        for (int w = 0; w < kConsumerWarps; ++w) A = fmaf(sm.wacc[w][d], fw[w], A);
        a.out[(int64_t)bh * kHeadDim + d] = L > 0.f ? A / L : 0.f;
      }
      if (tid == 0 && a.lse) a.lse[bh] = L > 0.f ? (M + log2f(L)) * kLn2 : -INFINITY;
    } else {
      float* rec = a.partials + ((int64_t)bh * a.splits + split) * (kHeadDim + 2);
      for (int d = tid; d < kHeadDim; d += kConsumerThreads) {
        float A = 0.f;
#pragma unroll
        for (int w = 0; w < kConsumerWarps; ++w) A = fmaf(sm.wacc[w][d], fw[w], A);
        rec[2 + d] = A;
      }
      if (tid == 0) {
        rec[0] = M;
        rec[1] = L;
      }
      __threadfence();
      consumer_sync();
      if (tid == 0) sm.is_last = (atomicAdd(&a.counters[bh], 1) == a.splits - 1);
      consumer_sync();
      if (sm.is_last) {
        __threadfence();
        const float* recs = a.partials + (int64_t)bh * a.splits * (kHeadDim + 2);
        float Mg = -INFINITY;
        for (int s = 0; s < a.splits; ++s) Mg = fmaxf(Mg, __ldcg(recs + s * (kHeadDim + 2)));
        float Lg = 0.f;
        if (Mg > -INFINITY)
          for (int s = 0; s < a.splits; ++s) {
            const float* r = recs + s * (kHeadDim + 2);
            Lg = fmaf(__ldcg(r + 1), exp2f(__ldcg(r) - Mg), Lg);
          }
        for (int d = tid; d < kHeadDim; d += kConsumerThreads) {
          float Ag = 0.f;
          if (Mg > -INFINITY)
            for (int s = 0; s < a.splits; ++s) {
              const float* r = recs + s * (kHeadDim + 2);
              Ag = fmaf(__ldcg(r + 2 + d), exp2f(__ldcg(r) - Mg), Ag);
            }
          a.out[(int64_t)bh * kHeadDim + d] = Lg > 0.f ? Ag / Lg : 0.f;
        }
        if (tid == 0) {
          if (a.lse) a.lse[bh] = Lg > 0.f ? (Mg + log2f(Lg)) * kLn2 : -INFINITY;
          a.counters[bh] = 0;
        }
      }
    }
    consumer_sync();  // the merge buffers are rewritten by the next item
  }
}

}  // namespace

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
  static unsigned long long done_sparse = 0, done_dense = 0;
  cudaError_t e = sparse ? ensure_smem_limit(decode_kernel<true>, smem, &done_sparse)
                         : ensure_smem_limit(decode_kernel<false>, smem, &done_dense);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  fill_launch_config(cfg, attr, dim3(grid), dim3(kDecodeThreads), smem, stream);
  if (sparse) return cudaLaunchKernelEx(&cfg, decode_kernel<true>, a);
  return cudaLaunchKernelEx(&cfg, decode_kernel<false>, a);
}

}  // namespace rswa
