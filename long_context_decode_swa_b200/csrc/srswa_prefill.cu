// srswa_prefill.cu -- SR-SWA chunked prefill on sm_100a tensor cores.
//
// Every output-side query of a chunk is routed by itself (the serving notes size prefill
// memory by a per-token router score tensor of about [tokens, context / 32]); query i
// attends to its routed prefix blocks, each with bias ln p (Unlimited-OCR-2 SR-SWA explainer,
// 稀疏路由 step 4), and to the causal band of the chunk's outputs i - n < j <= i, positions
// before the chunk coming from the ring. The two key sets are disjoint, so the softmax over
// their union is the log-sum-exp merge of a softmax over each:
//   * band and ring: the dense tcgen05 prefill kernel with the prefix left out writes
//     (out, lse) for every query;
//   * routed blocks: queries whose routes select the same set of blocks share their K and V
//     tiles, so a chunk's queries are grouped by block set (group_kernel) and each group of
//     up to 128 queries runs, per head, as one 128-row tcgen05 tile against its blocks' keys
//     with a per-(query, block) bias ln p (routed_kernel), merging its result into (out, lse).
//     A query alone in its block set is a group of one (the tile's other rows are idle).
#include <cuda.h>
#include <cuda_bf16.h>

#include <cmath>

#include "common.cuh"
#include "internal.h"
#include "tcgen05.cuh"

namespace rswa {

namespace {

constexpr int kGroupThreads = 512;
constexpr int kGroupRows = 128;        // queries per group: one tcgen05 M = 128 tile
constexpr int kChunkBlocks = 16;       // blocks per pass: 4 key tiles of 128 keys, S of all in TMEM
constexpr int kRec = 4 + kMaxTopk;     // group record: b, count, qoff, nblk, blocks (ascending)
constexpr float kLog2eR = 1.4426950408889634f;
constexpr float kLn2R = 0.6931471805599453f;

// splitmix64's output function (Steele, Lea and Flood 2014): a 64-bit bit mixer.
__device__ __forceinline__ uint64_t mix64(uint64_t x) {
  x += 0x9e3779b97f4a7c15ull;
  x = (x ^ (x >> 30)) * 0xbf58476d1ce4e5b9ull;
  x = (x ^ (x >> 27)) * 0x94d049bb133111ebull;
  return x ^ (x >> 31);
}

// A route entry counts when it names a block and its probability is not zero.
__device__ __forceinline__ bool entry_valid(int c, float lp) { return c >= 0 && lp > -INFINITY; }

// A query's route held in registers: its valid entries' blocks (ascending) and their ln p,
// k valid entries; slots past k hold block INT_MAX and -inf.
struct RouteRegs {
  int blk[kMaxTopk];
  float lp[kMaxTopk];
  int k;
};

__device__ __forceinline__ void load_route(const int32_t* blk, const float* logp, int64_t r, int topk, RouteRegs& q) {
#pragma unroll
  for (int j = 0; j < kMaxTopk; ++j) {
    const int c = j < topk ? blk[r + j] : -1;
    const float l = j < topk ? logp[r + j] : -INFINITY;
    const bool v = entry_valid(c, l);
    q.blk[j] = v ? c : 0x7fffffff;
    q.lp[j] = v ? l : -INFINITY;
  }
  // bitonic sorting network by block, ascending (invalid entries, INT_MAX, last)
#pragma unroll
  for (int k2 = 2; k2 <= kMaxTopk; k2 <<= 1)
#pragma unroll
    for (int j = k2 >> 1; j > 0; j >>= 1)
#pragma unroll
      for (int i = 0; i < kMaxTopk; ++i) {
        const int l = i ^ j;
        if (l > i && ((q.blk[i] > q.blk[l]) == ((i & k2) == 0))) {
          const int tb = q.blk[i];
          q.blk[i] = q.blk[l];
          q.blk[l] = tb;
          const float tl = q.lp[i];
          q.lp[i] = q.lp[l];
          q.lp[l] = tl;
        }
      }
  int k = 0;
#pragma unroll
  for (int j = 0; j < kMaxTopk; ++j) k += q.blk[j] != 0x7fffffff ? 1 : 0;
  q.k = k;
}

struct GroupArgs {
  int B, T, topk;
  int64_t cap;
  const int32_t* prefix_len;
  int32_t* status;
  const int32_t* blk;    // [B][T][topk]
  const float* logp;
  int32_t* rec;          // [B * T][kRec]
  int32_t* gq;           // [B * T]: query positions, group after group
  int32_t* gblk;         // [B * T][kMaxTopk]: per query, its route's blocks ascending (INT_MAX past them)
  float* gbias;          // [B * T][kMaxTopk]: per query, ln p of those blocks in that order
  int32_t* counts;       // [0] groups, [1] gq entries (zeroed before the launch)
  uint64_t* keys;        // [B * T]: per query, its sort key (group_prep_kernel -> group_kernel)
};

// Block-wide inclusive prefix sum of three counters over the threads
__device__ __forceinline__ int3 block_scan3(int3 v, int3* wsum, int3& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int3 inc = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int x = __shfl_up_sync(0xffffffffu, inc.x, o), y = __shfl_up_sync(0xffffffffu, inc.y, o),
              z = __shfl_up_sync(0xffffffffu, inc.z, o);
    if (lane >= o) {
      inc.x += x;
      inc.y += y;
      inc.z += z;
    }
  }
  __syncthreads();
  if (lane == 31) wsum[warp] = inc;
  __syncthreads();
  int3 before = make_int3(0, 0, 0);
  total = make_int3(0, 0, 0);
  for (int w = 0; w < kGroupThreads / 32; ++w) {
    const int3 s = wsum[w];
    if (w < warp) {
      before.x += s.x;
      before.y += s.y;
      before.z += s.z;
    }
    total.x += s.x;
    total.y += s.y;
    total.z += s.z;
  }
  return make_int3(before.x + inc.x, before.y + inc.y, before.z + inc.z);
}

// One thread per query of the chunk, over the whole grid: the query's route sorted by block into
// its scratch rows (blocks ascending, INT_MAX past them; ln p in the same order) and its sort
// key: a hash of the sorted block list in the high bits (equal sets, equal hashes) and the
// position in the low 13 (keys of empty routes sort last). Route entries past the prefix are
// flagged (their rows lie outside it: they are read as masked).
constexpr int kPrepThreads = 128;

__global__ void __launch_bounds__(kPrepThreads) group_prep_kernel(const GroupArgs a) {
  griddep_wait();
  griddep_launch_dependents();
  const int64_t qi = (int64_t)blockIdx.x * kPrepThreads + threadIdx.x;
  if (qi >= (int64_t)a.B * a.T) return;
  const int b = (int)(qi / a.T), t = (int)(qi - (int64_t)b * a.T);
  const int m_b = a.prefix_len[b];
  const int NB = (m_b < 0 || m_b > a.cap) ? 0 : (m_b + 31) / 32;
  RouteRegs rq;
  load_route(a.blk, a.logp, qi * a.topk, a.topk, rq);
  int4* gb = reinterpret_cast<int4*>(a.gblk + qi * kMaxTopk);
  float4* gl = reinterpret_cast<float4*>(a.gbias + qi * kMaxTopk);
#pragma unroll
  for (int j = 0; j < kMaxTopk; j += 4) {
    gb[j / 4] = make_int4(rq.blk[j], rq.blk[j + 1], rq.blk[j + 2], rq.blk[j + 3]);
    gl[j / 4] = make_float4(rq.lp[j], rq.lp[j + 1], rq.lp[j + 2], rq.lp[j + 3]);
  }
  uint64_t h = 0;
  int top = -1;
#pragma unroll
  for (int j = 0; j < kMaxTopk; ++j)
    if (j < rq.k) {
      h = mix64(h ^ (uint64_t)(uint32_t)rq.blk[j]);
      top = rq.blk[j];
    }
  a.keys[qi] = rq.k > 0 ? (mix64(h + (uint64_t)rq.k) & ~0x1FFFull) | (uint64_t)t : ~0ull;
  if (top >= NB) set_status(a.status, RSWA_DEVICE_BAD_BLOCK_IDX);  // the largest valid block lies past the prefix
}

__device__ __forceinline__ uint64_t shfl_xor_u64(uint64_t v, int m) {
  const uint32_t lo = __shfl_xor_sync(0xffffffffu, (uint32_t)v, m);
  const uint32_t hi = __shfl_xor_sync(0xffffffffu, (uint32_t)(v >> 32), m);
  return ((uint64_t)hi << 32) | lo;
}

// Stage (k2, J) of the bitonic network for the pairs inside one thread's registers (J < E).
template <int E, int J>
__device__ __forceinline__ void sort_stage_regs(uint64_t (&x)[E], int t, int k2) {
#pragma unroll
  for (int e = 0; e < E; ++e)
    if ((e & J) == 0) {
      const bool ascending = ((t * E + e) & k2) == 0;
      const uint64_t u = x[e], v = x[e | J];
      if ((u > v) == ascending) {
        x[e] = v;
        x[e | J] = u;
      }
    }
}

// Ascending bitonic sort of the chunk's keys of sequence b (padded with ~0 to
// kGroupThreads * E), held E per thread: thread t holds logical elements t * E + e. Strides
// below E are exchanged in registers, strides up to 32 E between the lanes of a warp by
// shuffles, larger ones through shared memory (element-major there: logical t * E + e at
// e * kGroupThreads + t, so the writes and the partner reads are both conflict-free).
// The sorted keys end in keys[0, kGroupThreads * E) in logical order. Every thread calls it.
template <int E>
__device__ void sort_keys(const uint64_t* g, int T, uint64_t* keys) {
  const int t = threadIdx.x;
  constexpr int N = kGroupThreads * E;
  uint64_t x[E];
#pragma unroll
  for (int e = 0; e < E; ++e) x[e] = t * E + e < T ? g[t * E + e] : ~0ull;
  for (int k2 = 2; k2 <= N; k2 <<= 1)
    for (int j = k2 >> 1; j > 0; j >>= 1) {
      if (j < E) {
        if (j == 1) sort_stage_regs<E, 1>(x, t, k2);
        if constexpr (E > 2) if (j == 2) sort_stage_regs<E, 2>(x, t, k2);
        if constexpr (E > 4) if (j == 4) sort_stage_regs<E, 4>(x, t, k2);
        if constexpr (E > 8) if (j == 8) sort_stage_regs<E, 8>(x, t, k2);
      } else {
        const bool in_warp = j < 32 * E;
        if (!in_warp) {  // partner in another warp
          __syncthreads();  // the previous stage's readers are done
#pragma unroll
          for (int e = 0; e < E; ++e) keys[e * kGroupThreads + t] = x[e];
          __syncthreads();
        }
        const int m = j / E;  // the partner thread: t ^ m
#pragma unroll
        for (int e = 0; e < E; ++e) {
          const int i = t * E + e;
          const uint64_t y = in_warp ? shfl_xor_u64(x[e], m) : keys[e * kGroupThreads + (t ^ m)];
          const bool keep_min = ((i & k2) == 0) == ((i & j) == 0);
          x[e] = keep_min ? (x[e] < y ? x[e] : y) : (x[e] < y ? y : x[e]);
        }
      }
    }
  __syncthreads();
#pragma unroll
  for (int e = 0; e < E; ++e) keys[t * E + e] = x[e];
  __syncthreads();
}

// One CTA per sequence: sorts the chunk's queries by their keys (the hash only brings equal
// sets together; adjacent queries are compared set for set) and cuts every run of equal sets
// into groups of up to 128 queries. Queries with an empty route join none.
__global__ void __launch_bounds__(kGroupThreads, 1) group_kernel(const GroupArgs a) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  __shared__ int3 wsum[kGroupThreads / 32];
  __shared__ int s_base[3];
  const int b = blockIdx.x, tid = threadIdx.x;
  const int T = a.T;
  int np2 = kGroupThreads;
  while (np2 < T) np2 <<= 1;
  uint64_t* keys = reinterpret_cast<uint64_t*>(smem_raw);  // np2 sort keys: hash (high bits) | position
  int* hp = reinterpret_cast<int*>(keys + np2);              // segment starts (T + 1)
  griddep_wait();
  griddep_launch_dependents();
  const int m_b = a.prefix_len[b];
  if (tid == 0 && (m_b < 0 || m_b > a.cap)) set_status(a.status, RSWA_DEVICE_BAD_PREFIX_LEN);
  const uint64_t* gkeys = a.keys + (int64_t)b * T;
  switch (np2 / kGroupThreads) {  // uniform over the CTA
    case 1: sort_keys<1>(gkeys, T, keys); break;
    case 2: sort_keys<2>(gkeys, T, keys); break;
    case 4: sort_keys<4>(gkeys, T, keys); break;
    case 8: sort_keys<8>(gkeys, T, keys); break;
    default: sort_keys<16>(gkeys, T, keys); break;
  }
  // positions [p0, p1) per thread (contiguous, so the scans give ranks in position order)
  const int per = (T + kGroupThreads - 1) / kGroupThreads;
  const int p0 = min(T, tid * per), p1 = min(T, p0 + per);
  auto valid_at = [&](int p) { return keys[p] != ~0ull; };
  auto pos_at = [&](int p) { return (int)(keys[p] & 0x1FFFull); };
  uint8_t* hf = reinterpret_cast<uint8_t*>(hp + T + 1);  // per position: segment head
  // a position starts a segment unless its neighbour below has the same hash and, compared
  // block by block, the same set (rows hold the blocks ascending, INT_MAX past the valid
  // ones, so the first topk entries decide); positions strided over the threads, so that each
  // thread's row loads are independent
  const int chunks = (a.topk + 3) / 4;
#pragma unroll 2
  for (int p = tid; p < T; p += kGroupThreads) {
    bool head = false;
    if (valid_at(p)) {
      head = p == 0 || (keys[p] >> 13) != (keys[p - 1] >> 13);
      if (!head) {
        const int4* u = reinterpret_cast<const int4*>(a.gblk + ((int64_t)b * T + pos_at(p)) * kMaxTopk);
        const int4* v = reinterpret_cast<const int4*>(a.gblk + ((int64_t)b * T + pos_at(p - 1)) * kMaxTopk);
        bool same = true;
#pragma unroll
        for (int c = 0; c < kMaxTopk / 4; ++c)
          if (c < chunks) {
            const int4 x = u[c], y = v[c];
            same &= x.x == y.x && x.y == y.y && x.z == y.z && x.w == y.w;
          }
        head = !same;
      }
    }
    hf[p] = head ? 1 : 0;
  }
  __syncthreads();
  int nh = 0, nv = 0;
  for (int p = p0; p < p1; ++p) {
    nh += hf[p];
    nv += valid_at(p) ? 1 : 0;
  }
  int3 tot;
  int3 inc = block_scan3(make_int3(nh, nv, 0), wsum, tot);
  {  // segment starts: hp[s] for segment s, hp[nseg] = number of valid positions
    int s = inc.x - nh;
    for (int p = p0; p < p1; ++p)
      if (hf[p]) hp[s++] = p;
    if (tid == 0) hp[tot.x] = tot.y;
  }
  __syncthreads();
  // per position: its segment [start, end) and the groups of 128 cut from it
  int ng = 0, nq = 0;
  {
    int s = inc.x - nh - 1;
    for (int p = p0; p < p1; ++p) {
      if (!valid_at(p)) continue;
      if (hf[p]) ++s;
      ++nq;
      ng += ((p - hp[s]) % kGroupRows == 0) ? 1 : 0;
    }
  }
  const int3 ex = block_scan3(make_int3(ng, nq, 0), wsum, tot);
  if (tid == 0) {
    s_base[0] = atomicAdd(a.counts + 0, tot.x);
    s_base[1] = atomicAdd(a.counts + 1, tot.y);
  }
  __syncthreads();
  int g = s_base[0] + ex.x - ng, q = s_base[1] + ex.y - nq;
  int s = inc.x - nh - 1;
  for (int p = p0; p < p1; ++p) {
    if (!valid_at(p)) continue;
    if (hf[p]) ++s;
    const int st = hp[s], en = hp[s + 1];
    const int t = pos_at(p);
    if ((p - st) % kGroupRows == 0) {  // a group starts here: its record, blocks ascending
      const int32_t* gb = a.gblk + ((int64_t)b * T + t) * kMaxTopk;
      int32_t* rec = a.rec + (int64_t)g * kRec;
      int k = 0;
#pragma unroll
      for (int j = 0; j < kMaxTopk; ++j) {
        const int c = gb[j];
        rec[4 + j] = c == 0x7fffffff ? -1 : c;
        k += c == 0x7fffffff ? 0 : 1;
      }
      rec[0] = b;
      rec[1] = min(kGroupRows, en - p);
      rec[2] = q;
      rec[3] = k;
      ++g;
    }
    a.gq[q++] = t;  // its biases stay in the scratch row of (b, t), in the group's block order
  }
}

// ---- routed part: one (group, head) per work unit, persistent CTAs ------------------------
//   warp 0, lane 0 : TMA producer of the unit's K tiles, then its V tiles, through a
//                    4-stage ring (a tile is 4 routed blocks of 32 rows, one box each half)
//   warp 1         : allocates TMEM; lane 0 issues tcgen05.mma; the warp zeroes V rows that
//                    no query may see (past the prefix, or a missing block slot)
//   warps 2-3      : gather the group's query rows into the 128B-swizzled Q tile
//   warps 4-7      : softmax (thread r owns query row r) and the merge with the band part
// TMEM: S of the (up to) 4 key tiles in columns [0, 512); the exact row maximum is taken
// over all of them first (pass 1), then P = 2^(s - max) is written as bf16 pairs over the
// S columns already read (P of tile t at [64 t, 64 t + 64)), and O accumulates at
// [256, 384) once S has been read: no running rescale is needed.

constexpr int kRoutedThreads = 256;
constexpr int kKV = 4;                         // K / V tile stages
constexpr int kRowsR = 128;
constexpr int kRegionR = kRowsR * 128;         // one 64-column SW128 region of a 128-row tile
constexpr int kTileR = 2 * kRegionR;           // 128 x 128 bf16
constexpr int kBlockBox = 32 * 128;            // one 32-row box of one region
constexpr uint32_t kColOR = 256;

struct __align__(1024) RoutedSmem {
  uint8_t q[kTileR];
  uint8_t kv[kKV][kTileR];
  uint64_t q_full, q_empty;
  uint64_t kv_full[kKV], kv_empty[kKV];
  uint64_t s_full[kChunkBlocks / 4];  // S of key tile t of the pass is in TMEM
  uint64_t p_full, o_full, o_free;
  uint32_t tmem_base;
  int abort_flag;
};

struct RoutedArgs {
  int H, T, topk;
  int64_t cap;
  const int32_t* prefix_len;
  const uint16_t* q;       // [B][H][T][D]
  const int32_t* rec;
  const int32_t* gq;
  const float* gbias;      // per (b, t): ln p of the query's blocks, in the group record's order
  const int32_t* counts;
  float qk_scale_log2;
  float* out;              // [B][H][T][D]: the band part in, the merged result out
  float* lse;              // [B][H][T]
  int32_t* status;
};

// A work unit is (group, head); its blocks are taken in passes of up to 16 (4 key tiles),
// each merged into (out, lse) in turn by the same CTA.
struct Unit {
  int b, h, count, qoff, nblk, m;
  int blocks[kMaxTopk];  // read with compile-time indices only (see unit_block), so it stays in registers
};

__device__ __forceinline__ Unit unit_at(const RoutedArgs& a, int u) {
  Unit w;
  const int g = u / a.H;
  w.h = u - g * a.H;
  const int4* rec = reinterpret_cast<const int4*>(a.rec + (int64_t)g * kRec);  // 16-byte aligned records
  const int4 hd = rec[0];
  w.b = hd.x;
  w.count = hd.y;
  w.qoff = hd.z;
  w.nblk = hd.w;
#pragma unroll
  for (int j = 0; j < kMaxTopk; j += 4) {
    const int4 v = rec[1 + j / 4];
    w.blocks[j] = v.x;
    w.blocks[j + 1] = v.y;
    w.blocks[j + 2] = v.z;
    w.blocks[j + 3] = v.w;
  }
  const int m = a.prefix_len[w.b];
  w.m = (m < 0 || m > a.cap) ? 0 : m;
  return w;
}

// Block of slot j (compile-time) of pass c.
__device__ __forceinline__ int unit_block(const Unit& w, int c, int j) {
  return c == 0 ? w.blocks[j] : w.blocks[kChunkBlocks + j];
}

__device__ __forceinline__ int unit_passes(const Unit& w) { return (w.nblk + kChunkBlocks - 1) / kChunkBlocks; }

// Blocks of pass c of a unit.
__device__ __forceinline__ int pass_blocks(const Unit& w, int c) { return min(kChunkBlocks, w.nblk - c * kChunkBlocks); }

__device__ __forceinline__ bool routed_wait(RoutedSmem& sm, uint64_t* bar, uint32_t parity, int32_t* status) {
  if (*reinterpret_cast<volatile int*>(&sm.abort_flag)) return false;
  if (mbar_wait(bar, parity)) return true;
  sm.abort_flag = 1;
  set_status(status, RSWA_DEVICE_WAIT_TIMEOUT);
  return false;
}

// Element j (run-time) of a 16-entry register array, by selects (an indexed read would move the
// array to local memory).
template <typename V>
__device__ __forceinline__ V pick16(const V (&x)[kChunkBlocks], int j) {
  V r = x[0];
#pragma unroll
  for (int i = 1; i < kChunkBlocks; ++i) r = j == i ? x[i] : r;
  return r;
}

// Valid rows of block slot j of pass c: 0 for a missing slot, else the block's rows inside the prefix.
__device__ __forceinline__ int slot_rows(const Unit& w, int c, int j) {
  if (j >= kChunkBlocks || c * kChunkBlocks + j >= w.nblk) return 0;
  return max(0, min(32, w.m - 32 * unit_block(w, c, j)));
}

__global__ void __launch_bounds__(kRoutedThreads, 1)
    routed_kernel(const __grid_constant__ RoutedArgs a, const __grid_constant__ CUtensorMap tm_pk,
                  const __grid_constant__ CUtensorMap tm_pv) {
  extern __shared__ uint8_t smem_raw[];
  RoutedSmem& sm = *reinterpret_cast<RoutedSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    sm.abort_flag = 0;
    mbar_init(&sm.q_full, 64);
    mbar_init(&sm.q_empty, 1);
    for (int s = 0; s < kKV; ++s) {
      mbar_init(&sm.kv_full[s], 1);
      mbar_init(&sm.kv_empty[s], 1);
    }
    for (int t = 0; t < kChunkBlocks / 4; ++t) mbar_init(&sm.s_full[t], 1);
    mbar_init(&sm.p_full, 128);
    mbar_init(&sm.o_full, 1);
    mbar_init(&sm.o_free, 128);
    fence_mbar_init();
  }
  griddep_wait();  // the groups and the band part come from the previous kernels (and their TMEM is free)
  griddep_launch_dependents();
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(&sm.tmem_base)),
                 "r"(512)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  const int n_units = a.counts[0] * a.H;
  const int grid = gridDim.x;

  // Every role walks the same (unit, pass) sequence; `it` counts the passes, which each
  // complete one phase of q_full, q_empty, s_full, p_full, o_full and o_free.
  if (warp == 0) {
    if (lane == 0) {
      // ---------------- producer: K tiles then V tiles of each pass ----------------
      int idx = 0;  // tiles through the ring so far
      bool ok = true;
      Unit wn;  // the next unit's record, loaded one unit ahead
      if ((int)blockIdx.x < n_units) wn = unit_at(a, blockIdx.x);
      for (int u = blockIdx.x; ok && u < n_units; u += grid) {
        const Unit w = wn;
        if (u + grid < n_units) wn = unit_at(a, u + grid);
        const int64_t row0 = ((int64_t)w.b * a.H + w.h) * a.cap;
        for (int c = 0; ok && c < unit_passes(w); ++c) {
          const int nkt = (pass_blocks(w, c) + 3) / 4;
          for (int kvsel = 0; ok && kvsel < 2; ++kvsel) {
            const CUtensorMap* map = kvsel == 0 ? &tm_pk : &tm_pv;
#pragma unroll
            for (int t = 0; t < kChunkBlocks / 4; ++t) {
              if (t >= nkt) break;
              const int s = idx % kKV;
              if (idx >= kKV && !(ok = routed_wait(sm, &sm.kv_empty[s], ((idx / kKV) - 1) & 1, a.status))) break;
              ++idx;
              const int nb = min(4, pass_blocks(w, c) - 4 * t);  // block slots of the tile
              mbar_arrive_expect_tx(&sm.kv_full[s], (uint32_t)nb * 2 * kBlockBox);
#pragma unroll
              for (int j = 0; j < 4; ++j)
                if (j < nb) {
                  const int row = (int)(row0 + 32 * unit_block(w, c, 4 * t + j));
                  tma_load_2d(sm.kv[s] + j * kBlockBox, map, 0, row, &sm.kv_full[s]);
                  tma_load_2d(sm.kv[s] + kRegionR + j * kBlockBox, map, 64, row, &sm.kv_full[s]);
                }
            }
          }
        }
      }
      if (sm.abort_flag)  // let copies in flight land before shared memory is released
        for (int i = max(0, idx - kKV); i < idx; ++i) mbar_wait(&sm.kv_full[i % kKV], (i / kKV) & 1);
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer (lane 0) + V-row zeroing (whole warp) ----------------
    constexpr uint32_t kIdescQK = idesc_bf16_m128_n128(0);
    constexpr uint32_t kIdescPV = idesc_bf16_m128_n128(1);
    int idx = 0, it = 0;
    bool ok = true;
    Unit wn;  // the next unit's record, loaded one unit ahead
    if ((int)blockIdx.x < n_units) wn = unit_at(a, blockIdx.x);
    for (int u = blockIdx.x; ok && u < n_units; u += grid) {
      const Unit w = wn;
      if (u + grid < n_units) wn = unit_at(a, u + grid);
      for (int c = 0; ok && c < unit_passes(w); ++c, ++it) {
        const int nkt = (pass_blocks(w, c) + 3) / 4;
        ok = __all_sync(0xffffffffu, routed_wait(sm, &sm.q_full, it & 1, a.status));
        if (!ok) break;
        tc_fence_after();
        for (int t = 0; ok && t < nkt; ++t, ++idx) {
          const int s = idx % kKV;
          ok = __all_sync(0xffffffffu, routed_wait(sm, &sm.kv_full[s], (idx / kKV) & 1, a.status));
          // S of tile 2 overwrites the columns of the previous pass's O: its merge must be done
          if (ok && t == 2 && it > 0)
            ok = __all_sync(0xffffffffu, routed_wait(sm, &sm.o_free, (it - 1) & 1, a.status));
          if (!ok) break;
          tc_fence_after();
          // K rows of a missing block slot hold stale bytes: their scores are masked
          if (lane == 0) {
            const uint32_t q_addr = smem_addr(sm.q), k_addr = smem_addr(sm.kv[s]);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              const uint32_t off = (uint32_t)(kk >> 2) * kRegionR + (uint32_t)(kk & 3) * 32u;
              tc_mma_ss(tmem + (uint32_t)t * 128u, smem_desc_sw128(q_addr + off, 16, 1024),
                        smem_desc_sw128(k_addr + off, 16, 1024), kIdescQK, kk > 0);
            }
            tc_commit(&sm.kv_empty[s]);
            tc_commit(&sm.s_full[t]);  // the softmax's first pass follows tile by tile
          }
          __syncwarp();
        }
        if (!ok) break;
        // a pass of fewer than 3 key tiles still frees the previous O before PV writes it
        if (nkt < 3 && it > 0) ok = __all_sync(0xffffffffu, routed_wait(sm, &sm.o_free, (it - 1) & 1, a.status));
        if (!ok) break;
        if (lane == 0) tc_commit(&sm.q_empty);
        __syncwarp();
        ok = __all_sync(0xffffffffu, routed_wait(sm, &sm.p_full, it & 1, a.status));
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int t = 0; t < kChunkBlocks / 4; ++t) {
          if (!ok || t >= nkt) break;
          const int s = idx % kKV;
          ok = __all_sync(0xffffffffu, routed_wait(sm, &sm.kv_full[s], (idx / kKV) & 1, a.status));
          ++idx;
          if (!ok) break;
          // zero V rows that no query may see (their P is 0; 0 * NaN would still reach O)
          bool zeroed = false;
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            const int r = lane + 32 * q4;
            if (lane >= slot_rows(w, c, 4 * t + q4)) {
              uint4* row0 = reinterpret_cast<uint4*>(sm.kv[s] + r * 128);
              uint4* row1 = reinterpret_cast<uint4*>(sm.kv[s] + kRegionR + r * 128);
#pragma unroll
              for (int e = 0; e < 8; ++e) {
                row0[e] = make_uint4(0, 0, 0, 0);
                row1[e] = make_uint4(0, 0, 0, 0);
              }
              zeroed = true;
            }
          }
          if (__any_sync(0xffffffffu, zeroed)) fence_async_smem();
          __syncwarp();
          tc_fence_after();
          if (lane == 0) {
            const uint32_t v_addr = smem_addr(sm.kv[s]);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)  // 16 keys per step: 8 packed TMEM columns of P, two 8-row groups of V
              tc_mma_ts(tmem + kColOR, tmem + (uint32_t)t * 64u + (uint32_t)kk * 8u,
                        smem_desc_sw128(v_addr + (uint32_t)kk * 2048u, kRegionR, 1024), kIdescPV,
                        (t > 0 || kk > 0) ? 1u : 0u);
            tc_commit(&sm.kv_empty[s]);
          }
          __syncwarp();
        }
        if (!ok) break;
        if (lane == 0) tc_commit(&sm.o_full);
        __syncwarp();
      }
    }
    if (!ok && lane == 0) {  // o_full's next phase fires once every issued MMA is done: TMEM can go
      tc_commit(&sm.o_full);
      mbar_wait(&sm.o_full, it & 1);
    }
  } else if (warp < 4) {
    // ---------------- Q gather: the group's query rows, 128B-swizzled ----------------
    const int gt = tid - 64;  // 0..63
    int it = 0;
    bool ok = true;
    for (int u = blockIdx.x; ok && u < n_units; u += grid) {
      const Unit w = unit_at(a, u);
      const int64_t qrow0 = ((int64_t)w.b * a.H + w.h) * a.T;
      for (int c = 0; c < unit_passes(w); ++c, ++it) {
        if (it > 0 && !(ok = routed_wait(sm, &sm.q_empty, (it - 1) & 1, a.status))) break;
        for (int r = gt; r < kRowsR; r += 64) {  // a row per thread: its 16 chunks of 16 bytes in flight together
          uint4 v[16];
          if (r < w.count) {
            const uint4* src = reinterpret_cast<const uint4*>(a.q + (qrow0 + a.gq[w.qoff + r]) * kHeadDim);
#pragma unroll
            for (int c16 = 0; c16 < 16; ++c16) v[c16] = __ldg(src + c16);
          } else {
#pragma unroll
            for (int c16 = 0; c16 < 16; ++c16) v[c16] = make_uint4(0, 0, 0, 0);
          }
#pragma unroll
          for (int c16 = 0; c16 < 16; ++c16) {
            const int region = c16 >> 3, ch = c16 & 7;
            *reinterpret_cast<uint4*>(sm.q + region * kRegionR + r * 128 + ((ch ^ (r & 7)) << 4)) = v[c16];
          }
        }
        fence_async_smem();
        mbar_arrive(&sm.q_full);
      }
    }
  } else {
    // ---------------- softmax and merge: thread r owns query row r ----------------
    const int r = tid - 128;
    const uint32_t lane_base = (uint32_t)((warp - 4) * 32) << 16;
    int it = 0;
    uint32_t s_phase = 0;  // bit t: parity of the next completion of s_full[t]
    bool ok = true;
    for (int u = blockIdx.x; ok && u < n_units; u += grid) {
      const Unit w = unit_at(a, u);
      const bool live = r < w.count;
      const int t_q = live ? a.gq[w.qoff + r] : 0;
      for (int c = 0; c < unit_passes(w); ++c, ++it) {
        const int nkt = (pass_blocks(w, c) + 3) / 4;
        // the row's bias per block slot of the pass (log2 domain), from its own route in the
        // group's block order, and the slot's valid rows
        float bias[kChunkBlocks];
        int rows[kChunkBlocks];
        {
          const float4* gb = reinterpret_cast<const float4*>(a.gbias + ((int64_t)w.b * a.T + t_q) * kMaxTopk +
                                                             c * kChunkBlocks);
#pragma unroll
          for (int j = 0; j < kChunkBlocks; j += 4) {
            const float4 v = __ldg(gb + j / 4);
            bias[j] = v.x * kLog2eR;
            bias[j + 1] = v.y * kLog2eR;
            bias[j + 2] = v.z * kLog2eR;
            bias[j + 3] = v.w * kLog2eR;
          }
#pragma unroll
          for (int j = 0; j < kChunkBlocks; ++j) {
            rows[j] = slot_rows(w, c, j);
            if (!live) bias[j] = -INFINITY;
          }
        }
        // pass 1: the row maximum over every routed key of the pass, key tile by key tile as the
        // tensor core finishes them; two 32-column chunks (block slots) per TMEM wait
        float mx = -INFINITY;
#pragma unroll 1
        for (int j = 0; j < 4 * nkt; j += 2) {
          if ((j & 3) == 0) {
            // s_full[t] completes once per pass that has key tile t: its own phase bit
            const int t = j >> 2;
            if (!(ok = __all_sync(0xffffffffu, routed_wait(sm, &sm.s_full[t], (s_phase >> t) & 1u, a.status))))
              break;
            s_phase ^= 1u << t;
            tc_fence_after();
          }
          uint32_t rv[32], rw[32];
          tmem_ld32(tmem + lane_base + (uint32_t)(j * 32), rv);
          tmem_ld32(tmem + lane_base + (uint32_t)(j * 32 + 32), rw);
          tmem_wait_ld();
          const float bj = pick16(bias, j), bk = pick16(bias, j + 1);
          const int nr = pick16(rows, j), ns = pick16(rows, j + 1);
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            if (e < nr) mx = fmaxf(mx, fmaf(__uint_as_float(rv[e]), a.qk_scale_log2, bj));
            if (e < ns) mx = fmaxf(mx, fmaf(__uint_as_float(rw[e]), a.qk_scale_log2, bk));
          }
        }
        if (!ok) break;
        const float msub = mx == -INFINITY ? 0.f : mx;
        // pass 2: P = 2^(s - max) as bf16 pairs over the S columns already read; two chunks per
        // TMEM wait (P of chunk j lands in columns [16 j, 16 j + 16), inside chunks already read)
        float l = 0.f, lu = 0.f;
        auto p_chunk = [&](const uint32_t (&rv)[32], float bj, int nr, uint32_t (&pk)[16]) {
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const float x0 = 2 * e < nr ? fmaf(__uint_as_float(rv[2 * e]), a.qk_scale_log2, bj) - msub : -INFINITY;
            const float x1 =
                2 * e + 1 < nr ? fmaf(__uint_as_float(rv[2 * e + 1]), a.qk_scale_log2, bj) - msub : -INFINITY;
            const float p0 = ex2(x0), p1 = ex2(x1);  // MUFU 2^x (2^-inf = 0), as in the dense prefill
            const __nv_bfloat162 pb = __floats2bfloat162_rn(p0, p1);
            pk[e] = *reinterpret_cast<const uint32_t*>(&pb);
            l += __uint_as_float(pk[e] << 16) + __uint_as_float(pk[e] & 0xffff0000u);
            lu += p0 + p1;
          }
        };
#pragma unroll 1
        for (int j = 0; j < 4 * nkt; j += 2) {
          uint32_t rv[32], rw[32], pk[16];
          tmem_ld32(tmem + lane_base + (uint32_t)(j * 32), rv);
          tmem_ld32(tmem + lane_base + (uint32_t)(j * 32 + 32), rw);
          tmem_wait_ld();
          p_chunk(rv, pick16(bias, j), pick16(rows, j), pk);
          tmem_st16(tmem + lane_base + (uint32_t)(j * 16), pk);
          p_chunk(rw, pick16(bias, j + 1), pick16(rows, j + 1), pk);
          tmem_st16(tmem + lane_base + (uint32_t)(j * 16 + 16), pk);
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&sm.p_full);
        // the band part's row: brought into L1 while the tensor core runs P.V, read at the merge
        // (held in registers instead, it would leave too few for the paired TMEM loads)
        const int64_t vq = ((int64_t)w.b * a.H + w.h) * a.T + t_q;
        float* orow = a.out + vq * kHeadDim;
        float lse_a = -INFINITY;
        if (live) {
#pragma unroll
          for (int e = 0; e < kHeadDim; e += 32) asm volatile("prefetch.global.L1 [%0];" ::"l"(orow + e));
          lse_a = a.lse[vq];
        }
        if (!(ok = __all_sync(0xffffffffu, routed_wait(sm, &sm.o_full, it & 1, a.status)))) break;
        tc_fence_after();
        // merge into (out, lse): a softmax over the union of disjoint key sets
        const float lse_r = (lu > 0.f) ? (mx + log2f(lu)) * kLn2R : -INFINITY;
        float wa = 0.f, wr = 0.f, lse_new = 0.f;
        if (live) {
          const float mm = fmaxf(lse_a, lse_r);
          wa = lse_a > -INFINITY ? expf(lse_a - mm) : 0.f;
          wr = lse_r > -INFINITY ? expf(lse_r - mm) : 0.f;
          const float ws = wa + wr;
          lse_new = ws > 0.f ? mm + logf(ws) : -INFINITY;
          if (ws > 0.f) {
            wa /= ws;
            wr /= ws;
          }
        }
        const float inv_l = l > 0.f ? wr / l : 0.f;
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
          uint32_t rv[32];
          tmem_ld32(tmem + lane_base + kColOR + (uint32_t)ch * 32u, rv);
          tmem_wait_ld();
          if (live) {
            float4 ob[8];  // the band part's values of these 32 columns
#pragma unroll
            for (int e = 0; e < 8; ++e) ob[e] = reinterpret_cast<const float4*>(orow + ch * 32)[e];
#pragma unroll
            for (int e = 0; e < 32; e += 4) {
              float4 o = ob[e / 4];
              o.x = fmaf(o.x, wa, __uint_as_float(rv[e]) * inv_l);
              o.y = fmaf(o.y, wa, __uint_as_float(rv[e + 1]) * inv_l);
              o.z = fmaf(o.z, wa, __uint_as_float(rv[e + 2]) * inv_l);
              o.w = fmaf(o.w, wa, __uint_as_float(rv[e + 3]) * inv_l);
              *reinterpret_cast<float4*>(orow + ch * 32 + e) = o;
            }
          }
        }
        if (live) a.lse[vq] = lse_new;
        tc_fence_before();
        mbar_arrive(&sm.o_free);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512) : "memory");
}

}  // namespace

// Workspace of srswa_prefill past its status area: [counts 256 B][group records][gq][gblk][gbias][lse scratch]
// [sort keys].
size_t srswa_prefill_scratch_bytes(int B, int H, int T) {
  const size_t bt = (size_t)B * T;
  return 256 + (bt * kRec * 4 + 255) / 256 * 256 + (bt * 4 + 255) / 256 * 256 + bt * kMaxTopk * 8 +
         ((size_t)B * H * T * 4 + 255) / 256 * 256 + bt * 8;
}

int srswa_prefill_group_rec_ints() { return kRec; }

cudaError_t launch_srswa_group(int B, int T, int topk, int64_t cap, const int32_t* prefix_len, const int32_t* blk,
                               const float* logp, int32_t* rec, int32_t* gq, int32_t* gblk, float* gbias,
                               int32_t* counts, uint64_t* keys, int32_t* status, cudaStream_t stream) {
  GroupArgs a{B, T, topk, cap, prefix_len, status, blk, logp, rec, gq, gblk, gbias, counts, keys};
  {  // the per-query part over the whole grid, then the per-sequence sort and cut
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    const int64_t queries = (int64_t)B * T;
    fill_launch_config(cfg, attr, dim3((unsigned)((queries + kPrepThreads - 1) / kPrepThreads)), dim3(kPrepThreads),
                       0, stream);
    cudaError_t e = cudaLaunchKernelEx(&cfg, group_prep_kernel, a);
    if (e != cudaSuccess) return e;
  }
  int np2 = 1;
  while (np2 < T) np2 <<= 1;
  if (np2 < kGroupThreads) np2 = kGroupThreads;
  const size_t smem = (size_t)np2 * 8 + (size_t)(T + 1) * 4 + (size_t)T;
  static unsigned long long done = 0;
  cudaError_t e = ensure_smem_limit(group_kernel, (size_t)8192 * 8 + 8193 * 4 + 8192, &done);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  fill_launch_config(cfg, attr, dim3(B), dim3(kGroupThreads), smem, stream);
  return cudaLaunchKernelEx(&cfg, group_kernel, a);
}

cudaError_t launch_srswa_routed(int B, int H, int T, int topk, int64_t cap, const int32_t* prefix_len, const void* q,
                                const void* pk, const void* pv, const int32_t* rec, const int32_t* gq,
                                const float* gbias, const int32_t* counts, float scale, float* out, float* lse,
                                int32_t* status, cudaStream_t stream) {
  CUtensorMap tpk, tpv;
  const int64_t rows = (int64_t)B * H * cap;
  cudaError_t e;
  if ((e = make_rows_map(&tpk, pk, rows, 32)) != cudaSuccess) return e;
  if ((e = make_rows_map(&tpv, pv, rows, 32)) != cudaSuccess) return e;
  RoutedArgs a;
  a.H = H;
  a.T = T;
  a.topk = topk;
  a.cap = cap;
  a.prefix_len = prefix_len;
  a.q = static_cast<const uint16_t*>(q);
  a.rec = rec;
  a.gq = gq;
  a.gbias = gbias;
  a.counts = counts;
  a.qk_scale_log2 = scale * kLog2eR;
  a.out = out;
  a.lse = lse;
  a.status = status;
  const size_t smem = sizeof(RoutedSmem) + 1024;
  static unsigned long long done = 0;
  if ((e = ensure_smem_limit(routed_kernel, smem, &done)) != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  fill_launch_config(cfg, attr, dim3(device_sm_count()), dim3(kRoutedThreads), smem, stream);
  return cudaLaunchKernelEx(&cfg, routed_kernel, a, tpk, tpv);
}

}  // namespace rswa
