// prefill.cu -- chunked R-SWA prefill on sm_100a tensor cores (tcgen05 + TMEM).
//
// Output-side query i of a chunk attends to every reference-prefix token and to
// the output tokens j with i - n < j <= i ("百度 Unlimited OCR 深度实战" tutorial
// §3.3.1: reference positions always visible, only the most recent n output
// positions visible). Positions j < 0 belong to a previous chunk and are read
// from the ring (the r-th most recent slot is (wp - r) mod n, present when
// r <= fill).
//
// This is the path's one dense contraction, so it runs on the 5th-generation
// tensor cores. One CTA owns two 128-row query tiles (A and B) of one
// (sequence, head) and walks the key tiles (128 keys each) both need:
//   warp 0, lane 0  : TMA producer of Q (both tiles) and of the K tiles (3 stages)
//   warp 2, lane 0  : TMA producer of the V tiles (2 stages)
//   warp 1          : allocates TMEM; lane 0 issues tcgen05.mma; the warp zeroes
//                     the V rows of keys no query may see (their P is 0, their
//                     bytes may be anything, and 0 * NaN would reach O)
//   warps 4-7 / 8-11: softmax of tile A / tile B; thread r owns query row r, i.e.
//                     TMEM lane r of its tile's S, P and O.
// TMEM (512 columns): S_A [0,128), S_B [128,256), O_A [256,384), O_B [384,512).
// P (bf16, two per 32-bit column) is written over the first 64 columns of its
// tile's S once those scores have been read, and the P.V product takes its A
// operand straight from TMEM. The MMA thread issues, per key tile t,
//   PV_A(t), S_A(t+1), PV_B(t), S_B(t+1)
// so while one tile's softmax runs the tensor core works on the other tile.
// Tensor-core operations of one thread execute in issue order, so S_A(t+1) may
// overwrite P_A(t) right after PV_A(t) is issued, and a softmax that sees S_X(t)
// complete also knows PV_X(t-1) has completed (the commit covers every earlier
// operation): the O rescale it may then do needs no further wait.
// The running max only moves when it grows by more than 2^8 (log2 units); the
// exponentials stay below 256 and the final O / l is the same quotient, so this
// lazy rescale is exact and the O read-modify-write through TMEM is rare.
// (query tile, key tile) pairs in which every score is masked are skipped by the
// MMA thread and the softmax alike.
// Every mbarrier wait is bounded; on expiry the kernel flags
// RSWA_DEVICE_WAIT_TIMEOUT, drains what it issued and frees its TMEM.
#include <cuda.h>
#include <cuda_bf16.h>

#include <cmath>

#include "common.cuh"
#include "internal.h"
#include "tcgen05.cuh"

namespace rswa {

namespace {

constexpr int kTileRows = 128;                 // query rows per tile, keys per key tile
constexpr int kQTiles = 2;                     // query tiles per CTA
constexpr int kRegionBytes = kTileRows * 128;  // one 64-column SW128 region of a 128-row tile
constexpr int kTileBytes = 2 * kRegionBytes;   // 128 x 128 bf16
constexpr int kKStages = 3;
constexpr int kVStages = 2;
constexpr int kPrefillThreads = 384;
constexpr int kSoftmaxWarp0 = 4;               // warps 4-7: tile A, 8-11: tile B
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 256;                // O_A at 256, O_B at 384
constexpr float kLazyRescaleLog2 = 8.f;
constexpr float kLog2eP = 1.4426950408889634f;
constexpr float kLn2P = 0.6931471805599453f;

struct PrefillCtx {
  int m, n, fill, wp, T, i0;  // i0: first query row of the CTA (tile A)
  int np, nr, jt0, jt1, total;
  int has_ring;
};

struct __align__(1024) PrefillSmem {
  uint8_t q[kQTiles][kTileBytes];
  uint8_t k[kKStages][kTileBytes];
  uint8_t v[kVStages][kTileBytes];
  uint64_t q_full;
  uint64_t k_full[kKStages], k_empty[kKStages];
  uint64_t v_full[kVStages], v_empty[kVStages];
  uint64_t s_full[kQTiles], p_full[kQTiles], o_done[kQTiles];
  uint32_t tmem_base;
  int abort_flag;
  PrefillCtx ctx;
};

// ---- key-tile enumeration shared by every role -----------------------------------
// kind 0: prefix rows [start, start+128); kind 1: ring slots [start, start+128);
// kind 2: output rows [start, start+128) of this chunk.
__device__ __forceinline__ void tile_kind(const PrefillCtx& c, int t, int& kind, int& start) {
  if (t < c.np) {
    kind = 0;
    start = t * kTileRows;
  } else if (t < c.np + c.nr) {
    kind = 1;
    start = (t - c.np) * kTileRows;
  } else {
    kind = 2;
    start = (c.jt0 + t - c.np - c.nr) * kTileRows;
  }
}

// Age of ring slot s: 1 for the most recently written slot.
__device__ __forceinline__ int ring_age(const PrefillCtx& c, int s) {
  int a = (c.wp - 1 - s) % c.n;
  if (a < 0) a += c.n;
  return a + 1;
}

// Can any query of the chunk see key row `row` of tile (kind, start)?
__device__ __forceinline__ bool key_exists(const PrefillCtx& c, int kind, int start, int row) {
  const int x = start + row;
  if (kind == 0) return x < c.m;
  if (kind == 1) return x < c.n && ring_age(c, x) <= c.fill;
  return x < c.T;
}

// Is key row `row` of tile (kind, start) visible to query position i?
__device__ __forceinline__ bool key_visible(const PrefillCtx& c, int kind, int start, int row, int i) {
  const int x = start + row;
  if (kind == 0) return x < c.m;
  if (kind == 1) {
    if (x >= c.n) return false;
    const int age = ring_age(c, x);
    return age <= c.fill && age < c.n - i;
  }
  return x < c.T && x <= i && x > i - c.n;
}

// Does query tile X see anything of key tile t?
__device__ __forceinline__ bool tile_visible(const PrefillCtx& c, int X, int t) {
  const int ilo = c.i0 + X * kTileRows;
  if (ilo >= c.T) return false;
  const int ihi = min(ilo + kTileRows - 1, c.T - 1);
  int kind, start;
  tile_kind(c, t, kind, start);
  if (kind == 0) return true;
  if (kind == 1) return ilo <= c.n - 2;
  const int jhi = min(start + kTileRows - 1, c.T - 1);
  return start <= ihi && jhi >= ilo - c.n + 1;
}

struct PrefillArgs {
  int B, H, n, T;
  int64_t cap;
  const int32_t* prefix_len;
  const int32_t* wp;
  const int32_t* fill;
  int has_ring;
  int ignore_prefix;  // 1: no query sees the prefix (the SR-SWA prefill's band and ring part)
  float qk_scale_log2;
  float* out;
  float* lse;
  int32_t* status;
};

__device__ __forceinline__ bool wait_or_abort(PrefillSmem& sm, uint64_t* bar, uint32_t parity, int32_t* status) {
  if (*reinterpret_cast<volatile int*>(&sm.abort_flag)) return false;
  if (mbar_wait(bar, parity)) return true;
  sm.abort_flag = 1;
  set_status(status, RSWA_DEVICE_WAIT_TIMEOUT);
  return false;
}

// Masked, scaled scores of one 32-column chunk of a tile (log2 domain).
__device__ __forceinline__ void mask_chunk(const PrefillCtx& c, int kind, int start, int i, int col0, float scale,
                                           const uint32_t (&r)[32], float (&x)[32]) {
  if (kind == 1) {
#pragma unroll
    for (int e = 0; e < 32; ++e)
      x[e] = key_visible(c, kind, start, col0 + e, i) ? __uint_as_float(r[e]) * scale : -INFINITY;
  } else {
    // visible columns form one interval (lo, hi]: prefix rows below m; outputs i - n < j <= i, j < T
    const int hi = (kind == 0 ? min(127, c.m - start - 1) : min(127, min(i, c.T - 1) - start)) - col0;
    const int lo = (kind == 0 ? -1 : max(-1, i - c.n - start)) - col0;
#pragma unroll
    for (int e = 0; e < 32; ++e) x[e] = (e > lo && e <= hi) ? __uint_as_float(r[e]) * scale : -INFINITY;
  }
}

__global__ void __launch_bounds__(kPrefillThreads, 1)
    prefill_kernel(const __grid_constant__ PrefillArgs a, const __grid_constant__ CUtensorMap tm_q,
                   const __grid_constant__ CUtensorMap tm_ko, const __grid_constant__ CUtensorMap tm_vo,
                   const __grid_constant__ CUtensorMap tm_pk, const __grid_constant__ CUtensorMap tm_pv,
                   const __grid_constant__ CUtensorMap tm_rk, const __grid_constant__ CUtensorMap tm_rv) {
  extern __shared__ uint8_t smem_raw[];
  PrefillSmem& sm = *reinterpret_cast<PrefillSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

  const int qt = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t bh = (int64_t)b * a.H + h;

  __shared__ int s_skip;
  griddep_wait();
  griddep_launch_dependents();
  if (tid == 0) {
    // a CTA of this launch already gave up on a wait: skip the work (the output is flagged invalid)
    s_skip = a.status != nullptr && (*reinterpret_cast<volatile int32_t*>(a.status) & RSWA_DEVICE_WAIT_TIMEOUT);
  }
  __syncthreads();
  if (s_skip) return;

  if (tid == 0) {
    PrefillCtx c;
    int m = a.ignore_prefix ? 0 : a.prefix_len[b];
    if (m < 0 || m > a.cap) {
      if (qt == 0 && h == 0) set_status(a.status, RSWA_DEVICE_BAD_PREFIX_LEN);
      m = 0;
    }
    c.m = m;
    c.n = a.n;
    c.T = a.T;
    c.i0 = qt * kQTiles * kTileRows;
    c.wp = 0;
    c.fill = 0;
    c.has_ring = 0;
    if (a.has_ring) {
      const int w = a.wp[b], f = a.fill[b];
      if (w < 0 || w >= a.n || f < 0 || f > a.n) {
        if (qt == 0 && h == 0) set_status(a.status, RSWA_DEVICE_BAD_RING_STATE);
      } else {
        c.wp = w;
        c.fill = f;
        c.has_ring = f > 0 && c.i0 <= a.n - 2;  // some query of the CTA can still see a ring slot
      }
    }
    c.np = (m + kTileRows - 1) / kTileRows;
    c.nr = c.has_ring ? (a.n + kTileRows - 1) / kTileRows : 0;
    const int jlo = c.i0 - a.n + 1;
    c.jt0 = jlo > 0 ? jlo / kTileRows : 0;
    const int last_row = min(c.i0 + kQTiles * kTileRows - 1, a.T - 1);
    c.jt1 = last_row / kTileRows;
    c.total = c.np + c.nr + (c.jt1 - c.jt0 + 1);
    sm.ctx = c;
    sm.abort_flag = 0;
    mbar_init(&sm.q_full, 1);
    for (int s = 0; s < kKStages; ++s) {
      mbar_init(&sm.k_full[s], 1);
      mbar_init(&sm.k_empty[s], 1);
    }
    for (int s = 0; s < kVStages; ++s) {
      mbar_init(&sm.v_full[s], 1);
      mbar_init(&sm.v_empty[s], 1);
    }
    for (int x = 0; x < kQTiles; ++x) {
      mbar_init(&sm.s_full[x], 1);
      mbar_init(&sm.p_full[x], 128);
      mbar_init(&sm.o_done[x], 1);
    }
    fence_mbar_init();
  }
  if (warp == 1) {  // TMEM allocation: one warp, result written to shared memory
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(&sm.tmem_base)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const PrefillCtx c = sm.ctx;
  const uint32_t tmem = sm.tmem_base;
  const int total = c.total;

  if (warp == 0 && lane == 0) {
    // ---------------- producer: Q (both tiles) and K tiles ----------------
    const int qrow = (int)(bh * a.T) + c.i0;
    mbar_arrive_expect_tx(&sm.q_full, kQTiles * kTileBytes);
    for (int x = 0; x < kQTiles; ++x) {
      tma_load_2d(sm.q[x], &tm_q, 0, qrow + x * kTileRows, &sm.q_full);
      tma_load_2d(sm.q[x] + kRegionBytes, &tm_q, 64, qrow + x * kTileRows, &sm.q_full);
    }
    int issued = 0;
    for (int t = 0; t < total; ++t) {
      const int s = t % kKStages;
      if (t >= kKStages && !wait_or_abort(sm, &sm.k_empty[s], ((t / kKStages) - 1) & 1, a.status)) break;
      int kind, start;
      tile_kind(c, t, kind, start);
      const CUtensorMap* map = kind == 0 ? &tm_pk : (kind == 1 ? &tm_rk : &tm_ko);
      const int row =
          kind == 0 ? (int)(bh * a.cap) + start : (kind == 1 ? (int)(bh * a.n) + start : (int)(bh * a.T) + start);
      mbar_arrive_expect_tx(&sm.k_full[s], kTileBytes);
      tma_load_2d(sm.k[s], map, 0, row, &sm.k_full[s]);
      tma_load_2d(sm.k[s] + kRegionBytes, map, 64, row, &sm.k_full[s]);
      issued = t + 1;
    }
    if (sm.abort_flag) {  // let the copies in flight land before shared memory is released
      mbar_wait(&sm.q_full, 0);
      for (int t = max(0, issued - kKStages); t < issued; ++t)
        mbar_wait(&sm.k_full[t % kKStages], (t / kKStages) & 1);
    }
  } else if (warp == 2 && lane == 0) {
    // ---------------- producer: V tiles ----------------
    int issued = 0;
    for (int t = 0; t < total; ++t) {
      const int s = t % kVStages;
      if (t >= kVStages && !wait_or_abort(sm, &sm.v_empty[s], ((t / kVStages) - 1) & 1, a.status)) break;
      int kind, start;
      tile_kind(c, t, kind, start);
      const CUtensorMap* map = kind == 0 ? &tm_pv : (kind == 1 ? &tm_rv : &tm_vo);
      const int row =
          kind == 0 ? (int)(bh * a.cap) + start : (kind == 1 ? (int)(bh * a.n) + start : (int)(bh * a.T) + start);
      mbar_arrive_expect_tx(&sm.v_full[s], kTileBytes);
      tma_load_2d(sm.v[s], map, 0, row, &sm.v_full[s]);
      tma_load_2d(sm.v[s] + kRegionBytes, map, 64, row, &sm.v_full[s]);
      issued = t + 1;
    }
    if (sm.abort_flag)
      for (int t = max(0, issued - kVStages); t < issued; ++t)
        mbar_wait(&sm.v_full[t % kVStages], (t / kVStages) & 1);
  } else if (warp == 1) {
    // ---------------- MMA issuer (lane 0) + V-row zeroing (whole warp) ----------------
    constexpr uint32_t kIdescQK = idesc_bf16_m128_n128(0);
    constexpr uint32_t kIdescPV = idesc_bf16_m128_n128(1);
    int n_s[kQTiles] = {0, 0};   // S issued per query tile
    int n_pv[kQTiles] = {0, 0};  // P.V issued per query tile
    bool ok = __all_sync(0xffffffffu, wait_or_abort(sm, &sm.q_full, 0, a.status));
    auto issue_s = [&](int x, int t) {  // S_x = Q_x K_t^T
      const uint32_t q_addr = smem_addr(sm.q[x]);
      const uint32_t k_addr = smem_addr(sm.k[t % kKStages]);
      if (lane == 0) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = (uint32_t)(kk >> 2) * kRegionBytes + (uint32_t)(kk & 3) * 32u;
          tc_mma_ss(tmem + (uint32_t)x * 128u, smem_desc_sw128(q_addr + off, 16, 1024),
                    smem_desc_sw128(k_addr + off, 16, 1024), kIdescQK, kk > 0);
        }
        tc_commit(&sm.s_full[x]);
      }
      __syncwarp();
      ++n_s[x];
    };
    // key tile 0: S for both query tiles
    if (ok) {
      ok = __all_sync(0xffffffffu, wait_or_abort(sm, &sm.k_full[0], 0, a.status));
      if (ok) {
        tc_fence_after();
        for (int x = 0; x < kQTiles; ++x)
          if (tile_visible(c, x, 0)) issue_s(x, 0);
        if (lane == 0) tc_commit(&sm.k_empty[0]);
        __syncwarp();
      }
    }
    for (int t = 0; ok && t < total; ++t) {
      const int vs = t % kVStages;
      ok = __all_sync(0xffffffffu, wait_or_abort(sm, &sm.v_full[vs], (t / kVStages) & 1, a.status));
      if (!ok) break;
      int kind, start;
      tile_kind(c, t, kind, start);
      bool zeroed = false;
      for (int r = lane; r < kTileRows; r += 32) {
        if (!key_exists(c, kind, start, r)) {
          uint4* row0 = reinterpret_cast<uint4*>(sm.v[vs] + r * 128);
          uint4* row1 = reinterpret_cast<uint4*>(sm.v[vs] + kRegionBytes + r * 128);
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
      const bool next = t + 1 < total;
      bool k_next_ready = false;
      for (int x = 0; ok && x < kQTiles; ++x) {
        if (tile_visible(c, x, t)) {
          ok = __all_sync(0xffffffffu, wait_or_abort(sm, &sm.p_full[x], n_pv[x] & 1, a.status));
          if (!ok) break;
          tc_fence_after();
          if (lane == 0) {
            const uint32_t v_addr = smem_addr(sm.v[vs]);
            const uint32_t p_tmem = tmem + (uint32_t)x * 128u;
            const uint32_t o_tmem = tmem + kColO + (uint32_t)x * 128u;
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)  // 16 keys per step: 8 packed TMEM columns of P, two 8-row groups of V
              tc_mma_ts(o_tmem, p_tmem + (uint32_t)kk * 8u, smem_desc_sw128(v_addr + (uint32_t)kk * 2048u, kRegionBytes, 1024),
                        kIdescPV, (n_pv[x] > 0 || kk > 0) ? 1u : 0u);
            tc_commit(&sm.o_done[x]);
          }
          __syncwarp();
          ++n_pv[x];
        }
        if (next && tile_visible(c, x, t + 1)) {
          if (!k_next_ready) {
            ok = __all_sync(0xffffffffu,
                            wait_or_abort(sm, &sm.k_full[(t + 1) % kKStages], ((t + 1) / kKStages) & 1, a.status));
            if (!ok) break;
            tc_fence_after();
            k_next_ready = true;
          }
          issue_s(x, t + 1);
        }
      }
      if (!ok) break;
      if (lane == 0) tc_commit(&sm.v_empty[vs]);
      if (next) {
        if (!k_next_ready) {  // no query tile needed it: still let the copy land before freeing the stage
          ok = __all_sync(0xffffffffu,
                          wait_or_abort(sm, &sm.k_full[(t + 1) % kKStages], ((t + 1) / kKStages) & 1, a.status));
          if (!ok) break;
        }
        if (lane == 0) tc_commit(&sm.k_empty[(t + 1) % kKStages]);
      }
      __syncwarp();
    }
    if (!ok && lane == 0) tc_commit(&sm.o_done[0]);  // drain: the barrier fires once every issued MMA is done
  } else if (warp >= kSoftmaxWarp0) {
    // ---------------- softmax: warps 4-7 own tile A, 8-11 tile B; thread r owns row r ----------------
    const int x = (warp - kSoftmaxWarp0) / 4;
    const int r = tid - (kSoftmaxWarp0 + 4 * x) * 32;
    const int i = c.i0 + x * kTileRows + r;
    const uint32_t lane_base = (uint32_t)(((warp - kSoftmaxWarp0) & 3) * 32) << 16;
    const uint32_t s_cols = tmem + lane_base + (uint32_t)x * 128u;
    const uint32_t o_cols = tmem + lane_base + kColO + (uint32_t)x * 128u;
    // l normalises O with the same bf16-rounded weights the MMA used (a peaked softmax
    // would otherwise carry the rounding of its dominant weight into O's scale);
    // lu, the sum of the unrounded exponentials, gives lse
    float m_used = -INFINITY, l = 0.f, lu = 0.f;
    int j = 0;  // visible key tiles seen so far
    bool ok = true;
    for (int t = 0; t < total; ++t) {
      if (!tile_visible(c, x, t)) continue;
      ok = __all_sync(0xffffffffu, wait_or_abort(sm, &sm.s_full[x], j & 1, a.status));
      if (!ok) break;
      tc_fence_after();
      int kind, start;
      tile_kind(c, t, kind, start);
      // a prefix tile that lies wholly inside the prefix is visible to every row: no mask
      const bool full = kind == 0 && start + kTileRows <= c.m;
      // pass 1: the tile's row maximum (on raw scores for a full tile: the scale is positive)
      float tmax = -INFINITY;
#pragma unroll 1
      for (int ch = 0; ch < 4; ++ch) {
        uint32_t rr[32];
        tmem_ld32(s_cols + (uint32_t)ch * 32u, rr);
        tmem_wait_ld();
        float m0 = tmax, m1 = -INFINITY;  // two chains of three-input maxima
        if (full) {
#pragma unroll
          for (int e = 0; e < 32; e += 4) {
            m0 = max3(m0, __uint_as_float(rr[e]), __uint_as_float(rr[e + 1]));
            m1 = max3(m1, __uint_as_float(rr[e + 2]), __uint_as_float(rr[e + 3]));
          }
        } else {
          float xv[32];
          mask_chunk(c, kind, start, i, ch * 32, a.qk_scale_log2, rr, xv);
#pragma unroll
          for (int e = 0; e < 32; e += 4) {
            m0 = max3(m0, xv[e], xv[e + 1]);
            m1 = max3(m1, xv[e + 2], xv[e + 3]);
          }
        }
        tmax = fmaxf(m0, m1);
      }
      if (full) tmax *= a.qk_scale_log2;
      const bool rescale = tmax > m_used + kLazyRescaleLog2;
      float alpha = 1.f;
      if (rescale) {
        alpha = ex2(m_used - tmax);  // 0 while nothing has been seen
        l *= alpha;
        lu *= alpha;
        m_used = tmax;
      }
      // tcgen05.ld/st are warp-collective (.sync.aligned): the whole warp rescales its O rows
      // together, lanes that keep their max with alpha = 1. PV of the previous visible tile is
      // complete (see the header).
      if (j > 0 && __any_sync(0xffffffffu, rescale)) {
#pragma unroll 1
        for (int ch = 0; ch < 4; ++ch) {
          uint32_t rr[32];
          tmem_ld32(o_cols + (uint32_t)ch * 32u, rr);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) rr[e] = __float_as_uint(__uint_as_float(rr[e]) * alpha);
          tmem_st32(o_cols + (uint32_t)ch * 32u, rr);
        }
      }
      const float m_sub = m_used == -INFINITY ? 0.f : m_used;  // a row with nothing visible yet: exp2(-inf) = 0
      // pass 2: P = 2^(s - m) as bf16 pairs, written over the first 64 columns of this tile's S
      // (pairs of columns go through paired f32 FMA / add instructions)
      float2 lsum = make_float2(0.f, 0.f), lusum = make_float2(0.f, 0.f);
      const float2 neg_m = make_float2(-m_sub, -m_sub);
      const float2 scale2 = make_float2(a.qk_scale_log2, a.qk_scale_log2);
#pragma unroll 1
      for (int ch = 0; ch < 4; ++ch) {
        uint32_t rr[32];
        tmem_ld32(s_cols + (uint32_t)ch * 32u, rr);
        tmem_wait_ld();
        uint32_t pk[16];
        if (full) {
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const float2 x2 = __ffma2_rn(make_float2(__uint_as_float(rr[2 * e]), __uint_as_float(rr[2 * e + 1])),
                                         scale2, neg_m);
            const float2 p2 = make_float2(ex2(x2.x), ex2(x2.y));
            const __nv_bfloat162 pb = __floats2bfloat162_rn(p2.x, p2.y);
            pk[e] = *reinterpret_cast<const uint32_t*>(&pb);
            lsum = __fadd2_rn(lsum, make_float2(__uint_as_float(pk[e] << 16), __uint_as_float(pk[e] & 0xffff0000u)));
            lusum = __fadd2_rn(lusum, p2);
          }
        } else {
          float xv[32];
          mask_chunk(c, kind, start, i, ch * 32, a.qk_scale_log2, rr, xv);
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const float2 x2 = __fadd2_rn(make_float2(xv[2 * e], xv[2 * e + 1]), neg_m);
            const float2 p2 = make_float2(ex2(x2.x), ex2(x2.y));
            const __nv_bfloat162 pb = __floats2bfloat162_rn(p2.x, p2.y);
            pk[e] = *reinterpret_cast<const uint32_t*>(&pb);
            lsum = __fadd2_rn(lsum, make_float2(__uint_as_float(pk[e] << 16), __uint_as_float(pk[e] & 0xffff0000u)));
            lusum = __fadd2_rn(lusum, p2);
          }
        }
        tmem_st16(s_cols + (uint32_t)ch * 16u, pk);
      }
      l += lsum.x + lsum.y;
      lu += lusum.x + lusum.y;
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&sm.p_full[x]);
      ++j;
    }
    if (ok && j > 0) ok = __all_sync(0xffffffffu, wait_or_abort(sm, &sm.o_done[x], (j - 1) & 1, a.status));
    if (ok && j > 0) {
      tc_fence_after();
      const float inv = l > 0.f ? 1.f / l : 0.f;
      float* orow = a.out + (bh * a.T + i) * kHeadDim;
#pragma unroll 1
      for (int ch = 0; ch < 4; ++ch) {
        uint32_t rr[32];
        tmem_ld32(o_cols + (uint32_t)ch * 32u, rr);
        tmem_wait_ld();
        if (i < c.T) {
#pragma unroll
          for (int e = 0; e < 32; e += 4)
            *reinterpret_cast<float4*>(orow + ch * 32 + e) =
                make_float4(__uint_as_float(rr[e]) * inv, __uint_as_float(rr[e + 1]) * inv,
                            __uint_as_float(rr[e + 2]) * inv, __uint_as_float(rr[e + 3]) * inv);
        }
      }
      if (i < c.T && a.lse) a.lse[bh * a.T + i] = lu > 0.f ? (m_used + log2f(lu)) * kLn2P : -INFINITY;
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    if (sm.abort_flag && lane == 0) mbar_wait(&sm.o_done[0], 0);  // bounded; MMAs drain before TMEM is freed
    __syncwarp();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
  }
}

// ---- writes the chunk's last min(T, n) output K/V rows into the ring ----------
__global__ void ring_from_outputs_kernel(int H, int n, int T, const uint16_t* __restrict__ k_out,
                                         const uint16_t* __restrict__ v_out, uint16_t* __restrict__ ring_k,
                                         uint16_t* __restrict__ ring_v, int32_t* wp, int32_t* fill, int32_t* status) {
  __shared__ int s_wp;
  const int b = blockIdx.x;
  griddep_wait();
  if (threadIdx.x == 0) {
    const int w = wp[b], f = fill[b];
    const bool ok = w >= 0 && w < n && f >= 0 && f <= n;
    if (!ok) set_status(status, RSWA_DEVICE_BAD_RING_STATE);
    s_wp = ok ? w : -1;
  }
  __syncthreads();
  const int w = s_wp;
  if (w < 0) return;
  const int keep = min(T, n);
  constexpr int kVec = kHeadDim / 8;
  const int work = keep * H * kVec * 2;
  for (int idx = threadIdx.x; idx < work; idx += blockDim.x) {
    const int which = idx / (keep * H * kVec);
    const int rem = idx - which * keep * H * kVec;
    const int k = rem / (H * kVec);
    const int hh = (rem / kVec) % H;
    const int e = rem % kVec;
    const int tok = T - keep + k;                           // output position
    const int slot = (int)(((int64_t)w + tok) % n);         // the slot the tok-th append would write
    const int64_t bh = (int64_t)b * H + hh;
    const uint4* src = reinterpret_cast<const uint4*>((which ? v_out : k_out) + (bh * T + tok) * kHeadDim) + e;
    uint4* dst = reinterpret_cast<uint4*>((which ? ring_v : ring_k) + (bh * n + slot) * kHeadDim) + e;
    *dst = *src;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    wp[b] = (int)(((int64_t)w + T) % n);
    const int64_t nf = (int64_t)fill[b] + T;
    fill[b] = (int)(nf < n ? nf : n);
  }
}

}  // namespace

size_t prefill_smem_bytes() { return sizeof(PrefillSmem) + 1024; }

cudaError_t launch_prefill(const PrefillLaunch& L, cudaStream_t stream) {
  CUtensorMap tq, tko, tvo, tpk, tpv, trk, trv;
  const int64_t bh = (int64_t)L.B * L.H;
  cudaError_t e;
  if ((e = make_rows_map(&tq, L.q, bh * L.T)) != cudaSuccess) return e;
  if ((e = make_rows_map(&tko, L.k_out, bh * L.T)) != cudaSuccess) return e;
  if ((e = make_rows_map(&tvo, L.v_out, bh * L.T)) != cudaSuccess) return e;
  const int64_t prows = bh * L.cap > 0 ? bh * L.cap : 1;
  if ((e = make_rows_map(&tpk, L.cap > 0 ? L.pk : L.q, L.cap > 0 ? prows : bh * L.T)) != cudaSuccess) return e;
  if ((e = make_rows_map(&tpv, L.cap > 0 ? L.pv : L.q, L.cap > 0 ? prows : bh * L.T)) != cudaSuccess) return e;
  const bool ring = L.ring_k != nullptr;
  if ((e = make_rows_map(&trk, ring ? L.ring_k : L.q, ring ? bh * L.n : bh * L.T)) != cudaSuccess) return e;
  if ((e = make_rows_map(&trv, ring ? L.ring_v : L.q, ring ? bh * L.n : bh * L.T)) != cudaSuccess) return e;
  PrefillArgs a;
  a.B = L.B;
  a.H = L.H;
  a.n = L.n;
  a.T = L.T;
  a.cap = L.cap;
  a.prefix_len = L.prefix_len;
  a.wp = L.wp;
  a.fill = L.fill;
  a.has_ring = ring ? 1 : 0;
  a.ignore_prefix = L.ignore_prefix;
  a.qk_scale_log2 = L.scale * kLog2eP;
  a.out = L.out;
  a.lse = L.lse;
  a.status = L.status;
  const size_t smem = prefill_smem_bytes();
  static unsigned long long done = 0;
  if ((e = ensure_smem_limit(prefill_kernel, smem, &done)) != cudaSuccess) return e;
  const dim3 grid((L.T + kQTiles * kTileRows - 1) / (kQTiles * kTileRows), L.H, L.B);
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  fill_launch_config(cfg, attr, grid, dim3(kPrefillThreads), smem, stream);
  if ((e = cudaLaunchKernelEx(&cfg, prefill_kernel, a, tq, tko, tvo, tpk, tpv, trk, trv)) != cudaSuccess) return e;
  if (L.write_ring) {
    ring_from_outputs_kernel<<<L.B, 256, 0, stream>>>(L.H, L.n, L.T, static_cast<const uint16_t*>(L.k_out),
                                                      static_cast<const uint16_t*>(L.v_out),
                                                      static_cast<uint16_t*>(L.ring_k_w),
                                                      static_cast<uint16_t*>(L.ring_v_w), L.wp_w, L.fill_w, L.status);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace rswa
