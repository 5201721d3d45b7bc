// route.cu -- SR-SWA router on sm_100a: block index keys, block scores,
// exact 1.5-entmax threshold, top-k and log-probability bias.
//
// Unlimited-OCR-2 SR-SWA explainer, 稀疏路由: the history is cut into 32-token
// blocks (step 1); a low-dimensional index projection scores each block
// against the query (step 2); a 1.5-entmax turns the scores into a sparse
// distribution (step 3); the top-16 blocks are read and each enters the
// attention scores with a log(prob) bias (step 4, 偏置融合).
//
// The entmax is p = max(z/2 - tau, 0)^2 with tau fixed by sum p = 1 (the
// alpha = 1.5 member of alpha-entmax, Peters, Niculae & Martins 2019). It is
// solved exactly, by the sort-based rule, on the device:
//   * only blocks with z/2 > max(z/2) - 1 can have p > 0 (tau >= max - 1,
//     since the largest term alone reaches 1 there), so those are gathered;
//   * the candidates are ranked (descending, ties to the smaller block), and
//     each rank k takes prefix sums S1, S2 of the shifted values y = x - max x
//     in rank order, delta_k = (1 - (S2 - S1^2/k)) / k and
//     tau_k = S1/k - sqrt(delta_k);
//   * the support size is the largest k with delta_k >= 0 and tau_k < y_(k).
// Shifting by max x keeps the fp32 sums small (shift invariance of entmax).
//
// Top-k and candidates come from one set: the CTAs of a sequence's cluster
// exchange their maxima, then each sends CTA 0 its candidates (z > max z - 2
// over the sequence). When the sequence has at least k candidates they hold
// its k largest scores; otherwise every CTA also sends the rest of its sorted
// top-32 (warp bitonic networks and a merge tree), which holds its top-k.
// CTA 0 ranks the union by counting (a bitonic network past 1024 entries),
// reads the top-k off the front and takes the prefix sums with a block scan.
#include <cooperative_groups.h>

#include <cmath>

#include "common.cuh"
#include "internal.h"

namespace rswa {

namespace {

constexpr int kPoolWarps = 8;
constexpr int kRouteThreads = 512;
constexpr int kRouteWarps = kRouteThreads / 32;

// Index keys: one warp per 32-token block; lane (tg, dq) sums tokens tg, tg+8, ...
// over dims 8dq..8dq+7, then the eight token groups are folded with shuffles.
__global__ void __launch_bounds__(kPoolWarps * 32) index_pool_kernel(int64_t cap, int nb_cap,
                                                                     const uint16_t* __restrict__ k_idx,
                                                                     const int32_t* __restrict__ prefix_len,
                                                                     float* __restrict__ kbar) {
  const int b = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  griddep_wait();
  const int c = blockIdx.x * kPoolWarps + warp;
  if (c >= nb_cap) return;
  int64_t m = prefix_len[b];
  m = m < 0 ? 0 : (m > cap ? cap : m);
  const int64_t t0 = (int64_t)c * kBlock;
  const int cnt = (int)(m - t0 < kBlock ? (m - t0 > 0 ? m - t0 : 0) : kBlock);
  const int tg = lane >> 2, dq = lane & 3;
  float s[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) s[e] = 0.f;
  for (int t = tg; t < cnt; t += 8) {
    const uint4 w = *reinterpret_cast<const uint4*>(k_idx + ((int64_t)b * cap + t0 + t) * kIndexDim + dq * 8);
    s[0] += bf16lo(w.x);
    s[1] += bf16hi(w.x);
    s[2] += bf16lo(w.y);
    s[3] += bf16hi(w.y);
    s[4] += bf16lo(w.z);
    s[5] += bf16hi(w.z);
    s[6] += bf16lo(w.w);
    s[7] += bf16hi(w.w);
  }
#pragma unroll
  for (int off = 4; off < 32; off <<= 1)
#pragma unroll
    for (int e = 0; e < 8; ++e) s[e] += __shfl_xor_sync(0xffffffffu, s[e], off);
  if (tg == 0) {
    float r[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) r[e] = cnt > 0 ? s[e] / (float)cnt : 0.f;
    float4* dst = reinterpret_cast<float4*>(kbar + ((int64_t)b * nb_cap + c) * kIndexDim + dq * 8);
    dst[0] = make_float4(r[0], r[1], r[2], r[3]);
    dst[1] = make_float4(r[4], r[5], r[6], r[7]);
  }
}

// Strict total order of the top-k: larger score first, then smaller block.
__device__ __forceinline__ bool ranks_before(float za, int ia, float zb, int ib) {
  return za > zb || (za == zb && ia < ib);
}

constexpr int kNone = 0x7fffffff;
constexpr int kRankByCounting = 1024;  // larger unions are sorted with a bitonic network instead
constexpr int kMaxClusterCtas = 8;  // portable cluster size: up to 8 x 1024 = 8192 blocks
constexpr int kList = 32;  // sorted candidates kept per warp / per chunk (>= the largest topk)

// Compare-exchange with the lane `j` apart: the lane whose bit j equals `keep_better_bit`
// keeps the better of the pair, its partner the worse.
__device__ __forceinline__ void cmp_xchg(float& z, int& i, int j, bool keep_better) {
  const float oz = __shfl_xor_sync(0xffffffffu, z, j);
  const int oi = __shfl_xor_sync(0xffffffffu, i, j);
  const bool other_better = ranks_before(oz, oi, z, i);
  if (other_better == keep_better) {
    z = oz;
    i = oi;
  }
}

// Bitonic sort of one (z, i) pair per lane; afterwards lane 0 holds the best.
__device__ __forceinline__ void warp_sort(float& z, int& i, int lane) {
#pragma unroll
  for (int k = 2; k <= 32; k <<= 1)
#pragma unroll
    for (int j = k >> 1; j > 0; j >>= 1) cmp_xchg(z, i, j, ((lane & j) == 0) == ((lane & k) == 0));
}

// Top 32 of two sorted lists: lane l holds A[l] and B[31 - l] (a bitonic pair); keep the
// better, then merge the resulting bitonic sequence across the warp.
__device__ __forceinline__ void warp_merge(float& z, int& i, float bz, int bi, int lane) {
  if (ranks_before(bz, bi, z, i)) {
    z = bz;
    i = bi;
  }
#pragma unroll
  for (int j = 16; j > 0; j >>= 1) cmp_xchg(z, i, j, (lane & j) == 0);
}

// Slots of the compacted union on CTA 0: the next power of two of csize * 1024.
__host__ __device__ __forceinline__ int route_sort_capacity(int csize) {
  int p = kRouteThreads * 2;
  while (p < csize * kRouteThreads * 2) p <<= 1;
  return p;
}

struct RouteArgs {
  int64_t cap;
  int tokens;  // router queries per sequence: 1 (decode) or the chunk length (per-token prefill routing)
  int nb_cap, csize, topk;  // csize: CTAs per sequence (the cluster size)
  float idx_scale;
  const float* q_idx;
  const float* kbar;
  const int32_t* prefix_len;
  int32_t* blk_idx;
  float* blk_logp;
  float* probs;
  float* tau;
  int32_t* status;
};

// Merges `n` sorted lists of kList held in (lz, li) shared arrays into lists[0]; every
// warp of the CTA must call it (it synchronises the CTA).
__device__ void merge_lists(float (*lz)[kList], int (*li)[kList], int n, int warp, int lane) {
  for (int width = 1; width < n; width <<= 1) {
    const int pairs = (n + 2 * width - 1) / (2 * width);
    if (warp < pairs) {
      const int a = 2 * width * warp, bidx = a + width;
      float z = lz[a][lane];
      int i = li[a][lane];
      float bz = -INFINITY;
      int bi = kNone;
      if (bidx < n) {
        bz = lz[bidx][kList - 1 - lane];
        bi = li[bidx][kList - 1 - lane];
      }
      __syncwarp();
      warp_merge(z, i, bz, bi, lane);
      lz[a][lane] = z;
      li[a][lane] = i;
    }
    __syncthreads();
  }
}

// One thread-block cluster per sequence (grid = csize x B, cluster = csize x 1).
// CTA r scores blocks [1024 r, 1024 r + 1024) (two per thread), keeps their sorted
// top-32 and the candidates z > (its own max) - 2, and stores list, maximum and
// candidates into CTA 0's shared memory over DSMEM (the global candidates
// z > max z - 2 are among them: every CTA's max is at most the global one).
// After one cluster barrier CTA 0 merges the lists and solves the threshold.
// With probs requested, CTA 0 sends tau back and every CTA writes its blocks' p.
__global__ void __launch_bounds__(kRouteThreads) route_kernel(const RouteArgs a) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  __shared__ float lz[kRouteWarps][kList];
  __shared__ int li[kRouteWarps][kList];
  __shared__ float cl_max[kMaxClusterCtas];  // every CTA's maximum (on every CTA)
  __shared__ int cl_cnt[kMaxClusterCtas];    // every CTA's candidate count (on every CTA)
  __shared__ int cl_send[kMaxClusterCtas];   // on CTA 0: entries each CTA sent, lists included
  __shared__ float red[kRouteWarps];
  __shared__ float scan2[kRouteWarps];
  __shared__ int red_i[kRouteWarps];
  __shared__ int s_cnt;
  __shared__ float s_tau_y, s_xmax;
  namespace cg = cooperative_groups;
  cg::cluster_group cluster = cg::this_cluster();

  // blockIdx.y is the router query: (sequence b, token t) with t < a.tokens (1 for decode)
  const int rank = (int)cluster.block_rank(), row = blockIdx.y, b = row / a.tokens;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int region = kRouteThreads * 2;  // blocks per CTA
  // on CTA 0: what CTA r sends lands at [r * region, ...) of (cand_z, cand_i); the union
  // is compacted into (uz, ui), whose size is a power of two for the bitonic sort
  float* cand_z = reinterpret_cast<float*>(smem_raw);
  int* cand_i = reinterpret_cast<int*>(cand_z + a.csize * region);
  float* uz = reinterpret_cast<float*>(cand_i + a.csize * region);
  int* ui = reinterpret_cast<int*>(uz + route_sort_capacity(a.csize));

  griddep_wait();
  griddep_launch_dependents();
  if (tid == 0) s_cnt = 1;
  int64_t m64 = a.prefix_len[b];
  // ---- score: warp w covers blocks [64 w, 64 w + 64) of the CTA's region ----
  // The keys are read coalesced, four blocks (512 B) per warp load: octet o = lane / 8
  // reads block 4i + o of the warp's range, lane j = lane % 8 its dims 4j..4j+3. The
  // 16 partial dots of a lane are then reduce-scattered over the octet (xor 4, 2, 1),
  // leaving lane j with the full dots of groups 2j and 2j + 1, i.e. of blocks
  // 8j + o and 8j + 4 + o. The loads depend only on the capacity, so they are in
  // flight while prefix_len is still being read.
  float dot[2];
  int cpos[2];
  {
    const int o = lane >> 3, j = lane & 7;
    const int wbase = rank * region + warp * 64;
    const float4 qv = reinterpret_cast<const float4*>(a.q_idx + (int64_t)row * kIndexDim)[j];
    const float4* k4 = reinterpret_cast<const float4*>(a.kbar + (int64_t)b * a.nb_cap * kIndexDim);
    float4 kv[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const int c = wbase + 4 * i + o;
      kv[i] = c < a.nb_cap ? k4[(int64_t)c * 8 + j] : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    asm volatile("" ::: "memory");  // all 16 loads are issued before the first use
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
#pragma unroll
    for (int s2 = 0; s2 < 2; ++s2) {
      cpos[s2] = wbase + 4 * (2 * j + s2) + o;
      dot[s2] = v[s2];
    }
  }
  if (m64 < 0 || m64 > a.cap) {
    if (tid == 0 && rank == 0) set_status(a.status, RSWA_DEVICE_BAD_PREFIX_LEN);
    m64 = 0;
  }
  const int NB = (int)((m64 + kBlock - 1) / kBlock);
  if (NB == 0) {  // uniform over the cluster: no barrier is reached
    if (rank == 0) {
      if (tid < a.topk) {
        a.blk_idx[(int64_t)row * a.topk + tid] = -1;
        a.blk_logp[(int64_t)row * a.topk + tid] = -INFINITY;
      }
      if (a.probs)
        for (int c = tid; c < a.nb_cap; c += kRouteThreads) a.probs[(int64_t)row * a.nb_cap + c] = 0.f;
      if (a.tau && tid == 0) a.tau[row] = NAN;
    }
    return;
  }

  float z[2];
  int cidx[2];
#pragma unroll
  for (int s2 = 0; s2 < 2; ++s2) {
    cidx[s2] = cpos[s2] < NB ? cpos[s2] : kNone;
    z[s2] = cpos[s2] < NB ? a.idx_scale * dot[s2] : -INFINITY;
  }
  // ---- the sequence's maximum: every CTA of the cluster receives every CTA's ----
  const float wmax = warp_max(fmaxf(z[0], z[1]));
  if (lane == 0) red[warp] = wmax;
  __syncthreads();
  float zmax = red[0];
#pragma unroll
  for (int w = 1; w < kRouteWarps; ++w) zmax = fmaxf(zmax, red[w]);
  if (a.csize > 1) {  // uniform over the cluster
    if (tid < a.csize) cluster.map_shared_rank(cl_max, tid)[rank] = zmax;
    cluster.sync();
    for (int r = 0; r < a.csize; ++r) zmax = fmaxf(zmax, cl_max[r]);
  }
  // ---- this CTA's candidates z > zmax - 2 go to CTA 0; every CTA learns every count ----
  const bool cand0 = cidx[0] != kNone && z[0] > zmax - 2.f;
  const bool cand1 = cidx[1] != kNone && z[1] > zmax - 2.f;
  const unsigned bal0 = __ballot_sync(0xffffffffu, cand0), bal1 = __ballot_sync(0xffffffffu, cand1);
  if (lane == 0) red_i[warp] = __popc(bal0) + __popc(bal1);
  __syncthreads();
  int n_cand = 0, before = 0;
#pragma unroll
  for (int w = 0; w < kRouteWarps; ++w) {
    before += w < warp ? red_i[w] : 0;
    n_cand += red_i[w];
  }
  float* r_cand_z = cluster.map_shared_rank(cand_z, 0) + rank * region;
  int* r_cand_i = cluster.map_shared_rank(cand_i, 0) + rank * region;
  {
    const unsigned lt = (1u << lane) - 1u;
    if (cand0) {
      const int k = before + __popc(bal0 & lt);
      r_cand_z[k] = z[0];
      r_cand_i[k] = cidx[0];
    }
    if (cand1) {
      const int k = before + __popc(bal0) + __popc(bal1 & lt);
      r_cand_z[k] = z[1];
      r_cand_i[k] = cidx[1];
    }
  }
  if (tid < a.csize) cluster.map_shared_rank(cl_cnt, tid)[rank] = n_cand;
  if (a.csize > 1)
    cluster.sync();
  else
    __syncthreads();
  int total = 0;
  for (int r = 0; r < a.csize; ++r) total += cl_cnt[r];
  // ---- fewer than topk candidates in all: each CTA adds the rest of its sorted top-32 ----
  // (the global top-k is within the CTAs' top-k; a CTA's candidates are its first n_cand)
  const bool with_lists = total < a.topk;  // uniform over the cluster
  if (with_lists) {
    float za = z[0], zb = z[1];
    int ia = cidx[0], ib = cidx[1];
    warp_sort(za, ia, lane);
    warp_sort(zb, ib, lane);
    {  // merge the two sorted columns: lane l pairs A[l] with B[31 - l]
      const float rz = __shfl_sync(0xffffffffu, zb, 31 - lane);
      const int ri = __shfl_sync(0xffffffffu, ib, 31 - lane);
      warp_merge(za, ia, rz, ri, lane);
    }
    lz[warp][lane] = za;
    li[warp][lane] = ia;
    __syncthreads();
    merge_lists(lz, li, kRouteWarps, warp, lane);
    // the valid entries are a prefix of the sorted list (missing blocks carry kNone, -inf)
    const int n_valid = __popc(__ballot_sync(0xffffffffu, li[0][lane] != kNone));
    if (warp == 0 && lane >= n_cand && lane < n_valid) {
      r_cand_z[lane] = lz[0][lane];
      r_cand_i[lane] = li[0][lane];
    }
    if (tid == 0) cluster.map_shared_rank(cl_send, 0)[rank] = max(n_valid, n_cand);
    if (a.csize > 1)
      cluster.sync();
    else
      __syncthreads();
  }

  if (rank != 0) {
    if (a.probs == nullptr) return;
    cluster.sync();  // CTA 0 sends tau
    for (int s2 = 0; s2 < 2; ++s2) {
      const int c = cpos[s2];
      if (c < a.nb_cap) {
        float pr = 0.f;
        if (c < NB) {
          const float r = fmaf(z[s2], 0.5f, -s_xmax) - s_tau_y;
          pr = r > 0.f ? r * r : 0.f;
        }
        a.probs[(int64_t)row * a.nb_cap + c] = pr;
      }
    }
    return;
  }

  // ---- CTA 0: the union U of what the CTAs sent, in rank order ----
  int n_u = 0;
  for (int r = 0; r < a.csize; ++r) n_u += with_lists ? cl_send[r] : cl_cnt[r];
  const float xmax = 0.5f * zmax;
  {  // compact U into (uz, ui)
    int off = 0;
    for (int r = 0; r < a.csize; ++r) {
      const int cnt = with_lists ? cl_send[r] : cl_cnt[r];
      for (int k = tid; k < cnt; k += kRouteThreads) {
        uz[off + k] = cand_z[r * region + k];
        ui[off + k] = cand_i[r * region + k];
      }
      off += cnt;
    }
  }
  __syncthreads();
  const float* oz;  // U sorted: larger score first, ties to the smaller block
  const int* oi;
  if (n_u <= kRankByCounting) {
    for (int i = tid; i < n_u; i += kRouteThreads) {
      const float zi = uz[i];
      const int ii = ui[i];
      int r = 0;
      for (int j = 0; j < n_u; ++j) r += ranks_before(uz[j], ui[j], zi, ii) ? 1 : 0;
      cand_z[r] = zi;
      cand_i[r] = ii;
    }
    oz = cand_z;
    oi = cand_i;
  } else {  // bitonic sort of U in place, padded to a power of two
    int np2 = 1;
    while (np2 < n_u) np2 <<= 1;
    for (int i = n_u + tid; i < np2; i += kRouteThreads) {
      uz[i] = -INFINITY;
      ui[i] = kNone;
    }
    for (int k = 2; k <= np2; k <<= 1)
      for (int j = k >> 1; j > 0; j >>= 1) {
        __syncthreads();
        for (int i = tid; i < np2; i += kRouteThreads) {
          const int p = i ^ j;
          if (p > i) {
            const bool first_better = ranks_before(uz[i], ui[i], uz[p], ui[p]);
            // ascending blocks of the network put the better element first
            if (first_better != ((i & k) == 0)) {
              const float tz = uz[i];
              uz[i] = uz[p];
              uz[p] = tz;
              const int ti = ui[i];
              ui[i] = ui[p];
              ui[p] = ti;
            }
          }
        }
      }
    oz = uz;
    oi = ui;
  }
  __syncthreads();

  // ---- exact threshold over the candidates y = z/2 - max(z/2) > -1, a prefix of U ----
  for (int r = tid; r < n_u; r += kRouteThreads) {
    const bool in = fmaf(oz[r], 0.5f, -xmax) > -1.f;
    const bool next_in = r + 1 < n_u && fmaf(oz[r + 1], 0.5f, -xmax) > -1.f;
    if (in && !next_in) s_cnt = r + 1;
  }
  __syncthreads();
  const int K = s_cnt;  // >= 1: the maximum itself has y = 0
  // prefix sums of y and y^2 in rank order: thread t takes a contiguous run of ranks
  const int per = (K + kRouteThreads - 1) / kRouteThreads;
  const int r0 = min(K, tid * per), r1 = min(K, r0 + per);
  float s1 = 0.f, s2 = 0.f;
  for (int r = r0; r < r1; ++r) {
    const float y = fmaf(oz[r], 0.5f, -xmax);
    s1 += y;
    s2 = fmaf(y, y, s2);
  }
  float i1 = s1, i2 = s2;  // inclusive scan over the warp
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const float t1 = __shfl_up_sync(0xffffffffu, i1, o), t2 = __shfl_up_sync(0xffffffffu, i2, o);
    if (lane >= o) {
      i1 += t1;
      i2 += t2;
    }
  }
  if (lane == 31) {
    red[warp] = i1;
    scan2[warp] = i2;
  }
  __syncthreads();
  float e1 = i1 - s1, e2 = i2 - s2;  // exclusive prefix of this thread's run
  for (int w = 0; w < warp; ++w) {
    e1 += red[w];
    e2 += scan2[w];
  }
  float* tau_r = uz == oz ? reinterpret_cast<float*>(cand_z) : uz;  // tau_k by rank k - 1
  int best = 0;
  for (int r = r0; r < r1; ++r) {
    const float y = fmaf(oz[r], 0.5f, -xmax);
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
  if (lane == 0) red_i[warp] = best;
  __syncthreads();
#pragma unroll
  for (int w = 0; w < kRouteWarps; ++w) best = max(best, red_i[w]);
  const float tau_y = best > 0 ? tau_r[best - 1] : 0.f;
  if (a.tau && tid == 0) a.tau[row] = tau_y + xmax;
  if (tid < a.topk) {
    const int64_t o = (int64_t)row * a.topk + tid;
    const int bi = tid < n_u ? oi[tid] : kNone;
    if (bi == kNone) {
      a.blk_idx[o] = -1;
      a.blk_logp[o] = -INFINITY;
    } else {
      const float d = fmaf(oz[tid], 0.5f, -xmax) - tau_y;
      const float pr = d > 0.f ? d * d : 0.f;
      a.blk_idx[o] = bi;
      a.blk_logp[o] = pr > 0.f ? logf(pr) : -INFINITY;
    }
  }
  if (a.probs != nullptr) {
    if (tid < a.csize) {
      cluster.map_shared_rank(&s_tau_y, tid)[0] = tau_y;
      cluster.map_shared_rank(&s_xmax, tid)[0] = xmax;
    }
    if (a.csize > 1)
      cluster.sync();
    else
      __syncthreads();
    for (int s2i = 0; s2i < 2; ++s2i) {
      const int c = cpos[s2i];
      if (c < a.nb_cap) {
        float pr = 0.f;
        if (c < NB) {
          const float r = fmaf(z[s2i], 0.5f, -xmax) - tau_y;
          pr = r > 0.f ? r * r : 0.f;
        }
        a.probs[(int64_t)row * a.nb_cap + c] = pr;
      }
    }
  }
}

// ---------------------------------------------------------------------------------------
// Per-token router of the chunked prefill (T router queries per sequence, at most 1024
// blocks): the same result as route_kernel row by row (the same z arithmetic; the same
// sort-based threshold whenever at most 32 blocks are candidates), organised for many rows
// that share one sequence's block keys. A CTA takes one sequence and a run of its tokens:
// it stages the sequence's keys in shared memory once (bulk copies on an mbarrier), and each
// warp routes two tokens at a time from there: both rows' scores come from the same key
// loads (the octet layout of route_kernel), go to the warp's two score rows in shared
// memory, and each row is then finished by the warp alone, without block barriers:
//   * max z and the candidate count (z > max z - 2) by warp reductions;
//   * at most 32 candidates (the usual case): compacted by ballots, sorted by one warp
//     bitonic network (larger score first, ties to the smaller block), the threshold by the
//     sort-based rule over a warp scan; the top-k is the front of that list, completed, when
//     fewer than k blocks are candidates, by argmax rounds over the rest of the row;
//   * more than 32 candidates: the root of sum (y - tau)_+^2 = 1 (y = z/2 - max z/2) is
//     bracketed by bisection on [-1, 0], the support is {y > the bracket's low end}, and tau
//     is the closed form over that support (the value the sort-based rule reaches); the top-k
//     comes from argmax rounds.
// ---------------------------------------------------------------------------------------
constexpr int kTokWarps = 12;
constexpr int kTokThreads = kTokWarps * 32;
constexpr int kTokMaxBlocks = 1024;       // 32 scores per lane per row
constexpr uint32_t kTokCopyBytes = 32768;  // bulk copies of the keys in pieces of this size

__host__ __device__ __forceinline__ int tok_padded_blocks(int nb_cap) { return (nb_cap + 63) / 64 * 64; }

__host__ __device__ __forceinline__ size_t tok_smem_bytes(int nb_cap) {
  const size_t nbr = (size_t)tok_padded_blocks(nb_cap);
  return nbr * kIndexDim * 4 + (size_t)kTokWarps * 2 * nbr * 4 + 16;
}

// Finishes one router row from its scores zs[0, NB) in shared memory (warp-collective; the
// row's buffer is reused as scratch).
__device__ void tok_finish_row(const RouteArgs& a, float* zs, int NB, int64_t row, int lane) {
  float zr[32];
#pragma unroll
  for (int t = 0; t < 32; ++t) {
    const int c = lane + 32 * t;
    zr[t] = c < NB ? zs[c] : -INFINITY;
  }
  float mx = zr[0];
#pragma unroll
  for (int t = 1; t < 32; ++t) mx = fmaxf(mx, zr[t]);
  const float zmax = warp_max(mx);
  const float cut = zmax - 2.f;  // candidates: z / 2 > max z / 2 - 1
  int cnt = 0;
#pragma unroll
  for (int t = 0; t < 32; ++t) cnt += zr[t] > cut ? 1 : 0;
  const int C = (int)__reduce_add_sync(0xffffffffu, (unsigned)cnt);  // >= 1: the maximum
  const float xmax = 0.5f * zmax;
  __syncwarp();  // the row is in registers: its buffer now holds the candidate list
  float* lz = zs;
  int* li = reinterpret_cast<int*>(zs + 32);
  float sz = -INFINITY;  // lane r: the r-th entry of the top list (best first)
  int si = kNone;
  int have = 0;          // entries of the top list already in place
  float tau_y;
  if (C <= 32) {
    int base = 0;
    const unsigned lt = (1u << lane) - 1u;
#pragma unroll
    for (int t = 0; t < 32; ++t) {
      const bool in = zr[t] > cut;
      const unsigned bal = __ballot_sync(0xffffffffu, in);
      if (in) {
        const int k = base + __popc(bal & lt);
        lz[k] = zr[t];
        li[k] = lane + 32 * t;
      }
      base += __popc(bal);
    }
    __syncwarp();
    if (lane < C) {
      sz = lz[lane];
      si = li[lane];
    }
    warp_sort(sz, si, lane);
    // sort-based rule: prefix sums of y and y^2 in rank order, tau_k per rank, support size =
    // the largest k with delta_k >= 0 and tau_k < y_(k)
    const float y = lane < C ? fmaf(sz, 0.5f, -xmax) : 0.f;
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
    const float tk = mean - sqrtf(fmaxf(delta, 0.f));
    const unsigned ok = __ballot_sync(0xffffffffu, lane < C && delta >= 0.f && tk < y);
    const int best = ok ? 32 - __clz(ok) : 0;
    const float tb = __shfl_sync(0xffffffffu, tk, best > 0 ? best - 1 : 0);
    tau_y = best > 0 ? tb : 0.f;
    have = C;
  } else {
    // f(tau) = sum (y - tau)_+^2 falls from f(-1) >= 1 (the maximum has y = 0) to f(0) = 0
    float lo = -1.f, hi = 0.f;
#pragma unroll 1
    for (int it = 0; it < 30; ++it) {
      const float mid = 0.5f * (lo + hi);
      float f = 0.f;
#pragma unroll
      for (int t = 0; t < 32; ++t) {
        const float d = fmaf(zr[t], 0.5f, -xmax) - mid;
        f = d > 0.f ? fmaf(d, d, f) : f;
      }
      if (warp_sum(f) >= 1.f)
        lo = mid;
      else
        hi = mid;
    }
    float n = 0.f, s1 = 0.f, s2 = 0.f;
#pragma unroll
    for (int t = 0; t < 32; ++t) {
      const float y = fmaf(zr[t], 0.5f, -xmax);
      if (y > lo) {
        n += 1.f;
        s1 += y;
        s2 = fmaf(y, y, s2);
      }
    }
    n = warp_sum(n);
    s1 = warp_sum(s1);
    s2 = warp_sum(s2);
    const float mean = s1 / n;
    const float delta = (1.f - (s2 - s1 * mean)) / n;
    tau_y = mean - sqrtf(fmaxf(delta, 0.f));
  }
  if (have < a.topk) {
    // argmax rounds: each takes the best entry ranking after the previous round's
    float pz = have > 0 ? __shfl_sync(0xffffffffu, sz, have - 1) : INFINITY;
    int pi = have > 0 ? __shfl_sync(0xffffffffu, si, have - 1) : -1;
#pragma unroll 1
    for (int r = have; r < a.topk; ++r) {
      float bz = -INFINITY;
      int bi = kNone;
#pragma unroll
      for (int t = 0; t < 32; ++t) {
        const float z = zr[t];
        const int i = lane + 32 * t;
        const bool after = z < pz || (z == pz && i > pi);
        if (after && i < NB && ranks_before(z, i, bz, bi)) {
          bz = z;
          bi = i;
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const float oz = __shfl_xor_sync(0xffffffffu, bz, o);
        const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
        if (ranks_before(oz, oi, bz, bi)) {
          bz = oz;
          bi = oi;
        }
      }
      if (lane == r) {
        sz = bz;
        si = bi;
      }
      pz = bz;
      pi = bi;
    }
  }
  if (lane < a.topk) {
    const int64_t o = row * a.topk + lane;
    if (si == kNone) {
      a.blk_idx[o] = -1;
      a.blk_logp[o] = -INFINITY;
    } else {
      const float d = fmaf(sz, 0.5f, -xmax) - tau_y;
      const float pr = d > 0.f ? d * d : 0.f;
      a.blk_idx[o] = si;
      a.blk_logp[o] = pr > 0.f ? logf(pr) : -INFINITY;
    }
  }
  __syncwarp();  // the buffer is rewritten by the warp's next rows
}

__global__ void __launch_bounds__(kTokThreads, 1) route_tokens_kernel(const RouteArgs a, int rows_per_cta) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  const int nbr = tok_padded_blocks(a.nb_cap);
  float* kb = reinterpret_cast<float*>(smem_raw);                                    // [nbr][32] keys
  float* zb = kb + (size_t)nbr * kIndexDim;                                          // [warps][2][nbr]
  uint64_t* bar = reinterpret_cast<uint64_t*>(zb + (size_t)kTokWarps * 2 * nbr);
  const int b = blockIdx.y;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int t_begin = blockIdx.x * rows_per_cta;
  const int t_end = min(a.tokens, t_begin + rows_per_cta);
  if (tid == 0) {
    mbar_init(bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  griddep_wait();
  griddep_launch_dependents();
  int64_t m64 = a.prefix_len[b];
  if (m64 < 0 || m64 > a.cap) {
    if (tid == 0 && blockIdx.x == 0) set_status(a.status, RSWA_DEVICE_BAD_PREFIX_LEN);
    m64 = 0;
  }
  const int NB = (int)((m64 + kBlock - 1) / kBlock);
  bool staged = true;
  if (NB > 0) {
    if (tid == 0) {
      const uint32_t bytes = (uint32_t)NB * kIndexDim * 4;
      mbar_arrive_expect_tx(bar, bytes);
      const uint8_t* src = reinterpret_cast<const uint8_t*>(a.kbar + (int64_t)b * a.nb_cap * kIndexDim);
      for (uint32_t off = 0; off < bytes; off += kTokCopyBytes)
        bulk_copy_g2s(reinterpret_cast<uint8_t*>(kb) + off, src + off, min(kTokCopyBytes, bytes - off), bar);
    }
    staged = mbar_wait(bar, 0);
  }
  if (!__syncthreads_and(staged)) {  // the whole CTA gives up together
    if (tid == 0) set_status(a.status, RSWA_DEVICE_WAIT_TIMEOUT);
    if (!staged) (void)mbar_wait(bar, 0);  // the copies in flight land before the CTA leaves
    return;
  }
  const int o = lane >> 3, j = lane & 7;
  float* zw = zb + (size_t)warp * 2 * nbr;
  const int n_pairs = (max(0, t_end - t_begin) + 1) / 2;
  for (int p = warp; p < n_pairs; p += kTokWarps) {
    const int r0 = t_begin + 2 * p;
    const bool two = r0 + 1 < t_end;
    const int64_t row0 = (int64_t)b * a.tokens + r0;
    if (NB == 0) {
      if (lane < a.topk) {
        a.blk_idx[row0 * a.topk + lane] = -1;
        a.blk_logp[row0 * a.topk + lane] = -INFINITY;
        if (two) {
          a.blk_idx[(row0 + 1) * a.topk + lane] = -1;
          a.blk_logp[(row0 + 1) * a.topk + lane] = -INFINITY;
        }
      }
      continue;
    }
    const float4 qa = reinterpret_cast<const float4*>(a.q_idx + row0 * kIndexDim)[j];
    const float4 qb = two ? reinterpret_cast<const float4*>(a.q_idx + (row0 + 1) * kIndexDim)[j] : qa;
    for (int base = 0; base < NB; base += 64) {
      // octet o reads block base + 4i + o, lane j its dims 4j..4j+3 (512 contiguous bytes per
      // warp load); both rows' 16 partial dots are reduce-scattered over the octet, leaving
      // lane j the dots of blocks base + 8j + o and base + 8j + 4 + o, as in route_kernel
      float4 kv[16];
#pragma unroll
      for (int i = 0; i < 16; ++i)
        kv[i] = reinterpret_cast<const float4*>(kb)[(size_t)(base + 4 * i + o) * 8 + j];
      float va[16], vb[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        float d = qa.x * kv[i].x;
        d = fmaf(qa.y, kv[i].y, d);
        d = fmaf(qa.z, kv[i].z, d);
        va[i] = fmaf(qa.w, kv[i].w, d);
        float e = qb.x * kv[i].x;
        e = fmaf(qb.y, kv[i].y, e);
        e = fmaf(qb.z, kv[i].z, e);
        vb[i] = fmaf(qb.w, kv[i].w, e);
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const bool up = j & 4;
        va[i] = (up ? va[i + 8] : va[i]) + __shfl_xor_sync(0xffffffffu, up ? va[i] : va[i + 8], 4);
        vb[i] = (up ? vb[i + 8] : vb[i]) + __shfl_xor_sync(0xffffffffu, up ? vb[i] : vb[i + 8], 4);
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const bool up = j & 2;
        va[i] = (up ? va[i + 4] : va[i]) + __shfl_xor_sync(0xffffffffu, up ? va[i] : va[i + 4], 2);
        vb[i] = (up ? vb[i + 4] : vb[i]) + __shfl_xor_sync(0xffffffffu, up ? vb[i] : vb[i + 4], 2);
      }
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const bool up = j & 1;
        va[i] = (up ? va[i + 2] : va[i]) + __shfl_xor_sync(0xffffffffu, up ? va[i] : va[i + 2], 1);
        vb[i] = (up ? vb[i + 2] : vb[i]) + __shfl_xor_sync(0xffffffffu, up ? vb[i] : vb[i + 2], 1);
      }
#pragma unroll
      for (int s2 = 0; s2 < 2; ++s2) {
        const int c = base + 8 * j + 4 * s2 + o;
        zw[c] = c < NB ? a.idx_scale * va[s2] : -INFINITY;
        zw[nbr + c] = c < NB ? a.idx_scale * vb[s2] : -INFINITY;
      }
    }
    __syncwarp();
    tok_finish_row(a, zw, NB, row0, lane);
    if (two) tok_finish_row(a, zw + nbr, NB, row0 + 1, lane);
  }
}

}  // namespace

cudaError_t launch_index_pool(int B, int64_t cap, const uint16_t* k_idx, const int32_t* prefix_len, float* kbar,
                              cudaStream_t stream) {
  const int nb_cap = (int)((cap + kBlock - 1) / kBlock);
  const dim3 grid((nb_cap + kPoolWarps - 1) / kPoolWarps, B);
  index_pool_kernel<<<grid, kPoolWarps * 32, 0, stream>>>(cap, nb_cap, k_idx, prefix_len, kbar);
  return cudaGetLastError();
}

int route_cluster_size(int64_t cap) {
  const int nb_cap = (int)((cap + kBlock - 1) / kBlock);
  const int per = kRouteThreads * 2;
  return (nb_cap + per - 1) / per;
}

cudaError_t launch_route(int B, int tokens, int64_t cap, const float* q_idx, const float* kbar,
                         const int32_t* prefix_len, float idx_scale, int topk, int32_t* blk_idx, float* blk_logp,
                         float* probs, float* tau, int32_t* status, cudaStream_t stream) {
  RouteArgs a;
  a.cap = cap;
  a.tokens = tokens;
  a.nb_cap = (int)((cap + kBlock - 1) / kBlock);
  a.csize = route_cluster_size(cap);
  a.topk = topk;
  a.idx_scale = idx_scale;
  a.q_idx = q_idx;
  a.kbar = kbar;
  a.prefix_len = prefix_len;
  a.blk_idx = blk_idx;
  a.blk_logp = blk_logp;
  a.probs = probs;
  a.tau = tau;
  a.status = status;
  if (tokens > 1 && a.nb_cap <= kTokMaxBlocks && probs == nullptr && tau == nullptr) {
    // many router queries per sequence: the per-token kernel; CTAs per sequence so that the
    // grid fills the SMs, each with a run of the sequence's tokens
    const size_t smem = tok_smem_bytes(a.nb_cap);
    static unsigned long long tok_done = 0;
    cudaError_t e = ensure_smem_limit(route_tokens_kernel, tok_smem_bytes(kTokMaxBlocks), &tok_done);
    if (e != cudaSuccess) return e;
    const int slots = device_sm_count();  // one CTA per SM (its registers alone fill most of one)
    const int by_rows = (tokens + 2 * kTokWarps - 1) / (2 * kTokWarps);  // a full pass of every warp at least
    const int by_sms = (slots + B - 1) / B;
    int gx = by_rows < by_sms ? by_rows : by_sms;
    if (gx < 1) gx = 1;
    const int rows_per_cta = (tokens + gx - 1) / gx;
    gx = (tokens + rows_per_cta - 1) / rows_per_cta;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    fill_launch_config(cfg, attr, dim3(gx, B), dim3(kTokThreads), smem, stream);
    return cudaLaunchKernelEx(&cfg, route_tokens_kernel, a, rows_per_cta);
  }
  const size_t smem = (size_t)a.csize * kRouteThreads * 2 * 8 + (size_t)route_sort_capacity(a.csize) * 8;
  static unsigned long long done = 0;
  cudaError_t e = ensure_smem_limit(
      route_kernel, (size_t)kMaxClusterCtas * kRouteThreads * 2 * 8 + (size_t)route_sort_capacity(kMaxClusterCtas) * 8,
      &done);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  fill_launch_config(cfg, attr, dim3(a.csize, B * tokens), dim3(kRouteThreads), smem, stream);
  attr[cfg.numAttrs].id = cudaLaunchAttributeClusterDimension;
  attr[cfg.numAttrs].val.clusterDim.x = a.csize;
  attr[cfg.numAttrs].val.clusterDim.y = 1;
  attr[cfg.numAttrs].val.clusterDim.z = 1;
  cfg.numAttrs += 1;
  return cudaLaunchKernelEx(&cfg, route_kernel, a);
}

}  // namespace rswa
