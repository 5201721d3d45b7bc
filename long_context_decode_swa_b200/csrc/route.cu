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

struct RouteArgs {
  int64_t cap;
  int nb_cap, chunks_cap, topk;
  float idx_scale;
  const float* q_idx;
  const float* kbar;
  const int32_t* prefix_len;
  int32_t* blk_idx;
  float* blk_logp;
  float* probs;
  float* tau;
  int32_t* status;
  int32_t* counters;  // [B]
  float* cmax;        // [B][chunks_cap]
  float2* cand;       // [B][chunks_cap][kList]: (z, block index as int bits)
  float* zbuf;        // [B][nb_cap]
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

// One CTA scores kRouteThreads blocks of one sequence (grid = chunks x B), keeps their
// sorted top-kList, and the last CTA of the sequence merges the chunk lists and solves
// the 1.5-entmax threshold exactly.
__global__ void __launch_bounds__(kRouteThreads) route_kernel(const RouteArgs a) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  __shared__ float lz[kRouteWarps][kList];
  __shared__ int li[kRouteWarps][kList];
  __shared__ float red[kRouteWarps];
  __shared__ int s_last, s_count;
  __shared__ unsigned long long s_best;  // (support size << 32) | bits(tau_y)

  const int chunk = blockIdx.x, b = blockIdx.y;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  griddep_wait();
  griddep_launch_dependents();
  int64_t m64 = a.prefix_len[b];
  if (m64 < 0 || m64 > a.cap) {
    if (tid == 0 && chunk == 0) set_status(a.status, RSWA_DEVICE_BAD_PREFIX_LEN);
    m64 = 0;
  }
  const int NB = (int)((m64 + kBlock - 1) / kBlock);
  const int chunks = (NB + kRouteThreads - 1) / kRouteThreads;
  if (NB == 0) {
    if (chunk == 0) {
      if (tid < a.topk) {
        a.blk_idx[(int64_t)b * a.topk + tid] = -1;
        a.blk_logp[(int64_t)b * a.topk + tid] = -INFINITY;
      }
      if (a.probs)
        for (int c = tid; c < a.nb_cap; c += kRouteThreads) a.probs[(int64_t)b * a.nb_cap + c] = 0.f;
      if (a.tau && tid == 0) a.tau[b] = NAN;
    }
    return;
  }
  if (chunk >= chunks) return;

  // ---- score one block per thread ----
  const int c = chunk * kRouteThreads + tid;
  float z = -INFINITY;
  int ci = kNone;
  if (c < NB) {
    const float4* q4 = reinterpret_cast<const float4*>(a.q_idx + (int64_t)b * kIndexDim);
    const float4* k4 = reinterpret_cast<const float4*>(a.kbar + ((int64_t)b * a.nb_cap + c) * kIndexDim);
    float4 kv[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) kv[u] = k4[u];
    float d = 0.f;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const float4 qv = q4[u];
      d = fmaf(qv.x, kv[u].x, d);
      d = fmaf(qv.y, kv[u].y, d);
      d = fmaf(qv.z, kv[u].z, d);
      d = fmaf(qv.w, kv[u].w, d);
    }
    z = a.idx_scale * d;
    ci = c;
    a.zbuf[(int64_t)b * a.nb_cap + c] = z;
  }
  const float wmax = warp_max(z);
  if (lane == 0) red[warp] = wmax;
  warp_sort(z, ci, lane);
  lz[warp][lane] = z;
  li[warp][lane] = ci;
  __syncthreads();
  merge_lists(lz, li, kRouteWarps, warp, lane);
  float2* my_list = a.cand + ((int64_t)b * a.chunks_cap + chunk) * kList;
  if (warp == 0) my_list[lane] = make_float2(lz[0][lane], __int_as_float(li[0][lane]));
  if (tid == 0) {
    float mx = red[0];
    for (int w = 1; w < kRouteWarps; ++w) mx = fmaxf(mx, red[w]);
    a.cmax[(int64_t)b * a.chunks_cap + chunk] = mx;
  }
  __threadfence();
  __syncthreads();
  if (tid == 0) s_last = atomicAdd(&a.counters[b], 1) == chunks - 1;
  __syncthreads();
  if (!s_last) return;
  __threadfence();

  // ---- last CTA of the sequence: merge the chunk lists ----
  if (warp < chunks) {
    const float2 e = __ldcg(a.cand + ((int64_t)b * a.chunks_cap + warp) * kList + lane);
    lz[warp][lane] = e.x;
    li[warp][lane] = __float_as_int(e.y);
  }
  if (tid == 0) {
    float mx = -INFINITY;
    for (int k = 0; k < chunks; ++k) mx = fmaxf(mx, __ldcg(a.cmax + (int64_t)b * a.chunks_cap + k));
    red[0] = 0.5f * mx;
    s_count = 0;
    s_best = 0ull;
  }
  __syncthreads();
  merge_lists(lz, li, chunks, warp, lane);
  const float xmax = red[0];

  // ---- 1.5-entmax over all NB blocks: candidates x > max x - 1, ranked, prefix sums ----
  float* cy = reinterpret_cast<float*>(smem_raw);  // [NB] shifted candidates y = x - max x
  int* cix = reinterpret_cast<int*>(cy + a.nb_cap);
  float* sy = reinterpret_cast<float*>(cix + a.nb_cap);
  const float* zb = a.zbuf + (int64_t)b * a.nb_cap;
  for (int k = tid; k < NB; k += kRouteThreads) {
    const float y = fmaf(__ldcg(zb + k), 0.5f, -xmax);
    if (y > -1.f) {
      const int slot = atomicAdd(&s_count, 1);
      cy[slot] = y;
      cix[slot] = k;
    }
  }
  __syncthreads();
  const int K = s_count;
  for (int i = tid; i < K; i += kRouteThreads) {
    const float yi = cy[i];
    const int ii = cix[i];
    int r = 0;
    for (int j = 0; j < K; ++j) r += ranks_before(cy[j], cix[j], yi, ii) ? 1 : 0;
    sy[r] = yi;
  }
  __syncthreads();
  for (int r = tid; r < K; r += kRouteThreads) {
    float s1 = 0.f, s2 = 0.f;
    for (int j = 0; j <= r; ++j) {
      const float y = sy[j];
      s1 += y;
      s2 = fmaf(y, y, s2);
    }
    const float k = (float)(r + 1);
    const float mean = s1 / k;
    const float delta = (1.f - (s2 - s1 * mean)) / k;
    if (delta >= 0.f) {
      const float t = mean - sqrtf(delta);
      if (t < sy[r])
        atomicMax(&s_best, ((unsigned long long)(r + 1) << 32) | (unsigned long long)__float_as_uint(t));
    }
  }
  __syncthreads();
  const float tau_y = __uint_as_float((unsigned)(s_best & 0xffffffffull));
  if (a.tau && tid == 0) a.tau[b] = tau_y + xmax;
  if (a.probs) {
    for (int k = tid; k < a.nb_cap; k += kRouteThreads) {
      float pr = 0.f;
      if (k < NB) {
        const float r = fmaf(__ldcg(zb + k), 0.5f, -xmax) - tau_y;
        pr = r > 0.f ? r * r : 0.f;
      }
      a.probs[(int64_t)b * a.nb_cap + k] = pr;
    }
  }
  if (warp == 0 && lane < a.topk) {
    const int64_t o = (int64_t)b * a.topk + lane;
    const int bi = li[0][lane];
    if (bi == kNone) {
      a.blk_idx[o] = -1;
      a.blk_logp[o] = -INFINITY;
    } else {
      const float d = fmaf(lz[0][lane], 0.5f, -xmax) - tau_y;
      const float pr = d > 0.f ? d * d : 0.f;
      a.blk_idx[o] = bi;
      a.blk_logp[o] = pr > 0.f ? logf(pr) : -INFINITY;
    }
  }
  if (tid == 0) a.counters[b] = 0;
}

}  // namespace

cudaError_t launch_index_pool(int B, int64_t cap, const uint16_t* k_idx, const int32_t* prefix_len, float* kbar,
                              cudaStream_t stream) {
  const int nb_cap = (int)((cap + kBlock - 1) / kBlock);
  const dim3 grid((nb_cap + kPoolWarps - 1) / kPoolWarps, B);
  index_pool_kernel<<<grid, kPoolWarps * 32, 0, stream>>>(cap, nb_cap, k_idx, prefix_len, kbar);
  return cudaGetLastError();
}

RouteWorkspace plan_route_workspace(int B, int64_t cap) {
  RouteWorkspace w;
  w.nb_cap = (int)((cap + kBlock - 1) / kBlock);
  w.chunks_cap = (w.nb_cap + kRouteThreads - 1) / kRouteThreads;
  size_t off = 256;  // status word
  w.counters_off = off;
  off += ((size_t)B * 4 + 255) / 256 * 256;
  w.cmax_off = off;
  off += ((size_t)B * w.chunks_cap * 4 + 255) / 256 * 256;
  w.cand_off = off;
  off += (size_t)B * w.chunks_cap * kList * 8;
  w.zbuf_off = off;
  off += (size_t)B * w.nb_cap * 4;
  w.bytes = off;
  return w;
}

cudaError_t launch_route(int B, int64_t cap, const float* q_idx, const float* kbar, const int32_t* prefix_len,
                         float idx_scale, int topk, int32_t* blk_idx, float* blk_logp, float* probs, float* tau,
                         void* workspace, cudaStream_t stream) {
  const RouteWorkspace w = plan_route_workspace(B, cap);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  RouteArgs a;
  a.cap = cap;
  a.nb_cap = w.nb_cap;
  a.chunks_cap = w.chunks_cap;
  a.topk = topk;
  a.idx_scale = idx_scale;
  a.q_idx = q_idx;
  a.kbar = kbar;
  a.prefix_len = prefix_len;
  a.blk_idx = blk_idx;
  a.blk_logp = blk_logp;
  a.probs = probs;
  a.tau = tau;
  a.status = reinterpret_cast<int32_t*>(ws);
  a.counters = reinterpret_cast<int32_t*>(ws + w.counters_off);
  a.cmax = reinterpret_cast<float*>(ws + w.cmax_off);
  a.cand = reinterpret_cast<float2*>(ws + w.cand_off);
  a.zbuf = reinterpret_cast<float*>(ws + w.zbuf_off);
  const size_t smem = (size_t)w.nb_cap * 12;
  static unsigned long long done = 0;
  cudaError_t e = ensure_smem_limit(route_kernel, (size_t)kMaxRouteBlocks * 12, &done);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  fill_launch_config(cfg, attr, dim3(w.chunks_cap, B), dim3(kRouteThreads), smem, stream);
  return cudaLaunchKernelEx(&cfg, route_kernel, a);
}

}  // namespace rswa
