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
constexpr int kScoreUnroll = 8;

// Index keys: one warp per 32-token block; lane (tg, dq) sums tokens tg, tg+8, ...
// over dims 8dq..8dq+7, then the eight token groups are folded with shuffles.
__global__ void __launch_bounds__(kPoolWarps * 32) index_pool_kernel(int64_t cap, int nb_cap,
                                                                     const uint16_t* __restrict__ k_idx,
                                                                     const int32_t* __restrict__ prefix_len,
                                                                     float* __restrict__ kbar) {
  const int b = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
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

__device__ __forceinline__ void warp_best(float& z, int& i) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    const float oz = __shfl_xor_sync(0xffffffffu, z, off);
    const int oi = __shfl_xor_sync(0xffffffffu, i, off);
    if (ranks_before(oz, oi, z, i)) {
      z = oz;
      i = oi;
    }
  }
}

constexpr int kNone = 0x7fffffff;

__global__ void __launch_bounds__(kRouteThreads) route_kernel(int64_t cap, int nb_cap, const float* __restrict__ q_idx,
                                                              const float* __restrict__ kbar,
                                                              const int32_t* __restrict__ prefix_len, float idx_scale,
                                                              int topk, int32_t* __restrict__ blk_idx,
                                                              float* __restrict__ blk_logp, float* __restrict__ probs,
                                                              float* __restrict__ tau_out, int32_t* status) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  float* z = reinterpret_cast<float*>(smem_raw);  // [nb_cap] block scores
  float* cy = z + nb_cap;                         // [nb_cap] candidates: y = z/2 - max(z/2)
  int* ci = reinterpret_cast<int*>(cy + nb_cap);  // [nb_cap] candidates: block index
  float* sy = reinterpret_cast<float*>(ci + nb_cap);  // [nb_cap] candidates sorted by rank
  __shared__ float red[kRouteWarps];
  __shared__ float s_xmax;
  __shared__ int s_count;
  __shared__ unsigned long long s_best;  // (support size << 32) | bits(tau_y)
  __shared__ float wz[kRouteWarps][kMaxTopk];
  __shared__ int wi[kRouteWarps][kMaxTopk];

  const int b = blockIdx.x;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  int64_t m64 = prefix_len[b];
  if (m64 < 0 || m64 > cap) {
    if (tid == 0) set_status(status, RSWA_DEVICE_BAD_PREFIX_LEN);
    m64 = 0;
  }
  const int NB = (int)((m64 + kBlock - 1) / kBlock);
  if (NB == 0) {
    if (tid < topk) {
      blk_idx[(int64_t)b * topk + tid] = -1;
      blk_logp[(int64_t)b * topk + tid] = -INFINITY;
    }
    if (probs)
      for (int c = tid; c < nb_cap; c += kRouteThreads) probs[(int64_t)b * nb_cap + c] = 0.f;
    if (tau_out && tid == 0) tau_out[b] = NAN;
    return;
  }

  // ---- 1. block scores z_c = idx_scale * <q_idx, kbar_c>: 8 lanes per block ----
  const int sub = lane >> 3, dq = lane & 7;
  const float4 q4 = reinterpret_cast<const float4*>(q_idx + (int64_t)b * kIndexDim)[dq];
  const float* kb = kbar + (int64_t)b * nb_cap * kIndexDim;
  float lmax = -INFINITY;
  for (int c0 = warp * 4 * kScoreUnroll; c0 < NB; c0 += kRouteWarps * 4 * kScoreUnroll) {
    float4 k4[kScoreUnroll];
#pragma unroll
    for (int u = 0; u < kScoreUnroll; ++u) {
      const int c = c0 + u * 4 + sub;
      k4[u] = c < NB ? reinterpret_cast<const float4*>(kb + (int64_t)c * kIndexDim)[dq]
                     : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int u = 0; u < kScoreUnroll; ++u) {
      const int c = c0 + u * 4 + sub;
      float d = q4.x * k4[u].x;
      d = fmaf(q4.y, k4[u].y, d);
      d = fmaf(q4.z, k4[u].z, d);
      d = fmaf(q4.w, k4[u].w, d);
      d += __shfl_xor_sync(0xffffffffu, d, 1);
      d += __shfl_xor_sync(0xffffffffu, d, 2);
      d += __shfl_xor_sync(0xffffffffu, d, 4);
      if (c < NB) {
        const float zc = idx_scale * d;
        if (dq == 0) z[c] = zc;
        lmax = fmaxf(lmax, zc);
      }
    }
  }
  lmax = warp_max(lmax);
  if (lane == 0) red[warp] = lmax;
  __syncthreads();
  if (tid == 0) {
    float mx = red[0];
    for (int w = 1; w < kRouteWarps; ++w) mx = fmaxf(mx, red[w]);
    s_xmax = 0.5f * mx;
    s_count = 0;
    s_best = 0ull;
  }
  __syncthreads();
  const float xmax = s_xmax;

  // ---- 2. gather the candidates x_c > max x - 1 ----
  for (int c = tid; c < NB; c += kRouteThreads) {
    const float y = fmaf(z[c], 0.5f, -xmax);
    if (y > -1.f) {
      const int k = atomicAdd(&s_count, 1);
      cy[k] = y;
      ci[k] = c;
    }
  }
  __syncthreads();
  const int K = s_count;

  // ---- 3. rank the candidates (descending y, ties to the smaller block) ----
  for (int i = tid; i < K; i += kRouteThreads) {
    const float yi = cy[i];
    const int ii = ci[i];
    int r = 0;
    for (int j = 0; j < K; ++j) r += ranks_before(cy[j], ci[j], yi, ii) ? 1 : 0;
    sy[r] = yi;
  }
  __syncthreads();

  // ---- 4. sort-based threshold: prefix sums in rank order ----
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
  if (tau_out && tid == 0) tau_out[b] = tau_y + xmax;
  if (probs) {
    for (int c = tid; c < nb_cap; c += kRouteThreads) {
      float p = 0.f;
      if (c < NB) {
        const float r = fmaf(z[c], 0.5f, -xmax) - tau_y;
        p = r > 0.f ? r * r : 0.f;
      }
      probs[(int64_t)b * nb_cap + c] = p;
    }
  }

  // ---- 5. top-k: each warp selects from its slice, warp 0 merges ----
  {
    const int chunk = (NB + kRouteWarps - 1) / kRouteWarps;
    const int lo = warp * chunk, hi = min(NB, lo + chunk);
    float pz = INFINITY;
    int pi = -1;
    for (int r = 0; r < topk; ++r) {
      float bz = -INFINITY;
      int bi = kNone;
      for (int c = lo + lane; c < hi; c += 32) {
        const float zc = z[c];
        if (ranks_before(pz, pi, zc, c) && ranks_before(zc, c, bz, bi)) {
          bz = zc;
          bi = c;
        }
      }
      warp_best(bz, bi);
      if (lane == 0) {
        wz[warp][r] = bz;
        wi[warp][r] = bi;
      }
      pz = bz;
      pi = bi;
    }
  }
  __syncthreads();
  if (warp == 0) {
    float pz = INFINITY;
    int pi = -1;
    for (int r = 0; r < topk; ++r) {
      float bz = -INFINITY;
      int bi = kNone;
      for (int e = lane; e < kRouteWarps * topk; e += 32) {
        const float zc = wz[e / topk][e % topk];
        const int c = wi[e / topk][e % topk];
        if (c != kNone && ranks_before(pz, pi, zc, c) && ranks_before(zc, c, bz, bi)) {
          bz = zc;
          bi = c;
        }
      }
      warp_best(bz, bi);
      if (lane == 0) {
        const int64_t o = (int64_t)b * topk + r;
        if (bi == kNone) {
          blk_idx[o] = -1;
          blk_logp[o] = -INFINITY;
        } else {
          const float d = fmaf(z[bi], 0.5f, -xmax) - tau_y;
          const float p = d > 0.f ? d * d : 0.f;
          blk_idx[o] = bi;
          blk_logp[o] = p > 0.f ? logf(p) : -INFINITY;
        }
      }
      pz = bz;
      pi = bi;
    }
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

cudaError_t launch_route(int B, int64_t cap, const float* q_idx, const float* kbar, const int32_t* prefix_len,
                         float idx_scale, int topk, int32_t* blk_idx, float* blk_logp, float* probs, float* tau,
                         int32_t* status, cudaStream_t stream) {
  const int nb_cap = (int)((cap + kBlock - 1) / kBlock);
  const size_t smem = (size_t)nb_cap * 16;
  static unsigned long long done = 0;
  // one-time raise to the largest size the router supports
  cudaError_t e = ensure_smem_limit(route_kernel, (size_t)kMaxRouteBlocks * 16, &done);
  if (e != cudaSuccess) return e;
  route_kernel<<<B, kRouteThreads, smem, stream>>>(cap, nb_cap, q_idx, kbar, prefix_len, idx_scale, topk, blk_idx,
                                                   blk_logp, probs, tau, status);
  return cudaGetLastError();
}

}  // namespace rswa
