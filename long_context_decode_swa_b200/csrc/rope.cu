// rope.cu -- page2d rotary position encoding of query / key rows.
//
// Two rotary axes share the head dimension: a token axis driven by the
// token's offset inside its page and a page axis driven by the page number
// (Unlimited-OCR-2 SR-SWA explainer, 2D 位置编码: sparse_rope_mode page2d,
// page_mod 2). The pages give neither frequencies nor the split; this library
// reads them as the LLaMA family's rotary encoding with the pairs shared out:
// pair i couples dims i and i + D/2 and turns by position * base^(-2i/D);
// it follows the page axis when i mod page_mod == page_mod - 1 and the token
// axis otherwise (page_mod 0: token axis only).
//
// HBM-bound: every element is read once and written once. A CTA takes G
// consecutive tokens at a time (G = 4 at 16 heads x 128 dims, q and k): each
// thread issues the 16-byte loads of up to four 8-pair chunks (dims 8c..8c+7
// and D/2+8c..D/2+8c+7 of one head), the whole CTA meanwhile computes the G
// tokens' pair angles (fp64 angle and sincos, one (token, pair) per thread,
// from a per-CTA table of the D/2 frequencies) and rounds cos / sin to fp32
// into shared memory; after one barrier each thread rotates its pairs in fp32
// (two FMAs per output) and stores bf16 (round to nearest even).
#include <cuda_bf16.h>

#include "common.cuh"
#include "internal.h"

namespace rswa {

namespace {

constexpr int kRopeThreads = 256;
constexpr int kRopeMaxHalf = 128;  // D <= 256
constexpr int kRopeCtasPerSm = 4;   // resident CTAs per SM (64 registers a thread)
constexpr int kRopeMaxGroup = 8;    // tokens per CTA iteration
constexpr int kRopeUnits = 4;       // chunk pairs a thread holds per pass

// Frequencies base^(-2i/D) = 2^(-(2i/D) log2(base)) of the D/2 pairs (log2(base) from the host).
__device__ __forceinline__ void pair_freqs(int D, double log2_base, double* th) {
  for (int i = threadIdx.x; i < (D >> 1); i += blockDim.x) th[i] = exp2(-(2.0 * i / D) * log2_base);
}

// cos / sin (rounded to fp32) of pair i of a token at (tok, pg).
__device__ __forceinline__ float2 pair_cos_sin(int i, int tok, int pg, int page_mod, const double* th) {
  const bool on_page = page_mod > 0 && i % page_mod == page_mod - 1;
  double s, c;
  sincos((double)(on_page ? pg : tok) * th[i], &s, &c);
  return make_float2((float)c, (float)s);
}

// Rotates eight pairs in place: lo holds their first halves (dims 8c + e), hi their second
// halves (dims D/2 + 8c + e), cs their cos / sin.
__device__ __forceinline__ void rotate8(uint4& lo, uint4& hi, const float2* cs) {
  uint32_t* l = reinterpret_cast<uint32_t*>(&lo);
  uint32_t* h = reinterpret_cast<uint32_t*>(&hi);
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    const float2 a0 = cs[2 * w], a1 = cs[2 * w + 1];
    const float x0 = bf16lo(l[w]), x1 = bf16hi(l[w]);
    const float y0 = bf16lo(h[w]), y1 = bf16hi(h[w]);
    const __nv_bfloat162 lo2 = __floats2bfloat162_rn(fmaf(x0, a0.x, -y0 * a0.y), fmaf(x1, a1.x, -y1 * a1.y));
    const __nv_bfloat162 hi2 = __floats2bfloat162_rn(fmaf(y0, a0.x, x0 * a0.y), fmaf(y1, a1.x, x1 * a1.y));
    l[w] = *reinterpret_cast<const uint32_t*>(&lo2);
    h[w] = *reinterpret_cast<const uint32_t*>(&hi2);
  }
}

// rows x [H][D] of q (and k): one row per token with positions tok_pos[r], page[r].
__global__ void __launch_bounds__(kRopeThreads, kRopeCtasPerSm) rope_kernel(int64_t rows, int H, int D, int group, const uint16_t* q,
                                                           uint16_t* q_out, const uint16_t* k, uint16_t* k_out,
                                                           const int32_t* __restrict__ tok_pos,
                                                           const int32_t* __restrict__ page, double log2_base,
                                                           int page_mod) {
  __shared__ double th[kRopeMaxHalf];
  __shared__ float2 cs[kRopeMaxGroup][kRopeMaxHalf];
  griddep_wait();  // inputs may come from, and outputs be read by, the neighbouring launches
  griddep_launch_dependents();
  pair_freqs(D, log2_base, th);
  __syncthreads();
  const int half = D >> 1;
  const int chunks = D >> 4;                 // 8-pair chunks per head
  const int per_tensor = H * chunks;
  const int items = (k != nullptr ? 2 : 1) * per_tensor;  // chunk pairs per token
  for (int64_t r0 = (int64_t)blockIdx.x * group; r0 < rows; r0 += (int64_t)gridDim.x * group) {
    const int g_rows = (int)(rows - r0 < group ? rows - r0 : group);
    const int units = g_rows * items;
    for (int u0 = 0; u0 < units; u0 += kRopeUnits * kRopeThreads) {
      uint4 lo[kRopeUnits], hi[kRopeUnits];
#pragma unroll
      for (int j = 0; j < kRopeUnits; ++j) {
        const int u = u0 + j * kRopeThreads + (int)threadIdx.x;
        if (u < units) {
          const int g = u / items, it = u - g * items;
          const int which = it / per_tensor, jt = it - which * per_tensor;
          const int h = jt / chunks, c = jt - h * chunks;
          const int64_t off = ((r0 + g) * H + h) * (int64_t)D + 8 * c;
          const uint16_t* src = which ? k : q;
          lo[j] = *reinterpret_cast<const uint4*>(src + off);
          hi[j] = *reinterpret_cast<const uint4*>(src + off + half);
        }
      }
      if (u0 == 0) {  // the group's angles, while its loads are in flight
        for (int a = threadIdx.x; a < g_rows * half; a += kRopeThreads) {
          const int g = a / half, i = a - g * half;
          cs[g][i] = pair_cos_sin(i, tok_pos[r0 + g], page[r0 + g], page_mod, th);
        }
        __syncthreads();
      }
#pragma unroll
      for (int j = 0; j < kRopeUnits; ++j) {
        const int u = u0 + j * kRopeThreads + (int)threadIdx.x;
        if (u < units) {
          const int g = u / items, it = u - g * items;
          const int which = it / per_tensor, jt = it - which * per_tensor;
          const int h = jt / chunks, c = jt - h * chunks;
          const int64_t off = ((r0 + g) * H + h) * (int64_t)D + 8 * c;
          rotate8(lo[j], hi[j], &cs[g][8 * c]);
          uint16_t* dst = which ? k_out : q_out;
          *reinterpret_cast<uint4*>(dst + off) = lo[j];
          *reinterpret_cast<uint4*>(dst + off + half) = hi[j];
        }
      }
    }
    __syncthreads();  // cs is rewritten by the next group
  }
}

// Ring append of one token per sequence with its key rotated on the way and its query
// rotated into q_out; v_new is copied unchanged (D = 128).
__global__ void __launch_bounds__(kRopeThreads) append_rope_kernel(
    int H, int n, uint16_t* __restrict__ ring_k, uint16_t* __restrict__ ring_v, const uint16_t* k_new,
    const uint16_t* __restrict__ v_new, const uint16_t* q, uint16_t* q_out, const int32_t* __restrict__ tok_pos,
    const int32_t* __restrict__ page, double log2_base, int page_mod, int32_t* wp, int32_t* fill, int32_t* slot_out,
    int32_t* status) {
  __shared__ float2 cs[kHeadDim / 2];
  __shared__ int s_slot;
  const int b = blockIdx.x;
  griddep_wait();  // the previous kernel may still be reading the slot this one overwrites
  griddep_launch_dependents();
  constexpr int kChunks = kHeadDim / 16;
  constexpr int kVecPerRow = kHeadDim / 8;
  const int per_tensor = H * kChunks;  // 8-pair chunks of q (then of k)
  const int vvec = H * kVecPerRow;     // uint4 of v_new
  int w = 0, f = 0;
  if (threadIdx.x == 0) {
    w = wp[b];
    f = fill[b];
  }
  // first pass held in registers across the ring-state read: one q/k chunk pair and two
  // v vectors per thread (all of them for H <= 16)
  const int it0 = threadIdx.x;
  const bool has_qk = it0 < 2 * per_tensor;
  const int which0 = has_qk ? it0 / per_tensor : 0;
  const int j0 = it0 - which0 * per_tensor;
  const int h0 = j0 / kChunks, c0 = j0 - h0 * kChunks;
  const int64_t off0 = ((int64_t)b * H + h0) * kHeadDim + 8 * c0;
  uint4 lo = make_uint4(0, 0, 0, 0), hi = lo, v0 = lo, v1 = lo;
  if (has_qk) {
    const uint16_t* src = which0 ? k_new : q;
    lo = *reinterpret_cast<const uint4*>(src + off0);
    hi = *reinterpret_cast<const uint4*>(src + off0 + kHeadDim / 2);
  }
  const uint4* vsrc = reinterpret_cast<const uint4*>(v_new + (int64_t)b * H * kHeadDim);
  if (it0 < vvec) v0 = vsrc[it0];
  if (it0 + kRopeThreads < vvec) v1 = vsrc[it0 + kRopeThreads];
  if (threadIdx.x < kHeadDim / 2) {
    const int i = threadIdx.x;
    const bool on_page = page_mod > 0 && i % page_mod == page_mod - 1;
    double s, c;
    sincos((double)(on_page ? page[b] : tok_pos[b]) * exp2(-(2.0 * i / kHeadDim) * log2_base), &s, &c);
    cs[i] = make_float2((float)c, (float)s);
  }
  if (threadIdx.x == 0) {
    const bool ok = w >= 0 && w < n && f >= 0 && f <= n;
    if (!ok) set_status(status, RSWA_DEVICE_BAD_RING_STATE);
    s_slot = ok ? w : -1;
    if (ok) {
      wp[b] = (w + 1 == n) ? 0 : w + 1;
      fill[b] = min(f + 1, n);
      if (slot_out) slot_out[b] = w;
    }
  }
  __syncthreads();
  const int slot = s_slot;
  // q is rotated whatever the ring state; k and v go to the ring only with a valid slot
  auto put_qk = [&](int which, int h, int c, int64_t off, uint4 a, uint4 z) {
    rotate8(a, z, cs + 8 * c);
    uint16_t* dst;
    if (which == 0) {
      dst = q_out + off;
    } else {
      if (slot < 0) return;
      dst = ring_k + (((int64_t)b * H + h) * n + slot) * kHeadDim + 8 * c;
    }
    *reinterpret_cast<uint4*>(dst) = a;
    *reinterpret_cast<uint4*>(dst + kHeadDim / 2) = z;
  };
  auto put_v = [&](int i, uint4 val) {
    const int h = i / kVecPerRow, e = i - h * kVecPerRow;
    reinterpret_cast<uint4*>(ring_v + (((int64_t)b * H + h) * n + slot) * kHeadDim)[e] = val;
  };
  if (has_qk) put_qk(which0, h0, c0, off0, lo, hi);
  if (slot >= 0) {
    if (it0 < vvec) put_v(it0, v0);
    if (it0 + kRopeThreads < vvec) put_v(it0 + kRopeThreads, v1);
  }
  // heads beyond what the first pass held (H > 16)
  for (int it = it0 + kRopeThreads; it < 2 * per_tensor; it += kRopeThreads) {
    const int which = it / per_tensor;
    const int j = it - which * per_tensor;
    const int h = j / kChunks, c = j - h * kChunks;
    const int64_t off = ((int64_t)b * H + h) * kHeadDim + 8 * c;
    const uint16_t* src = which ? k_new : q;
    put_qk(which, h, c, off, *reinterpret_cast<const uint4*>(src + off),
           *reinterpret_cast<const uint4*>(src + off + kHeadDim / 2));
  }
  if (slot >= 0)
    for (int i = it0 + 2 * kRopeThreads; i < vvec; i += kRopeThreads) put_v(i, vsrc[i]);
}

}  // namespace

cudaError_t launch_rope(int64_t rows, int H, int D, const uint16_t* q, uint16_t* q_out, const uint16_t* k,
                        uint16_t* k_out, const int32_t* tok_pos, const int32_t* page, double base, int page_mod,
                        cudaStream_t stream) {
  // tokens per CTA iteration: about 1024 chunk pairs (four per thread), 1..8 tokens
  const int items = (k != nullptr ? 2 : 1) * H * (D / 16);
  int group = (kRopeUnits * kRopeThreads) / items;
  group = group < 1 ? 1 : (group > kRopeMaxGroup ? kRopeMaxGroup : group);
  const int64_t groups = (rows + group - 1) / group;
  const int64_t most = (int64_t)device_sm_count() * kRopeCtasPerSm;
  const int grid = (int)(groups < most ? groups : most);
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  fill_launch_config(cfg, attr, dim3(grid), dim3(kRopeThreads), 0, stream);
  return cudaLaunchKernelEx(&cfg, rope_kernel, rows, H, D, group, q, q_out, k, k_out, tok_pos, page, log2(base),
                            page_mod);
}

cudaError_t launch_append_rope(int B, int H, int n, uint16_t* ring_k, uint16_t* ring_v, const uint16_t* k_new,
                               const uint16_t* v_new, const uint16_t* q, uint16_t* q_out, const int32_t* tok_pos,
                               const int32_t* page, double base, int page_mod, int32_t* wp, int32_t* fill,
                               int32_t* slot_out, int32_t* status, cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  fill_launch_config(cfg, attr, dim3(B), dim3(kRopeThreads), 0, stream);
  return cudaLaunchKernelEx(&cfg, append_rope_kernel, H, n, ring_k, ring_v, k_new, v_new, q, q_out, tok_pos, page,
                            log2(base), page_mod, wp, fill, slot_out, status);
}

}  // namespace rswa
