// quant.cu -- FP8 (E4M3) prefix quantisation with per-(sequence, head, block) scales.
//
// The Unlimited-OCR technical analysis page lists quantised KV-cache compression among
// its memory measures (内存使用效率, KV缓存压缩) without a format; this library's
// reading: E4M3 codes with one
// f32 scale per (sequence, head, 32-token block) for K and one for V, scale = amax / 448
// over the block's valid rows, code = E4M3(x / scale) rounded to nearest even and
// saturating at +-448, both steps in f32 (IEEE division, as written). Rows of a partial
// block past prefix_len get code 0; blocks past it are not written.
//
// One warp per (block, sequence, head, K or V): lane l holds dims 4l..4l+3 of the 32
// rows (one coalesced 256-byte read per row), the warp reduces amax with shuffles, and
// each lane writes its 4 codes of a row as one 32-bit store (128 bytes per row).
#include <cuda_fp8.h>

#include "common.cuh"
#include "internal.h"

namespace rswa {

namespace {

constexpr int kQuantWarps = 4;

__global__ void __launch_bounds__(kQuantWarps * 32)
    quantize_kernel(int H, int64_t cap, int64_t nb_cap, const uint16_t* __restrict__ pk,
                    const uint16_t* __restrict__ pv, const int32_t* __restrict__ prefix_len, uint8_t* __restrict__ pk8,
                    uint8_t* __restrict__ pv8, float* __restrict__ k_scale, float* __restrict__ v_scale,
                    int32_t* status) {
  griddep_wait();
  griddep_launch_dependents();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t c = (int64_t)blockIdx.x * kQuantWarps + warp;
  const int64_t bh = blockIdx.y;
  const int b = (int)(bh / H);
  const bool is_v = blockIdx.z != 0;
  int64_t m = prefix_len[b];
  if (m < 0 || m > cap) {
    if (c == 0 && lane == 0 && !is_v && bh % H == 0) set_status(status, RSWA_DEVICE_BAD_PREFIX_LEN);
    return;
  }
  if (c >= nb_cap || c * kBlock >= m) return;  // warp-uniform
  const int rows = m - c * kBlock < kBlock ? (int)(m - c * kBlock) : kBlock;
  const uint16_t* src = (is_v ? pv : pk) + (bh * cap + c * kBlock) * kHeadDim;
  uint8_t* dst = (is_v ? pv8 : pk8) + (bh * cap + c * kBlock) * kHeadDim;
  uint2 x[kBlock];
  float amax = 0.f;
#pragma unroll
  for (int r = 0; r < kBlock; ++r) {
    x[r] = r < rows ? reinterpret_cast<const uint2*>(src + (int64_t)r * kHeadDim)[lane] : make_uint2(0, 0);
    amax = fmaxf(amax, fmaxf(fmaxf(fabsf(bf16lo(x[r].x)), fabsf(bf16hi(x[r].x))),
                             fmaxf(fabsf(bf16lo(x[r].y)), fabsf(bf16hi(x[r].y)))));
  }
  amax = warp_max(amax);
  const float scale = amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f;
  if (lane == 0) (is_v ? v_scale : k_scale)[bh * nb_cap + c] = scale;
#pragma unroll
  for (int r = 0; r < kBlock; ++r) {
    if (c * kBlock + r >= cap) break;
    uint32_t word = 0;
    if (r < rows) {
      const float2 lo = make_float2(__fdiv_rn(bf16lo(x[r].x), scale), __fdiv_rn(bf16hi(x[r].x), scale));
      const float2 hi = make_float2(__fdiv_rn(bf16lo(x[r].y), scale), __fdiv_rn(bf16hi(x[r].y), scale));
      word = (uint32_t)__nv_cvt_float2_to_fp8x2(lo, __NV_SATFINITE, __NV_E4M3) |
             ((uint32_t)__nv_cvt_float2_to_fp8x2(hi, __NV_SATFINITE, __NV_E4M3) << 16);
    }
    reinterpret_cast<uint32_t*>(dst + (int64_t)r * kHeadDim)[lane] = word;
  }
}

// Ring append into an FP8 ring: one CTA per sequence, one warp per (head, K or V) row: lane l
// holds dims 4l..4l+3, the warp reduces the row's amax, and the row is written as codes with
// its own scale (the ring is written one token at a time, so a row is the unit that is
// complete when written). Thread 0 reads and advances wp / fill, as append_kernel does.
constexpr int kAppend8Warps = 8;

__global__ void __launch_bounds__(kAppend8Warps * 32)
    append_fp8_kernel(int H, int n, uint8_t* __restrict__ ring_k8, uint8_t* __restrict__ ring_v8,
                      float* __restrict__ ring_ks, float* __restrict__ ring_vs, const uint16_t* __restrict__ k_new,
                      const uint16_t* __restrict__ v_new, int32_t* wp, int32_t* fill, int32_t* slot_out,
                      int32_t* status) {
  __shared__ int s_slot;
  const int b = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  griddep_wait();  // the previous kernel may still be reading the slot this one overwrites
  griddep_launch_dependents();
  if (threadIdx.x == 0) {
    const int w = wp[b], f = fill[b];
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
  if (slot < 0) return;
  for (int r = warp; r < 2 * H; r += kAppend8Warps) {  // warp-uniform
    const int h = r >> 1;
    const bool is_v = r & 1;
    const int64_t bh = (int64_t)b * H + h;
    const uint2 x = reinterpret_cast<const uint2*>((is_v ? v_new : k_new) + bh * kHeadDim)[lane];
    float amax = fmaxf(fmaxf(fabsf(bf16lo(x.x)), fabsf(bf16hi(x.x))), fmaxf(fabsf(bf16lo(x.y)), fabsf(bf16hi(x.y))));
    amax = warp_max(amax);
    const float scale = amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f;
    const int64_t row = bh * n + slot;
    if (lane == 0) (is_v ? ring_vs : ring_ks)[row] = scale;
    const float2 lo = make_float2(__fdiv_rn(bf16lo(x.x), scale), __fdiv_rn(bf16hi(x.x), scale));
    const float2 hi = make_float2(__fdiv_rn(bf16lo(x.y), scale), __fdiv_rn(bf16hi(x.y), scale));
    const uint32_t word = (uint32_t)__nv_cvt_float2_to_fp8x2(lo, __NV_SATFINITE, __NV_E4M3) |
                          ((uint32_t)__nv_cvt_float2_to_fp8x2(hi, __NV_SATFINITE, __NV_E4M3) << 16);
    reinterpret_cast<uint32_t*>((is_v ? ring_v8 : ring_k8) + row * kHeadDim)[lane] = word;
  }
}

}  // namespace

cudaError_t launch_append_fp8(int B, int H, int n, uint8_t* ring_k8, uint8_t* ring_v8, float* ring_ks, float* ring_vs,
                              const uint16_t* k_new, const uint16_t* v_new, int32_t* wp, int32_t* fill,
                              int32_t* slot_out, int32_t* status, cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  fill_launch_config(cfg, attr, dim3(B), dim3(kAppend8Warps * 32), 0, stream);
  return cudaLaunchKernelEx(&cfg, append_fp8_kernel, H, n, ring_k8, ring_v8, ring_ks, ring_vs, k_new, v_new, wp,
                            fill, slot_out, status);
}

cudaError_t launch_quantize_prefix(int B, int H, int64_t cap, const uint16_t* pk, const uint16_t* pv,
                                   const int32_t* prefix_len, uint8_t* pk8, uint8_t* pv8, float* k_scale,
                                   float* v_scale, int32_t* status, cudaStream_t stream) {
  const int64_t nb_cap = (cap + kBlock - 1) / kBlock;
  if (nb_cap == 0) return cudaSuccess;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  fill_launch_config(cfg, attr, dim3((unsigned)((nb_cap + kQuantWarps - 1) / kQuantWarps), (unsigned)(B * H), 2),
                     dim3(kQuantWarps * 32), 0, stream);
  return cudaLaunchKernelEx(&cfg, quantize_kernel, H, cap, nb_cap, pk, pv, prefix_len, pk8, pv8, k_scale, v_scale,
                            status);
}

}  // namespace rswa
