// append.cu -- ring-buffer append of one generated token per sequence.
//
// The newest token's K/V overwrite the ring slot at the write pointer of every
// head, the pointer advances cyclically and the valid count saturates at n
// (Unlimited-OCR-2 SR-SWA explainer, 环形缓冲; "百度 Unlimited OCR 深度实战"
// tutorial §3.3.2). One CTA per sequence copies its H x 256 B of K and of V
// with 16-byte loads/stores; thread 0 alone reads and advances wp/fill, so no
// other thread of the launch touches them.
#include "common.cuh"
#include "internal.h"

namespace rswa {

namespace {

constexpr int kAppendThreads = 128;

__global__ void __launch_bounds__(kAppendThreads) append_kernel(int H, int n, uint16_t* __restrict__ ring_k,
                                                                uint16_t* __restrict__ ring_v,
                                                                const uint16_t* __restrict__ k_new,
                                                                const uint16_t* __restrict__ v_new, int32_t* wp,
                                                                int32_t* fill, int32_t* slot_out, int32_t* status) {
  __shared__ int s_slot;
  const int b = blockIdx.x;
  griddep_wait();  // the previous kernel may still be reading the slot this one overwrites
  griddep_launch_dependents();
  if (threadIdx.x == 0) {
    const int w = wp[b], f = fill[b];
    const bool ok = w >= 0 && w < n && f >= 0 && f <= n;
    if (!ok) set_status(status, RSWA_DEVICE_BAD_RING_STATE);
    s_slot = ok ? w : -1;
  }
  __syncthreads();
  const int slot = s_slot;
  if (slot < 0) return;
  constexpr int kVecPerRow = kHeadDim / 8;  // uint4 per 128-dim bf16 row
  const int per_tensor = H * kVecPerRow;
  for (int i = threadIdx.x; i < 2 * per_tensor; i += kAppendThreads) {
    const int which = i / per_tensor;
    const int j = i - which * per_tensor;
    const int h = j / kVecPerRow, e = j - h * kVecPerRow;
    const int64_t bh = (int64_t)b * H + h;
    const uint4* src = reinterpret_cast<const uint4*>((which ? v_new : k_new) + bh * kHeadDim) + e;
    uint4* dst = reinterpret_cast<uint4*>((which ? ring_v : ring_k) + (bh * n + slot) * kHeadDim) + e;
    *dst = *src;
  }
  if (threadIdx.x == 0) {
    wp[b] = (slot + 1 == n) ? 0 : slot + 1;
    fill[b] = min(fill[b] + 1, n);
    if (slot_out) slot_out[b] = slot;
  }
}

}  // namespace

cudaError_t launch_append(int B, int H, int n, uint16_t* ring_k, uint16_t* ring_v, const uint16_t* k_new,
                          const uint16_t* v_new, int32_t* wp, int32_t* fill, int32_t* slot_out, int32_t* status,
                          cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  fill_launch_config(cfg, attr, dim3(B), dim3(kAppendThreads), 0, stream);
  return cudaLaunchKernelEx(&cfg, append_kernel, H, n, ring_k, ring_v, k_new, v_new, wp, fill, slot_out, status);
}

}  // namespace rswa
