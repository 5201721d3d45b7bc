// append.cu -- ring-buffer append of one generated token per sequence.
//
// The newest token's K/V overwrite the ring slot at the write pointer of every
// head, the pointer advances cyclically and the valid count saturates at n
// (Unlimited-OCR-2 SR-SWA explainer, 环形缓冲; "百度 Unlimited OCR 深度实战"
// tutorial §3.3.2). One CTA per sequence copies its H x 256 B of K and of V
// with 16-byte loads/stores; the rows are loaded while thread 0 reads wp/fill,
// so the kernel costs one memory round trip before its stores. Thread 0 alone
// reads and advances wp/fill, so no other thread of the launch touches them.
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
  // the new rows are loaded while thread 0 reads the ring state (one round trip, not two)
  constexpr int kVecPerRow = kHeadDim / 8;  // uint4 per 128-dim bf16 row
  constexpr int kMaxVec = 4;  // rows held in registers: 4 x 128 uint4 covers K and V of H <= 16 heads
  const int per_tensor = H * kVecPerRow;
  int w = 0, f = 0;
  if (threadIdx.x == 0) {
    w = wp[b];
    f = fill[b];
  }
  uint4 row[kMaxVec];
  int cnt = 0;
#pragma unroll
  for (int u = 0; u < kMaxVec; ++u) {
    const int i = threadIdx.x + u * kAppendThreads;
    if (i < 2 * per_tensor) {
      const int which = i / per_tensor;
      const int j = i - which * per_tensor;
      row[u] = reinterpret_cast<const uint4*>((which ? v_new : k_new) + (int64_t)b * H * kHeadDim)[j];
      cnt = u + 1;
    }
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
  if (slot < 0) return;
#pragma unroll
  for (int u = 0; u < kMaxVec; ++u) {
    if (u >= cnt) break;
    const int i = threadIdx.x + u * kAppendThreads;
    const int which = i / per_tensor;
    const int j = i - which * per_tensor;
    const int h = j / kVecPerRow, e = j - h * kVecPerRow;
    const int64_t bh = (int64_t)b * H + h;
    reinterpret_cast<uint4*>((which ? ring_v : ring_k) + (bh * n + slot) * kHeadDim)[e] = row[u];
  }
  // rows beyond what the registers held (H > 16): plain copy
  for (int i = threadIdx.x + kMaxVec * kAppendThreads; i < 2 * per_tensor; i += kAppendThreads) {
    const int which = i / per_tensor;
    const int j = i - which * per_tensor;
    const int h = j / kVecPerRow, e = j - h * kVecPerRow;
    const int64_t bh = (int64_t)b * H + h;
    reinterpret_cast<uint4*>((which ? ring_v : ring_k) + (bh * n + slot) * kHeadDim)[e] =
        reinterpret_cast<const uint4*>((which ? v_new : k_new) + bh * kHeadDim)[e];
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
