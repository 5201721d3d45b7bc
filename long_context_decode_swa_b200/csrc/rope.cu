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
// HBM-bound: every element is read once and written once. A CTA works one row
// (one token, all heads, q and k) at a time: its threads issue the row's
// 16-byte loads (dims 8c..8c+7 and D/2+8c..D/2+8c+7 of one head, the two
// halves of eight pairs), D/2 threads meanwhile compute the row's angles in
// fp64 into shared memory, then each thread rotates its eight pairs and
// stores them. The rotation runs in fp64 and is rounded once to bf16, so the
// output is the correctly rounded rotation of the bf16 inputs up to the last
// bits of the angle; fp64 costs nothing against the memory traffic here.
#include <cuda_bf16.h>

#include "common.cuh"
#include "internal.h"

namespace rswa {

namespace {

constexpr int kRopeThreads = 256;
constexpr int kRopeMaxHalf = 128;  // D <= 256
constexpr int kRopeCtasPerSm = 8;

// cos / sin of the D/2 pair angles of one token (threads stride over the pairs).
__device__ __forceinline__ void pair_angles(int D, int tok, int pg, double base, int page_mod, double2* cs) {
  const int half = D >> 1;
  for (int i = threadIdx.x; i < half; i += blockDim.x) {
    const bool on_page = page_mod > 0 && i % page_mod == page_mod - 1;
    const double pos = on_page ? (double)pg : (double)tok;
    const double theta = pow(base, -2.0 * i / D);
    double s, c;
    sincos(pos * theta, &s, &c);
    cs[i] = make_double2(c, s);
  }
}

__device__ __forceinline__ uint32_t pack_bf16x2(double a, double b) {
  return (uint32_t)__bfloat16_as_ushort(__double2bfloat16(a)) |
         ((uint32_t)__bfloat16_as_ushort(__double2bfloat16(b)) << 16);
}

// Rotates eight pairs in place: lo holds their first halves (dims 8c + e), hi their second
// halves (dims D/2 + 8c + e), cs their cos / sin.
__device__ __forceinline__ void rotate8(uint4& lo, uint4& hi, const double2* cs) {
  uint32_t* l = reinterpret_cast<uint32_t*>(&lo);
  uint32_t* h = reinterpret_cast<uint32_t*>(&hi);
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    const double2 a0 = cs[2 * w], a1 = cs[2 * w + 1];
    const double x0 = bf16lo(l[w]), x1 = bf16hi(l[w]);
    const double y0 = bf16lo(h[w]), y1 = bf16hi(h[w]);
    l[w] = pack_bf16x2(x0 * a0.x - y0 * a0.y, x1 * a1.x - y1 * a1.y);
    h[w] = pack_bf16x2(y0 * a0.x + x0 * a0.y, y1 * a1.x + x1 * a1.y);
  }
}

// rows x [H][D] of q (and k): one row per token with positions tok_pos[r], page[r].
__global__ void __launch_bounds__(kRopeThreads) rope_kernel(int64_t rows, int H, int D, const uint16_t* q,
                                                           uint16_t* q_out, const uint16_t* k, uint16_t* k_out,
                                                           const int32_t* __restrict__ tok_pos,
                                                           const int32_t* __restrict__ page, double base,
                                                           int page_mod) {
  __shared__ double2 cs[kRopeMaxHalf];
  griddep_wait();  // inputs may come from, and outputs be read by, the neighbouring launches
  griddep_launch_dependents();
  const int chunks = D >> 4;                 // 8-pair chunks per head
  const int per_tensor = H * chunks;
  const int items = (k != nullptr ? 2 : 1) * per_tensor;
  const int half = D >> 1;
  for (int64_t r = blockIdx.x; r < rows; r += gridDim.x) {
    for (int base_item = 0; base_item < items; base_item += blockDim.x) {
      const int it = base_item + threadIdx.x;
      const bool mine = it < items;
      const int which = mine ? it / per_tensor : 0;
      const int j = it - which * per_tensor;
      const int h = j / chunks, c = j - h * chunks;
      const int64_t off = (r * H + h) * (int64_t)D + 8 * c;
      uint4 lo = make_uint4(0, 0, 0, 0), hi = lo;
      if (mine) {
        const uint16_t* src = which ? k : q;
        lo = *reinterpret_cast<const uint4*>(src + off);
        hi = *reinterpret_cast<const uint4*>(src + off + half);
      }
      if (base_item == 0) {  // the row's angles, while its loads are in flight
        pair_angles(D, tok_pos[r], page[r], base, page_mod, cs);
        __syncthreads();
      }
      if (mine) {
        rotate8(lo, hi, cs + 8 * c);
        uint16_t* dst = which ? k_out : q_out;
        *reinterpret_cast<uint4*>(dst + off) = lo;
        *reinterpret_cast<uint4*>(dst + off + half) = hi;
      }
    }
    __syncthreads();  // cs is rewritten by the next row
  }
}

// Ring append of one token per sequence with its key rotated on the way and its query
// rotated into q_out; v_new is copied unchanged (D = 128).
__global__ void __launch_bounds__(kRopeThreads) append_rope_kernel(
    int H, int n, uint16_t* __restrict__ ring_k, uint16_t* __restrict__ ring_v, const uint16_t* k_new,
    const uint16_t* __restrict__ v_new, const uint16_t* q, uint16_t* q_out, const int32_t* __restrict__ tok_pos,
    const int32_t* __restrict__ page, double base, int page_mod, int32_t* wp, int32_t* fill, int32_t* slot_out,
    int32_t* status) {
  __shared__ double2 cs[kHeadDim / 2];
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
  pair_angles(kHeadDim, tok_pos[b], page[b], base, page_mod, cs);
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
  const int64_t most = (int64_t)device_sm_count() * kRopeCtasPerSm;
  const int grid = (int)(rows < most ? rows : most);
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  fill_launch_config(cfg, attr, dim3(grid), dim3(kRopeThreads), 0, stream);
  return cudaLaunchKernelEx(&cfg, rope_kernel, rows, H, D, q, q_out, k, k_out, tok_pos, page, base, page_mod);
}

cudaError_t launch_append_rope(int B, int H, int n, uint16_t* ring_k, uint16_t* ring_v, const uint16_t* k_new,
                               const uint16_t* v_new, const uint16_t* q, uint16_t* q_out, const int32_t* tok_pos,
                               const int32_t* page, double base, int page_mod, int32_t* wp, int32_t* fill,
                               int32_t* slot_out, int32_t* status, cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  fill_launch_config(cfg, attr, dim3(B), dim3(kRopeThreads), 0, stream);
  return cudaLaunchKernelEx(&cfg, append_rope_kernel, H, n, ring_k, ring_v, k_new, v_new, q, q_out, tok_pos, page,
                            base, page_mod, wp, fill, slot_out, status);
}

}  // namespace rswa
