// Unpermute + top-k weighted combine: y[t] = BF16( sum_j w[t][j] * D[inv_perm[t][j]] ).
//
// The sum runs in FP32 in slot order j = 0..k-1 for every token, independent
// of how the tokens were batched or grouped -- the fixed reduction order the
// pages' strict-alignment mode needs (news.hamidun.com, "diagnostics,
// alignment and fast kernels": order of computation is part of the policy).
//
// One warp per token; each lane owns 8 consecutive BF16 columns per step
// (128-bit loads and stores), so a warp moves 512 contiguous bytes per row.
// For k <= 8 the k row loads of a step are all issued before the first
// multiply-add (the kernel is bound by HBM latency otherwise); the sum itself
// still runs in slot order.
#include "common.cuh"
#include "internal.h"

namespace nvfp4moe {

namespace {

constexpr int kCombineWarps = 8;
constexpr int kSlotsUnrolled = 8;   // top-k up to this many: all row loads in flight at once

// KU > 0: k <= KU, the k row loads of a column chunk are issued before the
// first multiply-add; KU == 0: any k, one row at a time.
template <int KU>
__global__ void __launch_bounds__(kCombineWarps * 32)
    k_combine(const uint4 *__restrict__ d, const int32_t *__restrict__ inv_perm,
              const float *__restrict__ w, int64_t T, int k, int64_t H, int64_t rows_cap,
              uint4 *__restrict__ y) {
  const int lane = threadIdx.x & 31;
  const int64_t t = (int64_t)blockIdx.x * kCombineWarps + (threadIdx.x >> 5);
  if (t >= T) return;
  const int64_t hv = H >> 3;                 // uint4 per row
  int32_t my_row = -1;
  float my_w = 0.0f;
  if (lane < k) {
    my_row = __ldg(inv_perm + t * k + lane);
    my_w = __ldg(w + t * k + lane);
  }
  if constexpr (KU > 0) {
    // row and weight of every slot in registers; an invalid routing entry adds nothing
    const uint4 *src[KU];
    float wj[KU];
    bool use[KU];
#pragma unroll
    for (int j = 0; j < KU; ++j) {
      const int64_t row = __shfl_sync(0xffffffffu, my_row, j);
      wj[j] = __shfl_sync(0xffffffffu, my_w, j);
      use[j] = j < k && row >= 0 && row < rows_cap;
      src[j] = d + (use[j] ? row : 0) * hv;
    }
    for (int64_t c = lane; c < hv; c += 32) {
      uint4 v[KU];
#pragma unroll
      for (int j = 0; j < KU; ++j) v[j] = use[j] ? __ldg(src[j] + c) : make_uint4(0, 0, 0, 0);
      float acc[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] = 0.0f;
#pragma unroll
      for (int j = 0; j < KU; ++j) {
        if (!use[j]) continue;
        const uint32_t u[4] = {v[j].x, v[j].y, v[j].z, v[j].w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          acc[2 * i] = __fmaf_rn(wj[j], bf16_lo(u[i]), acc[2 * i]);
          acc[2 * i + 1] = __fmaf_rn(wj[j], bf16_hi(u[i]), acc[2 * i + 1]);
        }
      }
      uint4 o;
      o.x = pack_bf16x2(acc[0], acc[1]);
      o.y = pack_bf16x2(acc[2], acc[3]);
      o.z = pack_bf16x2(acc[4], acc[5]);
      o.w = pack_bf16x2(acc[6], acc[7]);
      y[t * hv + c] = o;
    }
  } else {
    for (int64_t c = lane; c < hv; c += 32) {
      float acc[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] = 0.0f;
      for (int j = 0; j < k; ++j) {
        const int64_t row = __shfl_sync(0xffffffffu, my_row, j);
        const float wj = __shfl_sync(0xffffffffu, my_w, j);
        if (row < 0 || row >= rows_cap) continue;   // an invalid routing entry adds nothing
        const uint4 v = __ldg(d + row * hv + c);
        const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          acc[2 * i] = __fmaf_rn(wj, bf16_lo(u[i]), acc[2 * i]);
          acc[2 * i + 1] = __fmaf_rn(wj, bf16_hi(u[i]), acc[2 * i + 1]);
        }
      }
      uint4 o;
      o.x = pack_bf16x2(acc[0], acc[1]);
      o.y = pack_bf16x2(acc[2], acc[3]);
      o.z = pack_bf16x2(acc[4], acc[5]);
      o.w = pack_bf16x2(acc[6], acc[7]);
      y[t * hv + c] = o;
    }
  }
}

// y = BF16(acc), 8 values per thread (the non-strict combine's last step).
__global__ void k_f32_to_bf16(const float4 *__restrict__ src, int64_t n8, uint4 *__restrict__ dst) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n8; i += (int64_t)gridDim.x * blockDim.x) {
    const float4 a = __ldg(src + 2 * i), b = __ldg(src + 2 * i + 1);
    dst[i] = make_uint4(pack_bf16x2(a.x, a.y), pack_bf16x2(a.z, a.w), pack_bf16x2(b.x, b.y), pack_bf16x2(b.z, b.w));
  }
}

}  // namespace

cudaError_t launch_f32_to_bf16(const float *src, int64_t n, void *dst, cudaStream_t s) {
  if (n <= 0) return cudaSuccess;
  if (n % 8 != 0) return cudaErrorInvalidValue;
  int64_t blocks = (n / 8 + 255) / 256;
  const int64_t cap = (int64_t)num_sms() * 8;
  if (blocks > cap) blocks = cap;
  k_f32_to_bf16<<<(unsigned)blocks, 256, 0, s>>>(reinterpret_cast<const float4 *>(src), n / 8,
                                                  static_cast<uint4 *>(dst));
  return cudaGetLastError();
}

cudaError_t launch_combine(const void *d, const int32_t *inv_perm, const float *w, int64_t T, int k,
                           int64_t H, void *y, cudaStream_t s) {
  if (T <= 0) return cudaSuccess;
  const int64_t blocks = (T + kCombineWarps - 1) / kCombineWarps;
  if (k <= kSlotsUnrolled)
    k_combine<kSlotsUnrolled><<<(unsigned)blocks, kCombineWarps * 32, 0, s>>>(
        static_cast<const uint4 *>(d), inv_perm, w, T, k, H, T * k, static_cast<uint4 *>(y));
  else
    k_combine<0><<<(unsigned)blocks, kCombineWarps * 32, 0, s>>>(
        static_cast<const uint4 *>(d), inv_perm, w, T, k, H, T * k, static_cast<uint4 *>(y));
  return cudaGetLastError();
}

}  // namespace nvfp4moe
