// Backward of the MoE expert layer in the BF16-backward mode: the gather of
// the rows into the padded grouped layout and the reduction of the routing
// weights' gradient.  The GEMMs are in gemm_bf16.cu, the dx sum reuses the
// slot-ordered combine.
//
// The pages time "NVFP4 forward, BF16 backward" (www.aib.vote "miniTE
// report, NVFP4 RL stability", paragraph 1) without formulas; this follows
// the plain reading: the exact gradient of the unquantized layer on its BF16
// operands, the forward's quantizers treated as the identity, the routing
// choice not differentiated and the routing weights differentiated.
#include "common.cuh"
#include "internal.h"

namespace nvfp4moe {

namespace {

constexpr int kGatherWarps = 8;

__device__ __forceinline__ int find_group_dev(const int32_t *padded, int E, int64_t row) {
  int lo = 0, hi = E;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if ((int64_t)__ldg(padded + mid) <= row) lo = mid; else hi = mid;
  }
  return lo;
}

// One warp per padded row p < padded_offsets[E]: the row's token t (from the
// permutation) gives x_rows[p] = x[t], dy_rows[p] = dy[t], w_rows[p] =
// topk_w[t][j]; padding rows get zeros.  ones[r] = 1 for every routed row.
// dy / dy_rows, w_rows and ones are optional (the W4A16 / W4A8 forward
// gathers x alone); with mxfp8_x the x rows are MXFP8 quantize-dequantized
// (W4A8), each of the token's k rows from the same values.
__global__ void __launch_bounds__(kGatherWarps * 32) k_bwd_gather(const BwdGatherParams p) {
  const int lane = threadIdx.x & 31;
  const int64_t row = (int64_t)blockIdx.x * kGatherWarps + (threadIdx.x >> 5);
  const int64_t R = p.T * p.k;
  if (p.ones != nullptr)
    for (int64_t r = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; r < R; r += (int64_t)gridDim.x * blockDim.x)
      p.ones[r] = 1.0f;
  int64_t used = __ldg(p.padded_offsets + p.E);
  if (used > p.rows_cap) used = p.rows_cap;
  if (row >= used) return;
  const int e = find_group_dev(p.padded_offsets, p.E, row);
  const int64_t rel = row - __ldg(p.padded_offsets + e);
  const int64_t cnt = (int64_t)__ldg(p.offsets + e + 1) - __ldg(p.offsets + e);
  int64_t t = -1;
  float w = 0.0f;
  if (rel < cnt) {
    const int64_t slot = __ldg(p.perm + __ldg(p.offsets + e) + rel);
    if (slot >= 0 && slot < R) {
      t = slot / p.k;
      w = __ldg(p.topk_w + slot);
    }
  }
  const int64_t hv = p.H >> 3;   // uint4 per row
  uint4 *xo = static_cast<uint4 *>(p.x_rows) + row * hv;
  const uint4 z = make_uint4(0, 0, 0, 0);
  const uint4 *xs = static_cast<const uint4 *>(p.x) + (t >= 0 ? t : 0) * hv;
  if (p.mxfp8_x) {
    // one 32-element MXFP8 block (four 16-byte chunks) per lane and step
    for (int64_t b = lane; b < hv / 4; b += 32) {
      if (t < 0) {
#pragma unroll
        for (int q = 0; q < 4; ++q) xo[4 * b + q] = z;
        continue;
      }
      float v[32];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint4 u = __ldg(xs + 4 * b + q);
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          v[8 * q + 2 * i] = bf16_lo(w[i]);
          v[8 * q + 2 * i + 1] = bf16_hi(w[i]);
        }
      }
      uint32_t o[16];
      mxfp8_qdq32(v, o);
#pragma unroll
      for (int q = 0; q < 4; ++q) xo[4 * b + q] = make_uint4(o[4 * q], o[4 * q + 1], o[4 * q + 2], o[4 * q + 3]);
    }
  } else {
    for (int64_t c = lane; c < hv; c += 32) xo[c] = t >= 0 ? __ldg(xs + c) : z;
  }
  if (p.dy_rows != nullptr) {
    uint4 *dyo = static_cast<uint4 *>(p.dy_rows) + row * hv;
    const uint4 *dys = static_cast<const uint4 *>(p.dy) + (t >= 0 ? t : 0) * hv;
    for (int64_t c = lane; c < hv; c += 32) dyo[c] = t >= 0 ? __ldg(dys + c) : z;
  }
  if (lane == 0 && p.w_rows != nullptr) p.w_rows[row] = w;
}

// dw[t][j] = sum over the row's partials (I/128 of them, in column order) of
// <dh', h>: the gradient of the routing weight, <dy[t], D[t][j]>.
__global__ void k_bwd_dw(const float *__restrict__ dw_part, int64_t nparts, const int32_t *__restrict__ inv_perm,
                         const int32_t *__restrict__ topk_idx, const int32_t *__restrict__ offsets,
                         const int32_t *__restrict__ padded, int64_t T, int k, int E, float *__restrict__ dw) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= T * k) return;
  const int e = __ldg(topk_idx + i);
  const int32_t r = __ldg(inv_perm + i);
  float s = 0.0f;
  if (e >= 0 && e < E && r >= 0) {
    const int64_t prow = (int64_t)r - __ldg(offsets + e) + __ldg(padded + e);
    for (int64_t c = 0; c < nparts; ++c) s += __ldg(dw_part + prow * nparts + c);
  }
  dw[i] = s;
}

}  // namespace

cudaError_t launch_bwd_gather(const BwdGatherParams &p, cudaStream_t s) {
  if (p.rows_cap <= 0) return cudaSuccess;
  const int64_t blocks = (p.rows_cap + kGatherWarps - 1) / kGatherWarps;
  k_bwd_gather<<<(unsigned)blocks, kGatherWarps * 32, 0, s>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_bwd_dw(const float *dw_part, int64_t nparts, const int32_t *inv_perm, const int32_t *topk_idx,
                          const int32_t *offsets, const int32_t *padded_offsets, int64_t T, int k, int E,
                          float *dw, cudaStream_t s) {
  const int64_t n = T * k;
  if (n <= 0) return cudaSuccess;
  k_bwd_dw<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(dw_part, nparts, inv_perm, topk_idx, offsets, padded_offsets,
                                                       T, k, E, dw);
  return cudaGetLastError();
}

}  // namespace nvfp4moe
