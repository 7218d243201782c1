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

// Token-major: warp w < T takes token t = w, reads its x (and dy) row once
// and writes it to the token's k rows of the padded grouped layout (the
// compact row inv_perm[t][j] of expert e sits at padded row inv_perm -
// offsets[e] + padded_offsets[e]), with w_rows = topk_w[t][j].  The warps of
// the blocks after the token blocks zero the padding rows: warp (e, j) the
// j-th padding row of expert e (at most 127 per expert).  ones[r] = 1 for
// every routed row.  dy / dy_rows, w_rows and ones are optional (the W4A16 /
// W4A8 forward gathers x alone); with mxfp8_x the x rows are MXFP8
// quantize-dequantized (W4A8), once per token for all its rows.
__global__ void __launch_bounds__(kGatherWarps * 32) k_bwd_gather(const BwdGatherParams p, int64_t tok_blocks) {
  const int lane = threadIdx.x & 31;
  const int64_t gw = (int64_t)blockIdx.x * kGatherWarps + (threadIdx.x >> 5);
  const int64_t R = p.T * p.k;
  if (p.ones != nullptr)
    for (int64_t r = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; r < R; r += (int64_t)gridDim.x * blockDim.x)
      p.ones[r] = 1.0f;
  const int64_t hv = p.H >> 3;   // uint4 per row
  const uint4 z = make_uint4(0, 0, 0, 0);
  if ((int64_t)blockIdx.x >= tok_blocks) {
    // ---- padding rows: zero rows and weights
    const int64_t pw = gw - tok_blocks * kGatherWarps;
    const int e = (int)(pw / 128), j = (int)(pw % 128);
    if (e >= p.E) return;
    const int64_t cnt = (int64_t)__ldg(p.offsets + e + 1) - __ldg(p.offsets + e);
    const int64_t row = (int64_t)__ldg(p.padded_offsets + e) + cnt + j;
    int64_t end = __ldg(p.padded_offsets + e + 1);
    if (end > p.rows_cap) end = p.rows_cap;
    if (row >= end) return;
    uint4 *xo = static_cast<uint4 *>(p.x_rows) + row * hv;
    for (int64_t c = lane; c < hv; c += 32) xo[c] = z;
    if (p.dy_rows != nullptr) {
      uint4 *dyo = static_cast<uint4 *>(p.dy_rows) + row * hv;
      for (int64_t c = lane; c < hv; c += 32) dyo[c] = z;
    }
    if (lane == 0 && p.w_rows != nullptr) p.w_rows[row] = 0.0f;
    return;
  }
  // ---- a token: its k destination rows (lane j holds row j)
  const int64_t t = gw;
  if (t >= p.T) return;
  int64_t my_row = -1;
  if (lane < p.k) {
    const int64_t slot = t * p.k + lane;
    const int e = __ldg(p.topk_idx + slot);
    const int32_t r = __ldg(p.inv_perm + slot);
    if (e >= 0 && e < p.E && r >= 0) {
      const int64_t prow = (int64_t)r - __ldg(p.offsets + e) + __ldg(p.padded_offsets + e);
      if (prow >= 0 && prow < p.rows_cap) my_row = prow;
    }
    if (my_row >= 0 && p.w_rows != nullptr) p.w_rows[my_row] = __ldg(p.topk_w + slot);
  }
  // the row's 16-byte chunks c = c0 + 32 i + lane, eight per lane in flight,
  // then stored to every destination row
  constexpr int kBatch = 8;
  auto scatter = [&](const uint4 *src, void *dst_base) {
    uint4 *dst = static_cast<uint4 *>(dst_base);
    for (int64_t c0 = 0; c0 < hv; c0 += 32 * kBatch) {
      uint4 v[kBatch];
#pragma unroll
      for (int i = 0; i < kBatch; ++i) {
        const int64_t c = c0 + 32 * i + lane;
        v[i] = c < hv ? __ldg(src + c) : z;
      }
      for (int j = 0; j < p.k; ++j) {
        const int64_t row = __shfl_sync(0xffffffffu, my_row, j);
        if (row < 0) continue;
#pragma unroll
        for (int i = 0; i < kBatch; ++i) {
          const int64_t c = c0 + 32 * i + lane;
          if (c < hv) dst[row * hv + c] = v[i];
        }
      }
    }
  };
  const uint4 *xs = static_cast<const uint4 *>(p.x) + t * hv;
  if (p.mxfp8_x) {
    // one 32-element MXFP8 block (four 16-byte chunks) per lane and step
    uint4 *xo = static_cast<uint4 *>(p.x_rows);
    const int64_t nb = hv / 4;
    for (int64_t b0 = 0; b0 < nb; b0 += 32) {   // warp-uniform trip count (the shuffles below)
      const int64_t b = b0 + lane;
      const bool live = b < nb;
      float v[32];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint4 u = live ? __ldg(xs + 4 * b + q) : z;
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          v[8 * q + 2 * i] = bf16_lo(w[i]);
          v[8 * q + 2 * i + 1] = bf16_hi(w[i]);
        }
      }
      uint32_t o[16];
      mxfp8_qdq32(v, o);
      for (int j = 0; j < p.k; ++j) {
        const int64_t row = __shfl_sync(0xffffffffu, my_row, j);
        if (row < 0 || !live) continue;
#pragma unroll
        for (int q = 0; q < 4; ++q)
          xo[row * hv + 4 * b + q] = make_uint4(o[4 * q], o[4 * q + 1], o[4 * q + 2], o[4 * q + 3]);
      }
    }
  } else {
    scatter(xs, p.x_rows);
  }
  if (p.dy_rows != nullptr) scatter(static_cast<const uint4 *>(p.dy) + t * hv, p.dy_rows);
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
  if (p.rows_cap <= 0 || p.T <= 0) return cudaSuccess;
  if (p.inv_perm == nullptr || (p.H / 8) % 4 != 0) return cudaErrorInvalidValue;
  const int64_t tok_blocks = (p.T + kGatherWarps - 1) / kGatherWarps;
  const int64_t pad_blocks = ((int64_t)p.E * 128 + kGatherWarps - 1) / kGatherWarps;
  k_bwd_gather<<<(unsigned)(tok_blocks + pad_blocks), kGatherWarps * 32, 0, s>>>(p, tok_blocks);
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
