// NVFP4 quantizer kernels: amax reduction and the row quantizer.
//
// The token-wise NVFP4 path (www.aib.vote "miniTE report, NVFP4 RL
// stability", paragraph 4): every token row is quantized once -- its amax
// computed once and reused for all of its copies -- and written straight into
// the contiguous per-expert layout the grouped GEMM reads.
//
// One warp owns one row.  Lane l handles the 16-element blocks l, l+32, ...;
// a block is 32 contiguous bytes of BF16, so a warp reads 1 KB per step with
// 128-bit coalesced loads, and writes 256 contiguous bytes of codes.  The
// per-row amax is a warp shuffle reduction; rows of up to 4096 elements are
// loaded into registers up front, before the amax is known.
//
// Arithmetic per block (one binary32 operation each, round to nearest even):
//   bamax = max|x|, t = (bamax / 6) * S_enc, sf = UE4M3(t),
//   r = S_enc / sf, code_i = E2M1(x_i * r); a block with sf == 0 is all +0.
#include "common.cuh"
#include "internal.h"

namespace nvfp4moe {

namespace {

constexpr int kQuantWarps = 8;     // rows per 256-thread block

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// max |x| of 8 BF16 values on packed pairs (exact: a max of BF16 values)
__device__ __forceinline__ float abs_max8(uint4 v) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  __nv_bfloat162 m = __habs2(*reinterpret_cast<const __nv_bfloat162 *>(&w[0]));
#pragma unroll
  for (int i = 1; i < 4; ++i) m = __hmax2(m, __habs2(*reinterpret_cast<const __nv_bfloat162 *>(&w[i])));
  return fmaxf(__low2float(m), __high2float(m));
}

// Byte offset of scale (row, block b) in the given SfLayout.
__device__ __forceinline__ int64_t sf_offset(int layout, int64_t row, int64_t b, int64_t K, int64_t rows_cap) {
  if (layout == kSfMma) return sf_mma_offset(row, b, K);
  if (layout == kSfKStep) return ((b >> 4) * rows_cap + row) * 16 + (b & 15);
  return row * (K >> 4) + b;
}

// amax of `nseg` segments of seg_len BF16 each; out[seg] must be 0 beforehand
// (max of non-negative floats = max of their bit patterns as unsigned).
__global__ void k_amax(const uint4 *__restrict__ x, int64_t seg_vec, float *__restrict__ out) {
  const int64_t seg = blockIdx.y;
  const uint4 *base = x + seg * seg_vec;
  float m = 0.0f;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < seg_vec;
       i += (int64_t)gridDim.x * blockDim.x) {
    m = fmaxf(m, abs_max8(__ldg(base + i)));
  }
  m = warp_max(m);
  __shared__ float red[32];
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  if (l == 0) red[w] = m;
  __syncthreads();
  if (w == 0) {
    m = l < (int)(blockDim.x >> 5) ? red[l] : 0.0f;
    m = warp_max(m);
    if (l == 0 && m > 0.0f) atomicMax(reinterpret_cast<unsigned int *>(out + seg), __float_as_uint(m));
  }
}

// NB: 16-element blocks per lane held in registers (0 = re-read).
// KD > 0: at most KD destination rows whose byte offsets fit 32 bits, kept in
// registers for the whole row; KD == 0: any number, looked up per store.
template <int NB, int KD>
__global__ void __launch_bounds__(kQuantWarps * 32) k_quant(const QuantParams p) {
  const int lane = threadIdx.x & 31;
  const int64_t task = (int64_t)blockIdx.x * kQuantWarps + (threadIdx.x >> 5);
  if (task >= p.tasks) return;
  const int64_t K = p.K;
  const int64_t nblk = K >> 4;
  const __nv_bfloat16 *xb = static_cast<const __nv_bfloat16 *>(p.x);

  // ---- source row (plain, scatter, weights: the task's own row) ------------
  int64_t my_dest = -1;          // lane j < ndest holds destination j
  int ndest = 1;
  int64_t amax_index = 0;
  int64_t expert = 0;
  const uint4 *src = reinterpret_cast<const uint4 *>(xb + task * K);

  // ---- load the row (registers when it fits) before anything that waits ---
  uint4 cache[NB > 0 ? NB : 1][2];
  if constexpr (NB > 0) {
#pragma unroll
    for (int c = 0; c < NB; ++c) {
      const int64_t b = (int64_t)c * 32 + lane;
      cache[c][0] = make_uint4(0, 0, 0, 0);
      cache[c][1] = cache[c][0];
      if (b < nblk) {
        cache[c][0] = __ldg(src + b * 2);
        cache[c][1] = __ldg(src + b * 2 + 1);
      }
    }
  }

  // ---- destination row(s), amax source ----------------------------------
  if (p.mode == kQuantPlain) {
    my_dest = task;
    amax_index = p.amax_rows ? task : 0;
  } else if (p.mode == kQuantScatter) {
    ndest = p.k;
    amax_index = p.amax_rows ? task : 0;
    if (lane < p.k) {
      const int64_t slot = task * p.k + lane;
      const int e = __ldg(p.topk_idx + slot);
      if (p.local_rank != nullptr) p.inv_perm_out[slot] = -1;   // overwritten below when valid
      if (e >= 0 && e < p.E) {
        int64_t r;
        if (p.local_rank != nullptr) {
          const int64_t blk = task / kRankTokens;
          const int32_t lr = __ldg(p.local_rank + slot);
          r = (int64_t)__ldg(p.offsets + e) + __ldg(p.block_base + blk * p.E + e) + lr;
          if (lr < 0 || r < 0 || r >= p.tasks * p.k) r = -1;
          if (r >= 0) {
            p.perm_out[r] = (int32_t)slot;
            p.inv_perm_out[slot] = (int32_t)r;
          }
        } else {
          r = __ldg(p.inv_perm + slot);
        }
        const int64_t pr = r < 0 ? -1 : r - __ldg(p.offsets + e) + __ldg(p.padded_offsets + e);
        if (pr >= 0 && pr < p.rows_cap) my_dest = pr;
      }
    }
  } else {  // kQuantWeights
    expert = task / p.N;
    const int64_t n = task - expert * p.N;
    int64_t nd = n;
    if (p.gate_up) {
      const int64_t half = p.N >> 1;
      const int64_t j = n < half ? n : n - half;
      nd = (j >> 7) * 256 + (n < half ? 0 : 128) + (j & 127);
    }
    my_dest = expert * p.N + nd;
    amax_index = expert;
  }

  // ---- amax ---------------------------------------------------------------
  float amax;
  if (p.compute_row_amax) {
    float m = 0.0f;
    if constexpr (NB > 0) {
#pragma unroll
      for (int c = 0; c < NB; ++c) m = fmaxf(m, fmaxf(abs_max8(cache[c][0]), abs_max8(cache[c][1])));
    } else {
      for (int64_t b = lane; b < nblk; b += 32) {
        m = fmaxf(m, fmaxf(abs_max8(__ldg(src + b * 2)), abs_max8(__ldg(src + b * 2 + 1))));
      }
    }
    amax = warp_max(m);
    if (p.amax_out != nullptr && lane == 0) p.amax_out[task] = amax;
  } else {
    amax = __ldg(p.amax_src + amax_index);
  }
  float s_enc, s_dec;
  global_scales(amax, s_enc, s_dec);

  // ---- per-destination bookkeeping --------------------------------------
  if (lane < ndest && my_dest >= 0) {
    if (p.s_dec_rows) p.s_dec[my_dest] = s_dec;
    if (p.zero_rows != nullptr) p.zero_rows[my_dest] = 0.0f;
  }
  if (!p.s_dec_rows && lane == 0) {
    if (p.mode == kQuantPlain && task == 0) p.s_dec[0] = s_dec;
    if (p.mode == kQuantWeights && (task - expert * p.N) == 0) p.s_dec[expert] = s_dec;
  }

  // ---- destination offsets (codes, scale row part) ------------------------
  uint32_t qoff[KD > 0 ? KD : 1], soff[KD > 0 ? KD : 1];
  bool dvalid[KD > 0 ? KD : 1];
  if constexpr (KD > 0) {
#pragma unroll
    for (int d = 0; d < KD; ++d) {
      const int64_t row = __shfl_sync(0xffffffffu, my_dest, d);
      dvalid[d] = d < ndest && row >= 0;
      const uint32_t r32 = dvalid[d] ? (uint32_t)row : 0u;
      qoff[d] = r32 * (uint32_t)(K >> 1);
      soff[d] = p.sf_layout == kSfMma ? ((r32 >> 7) * (uint32_t)(K >> 6) * 512u + (r32 & 31u) * 16u +
                                         ((r32 & 127u) >> 5) * 4u)
                : p.sf_layout == kSfKStep ? r32 * 16u
                                          : r32 * (uint32_t)nblk;
    }
  }

  // ---- encode ------------------------------------------------------------
  auto encode_chunk = [&](int64_t c, uint4 v0, uint4 v1) {
    const int64_t b = c * 32 + lane;
    const bool valid = b < nblk;
    const float bamax = fmaxf(abs_max8(v0), abs_max8(v1));
    const float t = __fmul_rn(__fdiv_rn(bamax, 6.0f), s_enc);
    const uint32_t sfc = cvt_ue4m3(t);
    uint2 codes = make_uint2(0, 0);
    if (sfc != 0) {
      const float r = __fdiv_rn(s_enc, ue4m3_value(sfc));
      const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
      float y[8];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        y[2 * i] = __fmul_rn(bf16_lo(w[i]), r);
        y[2 * i + 1] = __fmul_rn(bf16_hi(w[i]), r);
      }
      codes.x = cvt_e2m1x8(y);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        y[2 * i] = __fmul_rn(bf16_lo(w[4 + i]), r);
        y[2 * i + 1] = __fmul_rn(bf16_hi(w[4 + i]), r);
      }
      codes.y = cvt_e2m1x8(y);
    }
    // gather the four scales of blocks 4i..4i+3 into lane 4i
    const int base = lane & ~3;
    const uint32_t s0 = __shfl_sync(0xffffffffu, sfc, base);
    const uint32_t s1 = __shfl_sync(0xffffffffu, sfc, base + 1);
    const uint32_t s2 = __shfl_sync(0xffffffffu, sfc, base + 2);
    const uint32_t s3 = __shfl_sync(0xffffffffu, sfc, base + 3);
    const uint32_t sfw = s0 | (s1 << 8) | (s2 << 16) | (s3 << 24);
    if constexpr (KD > 0) {
      const uint32_t qb = (uint32_t)b * 8u;
      const uint32_t sb = p.sf_layout == kSfMma ? ((uint32_t)b >> 2) * 512u
                          : p.sf_layout == kSfKStep ? ((uint32_t)b >> 4) * (uint32_t)p.rows_cap * 16u + ((uint32_t)b & 15u)
                                                    : (uint32_t)b;
#pragma unroll
      for (int d = 0; d < KD; ++d) {
        if (!dvalid[d] || !valid) continue;
        *reinterpret_cast<uint2 *>(p.q + qoff[d] + qb) = codes;
        if ((lane & 3) == 0) *reinterpret_cast<uint32_t *>(p.sf + soff[d] + sb) = sfw;
      }
    } else {
      for (int d = 0; d < ndest; ++d) {
        const int64_t row = __shfl_sync(0xffffffffu, my_dest, d);
        if (row < 0 || !valid) continue;
        *reinterpret_cast<uint2 *>(p.q + row * (K >> 1) + b * 8) = codes;
        if ((lane & 3) == 0) {
          const int64_t off = sf_offset(p.sf_layout, row, b, K, p.rows_cap);
          *reinterpret_cast<uint32_t *>(p.sf + off) = sfw;
        }
      }
    }
  };

  const int64_t nchunks = (nblk + 31) >> 5;
  if constexpr (NB > 0) {
#pragma unroll
    for (int c = 0; c < NB; ++c)
      if (c < nchunks) encode_chunk(c, cache[c][0], cache[c][1]);
  } else {
    for (int64_t c = 0; c < nchunks; ++c) {
      const int64_t b = c * 32 + lane;
      uint4 v0 = make_uint4(0, 0, 0, 0), v1 = v0;
      if (b < nblk) {
        v0 = __ldg(src + b * 2);
        v1 = __ldg(src + b * 2 + 1);
      }
      encode_chunk(c, v0, v1);
    }
  }
}

// Requantization of the padded rows of h with the amax the GEMM epilogue
// reduced (amax reuse): thread per two consecutive 16-element blocks of a row
// (the row's global scales are then computed once for both), grid-stride over
// the padded rows [0, padded_offsets[E]) so no lane searches the group
// offsets.  A row whose amax is 0 -- a padding row (the route scan zeroes
// their amax) or an all-zero row -- gets zero codes, zero scales and S_dec = 1,
// exactly what quantizing a zero row gives, without reading h.  (r, b2) of a
// lane advance by the fixed stride, so the loop divides once.  At most 40
// registers, so that six CTAs (48 warps) stay resident per SM: on the
// Qwen3-30B-A3B-shaped layer 54 us, against 57 us at 44 registers (five CTAs)
// and 61 us with one block per thread.
__global__ void __launch_bounds__(256, 6) k_requant_blocks(const QuantParams p, uint32_t npair) {
  const int lane = threadIdx.x & 31;
  const int64_t K = p.K;
  int64_t rows = __ldg(p.padded_offsets + p.E);
  if (rows > p.rows_cap) rows = p.rows_cap;
  if (rows < 0) rows = 0;
  const uint32_t total = (uint32_t)rows * npair;
  const uint32_t stride = gridDim.x * blockDim.x;        // a multiple of 32
  const uint32_t step_r = stride / npair, step_b = stride - step_r * npair;
  uint32_t i = blockIdx.x * blockDim.x + threadIdx.x;
  uint32_t r = i / npair, b2 = i - r * npair;
  // warp-uniform trip count: the shuffle below needs every lane
  for (uint32_t base = i - lane; base < total; base += stride) {
    const bool valid = i < total;
    const float amax = valid ? __ldg(p.amax_src + (p.amax_rows ? r : 0)) : 0.0f;
    float s_dec = 1.0f;
    uint32_t sf2 = 0;                 // the two blocks' UE4M3 scales, block 2 b2 in the low byte
    uint4 codes = make_uint4(0, 0, 0, 0);
    if (amax > 0.0f) {
      const uint4 *src = reinterpret_cast<const uint4 *>(static_cast<const __nv_bfloat16 *>(p.x) +
                                                         (int64_t)r * K) + b2 * 4;
      uint4 v[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) v[j] = __ldg(src + j);
      float s_enc;
      global_scales(amax, s_enc, s_dec);
      uint32_t cw[4];
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        const uint32_t w[8] = {v[2 * q].x, v[2 * q].y, v[2 * q].z, v[2 * q].w,
                               v[2 * q + 1].x, v[2 * q + 1].y, v[2 * q + 1].z, v[2 * q + 1].w};
        // block amax on packed BF16 pairs (exact: a max of BF16 values)
        __nv_bfloat162 m2 = __habs2(*reinterpret_cast<const __nv_bfloat162 *>(&w[0]));
#pragma unroll
        for (int j = 1; j < 8; ++j) m2 = __hmax2(m2, __habs2(*reinterpret_cast<const __nv_bfloat162 *>(&w[j])));
        const float bamax = fmaxf(__low2float(m2), __high2float(m2));
        const uint32_t sfc = cvt_ue4m3(__fmul_rn(__fdiv_rn(bamax, 6.0f), s_enc));
        cw[2 * q] = cw[2 * q + 1] = 0;
        if (sfc != 0) {
          const float rr = __fdiv_rn(s_enc, ue4m3_value(sfc));
          float y[8];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            y[2 * j] = __fmul_rn(bf16_lo(w[j]), rr);
            y[2 * j + 1] = __fmul_rn(bf16_hi(w[j]), rr);
          }
          cw[2 * q] = cvt_e2m1x8(y);
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            y[2 * j] = __fmul_rn(bf16_lo(w[4 + j]), rr);
            y[2 * j + 1] = __fmul_rn(bf16_hi(w[4 + j]), rr);
          }
          cw[2 * q + 1] = cvt_e2m1x8(y);
        }
        sf2 |= sfc << (8 * q);
      }
      codes = make_uint4(cw[0], cw[1], cw[2], cw[3]);
    }
    // the four blocks 4m..4m+3 of a row sit in lanes 2j, 2j+1: a row's pairs
    // start at an even index (npair is even) and the stride and the warp
    // bases are multiples of 32
    const uint32_t sf_hi = __shfl_down_sync(0xffffffffu, sf2, 1);
    if (valid) {
      if (b2 == 0) p.s_dec[r] = s_dec;
      *reinterpret_cast<uint4 *>(p.q + (int64_t)r * (K >> 1) + (int64_t)b2 * 16) = codes;
      if ((lane & 1) == 0)
        *reinterpret_cast<uint32_t *>(p.sf + sf_offset(p.sf_layout, r, 2 * (int64_t)b2, K, p.rows_cap)) =
            sf2 | (sf_hi << 16);
    }
    i += stride;
    r += step_r;
    b2 += step_b;
    if (b2 >= npair) {
      b2 -= npair;
      ++r;
    }
  }
}

template <int NB>
cudaError_t launch_quant_nb(const QuantParams &p, cudaStream_t s) {
  const int64_t blocks = (p.tasks + kQuantWarps - 1) / kQuantWarps;
  // every mode writes rows below rows_cap; 32-bit byte offsets when they fit
  const int ndest = p.mode == kQuantScatter ? p.k : 1;
  const bool small = p.rows_cap * (p.K >> 1) < ((int64_t)1 << 31);
  if (small && ndest <= 1)
    k_quant<NB, 1><<<(unsigned)blocks, kQuantWarps * 32, 0, s>>>(p);
  else if (small && ndest <= 8)
    k_quant<NB, 8><<<(unsigned)blocks, kQuantWarps * 32, 0, s>>>(p);
  else
    k_quant<NB, 0><<<(unsigned)blocks, kQuantWarps * 32, 0, s>>>(p);
  return cudaGetLastError();
}

__global__ void k_encode_e2m1(const float *__restrict__ y, int64_t n, uint8_t *__restrict__ codes) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    float v[8] = {y[i], 0, 0, 0, 0, 0, 0, 0};
    codes[i] = (uint8_t)(cvt_e2m1x8(v) & 0xFu);
  }
}

__global__ void k_encode_ue4m3(const float *__restrict__ v, int64_t n, uint8_t *__restrict__ codes) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    codes[i] = (uint8_t)cvt_ue4m3(v[i]);
  }
}

}  // namespace

cudaError_t launch_amax(const void *x, int64_t seg_len, int64_t nseg, float *out, cudaStream_t s) {
  if (seg_len <= 0 || nseg <= 0) return cudaSuccess;
  const int64_t seg_vec = seg_len / 8;
  int64_t per_seg = (seg_vec + 255) / 256;
  const int64_t target = (int64_t)num_sms() * 4;
  int64_t bx = per_seg < target / nseg + 1 ? per_seg : target / nseg + 1;
  if (bx < 1) bx = 1;
  dim3 grid((unsigned)bx, (unsigned)nseg);
  k_amax<<<grid, 256, 0, s>>>(static_cast<const uint4 *>(x), seg_vec, out);
  return cudaGetLastError();
}

cudaError_t launch_quant(const QuantParams &p, cudaStream_t s) {
  if (p.tasks <= 0) return cudaSuccess;
  if (p.mode == kQuantRequant) {
    // h is requantized with the amax the GEMM epilogue reduced; there is no
    // requantization that computes its own amax
    if (p.compute_row_amax) return cudaErrorInvalidValue;
    // two 16-element blocks per thread; a row holds a multiple of four blocks
    if (p.K % 64 != 0) return cudaErrorInvalidValue;
    const uint32_t npair = (uint32_t)(p.K / 32);
    // every padded row below rows_cap, every pair of blocks; 32-bit indices
    if (p.rows_cap * (int64_t)npair >= ((int64_t)1 << 31)) return cudaErrorInvalidValue;
    int64_t blocks = (p.rows_cap * npair + 255) / 256;
    // 16 CTAs of 256 threads per SM, in waves of the six that fit (with one
    // block per thread, 16 per SM ran 4-5 us faster on the moe30b layer than
    // one resident wave of 8, and 4 per SM slower)
    const int64_t persistent = (int64_t)num_sms() * 16;
    if (blocks > persistent) blocks = persistent;
    if (blocks < 1) blocks = 1;
    k_requant_blocks<<<(unsigned)blocks, 256, 0, s>>>(p, npair);
    return cudaGetLastError();
  }
  const int64_t nb = (p.K + 511) / 512;   // 16-element blocks per lane
  if (nb <= 1) return launch_quant_nb<1>(p, s);
  if (nb <= 2) return launch_quant_nb<2>(p, s);
  if (nb <= 4) return launch_quant_nb<4>(p, s);
  if (nb <= 8) return launch_quant_nb<8>(p, s);
  return launch_quant_nb<0>(p, s);
}

cudaError_t launch_encode_e2m1(const float *y, int64_t n, uint8_t *codes, cudaStream_t s) {
  if (n <= 0) return cudaSuccess;
  int64_t blocks = (n + 255) / 256;
  if (blocks > 65535) blocks = 65535;
  k_encode_e2m1<<<(unsigned)blocks, 256, 0, s>>>(y, n, codes);
  return cudaGetLastError();
}

cudaError_t launch_encode_ue4m3(const float *v, int64_t n, uint8_t *codes, cudaStream_t s) {
  if (n <= 0) return cudaSuccess;
  int64_t blocks = (n + 255) / 256;
  if (blocks > 65535) blocks = 65535;
  k_encode_ue4m3<<<(unsigned)blocks, 256, 0, s>>>(v, n, codes);
  return cudaGetLastError();
}

}  // namespace nvfp4moe
