// Persistent block-scaled NVFP4 grouped GEMM over the experts (sm_100a).
//
// The grouped matrix multiplication of the token-wise NVFP4 path
// (www.aib.vote "miniTE report, NVFP4 RL stability", paragraph 4) and the
// grouped GEMMs of the MoE learner (news.hamidun.com, "diagnostics, alignment
// and fast kernels").  One launch covers every expert; the group sizes are
// read on the device from padded_offsets, so the host never synchronizes.
//
// Design (B200):
//   * tile 128 x 256 x 256 (M x N x K elements); A rows come from the padded
//     grouped layout, where every expert's group starts on a 128-row boundary,
//     so a tile never straddles two experts.
//   * warp 0, one thread: TMA producer.  Per K-step it loads the A tile
//     (16 KB) and the B tile (32 KB) with 128-byte-swizzled tensor copies and
//     the scale factors (2 KB + 4 KB, already stored in the MMA atom layout)
//     with plain bulk copies, into a 4-stage shared-memory ring.
//   * warp 1, one thread: copies the scale factors into TMEM (tcgen05.cp) and
//     issues tcgen05.mma kind::mxf4nvf4 with 16-element UE4M3 scale blocks,
//     FP32 accumulators in TMEM (256 columns), then commits the stage back to
//     the producer and, after the last K-step, the accumulator to the epilogue.
//   * warps 2-9: epilogue.  Each warp reads its 32-lane quarter of the
//     accumulator (half of the columns), releases TMEM at once so the next
//     tile's MMAs overlap the rest of the epilogue, scales by
//     S_dec_a(row) * S_dec_w(expert) and stores BF16 / FP32 rows, or applies
//     SwiGLU (gate and up columns sit in the two 128-column halves of the
//     tile), stores h in BF16 and max-reduces |h| for the requantization.
//   * persistent grid: one CTA per SM walks tiles t = blockIdx.x, +gridDim.x,
//     ...; t enumerates (m-tile, n-tile) with n fastest so CTAs working at the
//     same time share A tiles and expert weights through L2.
//   * every wait is bounded (common.cuh); a timeout records an error word and
//     the CTA drains its in-flight copies and MMAs before freeing TMEM.
#include <cudaTypedefs.h>

#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace nvfp4moe {

namespace {

constexpr int BM = 128, BN = 256, BK = 256;
constexpr int kStages = 4;
constexpr int kABytes = BM * BK / 2;      // 16384
constexpr int kBBytes = BN * BK / 2;      // 32768
constexpr int kSfaBytes = BM * BK / 16;   // 2048: four 512-byte atoms
constexpr int kSfbBytes = BN * BK / 16;   // 4096: two 128-row halves x four atoms
constexpr int kStageBytes = kABytes + kBBytes + kSfaBytes + kSfbBytes;
constexpr int kEpiWarps = 8;
constexpr int kThreads = 32 * (2 + kEpiWarps);
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kAccCol = 0;       // 256 FP32 accumulator columns
constexpr uint32_t kSfaCol = 256;     // 4 K-blocks x 4 columns
constexpr uint32_t kSfbCol = 272;     // 4 K-blocks x 8 columns
constexpr size_t kSmemBytes = (size_t)kStages * kStageBytes + 1024 + 256;

// Instruction descriptor, kind::mxf4nvf4: A and B E2M1 (format 1), K-major,
// UE4M3 scales (bit 23 = 0), N >> 3 at bit 17, M >> 4 at bit 24, dense, K = 64.
constexpr uint32_t kIdesc = (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
                            ((uint32_t)(BM >> 4) << 24);

struct __align__(64) KParams {
  CUtensorMap tmap_a;
  CUtensorMap tmap_b;
  GemmArgs a;
};

__device__ __forceinline__ int find_group(const int32_t *padded, int E, int64_t row) {
  int lo = 0, hi = E;  // padded[lo] <= row < padded[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if ((int64_t)__ldg(padded + mid) <= row) lo = mid; else hi = mid;
  }
  return lo;
}

__device__ __forceinline__ float fmax_abs_bf16(float m, uint32_t packed) {
  return fmaxf(m, fmaxf(fabsf(bf16_lo(packed)), fabsf(bf16_hi(packed))));
}

__global__ void __launch_bounds__(kThreads, 1) k_grouped_gemm(const __grid_constant__ KParams P) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + (size_t)kStages * kStageBytes);
  uint64_t *empty = full + kStages;
  uint64_t *acc_full = empty + kStages;
  uint64_t *acc_empty = acc_full + 1;
  uint64_t *drain = acc_empty + 1;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
  int *never = reinterpret_cast<int *>(tmem_slot + 2);   // an abort flag nothing raises

  const GemmArgs &a = P.a;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, kEpiWarps);
    mbar_init(drain, 1);
    *abort_flag = 0;
    *never = 0;
    fence_mbarrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensor_map(&P.tmap_a);
    prefetch_tensor_map(&P.tmap_b);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  const int n_tiles = (int)(a.N / BN);
  const int kt_count = (int)(a.K / BK);
  // never walk past the rows the caller allocated, whatever the offsets say
  int64_t rows_used = __ldg(a.padded_offsets + a.E);
  if (rows_used > a.rows_cap) rows_used = a.rows_cap;
  if (rows_used < 0) rows_used = 0;
  const int64_t total = (rows_used / BM) * n_tiles;
  const int64_t rows_total = __ldg(a.offsets + a.E);
  const int64_t k_atoms = a.K >> 6;      // 512-byte scale atoms per 128 rows

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t stage = 0, phase = 0;
      uint32_t last_phase[kStages];
      bool used[kStages];
      for (int s = 0; s < kStages; ++s) { used[s] = false; last_phase[s] = 0; }
      bool ok = true;
      for (int64_t t = blockIdx.x; t < total && ok; t += gridDim.x) {
        const int64_t mt = t / n_tiles;
        const int nt = (int)(t - mt * n_tiles);
        const int64_t row0 = mt * BM;
        const int e = find_group(a.padded_offsets, a.E, row0);
        const int32_t wrow0 = (int32_t)((int64_t)e * a.N + (int64_t)nt * BN);
        const uint8_t *sfa_src = a.sf_a + mt * k_atoms * 512;
        const uint8_t *sfb_src0 = a.sf_w + ((int64_t)e * (a.N >> 7) + 2 * nt) * k_atoms * 512;
        const uint8_t *sfb_src1 = sfb_src0 + k_atoms * 512;
        for (int kt = 0; kt < kt_count; ++kt) {
          if (!mbar_wait_bounded(&empty[stage], phase ^ 1u, abort_flag, a.err, 100)) { ok = false; break; }
          uint8_t *sb = smem + (size_t)stage * kStageBytes;
          mbar_arrive_expect_tx(&full[stage], kStageBytes);
          tma_load_2d(sb, &P.tmap_a, kt * (BK / 2), (int32_t)row0, &full[stage]);
          tma_load_2d(sb + kABytes, &P.tmap_b, kt * (BK / 2), wrow0, &full[stage]);
          bulk_load(sb + kABytes + kBBytes, sfa_src + (int64_t)kt * kSfaBytes, kSfaBytes, &full[stage]);
          bulk_load(sb + kABytes + kBBytes + kSfaBytes, sfb_src0 + (int64_t)kt * 2048, 2048, &full[stage]);
          bulk_load(sb + kABytes + kBBytes + kSfaBytes + 2048, sfb_src1 + (int64_t)kt * 2048, 2048,
                    &full[stage]);
          used[stage] = true;
          last_phase[stage] = phase;
          if (++stage == kStages) { stage = 0; phase ^= 1u; }
        }
      }
      // drain: every copy issued must have landed before the CTA exits
      for (int s = 0; s < kStages; ++s)
        if (used[s]) mbar_wait_bounded(&full[s], last_phase[s], never, a.err, 101);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------- MMA
    if (lane == 0) {
      uint32_t stage = 0, phase = 0, acc_phase = 0;
      bool ok = true;
      for (int64_t t = blockIdx.x; t < total && ok; t += gridDim.x) {
        if (!mbar_wait_bounded(acc_empty, acc_phase ^ 1u, abort_flag, a.err, 200)) break;
        tc_fence_after();
        for (int kt = 0; kt < kt_count; ++kt) {
          if (!mbar_wait_bounded(&full[stage], phase, abort_flag, a.err, 201)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smem + (size_t)stage * kStageBytes);
          const uint32_t b_addr = a_addr + kABytes;
          const uint32_t sfa_addr = b_addr + kBBytes;
          const uint32_t sfb_addr = sfa_addr + kSfaBytes;
#pragma unroll
          for (int kb = 0; kb < 4; ++kb) {
            tmem_cp_sf_atom(tmem + kSfaCol + 4 * kb, smem_desc(sfa_addr + kb * 512, 0, 128, 0));
            tmem_cp_sf_atom(tmem + kSfbCol + 8 * kb, smem_desc(sfb_addr + kb * 512, 0, 128, 0));
            tmem_cp_sf_atom(tmem + kSfbCol + 8 * kb + 4,
                            smem_desc(sfb_addr + 2048 + kb * 512, 0, 128, 0));
          }
#pragma unroll
          for (int kb = 0; kb < 4; ++kb) {
            const uint64_t adesc = smem_desc(a_addr + kb * 32, 16, 1024, 2);
            const uint64_t bdesc = smem_desc(b_addr + kb * 32, 16, 1024, 2);
            mma_nvfp4(tmem + kAccCol, adesc, bdesc, kIdesc, tmem + kSfaCol + 4 * kb,
                      tmem + kSfbCol + 8 * kb, (kt | kb) != 0 ? 1u : 0u);
          }
          tc_commit(&empty[stage]);
          if (++stage == kStages) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        tc_commit(acc_full);
        acc_phase ^= 1u;
      }
      // drain: all MMAs and TMEM copies this thread issued have completed
      tc_commit(drain);
      mbar_wait_bounded(drain, 0, never, a.err, 202);
    }
  } else {
    // -------------------------------------------------------- epilogue
    const int ew = warp - 2;
    const int quad = warp & 3;              // TMEM lanes this warp may read
    const int half = ew >> 2;               // which half of the columns
    const int rit = quad * 32 + lane;       // row inside the tile
    const uint32_t tlane = tmem + ((uint32_t)(quad * 32) << 16);
    uint32_t acc_phase = 0;
    for (int64_t t = blockIdx.x; t < total; t += gridDim.x) {
      const int64_t mt = t / n_tiles;
      const int nt = (int)(t - mt * n_tiles);
      const int64_t row0 = mt * BM;
      const int e = find_group(a.padded_offsets, a.E, row0);
      const int64_t g_pad = __ldg(a.padded_offsets + e);
      const int64_t g_off = __ldg(a.offsets + e);
      const int64_t g_cnt = (int64_t)__ldg(a.offsets + e + 1) - g_off;
      const int64_t rel = row0 - g_pad + rit;
      const bool valid = rel < g_cnt && g_off + rel < rows_total;
      const int64_t prow = row0 + rit;

      if (!mbar_wait_bounded(acc_full, acc_phase, abort_flag, a.err, 300)) break;
      tc_fence_after();
      uint32_t v[4][32];
      if (a.epilogue == kEpiSwiGLU) {
        tmem_ld_32cols(tlane + kAccCol + half * 64, v[0]);
        tmem_ld_32cols(tlane + kAccCol + half * 64 + 32, v[1]);
        tmem_ld_32cols(tlane + kAccCol + 128 + half * 64, v[2]);
        tmem_ld_32cols(tlane + kAccCol + 128 + half * 64 + 32, v[3]);
      } else {
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld_32cols(tlane + kAccCol + half * 128 + c * 32, v[c]);
      }
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acc_empty);
      acc_phase ^= 1u;

      const float sa = valid ? __ldg(a.s_dec_a + (a.s_dec_a_rows ? prow : 0)) : 0.0f;
      const float scale = __fmul_rn(sa, __ldg(a.s_dec_w + e));
      if (a.epilogue == kEpiSwiGLU) {
        const int64_t hcols = a.N >> 1;
        uint32_t hp[32];
        float m = 0.0f;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
#pragma unroll
          for (int i = 0; i < 32; i += 2) {
            float hh[2];
#pragma unroll
            for (int q = 0; q < 2; ++q) {
              const float g = __fmul_rn(__uint_as_float(v[c][i + q]), scale);
              const float u = __fmul_rn(__uint_as_float(v[c + 2][i + q]), scale);
              const float sg = __fdiv_rn(g, __fadd_rn(1.0f, expf(-g)));
              hh[q] = __fmul_rn(sg, u);
            }
            hp[c * 16 + i / 2] = pack_bf16x2(hh[0], hh[1]);
          }
        }
#pragma unroll
        for (int i = 0; i < 32; ++i) m = fmax_abs_bf16(m, hp[i]);
        if (valid) {
          uint4 *dst = reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(a.out_bf16) +
                                                 prow * hcols + (int64_t)nt * 128 + half * 64);
#pragma unroll
          for (int i = 0; i < 8; ++i)
            dst[i] = make_uint4(hp[4 * i], hp[4 * i + 1], hp[4 * i + 2], hp[4 * i + 3]);
        }
        if (a.amax_h != nullptr) {
          if (a.amax_h_rows) {
            if (valid) atomicMax(reinterpret_cast<unsigned int *>(a.amax_h + prow), __float_as_uint(m));
          } else {
            float mm = valid ? m : 0.0f;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) mm = fmaxf(mm, __shfl_xor_sync(0xffffffffu, mm, o));
            if (lane == 0 && mm > 0.0f)
              atomicMax(reinterpret_cast<unsigned int *>(a.amax_h), __float_as_uint(mm));
          }
        }
      } else if (valid) {
        const int64_t orow = a.out_padded ? prow : g_off + rel;
        const int64_t col0 = (int64_t)nt * BN + half * 128;
        if (a.out_bf16 != nullptr) {
          uint4 *dst = reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(a.out_bf16) +
                                                 orow * a.N + col0);
#pragma unroll
          for (int c = 0; c < 4; ++c) {
#pragma unroll
            for (int i = 0; i < 32; i += 8) {
              uint4 o;
              o.x = pack_bf16x2(__fmul_rn(__uint_as_float(v[c][i + 0]), scale),
                                __fmul_rn(__uint_as_float(v[c][i + 1]), scale));
              o.y = pack_bf16x2(__fmul_rn(__uint_as_float(v[c][i + 2]), scale),
                                __fmul_rn(__uint_as_float(v[c][i + 3]), scale));
              o.z = pack_bf16x2(__fmul_rn(__uint_as_float(v[c][i + 4]), scale),
                                __fmul_rn(__uint_as_float(v[c][i + 5]), scale));
              o.w = pack_bf16x2(__fmul_rn(__uint_as_float(v[c][i + 6]), scale),
                                __fmul_rn(__uint_as_float(v[c][i + 7]), scale));
              dst[c * 4 + i / 8] = o;
            }
          }
        }
        if (a.out_f32 != nullptr) {
          float4 *dst = reinterpret_cast<float4 *>(a.out_f32 + orow * a.N + col0);
#pragma unroll
          for (int c = 0; c < 4; ++c) {
#pragma unroll
            for (int i = 0; i < 32; i += 4) {
              dst[c * 8 + i / 4] = make_float4(__fmul_rn(__uint_as_float(v[c][i]), scale),
                                               __fmul_rn(__uint_as_float(v[c][i + 1]), scale),
                                               __fmul_rn(__uint_as_float(v[c][i + 2]), scale),
                                               __fmul_rn(__uint_as_float(v[c][i + 3]), scale));
            }
          }
        }
      }
    }
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

bool encode_2d_u8(CUtensorMap *map, const void *base, uint64_t inner_bytes, uint64_t rows,
                  uint32_t box_inner, uint32_t box_rows) {
  auto fn = get_encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[2] = {inner_bytes, rows};
  const cuuint64_t strides[1] = {inner_bytes};
  const cuuint32_t box[2] = {box_inner, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), dims, strides,
                        box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace

cudaError_t launch_grouped_gemm(const GemmArgs &a, cudaStream_t s) {
  if (a.rows_cap <= 0) return cudaSuccess;
  static thread_local int configured_device = -1;
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (configured_device != dev) {
    err = cudaFuncSetAttribute(k_grouped_gemm, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)kSmemBytes);
    if (err != cudaSuccess) return err;
    configured_device = dev;
  }
  KParams P;
  P.a = a;
  if (!encode_2d_u8(&P.tmap_a, a.q_a, (uint64_t)(a.K / 2), (uint64_t)a.rows_cap, BK / 2, BM))
    return cudaErrorInvalidValue;
  if (!encode_2d_u8(&P.tmap_b, a.q_w, (uint64_t)(a.K / 2), (uint64_t)(a.E * a.N), BK / 2, BN))
    return cudaErrorInvalidValue;
  const int64_t max_tiles = (a.rows_cap / BM) * (a.N / BN);
  int64_t grid = num_sms();
  if (grid > max_tiles) grid = max_tiles;
  if (grid < 1) grid = 1;
  k_grouped_gemm<<<(unsigned)grid, kThreads, kSmemBytes, s>>>(P);
  return cudaGetLastError();
}

}  // namespace nvfp4moe
