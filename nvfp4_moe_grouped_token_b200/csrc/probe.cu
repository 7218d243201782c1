// Tensor-core throughput probe for the block-scaled FP4 MMA.
//
// Measures the roofline denominator of the grouped GEMM on the GPU at hand:
// one CTA per SM issues `iters` K-steps, each of 4 tcgen05.mma
// kind::mxf4nvf4 (M = 128, N = n, K = 64) on operands already resident in
// shared memory, optionally preceded by the tcgen05.cp scale-factor copies
// the GEMM issues per K-step.  No global memory is read; the operand bytes
// are whatever the CTA wrote into shared memory (zeros), so only timing is
// meaningful.  Each CTA records its elapsed SM cycles.  `mode` selects how
// the copies and MMAs are ordered (see the kernel).  Mode 12 also reads a
// 54 KB global buffer (the workspace past its first 256 bytes) with bulk
// copies, to measure how shared-memory fills interfere with the MMAs.
#include "common.cuh"
#include "internal.h"

namespace nvfp4moe {

namespace {

constexpr int kProbeOps = 16384 + 32768 + 2048 + 4096;   // operand + scale bytes
constexpr int kProbeLand = 55296;                         // landing zone for bulk copies
constexpr int kProbeSmem = kProbeOps + kProbeLand + 1024 + 64;

__global__ void __launch_bounds__(160, 1)
    k_mma_probe(int iters, int n, int sf_a_copies, int sf_b_copies, int mode, long long *cycles,
                int *err, const uint8_t *gsrc) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t *done = reinterpret_cast<uint64_t *>(smem + kProbeOps + kProbeLand);
  uint32_t *slot = reinterpret_cast<uint32_t *>(done + 1);
  int *never = reinterpret_cast<int *>(slot + 1);
  unsigned long long *span = reinterpret_cast<unsigned long long *>(slot + 4);   // [2]
  uint64_t *landed = reinterpret_cast<uint64_t *>(slot + 8);                      // [3]
  const int warp = threadIdx.x >> 5;
  for (int i = threadIdx.x; i < (16384 + 32768 + 2048 + 4096) / 16; i += blockDim.x)
    reinterpret_cast<uint4 *>(smem)[i] = make_uint4(0, 0, 0, 0);
  if (threadIdx.x == 0) {
    mbar_init(done, 1);
    *never = 0;
    span[0] = 0;
    span[1] = 0;
    for (int b = 0; b < 3; ++b) mbar_init(&landed[b], 1);
    fence_mbarrier_init();
  }
  fence_proxy_async_smem();
  if (warp == 0) {
    tmem_alloc(slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *slot;
  if (mode >= 8) {
    // mode 8: warps 0-3 write 48 scale columns per K-step into TMEM with
    //         tcgen05.st (16 + 32 columns per lane), no MMAs
    // mode 9: the same writes (into columns the MMAs do not read) while warp 4
    //         issues 4 MMAs per K-step
    const long long t0 = clock64();
    if (warp < 4 && mode <= 11) {
      uint32_t r16[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) r16[i] = 0x38383838u ^ (uint32_t)(i * 0x01010101u);
      const uint32_t lanes = (uint32_t)(warp * 32) << 16;
      const int lane = threadIdx.x & 31;
      const uint4 *sf_smem = reinterpret_cast<const uint4 *>(smem + 16384 + 32768);   // 6 KB of scales
      for (int it = 0; it < iters; ++it) {
        const uint32_t col = 320u + 48u * (uint32_t)(it & 1);
        if (mode >= 10) {
          // mode 10/11: each lane reads its 16-byte record of the 12 atoms from shared memory first
          uint32_t v[48];
#pragma unroll
          for (int c = 0; c < 12; ++c) {
            const uint4 q = sf_smem[c * 32 + lane];
            v[4 * c] = q.x; v[4 * c + 1] = q.y; v[4 * c + 2] = q.z; v[4 * c + 3] = q.w;
          }
          uint32_t (&a0)[16] = *reinterpret_cast<uint32_t (*)[16]>(&v[0]);
          uint32_t (&a1)[16] = *reinterpret_cast<uint32_t (*)[16]>(&v[16]);
          uint32_t (&a2)[16] = *reinterpret_cast<uint32_t (*)[16]>(&v[32]);
          tmem_st_16cols(tmem + lanes + col, a0);
          tmem_st_16cols(tmem + lanes + col + 16, a1);
          tmem_st_16cols(tmem + lanes + col + 32, a2);
        } else {
          tmem_st_16cols(tmem + lanes + col, r16);
          tmem_st_16cols(tmem + lanes + col + 16, r16);
          tmem_st_16cols(tmem + lanes + col + 32, r16);
        }
        tmem_st_wait();
      }
    } else if (warp == 4 && (threadIdx.x & 31) == 0 && mode == 12) {
      // mode 12: bulk global->shared copies, three 18 KB batches in flight
      // (sf_a_copies * 4.5 KB each... see below), for as long as the MMAs run
      const int chunk = 4608 * (sf_a_copies > 0 ? sf_a_copies : 1);   // bytes per batch
      uint64_t *bars = landed;                                       // 3 barriers
      const int nb = kProbeLand / chunk < 3 ? kProbeLand / chunk : 3;
      int issued = 0;
      for (int it = 0; it < iters * 3; ++it) {
        const int b = it % nb;
        if (it >= nb) mbar_wait_bounded(&bars[b], (uint32_t)(((it / nb) - 1) & 1), never, err, 902);
        mbar_arrive_expect_tx(&bars[b], chunk);
        bulk_load(smem + kProbeOps + b * chunk, gsrc + b * chunk, chunk, &bars[b]);
        issued = it + 1;
        if (*reinterpret_cast<volatile unsigned long long *>(span + 1) != 0) break;   // MMAs done
      }
      // let the batches still in flight land: batch j completed phase j / nb of its barrier
      for (int j = issued - nb > 0 ? issued - nb : 0; j < issued; ++j)
        mbar_wait_bounded(&bars[j % nb], (uint32_t)((j / nb) & 1), never, err, 904);
    }
    if (mode == 12 && warp == 0 && (threadIdx.x & 31) == 0) {
      const uint32_t a_addr = smem_u32(smem);
      const uint32_t b_addr = a_addr + 16384;
      const uint32_t idesc = (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
      const long long m0 = clock64();
      for (int it = 0; it < iters; ++it) {
#pragma unroll
        for (int kb = 0; kb < 4; ++kb)
          mma_nvfp4(tmem, smem_desc(a_addr + kb * 32, 16, 1024, 2), smem_desc(b_addr + kb * 32, 16, 1024, 2),
                    idesc, tmem + 256 + 4 * kb, tmem + 272 + 8 * kb, (it | kb) != 0 ? 1u : 0u);
      }
      tc_commit(done);
      mbar_wait_bounded(done, 0, never, err, 903);
      const long long m1 = clock64();
      *reinterpret_cast<volatile unsigned long long *>(span + 1) = (unsigned long long)(m1 - m0);
      cycles[blockIdx.x] = m1 - m0;   // the MMA thread's own time
    }
    if (false) {
    } else if (warp == 4 && (threadIdx.x & 31) == 0 && (mode == 9 || mode == 11)) {
      const uint32_t a_addr = smem_u32(smem);
      const uint32_t b_addr = a_addr + 16384;
      const uint32_t idesc = (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
      for (int it = 0; it < iters; ++it) {
#pragma unroll
        for (int kb = 0; kb < 4; ++kb)
          mma_nvfp4(tmem, smem_desc(a_addr + kb * 32, 16, 1024, 2), smem_desc(b_addr + kb * 32, 16, 1024, 2),
                    idesc, tmem + 256 + 4 * kb, tmem + 272 + 8 * kb, (it | kb) != 0 ? 1u : 0u);
      }
      tc_commit(done);
      mbar_wait_bounded(done, 0, never, err, 901);
    }
    if ((threadIdx.x & 31) == 0) atomicMax(span, (unsigned long long)(clock64() - t0));
    tc_fence_before();
    __syncthreads();
    if (threadIdx.x == 0 && mode != 12) cycles[blockIdx.x] = (long long)span[0];
  }
  if (threadIdx.x == 0 && mode < 8) {
    const uint32_t a_addr = smem_u32(smem);
    const uint32_t b_addr = a_addr + 16384;
    const uint32_t sfa_addr = b_addr + 32768;
    const uint32_t sfb_addr = sfa_addr + 2048;
    const uint32_t idesc = (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
    const uint32_t sfa_col = 256, sfb_col = 272;
    const long long t0 = clock64();
    // mode 0: a K-step's copies, then its 4 MMAs
    // mode 1: per K-block: its copies, then its MMA
    // mode 2: copies for K-step it+1 (second SF buffer) issued before the MMAs of K-step it
    // mode 3: copies only, no MMAs
    // mode 4: mode 0 with precomputed descriptors, 4 + 8 copies unrolled
    // mode 5: mode 3 with precomputed descriptors, 4 + 8 copies unrolled
    // mode 6: four 128x128b copies (2 KB each, no replication) only
    // mode 7: four 64x128b.warpx2 copies (1 KB each, replicated twice) only
    if (mode >= 4) {
      // precomputed descriptors, fully unrolled: 4 SFA + 8 SFB atoms
      uint64_t dA[4], dB[8];
#pragma unroll
      for (int c = 0; c < 4; ++c) dA[c] = smem_desc(sfa_addr + c * 512, 0, 128, 0);
#pragma unroll
      for (int c = 0; c < 8; ++c) dB[c] = smem_desc(sfb_addr + c * 512, 0, 128, 0);
      uint64_t ad[4], bd[4];
#pragma unroll
      for (int kb = 0; kb < 4; ++kb) {
        ad[kb] = smem_desc(a_addr + kb * 32, 16, 1024, 2);
        bd[kb] = smem_desc(b_addr + kb * 32, 16, 1024, 2);
      }
      for (int it = 0; it < iters; ++it) {
        if (mode == 4 || mode == 5) {
#pragma unroll
          for (int c = 0; c < 4; ++c) tmem_cp_sf_atom(tmem + sfa_col + 4 * c, dA[c]);
#pragma unroll
          for (int c = 0; c < 8; ++c) tmem_cp_sf_atom(tmem + sfb_col + 4 * c, dB[c]);
        } else if (mode == 6) {
#pragma unroll
          for (int c = 0; c < 4; ++c)
            asm volatile("tcgen05.cp.cta_group::1.128x128b [%0], %1;" ::"r"(tmem + sfa_col + 4 * c),
                         "l"(smem_desc(sfa_addr, 0, 128, 0)) : "memory");
        } else {
#pragma unroll
          for (int c = 0; c < 4; ++c)
            asm volatile("tcgen05.cp.cta_group::1.64x128b.warpx2::02_13 [%0], %1;" ::"r"(tmem + sfa_col + 4 * c),
                         "l"(smem_desc(sfa_addr, 0, 128, 0)) : "memory");
        }
        if (mode == 4) {
#pragma unroll
          for (int kb = 0; kb < 4; ++kb)
            mma_nvfp4(tmem, ad[kb], bd[kb], idesc, tmem + sfa_col + 4 * kb, tmem + sfb_col + 8 * kb,
                      (it | kb) != 0 ? 1u : 0u);
        }
      }
    }
    for (int it = 0; it < (mode >= 4 ? 0 : iters); ++it) {
      const uint32_t buf = (mode == 2) ? 48u * (uint32_t)((it + 1) & 1) : 0u;
      const uint32_t rbuf = (mode == 2) ? 48u * (uint32_t)(it & 1) : 0u;
      if (mode != 1) {
        for (int c = 0; c < sf_a_copies; ++c)
          tmem_cp_sf_atom(tmem + sfa_col + buf + 4 * (c & 3), smem_desc(sfa_addr + (c & 3) * 512, 0, 128, 0));
        for (int c = 0; c < sf_b_copies; ++c)
          tmem_cp_sf_atom(tmem + sfb_col + buf + 4 * (c & 7), smem_desc(sfb_addr + (c & 7) * 512, 0, 128, 0));
      }
      if (mode == 3) continue;
#pragma unroll
      for (int kb = 0; kb < 4; ++kb) {
        if (mode == 1) {
          if (kb < sf_a_copies)
            tmem_cp_sf_atom(tmem + sfa_col + 4 * kb, smem_desc(sfa_addr + kb * 512, 0, 128, 0));
          for (int h = 0; h < sf_b_copies / 4; ++h)
            tmem_cp_sf_atom(tmem + sfb_col + 8 * kb + 4 * h, smem_desc(sfb_addr + (2 * kb + h) * 512, 0, 128, 0));
        }
        const uint64_t adesc = smem_desc(a_addr + kb * 32, 16, 1024, 2);
        const uint64_t bdesc = smem_desc(b_addr + kb * 32, 16, 1024, 2);
        mma_nvfp4(tmem, adesc, bdesc, idesc, tmem + sfa_col + rbuf + 4 * kb, tmem + sfb_col + rbuf + 8 * kb,
                  (it | kb) != 0 ? 1u : 0u);
      }
    }
    tc_commit(done);
    mbar_wait_bounded(done, 0, never, err, 900);
    cycles[blockIdx.x] = clock64() - t0;
  }
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace

// Self-test of the bounded wait: one thread waits for a phase of an mbarrier
// that nothing arrives on, through the same routine every kernel of the
// library waits with.  After the bound it records kDevTimeout (detail 990)
// in the error word and the kernel returns; nothing faults or hangs.
__global__ void k_wait_selftest(int *err) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbarrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait_bounded(&bar, 0, &abort_flag, err, 990);
}

cudaError_t launch_wait_selftest(int *err, cudaStream_t s) {
  k_wait_selftest<<<1, 32, 0, s>>>(err);
  return cudaGetLastError();
}

cudaError_t launch_mma_probe(int iters, int n, int sf_a_copies, int sf_b_copies, int mode,
                             long long *cycles, int *err, const uint8_t *gsrc, int grid, cudaStream_t s) {
  cudaError_t e = cudaFuncSetAttribute(k_mma_probe, cudaFuncAttributeMaxDynamicSharedMemorySize, kProbeSmem);
  if (e != cudaSuccess) return e;
  k_mma_probe<<<grid, 160, kProbeSmem, s>>>(iters, n, sf_a_copies, sf_b_copies, mode, cycles, err, gsrc);
  return cudaGetLastError();
}

}  // namespace nvfp4moe
