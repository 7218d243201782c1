// Tensor-core throughput probe for the block-scaled FP4 MMA: the measured
// roofline denominator of the grouped GEMM on the GPU at hand.
//
// One CTA per SM issues `iters` K-steps of 4 tcgen05.mma kind::mxf4nvf4
// (M = 128, N = 256, K = 64) on operands already resident in shared memory
// (zeros: only the timing is meaningful), with FP32 accumulation in TMEM.
// With scale_writes, warps 0-3 meanwhile write a K-step's 48 scale columns
// into a spare TMEM slot with tcgen05.st, read from shared memory, exactly as
// the grouped GEMM's scale feeders do -- the rate the GEMM can reach when its
// operands are never late.  No global memory is read.  Each CTA records its
// elapsed SM cycles.
//
// Also here: the self-test kernel of the bounded-wait failure path.
#include "common.cuh"
#include "internal.h"

namespace nvfp4moe {

namespace {

constexpr int kProbeA = 16384, kProbeB = 32768, kProbeSf = 6144;
constexpr int kProbeSmem = kProbeA + kProbeB + kProbeSf + 1024 + 64;
constexpr int kProbeN = 256;

__global__ void __launch_bounds__(160, 1)
    k_mma_peak(int iters, int scale_writes, long long *cycles, int *err) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t *done = reinterpret_cast<uint64_t *>(smem + kProbeA + kProbeB + kProbeSf);
  uint32_t *slot = reinterpret_cast<uint32_t *>(done + 1);
  int *never = reinterpret_cast<int *>(slot + 1);
  unsigned long long *span = reinterpret_cast<unsigned long long *>(slot + 2);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int i = threadIdx.x; i < (kProbeA + kProbeB + kProbeSf) / 16; i += blockDim.x)
    reinterpret_cast<uint4 *>(smem)[i] = make_uint4(0, 0, 0, 0);
  if (threadIdx.x == 0) {
    mbar_init(done, 1);
    *never = 0;
    *span = 0;
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
  const long long t0 = clock64();
  if (warp < 4 && scale_writes) {
    // each lane reads its 16-byte records of the K-step's 12 scale atoms and
    // writes them as 48 columns of its TMEM lane (columns the MMAs do not read)
    const uint32_t lanes = (uint32_t)(warp * 32) << 16;
    const uint4 *sf_smem = reinterpret_cast<const uint4 *>(smem + kProbeA + kProbeB);
    for (int it = 0; it < iters; ++it) {
      const uint32_t col = 320u + 48u * (uint32_t)(it & 1);
      uint32_t v[48];
#pragma unroll
      for (int c = 0; c < 12; ++c) {
        const uint4 q = sf_smem[c * 32 + lane];
        v[4 * c] = q.x; v[4 * c + 1] = q.y; v[4 * c + 2] = q.z; v[4 * c + 3] = q.w;
      }
#pragma unroll
      for (int c = 0; c < 3; ++c)
        tmem_st_16cols(tmem + lanes + col + 16 * c, *reinterpret_cast<const uint32_t (*)[16]>(&v[16 * c]));
      tmem_st_wait();
    }
  } else if (warp == 4 && lane == 0) {
    const uint32_t a_addr = smem_u32(smem);
    const uint32_t b_addr = a_addr + kProbeA;
    const uint32_t idesc = (1u << 7) | (1u << 10) | ((uint32_t)(kProbeN >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
    for (int it = 0; it < iters; ++it) {
#pragma unroll
      for (int kb = 0; kb < 4; ++kb)
        mma_nvfp4(tmem, smem_desc(a_addr + kb * 32, 16, 1024, 2), smem_desc(b_addr + kb * 32, 16, 1024, 2),
                  idesc, tmem + 256 + 4 * kb, tmem + 272 + 8 * kb, (it | kb) != 0 ? 1u : 0u);
    }
    tc_commit(done);
    mbar_wait_bounded(done, 0, never, err, 901);
  }
  if (lane == 0) atomicMax(span, (unsigned long long)(clock64() - t0));
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0) cycles[blockIdx.x] = (long long)*span;
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

cudaError_t launch_mma_peak(int iters, int scale_writes, long long *cycles, int *err, int grid, cudaStream_t s) {
  cudaError_t e = cudaFuncSetAttribute(k_mma_peak, cudaFuncAttributeMaxDynamicSharedMemorySize, kProbeSmem);
  if (e != cudaSuccess) return e;
  k_mma_peak<<<grid, 160, kProbeSmem, s>>>(iters, scale_writes, cycles, err);
  return cudaGetLastError();
}

}  // namespace nvfp4moe
