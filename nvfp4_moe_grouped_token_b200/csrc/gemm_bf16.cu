// Persistent BF16 grouped GEMM over the experts on tcgen05 (sm_100a): the
// matrix products of the layer's BF16 backward.
//
// The pages time a mode that runs the forward in NVFP4 and the backward in
// BF16 (www.aib.vote "miniTE report, NVFP4 RL stability", paragraph 1:
// about 1.33-1.37x over BF16).  Its products, per expert e with G = [g | u]
// the gate_up output, h = silu(g) u, and rows r of the expert's group:
//   G      = x_rows W_gu,e^T          (recomputed, BF16 operands)
//   dh'    = dy_rows W_dn,e           (dgrad of down; B is MN-major)
//   dx_r   = dG W_gu,e                (dgrad of gate_up; B is MN-major)
//   dW_dn,e = dy_rows^T (w h)         (wgrad: K runs over the group's rows,
//   dW_gu,e = dG^T x_rows              both operands MN-major)
//
// Design (B200):
//   * tcgen05.mma.cta_group::1.kind::f16, M = 128, N = 256, K = 16, BF16
//     operands from shared memory, FP32 accumulation in TMEM.  With no scale
//     factors to stage, two 256-column accumulators fill TMEM, so the
//     epilogue of tile i overlaps the MMAs of tile i+1.
//   * operands are loaded by 128-byte-swizzled TMA tensor copies in either
//     orientation: K-major (a box of 64 K-elements x rows) or MN-major (boxes
//     of 64 M/N-elements x 64 K-rows, stacked 8 KB apart along M/N); the
//     shared-memory matrix descriptors and the instruction descriptor's
//     transpose bits say which.  So the backward reads every tensor where it
//     lies, with no transposed copies.
//   * K-step of 64 elements, a 4-stage ring (A 16 KB + B 32 KB per stage).
//   * warp 0: TMA producer (one thread); warp 1: TMEM owner and MMA issuer
//     (one thread); warps 4-11: epilogue, two per TMEM lane quarter, each
//     reading half of the 256 columns (setmaxnreg: 200 registers for the
//     epilogue warpgroups, 96 for the first).  BF16 outputs leave through
//     TMA tensor stores; the SwiGLU-backward epilogue instead runs each 32 x
//     32 chunk transposed through the warp's staging tile, so its loads of g
//     and u and its stores of dG and w h cover 8 rows x 64 bytes each.
//   * kBfRows: tiles over (m-tile, n-tile) of the padded grouped rows with n
//     fastest; the expert of an m-tile comes from padded_offsets.
//     kBfWgrad: tiles over (expert, m-tile, n-tile); the K loop covers the
//     expert's rows in steps of 64 (padding rows inside a group are zero, so
//     the step past the last row adds nothing); an empty expert's tile is
//     written as zeros.
//   * every wait is bounded (common.cuh).
#include <cudaTypedefs.h>

#include <cstring>

#include "common.cuh"
#include "internal.h"

namespace nvfp4moe {

// Shared tensor-map helpers of the FP4 GEMM (gemm.cu).
bool encode_2d_map(CUtensorMap *map, CUtensorMapDataType dtype, uint32_t esize, const void *base,
                   uint64_t inner, uint64_t rows, uint32_t box_inner, uint32_t box_rows,
                   CUtensorMapSwizzle swizzle);

namespace {

constexpr int BM = 128, BN = 256, BK = 64;
constexpr int STAGES = 4;
constexpr int ACC = 2;
constexpr int kThreads = 384;
constexpr int kEpiWarp0 = 4, kEpiWarps = 8;
// setmaxnreg: the first warpgroup (producer, MMA issuer, two idle warps)
// gives registers to the two epilogue warpgroups: 128 * 96 + 256 * 200 =
// 63488 of the 384 threads * 168 registers at launch.
constexpr uint32_t kRegsCtl = 96, kRegsEpi = 200;
static_assert(128 * kRegsCtl + 256 * kRegsEpi <= 384 * 168, "register split");
constexpr int kABytes = BM * BK * 2;          // 16 KB
constexpr int kBBytes = BN * BK * 2;          // 32 KB
constexpr int kStageBytes = kABytes + kBBytes;
constexpr int kMnBox = 64 * BK * 2;           // one MN-major box: 64 elements x 64 K-rows = 8 KB
constexpr int kStagingPerWarp = 4096;         // two 32 x 32 BF16 boxes
constexpr size_t kStagingOff = (size_t)STAGES * kStageBytes;
constexpr size_t kBarrierOff = kStagingOff + (size_t)kEpiWarps * kStagingPerWarp;
constexpr size_t kSmemBytes = kBarrierOff + 256 + 1024;   // + slack for 1 KB alignment
static_assert(kSmemBytes <= 232448, "shared memory budget");

// Instruction descriptor, kind::f16: FP32 accumulator (bits 4-5 = 1), A and
// B BF16 (bits 7-9, 10-12 = 1), transpose bits 15 (A MN-major) and 16 (B
// MN-major), N >> 3 at bit 17, M >> 4 at bit 24.
__host__ __device__ constexpr uint32_t idesc_bf16(int a_mn, int b_mn) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)a_mn << 15) | ((uint32_t)b_mn << 16) |
         ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);
}

struct __align__(64) BParams {
  CUtensorMap tmap_a;
  CUtensorMap tmap_b;
  CUtensorMap tmap_out;   // BF16 output, 32 x 32 boxes, 64-byte swizzle
  Bf16GemmArgs a;
};

__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t"
      "}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void stage_row(uint32_t box_addr, int lane, const uint32_t (&w)[16]) {
  const uint32_t base = box_addr + (uint32_t)lane * 64;
  const uint32_t sw = ((uint32_t)lane >> 1) & 3u;
#pragma unroll
  for (int q = 0; q < 4; ++q)
    st_shared_v4(base + (((uint32_t)q ^ sw) << 4), w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
}

__device__ __forceinline__ int find_group_g(const int32_t *padded, int E, int64_t row) {
  int lo = 0, hi = E;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if ((int64_t)__ldg(padded + mid) <= row) lo = mid; else hi = mid;
  }
  return lo;
}

// Tile t of the launch: expert, first row / output row block, n block, and
// the number of 64-element K-steps.
struct Tile {
  int e;
  int64_t m0;       // kBfRows: first padded row; kBfWgrad: first M index
  int64_t n0;
  int64_t k_rows0;  // kBfWgrad: first padded row of the group (the K origin)
  int ksteps;
};

__device__ __forceinline__ Tile tile_of(const Bf16GemmArgs &a, int64_t t, int n_tiles, int m_tiles) {
  Tile r;
  if (a.mode == kBfRows) {
    const int64_t mt = t / n_tiles;
    r.n0 = (t - mt * n_tiles) * BN;
    r.m0 = mt * BM;
    r.e = find_group_g(a.padded_offsets, a.E, r.m0);
    r.k_rows0 = 0;
    r.ksteps = (int)(a.K / BK);
  } else {
    const int64_t per_e = (int64_t)m_tiles * n_tiles;
    r.e = (int)(t / per_e);
    const int64_t rem = t - (int64_t)r.e * per_e;
    const int64_t mt = rem / n_tiles;
    r.m0 = mt * BM;
    r.n0 = (rem - mt * n_tiles) * BN;
    r.k_rows0 = __ldg(a.padded_offsets + r.e);
    const int64_t cnt = (int64_t)__ldg(a.offsets + r.e + 1) - __ldg(a.offsets + r.e);
    r.ksteps = (int)((cnt + BK - 1) / BK);
  }
  return r;
}

__global__ void __launch_bounds__(kThreads, 1) k_bf16_gemm(const __grid_constant__ BParams P) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + kBarrierOff);
  uint64_t *empty = full + STAGES;
  uint64_t *acc_full = empty + STAGES;
  uint64_t *acc_empty = acc_full + ACC;
  uint64_t *drain = acc_empty + ACC;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
  int *never = reinterpret_cast<int *>(tmem_slot + 2);

  const Bf16GemmArgs &a = P.a;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int a_mn = a.mode == kBfWgrad ? 1 : 0;
  const int b_mn = a.mode == kBfWgrad ? 1 : a.b_mn;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int s = 0; s < ACC; ++s) {
      mbar_init(&acc_full[s], 1);
      mbar_init(&acc_empty[s], kEpiWarps);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    *never = 0;
    fence_mbarrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensor_map(&P.tmap_a);
    prefetch_tensor_map(&P.tmap_b);
    prefetch_tensor_map(&P.tmap_out);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  const int n_tiles = (int)(a.N / BN);
  const int m_tiles = a.mode == kBfWgrad ? (int)(a.M / BM) : 0;
  int64_t total;
  if (a.mode == kBfRows) {
    int64_t rows_used = __ldg(a.padded_offsets + a.E);
    if (rows_used > a.rows_cap) rows_used = a.rows_cap;
    if (rows_used < 0) rows_used = 0;
    total = (rows_used / BM) * n_tiles;
  } else {
    total = (int64_t)a.E * m_tiles * n_tiles;
  }
  if (warp < kEpiWarp0) asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsCtl));
  if (warp == 0) {
    if (lane == 0) {
      // ---------------------------------------------------- TMA producer
      uint32_t p = 0;
      bool ok = true;
      for (int64_t t = blockIdx.x; t < total && ok; t += gridDim.x) {
        const Tile tl = tile_of(a, t, n_tiles, m_tiles);
        uint32_t st = p % STAGES, ph = (p / STAGES) & 1u;
        for (int kt = 0; kt < tl.ksteps; ++kt, ++p) {
          if (!mbar_wait_bounded(&empty[st], ph ^ 1u, abort_flag, a.err, 500)) { ok = false; break; }
          uint8_t *sa = smem + (size_t)st * kStageBytes;
          uint8_t *sb = sa + kABytes;
          mbar_arrive_expect_tx(&full[st], kStageBytes);
          if (a.mode == kBfRows) {
            tma_load_2d(sa, &P.tmap_a, kt * BK, (int32_t)tl.m0, &full[st]);
            if (b_mn) {
              // B_e[n][k] = W[e][k][n]: boxes of 64 n x 64 k-rows
              const int32_t krow = (int32_t)((int64_t)tl.e * a.K + (int64_t)kt * BK);
#pragma unroll
              for (int c = 0; c < BN / 64; ++c)
                tma_load_2d(sb + c * kMnBox, &P.tmap_b, (int32_t)(tl.n0 + 64 * c), krow, &full[st]);
            } else {
              tma_load_2d(sb, &P.tmap_b, kt * BK, (int32_t)((int64_t)tl.e * a.N + tl.n0), &full[st]);
            }
          } else {
            const int32_t krow = (int32_t)(tl.k_rows0 + (int64_t)kt * BK);
#pragma unroll
            for (int c = 0; c < BM / 64; ++c)
              tma_load_2d(sa + c * kMnBox, &P.tmap_a, (int32_t)(tl.m0 + 64 * c), krow, &full[st]);
#pragma unroll
            for (int c = 0; c < BN / 64; ++c)
              tma_load_2d(sb + c * kMnBox, &P.tmap_b, (int32_t)(tl.n0 + 64 * c), krow, &full[st]);
          }
          if (++st == STAGES) { st = 0; ph ^= 1u; }
        }
      }
      for (uint32_t q = p > STAGES ? p - STAGES : 0; q < p; ++q)
        mbar_wait_bounded(&full[q % STAGES], (q / STAGES) & 1u, never, a.err, 501);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------ MMA issuer
      // K-major: the 16-element K slice kk starts 32 bytes further in each
      // 128-byte row (LBO unused, SBO = 1024 between 8-row groups).
      // MN-major: slice kk starts 16 K-rows (2 KB) further; LBO = 8 KB
      // between 64-element M/N chunks, SBO = 1024 between 8-row K groups.
      const uint64_t dk = smem_desc(0, 16, 1024, 2);
      const uint64_t dmn = smem_desc(0, kMnBox, 1024, 2);
      const uint64_t da = a_mn ? dmn : dk, db = b_mn ? dmn : dk;
      const uint32_t step_a = a_mn ? 2048u >> 4 : 32u >> 4, step_b = b_mn ? 2048u >> 4 : 32u >> 4;
      const uint32_t idesc = idesc_bf16(a_mn, b_mn);
      const uint32_t smem0 = smem_u32(smem);
      uint32_t st = 0, ph = 0, it = 0;
      bool ok = true;
      for (int64_t t = blockIdx.x; t < total && ok; t += gridDim.x, ++it) {
        const Tile tl = tile_of(a, t, n_tiles, m_tiles);
        const uint32_t as = it % ACC;
        const uint32_t acc = tmem + as * BN;
        if (!mbar_wait_bounded(&acc_empty[as], ((it / ACC) & 1u) ^ 1u, abort_flag, a.err, 510)) break;
        tc_fence_after();
        for (int kt = 0; kt < tl.ksteps; ++kt) {
          if (!mbar_wait_bounded(&full[st], ph, abort_flag, a.err, 511)) { ok = false; break; }
          tc_fence_after();
          const uint64_t a16 = (smem0 + st * (uint32_t)kStageBytes) >> 4;
          const uint64_t b16 = a16 + kABytes / 16;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk)
            mma_bf16(acc, da | (a16 + kk * step_a), db | (b16 + kk * step_b), idesc, (kt | kk) != 0 ? 1u : 0u);
          tc_commit(&empty[st]);
          if (++st == STAGES) { st = 0; ph ^= 1u; }
        }
        if (ok) tc_commit(&acc_full[as]);
      }
      tc_commit(drain);
      mbar_wait_bounded(drain, 0, never, a.err, 512);
    }
  } else if (warp >= kEpiWarp0) {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsEpi));
    // -------------------------------------------------------- epilogue
    const int ew = warp - kEpiWarp0;
    const int quad = warp & 3;
    const int half = ew >> 2;
    const uint32_t tlane = tmem + ((uint32_t)(quad * 32) << 16);
    uint8_t *stg = smem + kStagingOff + (size_t)ew * kStagingPerWarp;
    const uint32_t stg_addr = smem_u32(stg);
    uint32_t chunk_id = 0, it = 0;
    auto store_box = [&](const uint32_t (&w16)[16], int32_t x, int32_t y) {
      const uint32_t box = stg_addr + (chunk_id & 1u) * 2048;
      if (lane == 0) bulk_wait_group_read<1>();
      __syncwarp();
      stage_row(box, lane, w16);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        tma_store_2d(&P.tmap_out, stg + (chunk_id & 1u) * 2048, x, y);
        bulk_commit_group();
      }
      ++chunk_id;
    };
    const int64_t rows_total = a.mode == kBfRows ? (int64_t)__ldg(a.offsets + a.E) : 0;
    for (int64_t t = blockIdx.x; t < total; t += gridDim.x, ++it) {
      const Tile tl = tile_of(a, t, n_tiles, m_tiles);
      const uint32_t as = it % ACC;
      // rows of this lane
      int64_t orow;            // output row index
      bool valid = true;
      int64_t prow = 0;        // padded row (kBfRows)
      bool slab_full = true;
      int64_t slab_row = 0;
      if (a.mode == kBfRows) {
        const int64_t g_pad = __ldg(a.padded_offsets + tl.e);
        const int64_t g_off = __ldg(a.offsets + tl.e);
        const int64_t g_cnt = (int64_t)__ldg(a.offsets + tl.e + 1) - g_off;
        const int64_t rel = tl.m0 - g_pad + quad * 32 + lane;
        valid = rel < g_cnt && g_off + rel < rows_total;
        prow = tl.m0 + quad * 32 + lane;
        orow = a.out_padded ? prow : g_off + rel;
        slab_full = a.out_padded || (tl.m0 - g_pad) + quad * 32 + 32 <= g_cnt;
        slab_row = a.out_padded ? tl.m0 + quad * 32 : g_off + (tl.m0 - g_pad) + quad * 32;
      } else {
        orow = (int64_t)tl.e * a.M + tl.m0 + quad * 32 + lane;
        slab_row = (int64_t)tl.e * a.M + tl.m0 + quad * 32;
      }
      // SwiGLU backward, processed transposed: each 32 x 32 chunk of dh'
      // goes through the warp's staging tile in shared memory, and lane l
      // then takes rows rl + 8 k (k < 4, rl = l / 4) of the warp's 32 and
      // columns 8 s .. 8 s + 7 (s = l % 4) of the chunk.  Every global access
      // of the chunk (g, u, dG, w h) then covers 8 rows x 64 contiguous bytes
      // instead of one row per lane.  g and u are loaded a chunk ahead, so
      // their HBM latency overlaps the previous chunk (chunk 0 before the
      // accumulator wait).
      const int64_t I = a.N;
      const int64_t col0 = tl.n0 + half * 128;
      const int s4 = lane & 3, rl = lane >> 2;
      const int64_t prow_t0 = tl.m0 + quad * 32 + rl;     // row of k = 0; k adds 8 k
      uint4 gq[4], uq[4];
      auto load_gu = [&](int c) {
#pragma unroll
        for (int k4 = 0; k4 < 4; ++k4) {
          const __nv_bfloat16 *gr = static_cast<const __nv_bfloat16 *>(a.g_u) + (prow_t0 + 8 * k4) * 2 * I +
                                    col0 + c * 32 + 8 * s4;
          gq[k4] = __ldg(reinterpret_cast<const uint4 *>(gr));
          uq[k4] = __ldg(reinterpret_cast<const uint4 *>(gr + I));
        }
      };
      float wr_t[4] = {0.0f, 0.0f, 0.0f, 0.0f};
      if (a.epilogue == kBfSwiGLUBwd) {
#pragma unroll
        for (int k4 = 0; k4 < 4; ++k4) wr_t[k4] = __ldg(a.w_rows + prow_t0 + 8 * k4);
        load_gu(0);
      }

      if (!mbar_wait_bounded(&acc_full[as], (it / ACC) & 1u, abort_flag, a.err, 520)) break;
      tc_fence_after();
      // Chunk by chunk (32 columns): with two accumulators the MMAs of the
      // next tile run in the other one, so this one is released after the
      // last chunk is read.  An empty expert's tile (no K-steps) is zeros.
      const bool zero_tile = tl.ksteps == 0;
      float dwp_t[4] = {0.0f, 0.0f, 0.0f, 0.0f};   // <dh', h> of rows rl + 8 k over this lane's columns
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        uint32_t v[32];
        if (!zero_tile) {
          tmem_ld_32cols(tlane + as * BN + half * 128 + c * 32, v);
          tmem_ld_wait();
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = 0u;
        }
        if (c == 3) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&acc_empty[as]);
        }
        if (a.epilogue == kBfStore) {
          if (a.out_bf16 != nullptr) {
            uint32_t w16[16];
#pragma unroll
            for (int i = 0; i < 16; ++i)
              w16[i] = pack_bf16x2(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
            if (slab_full) {
              store_box(w16, (int32_t)(col0 + c * 32), (int32_t)slab_row);
            } else if (valid) {
              uint4 *dst = reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(a.out_bf16) + orow * a.N +
                                                     col0 + c * 32);
#pragma unroll
              for (int q = 0; q < 4; ++q)
                dst[q] = make_uint4(w16[4 * q], w16[4 * q + 1], w16[4 * q + 2], w16[4 * q + 3]);
            }
          }
          const int64_t n_store = a.n_store ? a.n_store : a.N;
          if (a.out_f32 != nullptr && valid && col0 + c * 32 < n_store) {
            float4 *dst = reinterpret_cast<float4 *>(a.out_f32 + orow * (a.out_ld ? a.out_ld : a.N) + col0 + c * 32);
#pragma unroll
            for (int i = 0; i < 32; i += 4)
              dst[i / 4] = make_float4(__uint_as_float(v[i]), __uint_as_float(v[i + 1]), __uint_as_float(v[i + 2]),
                                       __uint_as_float(v[i + 3]));
          }
        } else {
          // SwiGLU backward, columns i0 .. i0+31 of I:
          //   dh' = accumulator (dy W_dn), s = sigmoid(g), h = BF16(g s u),
          //   dh = w dh', dg = dh u s (1 + g (1 - s)), du = dh g s,
          //   hw = BF16(w h), dw partial += dh' h
          const int64_t i0 = col0 + c * 32;
          if (a.out_f32 != nullptr) {     // dh' itself, for inspection (lane = row prow)
            float4 *dst = reinterpret_cast<float4 *>(a.out_f32 + prow * a.N + i0);
#pragma unroll
            for (int i = 0; i < 32; i += 4)
              dst[i / 4] = make_float4(__uint_as_float(v[i]), __uint_as_float(v[i + 1]), __uint_as_float(v[i + 2]),
                                       __uint_as_float(v[i + 3]));
          }
          // the chunk into the staging tile: 16-byte piece m of row `lane` at
          // piece m ^ (lane & 7) (conflict-free both ways)
          const uint32_t trow = stg_addr + (uint32_t)lane * 128;
#pragma unroll
          for (int m = 0; m < 8; ++m)
            st_shared_v4(trow + (((uint32_t)m ^ ((uint32_t)lane & 7u)) << 4), v[4 * m], v[4 * m + 1], v[4 * m + 2],
                         v[4 * m + 3]);
          __syncwarp();
          uint4 dq[4][2];
#pragma unroll
          for (int k4 = 0; k4 < 4; ++k4) {
            const uint32_t r = (uint32_t)(rl + 8 * k4);
            const uint32_t rb = stg_addr + r * 128;
            dq[k4][0] = ld_shared_v4(rb + (((uint32_t)(2 * s4) ^ (r & 7u)) << 4));
            dq[k4][1] = ld_shared_v4(rb + (((uint32_t)(2 * s4 + 1) ^ (r & 7u)) << 4));
          }
          __syncwarp();                         // the tile is free for the next chunk
          uint4 gc[4], uc[4];
#pragma unroll
          for (int k4 = 0; k4 < 4; ++k4) {
            gc[k4] = gq[k4];
            uc[k4] = uq[k4];
          }
          if (c < 3) load_gu(c + 1);           // the next chunk's g and u, in flight during this one
#pragma unroll
          for (int k4 = 0; k4 < 4; ++k4) {
            const uint32_t gw[4] = {gc[k4].x, gc[k4].y, gc[k4].z, gc[k4].w};
            const uint32_t uw[4] = {uc[k4].x, uc[k4].y, uc[k4].z, uc[k4].w};
            const uint32_t dw[8] = {dq[k4][0].x, dq[k4][0].y, dq[k4][0].z, dq[k4][0].w,
                                    dq[k4][1].x, dq[k4][1].y, dq[k4][1].z, dq[k4][1].w};
            const float wr = wr_t[k4];
            uint32_t o_dg[4], o_du[4], o_hw[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              float dg2[2], du2[2], hw2[2];
#pragma unroll
              for (int r = 0; r < 2; ++r) {
                const float g = r ? bf16_hi(gw[i]) : bf16_lo(gw[i]);
                const float u = r ? bf16_hi(uw[i]) : bf16_lo(uw[i]);
                const float dhp = __uint_as_float(dw[2 * i + r]);
                const float dh = wr * dhp;
                // sigmoid s = sc * sp without overflow: g >= 0: sp = 1/(1+e^-g);
                // g < 0: sp = e^g/(1+e^g); g < -64: sp = e^(g+64), sc = e^-64
                // (then 1 + e^g and 1 - s are 1 in binary32).  Fast exponential
                // and division (~2^-21 relative, the denominator in [1, 2]).
                const bool far = g < -64.0f;
                const float t = __expf(g >= 0.0f ? -g : (far ? g + 64.0f : g));
                const float sp = __fdividef(g >= 0.0f ? 1.0f : t, far ? 1.0f : 1.0f + t);
                const float sc = far ? kExpM64 : 1.0f;
                const float oms = far ? 1.0f : 1.0f - sp;
                const float gs = g * sp;
                const float hf = (gs * u) * sc;
                dg2[r] = (dh * u * (sp * (1.0f + g * oms))) * sc;
                du2[r] = (dh * gs) * sc;
                const float h = __bfloat162float(__float2bfloat16_rn(hf));
                hw2[r] = wr * h;
                dwp_t[k4] = __fmaf_rn(dhp, h, dwp_t[k4]);
              }
              o_dg[i] = pack_bf16x2(dg2[0], dg2[1]);
              o_du[i] = pack_bf16x2(du2[0], du2[1]);
              o_hw[i] = pack_bf16x2(hw2[0], hw2[1]);
            }
            const int64_t pr = prow_t0 + 8 * k4;
            __nv_bfloat16 *dgu = static_cast<__nv_bfloat16 *>(a.d_gu) + pr * 2 * I + i0 + 8 * s4;
            __nv_bfloat16 *hwp = static_cast<__nv_bfloat16 *>(a.hw) + pr * I + i0 + 8 * s4;
            *reinterpret_cast<uint4 *>(dgu) = make_uint4(o_dg[0], o_dg[1], o_dg[2], o_dg[3]);
            *reinterpret_cast<uint4 *>(dgu + I) = make_uint4(o_du[0], o_du[1], o_du[2], o_du[3]);
            *reinterpret_cast<uint4 *>(hwp) = make_uint4(o_hw[0], o_hw[1], o_hw[2], o_hw[3]);
          }
        }
      }
      if (a.epilogue == kBfSwiGLUBwd) {
        // each row's partial over the warp's 128 columns: the four lanes of
        // the row (s = 0..3) hold 32 columns each
#pragma unroll
        for (int k4 = 0; k4 < 4; ++k4) {
          float d = dwp_t[k4];
          d += __shfl_xor_sync(0xffffffffu, d, 1);
          d += __shfl_xor_sync(0xffffffffu, d, 2);
          if (s4 == 0) a.dw_part[(prow_t0 + 8 * k4) * (I / 128) + (col0 / 128)] = d;
        }
      }
    }
    if (lane == 0) bulk_wait_group_all();
    __syncwarp();
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}


// ---------------------------------------------------------------------------
// W4A16: BF16 activations x NVFP4 weights.  The weights stay 4-bit in HBM
// (codes + UE4M3 block scales, the layout the W4A4 GEMM reads); converter
// warps turn each K-step's weight tile into BF16 in shared memory, in the
// 128-byte-swizzled K-major layout a TMA load would have produced, and the
// MMAs are the kind::f16 ones above.  code x block scale is exact in BF16
// (at most 2 + 4 significant bits, exponents well inside the range), so the
// converted operand is exactly the dequantized weight divided by the
// per-expert S_dec, which the epilogue applies to the FP32 accumulator.
// (The decode multiplies code * 2^120 by scale * 2^-120 in BF16; the second
// factor is a BF16 subnormal for subnormal UE4M3 scales, which the BF16
// multiply keeps.)
//
// The conversion is the expensive part (about as many issue slots as the
// MMAs take time for a 128 x 256 tile), so each converted weight tile feeds
// two m-tiles of the same expert: a unit is (m-tile pair, 128 weight rows),
// two M = 128, N = 128 MMAs per K-slice share the B operand, and the
// conversion per FLOP halves.  An expert with an odd number of m-tiles ends
// with a single-m-tile unit.  For the gate_up weight (rows interleaved in
// blocks of 128 gate then 128 up) a unit's 128 rows are 64 gate rows and the
// 64 matching up rows, so the SwiGLU epilogue finds both in one tile.
//
//   raw ring (4 stages): A of both m-tiles 2 x 16 KB (TMA, swizzled) +
//     codes 4 KB (two TMA boxes of 64 rows x 32 bytes, unswizzled) + scales
//     1 KB (the two 512-byte atoms holding those rows, bulk copies)
//   converted ring (2 slots): B as BF16, 16 KB each
//   TMEM: two buffers of 2 x 128 accumulator columns (epilogue of one unit
//     overlaps the MMAs of the next)
//   warp 0: producer; warp 1: TMEM owner + MMA issuer; warps 2-9: epilogue
//   (m-tile = which half of the warps, TMEM lane quarter = warp % 4);
//   warps 10-17: converters, one half row per lane and K-step.
namespace w4 {
constexpr int kThreads = 576;
constexpr int kEpiWarp0 = 2, kConvWarp0 = 10, kConvWarps = 8;
constexpr int CS = 2;

// WN weight rows per unit: 128 (two accumulator buffers of 2 x 128 columns,
// 4 raw stages) or 256 (one buffer of 2 x 256 columns, 3 raw stages; fewer
// load rows and conversions per FLOP, the epilogue no longer overlapped).
template <int WN_>
struct Cfg {
  static constexpr int WN = WN_;
  static constexpr int RS = WN == 128 ? 4 : 3;
  static constexpr int ACC = WN == 128 ? 2 : 1;
  static constexpr int kA2Bytes = 2 * kABytes;             // A of two m-tiles
  static constexpr int kCodesBytes = WN * BK / 2;          // two boxes of WN/2 rows x 32 bytes
  static constexpr int kSfBytes = 2 * 512;                 // the two scale atoms holding those rows
  static constexpr int kRawBytes = kA2Bytes + kCodesBytes + kSfBytes;
  static constexpr int kConvBytes = WN * BK * 2;
  static constexpr int kAccCols = 2 * WN;                  // one buffer: two m-tiles
  static constexpr int kHalfRowsPerLane = WN / 128;        // converter: K-half rows per lane
  static constexpr size_t kConvOff = (size_t)RS * kRawBytes;
  static constexpr size_t kStagingOff = kConvOff + (size_t)CS * kConvBytes;
  static constexpr size_t kBarrierOff = kStagingOff + (size_t)kEpiWarps * kStagingPerWarp;
  static constexpr size_t kPairsOff = kBarrierOff + 256;   // + (E + 1) int32 pair prefix
  static constexpr size_t kSmemMax = kPairsOff + 4 * 1025 + 1024;   // + up to 1023 bytes of alignment
  // Instruction descriptor as idesc_bf16 with N = WN, both operands K-major.
  static constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(WN >> 3) << 17) |
                                     ((uint32_t)(BM >> 4) << 24);
  static_assert(WN == 128 || WN == 256, "unit width");
  static_assert(kRawBytes % 1024 == 0 && kConvBytes % 1024 == 0, "swizzled tiles need 1 KB alignment");
  static_assert(kSmemMax <= 232448, "shared memory budget");
  static_assert(kConvWarps * 32 * kHalfRowsPerLane == 2 * WN, "converter lanes cover the half rows");
  static_assert(ACC * kAccCols <= 512, "TMEM budget");
  static_assert((3 * RS + 2 * CS + 2 * ACC + 1) * 8 + 12 <= 256, "barrier area");
};

// A unit's m-tiles and weight rows.
struct Unit {
  int e;
  int64_t m0;       // first padded row of the first m-tile
  bool two;         // a second m-tile at m0 + 128
  int nt;           // weight-row tile
  int64_t wrow0;    // first weight row of each WN/2-row half (global row of the [E*N] codes)
  int64_t wrow1;
};

template <int WN>
__device__ __forceinline__ Unit unit_of(const Bf16GemmArgs &a, const int32_t *pairs, int64_t u, int n_tiles,
                                        int64_t rows_cap) {
  Unit r;
  const int64_t p = u / n_tiles;
  r.nt = (int)(u - p * n_tiles);
  int lo = 0, hi = a.E;                    // the expert whose pairs hold p
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if ((int64_t)pairs[mid] <= p) lo = mid; else hi = mid;
  }
  r.e = lo;
  const int64_t g_lo = min((int64_t)__ldg(a.padded_offsets + lo), rows_cap);
  const int64_t g_hi = min((int64_t)__ldg(a.padded_offsets + lo + 1), rows_cap);
  r.m0 = g_lo + 2 * BM * (p - pairs[lo]);
  r.two = r.m0 + BM < g_hi;
  if (a.epilogue == kBfSwiGLUFwd) {
    // WN/2 gate rows of a 256-row block (128 gate, then 128 up) and the matching up rows
    constexpr int per_block = 256 / WN;
    r.wrow0 = (int64_t)r.e * a.N + 256 * (r.nt / per_block) + (WN / 2) * (r.nt % per_block);
    r.wrow1 = r.wrow0 + 128;
  } else {
    r.wrow0 = (int64_t)r.e * a.N + (int64_t)WN * r.nt;
    r.wrow1 = r.wrow0 + WN / 2;
  }
  return r;
}
}  // namespace w4

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

// Eight E2M1 codes (one word; element 2b is the low nibble of byte b) ->
// four BF16 pairs in element order holding code * 2^120.  The 3-bit
// magnitude indexes two eight-entry byte tables held in registers: the low
// and the high byte of the BF16 value of 2^120 * {0, 0.5, 1, 1.5, 2, 3, 4, 6}.
// Each code's sign bit is moved to bit 7 of its high byte on the way (one
// byte permute gathers the four sign bits of four codes).
__device__ __forceinline__ void e2m1x8_to_bf16x2(uint32_t c, uint32_t (&w)[4]) {
  constexpr uint32_t kLo0 = 0xC0800000u, kLo1 = 0xC0804000u;   // low bytes 00 00 80 C0 | 00 40 80 C0
  constexpr uint32_t kHi0 = 0x7B7B7B00u, kHi1 = 0x7C7C7C7Cu;   // high bytes 00 7B 7B 7B | 7C 7C 7C 7C
  const uint32_t m = c & 0x77777777u;
  const uint32_t mh = m >> 16;
  const uint32_t c4 = c << 4;
  const uint32_t lo_a = prmt(kLo0, kLo1, m), lo_b = prmt(kLo0, kLo1, mh);
  // byte j of the sign word holds code j's sign at bit 7: bytes c4.b0, c.b0, c4.b1, c.b1 (codes 0-3)
  const uint32_t hi_a = prmt(kHi0, kHi1, m) | (prmt(c4, c, 0x5140) & 0x80808080u);
  const uint32_t hi_b = prmt(kHi0, kHi1, mh) | (prmt(c4, c, 0x7362) & 0x80808080u);
  w[0] = prmt(lo_a, hi_a, 0x5140);
  w[1] = prmt(lo_a, hi_a, 0x7362);
  w[2] = prmt(lo_b, hi_b, 0x5140);
  w[3] = prmt(lo_b, hi_b, 0x7362);
}

// Two UE4M3 block scales (bytes of sc) -> BF16 pairs (s0, s0) and (s1, s1)
// holding scale * 2^-120: a UE4M3 code b shifted left by 4 is, read as BF16
// bits, exactly its value times 2^-120 (normal codes: exponent e - 7 + 127 -
// 120; subnormal codes m * 2^-9 become BF16 subnormals m * 2^-129).  Times
// the table's 2^120 the products are exactly code * scale.
__device__ __forceinline__ void ue4m3x2_to_bf16x2(uint32_t sc, uint32_t &s0, uint32_t &s1) {
  const uint32_t u = prmt(sc, 0u, 0x4140) << 4;   // b0 << 4 in the low half, b1 << 4 in the high half
  s0 = prmt(u, 0u, 0x1010);
  s1 = prmt(u, 0u, 0x3232);
}

__device__ __forceinline__ uint32_t mul_bf16x2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

__device__ __forceinline__ uint32_t ld_shared_u16(uint32_t saddr) {
  uint16_t v;
  asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(saddr));
  return v;
}

template <class C>
__global__ void __launch_bounds__(w4::kThreads, 1) k_w4a16_gemm(const __grid_constant__ BParams P) {
  using namespace w4;
  constexpr int WN = C::WN, RS = C::RS, ACC = C::ACC;
  constexpr int kA2Bytes = C::kA2Bytes, kCodesBytes = C::kCodesBytes, kRawBytes = C::kRawBytes;
  constexpr int kConvBytes = C::kConvBytes, kAccCols = C::kAccCols;
  constexpr size_t kConvOff = C::kConvOff;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + C::kBarrierOff);
  uint64_t *empty = full + RS;
  uint64_t *cfull = empty + RS;
  uint64_t *cempty = cfull + CS;
  uint64_t *acc_full = cempty + CS;
  uint64_t *acc_empty = acc_full + ACC;
  uint64_t *drain = acc_empty + ACC;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
  int *never = reinterpret_cast<int *>(tmem_slot + 2);
  int32_t *pairs = reinterpret_cast<int32_t *>(smem + C::kPairsOff);   // [E + 1]

  const Bf16GemmArgs &a = P.a;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < RS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int s = 0; s < CS; ++s) {
      mbar_init(&cfull[s], kConvWarps);
      mbar_init(&cempty[s], 1);
    }
    for (int s = 0; s < ACC; ++s) {
      mbar_init(&acc_full[s], 1);
      mbar_init(&acc_empty[s], kEpiWarps);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    *never = 0;
    fence_mbarrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensor_map(&P.tmap_a);
    prefetch_tensor_map(&P.tmap_b);
    prefetch_tensor_map(&P.tmap_out);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  if (warp == 2) {
    // pairs[e] = m-tile pairs of the experts before e (groups clipped to rows_cap)
    int32_t carry = 0;
    if (lane == 0) pairs[0] = 0;
    for (int base = 0; base < a.E; base += 32) {
      const int e = base + lane;
      int32_t n = 0;
      if (e < a.E) {
        const int64_t lo = min((int64_t)__ldg(a.padded_offsets + e), a.rows_cap);
        const int64_t hi = min((int64_t)__ldg(a.padded_offsets + e + 1), a.rows_cap);
        const int64_t tiles = hi > lo ? (hi - lo) / BM : 0;
        n = (int32_t)((tiles + 1) / 2);
      }
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int32_t v = __shfl_up_sync(0xffffffffu, n, o);
        if (lane >= o) n += v;
      }
      if (e < a.E) pairs[e + 1] = carry + n;
      carry += __shfl_sync(0xffffffffu, n, 31);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  const int n_tiles = (int)(a.N / WN);
  const int64_t total = (int64_t)pairs[a.E] * n_tiles;
  const int ksteps = (int)(a.K / BK);
  const int64_t k_atoms = a.K >> 6;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------------------------------------------- TMA producer
      uint32_t p = 0;
      bool ok = true;
      for (int64_t t = blockIdx.x; t < total && ok; t += gridDim.x) {
        const Unit un = unit_of<WN>(a, pairs, t, n_tiles, a.rows_cap);
        const uint8_t *sf0 = a.b_sf + (un.wrow0 >> 7) * k_atoms * 512;
        const uint8_t *sf1 = a.b_sf + (un.wrow1 >> 7) * k_atoms * 512;
        const uint32_t bytes = un.two ? kRawBytes : kRawBytes - kABytes;
        uint32_t st = p % RS, ph = (p / RS) & 1u;
        for (int kt = 0; kt < ksteps; ++kt, ++p) {
          if (!mbar_wait_bounded(&empty[st], ph ^ 1u, abort_flag, a.err, 530)) { ok = false; break; }
          uint8_t *raw = smem + (size_t)st * kRawBytes;
          mbar_arrive_expect_tx(&full[st], bytes);
          tma_load_2d(raw, &P.tmap_a, kt * BK, (int32_t)un.m0, &full[st]);
          if (un.two) tma_load_2d(raw + kABytes, &P.tmap_a, kt * BK, (int32_t)(un.m0 + BM), &full[st]);
          tma_load_2d(raw + kA2Bytes, &P.tmap_b, kt * (BK / 2), (int32_t)un.wrow0, &full[st]);
          tma_load_2d(raw + kA2Bytes + kCodesBytes / 2, &P.tmap_b, kt * (BK / 2), (int32_t)un.wrow1, &full[st]);
          bulk_load(raw + kA2Bytes + kCodesBytes, sf0 + (int64_t)kt * 512, 512, &full[st]);
          bulk_load(raw + kA2Bytes + kCodesBytes + 512, sf1 + (int64_t)kt * 512, 512, &full[st]);
          if (++st == RS) { st = 0; ph ^= 1u; }
        }
      }
      for (uint32_t q = p > RS ? p - RS : 0; q < p; ++q)
        mbar_wait_bounded(&full[q % RS], (q / RS) & 1u, never, a.err, 531);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------ MMA issuer
      const uint64_t dk = smem_desc(0, 16, 1024, 2);
      const uint32_t smem0 = smem_u32(smem);
      uint32_t p = 0, it = 0;
      bool ok = true;
      for (int64_t t = blockIdx.x; t < total && ok; t += gridDim.x, ++it) {
        const Unit un = unit_of<WN>(a, pairs, t, n_tiles, a.rows_cap);
        const uint32_t as = it % ACC;
        const uint32_t acc = tmem + as * kAccCols;
        if (!mbar_wait_bounded(&acc_empty[as], ((it / ACC) & 1u) ^ 1u, abort_flag, a.err, 540)) break;
        tc_fence_after();
        for (int kt = 0; kt < ksteps; ++kt, ++p) {
          const uint32_t st = p % RS, cs = p % CS;
          if (!mbar_wait_bounded(&full[st], (p / RS) & 1u, abort_flag, a.err, 541) ||
              !mbar_wait_bounded(&cfull[cs], (p / CS) & 1u, abort_flag, a.err, 542)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t a16 = (smem0 + st * (uint32_t)kRawBytes) >> 4;
          const uint64_t b16 = (smem0 + (uint32_t)kConvOff + cs * (uint32_t)kConvBytes) >> 4;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint32_t accum = (kt | kk) != 0 ? 1u : 0u;
            mma_bf16(acc, dk | (a16 + kk * 2), dk | (b16 + kk * 2), C::kIdesc, accum);
            if (un.two) mma_bf16(acc + WN, dk | (a16 + kABytes / 16 + kk * 2), dk | (b16 + kk * 2), C::kIdesc, accum);
          }
          tc_commit(&empty[st]);
          tc_commit(&cempty[cs]);
        }
        if (ok) tc_commit(&acc_full[as]);
      }
      tc_commit(drain);
      mbar_wait_bounded(drain, 0, never, a.err, 543);
    }
  } else if (warp >= kConvWarp0) {
    // ------------------------------------------------------- converters
    // Lane l of converter warp w covers K-half (l & 1) of the B rows
    // r = 16 (kHalfRowsPerLane w + j) + l/2, j < kHalfRowsPerLane (rows below
    // WN/2 from the first box, the rest from the second): its 16-byte code
    // loads are contiguous across the warp, and its 16-byte stores land in
    // distinct banks within every quarter warp under the 128-byte swizzle.
    constexpr int HR = C::kHalfRowsPerLane;
    const int cw = warp - kConvWarp0;
    const int hk = lane & 1;
    const uint32_t smem0 = smem_u32(smem);
    int r[HR];
    uint32_t code_off[HR], dst_off[HR][4];
#pragma unroll
    for (int j = 0; j < HR; ++j) {
      r[j] = 16 * (HR * cw + j) + (lane >> 1);
      code_off[j] = (uint32_t)(kA2Bytes + r[j] * 32 + hk * 16);
#pragma unroll
      for (int i = 0; i < 4; ++i)
        dst_off[j][i] = (uint32_t)(r[j] * 128) + ((uint32_t)((4 * hk + i) ^ (r[j] & 7)) << 4);
    }
    uint32_t p = 0;
    bool ok = true;
    for (int64_t t = blockIdx.x; t < total && ok; t += gridDim.x) {
      const Unit un = unit_of<WN>(a, pairs, t, n_tiles, a.rows_cap);
      // each row's place in its 128-row scale atom
      uint32_t sf_off[HR];
#pragma unroll
      for (int j = 0; j < HR; ++j) {
        const int half_box = r[j] / (WN / 2);
        const int ra = (int)(((half_box ? un.wrow1 : un.wrow0) & 127) + (r[j] % (WN / 2)));
        sf_off[j] = (uint32_t)(kA2Bytes + kCodesBytes + half_box * 512 + (ra & 31) * 16 + (ra >> 5) * 4 + 2 * hk);
      }
      for (int kt = 0; kt < ksteps; ++kt, ++p) {
        const uint32_t st = p % RS, cs = p % CS;
        if (!mbar_wait_bounded(&full[st], (p / RS) & 1u, abort_flag, a.err, 550) ||
            !mbar_wait_bounded(&cempty[cs], ((p / CS) & 1u) ^ 1u, abort_flag, a.err, 551)) {
          ok = false;
          break;
        }
        const uint32_t raw = smem0 + st * (uint32_t)kRawBytes;
        const uint32_t dst = smem0 + (uint32_t)kConvOff + cs * (uint32_t)kConvBytes;
        uint4 q[HR];
        uint32_t sc[HR];
#pragma unroll
        for (int j = 0; j < HR; ++j) {
          q[j] = ld_shared_v4(raw + code_off[j]);
          sc[j] = ld_shared_u16(raw + sf_off[j]);
        }
#pragma unroll
        for (int j = 0; j < HR; ++j) {
          uint32_t s2[2];
          ue4m3x2_to_bf16x2(sc[j], s2[0], s2[1]);
          const uint32_t cw4[4] = {q[j].x, q[j].y, q[j].z, q[j].w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            uint32_t w[4];
            e2m1x8_to_bf16x2(cw4[i], w);
#pragma unroll
            for (int u = 0; u < 4; ++u) w[u] = mul_bf16x2(w[u], s2[i >> 1]);
            st_shared_v4(dst + dst_off[j][i], w[0], w[1], w[2], w[3]);
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&cfull[cs]);
      }
    }
  } else if (warp >= w4::kEpiWarp0) {
    // -------------------------------------------------------- epilogue
    const int ew = warp - w4::kEpiWarp0;
    const int quad = warp & 3;
    const int half = ew >> 2;              // which m-tile of the unit
    const uint32_t tlane = tmem + ((uint32_t)(quad * 32) << 16);
    uint8_t *stg = smem + C::kStagingOff + (size_t)ew * kStagingPerWarp;
    const uint32_t stg_addr = smem_u32(stg);
    uint32_t chunk_id = 0, it = 0;
    auto store_box = [&](const uint32_t (&w16)[16], int32_t x, int32_t y) {
      const uint32_t box = stg_addr + (chunk_id & 1u) * 2048;
      if (lane == 0) bulk_wait_group_read<1>();
      __syncwarp();
      stage_row(box, lane, w16);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        tma_store_2d(&P.tmap_out, stg + (chunk_id & 1u) * 2048, x, y);
        bulk_commit_group();
      }
      ++chunk_id;
    };
    auto release = [&](uint32_t as) {
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[as]);
    };
    const int64_t rows_total = (int64_t)__ldg(a.offsets + a.E);
    for (int64_t t = blockIdx.x; t < total; t += gridDim.x, ++it) {
      const Unit un = unit_of<WN>(a, pairs, t, n_tiles, a.rows_cap);
      const uint32_t as = it % ACC;
      const float scale = __ldg(a.s_dec_w + un.e);
      if (!mbar_wait_bounded(&acc_full[as], (it / ACC) & 1u, abort_flag, a.err, 560)) break;
      tc_fence_after();
      if (half == 1 && !un.two) {            // a single-m-tile unit
        release(as);
        continue;
      }
      const uint32_t tacc = tlane + as * kAccCols + half * WN;
      const int64_t mrow0 = un.m0 + half * BM;
      if (a.epilogue == kBfSwiGLUFwd) {
        // gate columns [0, WN/2), up columns [WN/2, WN) of the unit; h
        // columns (WN/2) nt + [0, WN/2), every padded row of the slab
#pragma unroll 1
        for (int c = 0; c < WN / 64; ++c) {
          uint32_t vg[32], vu[32];
          tmem_ld_32cols(tacc + c * 32, vg);
          tmem_ld_32cols(tacc + WN / 2 + c * 32, vu);
          tmem_ld_wait();
          if (c == WN / 64 - 1) release(as);
          uint32_t w16[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            float hh[2];
#pragma unroll
            for (int q = 0; q < 2; ++q)
              hh[q] = silu_mul(__fmul_rn(__uint_as_float(vg[2 * i + q]), scale),
                               __fmul_rn(__uint_as_float(vu[2 * i + q]), scale));
            w16[i] = pack_bf16x2(hh[0], hh[1]);
          }
          const int32_t hcol = (int32_t)((WN / 2) * un.nt + c * 32);
          if (a.mxfp8_h) {
            // W4A8: the BF16 h of these 32 columns is one MXFP8 block
            if (a.h_pre != nullptr) {
              uint4 *dst = reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(a.h_pre) +
                                                     (mrow0 + quad * 32 + lane) * (a.N / 2) + hcol);
#pragma unroll
              for (int q = 0; q < 4; ++q)
                dst[q] = make_uint4(w16[4 * q], w16[4 * q + 1], w16[4 * q + 2], w16[4 * q + 3]);
            }
            float hv[32];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              hv[2 * i] = bf16_lo(w16[i]);
              hv[2 * i + 1] = bf16_hi(w16[i]);
            }
            mxfp8_qdq32(hv, w16);
          }
          store_box(w16, hcol, (int32_t)(mrow0 + quad * 32));
        }
      } else {
        const int64_t g_pad = __ldg(a.padded_offsets + un.e);
        const int64_t g_off = __ldg(a.offsets + un.e);
        const int64_t g_cnt = (int64_t)__ldg(a.offsets + un.e + 1) - g_off;
        const int64_t rel = mrow0 - g_pad + quad * 32 + lane;
        const bool valid = rel < g_cnt && g_off + rel < rows_total;
        const int64_t prow = mrow0 + quad * 32 + lane;
        const int64_t orow = a.out_padded ? prow : g_off + rel;
        const bool slab_full = a.out_padded || (mrow0 - g_pad) + quad * 32 + 32 <= g_cnt;
        const int64_t slab_row = a.out_padded ? mrow0 + quad * 32 : g_off + (mrow0 - g_pad) + quad * 32;
        const int64_t col0 = (int64_t)WN * un.nt;
#pragma unroll 1
        for (int c = 0; c < WN / 32; ++c) {
          uint32_t v[32];
          tmem_ld_32cols(tacc + c * 32, v);
          tmem_ld_wait();
          if (c == WN / 32 - 1) release(as);
          uint32_t w16[16];
#pragma unroll
          for (int i = 0; i < 16; ++i)
            w16[i] = pack_bf16x2(__fmul_rn(__uint_as_float(v[2 * i]), scale),
                                 __fmul_rn(__uint_as_float(v[2 * i + 1]), scale));
          if (slab_full) {
            store_box(w16, (int32_t)(col0 + c * 32), (int32_t)slab_row);
          } else if (valid) {
            uint4 *dst = reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(a.out_bf16) + orow * a.N + col0 +
                                                   c * 32);
#pragma unroll
            for (int q = 0; q < 4; ++q)
              dst[q] = make_uint4(w16[4 * q], w16[4 * q + 1], w16[4 * q + 2], w16[4 * q + 3]);
          }
        }
      }
    }
    if (lane == 0) bulk_wait_group_all();
    __syncwarp();
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace

template <int WN>
static cudaError_t launch_w4a16_cfg(const Bf16GemmArgs &a, cudaStream_t s) {
  using C = w4::Cfg<WN>;
  if (a.mode != kBfRows || a.b_mn || a.s_dec_w == nullptr || a.out_bf16 == nullptr || a.K % BK != 0 ||
      a.E < 1 || a.E > 1024 || (a.epilogue != kBfStore && a.epilogue != kBfSwiGLUFwd) ||
      (a.epilogue == kBfSwiGLUFwd && (!a.out_padded || a.N % 256 != 0)) || a.N % WN != 0)
    return cudaErrorInvalidValue;
  static thread_local int configured_device = -1;
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (configured_device != dev) {
    err = cudaFuncSetAttribute(k_w4a16_gemm<C>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::kSmemMax);
    if (err != cudaSuccess) return err;
    configured_device = dev;
  }
  BParams P;
  P.a = a;
  const auto BF = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  if (!encode_2d_map(&P.tmap_a, BF, 2, a.a, (uint64_t)a.K, (uint64_t)a.rows_cap, BK, BM, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  // weight codes: boxes of WN/2 rows x 32 bytes (one K-step of half a unit)
  if (!encode_2d_map(&P.tmap_b, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a.b, (uint64_t)(a.K / 2), (uint64_t)(a.E * a.N),
                     BK / 2, WN / 2, CU_TENSOR_MAP_SWIZZLE_NONE))
    return cudaErrorInvalidValue;
  const uint64_t out_cols = a.epilogue == kBfSwiGLUFwd ? (uint64_t)(a.N / 2) : (uint64_t)a.N;
  if (!encode_2d_map(&P.tmap_out, BF, 2, a.out_bf16, out_cols, (uint64_t)a.rows_cap, 32, 32,
                     CU_TENSOR_MAP_SWIZZLE_64B))
    return cudaErrorInvalidValue;
  // units: at most (m-tiles + experts) / 2 pairs times the weight-row tiles
  const int64_t units = ((a.rows_cap / BM + a.E) / 2 + 1) * (a.N / WN);
  int64_t grid = num_sms();
  if (grid > units) grid = units;
  if (grid < 1) grid = 1;
  const size_t smem = C::kPairsOff + 4 * (size_t)(a.E + 1) + 1024;
  k_w4a16_gemm<C><<<(unsigned)grid, w4::kThreads, smem, s>>>(P);
  return cudaGetLastError();
}

static cudaError_t launch_w4a16_gemm(const Bf16GemmArgs &a, cudaStream_t s) {
  return a.w4_wide ? launch_w4a16_cfg<256>(a, s) : launch_w4a16_cfg<128>(a, s);
}

cudaError_t launch_bf16_gemm(const Bf16GemmArgs &a, cudaStream_t s) {
  if (a.rows_cap <= 0 || a.N % BN != 0) return a.rows_cap <= 0 ? cudaSuccess : cudaErrorInvalidValue;
  if (a.b_sf != nullptr) return launch_w4a16_gemm(a, s);
  static thread_local int configured_device = -1;
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (configured_device != dev) {
    err = cudaFuncSetAttribute(k_bf16_gemm, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
    if (err != cudaSuccess) return err;
    configured_device = dev;
  }
  BParams P;
  P.a = a;
  const auto BF = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const auto SW = CU_TENSOR_MAP_SWIZZLE_128B;
  int64_t tiles;
  if (a.mode == kBfRows) {
    if (a.K % BK != 0) return cudaErrorInvalidValue;
    if (!encode_2d_map(&P.tmap_a, BF, 2, a.a, (uint64_t)a.K, (uint64_t)(a.a_rows ? a.a_rows : a.rows_cap), BK, BM, SW))
      return cudaErrorInvalidValue;
    if (a.b_mn) {
      if (!encode_2d_map(&P.tmap_b, BF, 2, a.b, (uint64_t)a.N, (uint64_t)(a.E * a.K), 64, BK, SW))
        return cudaErrorInvalidValue;
    } else {
      if (!encode_2d_map(&P.tmap_b, BF, 2, a.b, (uint64_t)a.K, (uint64_t)(a.b_rows ? a.b_rows : a.E * a.N), BK, BN, SW))
        return cudaErrorInvalidValue;
    }
    tiles = (a.rows_cap / BM) * (a.N / BN);
  } else {
    if (a.M % BM != 0) return cudaErrorInvalidValue;
    if (!encode_2d_map(&P.tmap_a, BF, 2, a.a, (uint64_t)a.M, (uint64_t)a.rows_cap, 64, BK, SW))
      return cudaErrorInvalidValue;
    if (!encode_2d_map(&P.tmap_b, BF, 2, a.b, (uint64_t)a.N, (uint64_t)a.rows_cap, 64, BK, SW))
      return cudaErrorInvalidValue;
    tiles = (int64_t)a.E * (a.M / BM) * (a.N / BN);
  }
  std::memset(&P.tmap_out, 0, sizeof(P.tmap_out));
  if (a.epilogue == kBfStore && a.out_bf16 != nullptr) {
    const uint64_t rows = a.mode == kBfRows ? (uint64_t)a.rows_cap : (uint64_t)(a.E * a.M);
    if (!encode_2d_map(&P.tmap_out, BF, 2, a.out_bf16, (uint64_t)a.N, rows, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B))
      return cudaErrorInvalidValue;
  }
  int64_t grid = num_sms();
  if (grid > tiles) grid = tiles;
  if (grid < 1) grid = 1;
  k_bf16_gemm<<<(unsigned)grid, kThreads, kSmemBytes, s>>>(P);
  return cudaGetLastError();
}

}  // namespace nvfp4moe
