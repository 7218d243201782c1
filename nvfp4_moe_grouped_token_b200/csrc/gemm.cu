// Persistent block-scaled NVFP4 grouped GEMM over the experts (sm_100a).
//
// The grouped matrix multiplication of the token-wise NVFP4 path
// (www.aib.vote "miniTE report, NVFP4 RL stability", paragraph 4) and the
// grouped GEMMs of the MoE learner (news.hamidun.com, "diagnostics, alignment
// and fast kernels").  One launch covers every expert; the group sizes are
// read on the device from padded_offsets, so the host never synchronizes.
//
// Design (B200):
//   * tile 128 x 256 x 256 (M x N x K elements) with one 256-column TMEM
//     accumulator, for both GEMMs (the SwiGLU epilogue needs the gate and up
//     halves of a 256-wide tile).  A rows come from the padded grouped
//     layout, where every expert's group starts on a 128-row boundary, so a
//     tile never straddles two experts.
//   * 16 warps in four warpgroups:
//       warps 0-3   scale feeders: per K-step, each reads its 32-row quarter of
//                   the stage's scales from shared memory, rebuilds the MMA
//                   atom order in registers and writes the stage's TMEM scale
//                   slot with tcgen05.st;
//       warp 4      TMA producer (one thread): A tile (16 KB) and B tile
//                   (32 KB) by 128-byte-swizzled tensor copies, A's 2 KB of
//                   K-step-major scales and B's 4 KB of scale atoms by bulk
//                   copies, into a 4-stage (gate_up, while the group
//                   offsets still fit) or 3-stage shared-memory ring;
//       warp 5      MMA issuer (one thread): tcgen05.mma kind::mxf4nvf4 with
//                   16-element UE4M3 scale blocks read from TMEM, FP32
//                   accumulation in TMEM; commits each stage back to the
//                   producer and the finished accumulator to the epilogue;
//       warps 6-7   requantization workers (SwiGLU GEMM with fused requant);
//       warps 8-15  epilogue: each reads its 32-lane quarter of the
//                   accumulator (half of the columns), releases TMEM at once
//                   so the next tile's MMAs overlap the rest of the epilogue,
//                   scales by S_dec_a(row) * S_dec_w(expert) and stores BF16
//                   (or FP32) rows through TMA tensor stores (32 x 64
//                   boxes), or applies SwiGLU (gate and up sit in the two
//                   128-column halves of a tile), stores h in BF16 (32 x 32
//                   boxes, or 32 x 16 with the 4-stage ring's 1 KB of
//                   staging) and max-reduces |h| per row.
//   * fused requantization (per-row scales): the CTA walks its m-tiles with
//     all their n-tiles in a row, so a row of h -- and its amax -- is
//     complete inside one CTA once the m-tile's last n-tile is stored.  The
//     epilogue warps then count the m-tile done (shared memory); the two
//     worker warps (and, once their tiles are over, the epilogue warps) copy
//     the m-tile's h back from L2 into shared memory in pieces, NVFP4-quantize
//     it with the row amax (amax reuse) and write codes, scales and S_dec,
//     while the MMAs run the next m-tile -- so h makes no separate trip
//     through HBM for the requantization.  Optionally the h lines are then
//     dropped from L2 without a write-back (discard.global.L2).
//   * persistent grid, one CTA per SM.  Without the fused requantization the
//     CTA walks tiles t = blockIdx.x, +gridDim.x, ... over (m-tile, n-tile)
//     with n fastest, so CTAs working at the same time share A tiles and
//     expert weights through L2.  Every role walks its tiles by additions
//     (the group advances by a forward scan): no per-tile division or search.
//   * every wait is bounded (common.cuh); a timeout records an error word and
//     the CTA drains its in-flight copies and MMAs before freeing TMEM.
#include <cudaTypedefs.h>

#include <cstring>
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace nvfp4moe {

namespace {

constexpr int BM = 128, BK = 256;
// 16 warps in four warpgroups: 0-3 scale feeders (one per TMEM lane quarter),
// 4 the TMA producer, 5 the MMA issuer, 6-7 the requantization workers, 8-15
// the epilogue.  setmaxnreg moves registers from the first two warpgroups to
// the epilogue: 128 * 80 + 128 * 64 + 256 * 184 = 65536 launched (512 * 128).
constexpr int kFeedWarps = 4;
constexpr int kEpiWarps = 8;
constexpr int kEpiWarp0 = 8;
constexpr int kWorkWarp0 = 6;
constexpr int kThreads = 512;
constexpr uint32_t kRegsFeed = 80, kRegsCtl = 64, kRegsEpi = 184;
static_assert(128 * kRegsFeed + 128 * kRegsCtl + 256 * kRegsEpi <= 65536, "register split");
constexpr uint32_t kTmemCols = 512;
// Epilogue staging per warp (default): two 2 KB buffers of 32 rows x 32 BF16
// (64-byte swizzle) for h, or one 4 KB box of 32 x 64 (128-byte swizzle) for
// D, drained to global memory by TMA tensor stores.  The 4-stage gate_up
// kernel stages 1 KB per warp instead (Cfg::kStaging).
constexpr int kStagingPerWarp = 4096;
// Rows per slab of h: the unit of the fused requantization.
constexpr int kSlabRows = 32;
// Bytes of h a worker warp copies into shared memory per step (a multiple of
// 128, so a group of four 16-element blocks never straddles two pieces), two
// pieces in flight per warp.
constexpr uint32_t kReqPiece = 5632;

template <int BN_, int STAGES_, int ACC_, bool SWIGLU_, bool FUSED_ = false, int STG_ = kStagingPerWarp>
struct Cfg {
  static constexpr int BN = BN_;
  static constexpr int STAGES = STAGES_;
  static constexpr int ACC = ACC_;                   // TMEM accumulator buffers
  // the epilogue this instantiation carries: SwiGLU (gate_up) or the plain
  // store / FP32 reduction (down); compiling only one keeps the other's
  // registers out of the kernel
  static constexpr bool SWIGLU = SWIGLU_;
  // with the requantization of h fused into the launch (opt-in)
  static constexpr bool FUSED = FUSED_;
  // epilogue staging per warp: 4 KB (two 32 x 32 boxes of h, or one 32 x 64
  // box of D), or 1 KB (one 32 x 16 box of h) to make room for a fourth stage
  static constexpr int kStaging = STG_;
  static constexpr int kABytes = BM * BK / 2;        // 16 KB of E2M1 codes
  static constexpr int kBBytes = BN * BK / 2;
  static constexpr int kSfaBytes = BM * BK / 16;     // four 512-byte atoms
  static constexpr int kNAtoms = BN / 128;           // 128-row scale atoms in B
  static constexpr int kSfbBytes = BN * BK / 16;
  static constexpr int kStageBytes = kABytes + kBBytes + kSfaBytes + kSfbBytes;
  // per pipeline stage a TMEM slot of scale factors: SFA (4 K-blocks x 4
  // columns) then SFB (4 K-blocks x 4*kNAtoms columns)
  static constexpr uint32_t kSfSlotCols = 16 + 16 * kNAtoms;
  static constexpr uint32_t kSfCol0 = ACC * BN;
  static constexpr int kColsPerWarp = BN / 2;        // two warps share a TMEM lane quarter
  static constexpr int kChunks = kColsPerWarp / 32;
  static constexpr size_t kStagingOff = (size_t)STAGES * kStageBytes;
  static constexpr size_t kBarrierOff = kStagingOff + (size_t)kEpiWarps * kStaging;
  // fused requantization: each worker warp stages h through two buffers
  static constexpr size_t kReqOff = kBarrierOff + 512;   // barriers and flags: 512 bytes
  static constexpr size_t kOffsetsOff = kReqOff + (FUSED ? 4 * (size_t)kReqPiece : 0);
  // + up to 1023 bytes lost to aligning the dynamic shared memory to 1 KB
  static constexpr size_t kSmemFixed = kOffsetsOff + 1024;
  // the group offsets (two int32 per group) take the rest: up to kMaxE groups
  static constexpr int kMaxE = (int)((232448 - kSmemFixed) / 8) - 1;
  static constexpr size_t kSmemMax = kSmemFixed + (size_t)8 * (kMaxE + 1);
  // Instruction descriptor, kind::mxf4nvf4: A and B E2M1 (format 1), K-major,
  // UE4M3 scales (bit 23 = 0), N >> 3 at bit 17, M >> 4 at bit 24, dense, K = 64.
  static constexpr uint32_t kIdesc = (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
                                     ((uint32_t)(BM >> 4) << 24);
  static_assert(ACC * BN + STAGES * (16 + 16 * kNAtoms) <= (int)kTmemCols, "TMEM budget");
  static_assert(kMaxE >= 128 && kSmemMax <= 232448, "shared memory budget");
  static_assert(kStaging == 4096 || (kStaging == 1024 && SWIGLU && !FUSED), "staging layout");
  static_assert((3 * STAGES + 2 * ACC + 1) * 8 + 12 <= 192, "pipeline barriers overrun their area");
};

using CfgGateUp = Cfg<256, 3, 1, true>;
using CfgGateUp4 = Cfg<256, 4, 1, true, false, 1024>;
using CfgGateUpFused = Cfg<256, 3, 1, true, true>;
using CfgDown = Cfg<256, 3, 1, false>;

struct __align__(64) KParams {
  CUtensorMap tmap_a;
  CUtensorMap tmap_b;
  CUtensorMap tmap_out;   // BF16 output (D or h), 32 x 32 boxes, 64-byte swizzle
  GemmArgs a;
};

// Write one lane's 32 BF16 values (16 packed words) as row `lane` of a
// 32 x 32 staging box in the 64-byte swizzle the output tensor map uses:
// 16-byte chunk q of row r sits at chunk q ^ ((r >> 1) & 3).
__device__ __forceinline__ void stage_row(uint32_t box_addr, int lane, const uint32_t (&w)[16]) {
  const uint32_t base = box_addr + (uint32_t)lane * 64;
  const uint32_t sw = ((uint32_t)lane >> 1) & 3u;
#pragma unroll
  for (int q = 0; q < 4; ++q)
    st_shared_v4(base + (((uint32_t)q ^ sw) << 4), w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
}

__device__ __forceinline__ float fmax_abs_bf16(float m, uint32_t packed) {
  return fmaxf(m, fmaxf(fabsf(bf16_lo(packed)), fabsf(bf16_hi(packed))));
}

__device__ __forceinline__ uint32_t ld_volatile_u32(const uint32_t *p) {
  return *reinterpret_cast<const volatile uint32_t *>(p);
}

// Fused requantization bookkeeping, per CTA, in shared memory:
//   mt_done     +1 by each epilogue warp once its h stores and row-amax
//               updates for one of the CTA's m-tiles are complete (so the j-th
//               m-tile is ready when mt_done >= 8 (j + 1))
//   slab_next   slabs of the CTA's m-tiles claimed so far (4 per m-tile)
// Claim the CTA's next slab (one thread): returns its index k (m-tile k / 4
// of this CTA, slab k % 4 of it) once that m-tile is ready, or -1 when none
// is left (or the kernel is aborting).
__device__ __forceinline__ int64_t claim_slab(uint32_t *slab_next, const uint32_t *mt_done, int64_t nslabs,
                                              volatile int *abort_flag, int *err) {
  const int64_t k = atomicAdd(slab_next, 1u);
  if (k >= nslabs) return -1;
  const uint32_t need = (uint32_t)(kEpiWarps * (k / (BM / kSlabRows) + 1));
  if (ld_volatile_u32(mt_done) >= need) return k;
  const uint64_t t0 = global_timer_ns();
  for (uint32_t i = 1;; ++i) {
    __nanosleep(200);
    if (ld_volatile_u32(mt_done) >= need) return k;
    if ((i & 15u) == 0) {
      if (*abort_flag) return -1;
      if (global_timer_ns() - t0 > kWaitTimeoutNs) {
        set_device_error(err, kDevTimeout, 402);
        *abort_flag = 1;
        return -1;
      }
    }
  }
}

// NVFP4 quantization of one 16-element block of BF16 values (two uint4) under
// the row's S_enc, one binary32 operation per step, round to nearest even:
// sf = UE4M3((bamax / 6) * S_enc), code = E2M1(x * (S_enc / sf)), all +0
// when sf == 0.
__device__ __forceinline__ uint32_t encode_block16(const uint4 &v0, const uint4 &v1, float s_enc,
                                                   uint2 &codes) {
  const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
  __nv_bfloat162 m2 = __habs2(*reinterpret_cast<const __nv_bfloat162 *>(&w[0]));
#pragma unroll
  for (int j = 1; j < 8; ++j) m2 = __hmax2(m2, __habs2(*reinterpret_cast<const __nv_bfloat162 *>(&w[j])));
  const float bamax = fmaxf(__low2float(m2), __high2float(m2));
  const uint32_t sfc = cvt_ue4m3(__fmul_rn(__fdiv_rn(bamax, 6.0f), s_enc));
  codes = make_uint2(0, 0);
  if (sfc != 0) {
    const float rr = __fdiv_rn(s_enc, ue4m3_value(sfc));
    float y[8];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      y[2 * j] = __fmul_rn(bf16_lo(w[j]), rr);
      y[2 * j + 1] = __fmul_rn(bf16_hi(w[j]), rr);
    }
    codes.x = cvt_e2m1x8(y);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      y[2 * j] = __fmul_rn(bf16_lo(w[4 + j]), rr);
      y[2 * j + 1] = __fmul_rn(bf16_hi(w[4 + j]), rr);
    }
    codes.y = cvt_e2m1x8(y);
  }
  return sfc;
}

// Shared-memory staging of one warp for the requantization: two buffers of
// `piece` bytes with one mbarrier each; `loads[i]` counts the copies that
// buffer i has received (its barrier's phase), across slabs.
struct ReqStage {
  uint8_t *buf[2];
  uint64_t *bar[2];
  uint32_t piece;
  uint32_t loads[2];
};

// Requantize the 32 rows of h slab `slab` (rows slab*32 ..) with their
// per-row amax (reduced by the epilogue: amax reuse), one warp.  The slab's
// 32 rows are one contiguous run of 32 * I BF16; it is copied into shared
// memory in pieces (bulk copies, the next piece landing while this one is
// encoded), so the warp keeps whole pieces in flight instead of one row.  A
// row whose amax is 0 (a padding row, or an all-zero row) gets zero codes,
// zero scales and S_dec = 1.  Writes codes [rows][I/2], scales in the
// K-step-major layout and the row S_dec; then, if asked, drops the slab's h
// lines from L2 without writing them back.
__device__ __noinline__ void requant_slab(const GemmArgs &a, int32_t slab, int lane, ReqStage &rs,
                                          volatile int *abort_flag) {
  const int64_t I = a.N >> 1;
  const uint32_t nblk = (uint32_t)(I >> 4);
  const int64_t row0 = (int64_t)slab * kSlabRows;
  const uint8_t *src = reinterpret_cast<const uint8_t *>(static_cast<const __nv_bfloat16 *>(a.out_bf16) + row0 * I);
  const uint32_t total = (uint32_t)(kSlabRows * I * 2);
  const uint32_t npieces = (total + rs.piece - 1) / rs.piece;
  // lane r: the global scales of row row0 + r
  float my_enc, my_dec;
  const float my_amax = __ldcg(a.amax_h + row0 + lane);
  global_scales(my_amax, my_enc, my_dec);
  a.req_s_dec[row0 + lane] = my_dec;
  // the h just published by other CTAs is read through the async proxy
  asm volatile("fence.proxy.async.global;" ::: "memory");
  auto issue = [&](uint32_t pc) {
    if (lane == 0) {
      const uint32_t bi = pc & 1u;
      const uint32_t off = pc * rs.piece;
      const uint32_t n = total - off < rs.piece ? total - off : rs.piece;
      mbar_arrive_expect_tx(rs.bar[bi], n);
      bulk_load(rs.buf[bi], src + off, n, rs.bar[bi]);
    }
  };
  issue(0);
  for (uint32_t pc = 0; pc < npieces; ++pc) {
    const uint32_t bi = pc & 1u;
    if (pc + 1 < npieces) issue(pc + 1);     // into the buffer read in the previous step
    const bool ok = mbar_wait_bounded(rs.bar[bi], rs.loads[bi] & 1u, abort_flag, a.err, 403);
    ++rs.loads[bi];
    if (!__all_sync(0xffffffffu, ok)) {
      if (pc + 1 < npieces) {               // let the copy in flight land before leaving
        int never = 0;
        mbar_wait_bounded(rs.bar[bi ^ 1u], rs.loads[bi ^ 1u] & 1u, &never, a.err, 404);
        ++rs.loads[bi ^ 1u];
      }
      return;
    }
    const uint32_t off = pc * rs.piece;
    const uint32_t n = total - off < rs.piece ? total - off : rs.piece;
    const uint32_t nb = n / 32;            // 16-element blocks in this piece
    const uint4 *pbuf = reinterpret_cast<const uint4 *>(rs.buf[bi]);
    // two blocks per lane per step (blk and blk + 32): independent chains
    // the scheduler can interleave
    for (uint32_t j0 = 0; j0 < nb; j0 += 64) {
      uint2 codes[2];
      uint32_t sfc[2], rr[2], bb[2];
      bool valid[2];
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const uint32_t blk = j0 + 32 * u + (uint32_t)lane;
        valid[u] = blk < nb;
        const uint32_t gb = off / 32 + blk;    // block index inside the slab
        rr[u] = valid[u] ? gb / nblk : 0;
        bb[u] = gb - rr[u] * nblk;
      }
      float s_enc[2];
      bool live[2];
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        s_enc[u] = __shfl_sync(0xffffffffu, my_enc, (int)rr[u]);
        live[u] = __shfl_sync(0xffffffffu, my_amax, (int)rr[u]) > 0.0f;
      }
      uint4 v[2][2];
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        v[u][0] = make_uint4(0, 0, 0, 0);
        v[u][1] = v[u][0];
        if (valid[u] && live[u]) {
          const uint32_t blk = j0 + 32 * u + (uint32_t)lane;
          v[u][0] = pbuf[blk * 2];
          v[u][1] = pbuf[blk * 2 + 1];
        }
      }
#pragma unroll
      for (int u = 0; u < 2; ++u) sfc[u] = encode_block16(v[u][0], v[u][1], s_enc[u], codes[u]);
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        if (j0 + 32 * u >= nb) break;          // warp-uniform
        // the four scales of blocks 4i..4i+3 (one row: pieces and nblk are
        // multiples of 4 blocks) sit in lanes 4i..4i+3
        const int q4 = lane & ~3;
        const uint32_t s0 = __shfl_sync(0xffffffffu, sfc[u], q4);
        const uint32_t s1 = __shfl_sync(0xffffffffu, sfc[u], q4 + 1);
        const uint32_t s2 = __shfl_sync(0xffffffffu, sfc[u], q4 + 2);
        const uint32_t s3 = __shfl_sync(0xffffffffu, sfc[u], q4 + 3);
        if (valid[u]) {
          const int64_t row = row0 + rr[u];
          const uint32_t b = bb[u];
          *reinterpret_cast<uint2 *>(a.req_q + row * (I >> 1) + (int64_t)b * 8) = codes[u];
          if ((lane & 3) == 0)
            *reinterpret_cast<uint32_t *>(a.req_sf + (((int64_t)(b >> 4) * a.rows_cap + row) * 16 + (b & 15))) =
                s0 | (s1 << 8) | (s2 << 16) | (s3 << 24);
        }
      }
    }
    __syncwarp();                            // this buffer is free for piece pc + 2
  }
  if (a.discard_h) {
    const int64_t lines = (int64_t)total / 128;
    for (int64_t i = lane; i < lines; i += 32)
      asm volatile("discard.global.L2 [%0], 128;" ::"l"(src + i * 128) : "memory");
  }
}

template <class C>
__global__ void __launch_bounds__(kThreads, 1) k_grouped_gemm(const __grid_constant__ KParams P) {
  constexpr int BN = C::BN, STAGES = C::STAGES, ACC = C::ACC;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + C::kBarrierOff);
  uint64_t *empty = full + STAGES;
  uint64_t *sf_full = empty + STAGES;
  uint64_t *acc_full = sf_full + STAGES;
  uint64_t *acc_empty = acc_full + ACC;
  uint64_t *drain = acc_empty + ACC;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
  int *never = reinterpret_cast<int *>(tmem_slot + 2);   // an abort flag nothing raises
  // barrier area: pipeline barriers and flags [0, 192), the fused
  // requantization's worker barriers [192, 224), its epilogue-warp barriers
  // [224, 352), its counters at 384
  uint64_t *req_bar = reinterpret_cast<uint64_t *>(smem + C::kBarrierOff + 192);   // [2 workers][2]
  uint32_t *mt_done = reinterpret_cast<uint32_t *>(smem + C::kBarrierOff + 384);
  uint32_t *slab_next = mt_done + 1;
  int32_t *s_pad = reinterpret_cast<int32_t *>(smem + C::kOffsetsOff);
  int32_t *s_off = s_pad + (P.a.E + 1);

  const GemmArgs &a = P.a;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // requantize h inside this launch (SwiGLU epilogue, per-row amax)
  const bool fused_requant = C::FUSED && a.req_q != nullptr && a.amax_h != nullptr &&
                             a.amax_h_rows != 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
      mbar_init(&sf_full[s], kFeedWarps);
    }
    for (int s = 0; s < ACC; ++s) {
      mbar_init(&acc_full[s], 1);
      mbar_init(&acc_empty[s], kEpiWarps);
    }
    mbar_init(drain, 1);
    for (int i = 0; i < 4; ++i) mbar_init(&req_bar[i], 1);
    *mt_done = 0;
    *slab_next = 0;
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
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  for (int i = threadIdx.x; i <= a.E; i += blockDim.x) {
    s_pad[i] = __ldg(a.padded_offsets + i);
    s_off[i] = __ldg(a.offsets + i);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  const int n_tiles = (int)(a.N / BN);
  const int kt_count = (int)(a.K / BK);
  // never walk past the rows the caller allocated, whatever the offsets say
  int64_t rows_used = s_pad[a.E];
  if (rows_used > a.rows_cap) rows_used = a.rows_cap;
  if (rows_used < 0) rows_used = 0;
  const int64_t total = (rows_used / BM) * n_tiles;
  const int64_t rows_total = s_off[a.E];
  const int64_t k_atoms = a.K >> 6;      // 512-byte scale atoms per 128 rows

  const uint32_t smem0 = smem_u32(smem);
  // Tile order.  Default: t = blockIdx.x, +gridDim.x, ... over (m-tile,
  // n-tile) with n fastest, so the CTAs running together share A tiles and
  // expert weights through L2.  With the fused requantization: m-tile-major
  // per CTA (m-tiles blockIdx.x, +gridDim.x, ..., each with all its n-tiles in
  // order), so every row of h is completed by one CTA.
  const int64_t m_total = rows_used / BM;
  const bool m_major = fused_requant;
  const int64_t my_mtiles = m_total > (int64_t)blockIdx.x ? (m_total - 1 - blockIdx.x) / gridDim.x + 1 : 0;
  const int64_t my_tiles = m_major ? my_mtiles * n_tiles
                                   : (total > (int64_t)blockIdx.x ? (total - 1 - blockIdx.x) / gridDim.x + 1 : 0);
  // The walk over the CTA's tiles advances by additions, and the m-tile's
  // group by a short forward scan (m-tiles only grow along the walk): a
  // division and a binary search per tile cost the epilogue warps, which
  // redo them for every tile, a sizeable share of their time.
  struct TileWalk {
    int64_t mt;
    int nt;
    int e;
  };
  const int walk_dm = (int)(gridDim.x / n_tiles), walk_dn = (int)(gridDim.x % n_tiles);
  auto walk_group = [&](TileWalk &w) {
    while (w.e + 1 < a.E && (int64_t)s_pad[w.e + 1] <= w.mt * BM) ++w.e;
  };
  auto walk_start = [&]() {
    TileWalk w;
    w.mt = m_major ? (int64_t)blockIdx.x : (int64_t)(blockIdx.x / n_tiles);
    w.nt = m_major ? 0 : (int)(blockIdx.x % n_tiles);
    w.e = 0;
    walk_group(w);
    return w;
  };
  auto walk_next = [&](TileWalk &w) {
    if (m_major) {
      if (++w.nt == n_tiles) {
        w.nt = 0;
        w.mt += gridDim.x;
      }
    } else {
      w.mt += walk_dm;
      w.nt += walk_dn;
      if (w.nt >= n_tiles) {
        w.nt -= n_tiles;
        ++w.mt;
      }
    }
    walk_group(w);
  };
  const uint32_t steps = (uint32_t)(my_tiles * kt_count);

  if (warp < kFeedWarps) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsFeed));
    // --------------------------------------------------------- feeders
    // For every K-step: wait for the stage's TMA data, build this lane's
    // records of the stage's scales and write them into the stage's TMEM
    // scale slot with tcgen05.st (the MMA reads scales from TMEM).  The slot
    // holds the MMA atom layout: for K-block group kb (4 scale blocks), lane i
    // of every 32-lane quarter carries rows i, i+32, i+64, i+96.  A's scales
    // arrive as 128 rows x 16 bytes, so lane i reads those four 16-byte rows
    // and the 4x4 word transpose is a register renaming; B's arrive as atoms.  tcgen05.st
    // runs an order of magnitude faster than tcgen05.cp for these small
    // copies and overlaps the MMAs.
    const uint32_t tq = tmem + ((uint32_t)(warp * 32) << 16);
    uint32_t st = 0, ph = 0;
    for (uint32_t g = 0; g < steps; ++g, st = (st + 1 == STAGES) ? 0 : st + 1, ph ^= (st == 0)) {
      const bool ok = mbar_wait_bounded(&full[st], ph, abort_flag, a.err, 110 + warp);
      if (!__all_sync(0xffffffffu, ok)) break;
      const uint4 *sfa = reinterpret_cast<const uint4 *>(smem + (size_t)st * C::kStageBytes + C::kABytes +
                                                         C::kBBytes);
      const uint4 *sfb = sfa + C::kSfaBytes / 16;
      uint32_t w[C::kSfSlotCols];
#pragma unroll
      for (int j = 0; j < 4; ++j) {          // row lane + 32 j: 16 scales = word kb for group kb
        const uint4 v = sfa[j * 32 + lane];
        w[j] = v.x; w[4 + j] = v.y; w[8 + j] = v.z; w[12 + j] = v.w;
      }
#pragma unroll
      for (int kb = 0; kb < 4; ++kb) {
#pragma unroll
        for (int h = 0; h < C::kNAtoms; ++h) {
          const uint4 v = sfb[h * 128 + kb * 32 + lane];
          const int o = 16 + 4 * C::kNAtoms * kb + 4 * h;
          w[o] = v.x; w[o + 1] = v.y; w[o + 2] = v.z; w[o + 3] = v.w;
        }
      }
      const uint32_t slot = tq + C::kSfCol0 + st * C::kSfSlotCols;
#pragma unroll
      for (int c = 0; c < (int)C::kSfSlotCols / 16; ++c)
        tmem_st_16cols(slot + 16 * c, *reinterpret_cast<const uint32_t (*)[16]>(&w[16 * c]));
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sf_full[st]);
    }
  } else if (warp < kEpiWarp0) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsCtl));
    if (warp == 4 && lane == 0) {
      // ---------------------------------------------------- TMA producer
      // a single thread: tile coordinates are computed once per tile and the
      // per-step addresses advance by additions (a division or a search per
      // step costs this thread hundreds of cycles of latency)
      uint32_t p = 0;
      bool ok = true;
      TileWalk w = walk_start();
      for (int64_t i = 0; i < my_tiles && ok; ++i, walk_next(w)) {
        const int64_t mt = w.mt;
        const int nt = w.nt;
        const int e = w.e;
        const int32_t arow = (int32_t)(mt * BM);
        const int32_t wrow0 = (int32_t)((int64_t)e * a.N + (int64_t)nt * BN);
        const uint8_t *sfa_src = a.sf_a + mt * BM * 16;   // K-step 0 of the tile's rows
        const int64_t sfa_step = a.rows_cap * 16;           // one K-step further
        const uint8_t *sfb_src = a.sf_w + ((int64_t)e * (a.N >> 7) + C::kNAtoms * nt) * k_atoms * 512;
        const int64_t sfb_h = k_atoms * 512;
        uint32_t st = p % STAGES, ph = (p / STAGES) & 1u;
        for (int kt = 0; kt < kt_count; ++kt, ++p) {
          if (!mbar_wait_bounded(&empty[st], ph ^ 1u, abort_flag, a.err, 100)) { ok = false; break; }
          uint8_t *sb = smem + (size_t)st * C::kStageBytes;
          mbar_arrive_expect_tx(&full[st], C::kStageBytes);
          tma_load_2d(sb, &P.tmap_a, kt * (BK / 2), arow, &full[st]);
          tma_load_2d(sb + C::kABytes, &P.tmap_b, kt * (BK / 2), wrow0, &full[st]);
          bulk_load(sb + C::kABytes + C::kBBytes, sfa_src, C::kSfaBytes, &full[st]);
          sfa_src += sfa_step;
#pragma unroll
          for (int h = 0; h < C::kNAtoms; ++h)
            bulk_load(sb + C::kABytes + C::kBBytes + C::kSfaBytes + h * 2048, sfb_src + h * sfb_h, 2048,
                      &full[st]);
          sfb_src += 2048;
          if (++st == STAGES) { st = 0; ph ^= 1u; }
        }
      }
      // drain: every copy issued has landed before the CTA exits (in normal
      // operation the feeders consumed them all; this matters after an abort)
      for (uint32_t q = p > STAGES ? p - STAGES : 0; q < p; ++q)
        mbar_wait_bounded(&full[q % STAGES], (q / STAGES) & 1u, never, a.err, 101);
    } else if (warp == 5 && lane == 0) {
      // ------------------------------------------------------ MMA issuer
      const uint64_t op_desc0 = smem_desc(0, 16, 1024, 2);   // K-major, 128-byte swizzle
      uint32_t st = 0, ph = 0, it = 0;
      bool ok = true;
      for (int64_t i = 0; i < my_tiles && ok; ++i, ++it) {
        const uint32_t as = it % ACC;
        const uint32_t acc = tmem + as * BN;
        if (!mbar_wait_bounded(&acc_empty[as], ((it / ACC) & 1u) ^ 1u, abort_flag, a.err, 200)) break;
        for (int kt = 0; kt < kt_count; ++kt) {
          if (!mbar_wait_bounded(&sf_full[st], ph, abort_flag, a.err, 201)) { ok = false; break; }
          tc_fence_after();
          // only the start-address field (address >> 4) differs between descriptors
          const uint64_t a16 = (smem0 + st * (uint32_t)C::kStageBytes) >> 4;
          const uint64_t b16 = a16 + C::kABytes / 16;
          const uint32_t sf = tmem + C::kSfCol0 + st * C::kSfSlotCols;
#pragma unroll
          for (int kb = 0; kb < 4; ++kb)
            mma_nvfp4(acc, op_desc0 | (a16 + kb * 2), op_desc0 | (b16 + kb * 2), C::kIdesc, sf + 4 * kb,
                      sf + 16 + 4 * C::kNAtoms * kb, (kt | kb) != 0 ? 1u : 0u);
          tc_commit(&empty[st]);
          if (++st == STAGES) { st = 0; ph ^= 1u; }
        }
        if (ok) tc_commit(&acc_full[as]);
      }
      // drain: all MMAs this thread issued have completed
      tc_commit(drain);
      mbar_wait_bounded(drain, 0, never, a.err, 202);
    } else if (warp >= kWorkWarp0 && fused_requant) {
      // ------------------------------------------- requantization workers
      const int64_t nslabs = my_mtiles * (BM / kSlabRows);
      const int wk = warp - kWorkWarp0;
      ReqStage rs;
      rs.buf[0] = smem + C::kReqOff + (2 * wk) * (size_t)kReqPiece;
      rs.buf[1] = rs.buf[0] + kReqPiece;
      rs.bar[0] = &req_bar[2 * wk];
      rs.bar[1] = &req_bar[2 * wk + 1];
      rs.piece = kReqPiece;
      rs.loads[0] = rs.loads[1] = 0;
      for (;;) {
        int64_t k = -1;
        if (lane == 0) k = claim_slab(slab_next, mt_done, nslabs, abort_flag, a.err);
        k = __shfl_sync(0xffffffffu, k, 0);
        if (k < 0) break;
        __threadfence_block();   // pairs with the epilogue warps' release of mt_done
        const int64_t mt = (int64_t)blockIdx.x + (k / (BM / kSlabRows)) * gridDim.x;
        requant_slab(a, (int32_t)(mt * (BM / kSlabRows) + k % (BM / kSlabRows)), lane, rs, abort_flag);
      }
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsEpi));
    // -------------------------------------------------------- epilogue
    const int ew = warp - kEpiWarp0;
    const int quad = warp & 3;              // TMEM lanes this warp may read
    const int half = ew >> 2;               // which half of the columns
    const int rit = quad * 32 + lane;       // row inside the tile
    const uint32_t tlane = tmem + ((uint32_t)(quad * 32) << 16);
    uint8_t *stg = smem + C::kStagingOff + (size_t)ew * C::kStaging;
    const uint32_t stg_addr = smem_u32(stg);
    uint32_t chunk_id = 0;
    uint32_t it = 0;
    // stage 32 BF16 of this lane's row, then lane 0 stores the 32 x 32 box
    auto store_box = [&](const uint32_t (&w16)[16], int32_t x, int32_t y) {
      const uint32_t box = stg_addr + (chunk_id & 1u) * 2048;
      if (lane == 0) bulk_wait_group_read<1>();   // the buffer's previous store has read it
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
    // with 1 KB of staging: a 32 x 16 box (32-byte rows, no swizzle) of 8
    // packed words per lane, one buffer
    auto store_box16 = [&](const uint32_t *w8, int32_t x, int32_t y) {
      if (lane == 0) bulk_wait_group_read<0>();   // the buffer's previous store has read it
      __syncwarp();
      st_shared_v4(stg_addr + (uint32_t)lane * 32, w8[0], w8[1], w8[2], w8[3]);
      st_shared_v4(stg_addr + (uint32_t)lane * 32 + 16, w8[4], w8[5], w8[6], w8[7]);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        tma_store_2d(&P.tmap_out, stg, x, y);
        bulk_commit_group();
      }
    };
    // fused requantization: the warp's |h| maxima of a row are kept across
    // the n-tiles of an m-tile and folded into the row amax at its last
    // n-tile.  One tile later (its older bulk groups are then complete) lane
    // 0 makes the m-tile's h stores and amax updates visible and bumps
    // mt_done; the warp barrier before it orders every lane's updates.
    auto signal_mtile = [&](bool keep_two) {
      if (lane == 0) {
        if (keep_two) bulk_wait_group<2>(); else bulk_wait_group<0>();
        asm volatile("fence.proxy.async.global;" ::: "memory");
        __threadfence_block();
        atomicAdd(mt_done, 1u);
      }
      __syncwarp();
    };
    float row_amax = 0.0f;
    bool pending_mtile = false;
    TileWalk w = walk_start();
    for (int64_t i = 0; i < my_tiles; ++i, ++it, walk_next(w)) {
      const int64_t mt = w.mt;
      const int nt = w.nt;
      const int64_t row0 = mt * BM;
      const int e = w.e;
      const int64_t g_pad = s_pad[e];
      const int64_t g_off = s_off[e];
      const int64_t g_cnt = (int64_t)s_off[e + 1] - g_off;
      const int64_t rel = row0 - g_pad + rit;
      const bool valid = rel < g_cnt && g_off + rel < rows_total;
      const int64_t prow = row0 + rit;
      // scale loads issued before the wait so their latency hides under the MMAs
      const float sa = valid ? __ldg(a.s_dec_a + (a.s_dec_a_rows ? prow : 0)) : 0.0f;
      const float sw = __ldg(a.s_dec_w + e);
      const uint32_t as = it % ACC;

      if (!mbar_wait_bounded(&acc_full[as], (it / ACC) & 1u, abort_flag, a.err, 300)) break;
      tc_fence_after();
      uint32_t v[C::kChunks][32];
      const uint32_t tacc = tlane + as * BN;
      if constexpr (C::SWIGLU) {
        // gate columns [half*64, +64) and up columns [128 + half*64, +64)
#pragma unroll
        for (int c = 0; c < C::kChunks; ++c)
          tmem_ld_32cols(tacc + (c >> 1) * 128 + half * 64 + (c & 1) * 32, v[c]);
      } else {
#pragma unroll
        for (int c = 0; c < C::kChunks; ++c) tmem_ld_32cols(tacc + half * C::kColsPerWarp + c * 32, v[c]);
      }
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[as]);

      const float scale = __fmul_rn(sa, sw);
      // rows of this warp's 32-row slab all belong to the group?
      const bool slab_full = (row0 - g_pad) + quad * 32 + 32 <= g_cnt;
      if constexpr (C::SWIGLU) {
        float m = 0.0f;
        // h rows live at padded positions: the whole slab is stored (rows past
        // the group's end are padding that nothing reads); each 32-column
        // chunk is stored as soon as it is computed, which keeps the
        // epilogue's registers within its share
        auto swiglu = [&](auto silu2) {
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            uint32_t hp[16];
#pragma unroll
            for (int i = 0; i < 32; i += 2) {
              float hh[2], g[2], u[2];
              scale2(v[c][i], v[c][i + 1], scale, g[0], g[1]);
              scale2(v[(c + 2) % C::kChunks][i], v[(c + 2) % C::kChunks][i + 1], scale, u[0], u[1]);
              silu2(g[0], g[1], u[0], u[1], hh[0], hh[1]);
              hp[i / 2] = pack_bf16x2(hh[0], hh[1]);
              m = fmax_abs_bf16(m, hp[i / 2]);
            }
            const int32_t hx = (int32_t)(nt * 128 + half * 64 + c * 32), hy = (int32_t)(row0 + quad * 32);
            if constexpr (C::kStaging == 1024) {
              store_box16(hp, hx, hy);
              store_box16(hp + 8, hx + 16, hy);
            } else {
              store_box(hp, hx, hy);
            }
          }
        };
        // the fast SwiGLU form unless some gate value of the warp's tile
        // part is below -64 (scale >= 0, so the minimum decides)
        float gmin = __uint_as_float(v[0][0]);
#pragma unroll
        for (int c = 0; c < 2; ++c)
#pragma unroll
          for (int i = 0; i < 32; ++i) gmin = fminf(gmin, __uint_as_float(v[c][i]));
        if (__any_sync(0xffffffffu, __fmul_rn(gmin, scale) < -64.0f))
          swiglu([](float g0, float g1, float u0, float u1, float &h0, float &h1) {
            h0 = silu_mul(g0, u0);
            h1 = silu_mul(g1, u1);
          });
        else
          swiglu([](float g0, float g1, float u0, float u1, float &h0, float &h1) {
            silu_mul_fast2(g0, g1, u0, u1, h0, h1);
          });
        if (a.amax_h != nullptr) {
          if (a.amax_h_rows) {
            if (!fused_requant) {
              if (valid) atomicMax(reinterpret_cast<unsigned int *>(a.amax_h + prow), __float_as_uint(m));
            } else {
              row_amax = fmaxf(row_amax, m);
              __syncwarp();
              // this tile's two boxes are the newest bulk groups
              if (pending_mtile) signal_mtile(true);
              pending_mtile = false;
              if (nt == n_tiles - 1) {
                if (valid) atomicMax(reinterpret_cast<unsigned int *>(a.amax_h + prow), __float_as_uint(row_amax));
                row_amax = 0.0f;
                pending_mtile = true;
              }
            }
          } else {
            float mm = valid ? m : 0.0f;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) mm = fmaxf(mm, __shfl_xor_sync(0xffffffffu, mm, o));
            if (lane == 0 && mm > 0.0f)
              atomicMax(reinterpret_cast<unsigned int *>(a.amax_h), __float_as_uint(mm));
          }
        }
      } else if (a.red_y != nullptr) {
        // non-strict combine: y[t] += w[t][j] * D_row in FP32 reductions, in
        // whatever order the tiles finish (not bitwise reproducible)
        if (valid) {
          const int32_t slot = __ldg(a.red_perm + g_off + rel);
          const float wgt = __fmul_rn(__ldg(a.red_w + slot), scale);
          float *dst = a.red_y + (int64_t)(slot / a.red_k) * a.N + (int64_t)nt * BN + half * C::kColsPerWarp;
#pragma unroll
          for (int c = 0; c < C::kChunks; ++c)
#pragma unroll
            for (int i = 0; i < 32; i += 4)
              asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(dst + c * 32 + i),
                           "f"(__fmul_rn(__uint_as_float(v[c][i]), wgt)), "f"(__fmul_rn(__uint_as_float(v[c][i + 1]), wgt)),
                           "f"(__fmul_rn(__uint_as_float(v[c][i + 2]), wgt)), "f"(__fmul_rn(__uint_as_float(v[c][i + 3]), wgt))
                           : "memory");
        }
      } else {
        const int64_t orow = a.out_padded ? prow : g_off + rel;
        const int64_t col0 = (int64_t)nt * BN + half * C::kColsPerWarp;
        // FP32 first: the BF16 pass below then lets each chunk of v die as
        // soon as it is packed, which keeps the epilogue within its registers
        if (a.out_f32 != nullptr && valid) {
          float4 *dst = reinterpret_cast<float4 *>(a.out_f32 + orow * a.N + col0);
#pragma unroll
          for (int c = 0; c < C::kChunks; ++c) {
#pragma unroll
            for (int i = 0; i < 32; i += 4) {
              dst[c * 8 + i / 4] = make_float4(__fmul_rn(__uint_as_float(v[c][i]), scale),
                                               __fmul_rn(__uint_as_float(v[c][i + 1]), scale),
                                               __fmul_rn(__uint_as_float(v[c][i + 2]), scale),
                                               __fmul_rn(__uint_as_float(v[c][i + 3]), scale));
            }
          }
        }
        if (a.out_bf16 != nullptr) {
          const int64_t slab_row = a.out_padded ? row0 + quad * 32 : g_off + (row0 - g_pad) + quad * 32;
          // 32-row x 64-column boxes (128-byte rows, 128-byte swizzle: chunk
          // q of row r at q ^ (r & 7)) in one 4 KB buffer per warp; each
          // 32-column half is packed and staged on its own
          const uint32_t base = stg_addr + (uint32_t)lane * 128;
#pragma unroll
          for (int cc = 0; cc < C::kChunks / 2; ++cc) {
            if (slab_full) {
              if (lane == 0) bulk_wait_group_read<0>();   // the buffer's previous store has read it
              __syncwarp();
            }
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
              const int c = 2 * cc + hh;
              uint32_t w16[16];
#pragma unroll
              for (int i = 0; i < 16; ++i)
                w16[i] = scale_pack_bf16x2(v[c][2 * i], v[c][2 * i + 1], scale);
              if (slab_full) {
#pragma unroll
                for (int q = 0; q < 4; ++q)
                  st_shared_v4(base + (((uint32_t)(4 * hh + q) ^ ((uint32_t)lane & 7u)) << 4), w16[4 * q],
                               w16[4 * q + 1], w16[4 * q + 2], w16[4 * q + 3]);
              } else if (valid) {
                uint4 *dst = reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(a.out_bf16) + orow * a.N +
                                                       col0 + cc * 64 + hh * 32);
#pragma unroll
                for (int q = 0; q < 4; ++q)
                  dst[q] = make_uint4(w16[4 * q], w16[4 * q + 1], w16[4 * q + 2], w16[4 * q + 3]);
              }
            }
            if (slab_full) {
              fence_proxy_async_smem();
              __syncwarp();
              if (lane == 0) {
                tma_store_2d(&P.tmap_out, stg, (int32_t)(col0 + cc * 64), (int32_t)slab_row);
                bulk_commit_group();
              }
            }
          }
        }
      }
    }
    if (fused_requant) {
      if (pending_mtile) {
        __syncwarp();
        signal_mtile(false);
      }
      // then requantize this CTA's remaining slabs with the workers, staging
      // through this warp's two (now idle) output staging buffers
      const int64_t nslabs = my_mtiles * (BM / kSlabRows);
      if (lane == 0) bulk_wait_group_read<0>();
      __syncwarp();
      ReqStage rs;
      rs.buf[0] = stg;
      rs.buf[1] = stg + C::kStaging / 2;
      rs.bar[0] = reinterpret_cast<uint64_t *>(smem + C::kBarrierOff + 224) + 2 * ew;
      rs.bar[1] = rs.bar[0] + 1;
      rs.piece = C::kStaging / 2;
      rs.loads[0] = rs.loads[1] = 0;
      if (lane == 0) {
        mbar_init(rs.bar[0], 1);
        mbar_init(rs.bar[1], 1);
        fence_mbarrier_init();
      }
      __syncwarp();
      for (;;) {
        int64_t k = -1;
        if (lane == 0) k = claim_slab(slab_next, mt_done, nslabs, abort_flag, a.err);
        k = __shfl_sync(0xffffffffu, k, 0);
        if (k < 0) break;
        __threadfence_block();
        const int64_t mt = (int64_t)blockIdx.x + (k / (BM / kSlabRows)) * gridDim.x;
        requant_slab(a, (int32_t)(mt * (BM / kSlabRows) + k % (BM / kSlabRows)), lane, rs, abort_flag);
      }
    }
    // every tensor store this warp issued has finished before the CTA exits
    if (lane == 0) bulk_wait_group_all();
    __syncwarp();
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

bool encode_2d(CUtensorMap *map, CUtensorMapDataType dtype, uint32_t esize, const void *base,
               uint64_t inner, uint64_t rows, uint32_t box_inner, uint32_t box_rows,
               CUtensorMapSwizzle swizzle) {
  auto fn = get_encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[2] = {inner, rows};
  const cuuint64_t strides[1] = {inner * esize};
  const cuuint32_t box[2] = {box_inner, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(map, dtype, 2, const_cast<void *>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace

bool encode_2d_map(CUtensorMap *map, CUtensorMapDataType dtype, uint32_t esize, const void *base,
                   uint64_t inner, uint64_t rows, uint32_t box_inner, uint32_t box_rows,
                   CUtensorMapSwizzle swizzle) {
  return encode_2d(map, dtype, esize, base, inner, rows, box_inner, box_rows, swizzle);
}

namespace {

template <class C>
cudaError_t launch_cfg(const GemmArgs &a, cudaStream_t s) {
  static thread_local int configured_device = -1;
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (configured_device != dev) {
    err = cudaFuncSetAttribute(k_grouped_gemm<C>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)C::kSmemMax);
    if (err != cudaSuccess) return err;
    configured_device = dev;
  }
  KParams P;
  P.a = a;
  if (!encode_2d(&P.tmap_a, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a.q_a, (uint64_t)(a.K / 2),
                 (uint64_t)a.rows_cap, BK / 2, BM, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  if (!encode_2d(&P.tmap_b, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a.q_w, (uint64_t)(a.K / 2),
                 (uint64_t)(a.E * a.N), BK / 2, C::BN, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;

  std::memset(&P.tmap_out, 0, sizeof(P.tmap_out));
  if (a.out_bf16 != nullptr) {
    // D: [rows][N] (compact rows never exceed rows_cap); h: [rows_cap][N/2]
    const uint64_t cols = a.epilogue == kEpiSwiGLU ? (uint64_t)(a.N / 2) : (uint64_t)a.N;
    // h: 32 x 32 boxes, 64-byte swizzle (32 x 16, none, with 1 KB of
    // staging); D: 32 rows x 64 columns, 128-byte swizzle
    const bool wide = a.epilogue != kEpiSwiGLU;
    const uint32_t box_x = wide ? 64 : (C::kStaging == 1024 ? 16 : 32);
    const CUtensorMapSwizzle sw = wide ? CU_TENSOR_MAP_SWIZZLE_128B
                                       : (C::kStaging == 1024 ? CU_TENSOR_MAP_SWIZZLE_NONE : CU_TENSOR_MAP_SWIZZLE_64B);
    if (!encode_2d(&P.tmap_out, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.out_bf16, cols, (uint64_t)a.rows_cap, box_x,
                   32, sw))
      return cudaErrorInvalidValue;
  }
  const int64_t max_tiles = (a.rows_cap / BM) * (a.N / C::BN);
  int64_t grid = num_sms();
  if (grid > max_tiles) grid = max_tiles;
  if (grid < 1) grid = 1;
  const size_t smem = C::kSmemFixed + (size_t)8 * (a.E + 1);
  k_grouped_gemm<C><<<(unsigned)grid, kThreads, smem, s>>>(P);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_grouped_gemm(const GemmArgs &a, cudaStream_t s) {
  static_assert(CfgGateUp::kMaxE >= 1024 && CfgGateUpFused::kMaxE >= 1024 && CfgDown::kMaxE >= 1024,
                "the three-stage kernels take every group count the library accepts");
  if (a.rows_cap <= 0) return cudaSuccess;
  // both GEMMs use 128 x 256 tiles with one accumulator (the SwiGLU epilogue
  // reads gate and up from the two 128-column halves of a tile).  128 x 128
  // tiles with two accumulators (Cfg<128, 4, 2>) also pass the parity tests
  // but run the down GEMM of the Qwen3-30B-A3B-shaped layer in 239 us
  // instead of 183 us: its cost is per K-step, not the accumulator hand-over.
  // A fourth 54 KB stage for gate_up fits when each epilogue warp stages h
  // through one 1 KB box instead of two 2 KB ones: gate_up of that layer
  // then takes 220 us instead of 241 us.  (With plain 16-byte global stores
  // of h and no staging at all it was slower than three stages.)
  if (a.epilogue == kEpiSwiGLU) {
    // gate_up: a fourth stage in the room of the epilogue's staging (1 KB
    // boxes), as long as the group offsets of E experts still fit
    const bool fused = a.req_q != nullptr && a.amax_h != nullptr && a.amax_h_rows != 0;
    if (fused) return launch_cfg<CfgGateUpFused>(a, s);
    return a.E <= CfgGateUp4::kMaxE ? launch_cfg<CfgGateUp4>(a, s) : launch_cfg<CfgGateUp>(a, s);
  }
  return launch_cfg<CfgDown>(a, s);
}

}  // namespace nvfp4moe
