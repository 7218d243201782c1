// Persistent block-scaled NVFP4 grouped GEMM over the experts (sm_100a).
//
// The grouped matrix multiplication of the token-wise NVFP4 path
// (www.aib.vote "miniTE report, NVFP4 RL stability", paragraph 4) and the
// grouped GEMMs of the MoE learner (news.hamidun.com, "diagnostics, alignment
// and fast kernels").  One launch covers every expert; the group sizes are
// read on the device from padded_offsets, so the host never synchronizes.
//
// Design (B200):
//   * tile 128 x BN x 256 (M x N x K elements); BN = 256 with one TMEM
//     accumulator for both GEMMs (the SwiGLU epilogue needs the gate and up
//     halves of a 256-wide tile; BN = 128 with two accumulators measured
//     slower for down: twice the A re-reads).  A rows come
//     from the padded grouped layout, where every expert's group starts on a
//     128-row boundary, so a tile never straddles two experts.
//   * warp 4, one thread: TMA producer.  Per K-step it loads the A tile
//     (16 KB) and the B tile (32 KB) with 128-byte-swizzled tensor copies,
//     and the scales with plain bulk copies: A's 2 KB (the K-step-major
//     layout [K/256][rows][16] puts a tile's 128 rows x 16 scales of one
//     K-step in one contiguous run) and B's 4 KB (prepared in the MMA atom
//     layout), into a shared-memory ring.
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

#include <cstring>
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace nvfp4moe {

namespace {

constexpr int BM = 128, BK = 256;
// 16 warps in four warpgroups: 0-3 scale feeders (one per TMEM lane quarter),
// 4 the TMA producer, 5 the MMA issuer (6-7 idle), 8-15 the epilogue.
// setmaxnreg moves registers from the first two warpgroups to the epilogue:
// 128 * 96 + 128 * 56 + 256 * 176 = 64512 <= 65536 launched (512 * 128).
constexpr int kFeedWarps = 4;
constexpr int kEpiWarps = 8;
constexpr int kEpiWarp0 = 8;
constexpr int kThreads = 512;
constexpr uint32_t kRegsFeed = 96, kRegsCtl = 56, kRegsEpi = 176;
static_assert(128 * kRegsFeed + 128 * kRegsCtl + 256 * kRegsEpi <= 65536, "register split");
constexpr uint32_t kTmemCols = 512;
// Epilogue staging: per epilogue warp two 2 KB buffers of 32 rows x 32 BF16
// (64-byte swizzle), drained to global memory by TMA tensor stores.
constexpr int kStagingPerWarp = 4096;

template <int BN_, int STAGES_, int ACC_>
struct Cfg {
  static constexpr int BN = BN_;
  static constexpr int STAGES = STAGES_;
  static constexpr int ACC = ACC_;                   // TMEM accumulator buffers
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
  static constexpr size_t kBarrierOff = kStagingOff + (size_t)kEpiWarps * kStagingPerWarp;
  static constexpr size_t kSmemFixed = kBarrierOff + 1024 + 256;
  static constexpr size_t kSmemMax = kSmemFixed + (size_t)8 * 1025;   // + offsets of E <= 1024
  // Instruction descriptor, kind::mxf4nvf4: A and B E2M1 (format 1), K-major,
  // UE4M3 scales (bit 23 = 0), N >> 3 at bit 17, M >> 4 at bit 24, dense, K = 64.
  static constexpr uint32_t kIdesc = (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
                                     ((uint32_t)(BM >> 4) << 24);
  static_assert(ACC * BN + STAGES * (16 + 16 * kNAtoms) <= (int)kTmemCols, "TMEM budget");
  static_assert(kSmemMax <= 232448, "shared memory budget");
};

using CfgGateUp = Cfg<256, 3, 1>;
using CfgDown = Cfg<256, 3, 1>;

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

// Group of a padded row: padded[lo] <= row < padded[lo + 1] (shared memory).
__device__ __forceinline__ int find_group(const int32_t *padded, int E, int64_t row) {
  int lo = 0, hi = E;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if ((int64_t)padded[mid] <= row) lo = mid; else hi = mid;
  }
  return lo;
}

__device__ __forceinline__ float fmax_abs_bf16(float m, uint32_t packed) {
  return fmaxf(m, fmaxf(fabsf(bf16_lo(packed)), fabsf(bf16_hi(packed))));
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
  int32_t *s_pad = reinterpret_cast<int32_t *>(smem + C::kBarrierOff + 256);
  int32_t *s_off = s_pad + (P.a.E + 1);

  const GemmArgs &a = P.a;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

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
  // K-steps of this CTA: its tiles blockIdx.x, +gridDim.x, ... times kt_count
  const int64_t my_tiles = total > (int64_t)blockIdx.x ? (total - 1 - blockIdx.x) / gridDim.x + 1 : 0;
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
      for (int64_t t = blockIdx.x; t < total && ok; t += gridDim.x) {
        const int64_t mt = t / n_tiles;
        const int nt = (int)(t - mt * n_tiles);
        const int e = find_group(s_pad, a.E, mt * BM);
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
      for (int64_t t = blockIdx.x; t < total && ok; t += gridDim.x, ++it) {
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
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsEpi));
    // -------------------------------------------------------- epilogue
    const int ew = warp - kEpiWarp0;
    const int quad = warp & 3;              // TMEM lanes this warp may read
    const int half = ew >> 2;               // which half of the columns
    const int rit = quad * 32 + lane;       // row inside the tile
    const uint32_t tlane = tmem + ((uint32_t)(quad * 32) << 16);
    uint8_t *stg = smem + C::kStagingOff + (size_t)ew * kStagingPerWarp;
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
    for (int64_t t = blockIdx.x; t < total; t += gridDim.x, ++it) {
      const int64_t mt = t / n_tiles;
      const int nt = (int)(t - mt * n_tiles);
      const int64_t row0 = mt * BM;
      const int e = find_group(s_pad, a.E, row0);
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
      if (a.epilogue == kEpiSwiGLU) {
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
      if (BN == 256 && a.epilogue == kEpiSwiGLU) {
        uint32_t hp[2][16];
        float m = 0.0f;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
#pragma unroll
          for (int i = 0; i < 32; i += 2) {
            float hh[2];
#pragma unroll
            for (int q = 0; q < 2; ++q) {
              const float g = __fmul_rn(__uint_as_float(v[c][i + q]), scale);
              const float u = __fmul_rn(__uint_as_float(v[(c + 2) % C::kChunks][i + q]), scale);
              // silu(g) = g / (1 + e^-g); the fast exponential and division
              // are accurate to ~2^-21 relative, far below a BF16 ulp of h
              const float sg = __fdividef(g, 1.0f + __expf(-g));
              hh[q] = __fmul_rn(sg, u);
            }
            hp[c][i / 2] = pack_bf16x2(hh[0], hh[1]);
            m = fmax_abs_bf16(m, hp[c][i / 2]);
          }
        }
        // h rows live at padded positions: the whole slab is stored (rows past
        // the group's end are padding that nothing reads)
#pragma unroll
        for (int c = 0; c < 2; ++c)
          store_box(hp[c], (int32_t)(nt * 128 + half * 64 + c * 32), (int32_t)(row0 + quad * 32));
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
      } else {
        const int64_t orow = a.out_padded ? prow : g_off + rel;
        const int64_t col0 = (int64_t)nt * BN + half * C::kColsPerWarp;
        if (a.out_bf16 != nullptr) {
          const int64_t slab_row = a.out_padded ? row0 + quad * 32 : g_off + (row0 - g_pad) + quad * 32;
#pragma unroll
          for (int c = 0; c < C::kChunks; ++c) {
            uint32_t w16[16];
#pragma unroll
            for (int i = 0; i < 16; ++i)
              w16[i] = pack_bf16x2(__fmul_rn(__uint_as_float(v[c][2 * i]), scale),
                                   __fmul_rn(__uint_as_float(v[c][2 * i + 1]), scale));
            if (slab_full) {
              store_box(w16, (int32_t)(col0 + c * 32), (int32_t)slab_row);
            } else if (valid) {
              uint4 *dst = reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(a.out_bf16) +
                                                     orow * a.N + col0 + c * 32);
#pragma unroll
              for (int q = 0; q < 4; ++q)
                dst[q] = make_uint4(w16[4 * q], w16[4 * q + 1], w16[4 * q + 2], w16[4 * q + 3]);
            }
          }
        }
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
    if (!encode_2d(&P.tmap_out, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.out_bf16, cols,
                   (uint64_t)a.rows_cap, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B))
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
  if (a.rows_cap <= 0) return cudaSuccess;
  // the SwiGLU epilogue reads gate and up from the two halves of a 256-wide
  // tile; plain stores use 128-wide tiles with a double-buffered accumulator
  if (a.epilogue == kEpiSwiGLU) return launch_cfg<CfgGateUp>(a, s);
  return launch_cfg<CfgDown>(a, s);
}

}  // namespace nvfp4moe
