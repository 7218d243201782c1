// Shared device helpers for the sm_100a kernels: error word, bounded waits,
// mbarriers, TMA / bulk copies, tcgen05 (TMEM alloc, copy, MMA, commit, load)
// and the NVFP4 element / scale conversions.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/nvfp4moe.h"

namespace nvfp4moe {

// ------------------------------------------------------------ error word --
// The first 16 bytes of every workspace: word 0 holds the first device-side
// error (0 = none), word 1 a detail value (for example the bad expert id).
enum DeviceError : int {
  kDevOk = 0,
  kDevBadExpert = 1,     // expert id out of range
  kDevDupExpert = 2,     // one token lists the same expert twice
  kDevTimeout = 3,       // a bounded wait ran out
  kDevBadInput = 4,      // inconsistent counts or positions (expert-parallel exchange)
};

__device__ __forceinline__ void set_device_error(int *err, int code, int detail) {
  if (err != nullptr && atomicCAS(err, 0, code) == 0) {
    atomicExch(err + 1, detail);
  }
}

// Wall-clock bound on any single wait inside a kernel.
constexpr uint64_t kWaitTimeoutNs = 2000000000ull;  // 2 s

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

// ------------------------------------------------------------- mbarrier --
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_mbarrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Waits for the phase with the given parity to complete.  Gives up when
// *abort becomes nonzero or after kWaitTimeoutNs (then records kDevTimeout in
// err, raises *abort, and returns false).  Never spins without a bound.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t *bar, uint32_t parity,
                                                  volatile int *abort_flag, int *err,
                                                  int where) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 31u) == 0) {
      if (*abort_flag) return false;
      if (global_timer_ns() - t0 > kWaitTimeoutNs) {
        set_device_error(err, kDevTimeout, where);
        *abort_flag = 1;
        return false;
      }
    }
  }
}

// ---------------------------------------------------------- TMA / bulk ----
__device__ __forceinline__ void tma_load_2d(void *smem_dst, const CUtensorMap *map, int32_t x,
                                            int32_t y, uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void bulk_load(void *smem_dst, const void *gmem_src, uint32_t bytes,
                                          uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(smem_dst)),
      "l"(gmem_src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// Shared -> global tensor store of one box; completion tracked by bulk groups.
__device__ __forceinline__ void tma_store_2d(const CUtensorMap *map, const void *smem_src, int32_t x,
                                             int32_t y) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(x), "r"(y), "r"(smem_u32(smem_src))
               : "memory");
}

__device__ __forceinline__ void bulk_commit_group() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}

// Wait until at most N committed bulk stores still read shared memory.
template <int N>
__device__ __forceinline__ void bulk_wait_group_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}

// Wait until at most N committed bulk groups are incomplete (writes done).
template <int N>
__device__ __forceinline__ void bulk_wait_group() {
  asm volatile("cp.async.bulk.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void bulk_wait_group_all() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

// Make this thread's generic-proxy shared-memory writes visible to TMA.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void st_shared_v4(uint32_t saddr, uint32_t a, uint32_t b, uint32_t c,
                                             uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(saddr), "r"(a), "r"(b), "r"(c), "r"(d)
               : "memory");
}

__device__ __forceinline__ uint4 ld_shared_v4(uint32_t saddr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(saddr));
  return v;
}

__device__ __forceinline__ void prefetch_tensor_map(const CUtensorMap *map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// --------------------------------------------------------------- tcgen05 --
__device__ __forceinline__ void tmem_alloc(uint32_t *smem_slot, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(smem_slot)),
               "r"(ncols)
               : "memory");
}

__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Shared-memory matrix descriptor (tcgen05 "matrix descriptor"):
//   bits  0-13 start address >> 4, 16-29 leading byte offset >> 4,
//   32-45 stride byte offset >> 4, bit 46 = 1 (sm_100 descriptor version),
//   49-51 base offset, 61-63 swizzle mode (0 none, 2 = 128-byte).
__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes,
                                              uint32_t swizzle_mode) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo_bytes >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)(swizzle_mode & 7u) << 61;
  return d;
}

// D[tmem] (+)= A[smem] * B[smem]^T, NVFP4 operands with UE4M3 scales in TMEM,
// 16-element scale blocks.  accumulate == 0 overwrites D.
__device__ __forceinline__ void mma_nvfp4(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                          uint32_t idesc, uint32_t sfa_tmem, uint32_t sfb_tmem,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t"
      "}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
      : "memory");
}

// Arrive on an mbarrier once every tcgen05 operation this thread issued so
// far (MMAs and copies) has completed.
__device__ __forceinline__ void tc_commit(uint64_t *bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

// 32 lanes x 32 consecutive 32-bit columns: thread i of the warp receives
// columns [col, col+32) of TMEM lane (lane_base + i).
__device__ __forceinline__ void tmem_ld_32cols(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}

// 32 lanes x N consecutive 32-bit columns from registers: thread i of the
// warp writes columns [col, col+N) of TMEM lane (lane_base + i).
__device__ __forceinline__ void tmem_st_16cols(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}

__device__ __forceinline__ void tmem_st_wait() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_ld_wait() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// ------------------------------------------------------- NVFP4 numerics --
// Hardware round-to-nearest-even, saturating conversions.  cvt.*x2 puts its
// first source in the upper half of the result.
__device__ __forceinline__ uint32_t cvt_e2m1x8(const float (&v)[8]) {
  uint32_t out;
  asm volatile(
      "{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
      : "=r"(out)
      : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]));
  return out;
}

// UE4M3 code of a non-negative float, round-to-nearest-even, saturating at 448.
__device__ __forceinline__ uint32_t cvt_ue4m3(float v) {
  uint16_t out;
  asm volatile("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(out) : "f"(0.0f), "f"(v));
  return out & 0xFFu;
}

// Exact value of a non-negative E4M3 code (bias 7; subnormals m * 2^-9).
__device__ __forceinline__ float ue4m3_value(uint32_t code) {
  const uint32_t e = (code >> 3) & 0xFu, m = code & 7u;
  if (e == 0) return (float)m * 0.001953125f;  // 2^-9
  return __uint_as_float(((e + 120u) << 23) | (m << 20));
}

// Global scales from amax, one binary32 operation each:
//   S_enc = 2688 / amax (1 when amax == 0, FLT_MAX if it overflows), S_dec = 1 / S_enc.
__device__ __forceinline__ void global_scales(float amax, float &s_enc, float &s_dec) {
  float e = amax > 0.0f ? __fdiv_rn(2688.0f, amax) : 1.0f;
  if (isinf(e)) e = 3.402823466e38f;
  s_enc = e;
  s_dec = __fdiv_rn(1.0f, e);
}

__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&p);
}

// (x0 * s, x1 * s) rounded to nearest, as one paired binary32 multiply
// (mul.rn.f32x2: each lane of the pair is exactly __fmul_rn) packed to BF16x2.
__device__ __forceinline__ uint32_t scale_pack_bf16x2(uint32_t x0, uint32_t x1, float s) {
  uint64_t a, b, d;
  asm("mov.b64 %0, {%1, %2};" : "=l"(a) : "r"(x0), "r"(x1));
  asm("mov.b64 %0, {%1, %1};" : "=l"(b) : "f"(s));
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  float y0, y1;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(y0), "=f"(y1) : "l"(d));
  return pack_bf16x2(y0, y1);
}

// (x0 * s, x1 * s) rounded to nearest as one paired multiply, unpacked.
__device__ __forceinline__ void scale2(uint32_t x0, uint32_t x1, float s, float &y0, float &y1) {
  uint64_t a, b, d;
  asm("mov.b64 %0, {%1, %2};" : "=l"(a) : "r"(x0), "r"(x1));
  asm("mov.b64 %0, {%1, %1};" : "=l"(b) : "f"(s));
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  asm("mov.b64 {%0, %1}, %2;" : "=f"(y0), "=f"(y1) : "l"(d));
}

// e^-64 in binary32 (a normal number).
constexpr float kExpM64 = 1.60381089e-28f;

// silu(g) u for a pair (g0, u0), (g1, u1) with g >= -64: g / (1 + 2^(-g
// log2 e)) u from the MUFU's approximate base-2 exponential and reciprocal
// (ex2.approx / rcp.approx, a few ulp), the multiplies and the add paired
// (f32x2).  Beyond g = 87 the exponential flushes to 0 and h = g u; at
// g = -64 the denominator is 2^92, inside the reciprocal's range.
__device__ __forceinline__ void silu_mul_fast2(float g0, float g1, float u0, float u1, float &h0, float &h1) {
  constexpr float kNegLog2e = -1.44269504088896340736f;
  uint64_t gg, ll, x, d, one, r, q, uu, hh;
  asm("mov.b64 %0, {%1, %2};" : "=l"(gg) : "f"(g0), "f"(g1));
  asm("mov.b64 %0, {%1, %1};" : "=l"(ll) : "f"(kNegLog2e));
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(x) : "l"(gg), "l"(ll));
  float x0, x1, e0, e1;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(x0), "=f"(x1) : "l"(x));
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(e0) : "f"(x0));
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(e1) : "f"(x1));
  asm("mov.b64 %0, {%1, %2};" : "=l"(d) : "f"(e0), "f"(e1));
  asm("mov.b64 %0, {%1, %1};" : "=l"(one) : "f"(1.0f));
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(d), "l"(one));
  float d0, d1, r0, r1;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(d0), "=f"(d1) : "l"(d));
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r0) : "f"(d0));
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r1) : "f"(d1));
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(r0), "f"(r1));
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(q) : "l"(gg), "l"(r));
  asm("mov.b64 %0, {%1, %2};" : "=l"(uu) : "f"(u0), "f"(u1));
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(hh) : "l"(q), "l"(uu));
  asm("mov.b64 {%0, %1}, %2;" : "=f"(h0), "=f"(h1) : "l"(hh));
}

// silu(g) * u in binary32 with one fast exponential and one fast division
// (~2^-21 relative, far below a BF16 ulp), for every g:
//   g >= 0:        g / (1 + e^-g) * u
//   -64 <= g < 0:  g e^g / (1 + e^g) * u          (e^-g would overflow the
//                                                   fast division near -87)
//   g < -64:       ((g e^(g+64)) u) e^-64         (1 + e^g == 1 in binary32;
//                                                   the shift keeps e^(.)
//                                                   normal down to g = -151)
// so silu(g) u is not flushed to zero where it is still a BF16 number.
__device__ __forceinline__ float silu_mul(float g, float u) {
  const bool far = g < -64.0f;
  const float t = __expf(g >= 0.0f ? -g : (far ? g + 64.0f : g));
  const float num = g >= 0.0f ? g : __fmul_rn(g, t);
  const float h = __fmul_rn(__fdividef(num, far ? 1.0f : 1.0f + t), u);
  return far ? __fmul_rn(h, kExpM64) : h;
}

// MXFP8 quantize-dequantize of one 32-element block held by one thread (the
// public OCP MX definition; the activations of the W4A8 variant): the E8M0
// scale is 2^s with s = floor(log2 amax) - 8, clamped to [-127, 127] (-127
// for an all-zero block); each element becomes E4M3(v / 2^s) by the
// hardware's round-to-nearest-even saturating conversion (sign kept), and is
// returned as E4M3 * 2^s rounded to BF16 -- exact unless |E4M3 * 2^s| is
// below BF16's normal range (2^-126).  v: binary32 values; out: BF16 pairs.
__device__ __forceinline__ void mxfp8_qdq32(const float (&v)[32], uint32_t (&out)[16]) {
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(v[i]));
  const int eb = (int)(__float_as_uint(amax) >> 23);          // amax >= 0, finite
  const int s = eb == 0 ? -127 : max(eb - 135, -127);
  const float down = __uint_as_float((uint32_t)(127 - s) << 23);                      // 2^-s, s <= 119
  const float up = s > -127 ? __uint_as_float((uint32_t)(s + 127) << 23) : 0x1p-127f;  // 2^s
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    uint16_t q;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(q) : "f"(v[2 * i + 1] * down), "f"(v[2 * i] * down));
    uint32_t hp;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(hp) : "h"(q));
    const float lo = __half2float(__ushort_as_half((unsigned short)(hp & 0xFFFFu)));
    const float hi = __half2float(__ushort_as_half((unsigned short)(hp >> 16)));
    out[i] = pack_bf16x2(lo * up, hi * up);
  }
}

// Byte offset of scale (row, block b) in the MMA atom layout of a matrix whose
// rows hold K elements (K/64 atoms per 128-row group).
__device__ __forceinline__ int64_t sf_mma_offset(int64_t row, int64_t b, int64_t K) {
  const int64_t atom = (row >> 7) * (K >> 6) + (b >> 2);
  return atom * 512 + (row & 31) * 16 + ((row & 127) >> 5) * 4 + (b & 3);
}

}  // namespace nvfp4moe
