// Plain, slow CPU oracle of the NVFP4 W4A4 MoE expert layer, in C++.
//
// TEST INFRASTRUCTURE ONLY.  Built with g++ -O2 -ffp-contract=off
// -fno-fast-math (no fused multiply-add, IEEE binary32 / binary64 with
// round-to-nearest-even everywhere) into oracle/liboracle.so, and called
// through ctypes by tests/, __graft_entry__.smoke() and bench.py's CPU legs.
// Nothing in the product package links or calls it; it shares no code, table
// or helper with the CUDA path.
//
// What it computes follows the miniTE pages:
//   news.hamidun.com "miniTE ... 1.39x over BF16 on Qwen3-30B-A3B" (Arabic
//     and Russian editions), key facts: the learner runs native NVFP4 W4A4;
//     section "diagnostics, alignment and fast kernels": grouped GEMMs over
//     the experts of Qwen3-30B-A3B, strict alignment (the learner and the
//     rollout compute one policy, so the order of computation is fixed);
//   www.aib.vote "miniTE report, NVFP4 RL stability", paragraph 4: the
//     token-wise NVFP4 path -- contiguous layout, device-side metadata, amax
//     reuse, grouped matrix multiplication, fusion;
// plus the public NVFP4 format definition the pages name but do not print
// (E2M1 elements, one UE4M3 scale per 16 elements, one FP32 tensor scale).
//
// Readings where the pages are silent (the same numbering the design notes
// use):
//   R1  E2M1 magnitudes {0, .5, 1, 1.5, 2, 3, 4, 6}, bit 3 the sign.
//   R2  UE4M3: E4M3 with sign 0, bias 7, subnormals m * 2^-9, max 448; the
//       NaN code 0x7F is never produced.
//   R3  element 2i in the low nibble of byte i.
//   R4  S_enc = 2688 / amax in binary32 (1 when amax == 0, FLT_MAX when the
//       quotient overflows); S_dec = 1 / S_enc in binary32.
//   R5  sf = UE4M3_rne_satfinite((bamax / 6) * S_enc), two binary32 steps.
//   R6  code = E2M1_rne_satfinite(x * (S_enc / sf)); ties to the even code;
//       |y| > 6 saturates; a negative value that rounds to 0 keeps its sign
//       (code 0x8); a block with sf == 0 is all +0.
//   R7  per-token mode: amax per row.
//   R8  rows sorted by (expert, token, slot); each group padded to 128 rows.
//   R9  GEMM: sum over k of the dequantized products in fp64, one rounding.
//   R10 the fused gate_up weight of an expert is one [2I][H] tensor (gate
//       rows, then up rows) with one S_dec.
//   R11 h = silu(g) * u in fp64, silu(g) = g / (1 + exp(-g)), rounded once
//       to BF16; the requantization input is that BF16 h.
//   R12 D rows are BF16; y[t] = BF16(sum_j w[t][j] * D[t][j]), fp64 sum in
//       slot order.
//   R15 top-k routing: the k largest logits (ties to the lower expert id),
//       slots in descending order, weights = softmax over the chosen k.
//   R19 W4A16 variant (www.aib.vote "miniTE report, NVFP4 RL stability",
//       paragraph 3 measures W4A16 beside W4A8 and W4A4 without formulas):
//       the same NVFP4 weights, BF16 activations: x is not quantized and h is
//       not requantized; G = x W_gu^T on the dequantized weights in fp64,
//       h = BF16(silu(g) u), D = BF16(h W_dn^T), then the same combine.
//   R17 MXFP8 (W4A8 activations; the pages name the format only, this is the
//       public OCP MX definition): blocks of 32 consecutive elements along a
//       row share an E8M0 scale 2^s, s = floor(log2(block amax)) - 8
//       clamped to [-127, 127] (-127 for an all-zero block); elements are
//       E4M3(v / 2^s), round to nearest even, saturating at +-448, sign kept
//       (a negative value that rounds to 0 is code 0x80).
//   R20 W4A8 variant (the same paragraph 3 of the aib.vote report): the W4A4
//       layer's NVFP4 weights, activations x and h in MXFP8 (R17), each
//       dequantized exactly; h = BF16(silu(g) u) is the requantization input
//       as in R11.  Everything else as R19.
//   R16 backward, BF16-backward mode (www.aib.vote "miniTE report, NVFP4 RL
//       stability", paragraph 1 times "NVFP4 forward, BF16 backward" without
//       formulas): the exact gradient of the unquantized layer on its BF16
//       operands, every quantizer of the forward taken as the identity; the
//       routing choice is not differentiated, the routing weights are.
//
// Every step is written as a loop that can be checked against its definition
// by eye; no blocking or reordering beyond what the definition states.
#include <algorithm>
#include <cfloat>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <thread>
#include <vector>

namespace {

// ------------------------------------------------------------ formats --
// R1: the E2M1 magnitude of a 3-bit magnitude code.
const double kE2M1[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

// R2: value of a non-negative E4M3 code from its bit fields.
double ue4m3_value(int code) {
  const int e = (code >> 3) & 0xF, m = code & 7;
  if (e == 0) return std::ldexp((double)m, -9);
  return std::ldexp(1.0 + m / 8.0, e - 7);
}

// Index of the grid value nearest to a >= 0 over grid[0..n) (increasing),
// ties to the even index, saturating at the last value.  In both formats the
// lowest code bit is the lowest mantissa bit, so "ties to even mantissa" is
// "ties to the even index".  Differences are exact in fp64 for float inputs.
int nearest_even(double a, const double *grid, int n) {
  if (a >= grid[n - 1]) return n - 1;
  const int hi = (int)(std::lower_bound(grid, grid + n, a) - grid);   // grid[hi-1] < a <= grid[hi]
  if (hi == 0) return 0;
  const int lo = hi - 1;
  const double d_lo = a - grid[lo], d_hi = grid[hi] - a;
  if (d_hi < d_lo) return hi;
  if (d_lo < d_hi) return lo;
  return (hi % 2 == 0) ? hi : lo;
}

struct UE4M3Table {
  double v[127];
  UE4M3Table() {
    for (int c = 0; c < 127; ++c) v[c] = ue4m3_value(c);
  }
};
const UE4M3Table kUE4M3;

}  // namespace

extern "C" {

// R1, R6: E2M1 code of y (round to nearest even, saturating, sign kept).
uint8_t orc_e2m1_encode(float y) {
  const int mag = nearest_even(std::fabs((double)y), kE2M1, 8);
  const int sign = std::signbit(y) ? 8 : 0;
  return (uint8_t)(mag | sign);
}

double orc_e2m1_decode(uint8_t code) {
  const double m = kE2M1[code & 7];
  return (code & 8) ? -m : m;
}

// R2: UE4M3 code of v >= 0 (round to nearest even, saturating at 448).
uint8_t orc_ue4m3_encode(float v) { return (uint8_t)nearest_even((double)v, kUE4M3.v, 127); }

double orc_ue4m3_decode(uint8_t code) { return kUE4M3.v[code & 0x7F]; }

// Round a double to the nearest BF16 value (8 significant bits), ties to
// even, directly from the double (no intermediate binary32 rounding);
// overflow gives +-inf.  Returned as the (exact) binary32 value.
float orc_round_bf16(double v) {
  if (v == 0.0 || std::isnan(v) || std::isinf(v)) return (float)v;
  const double a = std::fabs(v);
  int e2;
  std::frexp(a, &e2);                 // a = f * 2^e2, f in [0.5, 1): floor(log2 a) = e2 - 1
  const int e = std::max(e2 - 1, -126);
  const double quantum = std::ldexp(1.0, e - 7);
  double r = std::nearbyint(a / quantum) * quantum;     // current rounding mode: to nearest even
  if (r > 3.3895313892515355e38) r = INFINITY;          // above the largest finite BF16
  return (float)std::copysign(r, v);
}

// R4: global encode / decode scales from amax, one binary32 operation each.
void orc_global_scales(float amax, float *s_enc, float *s_dec) {
  float e = 1.0f;
  if (amax > 0.0f) {
    e = 2688.0f / amax;
    if (std::isinf(e)) e = FLT_MAX;
  }
  *s_enc = e;
  *s_dec = 1.0f / e;
}

void orc_e2m1_encode_n(const float *y, int64_t n, uint8_t *out) {
  for (int64_t i = 0; i < n; ++i) out[i] = orc_e2m1_encode(y[i]);
}

void orc_ue4m3_encode_n(const float *v, int64_t n, uint8_t *out) {
  for (int64_t i = 0; i < n; ++i) out[i] = orc_ue4m3_encode(v[i]);
}

// Codes of the binary32 values whose bit patterns are start, start+1, ...,
// start+n-1 (the exhaustive sweeps of the hardware conversions compare these
// with the GPU's); threads split the range.
static void encode_bits_range(uint32_t start, int64_t n, uint8_t *out, int threads, bool e2m1) {
  auto work = [&](int64_t i0, int64_t i1) {
    for (int64_t i = i0; i < i1; ++i) {
      const uint32_t bits = start + (uint32_t)i;
      float v;
      std::memcpy(&v, &bits, 4);
      out[i] = e2m1 ? orc_e2m1_encode(v) : orc_ue4m3_encode(v);
    }
  };
  if (threads < 2) {
    work(0, n);
    return;
  }
  std::vector<std::thread> pool;
  const int64_t per = (n + threads - 1) / threads;
  for (int t = 0; t < threads; ++t) {
    const int64_t i0 = t * per, i1 = std::min(n, i0 + per);
    if (i0 < i1) pool.emplace_back(work, i0, i1);
  }
  for (auto &th : pool) th.join();
}

void orc_e2m1_encode_bits(uint32_t start, int64_t n, uint8_t *out, int threads) {
  encode_bits_range(start, n, out, threads, true);
}

// non-negative finite patterns only (start + n <= 0x7F800000)
void orc_ue4m3_encode_bits(uint32_t start, int64_t n, uint8_t *out, int threads) {
  encode_bits_range(start, n, out, threads, false);
}

void orc_round_bf16_n(const double *v, int64_t n, float *out) {
  for (int64_t i = 0; i < n; ++i) out[i] = orc_round_bf16(v[i]);
}

void orc_global_scales_n(const float *amax, int64_t n, float *s_enc, float *s_dec) {
  for (int64_t i = 0; i < n; ++i) orc_global_scales(amax[i], s_enc + i, s_dec + i);
}

// NVFP4 quantization of x [M][K] (BF16 values held as floats), R4-R7:
//   amax  = max |x| over the tensor, or over each row when per_token,
//           unless amax_in is given (amax reuse: [1] or [M], used as is)
//   S_enc = 2688 / amax, S_dec = 1 / S_enc
//   per 16-element block: bamax = max |x|, sf = UE4M3((bamax / 6) * S_enc),
//   r = S_enc / sf (0 when sf == 0), code = E2M1(x * r) (all +0 when sf == 0)
// Outputs: q [M][K/2] (R3 packing), sf [M][K/16] row-major, s_dec and amax
// [1] or [M].  Returns 0, or -1 when K is not a multiple of 16.
int orc_quantize(const float *x, int64_t M, int64_t K, int per_token, const float *amax_in,
                 uint8_t *q, uint8_t *sf, float *s_dec, float *amax_out) {
  if (K % 16 != 0 || M < 0) return -1;
  const int64_t nsc = per_token ? M : 1;       // number of global scales
  std::vector<float> amax(nsc, 0.0f), enc(nsc), dec(nsc);
  if (amax_in != nullptr) {
    for (int64_t i = 0; i < nsc; ++i) amax[i] = amax_in[i];
  } else {
    for (int64_t r = 0; r < M; ++r)
      for (int64_t c = 0; c < K; ++c) {
        const float a = std::fabs(x[r * K + c]);
        float &m = amax[per_token ? r : 0];
        if (a > m) m = a;
      }
  }
  for (int64_t i = 0; i < nsc; ++i) orc_global_scales(amax[i], &enc[i], &dec[i]);
  for (int64_t r = 0; r < M; ++r) {
    const float S_enc = enc[per_token ? r : 0];
    for (int64_t b = 0; b < K / 16; ++b) {
      const float *blk = x + r * K + b * 16;
      float bamax = 0.0f;
      for (int i = 0; i < 16; ++i) bamax = std::max(bamax, std::fabs(blk[i]));
      const float t1 = bamax / 6.0f;
      const float t = t1 * S_enc;
      const uint8_t sfc = orc_ue4m3_encode(t);
      sf[r * (K / 16) + b] = sfc;
      float rr = 0.0f;
      if (sfc != 0) rr = S_enc / (float)orc_ue4m3_decode(sfc);
      for (int i = 0; i < 16; i += 2) {
        uint8_t c0 = 0, c1 = 0;
        if (sfc != 0) {
          const float y0 = blk[i] * rr, y1 = blk[i + 1] * rr;
          c0 = orc_e2m1_encode(y0);
          c1 = orc_e2m1_encode(y1);
        }
        q[r * (K / 2) + b * 8 + i / 2] = (uint8_t)((c0 & 0xF) | ((c1 & 0xF) << 4));
      }
    }
  }
  for (int64_t i = 0; i < nsc; ++i) {
    s_dec[i] = dec[i];
    if (amax_out != nullptr) amax_out[i] = amax[i];
  }
  return 0;
}

// x_hat = e2m1(code) * sf * S_dec in fp64 (exact: 3 + 4 + 24 significant
// bits).  s_dec is [M] when per_row_sdec, else [1].
void orc_dequantize(const uint8_t *q, const uint8_t *sf, const float *s_dec, int64_t M, int64_t K,
                    int per_row_sdec, double *out) {
  for (int64_t r = 0; r < M; ++r) {
    const double S = s_dec[per_row_sdec ? r : 0];
    for (int64_t c = 0; c < K; ++c) {
      const uint8_t byte = q[r * (K / 2) + c / 2];
      const uint8_t code = (c % 2 == 0) ? (byte & 0xF) : (byte >> 4);
      out[r * K + c] = orc_e2m1_decode(code) * orc_ue4m3_decode(sf[r * (K / 16) + c / 16]) * S;
    }
  }
}

// R15: top-k routing from router logits [T][E] (FP32 values): the k largest
// logits with ties to the lower expert id, slots in descending order; the
// weights are exp(l_j - l_max) / sum over the chosen k of exp(l_i - l_max),
// in fp64.  Returns -1 unless 1 <= k <= E.
int orc_route_topk(const float *logits, int64_t T, int E, int k, int32_t *idx, double *w) {
  if (k < 1 || k > E) return -1;
  std::vector<char> taken(E);
  for (int64_t t = 0; t < T; ++t) {
    const float *l = logits + t * E;
    std::fill(taken.begin(), taken.end(), 0);
    for (int j = 0; j < k; ++j) {
      int best = -1;
      for (int e = 0; e < E; ++e) {
        if (taken[e]) continue;
        if (best < 0 || l[e] > l[best]) best = e;   // strict: the lower id wins a tie
      }
      taken[best] = 1;
      idx[t * k + j] = best;
    }
    const double top = l[idx[t * k]];
    double z = 0.0;
    for (int j = 0; j < k; ++j) z += std::exp((double)l[idx[t * k + j]] - top);
    for (int j = 0; j < k; ++j) w[t * k + j] = std::exp((double)l[idx[t * k + j]] - top) / z;
  }
  return 0;
}

// R8: the routed rows r = t*k + j in the stable order (expert, token, slot):
// a counting sort.  offsets[E+1], padded_offsets[E+1] (groups rounded up to
// 128 rows), perm[R] (perm[pos] = t*k + j) and inv_perm[T*k].  Returns -1 on
// an expert id out of range.
int orc_permutation(const int32_t *topk_idx, int64_t T, int k, int E, int32_t *offsets,
                    int32_t *padded_offsets, int32_t *perm, int32_t *inv_perm) {
  const int64_t R = T * k;
  std::vector<int64_t> count(E, 0);
  for (int64_t r = 0; r < R; ++r) {
    const int e = topk_idx[r];
    if (e < 0 || e >= E) return -1;
    ++count[e];
  }
  offsets[0] = 0;
  padded_offsets[0] = 0;
  for (int e = 0; e < E; ++e) {
    offsets[e + 1] = (int32_t)(offsets[e] + count[e]);
    padded_offsets[e + 1] = (int32_t)(padded_offsets[e] + (count[e] + 127) / 128 * 128);
  }
  std::vector<int64_t> next(E);
  for (int e = 0; e < E; ++e) next[e] = offsets[e];
  for (int64_t r = 0; r < R; ++r) {       // r = t*k + j ascending: token, then slot
    const int e = topk_idx[r];
    const int64_t pos = next[e]++;
    perm[pos] = (int32_t)r;
    inv_perm[r] = (int32_t)pos;
  }
  return 0;
}

// R9: out[r][n] = sum_{c=0..K-1} a[r][c] * w[n][c] in fp64, the sum taken in
// ascending c; out_abs (nullable) receives sum_c |a[r][c] * w[n][c]|, the
// scale of the GEMM tolerance.  Rows are split over `threads` threads.
void orc_gemm_rows(const double *a, int64_t R, const double *w, int64_t N, int64_t K, double *out,
                   double *out_abs, int threads) {
  auto work = [&](int64_t r0, int64_t r1) {
    for (int64_t r = r0; r < r1; ++r)
      for (int64_t n = 0; n < N; ++n) {
        double s = 0.0, sa = 0.0;
        for (int64_t c = 0; c < K; ++c) {
          const double p = a[r * K + c] * w[n * K + c];
          s += p;
          sa += std::fabs(p);
        }
        out[r * N + n] = s;
        if (out_abs != nullptr) out_abs[r * N + n] = sa;
      }
  };
  if (threads < 2 || R < 2) {
    work(0, R);
    return;
  }
  std::vector<std::thread> pool;
  const int64_t per = (R + threads - 1) / threads;
  for (int i = 0; i < threads; ++i) {
    const int64_t r0 = i * per, r1 = std::min(R, r0 + per);
    if (r0 < r1) pool.emplace_back(work, r0, r1);
  }
  for (auto &th : pool) th.join();
}

// R9 over experts: rows offsets[e]..offsets[e+1] of a times W_e^T, where
// w = [E][N][K] dequantized weights.
void orc_grouped_gemm(const double *a, const int32_t *offsets, int E, const double *w, int64_t N, int64_t K,
                      double *out, double *out_abs, int threads) {
  for (int e = 0; e < E; ++e) {
    const int64_t lo = offsets[e], hi = offsets[e + 1];
    if (hi > lo)
      orc_gemm_rows(a + lo * K, hi - lo, w + (int64_t)e * N * K, N, K, out + lo * N,
                    out_abs != nullptr ? out_abs + lo * N : nullptr, threads);
  }
}

// R11: h[r][i] = silu(g) * u with g = gu[r][i], u = gu[r][I + i], fp64.
void orc_swiglu(const double *gu, int64_t R, int64_t I, double *h) {
  for (int64_t r = 0; r < R; ++r)
    for (int64_t i = 0; i < I; ++i) {
      const double g = gu[r * 2 * I + i], u = gu[r * 2 * I + I + i];
      h[r * I + i] = g / (1.0 + std::exp(-g)) * u;
    }
}

// R12: y[t] = BF16( sum_{j=0..k-1} w[t][j] * D[inv_perm[t][j]] ), fp64 sum in
// slot order; D rows are BF16 values held as floats.
void orc_combine(const float *d, int64_t H, const int32_t *inv_perm, const float *w, int64_t T, int k,
                 float *y) {
  for (int64_t t = 0; t < T; ++t)
    for (int64_t c = 0; c < H; ++c) {
      double s = 0.0;
      for (int j = 0; j < k; ++j) s += (double)w[t * k + j] * (double)d[(int64_t)inv_perm[t * k + j] * H + c];
      y[t * H + c] = orc_round_bf16(s);
    }
}

// Intermediates of orc_expert_layer (every pointer nullable except y).
struct OrcLayerOut {
  float *y;             // [T][H]
  uint8_t *x_q;         // [T][H/2]      x quantized once per token (or per tensor)
  uint8_t *x_sf;        // [T][H/16]
  float *x_s_dec;       // [T] or [1]
  int32_t *offsets;     // [E+1]
  int32_t *padded_offsets;
  int32_t *perm;        // [T*k]
  int32_t *inv_perm;    // [T*k]
  float *h;             // [T*k][I]      BF16 h in sorted row order
  uint8_t *h_q;         // [T*k][I/2]
  uint8_t *h_sf;        // [T*k][I/16]
  float *h_s_dec;       // [T*k] or [1]
  float *d;             // [T*k][H]      BF16 D in sorted row order
};

// The W4A4 MoE expert layer end to end, in the pages' order:
//   1. quantize x once per token (amax reused for all k copies of a token)
//   2. permute the routed rows to the (expert, token, slot) layout
//   3. gate_up grouped GEMM on the dequantized operands (fp64)
//   4. SwiGLU, BF16 h, requantize h (per row in per-token mode, else one
//      scale over all routed rows)
//   5. down grouped GEMM -> BF16 D
//   6. weighted combine in slot order -> BF16 y
// Weights: w_gate_up [E][2I][H] and w_down [E][H][I] as BF16 values; each
// expert's matrix is quantized as one tensor (R10).  Returns 0, or -1 on a
// bad shape or routing entry.
int orc_expert_layer(const float *x, const int32_t *topk_idx, const float *topk_w, const float *w_gate_up,
                     const float *w_down, int64_t T, int64_t H, int64_t I, int E, int k, int per_token,
                     int threads, OrcLayerOut *out) {
  if (H % 16 != 0 || I % 16 != 0 || out == nullptr || out->y == nullptr) return -1;
  const int64_t R = T * k;
  // 1. x, quantized once
  std::vector<uint8_t> xq(T * H / 2), xsf(T * H / 16);
  std::vector<float> xsd(per_token ? std::max<int64_t>(T, 1) : 1), xam(xsd.size());
  orc_quantize(x, T, H, per_token, nullptr, xq.data(), xsf.data(), xsd.data(), xam.data());
  std::vector<double> x_hat(T * H);
  orc_dequantize(xq.data(), xsf.data(), xsd.data(), T, H, per_token, x_hat.data());
  // 2. permutation
  std::vector<int32_t> off(E + 1), pad(E + 1), perm(R), inv(R);
  if (orc_permutation(topk_idx, T, k, E, off.data(), pad.data(), perm.data(), inv.data()) != 0) return -1;
  std::vector<double> a(R * H);
  for (int64_t p = 0; p < R; ++p) {
    const int64_t t = perm[p] / k;
    std::memcpy(&a[p * H], &x_hat[t * H], H * sizeof(double));
  }
  // weights, dequantized
  std::vector<double> wgu((int64_t)E * 2 * I * H), wdn((int64_t)E * H * I);
  for (int e = 0; e < E; ++e) {
    std::vector<uint8_t> q(2 * I * H / 2), s(2 * I * H / 16);
    float sd, am;
    orc_quantize(w_gate_up + (int64_t)e * 2 * I * H, 2 * I, H, 0, nullptr, q.data(), s.data(), &sd, &am);
    orc_dequantize(q.data(), s.data(), &sd, 2 * I, H, 0, &wgu[(int64_t)e * 2 * I * H]);
    std::vector<uint8_t> q2(H * I / 2), s2(H * I / 16);
    orc_quantize(w_down + (int64_t)e * H * I, H, I, 0, nullptr, q2.data(), s2.data(), &sd, &am);
    orc_dequantize(q2.data(), s2.data(), &sd, H, I, 0, &wdn[(int64_t)e * H * I]);
  }
  // 3. gate_up
  std::vector<double> gu(R * 2 * I);
  orc_grouped_gemm(a.data(), off.data(), E, wgu.data(), 2 * I, H, gu.data(), nullptr, threads);
  // 4. SwiGLU, BF16, requantize
  std::vector<double> hd(R * I);
  orc_swiglu(gu.data(), R, I, hd.data());
  std::vector<float> h(R * I);
  orc_round_bf16_n(hd.data(), R * I, h.data());
  std::vector<uint8_t> hq(R * I / 2), hsf(R * I / 16);
  std::vector<float> hsd(per_token ? std::max<int64_t>(R, 1) : 1), ham(hsd.size());
  orc_quantize(h.data(), R, I, per_token, nullptr, hq.data(), hsf.data(), hsd.data(), ham.data());
  std::vector<double> h_hat(R * I);
  orc_dequantize(hq.data(), hsf.data(), hsd.data(), R, I, per_token, h_hat.data());
  // 5. down -> BF16 D
  std::vector<double> dd(R * H);
  orc_grouped_gemm(h_hat.data(), off.data(), E, wdn.data(), H, I, dd.data(), nullptr, threads);
  std::vector<float> d(R * H);
  orc_round_bf16_n(dd.data(), R * H, d.data());
  // 6. combine
  orc_combine(d.data(), H, inv.data(), topk_w, T, k, out->y);

  auto put = [](auto *dst, const auto &src) {
    if (dst != nullptr) std::copy(src.begin(), src.end(), dst);
  };
  put(out->x_q, xq);
  put(out->x_sf, xsf);
  put(out->x_s_dec, xsd);
  put(out->offsets, off);
  put(out->padded_offsets, pad);
  put(out->perm, perm);
  put(out->inv_perm, inv);
  put(out->h, h);
  put(out->h_q, hq);
  put(out->h_sf, hsf);
  put(out->h_s_dec, hsd);
  put(out->d, d);
  return 0;
}

// R19: the W4A16 variant of orc_expert_layer -- BF16 activations, NVFP4
// weights.  Outputs y, the permutation, h (BF16, sorted rows) and D.
int orc_expert_layer_w4a16(const float *x, const int32_t *topk_idx, const float *topk_w, const float *w_gate_up,
                           const float *w_down, int64_t T, int64_t H, int64_t I, int E, int k, int threads,
                           OrcLayerOut *out) {
  if (H % 16 != 0 || I % 16 != 0 || out == nullptr || out->y == nullptr) return -1;
  const int64_t R = T * k;
  std::vector<int32_t> off(E + 1), pad(E + 1), perm(R), inv(R);
  if (orc_permutation(topk_idx, T, k, E, off.data(), pad.data(), perm.data(), inv.data()) != 0) return -1;
  std::vector<double> a(R * H);
  for (int64_t p = 0; p < R; ++p) {
    const int64_t t = perm[p] / k;
    for (int64_t c = 0; c < H; ++c) a[p * H + c] = x[t * H + c];
  }
  std::vector<double> wgu((int64_t)E * 2 * I * H), wdn((int64_t)E * H * I);
  for (int e = 0; e < E; ++e) {
    std::vector<uint8_t> q(2 * I * H / 2), sc(2 * I * H / 16);
    float sd, am;
    orc_quantize(w_gate_up + (int64_t)e * 2 * I * H, 2 * I, H, 0, nullptr, q.data(), sc.data(), &sd, &am);
    orc_dequantize(q.data(), sc.data(), &sd, 2 * I, H, 0, &wgu[(int64_t)e * 2 * I * H]);
    std::vector<uint8_t> q2(H * I / 2), s2(H * I / 16);
    orc_quantize(w_down + (int64_t)e * H * I, H, I, 0, nullptr, q2.data(), s2.data(), &sd, &am);
    orc_dequantize(q2.data(), s2.data(), &sd, H, I, 0, &wdn[(int64_t)e * H * I]);
  }
  std::vector<double> gu(R * 2 * I), hd(R * I), hb(R * I), dd(R * H);
  orc_grouped_gemm(a.data(), off.data(), E, wgu.data(), 2 * I, H, gu.data(), nullptr, threads);
  orc_swiglu(gu.data(), R, I, hd.data());
  std::vector<float> h(R * I);
  orc_round_bf16_n(hd.data(), R * I, h.data());
  for (int64_t i = 0; i < R * I; ++i) hb[i] = h[i];
  orc_grouped_gemm(hb.data(), off.data(), E, wdn.data(), H, I, dd.data(), nullptr, threads);
  std::vector<float> d(R * H);
  orc_round_bf16_n(dd.data(), R * H, d.data());
  orc_combine(d.data(), H, inv.data(), topk_w, T, k, out->y);
  auto put = [](auto *dst, const auto &src) {
    if (dst != nullptr) std::copy(src.begin(), src.end(), dst);
  };
  put(out->offsets, off);
  put(out->padded_offsets, pad);
  put(out->perm, perm);
  put(out->inv_perm, inv);
  put(out->h, h);
  put(out->d, d);
  return 0;
}

// R17: MXFP8 quantization of rows x [M][K] (K % 32 == 0): codes [M][K]
// (E4M3, bit 7 the sign) and scales [M][K/32] (E8M0 code = s + 127).
int orc_mxfp8_quantize(const float *x, int64_t M, int64_t K, uint8_t *codes, uint8_t *scales) {
  if (K % 32 != 0) return -1;
  for (int64_t r = 0; r < M; ++r) {
    for (int64_t b = 0; b < K / 32; ++b) {
      const float *v = x + r * K + b * 32;
      double amax = 0.0;
      for (int i = 0; i < 32; ++i) amax = std::max(amax, std::fabs((double)v[i]));
      int s = -127;
      if (amax > 0.0) {
        int e2;
        std::frexp(amax, &e2);        // amax = f * 2^e2, f in [0.5, 1): floor(log2 amax) = e2 - 1
        s = std::min(127, std::max(-127, (e2 - 1) - 8));
      }
      scales[r * (K / 32) + b] = (uint8_t)(s + 127);
      for (int i = 0; i < 32; ++i) {
        const double y = std::ldexp((double)v[i], -s);   // exact: a power-of-two scale
        const int mag = nearest_even(std::fabs(y), kUE4M3.v, 127);
        codes[r * K + b * 32 + i] = (uint8_t)(mag | (std::signbit(y) ? 0x80 : 0));
      }
    }
  }
  return 0;
}

void orc_mxfp8_dequantize(const uint8_t *codes, const uint8_t *scales, int64_t M, int64_t K, double *out) {
  for (int64_t r = 0; r < M; ++r)
    for (int64_t c = 0; c < K; ++c) {
      const uint8_t q = codes[r * K + c];
      const double m = ue4m3_value(q & 0x7F);
      out[r * K + c] = std::ldexp((q & 0x80) ? -m : m, (int)scales[r * (K / 32) + c / 32] - 127);
    }
}

// R20: the W4A8 variant -- NVFP4 weights, MXFP8 activations (x and h).
// Outputs y, the permutation, h (BF16 before its MXFP8 requantization,
// sorted rows) and D.
int orc_expert_layer_w4a8(const float *x, const int32_t *topk_idx, const float *topk_w, const float *w_gate_up,
                          const float *w_down, int64_t T, int64_t H, int64_t I, int E, int k, int threads,
                          OrcLayerOut *out) {
  if (H % 32 != 0 || I % 32 != 0 || out == nullptr || out->y == nullptr) return -1;
  const int64_t R = T * k;
  std::vector<int32_t> off(E + 1), pad(E + 1), perm(R), inv(R);
  if (orc_permutation(topk_idx, T, k, E, off.data(), pad.data(), perm.data(), inv.data()) != 0) return -1;
  // x: MXFP8 per token, dequantized exactly
  std::vector<uint8_t> xc(T * H), xs(T * (H / 32));
  orc_mxfp8_quantize(x, T, H, xc.data(), xs.data());
  std::vector<double> xd(T * H);
  orc_mxfp8_dequantize(xc.data(), xs.data(), T, H, xd.data());
  std::vector<double> a(R * H);
  for (int64_t p = 0; p < R; ++p) {
    const int64_t t = perm[p] / k;
    for (int64_t c = 0; c < H; ++c) a[p * H + c] = xd[t * H + c];
  }
  std::vector<double> wgu((int64_t)E * 2 * I * H), wdn((int64_t)E * H * I);
  for (int e = 0; e < E; ++e) {
    std::vector<uint8_t> q(2 * I * H / 2), sc(2 * I * H / 16);
    float sd, am;
    orc_quantize(w_gate_up + (int64_t)e * 2 * I * H, 2 * I, H, 0, nullptr, q.data(), sc.data(), &sd, &am);
    orc_dequantize(q.data(), sc.data(), &sd, 2 * I, H, 0, &wgu[(int64_t)e * 2 * I * H]);
    std::vector<uint8_t> q2(H * I / 2), s2(H * I / 16);
    orc_quantize(w_down + (int64_t)e * H * I, H, I, 0, nullptr, q2.data(), s2.data(), &sd, &am);
    orc_dequantize(q2.data(), s2.data(), &sd, H, I, 0, &wdn[(int64_t)e * H * I]);
  }
  std::vector<double> gu(R * 2 * I), hd(R * I), dd(R * H);
  orc_grouped_gemm(a.data(), off.data(), E, wgu.data(), 2 * I, H, gu.data(), nullptr, threads);
  orc_swiglu(gu.data(), R, I, hd.data());
  std::vector<float> h(R * I);
  orc_round_bf16_n(hd.data(), R * I, h.data());
  // h: MXFP8 per row, dequantized exactly
  std::vector<uint8_t> hc(R * I), hs(R * (I / 32));
  orc_mxfp8_quantize(h.data(), R, I, hc.data(), hs.data());
  std::vector<double> hq(R * I);
  orc_mxfp8_dequantize(hc.data(), hs.data(), R, I, hq.data());
  orc_grouped_gemm(hq.data(), off.data(), E, wdn.data(), H, I, dd.data(), nullptr, threads);
  std::vector<float> d(R * H);
  orc_round_bf16_n(dd.data(), R * H, d.data());
  orc_combine(d.data(), H, inv.data(), topk_w, T, k, out->y);
  auto put = [](auto *dst, const auto &src) {
    if (dst != nullptr) std::copy(src.begin(), src.end(), dst);
  };
  put(out->offsets, off);
  put(out->padded_offsets, pad);
  put(out->perm, perm);
  put(out->inv_perm, inv);
  put(out->h, h);
  put(out->d, d);
  return 0;
}

// R16 pieces.  SwiGLU backward per element, fp64: with s = 1/(1+exp(-g)),
// silu = g s, h = silu u, dh = w dh':  dg = dh u s (1 + g (1 - s)),
// du = dh silu.  gu [R][2I] (gate, then up), dhp [R][I], w [R] -> dgu
// [R][2I], h [R][I].
void orc_swiglu_backward(const double *gu, const double *dhp, const double *w, int64_t R, int64_t I, double *dgu,
                         double *h) {
  for (int64_t r = 0; r < R; ++r)
    for (int64_t i = 0; i < I; ++i) {
      const double g = gu[r * 2 * I + i], u = gu[r * 2 * I + I + i];
      const double sg = 1.0 / (1.0 + std::exp(-g));
      const double silu = g * sg;
      const double dh = w[r] * dhp[r * I + i];
      dgu[r * 2 * I + i] = dh * u * (sg * (1.0 + g * (1.0 - sg)));
      dgu[r * 2 * I + I + i] = dh * silu;
      h[r * I + i] = silu * u;
    }
}

// R16: gradients of sum(dy * y) for the unquantized layer, all in fp64:
//   per routed row (t, j), e = topk_idx[t][j], in the sorted order of R8:
//   G = W_gu,e x[t] = [g | u], h = silu(g) u, D = W_dn,e h
//   dD = w[t][j] dy[t];  d topk_w[t][j] = <dy[t], D>
//   dh = W_dn,e^T dD;     dW_dn,e += dD h^T
//   dg = dh u silu'(g), du = dh silu(g)
//   dx[t] += W_gu,e^T [dg | du];  dW_gu,e += [dg | du] x[t]^T
// Inputs are BF16 values held as floats: x [T][H], dy [T][H], w_gate_up
// [E][2I][H], w_down [E][H][I], topk_w [T][k].  Outputs (fp64): dx [T][H],
// dtopk_w [T][k], dw_gate_up [E][2I][H], dw_down [E][H][I].
int orc_expert_layer_backward(const float *x, const int32_t *topk_idx, const float *topk_w, const float *w_gate_up,
                              const float *w_down, const float *dy, int64_t T, int64_t H, int64_t I, int E, int k,
                              int threads, double *dx, double *dtopk_w, double *dw_gate_up, double *dw_down) {
  const int64_t R = T * k;
  std::vector<int32_t> off(E + 1), pad(E + 1), perm(R), inv(R);
  if (orc_permutation(topk_idx, T, k, E, off.data(), pad.data(), perm.data(), inv.data()) != 0) return -1;
  std::vector<double> wgu((int64_t)E * 2 * I * H), wdn((int64_t)E * H * I), wguT((int64_t)E * H * 2 * I),
      wdnT((int64_t)E * I * H);
  for (int64_t i = 0; i < (int64_t)wgu.size(); ++i) wgu[i] = w_gate_up[i];
  for (int64_t i = 0; i < (int64_t)wdn.size(); ++i) wdn[i] = w_down[i];
  for (int e = 0; e < E; ++e) {
    for (int64_t n = 0; n < 2 * I; ++n)
      for (int64_t c = 0; c < H; ++c) wguT[((int64_t)e * H + c) * 2 * I + n] = wgu[((int64_t)e * 2 * I + n) * H + c];
    for (int64_t n = 0; n < H; ++n)
      for (int64_t c = 0; c < I; ++c) wdnT[((int64_t)e * I + c) * H + n] = wdn[((int64_t)e * H + n) * I + c];
  }
  // rows in sorted order
  std::vector<double> a(R * H), dyr(R * H), wr(R);
  for (int64_t p = 0; p < R; ++p) {
    const int64_t t = perm[p] / k;
    for (int64_t c = 0; c < H; ++c) {
      a[p * H + c] = x[t * H + c];
      dyr[p * H + c] = dy[t * H + c];
    }
    wr[p] = topk_w[perm[p]];
  }
  // forward, unquantized
  std::vector<double> gu(R * 2 * I), h(R * I), d(R * H);
  orc_grouped_gemm(a.data(), off.data(), E, wgu.data(), 2 * I, H, gu.data(), nullptr, threads);
  orc_swiglu(gu.data(), R, I, h.data());
  orc_grouped_gemm(h.data(), off.data(), E, wdn.data(), H, I, d.data(), nullptr, threads);
  // combine backward
  std::vector<double> dd(R * H);
  for (int64_t p = 0; p < R; ++p) {
    double s = 0.0;
    for (int64_t c = 0; c < H; ++c) {
      dd[p * H + c] = wr[p] * dyr[p * H + c];
      s += dyr[p * H + c] * d[p * H + c];
    }
    dtopk_w[perm[p]] = s;
  }
  // down: dgrad and wgrad
  std::vector<double> dh(R * I), ones(R, 1.0), dgu(R * 2 * I), hh(R * I);
  orc_grouped_gemm(dd.data(), off.data(), E, wdnT.data(), I, H, dh.data(), nullptr, threads);
  for (int e = 0; e < E; ++e)
    for (int64_t n = 0; n < H; ++n)
      for (int64_t c = 0; c < I; ++c) {
        double s = 0.0;
        for (int64_t p = off[e]; p < off[e + 1]; ++p) s += dd[p * H + n] * h[p * I + c];
        dw_down[((int64_t)e * H + n) * I + c] = s;
      }
  // SwiGLU (dh already carries the routing weight: w = 1 here)
  orc_swiglu_backward(gu.data(), dh.data(), ones.data(), R, I, dgu.data(), hh.data());
  // gate_up: dgrad to the rows, summed back to the tokens in slot order; wgrad
  std::vector<double> dxr(R * H);
  orc_grouped_gemm(dgu.data(), off.data(), E, wguT.data(), H, 2 * I, dxr.data(), nullptr, threads);
  for (int64_t t = 0; t < T; ++t)
    for (int64_t c = 0; c < H; ++c) {
      double s = 0.0;
      for (int j = 0; j < k; ++j) s += dxr[(int64_t)inv[t * k + j] * H + c];
      dx[t * H + c] = s;
    }
  for (int e = 0; e < E; ++e)
    for (int64_t n = 0; n < 2 * I; ++n)
      for (int64_t c = 0; c < H; ++c) {
        double s = 0.0;
        for (int64_t p = off[e]; p < off[e + 1]; ++p) s += dgu[p * 2 * I + n] * a[p * H + c];
        dw_gate_up[((int64_t)e * 2 * I + n) * H + c] = s;
      }
  return 0;
}

}  // extern "C"
