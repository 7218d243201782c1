// Internal launch interface between the C-ABI layer and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace nvfp4moe {

// Where the rows a quantize launch reads come from and where they go.
enum QuantMode : int {
  kQuantPlain = 0,     // row i -> row i (nvfp4_quantize)
  kQuantScatter = 1,   // token t -> its k rows in the padded grouped layout
  kQuantRequant = 2,   // padded row p of h -> row p, amax given (k_requant_blocks)
  kQuantWeights = 3,   // expert e row n -> expert e row interleave(n)
};

// Byte layouts of a scale matrix (one UE4M3 byte per 16 elements along K):
//   kSfRowMajor  [rows][K/16]
//   kSfMma       the 128-row x 4-scale atoms the block-scaled MMA reads
//   kSfKStep     [K/256][rows_cap][16]: the 16 scales of one 256-element
//                K-step of a row are 16 contiguous bytes, and the scales of
//                128 consecutive rows for one K-step are 2 KB contiguous
enum SfLayout : int { kSfRowMajor = 0, kSfMma = 1, kSfKStep = 2 };

struct QuantParams {
  const void *x = nullptr;          // BF16 source
  int64_t tasks = 0;                // rows (plain), tokens (scatter), E*N (weights); requant walks rows_cap
  int64_t K = 0;                    // elements per row
  int mode = kQuantPlain;
  // amax: amax_src is the per-tensor value (index 0), per-row values, or per
  // expert values (weights); amax_rows == 1 means per row.
  const float *amax_src = nullptr;
  int amax_rows = 0;
  int compute_row_amax = 0;         // per-row amax computed here (no amax_src)
  float *amax_out = nullptr;        // per-row amax written here (per-row modes)
  // outputs
  uint8_t *q = nullptr;
  uint8_t *sf = nullptr;
  int sf_layout = 0;                // SfLayout
  float *s_dec = nullptr;           // per tensor [1], per row, or per expert
  int s_dec_rows = 0;               // 1: one S_dec per destination row
  int64_t rows_cap = 0;             // destination rows allocated (bounds check)
  // grouped layout (scatter / requant)
  const int32_t *topk_idx = nullptr;
  const int32_t *inv_perm = nullptr;    // given positions (standalone scatter)
  const int32_t *offsets = nullptr;
  const int32_t *padded_offsets = nullptr;
  int k = 1;
  int E = 1;
  // fused ranks (layer path): positions from per-block bases + local ranks
  const int32_t *local_rank = nullptr;
  const int32_t *block_base = nullptr;
  int32_t *perm_out = nullptr;
  int32_t *inv_perm_out = nullptr;
  float *zero_rows = nullptr;       // per-row buffer zeroed at each destination
  // weights
  int64_t N = 0;
  int gate_up = 0;
  int *err = nullptr;
};

constexpr int kRankTokens = 128;    // tokens per routing block

cudaError_t launch_amax(const void *x, int64_t seg_len, int64_t nseg, float *out, cudaStream_t s);
cudaError_t launch_quant(const QuantParams &p, cudaStream_t s);
cudaError_t launch_encode_e2m1(const float *y, int64_t n, uint8_t *codes, cudaStream_t s);
cudaError_t launch_encode_ue4m3(const float *v, int64_t n, uint8_t *codes, cudaStream_t s);

struct PermuteParams {
  const int32_t *topk_idx;
  int64_t T;
  int k;
  int E;
  int32_t *block_counts;   // [nblk][E]
  int32_t *local_rank;     // [T*k]
  int32_t *offsets;        // [E+1]
  int32_t *padded_offsets; // [E+1]
  int32_t *perm;           // [T*k] (rank kernel)
  int32_t *inv_perm;       // [T*k] (rank kernel)
  int *err;
  // optional: per-row floats zeroed on every padding row [padded start + count,
  // padded end) of each group below rows_cap (scan kernel)
  float *zero_pad_rows = nullptr;
  int64_t rows_cap = 0;
  // optional: route from router logits [T][E] inside the count kernel; the
  // chosen ids / weights go to topk_idx_out (which topk_idx must equal) and
  // topk_w_out
  const float *logits = nullptr;
  int32_t *topk_idx_out = nullptr;
  float *topk_w_out = nullptr;
};
int64_t permute_blocks(int64_t T);
cudaError_t launch_route_count(const PermuteParams &p, cudaStream_t s);
cudaError_t launch_route_scan(const PermuteParams &p, cudaStream_t s);
cudaError_t launch_route_rank(const PermuteParams &p, cudaStream_t s);

enum GemmEpilogue : int { kEpiStore = 0, kEpiSwiGLU = 1 };

struct GemmArgs {
  const uint8_t *q_a, *sf_a;
  const float *s_dec_a;
  int s_dec_a_rows;
  const uint8_t *q_w, *sf_w;
  const float *s_dec_w;
  const int32_t *offsets, *padded_offsets;
  int E;
  int64_t rows_cap, N, K;
  int epilogue;
  void *out_bf16;
  float *out_f32;
  int out_padded;
  float *amax_h;      // SwiGLU: amax of h (per row [rows_cap] or [1])
  int amax_h_rows;
  // SwiGLU with per-row amax: requantize h inside the launch (nullable = no)
  uint8_t *req_q;         // [rows_cap][N/4] codes of h
  uint8_t *req_sf;        // K-step-major scales of h
  float *req_s_dec;       // [rows_cap]
  int discard_h;          // drop h's L2 lines once requantized (h undefined after)
  // plain-store epilogue, non-strict combine: y[t] += w * out_row (FP32
  // reductions) instead of storing the rows (nullable = store)
  float *red_y;           // [T][N]
  const int32_t *red_perm;  // perm[R]: compact sorted row -> t * k + j
  const float *red_w;       // topk_w [T * k]
  int red_k;
  int *err;
};
cudaError_t launch_grouped_gemm(const GemmArgs &a, cudaStream_t s);

// ---------------------------------------------------------------- BF16 ----
// BF16 x BF16 -> FP32 grouped GEMM on tcgen05 (kind::f16), for the layer's
// BF16 backward.
enum Bf16GemmMode : int {
  kBfRows = 0,    // per expert e: C[r][n] = sum_k A[r][k] * B_e[n][k], r over e's padded rows
  kBfWgrad = 1,   // per expert e: C_e[m][n] = sum_{r in group e} A[r][m] * B[r][n]
};
enum Bf16Epilogue : int {
  kBfStore = 0,       // BF16 and/or FP32 output
  kBfSwiGLUBwd = 1,   // backward of SwiGLU and of the combine's dot (see gemm_bf16.cu)
  kBfSwiGLUFwd = 2,   // W4A16 gate_up: h = BF16(silu(g) u) of the scaled accumulator
};

struct Bf16GemmArgs {
  int mode = kBfRows;
  // operand layouts: A is K-major [rows_cap][K] (kBfRows) or MN-major
  // [rows_cap][M] (kBfWgrad); B is K-major [E][N][K], MN-major [E][K][N]
  // (kBfRows), or MN-major [rows_cap][N] (kBfWgrad)
  int b_mn = 0;
  const void *a = nullptr;
  const void *b = nullptr;
  const int32_t *offsets = nullptr, *padded_offsets = nullptr;
  int E = 1;
  int64_t rows_cap = 0, M = 0, N = 0, K = 0;
  int epilogue = kBfStore;
  void *out_bf16 = nullptr;     // kBfRows: [rows][N] (padded or compact); kBfWgrad: [E][M][N]
  float *out_f32 = nullptr;
  int out_padded = 1;
  // kBfSwiGLUBwd (kBfRows, N = I): the accumulator is dh' = dy_rows W_dn
  const void *g_u = nullptr;    // BF16 [rows_cap][2I]: gate columns, then up columns
  const float *w_rows = nullptr;  // [rows_cap] routing weight of each row (0 on padding)
  void *d_gu = nullptr;         // BF16 [rows_cap][2I] (out)
  void *hw = nullptr;           // BF16 [rows_cap][I] (out): w * BF16(silu(g) u)
  float *dw_part = nullptr;     // [rows_cap][I/128] (out): partial <dh', h> per 128 columns
  // W4A16 (kBfRows, B K-major): B is NVFP4 -- b holds the E2M1 codes
  // [E][N][K/2], b_sf the UE4M3 block scales in the MMA atom layout, s_dec_w
  // the per-expert decode scale applied to the accumulator in the epilogue
  const uint8_t *b_sf = nullptr;
  const float *s_dec_w = nullptr;
  int w4_wide = 0;              // units of 256 weight rows (else 128)
  // kBfRows, K-major B (optional): the rows the A and B tensors really hold
  // (tile rows past them read as zeros), and the FP32 output's valid columns
  // and leading dimension (0: rows_cap, E * N, N and N)
  int64_t a_rows = 0, b_rows = 0, n_store = 0, out_ld = 0;
  // kBfSwiGLUFwd: h is MXFP8 quantize-dequantized (W4A8); h_pre (optional)
  // receives the BF16 h before that, [rows_cap][I]
  int mxfp8_h = 0;
  void *h_pre = nullptr;
  int *err = nullptr;
};
cudaError_t launch_bf16_gemm(const Bf16GemmArgs &a, cudaStream_t s);
// Expert parallelism (ep.cu): tables from the [G][El] row counts, the
// arrangement of received rows into the padded grouped layout, and the
// return of D rows in received order.
struct EpArrangeParams {
  const uint8_t *q_recv = nullptr, *sf_recv = nullptr;   // [rows_recv][H/2], row-major [rows_recv][H/16]
  const float *sdec_recv = nullptr;                       // [rows_recv]
  const int32_t *counts = nullptr;                        // [G][El]
  const int32_t *offsets = nullptr, *padded = nullptr;    // [El+1] (from the tables)
  const int32_t *tab = nullptr;                           // recv_start, pad_start, cmp_start, [G*El] each
  int G = 1, El = 1;
  int64_t rows_recv = 0, H = 0, rows_cap = 0;
  uint8_t *q_a = nullptr, *sf_a = nullptr;                // [rows_cap][H/2], K-step-major
  float *sdec_a = nullptr;                                // [rows_cap]
  int *err = nullptr;
};
cudaError_t launch_ep_tables(const int32_t *counts, int G, int El, int32_t *offsets, int32_t *padded, int32_t *tab,
                             int *err, cudaStream_t s);
cudaError_t launch_ep_arrange(const EpArrangeParams &a, cudaStream_t s);
cudaError_t launch_ep_return(const void *d, const int32_t *tab, int P, int64_t rows_recv, int64_t H, void *d_send,
                             int *err, cudaStream_t s);
// offsets {0, T} and padded offsets {0, Tpad} of the router GEMM's single group, in meta[0..3]
cudaError_t launch_router_meta(int32_t *meta, int64_t T, int64_t Tpad, cudaStream_t s);

// Backward helpers: gather x and dy rows into the padded grouped layout
// (zeros on padding rows), the row weights, and ones for the dx combine
// (dy / dy_rows, w_rows and ones may be null).
struct BwdGatherParams {
  const void *x, *dy;
  const float *topk_w;
  const int32_t *topk_idx, *perm, *offsets, *padded_offsets;
  const int32_t *inv_perm;   // [T][k] compact row of each (token, slot), -1 if unrouted
  int64_t T, H, rows_cap;
  int k, E;
  void *x_rows, *dy_rows;
  float *w_rows, *ones;
  int mxfp8_x = 0;   // x rows are MXFP8 quantize-dequantized (W4A8)
};
cudaError_t launch_bwd_gather(const BwdGatherParams &p, cudaStream_t s);
cudaError_t launch_bwd_dw(const float *dw_part, int64_t nparts, const int32_t *inv_perm, const int32_t *topk_idx,
                          const int32_t *offsets, const int32_t *padded_offsets, int64_t T, int k, int E,
                          float *dw, cudaStream_t s);

cudaError_t launch_combine(const void *d, const int32_t *inv_perm, const float *w, int64_t T, int k,
                           int64_t H, void *y, cudaStream_t s);
cudaError_t launch_f32_to_bf16(const float *src, int64_t n, void *dst, cudaStream_t s);

cudaError_t launch_wait_selftest(int *err, cudaStream_t s);
cudaError_t launch_mma_peak(int iters, int scale_writes, long long *cycles, int *err, int grid, cudaStream_t s);

int num_sms();

}  // namespace nvfp4moe
