/*
 * nvfp4moe -- NVFP4 W4A4 MoE expert layer for NVIDIA B200 (sm_100a).
 *
 * The operation is the MoE expert linear layer of miniTE's NVFP4 learner:
 *   news.hamidun.com "miniTE ... 1.39x over BF16 on Qwen3-30B-A3B" (Arabic and
 *   Russian editions), key facts: native NVFP4 W4A4 (4-bit weights and
 *   activations); section "diagnostics, alignment and fast kernels": grouped
 *   GEMMs over the many experts of Qwen3-30B-A3B; strict-alignment mode.
 *   www.aib.vote "miniTE report, NVFP4 RL stability", paragraph 4: the
 *   token-wise NVFP4 path of Transformer Engine -- contiguous data layout,
 *   device-side metadata, amax reuse, grouped matrix multiplication and
 *   operator fusion.
 *
 * Data formats (the pages name NVFP4; the format itself is the public NVFP4
 * definition):
 *   codes   E2M1, two per byte, element 2i in the low nibble of byte i
 *   scales  one UE4M3 byte per 16 consecutive elements along K
 *   S_dec   FP32 decode scale, per tensor or per row; x ~ e2m1 * sf * S_dec
 *   Quantization: amax -> S_enc = 2688/amax, S_dec = 1/S_enc (binary32);
 *   sf = UE4M3_rne_satfinite((bamax/6)*S_enc); code = E2M1_rne_satfinite(x*S_enc/sf).
 *
 * Scale-factor layouts
 *   row-major     scales[row][K/16]
 *   MMA layout    the 128-row x 4-scale atom the tcgen05 block-scaled MMA reads:
 *                 byte(row, b) = ((row/128)*(K/64) + b/4)*512 + (row%32)*16
 *                                + ((row%128)/32)*4 + b%4
 *                 (rows of a matrix padded to a multiple of 128).
 *   K-step-major  the activations' layout in the padded grouped layout:
 *                 byte(row, b) = ((b/16)*rows_cap + row)*16 + b%16, i.e.
 *                 [K/256][rows_cap][16] -- the 16 scales of a row's 256-element
 *                 K-step are contiguous, and a 128-row tile's scales for one
 *                 K-step are 2 KB contiguous (one bulk copy for the GEMM).
 *
 * Conventions for every entry point
 *   - Pointers are DEVICE pointers unless the comment says host.  The caller
 *     owns and allocates every buffer (workspace included); the library never
 *     allocates device memory and never synchronizes the host, except
 *     nvfp4moe_device_status() which says so.
 *   - All work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *     stream) and is stream-ordered.
 *   - Argument, shape and alignment errors are returned before anything is
 *     launched.  A CUDA launch error is returned as NVFP4MOE_ERR_CUDA.  Errors
 *     the kernels detect (an expert index out of range, a duplicate expert in
 *     one token's top-k, a wait that timed out) are recorded in an error word
 *     inside the caller's workspace and read with nvfp4moe_device_status().
 *   - Device pointers must be 16-byte aligned; sizes: K % 256 == 0 and
 *     N % 256 == 0 for the grouped GEMM, K % 64 == 0 for the quantizer.
 */
#ifndef NVFP4MOE_H
#define NVFP4MOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* A cudaStream_t, declared without the CUDA headers. */
typedef struct CUstream_st *nvfp4moe_stream_t;

typedef enum {
  NVFP4MOE_OK = 0,
  NVFP4MOE_ERR_INVALID_ARG = -1,      /* null pointer, negative size, bad flag   */
  NVFP4MOE_ERR_MISALIGNED = -2,       /* a pointer is not 16-byte aligned        */
  NVFP4MOE_ERR_UNSUPPORTED_SHAPE = -3,/* K, N or E outside what the kernels take */
  NVFP4MOE_ERR_CUDA = -4,             /* a CUDA runtime / driver call failed     */
  NVFP4MOE_ERR_DEVICE_TIMEOUT = -5,   /* a kernel wait ran out (device status)   */
  NVFP4MOE_ERR_WORKSPACE = -6,        /* workspace missing or too small          */
  NVFP4MOE_ERR_DEVICE_CHECK = -7      /* kernel-side input check failed (device status) */
} nvfp4moe_status;

/* ---------------------------------------------------------------- flags -- */
/* One FP32 global scale per row (token) instead of one per tensor. */
#define NVFP4MOE_SCALE_PER_TOKEN 0x1u
/* Strict alignment (the pages' strict-alignment mode): per-token scales and a
 * reduction order fixed per output element, so each token's output is bitwise
 * identical however the tokens are batched, ordered or grouped. */
#define NVFP4MOE_STRICT 0x2u
/* Scale factors are written / read in the MMA atom layout (see above). */
#define NVFP4MOE_SF_MMA_LAYOUT 0x4u
/* Grouped GEMM: write output rows at their padded positions instead of the
 * compact sorted positions. */
#define NVFP4MOE_OUT_PADDED 0x8u
/* nvfp4_prepare_weights: the matrix is a fused gate_up [2I][K] (gate rows
 * 0..I-1, up rows I..2I-1); store rows in the order the fused SwiGLU epilogue
 * reads (per 256-row tile: 128 gate rows then the matching 128 up rows). */
#define NVFP4MOE_W_GATE_UP 0x10u
/* moe_expert_layer with per-token scales: requantize h inside the gate_up
 * GEMM launch instead of a separate pass.  The GEMM then walks each CTA's
 * m-tiles with all their n-tiles in a row, so a row of h and its amax are
 * complete inside one CTA, and two worker warps per CTA requantize an m-tile
 * from L2 while the tensor cores run the next one.  Outputs are bitwise the
 * same as the separate pass.  Measured on the Qwen3-30B-A3B-shaped layer it
 * is slower than the separate pass (the requantization needs more warps than
 * a GEMM CTA can give it), so it is off by default. */
#define NVFP4MOE_FUSED_REQUANT 0x100u
/* With NVFP4MOE_FUSED_REQUANT: keep h (BF16) readable in the workspace.
 * Without it the fused path drops h's cache lines once requantized, without
 * writing them to HBM, and the workspace's h region holds undefined values
 * afterwards.  Outputs are identical either way. */
#define NVFP4MOE_KEEP_H 0x20u
/* moe_expert_layer, non-strict: the down GEMM's epilogue adds w[t][j] * D
 * (FP32, before any BF16 rounding) straight into an FP32 accumulator of y
 * with reductions (red.global.add), and a last pass rounds it to BF16, so D
 * never goes to memory.  The order of the additions follows the GEMM's tile
 * completion, so y is not bitwise reproducible: not allowed with
 * NVFP4MOE_STRICT (NVFP4MOE_ERR_INVALID_ARG). */
#define NVFP4MOE_FAST_COMBINE 0x80u

const char *nvfp4moe_status_string(int status);
int nvfp4moe_version(void);

/* Reads and clears the error word of a workspace (the first 16 bytes of every
 * workspace this library uses): synchronizes `stream`, copies the word to the
 * host, zeroes it, and returns NVFP4MOE_OK, NVFP4MOE_ERR_DEVICE_CHECK or
 * NVFP4MOE_ERR_DEVICE_TIMEOUT.  This is the one call that blocks the host. */
int nvfp4moe_device_status(void *workspace, nvfp4moe_stream_t stream);

/* Self-test of the failure path every kernel's waits share (no counterpart on
 * the pages): enqueues one kernel that waits on a barrier nothing completes.
 * After the wait bound (2 s) the kernel records a timeout in the error word
 * of `workspace` (16 bytes at least) and returns; nothing faults and the
 * context stays usable.  A following nvfp4moe_device_status() returns
 * NVFP4MOE_ERR_DEVICE_TIMEOUT. */
int nvfp4moe_wait_selftest(void *workspace, nvfp4moe_stream_t stream);

/* ------------------------------------------------------------ quantize -- */
/* NVFP4-quantize x [M][K] BF16 (row-major).  The token-wise NVFP4 path with
 * amax reuse (www.aib.vote "miniTE report", paragraph 4).
 *   amax_in   nullable.  Per-tensor mode: [1]; per-token: [M].  When given,
 *             it is used as is (amax reuse) and no amax pass runs.
 *   amax_out  nullable, same shape; receives the amax used.  In per-tensor
 *             mode without amax_in it is REQUIRED (the reduction target).
 *   q         [M][K/2] packed E2M1 codes (out)
 *   scales    UE4M3 scales, row-major [M][K/16] or, with
 *             NVFP4MOE_SF_MMA_LAYOUT, the MMA layout over roundup(M,128) rows
 *   s_dec     [1] (per tensor) or [M] (per token) FP32 decode scales (out)
 *   flags     NVFP4MOE_SCALE_PER_TOKEN | NVFP4MOE_STRICT | NVFP4MOE_SF_MMA_LAYOUT
 * Requirements: K % 64 == 0, M >= 0 (M == 0 is a no-op). */
int nvfp4_quantize(const void *x, int64_t M, int64_t K, const float *amax_in,
                   float *amax_out, uint8_t *q, uint8_t *scales, float *s_dec,
                   uint32_t flags, nvfp4moe_stream_t stream);

/* -------------------------------------------------------------- routing -- */
/* Top-k routing from router logits, on the device: the inputs of
 * moe_permute without a trip through the host.  The pages' MoE learner runs
 * Qwen3-30B-A3B (news.hamidun.com "miniTE ... 1.39x": 128 experts, 8 active
 * per token) and keeps the token-wise path's metadata on the device
 * (www.aib.vote "miniTE report", paragraph 4); the routing rule itself is not
 * on the pages and follows Qwen3-MoE: for each token the k experts with the
 * largest logits (ties to the lower expert id), slots in descending logit
 * order, weights = softmax over the chosen k.  The choice compares the FP32
 * logits exactly; the weights are FP32 (expf, one IEEE division each).
 *   logits    [T][E] FP32 router logits (the dense router GEMM's output,
 *             computed by the caller), finite values
 *   topk_idx  [T][k] int32 expert ids (out)
 *   topk_w    [T][k] FP32 weights, summing to 1 per token (out)
 * Requirements: 1 <= k <= min(E, 32), E <= 1024; T == 0 is a no-op.
 * NVFP4MOE_ERR_UNSUPPORTED_SHAPE beyond those limits. */
int moe_route_topk(const float *logits, int64_t T, int E, int k, int32_t *topk_idx,
                   float *topk_w, nvfp4moe_stream_t stream);

/* ------------------------------------------------------------- permute -- */
/* Token-to-expert permutation into a contiguous per-expert layout with
 * device-side group offsets (www.aib.vote "miniTE report", paragraph 4:
 * contiguous layout, device-side metadata).  Rows are ordered by
 * (expert, token, slot); the host never learns the group sizes.
 *   topk_idx        [T][k] int32 expert ids; each row holds k distinct ids
 *   offsets         [E+1] int32 (out): group e is rows offsets[e]..offsets[e+1]
 *   padded_offsets  [E+1] int32 (out): the same with every group rounded up
 *                   to a multiple of 128 rows (the GEMM tile height)
 *   perm            [T*k] int32 (out): perm[r] = t*k + j for sorted row r
 *   inv_perm        [T][k] int32 (out): inv_perm[t][j] = r
 *   workspace       moe_permute_workspace_size() bytes
 * Out-of-range or duplicate expert ids set NVFP4MOE_ERR_DEVICE_CHECK in the
 * workspace error word; such entries are skipped, nothing is written out of
 * bounds.  Requirements: 1 <= E <= 1024, 1 <= k <= 32. */
size_t moe_permute_workspace_size(int64_t T, int k, int E);
int moe_permute(const int32_t *topk_idx, int64_t T, int k, int E,
                int32_t *offsets, int32_t *padded_offsets, int32_t *perm,
                int32_t *inv_perm, void *workspace, size_t workspace_bytes,
                nvfp4moe_stream_t stream);

/* moe_permute for callers that cannot provide any scratch memory -- code
 * inside a host framework whose memory planner owns all device memory and
 * allows no allocation after start-up, or code running where cudaMalloc is
 * not allowed.  The pages have no counterpart of this entry point.
 * Same arguments and outputs as moe_permute, without the workspace: the
 * scratch is a static device array of the library (about 1 MB per GPU that
 * loads it, held until the process exits).  Limits: T*k <= 131072 and
 * ceil(T/128)*E <= 131072 (NVFP4MOE_ERR_WORKSPACE beyond them).  It allocates
 * nothing; its first call on a device looks up the array's address (make that
 * call before any stream capture).  Calls that overlap on the GPU race on the
 * shared array.  Bad or duplicate expert ids are skipped as in moe_permute
 * but not reported (there is no workspace error word to read). */
int moe_permute_noalloc(const int32_t *topk_idx, int64_t T, int k, int E,
                        int32_t *offsets, int32_t *padded_offsets,
                        int32_t *perm, int32_t *inv_perm,
                        nvfp4moe_stream_t stream);

/* Router and permutation in one pass: the top-k of the router logits is
 * taken inside the routing-histogram kernel (each warp routes its 32 tokens
 * and sets their expert masks directly), then the same scan and ranking as
 * moe_permute.  The pages' token-wise path fuses its operators and keeps its
 * metadata on the device (www.aib.vote "miniTE report", paragraph 4); the
 * routing rule is moe_route_topk's.
 *   logits    [T][E] FP32 router logits (finite)
 *   topk_idx  [T][k] int32 (out), topk_w [T][k] FP32 (out)
 *   offsets, padded_offsets, perm, inv_perm, workspace: as moe_permute
 * Requirements: 1 <= k <= min(E, 32), E <= 1024. */
int moe_route_permute(const float *logits, int64_t T, int E, int k,
                      int32_t *topk_idx, float *topk_w, int32_t *offsets,
                      int32_t *padded_offsets, int32_t *perm, int32_t *inv_perm,
                      void *workspace, size_t workspace_bytes,
                      nvfp4moe_stream_t stream);

/* Quantize each token of x [T][K] once and write its codes, scales and
 * decode scale to all k of its rows in the padded grouped layout (the fused
 * quantize + permute of the token-wise path: amax computed once, reused for
 * every copy).  Uses the inv_perm / offsets / padded_offsets of moe_permute.
 *   q_rows      [rows_cap][K/2] codes at padded row positions (out)
 *   sf_rows     scales in the K-step-major layout (out)
 *   s_dec_rows  [rows_cap] FP32 per-row decode scale (out; per-tensor mode
 *               writes the tensor's S_dec into every row)
 *   amax_in / amax_out as for nvfp4_quantize (per tensor [1], per token [T])
 *   rows_cap    allocated padded rows: >= roundup(T*k + E*127, 128)
 * flags: NVFP4MOE_SCALE_PER_TOKEN | NVFP4MOE_STRICT. */
int moe_quantize_permute(const void *x, int64_t T, int64_t K, int k, int E,
                         const int32_t *topk_idx, const int32_t *inv_perm,
                         const int32_t *offsets, const int32_t *padded_offsets,
                         const float *amax_in, float *amax_out, uint8_t *q_rows,
                         uint8_t *sf_rows, float *s_dec_rows, int64_t rows_cap,
                         uint32_t flags, nvfp4moe_stream_t stream);

/* --------------------------------------------------------- grouped GEMM -- */
/* Block-scaled FP4 x FP4 grouped GEMM over the experts, one launch, group
 * sizes read on the device (news.hamidun.com section "diagnostics, alignment
 * and fast kernels": grouped GEMMs for MoE; www.aib.vote paragraph 4).
 * For every expert e and every row r of its group:
 *   out[r][n] = S_dec_a(r) * S_dec_w[e] * sum_k a(r,k) * w(e,n,k)
 * with a, w the block-scaled E2M1 values; FP32 accumulation in the tensor
 * cores, one rounding to the output type.
 *   q_a, sf_a, s_dec_a  A in the padded grouped layout (moe_quantize_permute):
 *                       q_a [rows_cap][K/2], sf_a K-step-major, s_dec_a
 *                       [rows_cap] (NVFP4MOE_SCALE_PER_TOKEN) or [1]
 *   q_w, sf_w, s_dec_w  weights: q_w [E][N][K/2], sf_w MMA layout per expert
 *                       ([E][N/128][K/64][512] bytes), s_dec_w [E]
 *   offsets, padded_offsets  [E+1] device group offsets (moe_permute)
 *   out_bf16, out_f32   nullable (at least one): [R][N] compact sorted rows,
 *                       or [rows_cap][N] with NVFP4MOE_OUT_PADDED
 *   workspace           16 bytes at least (error word)
 * Requirements: K % 256 == 0, N % 256 == 0, 1 <= E. */
int nvfp4_grouped_gemm(const uint8_t *q_a, const uint8_t *sf_a,
                       const float *s_dec_a, const uint8_t *q_w,
                       const uint8_t *sf_w, const float *s_dec_w,
                       const int32_t *offsets, const int32_t *padded_offsets,
                       int E, int64_t rows_cap, int64_t N, int64_t K,
                       void *out_bf16, float *out_f32, uint32_t flags,
                       void *workspace, size_t workspace_bytes,
                       nvfp4moe_stream_t stream);

/* ------------------------------------------------------------- weights -- */
/* NVFP4 weights of one MoE linear, E experts of [N][K] each, every expert
 * one tensor (one S_dec per expert).  All pointers are device pointers. */
typedef struct {
  uint8_t *q;      /* [E][N][K/2] packed codes, rows in kernel order        */
  uint8_t *sf;     /* [E][N/128][K/64][512] UE4M3, MMA layout              */
  float *s_dec;    /* [E] decode scales                                     */
  float *amax;     /* [E] amax of each expert's BF16 matrix                 */
  int64_t E, N, K;
  uint32_t flags;  /* NVFP4MOE_W_GATE_UP when rows are gate/up interleaved  */
} nvfp4moe_weights;

/* Quantize BF16 weights w [E][N][K] into `out` (whose q/sf/s_dec/amax buffers
 * the caller allocated).  One-time preparation, not part of the layer step.
 * flags: NVFP4MOE_W_GATE_UP to store the fused gate_up rows interleaved.
 * Requirements: K % 256 == 0, N % 256 == 0 (gate_up: N/2 % 128 == 0). */
int nvfp4_prepare_weights(const void *w, int64_t E, int64_t N, int64_t K,
                          uint32_t flags, nvfp4moe_weights *out,
                          nvfp4moe_stream_t stream);

/* ------------------------------------------------------------- combine -- */
/* y[t] = BF16( sum_{j<k} topk_w[t][j] * D[inv_perm[t][j]] ), FP32 sum in slot
 * order j = 0..k-1 (a fixed order: the strict-alignment requirement).
 *   d        [R][H] BF16 expert outputs in compact sorted order
 *   inv_perm [T][k], topk_w [T][k] FP32, y [T][H] BF16 (out)
 * Requirements: H % 8 == 0. */
int moe_combine(const void *d, const int32_t *inv_perm, const float *topk_w,
                int64_t T, int k, int64_t H, void *y, nvfp4moe_stream_t stream);

/* --------------------------------------------------------- the layer ---- */
/* The whole W4A4 MoE expert layer, one stream, no host synchronization:
 *   quantize x once per token + permute (fused)  -> gate_up grouped GEMM with
 *   a fused SwiGLU epilogue that also reduces the amax of h  -> requantize h
 *   reusing that amax  -> down grouped GEMM  -> weighted combine.
 *   x         [T][H] BF16 activations
 *   topk_idx  [T][k] int32, topk_w [T][k] FP32 routing (router output, e.g.
 *             moe_route_topk)
 *   w_gate_up prepared with NVFP4MOE_W_GATE_UP: E x [2I][H]
 *   w_down    prepared plainly: E x [H][I]
 *   y         [T][H] BF16 (out)
 *   flags     NVFP4MOE_SCALE_PER_TOKEN | NVFP4MOE_STRICT
 *   workspace moe_expert_layer_workspace_size() bytes; its named regions
 *             (offsets, perm, h, ...) are laid out by
 *             moe_expert_layer_workspace_offsets() for inspection.
 * Requirements: H % 256 == 0, I % 256 == 0, 1 <= E <= 1024, 1 <= k <= 32. */
size_t moe_expert_layer_workspace_size(int64_t T, int64_t H, int64_t I, int E,
                                       int k, uint32_t flags);

/* Byte offsets of the regions inside the layer workspace, in this order:
 * [0] error word, [1] offsets, [2] padded_offsets, [3] perm, [4] inv_perm,
 * [5] x codes (padded rows), [6] x scales (K-step-major layout), [7] x row S_dec,
 * [8] h BF16 (padded rows), [9] h amax, [10] h codes, [11] h scales (K-step-major),
 * [12] h row S_dec, [13] D BF16 (compact rows), [14] rows_cap (a count, not an
 * offset), [15] total bytes.  `out` must hold 16 int64 (host memory). */
int moe_expert_layer_workspace_offsets(int64_t T, int64_t H, int64_t I, int E,
                                       int k, uint32_t flags, int64_t *out);

int moe_expert_layer(const void *x, const int32_t *topk_idx,
                     const float *topk_w, const nvfp4moe_weights *w_gate_up,
                     const nvfp4moe_weights *w_down, int64_t T, int64_t H,
                     int64_t I, int E, int k, void *y, uint32_t flags,
                     void *workspace, size_t workspace_bytes,
                     nvfp4moe_stream_t stream);

/* moe_expert_layer starting from router logits [T][E] (FP32): the top-k
 * routing (moe_route_topk's rule) runs inside the layer's routing-histogram
 * kernel and its result is written to topk_idx [T][k] and topk_w [T][k]
 * (outputs, also used by the combine).  Everything else is exactly
 * moe_expert_layer with that routing; the workspace is the same size.
 * Requirements: those of moe_expert_layer and k <= E. */
int moe_expert_layer_from_logits(const void *x, const float *logits,
                                 const nvfp4moe_weights *w_gate_up,
                                 const nvfp4moe_weights *w_down, int64_t T,
                                 int64_t H, int64_t I, int E, int k,
                                 int32_t *topk_idx, float *topk_w, void *y,
                                 uint32_t flags, void *workspace,
                                 size_t workspace_bytes,
                                 nvfp4moe_stream_t stream);

/* The dense router in front of the routing: logits = x W_r^T in FP32, with
 * BF16 operands on the tcgen05 tensor cores (kind::f16, FP32 accumulation).
 * The pages list fusion and device-side metadata for the token path
 * (www.aib.vote "miniTE report, NVFP4 RL stability", paragraph 4) and run
 * Qwen3-30B-A3B, whose MoE router is this product; moe_route_permute or
 * moe_expert_layer_from_logits take its output.
 *   x          [T][H] BF16;  w_router [E][H] BF16 (device, 16-byte aligned)
 *   logits     [T][E] FP32 (out)
 *   workspace  moe_router_logits_workspace_size() bytes (device): the error
 *              word at 0 (nvfp4moe_device_status), the GEMM's metadata
 * Requirements: H % 64 == 0, E % 32 == 0, 1 <= E <= 1024, T < 2^30.
 * Errors: NVFP4MOE_ERR_INVALID_ARG / _UNSUPPORTED_SHAPE / _MISALIGNED /
 * _WORKSPACE before any launch; a CUDA error as NVFP4MOE_ERR_CUDA. */
size_t moe_router_logits_workspace_size(void);
int moe_router_logits(const void *x, const void *w_router, int64_t T, int64_t H,
                      int E, float *logits, void *workspace,
                      size_t workspace_bytes, nvfp4moe_stream_t stream);

/* moe_expert_layer that also records CUDA events at its stage boundaries, so
 * a caller can time each kernel on the stream it runs on.  stage_events
 * (host array of 7 cudaEvent_t, entries may be NULL): [0] before the first
 * launch, [1] after routing (counts, amax, offsets), [2] after the fused
 * quantize + permute, [3] after the gate_up GEMM + SwiGLU, [4] after the
 * requantization of h, [5] after the down GEMM, [6] after the combine.
 * Everything else is exactly moe_expert_layer. */
int moe_expert_layer_profiled(const void *x, const int32_t *topk_idx,
                              const float *topk_w,
                              const nvfp4moe_weights *w_gate_up,
                              const nvfp4moe_weights *w_down, int64_t T,
                              int64_t H, int64_t I, int E, int k, void *y,
                              uint32_t flags, void *workspace,
                              size_t workspace_bytes, nvfp4moe_stream_t stream,
                              void *const *stage_events);

/* ------------------------------------------------------------ backward -- */
/* Backward of the MoE expert layer in the BF16-backward mode: the pages time
 * "NVFP4 forward, BF16 backward" at about 1.33-1.37x over BF16 (www.aib.vote
 * "miniTE report, NVFP4 RL stability", paragraph 1) and give no formulas.
 * This computes the exact gradient of the unquantized layer
 *   y[t] = sum_j w[t][j] * W_dn,e (silu(g) * u),  [g | u] = W_gu,e x[t],
 *   e = topk_idx[t][j],
 * on its BF16 operands (the forward's quantizers act as the identity): the
 * routing choice is not differentiated, the routing weights are.  It
 * recomputes [g | u] from x in BF16; all products run on the tensor cores in
 * BF16 with FP32 accumulation (tcgen05 kind::f16), intermediates (G, dG, w*h,
 * dx rows) are stored in BF16 and dx is summed over the k slots in slot order
 * in FP32.
 *   x          [T][H] BF16, topk_idx [T][k] int32, topk_w [T][k] FP32
 *   w_gate_up  [E][2I][H] BF16 (gate rows 0..I-1, up rows I..2I-1: the same
 *              BF16 weights nvfp4_prepare_weights quantizes)
 *   w_down     [E][H][I] BF16
 *   dy         [T][H] BF16, the gradient of the layer output
 *   dx         [T][H] BF16 (out)
 *   d_topk_w   [T][k] FP32 (out): <dy[t], D[t][j]>
 *   dw_gate_up [E][2I][H] weight gradient (out), BF16 and/or FP32 (at least
 *              one non-NULL); dw_down [E][H][I] likewise
 *   flags      NVFP4MOE_BWD_KEEP_DH keeps dh' = dy_rows W_dn (FP32) in the
 *              workspace for inspection
 *   workspace  moe_expert_layer_backward_workspace_size() bytes
 * Requirements: H % 256 == 0, I % 256 == 0, 1 <= E <= 1024, 1 <= k <= 32. */
#define NVFP4MOE_BWD_KEEP_DH 0x40u
size_t moe_expert_layer_backward_workspace_size(int64_t T, int64_t H, int64_t I,
                                                int E, int k, uint32_t flags);
/* Byte offsets of the backward workspace's regions: [0] error word,
 * [1] offsets, [2] padded_offsets, [3] perm, [4] inv_perm, [5] x rows and
 * [6] dy rows (BF16, padded grouped layout, zero padding rows), [7] row
 * weights (FP32), [8] G = x W_gu^T (BF16 [rows_cap][2I]), [9] dG (BF16),
 * [10] w*h (BF16 [rows_cap][I]), [11] <dh', h> partials (FP32
 * [rows_cap][I/128]), [12] dx rows (BF16, compact sorted rows), [13] dh'
 * (FP32 [rows_cap][I], with NVFP4MOE_BWD_KEEP_DH), [14] rows_cap (a count),
 * [15] total bytes.  `out` must hold 16 int64 (host memory). */
int moe_expert_layer_backward_workspace_offsets(int64_t T, int64_t H, int64_t I,
                                                int E, int k, uint32_t flags,
                                                int64_t *out);
int moe_expert_layer_backward(const void *x, const int32_t *topk_idx,
                              const float *topk_w, const void *w_gate_up,
                              const void *w_down, const void *dy, int64_t T,
                              int64_t H, int64_t I, int E, int k, void *dx,
                              float *d_topk_w, void *dw_gate_up_bf16,
                              float *dw_gate_up_f32, void *dw_down_bf16,
                              float *dw_down_f32, uint32_t flags,
                              void *workspace, size_t workspace_bytes,
                              nvfp4moe_stream_t stream);

/* The CUDA error code behind the last NVFP4MOE_ERR_CUDA returned on this host
 * thread (0 if none), with its name, description and the source line of the
 * failing call written to buf (NUL-terminated, at most len bytes; buf may be
 * NULL). */
int nvfp4moe_last_cuda_error(char *buf, size_t len);

/* --------------------------------------------------------------- W4A16 -- */
/* The MoE expert layer with BF16 activations and NVFP4 weights.  The
 * miniTE report on NVFP4 RL stability (www.aib.vote, paragraph 3) measures
 * this variant beside W4A8 and W4A4 and gives no formulas; this reads it as
 * the W4A4 layer without the activation quantizers:
 *   G = x_rows W_gu,e^T,  h = BF16(silu(g) * u),  D = BF16(h W_dn,e^T),
 *   y[t] = BF16(sum_j topk_w[t][j] * D[t][j])  (slot order, FP32),
 * with W the dequantized NVFP4 weights (codes x block scale x S_dec).  The
 * weights stay 4-bit in memory; each K-step of a weight tile is converted to
 * BF16 in shared memory and multiplied on the tensor cores (tcgen05
 * kind::f16, FP32 accumulation); S_dec is applied to the accumulator.
 *   x, topk_idx, topk_w, y, T, H, I, E, k   as for moe_expert_layer
 *   w_gate_up, w_down   prepared exactly as for moe_expert_layer
 *   flags      0 (reserved)
 *   workspace  moe_expert_layer_w4a16_workspace_size() bytes
 * Requirements: those of moe_expert_layer.  Errors: those of
 * moe_expert_layer; the device error word (nvfp4moe_device_status) reports
 * a bounded wait that gave up. */
size_t moe_expert_layer_w4a16_workspace_size(int64_t T, int64_t H, int64_t I,
                                             int E, int k, uint32_t flags);
/* Byte offsets of the W4A16 workspace's regions: [0] error word, [1] offsets,
 * [2] padded_offsets, [3] perm, [4] inv_perm, [5] x rows (BF16, padded
 * grouped layout, zero padding rows), [6] h (BF16 [rows_cap][I]), [7] D
 * (BF16, compact sorted rows), [8] h before its MXFP8 requantization (W4A8
 * with NVFP4MOE_KEEP_H; else 0), [9..13] 0, [14] rows_cap (a count), [15]
 * total bytes.  `out` must hold 16 int64 (host memory). */
int moe_expert_layer_w4a16_workspace_offsets(int64_t T, int64_t H, int64_t I,
                                             int E, int k, uint32_t flags,
                                             int64_t *out);
int moe_expert_layer_w4a16(const void *x, const int32_t *topk_idx,
                           const float *topk_w,
                           const nvfp4moe_weights *w_gate_up,
                           const nvfp4moe_weights *w_down, int64_t T,
                           int64_t H, int64_t I, int E, int k, void *y,
                           uint32_t flags, void *workspace,
                           size_t workspace_bytes, nvfp4moe_stream_t stream);

/* The MoE expert layer with NVFP4 weights and MXFP8 activations (W4A8),
 * the third variant the same paragraph of the aib.vote report compares.  The
 * weights are the W4A4 layer's NVFP4 weights; x (per token) and h (per row)
 * are quantized to MXFP8 -- blocks of 32 along the row, E8M0 scale 2^s with
 * s = floor(log2 amax) - 8, E4M3 elements, round to nearest even, saturating
 * at +-448 (the public OCP MX definition; the pages name the format only) --
 * and dequantized exactly.  The products then run as in
 * moe_expert_layer_w4a16 (BF16 operands, which hold E4M3 x 2^s exactly, on
 * the kind::f16 tensor cores with FP32 accumulation), so the result is the
 * W4A8 layer's up to FP32 summation order.  Dequantized activations below
 * BF16's normal range (2^-126) are rounded to BF16.
 *   arguments  as for moe_expert_layer_w4a16
 *   flags      0, or NVFP4MOE_KEEP_H: also keep the BF16 h before its MXFP8
 *              requantization in workspace region [8] (BF16 [rows_cap][I])
 *   workspace  moe_expert_layer_w4a8_workspace_size() bytes (with the same
 *              flags); regions as for the W4A16 layer, plus [8]. */
size_t moe_expert_layer_w4a8_workspace_size(int64_t T, int64_t H, int64_t I,
                                            int E, int k, uint32_t flags);
int moe_expert_layer_w4a8_workspace_offsets(int64_t T, int64_t H, int64_t I,
                                            int E, int k, uint32_t flags,
                                            int64_t *out);
int moe_expert_layer_w4a8(const void *x, const int32_t *topk_idx,
                          const float *topk_w,
                          const nvfp4moe_weights *w_gate_up,
                          const nvfp4moe_weights *w_down, int64_t T,
                          int64_t H, int64_t I, int E, int k, void *y,
                          uint32_t flags, void *workspace,
                          size_t workspace_bytes, nvfp4moe_stream_t stream);

/* ------------------------------------------------- expert parallelism -- */
/* The expert-parallel layer over G ranks, each owning El = E / G consecutive
 * experts (expert e on rank e / El).  The library provides the steps around
 * the two all-to-all exchanges, which the caller runs (NCCL over NVLink): the
 * forward layer's data movement when its rows cross GPUs, in NVFP4 (3.6x
 * fewer bytes than BF16).  Per-token scaling; results equal those of
 * moe_expert_layer with NVFP4MOE_STRICT, bit for bit, whatever G.
 *   1. source:  moe_ep_dispatch_pack: routing metadata and each token quantized
 *      once into its k rows in compact sorted order (expert, token, slot), so
 *      the rows for rank g are rows [offsets[g El], offsets[(g+1) El]).
 *   2. exchange the [G][El] row counts and the rows (codes, row-major scales,
 *      row S_dec), source-major on the receiver.
 *   3. destination: moe_ep_arrange, moe_ep_experts, moe_ep_return.
 *   4. exchange the D rows back (reverse splits); the source's concatenated
 *      returns are its compact sorted D rows: moe_combine with its inv_perm.
 * All pointers are device pointers, all buffers caller-allocated, all calls
 * stream-ordered; errors as for moe_expert_layer; device-side checks go to
 * each workspace's error word (nvfp4moe_device_status). */
size_t moe_ep_dispatch_workspace_size(int64_t T, int E, int k);
/*   x [T][H] BF16, topk_idx [T][k] (global expert ids)
 *   q_send [T*k][H/2], sf_send [T*k][H/16] (UE4M3, row-major), sdec_send
 *   [T*k] (FP32 per row), offsets [E+1] (compact, device), inv_perm [T][k]:
 *   all written.  H % 256 == 0, 1 <= E <= 1024, 1 <= k <= 32. */
int moe_ep_dispatch_pack(const void *x, const int32_t *topk_idx, int64_t T,
                         int64_t H, int E, int k, uint8_t *q_send,
                         uint8_t *sf_send, float *sdec_send, int32_t *offsets,
                         int32_t *inv_perm, void *workspace,
                         size_t workspace_bytes, nvfp4moe_stream_t stream);
/* Rows of the padded grouped layout needed for rows_recv received rows over
 * El local experts (each group padded to 128 rows). */
int64_t moe_ep_rows_cap(int64_t rows_recv, int El);
size_t moe_ep_arrange_workspace_size(int G, int El);
/*   q_recv, sf_recv, sdec_recv  the received rows, source-major, each
 *                source's rows in its (local expert, token, slot) order
 *   counts       [G][El] int32 (device): rows received from source s for
 *                local expert e
 *   q_a, sf_a, sdec_a  the padded grouped layout (out): q_a [rows_cap][H/2],
 *                sf_a K-step-major [H/256][rows_cap][16], sdec_a [rows_cap];
 *                padding rows are zero
 *   offsets, padded_offsets  [El+1] local groups (out)
 *   workspace    moe_ep_arrange_workspace_size(G, El) bytes; keep it for
 *                moe_ep_return (it holds the (source, expert) tables)
 * Requirements: G * El <= 1024, H % 256 == 0, rows_cap >= moe_ep_rows_cap()
 * and a multiple of 128. */
int moe_ep_arrange(const uint8_t *q_recv, const uint8_t *sf_recv,
                   const float *sdec_recv, const int32_t *counts, int G,
                   int El, int64_t rows_recv, int64_t H, int64_t rows_cap,
                   uint8_t *q_a, uint8_t *sf_a, float *sdec_a,
                   int32_t *offsets, int32_t *padded_offsets, void *workspace,
                   size_t workspace_bytes, nvfp4moe_stream_t stream);
size_t moe_ep_experts_workspace_size(int64_t rows_cap, int64_t H, int64_t I);
/* The local experts on the arranged rows: gate_up + SwiGLU, per-row NVFP4
 * requantization of h, down.  w_gate_up / w_down hold the El local experts
 * (prepared as for moe_expert_layer).  d [rows_recv][H] BF16 (out), compact
 * local order (expert, then source, then the source's order). */
int moe_ep_experts(const uint8_t *q_a, const uint8_t *sf_a,
                   const float *sdec_a, const int32_t *offsets,
                   const int32_t *padded_offsets, int El, int64_t rows_cap,
                   const nvfp4moe_weights *w_gate_up,
                   const nvfp4moe_weights *w_down, int64_t H, int64_t I,
                   void *d, void *workspace, size_t workspace_bytes,
                   nvfp4moe_stream_t stream);
/* d_send [rows_recv][H] BF16 (out): the D rows in received order, ready for
 * the reverse exchange.  workspace: the one moe_ep_arrange filled. */
int moe_ep_return(const void *d, int G, int El, int64_t rows_recv, int64_t H,
                  void *d_send, void *workspace, size_t workspace_bytes,
                  nvfp4moe_stream_t stream);

/* ---------------------------------------------------------- diagnostics -- */
/* The hardware conversions the quantizer uses, exposed so their rounding can
 * be checked against the format definition: codes[i] = E2M1_rne_satfinite(y[i])
 * (one code per byte, 0..15) and codes[i] = UE4M3_rne_satfinite(v[i]). */
int nvfp4moe_encode_e2m1(const float *y, int64_t n, uint8_t *codes,
                         nvfp4moe_stream_t stream);
int nvfp4moe_encode_ue4m3(const float *v, int64_t n, uint8_t *codes,
                          nvfp4moe_stream_t stream);

/* Tensor-core throughput probe: the measured roofline denominator of the
 * grouped GEMM (no counterpart on the pages).  `grid` CTAs (one per SM when
 * grid equals the SM count) each issue `iters` K-steps of 4 block-scaled FP4
 * MMAs (tcgen05.mma kind::mxf4nvf4, M = 128, N = 256, K = 64, 16-element
 * UE4M3 scale blocks) on operands resident in shared memory, the GEMM's
 * instruction and tile shape.  With scale_writes != 0, four warps meanwhile
 * write each K-step's 48 scale columns into TMEM with tcgen05.st, as the
 * GEMM's scale feeders do.  Reads no global memory.  cycles[grid] (device,
 * int64) receives each CTA's elapsed SM cycles; the FLOP count is
 * grid * iters * 4 * 2*128*256*64.  workspace: 16 bytes (error word). */
int nvfp4moe_mma_peak(int iters, int scale_writes, int grid, long long *cycles,
                      void *workspace, nvfp4moe_stream_t stream);

/* Number of SMs of the current device (the persistent grids' size). */
int nvfp4moe_num_sms(void);

#ifdef __cplusplus
}
#endif

#endif /* NVFP4MOE_H */
