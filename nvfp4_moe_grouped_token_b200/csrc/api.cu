// The C-ABI of nvfp4moe: argument checks, workspace layout and the layer's
// launch sequence.  Plain pointers and sizes only; see include/nvfp4moe.h.
#include <cstdio>
#include <cstring>
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace nvfp4moe {

int num_sms() {
  static int cache[64];
  static std::once_flag once;
  std::call_once(once, [] {
    for (int i = 0; i < 64; ++i) cache[i] = 0;
  });
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (cache[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    cache[dev] = n;
  }
  return cache[dev];
}

}  // namespace nvfp4moe

using namespace nvfp4moe;

namespace {

constexpr int64_t kAlign = 256;
constexpr int64_t kHeaderBytes = 256;     // error word, detail, x amax, h amax
constexpr int64_t kHdrXAmax = 16;         // byte offsets inside the header
constexpr int64_t kHdrHAmax = 20;

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
int64_t round_up(int64_t a, int64_t b) { return (a + b - 1) / b * b; }
// The CUDA error behind the last NVFP4MOE_ERR_CUDA of this host thread.
thread_local cudaError_t g_last_cuda_error = cudaSuccess;
thread_local int g_last_cuda_line = 0;

int cuda_fail(cudaError_t e, int line) {
  g_last_cuda_error = e;
  g_last_cuda_line = line;
  return NVFP4MOE_ERR_CUDA;
}

int cuda_rc(cudaError_t e) { return e == cudaSuccess ? NVFP4MOE_OK : cuda_fail(e, 0); }
cudaStream_t st(nvfp4moe_stream_t s) { return reinterpret_cast<cudaStream_t>(s); }

#define NVFP4MOE_TRY(expr)                              \
  do {                                                  \
    cudaError_t e_ = (expr);                            \
    if (e_ != cudaSuccess) return cuda_fail(e_, __LINE__); \
  } while (0)

// Bump allocator over a caller-provided workspace.
struct Carve {
  int64_t off = 0;
  int64_t take(int64_t bytes) {
    const int64_t o = off;
    off += round_up(bytes > 0 ? bytes : 0, kAlign);
    return o;
  }
};

struct PermuteLayout {
  int64_t hdr, counts, local_rank, total;
};

PermuteLayout permute_layout(int64_t T, int k, int E) {
  Carve c;
  PermuteLayout L;
  L.hdr = c.take(kHeaderBytes);
  L.counts = c.take(permute_blocks(T) * E * 4);
  L.local_rank = c.take(T * k * 4);
  L.total = c.off;
  return L;
}

int64_t layer_rows_cap(int64_t T, int k, int E) { return round_up(T * k + 127 * (int64_t)E, 128); }

struct LayerLayout {
  int64_t v[16];
  int64_t counts, local_rank;
  int64_t y_acc;     // FP32 [T][H]: the non-strict combine's accumulator
};

LayerLayout layer_layout(int64_t T, int64_t H, int64_t I, int E, int k) {
  const int64_t R = T * k;
  const int64_t cap = layer_rows_cap(T, k, E);
  Carve c;
  LayerLayout L;
  L.v[0] = c.take(kHeaderBytes);
  L.v[1] = c.take((E + 1) * 4);
  L.v[2] = c.take((E + 1) * 4);
  L.v[3] = c.take(R * 4);
  L.v[4] = c.take(R * 4);
  L.v[5] = c.take(cap * H / 2);
  L.v[6] = c.take(cap * H / 16);
  L.v[7] = c.take(cap * 4);
  L.v[8] = c.take(cap * I * 2);
  L.v[9] = c.take(cap * 4);
  L.v[10] = c.take(cap * I / 2);
  L.v[11] = c.take(cap * I / 16);
  L.v[12] = c.take(cap * 4);
  L.v[13] = c.take(R * H * 2);
  L.counts = c.take(permute_blocks(T) * E * 4);
  L.local_rank = c.take(R * 4);
  L.y_acc = c.take(T * H * 4);
  L.v[14] = cap;
  L.v[15] = c.off;
  return L;
}

struct BwdLayout {
  int64_t v[16];
  int64_t counts, local_rank, ones;
};

// Workspace of the backward: [0] header, [1] offsets, [2] padded offsets,
// [3] perm, [4] inv_perm, [5] x rows, [6] dy rows, [7] row weights, [8] G,
// [9] dG, [10] w*h, [11] <dh', h> partials, [12] dx rows (compact), [13] dh'
// (FP32, only with NVFP4MOE_BWD_KEEP_DH), [14] rows_cap, [15] total bytes.
BwdLayout bwd_layout(int64_t T, int64_t H, int64_t I, int E, int k, uint32_t flags) {
  const int64_t R = T * k;
  const int64_t cap = layer_rows_cap(T, k, E);
  Carve c;
  BwdLayout L;
  L.v[0] = c.take(kHeaderBytes);
  L.v[1] = c.take((E + 1) * 4);
  L.v[2] = c.take((E + 1) * 4);
  L.v[3] = c.take(R * 4);
  L.v[4] = c.take(R * 4);
  L.v[5] = c.take(cap * H * 2);
  L.v[6] = c.take(cap * H * 2);
  L.v[7] = c.take(cap * 4);
  L.v[8] = c.take(cap * 2 * I * 2);
  L.v[9] = c.take(cap * 2 * I * 2);
  L.v[10] = c.take(cap * I * 2);
  L.v[11] = c.take(cap * (I / 128) * 4);
  L.v[12] = c.take(R * H * 2);
  L.v[13] = c.take((flags & NVFP4MOE_BWD_KEEP_DH) ? cap * I * 4 : 0);
  L.counts = c.take(permute_blocks(T) * E * 4);
  L.local_rank = c.take(R * 4);
  L.ones = c.take(R * 4);
  L.v[14] = cap;
  L.v[15] = c.off;
  return L;
}

// Workspace of the W4A16 / W4A8 layer: [0] header, [1] offsets, [2] padded
// offsets, [3] perm, [4] inv_perm, [5] x rows (padded), [6] h (padded), [7] D
// (compact), [8] h before its MXFP8 requantization (W4A8 with KEEP_H),
// [14] rows_cap, [15] total bytes.
BwdLayout w4a16_layout(int64_t T, int64_t H, int64_t I, int E, int k, bool keep_h_pre = false) {
  const int64_t R = T * k;
  const int64_t cap = layer_rows_cap(T, k, E);
  Carve c;
  BwdLayout L;
  for (int i = 0; i < 16; ++i) L.v[i] = 0;
  L.v[0] = c.take(kHeaderBytes);
  L.v[1] = c.take((E + 1) * 4);
  L.v[2] = c.take((E + 1) * 4);
  L.v[3] = c.take(R * 4);
  L.v[4] = c.take(R * 4);
  L.v[5] = c.take(cap * H * 2);
  L.v[6] = c.take(cap * I * 2);
  L.v[7] = c.take(R * H * 2);
  L.v[8] = keep_h_pre ? c.take(cap * I * 2) : 0;
  L.counts = c.take(permute_blocks(T) * E * 4);
  L.local_rank = c.take(R * 4);
  L.ones = 0;
  L.v[14] = cap;
  L.v[15] = c.off;
  return L;
}

bool per_token(uint32_t flags) { return (flags & (NVFP4MOE_SCALE_PER_TOKEN | NVFP4MOE_STRICT)) != 0; }

int check_weights(const nvfp4moe_weights *w, int64_t E, int64_t N, int64_t K) {
  if (w == nullptr || w->q == nullptr || w->sf == nullptr || w->s_dec == nullptr) return NVFP4MOE_ERR_INVALID_ARG;
  if (w->E != E || w->N != N || w->K != K) return NVFP4MOE_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(w->q) || !aligned16(w->sf)) return NVFP4MOE_ERR_MISALIGNED;
  return NVFP4MOE_OK;
}

}  // namespace

extern "C" {

int nvfp4moe_last_cuda_error(char *buf, size_t len) {
  if (buf != nullptr && len > 0) {
    std::snprintf(buf, len, "%s (%s) at api.cu:%d", cudaGetErrorName(g_last_cuda_error),
                  cudaGetErrorString(g_last_cuda_error), g_last_cuda_line);
  }
  return (int)g_last_cuda_error;
}

const char *nvfp4moe_status_string(int status) {
  switch (status) {
    case NVFP4MOE_OK: return "ok";
    case NVFP4MOE_ERR_INVALID_ARG: return "invalid argument";
    case NVFP4MOE_ERR_MISALIGNED: return "pointer not 16-byte aligned";
    case NVFP4MOE_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
    case NVFP4MOE_ERR_CUDA: return "CUDA error";
    case NVFP4MOE_ERR_DEVICE_TIMEOUT: return "device wait timed out";
    case NVFP4MOE_ERR_WORKSPACE: return "workspace missing or too small";
    case NVFP4MOE_ERR_DEVICE_CHECK: return "device-side input check failed";
    default: return "unknown status";
  }
}

int nvfp4moe_version(void) { return 100; }

int nvfp4moe_wait_selftest(void *workspace, nvfp4moe_stream_t stream) {
  if (workspace == nullptr) return NVFP4MOE_ERR_INVALID_ARG;
  if (!aligned16(workspace)) return NVFP4MOE_ERR_MISALIGNED;
  NVFP4MOE_TRY(launch_wait_selftest(static_cast<int *>(workspace), st(stream)));
  return NVFP4MOE_OK;
}

int nvfp4moe_device_status(void *workspace, nvfp4moe_stream_t stream) {
  if (workspace == nullptr) return NVFP4MOE_ERR_INVALID_ARG;
  int words[2] = {0, 0};
  NVFP4MOE_TRY(cudaStreamSynchronize(st(stream)));
  NVFP4MOE_TRY(cudaMemcpy(words, workspace, sizeof(words), cudaMemcpyDeviceToHost));
  NVFP4MOE_TRY(cudaMemset(workspace, 0, sizeof(words)));
  if (words[0] == kDevOk) return NVFP4MOE_OK;
  if (words[0] == kDevTimeout) return NVFP4MOE_ERR_DEVICE_TIMEOUT;
  return NVFP4MOE_ERR_DEVICE_CHECK;
}

int nvfp4_quantize(const void *x, int64_t M, int64_t K, const float *amax_in, float *amax_out,
                   uint8_t *q, uint8_t *scales, float *s_dec, uint32_t flags,
                   nvfp4moe_stream_t stream) {
  if (M < 0 || K <= 0) return NVFP4MOE_ERR_INVALID_ARG;
  if (K % 64 != 0) return NVFP4MOE_ERR_UNSUPPORTED_SHAPE;
  if (M == 0) return NVFP4MOE_OK;
  if (x == nullptr || q == nullptr || scales == nullptr || s_dec == nullptr) return NVFP4MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(q) || !aligned16(scales)) return NVFP4MOE_ERR_MISALIGNED;
  const bool tok = per_token(flags);
  if (!tok && amax_in == nullptr && amax_out == nullptr) return NVFP4MOE_ERR_INVALID_ARG;
  cudaStream_t s = st(stream);
  QuantParams p;
  p.x = x;
  p.tasks = M;
  p.K = K;
  p.mode = kQuantPlain;
  p.q = q;
  p.sf = scales;
  p.sf_layout = (flags & NVFP4MOE_SF_MMA_LAYOUT) ? kSfMma : kSfRowMajor;
  p.s_dec = s_dec;
  p.s_dec_rows = tok ? 1 : 0;
  p.rows_cap = M;
  if (tok) {
    p.amax_rows = 1;
    if (amax_in != nullptr) {
      p.amax_src = amax_in;
      if (amax_out != nullptr && amax_out != amax_in)
        NVFP4MOE_TRY(cudaMemcpyAsync(amax_out, amax_in, M * 4, cudaMemcpyDeviceToDevice, s));
    } else {
      p.compute_row_amax = 1;
      p.amax_out = amax_out;
    }
  } else {
    if (amax_in != nullptr) {
      p.amax_src = amax_in;
      if (amax_out != nullptr && amax_out != amax_in)
        NVFP4MOE_TRY(cudaMemcpyAsync(amax_out, amax_in, 4, cudaMemcpyDeviceToDevice, s));
    } else {
      NVFP4MOE_TRY(cudaMemsetAsync(amax_out, 0, 4, s));
      NVFP4MOE_TRY(launch_amax(x, M * K, 1, amax_out, s));
      p.amax_src = amax_out;
    }
  }
  return cuda_rc(launch_quant(p, s));
}

size_t moe_permute_workspace_size(int64_t T, int k, int E) {
  if (T < 0 || k < 1 || E < 1) return 0;
  return (size_t)permute_layout(T, k, E).total;
}

int moe_permute(const int32_t *topk_idx, int64_t T, int k, int E, int32_t *offsets,
                int32_t *padded_offsets, int32_t *perm, int32_t *inv_perm, void *workspace,
                size_t workspace_bytes, nvfp4moe_stream_t stream) {
  if (T < 0 || k < 1 || k > 32 || E < 1) return NVFP4MOE_ERR_INVALID_ARG;
  if (E > 1024) return NVFP4MOE_ERR_UNSUPPORTED_SHAPE;
  if (offsets == nullptr || padded_offsets == nullptr || (T > 0 && (topk_idx == nullptr || perm == nullptr || inv_perm == nullptr)))
    return NVFP4MOE_ERR_INVALID_ARG;
  const PermuteLayout L = permute_layout(T, k, E);
  if (workspace == nullptr || (int64_t)workspace_bytes < L.total) return NVFP4MOE_ERR_WORKSPACE;
  if (!aligned16(workspace)) return NVFP4MOE_ERR_MISALIGNED;
  cudaStream_t s = st(stream);
  uint8_t *ws = static_cast<uint8_t *>(workspace);
  NVFP4MOE_TRY(cudaMemsetAsync(ws + L.hdr, 0, 16, s));
  PermuteParams p;
  p.topk_idx = topk_idx;
  p.T = T;
  p.k = k;
  p.E = E;
  p.block_counts = reinterpret_cast<int32_t *>(ws + L.counts);
  p.local_rank = reinterpret_cast<int32_t *>(ws + L.local_rank);
  p.offsets = offsets;
  p.padded_offsets = padded_offsets;
  p.perm = perm;
  p.inv_perm = inv_perm;
  p.err = reinterpret_cast<int *>(ws + L.hdr);
  NVFP4MOE_TRY(launch_route_count(p, s));
  NVFP4MOE_TRY(launch_route_scan(p, s));
  NVFP4MOE_TRY(launch_route_rank(p, s));
  return NVFP4MOE_OK;
}

int moe_quantize_permute(const void *x, int64_t T, int64_t K, int k, int E, const int32_t *topk_idx,
                         const int32_t *inv_perm, const int32_t *offsets,
                         const int32_t *padded_offsets, const float *amax_in, float *amax_out,
                         uint8_t *q_rows, uint8_t *sf_rows, float *s_dec_rows, int64_t rows_cap,
                         uint32_t flags, nvfp4moe_stream_t stream) {
  if (T < 0 || K <= 0 || k < 1 || k > 32 || E < 1 || rows_cap < 0) return NVFP4MOE_ERR_INVALID_ARG;
  if (K % 64 != 0) return NVFP4MOE_ERR_UNSUPPORTED_SHAPE;
  if (T == 0) return NVFP4MOE_OK;
  if (x == nullptr || topk_idx == nullptr || inv_perm == nullptr || offsets == nullptr ||
      padded_offsets == nullptr || q_rows == nullptr || sf_rows == nullptr || s_dec_rows == nullptr)
    return NVFP4MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(q_rows) || !aligned16(sf_rows)) return NVFP4MOE_ERR_MISALIGNED;
  const bool tok = per_token(flags);
  if (!tok && amax_in == nullptr && amax_out == nullptr) return NVFP4MOE_ERR_INVALID_ARG;
  cudaStream_t s = st(stream);
  QuantParams p;
  p.x = x;
  p.tasks = T;
  p.K = K;
  p.mode = kQuantScatter;
  p.q = q_rows;
  p.sf = sf_rows;
  p.sf_layout = kSfKStep;
  p.s_dec = s_dec_rows;
  p.s_dec_rows = 1;
  p.rows_cap = rows_cap;
  p.topk_idx = topk_idx;
  p.inv_perm = inv_perm;
  p.offsets = offsets;
  p.padded_offsets = padded_offsets;
  p.k = k;
  p.E = E;
  if (tok) {
    p.amax_rows = 1;
    if (amax_in != nullptr) {
      p.amax_src = amax_in;
    } else {
      p.compute_row_amax = 1;
      p.amax_out = amax_out;
    }
  } else {
    if (amax_in != nullptr) {
      p.amax_src = amax_in;
    } else {
      NVFP4MOE_TRY(cudaMemsetAsync(amax_out, 0, 4, s));
      NVFP4MOE_TRY(launch_amax(x, T * K, 1, amax_out, s));
      p.amax_src = amax_out;
    }
  }
  return cuda_rc(launch_quant(p, s));
}

int nvfp4_grouped_gemm(const uint8_t *q_a, const uint8_t *sf_a, const float *s_dec_a,
                       const uint8_t *q_w, const uint8_t *sf_w, const float *s_dec_w,
                       const int32_t *offsets, const int32_t *padded_offsets, int E, int64_t rows_cap,
                       int64_t N, int64_t K, void *out_bf16, float *out_f32, uint32_t flags,
                       void *workspace, size_t workspace_bytes, nvfp4moe_stream_t stream) {
  if (E < 1 || rows_cap < 0 || N <= 0 || K <= 0) return NVFP4MOE_ERR_INVALID_ARG;
  if (K % 256 != 0 || N % 256 != 0 || rows_cap % 128 != 0 || E > 1024)
    return NVFP4MOE_ERR_UNSUPPORTED_SHAPE;
  if (q_a == nullptr || sf_a == nullptr || s_dec_a == nullptr || q_w == nullptr || sf_w == nullptr ||
      s_dec_w == nullptr || offsets == nullptr || padded_offsets == nullptr ||
      (out_bf16 == nullptr && out_f32 == nullptr))
    return NVFP4MOE_ERR_INVALID_ARG;
  if (!aligned16(q_a) || !aligned16(sf_a) || !aligned16(q_w) || !aligned16(sf_w) ||
      !aligned16(out_bf16) || !aligned16(out_f32))
    return NVFP4MOE_ERR_MISALIGNED;
  if (workspace == nullptr || workspace_bytes < 16) return NVFP4MOE_ERR_WORKSPACE;
  if (rows_cap == 0) return NVFP4MOE_OK;
  cudaStream_t s = st(stream);
  NVFP4MOE_TRY(cudaMemsetAsync(workspace, 0, 16, s));
  GemmArgs a;
  std::memset(&a, 0, sizeof(a));
  a.q_a = q_a;
  a.sf_a = sf_a;
  a.s_dec_a = s_dec_a;
  a.s_dec_a_rows = per_token(flags) ? 1 : 0;
  a.q_w = q_w;
  a.sf_w = sf_w;
  a.s_dec_w = s_dec_w;
  a.offsets = offsets;
  a.padded_offsets = padded_offsets;
  a.E = E;
  a.rows_cap = rows_cap;
  a.N = N;
  a.K = K;
  a.epilogue = kEpiStore;
  a.out_bf16 = out_bf16;
  a.out_f32 = out_f32;
  a.out_padded = (flags & NVFP4MOE_OUT_PADDED) ? 1 : 0;
  a.err = static_cast<int *>(workspace);
  return cuda_rc(launch_grouped_gemm(a, s));
}

int nvfp4_prepare_weights(const void *w, int64_t E, int64_t N, int64_t K, uint32_t flags,
                          nvfp4moe_weights *out, nvfp4moe_stream_t stream) {
  if (w == nullptr || out == nullptr || E < 1 || N <= 0 || K <= 0) return NVFP4MOE_ERR_INVALID_ARG;
  if (out->q == nullptr || out->sf == nullptr || out->s_dec == nullptr || out->amax == nullptr)
    return NVFP4MOE_ERR_INVALID_ARG;
  if (K % 256 != 0 || N % 256 != 0) return NVFP4MOE_ERR_UNSUPPORTED_SHAPE;
  const bool gate_up = (flags & NVFP4MOE_W_GATE_UP) != 0;
  if (gate_up && (N / 2) % 128 != 0) return NVFP4MOE_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(w) || !aligned16(out->q) || !aligned16(out->sf)) return NVFP4MOE_ERR_MISALIGNED;
  cudaStream_t s = st(stream);
  NVFP4MOE_TRY(cudaMemsetAsync(out->amax, 0, E * 4, s));
  NVFP4MOE_TRY(launch_amax(w, N * K, E, out->amax, s));
  QuantParams p;
  p.x = w;
  p.tasks = E * N;
  p.K = K;
  p.mode = kQuantWeights;
  p.amax_src = out->amax;
  p.amax_rows = 1;
  p.q = out->q;
  p.sf = out->sf;
  p.sf_layout = kSfMma;
  p.s_dec = out->s_dec;
  p.s_dec_rows = 0;
  p.rows_cap = E * N;
  p.N = N;
  p.gate_up = gate_up ? 1 : 0;
  NVFP4MOE_TRY(launch_quant(p, s));
  out->E = E;
  out->N = N;
  out->K = K;
  out->flags = gate_up ? NVFP4MOE_W_GATE_UP : 0u;
  return NVFP4MOE_OK;
}

int moe_combine(const void *d, const int32_t *inv_perm, const float *topk_w, int64_t T, int k,
                int64_t H, void *y, nvfp4moe_stream_t stream) {
  if (T < 0 || k < 1 || k > 32 || H <= 0) return NVFP4MOE_ERR_INVALID_ARG;
  if (H % 8 != 0) return NVFP4MOE_ERR_UNSUPPORTED_SHAPE;
  if (T == 0) return NVFP4MOE_OK;
  if (d == nullptr || inv_perm == nullptr || topk_w == nullptr || y == nullptr) return NVFP4MOE_ERR_INVALID_ARG;
  if (!aligned16(d) || !aligned16(y)) return NVFP4MOE_ERR_MISALIGNED;
  return cuda_rc(launch_combine(d, inv_perm, topk_w, T, k, H, y, st(stream)));
}

size_t moe_expert_layer_workspace_size(int64_t T, int64_t H, int64_t I, int E, int k, uint32_t flags) {
  (void)flags;
  if (T < 0 || H <= 0 || I <= 0 || E < 1 || k < 1) return 0;
  return (size_t)layer_layout(T, H, I, E, k).v[15];
}

int moe_expert_layer_workspace_offsets(int64_t T, int64_t H, int64_t I, int E, int k, uint32_t flags,
                                       int64_t *out) {
  (void)flags;
  if (out == nullptr || T < 0 || H <= 0 || I <= 0 || E < 1 || k < 1) return NVFP4MOE_ERR_INVALID_ARG;
  const LayerLayout L = layer_layout(T, H, I, E, k);
  for (int i = 0; i < 16; ++i) out[i] = L.v[i];
  return NVFP4MOE_OK;
}

// logits == nullptr: topk_idx / topk_w are the given routing.  Otherwise the
// top-k of the router logits [T][E] is taken inside the routing-histogram
// kernel and written to topk_idx / topk_w (outputs).
static int expert_layer_impl(const void *x, const int32_t *topk_idx, const float *topk_w,
                             const nvfp4moe_weights *w_gate_up, const nvfp4moe_weights *w_down,
                             int64_t T, int64_t H, int64_t I, int E, int k, void *y, uint32_t flags,
                             void *workspace, size_t workspace_bytes, nvfp4moe_stream_t stream,
                             void *const *events, const float *logits = nullptr) {
  if (T < 0 || H <= 0 || I <= 0 || k < 1 || k > 32 || E < 1) return NVFP4MOE_ERR_INVALID_ARG;
  if (E > 1024 || H % 256 != 0 || I % 256 != 0) return NVFP4MOE_ERR_UNSUPPORTED_SHAPE;
  int rc = check_weights(w_gate_up, E, 2 * I, H);
  if (rc != NVFP4MOE_OK) return rc;
  if (!(w_gate_up->flags & NVFP4MOE_W_GATE_UP)) return NVFP4MOE_ERR_INVALID_ARG;
  rc = check_weights(w_down, E, H, I);
  if (rc != NVFP4MOE_OK) return rc;
  if (T == 0) return NVFP4MOE_OK;
  if (x == nullptr || topk_idx == nullptr || topk_w == nullptr || y == nullptr) return NVFP4MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(y) || !aligned16(workspace)) return NVFP4MOE_ERR_MISALIGNED;
  const LayerLayout L = layer_layout(T, H, I, E, k);
  if (workspace == nullptr || (int64_t)workspace_bytes < L.v[15]) return NVFP4MOE_ERR_WORKSPACE;
  const bool tok = per_token(flags);
  const bool fast_combine = (flags & NVFP4MOE_FAST_COMBINE) != 0;
  if (fast_combine && (flags & NVFP4MOE_STRICT)) return NVFP4MOE_ERR_INVALID_ARG;
  if (fast_combine && H % 8 != 0) return NVFP4MOE_ERR_UNSUPPORTED_SHAPE;
  const int64_t cap = L.v[14];
  cudaStream_t s = st(stream);
  uint8_t *ws = static_cast<uint8_t *>(workspace);
  int *err = reinterpret_cast<int *>(ws + L.v[0]);
  float *y_acc = reinterpret_cast<float *>(ws + L.y_acc);
  float *x_amax = reinterpret_cast<float *>(ws + L.v[0] + kHdrXAmax);
  float *h_amax_tensor = reinterpret_cast<float *>(ws + L.v[0] + kHdrHAmax);
  int32_t *offsets = reinterpret_cast<int32_t *>(ws + L.v[1]);
  int32_t *padded = reinterpret_cast<int32_t *>(ws + L.v[2]);
  int32_t *perm = reinterpret_cast<int32_t *>(ws + L.v[3]);
  int32_t *inv_perm = reinterpret_cast<int32_t *>(ws + L.v[4]);
  uint8_t *xq = ws + L.v[5];
  uint8_t *xsf = ws + L.v[6];
  float *xsd = reinterpret_cast<float *>(ws + L.v[7]);
  void *hb = ws + L.v[8];
  float *h_amax_rows = reinterpret_cast<float *>(ws + L.v[9]);
  uint8_t *hq = ws + L.v[10];
  uint8_t *hsf = ws + L.v[11];
  float *hsd = reinterpret_cast<float *>(ws + L.v[12]);
  void *d = ws + L.v[13];

  auto mark = [&](int i) -> cudaError_t {
    if (events == nullptr || events[i] == nullptr) return cudaSuccess;
    return cudaEventRecord(reinterpret_cast<cudaEvent_t>(events[i]), s);
  };
  NVFP4MOE_TRY(mark(0));
  NVFP4MOE_TRY(cudaMemsetAsync(ws + L.v[0], 0, kHeaderBytes, s));

  // 1-2. route counts, (per-tensor) amax of x, offsets
  PermuteParams pp;
  pp.topk_idx = topk_idx;
  pp.T = T;
  pp.k = k;
  pp.E = E;
  pp.block_counts = reinterpret_cast<int32_t *>(ws + L.counts);
  pp.local_rank = reinterpret_cast<int32_t *>(ws + L.local_rank);
  pp.offsets = offsets;
  pp.padded_offsets = padded;
  pp.perm = perm;
  pp.inv_perm = inv_perm;
  pp.err = err;
  // padding rows of h start with amax 0 (the requantizer skips them)
  pp.zero_pad_rows = tok ? h_amax_rows : nullptr;
  pp.rows_cap = cap;
  if (logits != nullptr) {
    if (k > E) return NVFP4MOE_ERR_UNSUPPORTED_SHAPE;
    pp.logits = logits;
    pp.topk_idx_out = const_cast<int32_t *>(topk_idx);
    pp.topk_w_out = const_cast<float *>(topk_w);
  }
  NVFP4MOE_TRY(launch_route_count(pp, s));
  if (!tok) NVFP4MOE_TRY(launch_amax(x, T * H, 1, x_amax, s));
  NVFP4MOE_TRY(launch_route_scan(pp, s));
  NVFP4MOE_TRY(mark(1));

  // 3. quantize each token once, scatter to its k rows, write perm / inv_perm
  QuantParams q;
  q.x = x;
  q.tasks = T;
  q.K = H;
  q.mode = kQuantScatter;
  q.q = xq;
  q.sf = xsf;
  q.sf_layout = kSfKStep;
  q.s_dec = xsd;
  q.s_dec_rows = 1;
  q.rows_cap = cap;
  q.topk_idx = topk_idx;
  q.offsets = offsets;
  q.padded_offsets = padded;
  q.k = k;
  q.E = E;
  q.local_rank = pp.local_rank;
  q.block_base = pp.block_counts;
  q.perm_out = perm;
  q.inv_perm_out = inv_perm;
  q.zero_rows = tok ? h_amax_rows : nullptr;
  if (tok) {
    q.amax_rows = 1;
    q.compute_row_amax = 1;
  } else {
    q.amax_src = x_amax;
  }
  NVFP4MOE_TRY(launch_quant(q, s));
  NVFP4MOE_TRY(mark(2));

  // 4. gate_up grouped GEMM + SwiGLU epilogue (h in BF16, amax of h)
  GemmArgs g;
  std::memset(&g, 0, sizeof(g));
  g.q_a = xq;
  g.sf_a = xsf;
  g.s_dec_a = xsd;
  g.s_dec_a_rows = 1;
  g.q_w = w_gate_up->q;
  g.sf_w = w_gate_up->sf;
  g.s_dec_w = w_gate_up->s_dec;
  g.offsets = offsets;
  g.padded_offsets = padded;
  g.E = E;
  g.rows_cap = cap;
  g.N = 2 * I;
  g.K = H;
  g.epilogue = kEpiSwiGLU;
  g.out_bf16 = hb;
  g.out_padded = 1;
  g.amax_h = tok ? h_amax_rows : h_amax_tensor;
  g.amax_h_rows = tok ? 1 : 0;
  g.err = err;
  const bool fused_requant = tok && (flags & NVFP4MOE_FUSED_REQUANT);
  if (fused_requant) {
    // 5 (fused). per-row scales: each m-tile of h is requantized inside the
    // GEMM launch as soon as all its columns and its row amax are final
    g.req_q = hq;
    g.req_sf = hsf;
    g.req_s_dec = hsd;
    g.discard_h = (flags & NVFP4MOE_KEEP_H) ? 0 : 1;
  }
  NVFP4MOE_TRY(launch_grouped_gemm(g, s));
  NVFP4MOE_TRY(mark(3));

  // 5. requantize h with the amax the epilogue reduced (amax reuse): a
  // separate pass unless it ran inside the GEMM (a per-tensor amax spans
  // every row, so it always needs the separate pass)
  if (!fused_requant) {
  QuantParams rq;
  rq.x = hb;
  rq.tasks = T * k;
  rq.K = I;
  rq.mode = kQuantRequant;
  rq.amax_src = tok ? h_amax_rows : h_amax_tensor;
  rq.amax_rows = tok ? 1 : 0;
  rq.q = hq;
  rq.sf = hsf;
  rq.sf_layout = kSfKStep;
  rq.s_dec = hsd;
  rq.s_dec_rows = 1;
  rq.rows_cap = cap;
  rq.offsets = offsets;
  rq.padded_offsets = padded;
  rq.E = E;
  NVFP4MOE_TRY(launch_quant(rq, s));
  }
  NVFP4MOE_TRY(mark(4));

  // 6. down grouped GEMM -> D (BF16, compact sorted rows)
  GemmArgs dn;
  std::memset(&dn, 0, sizeof(dn));
  dn.q_a = hq;
  dn.sf_a = hsf;
  dn.s_dec_a = hsd;
  dn.s_dec_a_rows = 1;
  dn.q_w = w_down->q;
  dn.sf_w = w_down->sf;
  dn.s_dec_w = w_down->s_dec;
  dn.offsets = offsets;
  dn.padded_offsets = padded;
  dn.E = E;
  dn.rows_cap = cap;
  dn.N = H;
  dn.K = I;
  dn.epilogue = kEpiStore;
  dn.out_bf16 = d;
  dn.out_padded = 0;
  dn.err = err;
  if (fast_combine) {
    // non-strict: the epilogue adds w * D_row into y_acc[t] (FP32 reductions)
    NVFP4MOE_TRY(cudaMemsetAsync(y_acc, 0, T * H * 4, s));
    dn.out_bf16 = nullptr;
    dn.red_y = y_acc;
    dn.red_perm = perm;
    dn.red_w = topk_w;
    dn.red_k = k;
  }
  NVFP4MOE_TRY(launch_grouped_gemm(dn, s));
  NVFP4MOE_TRY(mark(5));

  // 7. weighted combine in slot order (strict), or y = BF16(y_acc)
  if (fast_combine) NVFP4MOE_TRY(launch_f32_to_bf16(y_acc, T * H, y, s));
  else NVFP4MOE_TRY(launch_combine(d, inv_perm, topk_w, T, k, H, y, s));
  NVFP4MOE_TRY(mark(6));
  return NVFP4MOE_OK;
}

int moe_expert_layer(const void *x, const int32_t *topk_idx, const float *topk_w,
                     const nvfp4moe_weights *w_gate_up, const nvfp4moe_weights *w_down, int64_t T,
                     int64_t H, int64_t I, int E, int k, void *y, uint32_t flags, void *workspace,
                     size_t workspace_bytes, nvfp4moe_stream_t stream) {
  return expert_layer_impl(x, topk_idx, topk_w, w_gate_up, w_down, T, H, I, E, k, y, flags, workspace,
                           workspace_bytes, stream, nullptr);
}

int moe_expert_layer_profiled(const void *x, const int32_t *topk_idx, const float *topk_w,
                              const nvfp4moe_weights *w_gate_up, const nvfp4moe_weights *w_down,
                              int64_t T, int64_t H, int64_t I, int E, int k, void *y, uint32_t flags,
                              void *workspace, size_t workspace_bytes, nvfp4moe_stream_t stream,
                              void *const *stage_events) {
  return expert_layer_impl(x, topk_idx, topk_w, w_gate_up, w_down, T, H, I, E, k, y, flags, workspace,
                           workspace_bytes, stream, stage_events);
}

size_t moe_expert_layer_backward_workspace_size(int64_t T, int64_t H, int64_t I, int E, int k, uint32_t flags) {
  if (T < 0 || H <= 0 || I <= 0 || E < 1 || k < 1) return 0;
  return (size_t)bwd_layout(T, H, I, E, k, flags).v[15];
}

int moe_expert_layer_backward_workspace_offsets(int64_t T, int64_t H, int64_t I, int E, int k, uint32_t flags,
                                                int64_t *out) {
  if (out == nullptr || T < 0 || H <= 0 || I <= 0 || E < 1 || k < 1) return NVFP4MOE_ERR_INVALID_ARG;
  const BwdLayout L = bwd_layout(T, H, I, E, k, flags);
  for (int i = 0; i < 16; ++i) out[i] = L.v[i];
  return NVFP4MOE_OK;
}

int moe_expert_layer_backward(const void *x, const int32_t *topk_idx, const float *topk_w, const void *w_gate_up,
                              const void *w_down, const void *dy, int64_t T, int64_t H, int64_t I, int E, int k,
                              void *dx, float *d_topk_w, void *dw_gate_up_bf16, float *dw_gate_up_f32,
                              void *dw_down_bf16, float *dw_down_f32, uint32_t flags, void *workspace,
                              size_t workspace_bytes, nvfp4moe_stream_t stream) {
  if (T < 0 || H <= 0 || I <= 0 || k < 1 || k > 32 || E < 1) return NVFP4MOE_ERR_INVALID_ARG;
  if (E > 1024 || H % 256 != 0 || I % 256 != 0) return NVFP4MOE_ERR_UNSUPPORTED_SHAPE;
  if (T == 0) return NVFP4MOE_OK;
  if (x == nullptr || topk_idx == nullptr || topk_w == nullptr || w_gate_up == nullptr || w_down == nullptr ||
      dy == nullptr || dx == nullptr || d_topk_w == nullptr ||
      (dw_gate_up_bf16 == nullptr && dw_gate_up_f32 == nullptr) || (dw_down_bf16 == nullptr && dw_down_f32 == nullptr))
    return NVFP4MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(w_gate_up) || !aligned16(w_down) || !aligned16(dy) || !aligned16(dx) ||
      !aligned16(dw_gate_up_bf16) || !aligned16(dw_gate_up_f32) || !aligned16(dw_down_bf16) ||
      !aligned16(dw_down_f32) || !aligned16(workspace))
    return NVFP4MOE_ERR_MISALIGNED;
  const BwdLayout L = bwd_layout(T, H, I, E, k, flags);
  if (workspace == nullptr || (int64_t)workspace_bytes < L.v[15]) return NVFP4MOE_ERR_WORKSPACE;
  const int64_t cap = L.v[14];
  cudaStream_t s = st(stream);
  uint8_t *ws = static_cast<uint8_t *>(workspace);
  int *err = reinterpret_cast<int *>(ws + L.v[0]);
  int32_t *offsets = reinterpret_cast<int32_t *>(ws + L.v[1]);
  int32_t *padded = reinterpret_cast<int32_t *>(ws + L.v[2]);
  int32_t *perm = reinterpret_cast<int32_t *>(ws + L.v[3]);
  int32_t *inv_perm = reinterpret_cast<int32_t *>(ws + L.v[4]);
  void *x_rows = ws + L.v[5];
  void *dy_rows = ws + L.v[6];
  float *w_rows = reinterpret_cast<float *>(ws + L.v[7]);
  void *g = ws + L.v[8];
  void *dg = ws + L.v[9];
  void *hw = ws + L.v[10];
  float *dw_part = reinterpret_cast<float *>(ws + L.v[11]);
  void *dx_rows = ws + L.v[12];
  float *dh_keep = (flags & NVFP4MOE_BWD_KEEP_DH) ? reinterpret_cast<float *>(ws + L.v[13]) : nullptr;
  float *ones = reinterpret_cast<float *>(ws + L.ones);
  NVFP4MOE_TRY(cudaMemsetAsync(ws + L.v[0], 0, kHeaderBytes, s));

  // routing metadata: offsets, padded offsets, perm, inv_perm
  PermuteParams pp;
  pp.topk_idx = topk_idx;
  pp.T = T;
  pp.k = k;
  pp.E = E;
  pp.block_counts = reinterpret_cast<int32_t *>(ws + L.counts);
  pp.local_rank = reinterpret_cast<int32_t *>(ws + L.local_rank);
  pp.offsets = offsets;
  pp.padded_offsets = padded;
  pp.perm = perm;
  pp.inv_perm = inv_perm;
  pp.err = err;
  NVFP4MOE_TRY(launch_route_count(pp, s));
  NVFP4MOE_TRY(launch_route_scan(pp, s));
  NVFP4MOE_TRY(launch_route_rank(pp, s));

  // rows of x and dy in the padded grouped layout, row weights, ones
  BwdGatherParams gp{};
  gp.x = x;
  gp.dy = dy;
  gp.topk_w = topk_w;
  gp.topk_idx = topk_idx;
  gp.perm = perm;
  gp.inv_perm = inv_perm;
  gp.offsets = offsets;
  gp.padded_offsets = padded;
  gp.T = T;
  gp.H = H;
  gp.rows_cap = cap;
  gp.k = k;
  gp.E = E;
  gp.x_rows = x_rows;
  gp.dy_rows = dy_rows;
  gp.w_rows = w_rows;
  gp.ones = ones;
  NVFP4MOE_TRY(launch_bwd_gather(gp, s));

  Bf16GemmArgs base;
  base.offsets = offsets;
  base.padded_offsets = padded;
  base.E = E;
  base.rows_cap = cap;
  base.err = err;
  // G = x_rows W_gu^T (the forward's gate_up product, recomputed in BF16)
  Bf16GemmArgs g1 = base;
  g1.mode = kBfRows;
  g1.a = x_rows;
  g1.b = w_gate_up;
  g1.b_mn = 0;
  g1.N = 2 * I;
  g1.K = H;
  g1.out_bf16 = g;
  g1.out_padded = 1;
  NVFP4MOE_TRY(launch_bf16_gemm(g1, s));
  // dh' = dy_rows W_dn; epilogue: SwiGLU backward -> dG, w*h, <dh', h> partials
  Bf16GemmArgs g2 = base;
  g2.mode = kBfRows;
  g2.a = dy_rows;
  g2.b = w_down;
  g2.b_mn = 1;
  g2.N = I;
  g2.K = H;
  g2.epilogue = kBfSwiGLUBwd;
  g2.g_u = g;
  g2.w_rows = w_rows;
  g2.d_gu = dg;
  g2.hw = hw;
  g2.dw_part = dw_part;
  g2.out_f32 = dh_keep;
  NVFP4MOE_TRY(launch_bf16_gemm(g2, s));
  // dx rows = dG W_gu (compact sorted rows), then dx[t] = sum_j dx_rows[inv_perm[t][j]]
  Bf16GemmArgs g3 = base;
  g3.mode = kBfRows;
  g3.a = dg;
  g3.b = w_gate_up;
  g3.b_mn = 1;
  g3.N = H;
  g3.K = 2 * I;
  g3.out_bf16 = dx_rows;
  g3.out_padded = 0;
  NVFP4MOE_TRY(launch_bf16_gemm(g3, s));
  NVFP4MOE_TRY(launch_combine(dx_rows, inv_perm, ones, T, k, H, dx, s));
  // d topk_w[t][j] = <dy[t], D[t][j]> = sum of the row's partials
  NVFP4MOE_TRY(launch_bwd_dw(dw_part, I / 128, inv_perm, topk_idx, offsets, padded, T, k, E, d_topk_w, s));
  // dW_dn,e = sum over the group's rows of dy_r^T (w h)_r
  Bf16GemmArgs g4 = base;
  g4.mode = kBfWgrad;
  g4.a = dy_rows;
  g4.b = hw;
  g4.M = H;
  g4.N = I;
  g4.out_bf16 = dw_down_bf16;
  g4.out_f32 = dw_down_f32;
  NVFP4MOE_TRY(launch_bf16_gemm(g4, s));
  // dW_gu,e = sum over the group's rows of dG_r^T x_r
  Bf16GemmArgs g5 = base;
  g5.mode = kBfWgrad;
  g5.a = dg;
  g5.b = x_rows;
  g5.M = 2 * I;
  g5.N = H;
  g5.out_bf16 = dw_gate_up_bf16;
  g5.out_f32 = dw_gate_up_f32;
  NVFP4MOE_TRY(launch_bf16_gemm(g5, s));
  return NVFP4MOE_OK;
}

int moe_route_permute(const float *logits, int64_t T, int E, int k, int32_t *topk_idx, float *topk_w,
                      int32_t *offsets, int32_t *padded_offsets, int32_t *perm, int32_t *inv_perm, void *workspace,
                      size_t workspace_bytes, nvfp4moe_stream_t stream) {
  if (T < 0 || k < 1 || E < 1) return NVFP4MOE_ERR_INVALID_ARG;
  if (E > 1024 || k > 32 || k > E) return NVFP4MOE_ERR_UNSUPPORTED_SHAPE;
  if (offsets == nullptr || padded_offsets == nullptr ||
      (T > 0 && (logits == nullptr || topk_idx == nullptr || topk_w == nullptr || perm == nullptr ||
                 inv_perm == nullptr)))
    return NVFP4MOE_ERR_INVALID_ARG;
  const PermuteLayout L = permute_layout(T, k, E);
  if (workspace == nullptr || (int64_t)workspace_bytes < L.total) return NVFP4MOE_ERR_WORKSPACE;
  if (!aligned16(workspace)) return NVFP4MOE_ERR_MISALIGNED;
  cudaStream_t s = st(stream);
  uint8_t *ws = static_cast<uint8_t *>(workspace);
  NVFP4MOE_TRY(cudaMemsetAsync(ws + L.hdr, 0, 16, s));
  PermuteParams p;
  p.topk_idx = topk_idx;
  p.T = T;
  p.k = k;
  p.E = E;
  p.block_counts = reinterpret_cast<int32_t *>(ws + L.counts);
  p.local_rank = reinterpret_cast<int32_t *>(ws + L.local_rank);
  p.offsets = offsets;
  p.padded_offsets = padded_offsets;
  p.perm = perm;
  p.inv_perm = inv_perm;
  p.err = reinterpret_cast<int *>(ws + L.hdr);
  p.logits = logits;
  p.topk_idx_out = topk_idx;
  p.topk_w_out = topk_w;
  NVFP4MOE_TRY(launch_route_count(p, s));
  NVFP4MOE_TRY(launch_route_scan(p, s));
  NVFP4MOE_TRY(launch_route_rank(p, s));
  return NVFP4MOE_OK;
}

int moe_expert_layer_from_logits(const void *x, const float *logits, const nvfp4moe_weights *w_gate_up,
                                 const nvfp4moe_weights *w_down, int64_t T, int64_t H, int64_t I, int E, int k,
                                 int32_t *topk_idx, float *topk_w, void *y, uint32_t flags, void *workspace,
                                 size_t workspace_bytes, nvfp4moe_stream_t stream) {
  if (T > 0 && logits == nullptr) return NVFP4MOE_ERR_INVALID_ARG;
  return expert_layer_impl(x, topk_idx, topk_w, w_gate_up, w_down, T, H, I, E, k, y, flags, workspace,
                           workspace_bytes, stream, nullptr, logits);
}

int nvfp4moe_mma_peak(int iters, int scale_writes, int grid, long long *cycles, void *workspace,
                      nvfp4moe_stream_t stream) {
  if (iters < 1 || grid < 1 || cycles == nullptr || workspace == nullptr) return NVFP4MOE_ERR_INVALID_ARG;
  if (!aligned16(workspace)) return NVFP4MOE_ERR_MISALIGNED;
  cudaStream_t s = st(stream);
  NVFP4MOE_TRY(cudaMemsetAsync(workspace, 0, 16, s));
  return cuda_rc(launch_mma_peak(iters, scale_writes ? 1 : 0, cycles, static_cast<int *>(workspace), grid, s));
}

int nvfp4moe_num_sms(void) { return num_sms(); }

int nvfp4moe_encode_e2m1(const float *y, int64_t n, uint8_t *codes, nvfp4moe_stream_t stream) {
  if (n < 0 || (n > 0 && (y == nullptr || codes == nullptr))) return NVFP4MOE_ERR_INVALID_ARG;
  return cuda_rc(launch_encode_e2m1(y, n, codes, st(stream)));
}

int nvfp4moe_encode_ue4m3(const float *v, int64_t n, uint8_t *codes, nvfp4moe_stream_t stream) {
  if (n < 0 || (n > 0 && (v == nullptr || codes == nullptr))) return NVFP4MOE_ERR_INVALID_ARG;
  return cuda_rc(launch_encode_ue4m3(v, n, codes, st(stream)));
}


// ---------------------------------------------------------- W4A16 / W4A8 --

}  // extern "C"

namespace {

// The W4A16 layer, or with mxfp8 the W4A8 layer (x and h MXFP8
// quantize-dequantized in the gather and in the gate_up epilogue).
int w4ax_layer(const void *x, const int32_t *topk_idx, const float *topk_w, const nvfp4moe_weights *w_gate_up,
               const nvfp4moe_weights *w_down, int64_t T, int64_t H, int64_t I, int E, int k, void *y, uint32_t flags,
               void *workspace, size_t workspace_bytes, nvfp4moe_stream_t stream, bool mxfp8) {
  const uint32_t allowed = mxfp8 ? NVFP4MOE_KEEP_H : 0u;
  if (T < 0 || H <= 0 || I <= 0 || k < 1 || k > 32 || E < 1 || (flags & ~allowed) != 0)
    return NVFP4MOE_ERR_INVALID_ARG;
  if (E > 1024 || H % 256 != 0 || I % 256 != 0) return NVFP4MOE_ERR_UNSUPPORTED_SHAPE;
  int rc = check_weights(w_gate_up, E, 2 * I, H);
  if (rc != NVFP4MOE_OK) return rc;
  if (!(w_gate_up->flags & NVFP4MOE_W_GATE_UP)) return NVFP4MOE_ERR_INVALID_ARG;
  rc = check_weights(w_down, E, H, I);
  if (rc != NVFP4MOE_OK) return rc;
  if (T == 0) return NVFP4MOE_OK;
  if (x == nullptr || topk_idx == nullptr || topk_w == nullptr || y == nullptr) return NVFP4MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(y) || !aligned16(workspace)) return NVFP4MOE_ERR_MISALIGNED;
  const bool keep_h_pre = (flags & NVFP4MOE_KEEP_H) != 0;
  const BwdLayout L = w4a16_layout(T, H, I, E, k, keep_h_pre);
  if (workspace == nullptr || (int64_t)workspace_bytes < L.v[15]) return NVFP4MOE_ERR_WORKSPACE;
  const int64_t cap = L.v[14];
  cudaStream_t s = st(stream);
  uint8_t *ws = static_cast<uint8_t *>(workspace);
  int *err = reinterpret_cast<int *>(ws + L.v[0]);
  int32_t *offsets = reinterpret_cast<int32_t *>(ws + L.v[1]);
  int32_t *padded = reinterpret_cast<int32_t *>(ws + L.v[2]);
  int32_t *perm = reinterpret_cast<int32_t *>(ws + L.v[3]);
  int32_t *inv_perm = reinterpret_cast<int32_t *>(ws + L.v[4]);
  void *x_rows = ws + L.v[5];
  void *h = ws + L.v[6];
  void *d = ws + L.v[7];
  NVFP4MOE_TRY(cudaMemsetAsync(ws + L.v[0], 0, kHeaderBytes, s));

  // routing metadata, then the rows of x in the padded grouped layout
  PermuteParams pp;
  pp.topk_idx = topk_idx;
  pp.T = T;
  pp.k = k;
  pp.E = E;
  pp.block_counts = reinterpret_cast<int32_t *>(ws + L.counts);
  pp.local_rank = reinterpret_cast<int32_t *>(ws + L.local_rank);
  pp.offsets = offsets;
  pp.padded_offsets = padded;
  pp.perm = perm;
  pp.inv_perm = inv_perm;
  pp.err = err;
  NVFP4MOE_TRY(launch_route_count(pp, s));
  NVFP4MOE_TRY(launch_route_scan(pp, s));
  NVFP4MOE_TRY(launch_route_rank(pp, s));
  BwdGatherParams gp{};
  gp.x = x;
  gp.topk_w = topk_w;
  gp.topk_idx = topk_idx;
  gp.perm = perm;
  gp.inv_perm = inv_perm;
  gp.offsets = offsets;
  gp.padded_offsets = padded;
  gp.T = T;
  gp.H = H;
  gp.rows_cap = cap;
  gp.k = k;
  gp.E = E;
  gp.x_rows = x_rows;
  gp.mxfp8_x = mxfp8 ? 1 : 0;
  NVFP4MOE_TRY(launch_bwd_gather(gp, s));

  Bf16GemmArgs base;
  base.mode = kBfRows;
  base.offsets = offsets;
  base.padded_offsets = padded;
  base.E = E;
  base.rows_cap = cap;
  base.err = err;
  // gate_up with NVFP4 weights, SwiGLU epilogue -> h (padded rows)
  Bf16GemmArgs g1 = base;
  g1.a = x_rows;
  g1.b = w_gate_up->q;
  g1.b_sf = w_gate_up->sf;
  g1.s_dec_w = w_gate_up->s_dec;
  g1.N = 2 * I;
  g1.K = H;
  g1.epilogue = kBfSwiGLUFwd;
  g1.out_bf16 = h;
  g1.out_padded = 1;
  g1.mxfp8_h = mxfp8 ? 1 : 0;
  g1.w4_wide = 1;
  g1.h_pre = keep_h_pre ? ws + L.v[8] : nullptr;
  NVFP4MOE_TRY(launch_bf16_gemm(g1, s));
  // down with NVFP4 weights -> D (compact sorted rows)
  Bf16GemmArgs g2 = base;
  g2.a = h;
  g2.b = w_down->q;
  g2.b_sf = w_down->sf;
  g2.s_dec_w = w_down->s_dec;
  g2.N = H;
  g2.K = I;
  g2.epilogue = kBfStore;
  g2.out_bf16 = d;
  g2.out_padded = 0;
  g2.w4_wide = 1;
  NVFP4MOE_TRY(launch_bf16_gemm(g2, s));
  NVFP4MOE_TRY(launch_combine(d, inv_perm, topk_w, T, k, H, y, s));
  return NVFP4MOE_OK;
}

}  // namespace

extern "C" {

size_t moe_expert_layer_w4a16_workspace_size(int64_t T, int64_t H, int64_t I, int E, int k, uint32_t flags) {
  (void)flags;
  if (T < 0 || H <= 0 || I <= 0 || E < 1 || k < 1) return 0;
  return (size_t)w4a16_layout(T, H, I, E, k).v[15];
}

int moe_expert_layer_w4a16_workspace_offsets(int64_t T, int64_t H, int64_t I, int E, int k, uint32_t flags,
                                             int64_t *out) {
  (void)flags;
  if (out == nullptr || T < 0 || H <= 0 || I <= 0 || E < 1 || k < 1) return NVFP4MOE_ERR_INVALID_ARG;
  const BwdLayout L = w4a16_layout(T, H, I, E, k);
  for (int i = 0; i < 16; ++i) out[i] = L.v[i];
  return NVFP4MOE_OK;
}

int moe_expert_layer_w4a16(const void *x, const int32_t *topk_idx, const float *topk_w,
                           const nvfp4moe_weights *w_gate_up, const nvfp4moe_weights *w_down, int64_t T, int64_t H,
                           int64_t I, int E, int k, void *y, uint32_t flags, void *workspace, size_t workspace_bytes,
                           nvfp4moe_stream_t stream) {
  return w4ax_layer(x, topk_idx, topk_w, w_gate_up, w_down, T, H, I, E, k, y, flags, workspace, workspace_bytes,
                    stream, false);
}

size_t moe_expert_layer_w4a8_workspace_size(int64_t T, int64_t H, int64_t I, int E, int k, uint32_t flags) {
  if (T < 0 || H <= 0 || I <= 0 || E < 1 || k < 1) return 0;
  return (size_t)w4a16_layout(T, H, I, E, k, (flags & NVFP4MOE_KEEP_H) != 0).v[15];
}

int moe_expert_layer_w4a8_workspace_offsets(int64_t T, int64_t H, int64_t I, int E, int k, uint32_t flags,
                                            int64_t *out) {
  if (out == nullptr || T < 0 || H <= 0 || I <= 0 || E < 1 || k < 1) return NVFP4MOE_ERR_INVALID_ARG;
  const BwdLayout L = w4a16_layout(T, H, I, E, k, (flags & NVFP4MOE_KEEP_H) != 0);
  for (int i = 0; i < 16; ++i) out[i] = L.v[i];
  return NVFP4MOE_OK;
}

int moe_expert_layer_w4a8(const void *x, const int32_t *topk_idx, const float *topk_w,
                          const nvfp4moe_weights *w_gate_up, const nvfp4moe_weights *w_down, int64_t T, int64_t H,
                          int64_t I, int E, int k, void *y, uint32_t flags, void *workspace, size_t workspace_bytes,
                          nvfp4moe_stream_t stream) {
  return w4ax_layer(x, topk_idx, topk_w, w_gate_up, w_down, T, H, I, E, k, y, flags, workspace, workspace_bytes,
                    stream, true);
}

// ------------------------------------------------------------ router GEMM --

size_t moe_router_logits_workspace_size(void) { return 256; }

int moe_router_logits(const void *x, const void *w_router, int64_t T, int64_t H, int E, float *logits,
                      void *workspace, size_t workspace_bytes, nvfp4moe_stream_t stream) {
  if (T < 0 || H <= 0 || E < 1) return NVFP4MOE_ERR_INVALID_ARG;
  if (E > 1024 || E % 32 != 0 || H % 64 != 0 || T > (int64_t)1 << 30) return NVFP4MOE_ERR_UNSUPPORTED_SHAPE;
  if (T == 0) return NVFP4MOE_OK;
  if (x == nullptr || w_router == nullptr || logits == nullptr) return NVFP4MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(w_router) || !aligned16(logits) || !aligned16(workspace))
    return NVFP4MOE_ERR_MISALIGNED;
  if (workspace == nullptr || workspace_bytes < 256) return NVFP4MOE_ERR_WORKSPACE;
  cudaStream_t s = st(stream);
  // workspace: the error word at 0 (as in every workspace), the GEMM's group metadata at 64
  int *err = static_cast<int *>(workspace);
  int32_t *meta = reinterpret_cast<int32_t *>(static_cast<uint8_t *>(workspace) + 64);
  const int64_t t_pad = (T + 127) / 128 * 128;
  NVFP4MOE_TRY(cudaMemsetAsync(workspace, 0, 256, s));
  NVFP4MOE_TRY(launch_router_meta(meta, T, t_pad, s));
  // logits = x W_r^T: one group of T rows (A = x), B = W_r K-major; tile rows
  // past T and past E read as zeros (the tensor maps hold the true row
  // counts), and only the first E columns are stored, with leading dimension E
  Bf16GemmArgs g;
  g.mode = kBfRows;
  g.a = x;
  g.b = w_router;
  g.b_mn = 0;
  g.offsets = meta;
  g.padded_offsets = meta + 2;
  g.E = 1;
  g.rows_cap = t_pad;
  g.N = (E + 255) / 256 * 256;
  g.K = H;
  g.epilogue = kBfStore;
  g.out_f32 = logits;
  g.out_padded = 0;
  g.a_rows = T;
  g.b_rows = E;
  g.n_store = E;
  g.out_ld = E;
  g.err = err;
  NVFP4MOE_TRY(launch_bf16_gemm(g, s));
  return NVFP4MOE_OK;
}

// -------------------------------------------------- expert parallelism --

size_t moe_ep_dispatch_workspace_size(int64_t T, int E, int k) {
  if (T < 0 || E < 1 || k < 1) return 0;
  Carve c;
  c.take(kHeaderBytes);
  c.take((E + 1) * 4);                      // padded offsets (the compact layout does not use them)
  c.take(T * k * 4);                        // perm
  c.take(permute_blocks(T) * E * 4);        // routing block counts
  c.take(T * k * 4);                        // local ranks
  return (size_t)c.off;
}

int moe_ep_dispatch_pack(const void *x, const int32_t *topk_idx, int64_t T, int64_t H, int E, int k, uint8_t *q_send,
                         uint8_t *sf_send, float *sdec_send, int32_t *offsets, int32_t *inv_perm, void *workspace,
                         size_t workspace_bytes, nvfp4moe_stream_t stream) {
  if (T < 0 || H <= 0 || E < 1 || k < 1 || k > 32) return NVFP4MOE_ERR_INVALID_ARG;
  if (E > 1024 || H % 256 != 0) return NVFP4MOE_ERR_UNSUPPORTED_SHAPE;
  if (offsets == nullptr || workspace == nullptr) return NVFP4MOE_ERR_INVALID_ARG;
  if (T > 0 && (x == nullptr || topk_idx == nullptr || q_send == nullptr || sf_send == nullptr ||
                sdec_send == nullptr || inv_perm == nullptr))
    return NVFP4MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(q_send) || !aligned16(sf_send) || !aligned16(workspace))
    return NVFP4MOE_ERR_MISALIGNED;
  if (workspace_bytes < moe_ep_dispatch_workspace_size(T, E, k)) return NVFP4MOE_ERR_WORKSPACE;
  cudaStream_t s = st(stream);
  uint8_t *ws = static_cast<uint8_t *>(workspace);
  Carve c;
  int *err = reinterpret_cast<int *>(ws + c.take(kHeaderBytes));
  int32_t *padded = reinterpret_cast<int32_t *>(ws + c.take((E + 1) * 4));
  int32_t *perm = reinterpret_cast<int32_t *>(ws + c.take(T * k * 4));
  int32_t *block_counts = reinterpret_cast<int32_t *>(ws + c.take(permute_blocks(T) * E * 4));
  int32_t *local_rank = reinterpret_cast<int32_t *>(ws + c.take(T * k * 4));
  NVFP4MOE_TRY(cudaMemsetAsync(ws, 0, kHeaderBytes, s));
  if (T == 0) {
    NVFP4MOE_TRY(cudaMemsetAsync(offsets, 0, (E + 1) * 4, s));
    return NVFP4MOE_OK;
  }
  PermuteParams pp;
  pp.topk_idx = topk_idx;
  pp.T = T;
  pp.k = k;
  pp.E = E;
  pp.block_counts = block_counts;
  pp.local_rank = local_rank;
  pp.offsets = offsets;
  pp.padded_offsets = padded;
  pp.perm = perm;
  pp.inv_perm = inv_perm;
  pp.err = err;
  pp.rows_cap = layer_rows_cap(T, k, E);
  NVFP4MOE_TRY(launch_route_count(pp, s));
  NVFP4MOE_TRY(launch_route_scan(pp, s));
  // each token quantized once (per-token scale) and written to its k rows in
  // compact sorted order: the destination offsets are the compact ones
  QuantParams q;
  q.x = x;
  q.tasks = T;
  q.K = H;
  q.mode = kQuantScatter;
  q.q = q_send;
  q.sf = sf_send;
  q.sf_layout = kSfRowMajor;
  q.s_dec = sdec_send;
  q.s_dec_rows = 1;
  q.rows_cap = T * k;
  q.topk_idx = topk_idx;
  q.offsets = offsets;
  q.padded_offsets = offsets;
  q.k = k;
  q.E = E;
  q.local_rank = local_rank;
  q.block_base = block_counts;
  q.perm_out = perm;
  q.inv_perm_out = inv_perm;
  q.amax_rows = 1;
  q.compute_row_amax = 1;
  return cuda_rc(launch_quant(q, s));
}

int64_t moe_ep_rows_cap(int64_t rows_recv, int El) {
  if (rows_recv < 0 || El < 1) return 0;
  return layer_rows_cap(rows_recv, 1, El);
}

size_t moe_ep_arrange_workspace_size(int G, int El) {
  if (G < 1 || El < 1) return 0;
  return (size_t)(kHeaderBytes + round_up((int64_t)3 * G * El * 4, kAlign));
}

int moe_ep_arrange(const uint8_t *q_recv, const uint8_t *sf_recv, const float *sdec_recv, const int32_t *counts, int G,
                   int El, int64_t rows_recv, int64_t H, int64_t rows_cap, uint8_t *q_a, uint8_t *sf_a, float *sdec_a,
                   int32_t *offsets, int32_t *padded_offsets, void *workspace, size_t workspace_bytes,
                   nvfp4moe_stream_t stream) {
  if (G < 1 || El < 1 || rows_recv < 0 || H <= 0 || rows_cap < 0) return NVFP4MOE_ERR_INVALID_ARG;
  if ((int64_t)G * El > 1024 || H % 256 != 0 || rows_cap % 128 != 0) return NVFP4MOE_ERR_UNSUPPORTED_SHAPE;
  if (rows_cap < moe_ep_rows_cap(rows_recv, El)) return NVFP4MOE_ERR_WORKSPACE;
  if (counts == nullptr || q_a == nullptr || sf_a == nullptr || sdec_a == nullptr || offsets == nullptr ||
      padded_offsets == nullptr || workspace == nullptr ||
      (rows_recv > 0 && (q_recv == nullptr || sf_recv == nullptr || sdec_recv == nullptr)))
    return NVFP4MOE_ERR_INVALID_ARG;
  if (!aligned16(q_recv) || !aligned16(sf_recv) || !aligned16(q_a) || !aligned16(sf_a) || !aligned16(workspace))
    return NVFP4MOE_ERR_MISALIGNED;
  if (workspace_bytes < moe_ep_arrange_workspace_size(G, El)) return NVFP4MOE_ERR_WORKSPACE;
  cudaStream_t s = st(stream);
  uint8_t *ws = static_cast<uint8_t *>(workspace);
  int *err = reinterpret_cast<int *>(ws);
  int32_t *tab = reinterpret_cast<int32_t *>(ws + kHeaderBytes);
  NVFP4MOE_TRY(cudaMemsetAsync(ws, 0, kHeaderBytes, s));
  NVFP4MOE_TRY(launch_ep_tables(counts, G, El, offsets, padded_offsets, tab, err, s));
  EpArrangeParams a;
  a.q_recv = q_recv;
  a.sf_recv = sf_recv;
  a.sdec_recv = sdec_recv;
  a.counts = counts;
  a.offsets = offsets;
  a.padded = padded_offsets;
  a.tab = tab;
  a.G = G;
  a.El = El;
  a.rows_recv = rows_recv;
  a.H = H;
  a.rows_cap = rows_cap;
  a.q_a = q_a;
  a.sf_a = sf_a;
  a.sdec_a = sdec_a;
  a.err = err;
  NVFP4MOE_TRY(launch_ep_arrange(a, s));
  return NVFP4MOE_OK;
}

int moe_ep_return(const void *d, int G, int El, int64_t rows_recv, int64_t H, void *d_send, void *workspace,
                  size_t workspace_bytes, nvfp4moe_stream_t stream) {
  if (G < 1 || El < 1 || rows_recv < 0 || H <= 0) return NVFP4MOE_ERR_INVALID_ARG;
  if ((int64_t)G * El > 1024 || H % 8 != 0) return NVFP4MOE_ERR_UNSUPPORTED_SHAPE;
  if (workspace == nullptr || (rows_recv > 0 && (d == nullptr || d_send == nullptr))) return NVFP4MOE_ERR_INVALID_ARG;
  if (!aligned16(d) || !aligned16(d_send) || !aligned16(workspace)) return NVFP4MOE_ERR_MISALIGNED;
  if (workspace_bytes < moe_ep_arrange_workspace_size(G, El)) return NVFP4MOE_ERR_WORKSPACE;
  uint8_t *ws = static_cast<uint8_t *>(workspace);
  return cuda_rc(launch_ep_return(d, reinterpret_cast<const int32_t *>(ws + kHeaderBytes), G * El, rows_recv, H,
                                  d_send, reinterpret_cast<int *>(ws), st(stream)));
}

size_t moe_ep_experts_workspace_size(int64_t rows_cap, int64_t H, int64_t I) {
  (void)H;
  if (rows_cap < 0 || I <= 0) return 0;
  Carve c;
  c.take(kHeaderBytes);
  c.take(rows_cap * I * 2);                 // h BF16
  c.take(rows_cap * 4);                     // h row amax
  c.take(rows_cap * I / 2);                 // h codes
  c.take(rows_cap * I / 16);                // h scales (K-step-major)
  c.take(rows_cap * 4);                     // h row S_dec
  return (size_t)c.off;
}

int moe_ep_experts(const uint8_t *q_a, const uint8_t *sf_a, const float *sdec_a, const int32_t *offsets,
                   const int32_t *padded_offsets, int El, int64_t rows_cap, const nvfp4moe_weights *w_gate_up,
                   const nvfp4moe_weights *w_down, int64_t H, int64_t I, void *d, void *workspace,
                   size_t workspace_bytes, nvfp4moe_stream_t stream) {
  if (El < 1 || rows_cap < 0 || H <= 0 || I <= 0) return NVFP4MOE_ERR_INVALID_ARG;
  if (El > 1024 || H % 256 != 0 || I % 256 != 0 || rows_cap % 128 != 0) return NVFP4MOE_ERR_UNSUPPORTED_SHAPE;
  int rc = check_weights(w_gate_up, El, 2 * I, H);
  if (rc != NVFP4MOE_OK) return rc;
  if (!(w_gate_up->flags & NVFP4MOE_W_GATE_UP)) return NVFP4MOE_ERR_INVALID_ARG;
  rc = check_weights(w_down, El, H, I);
  if (rc != NVFP4MOE_OK) return rc;
  if (q_a == nullptr || sf_a == nullptr || sdec_a == nullptr || offsets == nullptr || padded_offsets == nullptr ||
      d == nullptr || workspace == nullptr)
    return NVFP4MOE_ERR_INVALID_ARG;
  if (!aligned16(q_a) || !aligned16(sf_a) || !aligned16(d) || !aligned16(workspace)) return NVFP4MOE_ERR_MISALIGNED;
  if (workspace_bytes < moe_ep_experts_workspace_size(rows_cap, H, I)) return NVFP4MOE_ERR_WORKSPACE;
  if (rows_cap == 0) return NVFP4MOE_OK;
  cudaStream_t s = st(stream);
  uint8_t *ws = static_cast<uint8_t *>(workspace);
  Carve c;
  int *err = reinterpret_cast<int *>(ws + c.take(kHeaderBytes));
  void *hb = ws + c.take(rows_cap * I * 2);
  float *h_amax = reinterpret_cast<float *>(ws + c.take(rows_cap * 4));
  uint8_t *hq = ws + c.take(rows_cap * I / 2);
  uint8_t *hsf = ws + c.take(rows_cap * I / 16);
  float *hsd = reinterpret_cast<float *>(ws + c.take(rows_cap * 4));
  NVFP4MOE_TRY(cudaMemsetAsync(ws, 0, kHeaderBytes, s));
  // padding rows keep amax 0: the requantization leaves them as zero codes
  NVFP4MOE_TRY(cudaMemsetAsync(h_amax, 0, rows_cap * 4, s));
  // gate_up grouped GEMM + SwiGLU epilogue (h in BF16, per-row amax of h)
  GemmArgs g;
  std::memset(&g, 0, sizeof(g));
  g.q_a = q_a;
  g.sf_a = sf_a;
  g.s_dec_a = sdec_a;
  g.s_dec_a_rows = 1;
  g.q_w = w_gate_up->q;
  g.sf_w = w_gate_up->sf;
  g.s_dec_w = w_gate_up->s_dec;
  g.offsets = offsets;
  g.padded_offsets = padded_offsets;
  g.E = El;
  g.rows_cap = rows_cap;
  g.N = 2 * I;
  g.K = H;
  g.epilogue = kEpiSwiGLU;
  g.out_bf16 = hb;
  g.out_padded = 1;
  g.amax_h = h_amax;
  g.amax_h_rows = 1;
  g.err = err;
  NVFP4MOE_TRY(launch_grouped_gemm(g, s));
  // requantize h per row with the amax the epilogue reduced
  QuantParams rq;
  rq.x = hb;
  rq.tasks = rows_cap;                      // the requantization walks the padded rows
  rq.K = I;
  rq.mode = kQuantRequant;
  rq.amax_src = h_amax;
  rq.amax_rows = 1;
  rq.q = hq;
  rq.sf = hsf;
  rq.sf_layout = kSfKStep;
  rq.s_dec = hsd;
  rq.s_dec_rows = 1;
  rq.rows_cap = rows_cap;
  rq.offsets = offsets;
  rq.padded_offsets = padded_offsets;
  rq.E = El;
  NVFP4MOE_TRY(launch_quant(rq, s));
  // down grouped GEMM -> D (BF16, compact local rows)
  GemmArgs dn;
  std::memset(&dn, 0, sizeof(dn));
  dn.q_a = hq;
  dn.sf_a = hsf;
  dn.s_dec_a = hsd;
  dn.s_dec_a_rows = 1;
  dn.q_w = w_down->q;
  dn.sf_w = w_down->sf;
  dn.s_dec_w = w_down->s_dec;
  dn.offsets = offsets;
  dn.padded_offsets = padded_offsets;
  dn.E = El;
  dn.rows_cap = rows_cap;
  dn.N = H;
  dn.K = I;
  dn.epilogue = kEpiStore;
  dn.out_bf16 = d;
  dn.out_padded = 0;
  dn.err = err;
  NVFP4MOE_TRY(launch_grouped_gemm(dn, s));
  return NVFP4MOE_OK;
}

}  // extern "C"
