// Top-k routing from FP32 router logits, on the device.
//
// The MoE learner's layer (news.hamidun.com "miniTE ... Qwen3-30B-A3B":
// 128 experts, 8 active per token) starts from each token's router logits.
// The pages say the token-wise path keeps its metadata on the device
// (www.aib.vote "miniTE report, NVFP4 RL stability", paragraph 4); this
// kernel turns logits into the topk_idx / topk_w the permutation consumes, so
// nothing about the routing goes through the host.  The rule (the pages give
// none; Qwen3-MoE style): the k experts with the largest logits, ties to the
// lower expert id, slots in descending order, weights = softmax renormalised
// over the chosen k.  The choice compares the FP32 logits exactly, so it is
// bit-reproducible; only the weights carry rounding (expf and one division).
//
// One warp per token (warp_topk in topk.cuh).  The fused variant that also
// builds the routing histogram lives in permute.cu.
#include "common.cuh"
#include "internal.h"
#include "topk.cuh"

namespace nvfp4moe {

namespace {

constexpr int kRouteWarps = 8;

template <int NE>   // logits per lane: E <= 32 * NE
__global__ void __launch_bounds__(kRouteWarps * 32)
    k_route_topk(const float *__restrict__ logits, int64_t T, int E, int k, int32_t *__restrict__ idx_out,
                 float *__restrict__ w_out) {
  const int lane = threadIdx.x & 31;
  const int64_t t = (int64_t)blockIdx.x * kRouteWarps + (threadIdx.x >> 5);
  if (t >= T) return;
  int my_id;
  float my_w;
  warp_topk<NE>(logits + t * E, E, k, lane, my_id, my_w);
  if (lane < k) {
    idx_out[t * k + lane] = my_id;
    w_out[t * k + lane] = my_w;
  }
}

template <int NE>
cudaError_t launch_topk(const float *logits, int64_t T, int E, int k, int32_t *idx, float *w, cudaStream_t s) {
  const int64_t blocks = (T + kRouteWarps - 1) / kRouteWarps;
  k_route_topk<NE><<<(unsigned)blocks, kRouteWarps * 32, 0, s>>>(logits, T, E, k, idx, w);
  return cudaGetLastError();
}

bool aligned16_ptr(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace nvfp4moe

namespace nvfp4moe {
namespace {
// The one-group metadata of the router GEMM: offsets {0, T}, padded {0, Tpad}.
__global__ void k_router_meta(int32_t *meta, int32_t T, int32_t Tpad) {
  if (threadIdx.x == 0) {
    meta[0] = 0;
    meta[1] = T;
    meta[2] = 0;
    meta[3] = Tpad;
  }
}
}  // namespace

cudaError_t launch_router_meta(int32_t *meta, int64_t T, int64_t Tpad, cudaStream_t s) {
  k_router_meta<<<1, 32, 0, s>>>(meta, (int32_t)T, (int32_t)Tpad);
  return cudaGetLastError();
}
}  // namespace nvfp4moe

using namespace nvfp4moe;

extern "C" int moe_route_topk(const float *logits, int64_t T, int E, int k, int32_t *topk_idx, float *topk_w,
                              nvfp4moe_stream_t stream) {
  if (T < 0 || E < 1 || k < 1) return NVFP4MOE_ERR_INVALID_ARG;
  if (E > 1024 || k > 32 || k > E) return NVFP4MOE_ERR_UNSUPPORTED_SHAPE;
  if (T == 0) return NVFP4MOE_OK;
  if (logits == nullptr || topk_idx == nullptr || topk_w == nullptr) return NVFP4MOE_ERR_INVALID_ARG;
  if (!aligned16_ptr(logits) || !aligned16_ptr(topk_idx) || !aligned16_ptr(topk_w))
    return NVFP4MOE_ERR_MISALIGNED;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e;
  if (E <= 32) e = launch_topk<1>(logits, T, E, k, topk_idx, topk_w, s);
  else if (E <= 64) e = launch_topk<2>(logits, T, E, k, topk_idx, topk_w, s);
  else if (E <= 128) e = launch_topk<4>(logits, T, E, k, topk_idx, topk_w, s);
  else if (E <= 256) e = launch_topk<8>(logits, T, E, k, topk_idx, topk_w, s);
  else if (E <= 512) e = launch_topk<16>(logits, T, E, k, topk_idx, topk_w, s);
  else e = launch_topk<32>(logits, T, E, k, topk_idx, topk_w, s);
  return e == cudaSuccess ? NVFP4MOE_OK : NVFP4MOE_ERR_CUDA;
}
