// moe_permute without a caller workspace: the scratch lives in a file-scope
// device array instead.
//
// Who needs this: callers that can hand over their own input and output
// buffers but cannot provide scratch memory -- code embedded in a host
// framework whose memory planner owns every device byte and allows no
// allocation after start-up, or code running where cudaMalloc is forbidden
// (for example while another component is capturing work).  This entry point
// and its array are an addition of this library; the pages describe no such
// interface.
//
// The array (kScratchBytes, about 1 MB) exists once per GPU that loads the
// library and stays until the process exits.  Its device address is looked up
// with cudaGetSymbolAddress the first time the entry point runs on a device
// (that device current); that first call should therefore come before any
// stream capture.  All calls share the array: two calls that overlap on the
// GPU race on it.
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace nvfp4moe {
namespace {

// Capacity of the static scratch.
constexpr int64_t kMaxRows = 131072;          // T * k routed rows (local ranks)
constexpr int64_t kMaxBlockCounts = 131072;   // ceil(T / 128) * E per-block expert counts
constexpr size_t kHeaderBytes = 256;
constexpr size_t kScratchBytes = kHeaderBytes + 4 * kMaxBlockCounts + 4 * kMaxRows;

__device__ __align__(256) uint8_t g_permute_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
uint8_t *g_scratch_addr[kMaxDevices] = {};
std::mutex g_scratch_mutex;

// Device address of the array on the current device (looked up once).
cudaError_t scratch_address(uint8_t **out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (g_scratch_addr[dev] == nullptr) {
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_permute_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_addr[dev] = static_cast<uint8_t *>(p);
  }
  *out = g_scratch_addr[dev];
  return cudaSuccess;
}

}  // namespace
}  // namespace nvfp4moe

using namespace nvfp4moe;

extern "C" int moe_permute_noalloc(const int32_t *topk_idx, int64_t T, int k, int E, int32_t *offsets,
                                   int32_t *padded_offsets, int32_t *perm, int32_t *inv_perm,
                                   nvfp4moe_stream_t stream) {
  if (T < 0 || k < 1 || k > 32 || E < 1) return NVFP4MOE_ERR_INVALID_ARG;
  if (E > 1024) return NVFP4MOE_ERR_UNSUPPORTED_SHAPE;
  if (offsets == nullptr || padded_offsets == nullptr ||
      (T > 0 && (topk_idx == nullptr || perm == nullptr || inv_perm == nullptr)))
    return NVFP4MOE_ERR_INVALID_ARG;
  // sizes beyond the static scratch are refused, never truncated
  if (T * k > kMaxRows || permute_blocks(T) * E > kMaxBlockCounts) return NVFP4MOE_ERR_WORKSPACE;
  uint8_t *scratch = nullptr;
  if (scratch_address(&scratch) != cudaSuccess) return NVFP4MOE_ERR_CUDA;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  // the error word is the one part that must start at zero (it is not
  // reported by this entry point; bad routing entries are skipped)
  if (cudaMemsetAsync(scratch, 0, 16, s) != cudaSuccess) return NVFP4MOE_ERR_CUDA;
  PermuteParams p;
  p.topk_idx = topk_idx;
  p.T = T;
  p.k = k;
  p.E = E;
  p.block_counts = reinterpret_cast<int32_t *>(scratch + kHeaderBytes);
  p.local_rank = reinterpret_cast<int32_t *>(scratch + kHeaderBytes + 4 * kMaxBlockCounts);
  p.offsets = offsets;
  p.padded_offsets = padded_offsets;
  p.perm = perm;
  p.inv_perm = inv_perm;
  p.err = reinterpret_cast<int *>(scratch);
  if (launch_route_count(p, s) != cudaSuccess) return NVFP4MOE_ERR_CUDA;
  if (launch_route_scan(p, s) != cudaSuccess) return NVFP4MOE_ERR_CUDA;
  if (launch_route_rank(p, s) != cudaSuccess) return NVFP4MOE_ERR_CUDA;
  return NVFP4MOE_OK;
}
