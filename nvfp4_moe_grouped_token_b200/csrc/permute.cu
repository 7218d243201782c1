// Token-to-expert permutation with device-side group offsets.
//
// The contiguous per-expert layout and device-side metadata of the token-wise
// path (www.aib.vote "miniTE report, NVFP4 RL stability", paragraph 4).  Rows
// are ordered by (expert, token, slot): a stable order that needs no sort and
// no atomics whose order could vary from run to run.
//
//   count  one block per 128 tokens.  Each warp marks, per expert, which of
//          its 32 tokens chose that expert (a 32-bit mask built with atomicOr,
//          whose result does not depend on the order of the ORs).  A token's
//          rank inside its block is the popcount of the masks of the earlier
//          warps plus that of its own warp below its lane.  Writes the
//          per-block count of every expert and each (token, slot)'s local rank.
//          The fused variant starts from router logits: each warp runs the
//          top-k of its 32 tokens (topk.cuh), writes topk_idx / topk_w and
//          sets the masks directly -- router and histogram in one pass.
//   scan   one block: exclusive prefix over blocks per expert (in place), the
//          expert totals, and their prefix sums -> offsets / padded_offsets.
//   rank   perm / inv_perm from offsets + block base + local rank (the fused
//          layer path does this inside the quantize-scatter kernel instead).
#include "common.cuh"
#include "internal.h"
#include "topk.cuh"

namespace nvfp4moe {

namespace {

constexpr int kScanThreads = 1024;

// NE == 0: the routing is given (topk_idx); NE > 0: top-k from the router
// logits first (E <= 32 * NE), written to topk_idx (== p.topk_idx) / topk_w.
template <int NE>
__global__ void __launch_bounds__(kRankTokens) k_route_count(const PermuteParams p) {
  extern __shared__ uint32_t smem_u[];
  const int E = p.E, k = p.k;
  uint32_t *masks = smem_u;                                   // [4][E]
  int32_t *wpre = reinterpret_cast<int32_t *>(smem_u + 4 * E);  // [4][E]
  for (int i = threadIdx.x; i < 4 * E; i += blockDim.x) masks[i] = 0;
  __syncthreads();
  const int64_t t = (int64_t)blockIdx.x * kRankTokens + threadIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool live = t < p.T;
  if constexpr (NE > 0) {
    // warp w: the block's tokens w*32 + i, one at a time; token i is bit i
    const int64_t t0 = (int64_t)blockIdx.x * kRankTokens + warp * 32;
    for (int i = 0; i < 32 && t0 + i < p.T; ++i) {
      int id;
      float w;
      warp_topk<NE>(p.logits + (t0 + i) * E, E, k, lane, id, w);
      if (lane < k) {
        p.topk_idx_out[(t0 + i) * k + lane] = id;
        p.topk_w_out[(t0 + i) * k + lane] = w;
        atomicOr(&masks[warp * E + id], 1u << i);
      }
    }
  } else if (live) {
    const int32_t *row = p.topk_idx + t * k;
    for (int j = 0; j < k; ++j) {
      const int e = __ldg(row + j);
      if (e < 0 || e >= E) {
        set_device_error(p.err, kDevBadExpert, e);
        continue;
      }
      bool dup = false;
      for (int jj = 0; jj < j; ++jj) dup |= (__ldg(row + jj) == e);
      if (dup) {
        set_device_error(p.err, kDevDupExpert, e);
        continue;
      }
      atomicOr(&masks[warp * E + e], 1u << lane);
    }
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int run = 0;
#pragma unroll
    for (int w = 0; w < kRankTokens / 32; ++w) {
      wpre[w * E + e] = run;
      run += __popc(masks[w * E + e]);
    }
    p.block_counts[(int64_t)blockIdx.x * E + e] = run;
  }
  __syncthreads();
  if (live) {
    // the fused variant wrote these ids in this launch: coherent loads there;
    // given ids are read-only here and sit in L1 since the first pass
    const int32_t *row = p.topk_idx + t * k;
    auto id_at = [&](int j) { return NE > 0 ? __ldcg(row + j) : __ldg(row + j); };
    const uint32_t below = (1u << lane) - 1u;
    for (int j = 0; j < k; ++j) {
      const int e = id_at(j);
      int32_t r = -1;
      if (e >= 0 && e < E) {
        bool dup = false;
        for (int jj = 0; jj < j; ++jj) dup |= (id_at(jj) == e);
        if (!dup) r = wpre[warp * E + e] + __popc(masks[warp * E + e] & below);
      }
      p.local_rank[t * k + j] = r;
    }
  }
}

__global__ void __launch_bounds__(kScanThreads) k_route_scan(const PermuteParams p, int64_t nblk) {
  __shared__ int32_t partial[kScanThreads];
  __shared__ int32_t scan_a[kScanThreads];
  __shared__ int32_t scan_b[kScanThreads];
  const int E = p.E;
  const int S = kScanThreads / E;          // segments per expert (E <= 1024)
  const int tid = threadIdx.x;
  const int e = tid % E, s = tid / E;
  const int64_t seg = (nblk + S - 1) / S;
  const int64_t b0 = (int64_t)s * seg;
  const int64_t b1 = b0 + seg < nblk ? b0 + seg : nblk;
  // eight loads in flight per step: one at a time, the segment's loads would
  // each wait out a full memory latency
  constexpr int kBatch = 8;
  int32_t sum = 0;
  if (s < S) {
    for (int64_t b = b0; b < b1; b += kBatch) {
      int32_t c[kBatch];
#pragma unroll
      for (int j = 0; j < kBatch; ++j) c[j] = b + j < b1 ? p.block_counts[(b + j) * E + e] : 0;
#pragma unroll
      for (int j = 0; j < kBatch; ++j) sum += c[j];
    }
    partial[s * E + e] = sum;
  }
  __syncthreads();
  int32_t total = 0;
  if (s < S) {
    int32_t base = 0;
    for (int ss = 0; ss < S; ++ss) {
      const int32_t v = partial[ss * E + e];
      if (ss < s) base += v;
      total += v;
    }
    for (int64_t b = b0; b < b1; b += kBatch) {
      int32_t c[kBatch];
#pragma unroll
      for (int j = 0; j < kBatch; ++j) c[j] = b + j < b1 ? p.block_counts[(b + j) * E + e] : 0;
#pragma unroll
      for (int j = 0; j < kBatch; ++j) {
        if (b + j < b1) p.block_counts[(b + j) * E + e] = base;
        base += c[j];
      }
    }
  }
  // inclusive scans of totals and padded totals over experts: a warp scan,
  // then a scan of the 32 warp sums (two block barriers)
  __shared__ int32_t wsum_a[kScanThreads / 32];
  __shared__ int32_t wsum_b[kScanThreads / 32];
  const int32_t v = (tid < E && s == 0) ? total : 0;
  const int32_t vp = (tid < E && s == 0) ? ((total + 127) / 128) * 128 : 0;
  const int lane = tid & 31, wid = tid >> 5;
  int32_t ia = v, ib = vp;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int32_t ya = __shfl_up_sync(0xffffffffu, ia, o);
    const int32_t yb = __shfl_up_sync(0xffffffffu, ib, o);
    if (lane >= o) {
      ia += ya;
      ib += yb;
    }
  }
  if (lane == 31) {
    wsum_a[wid] = ia;
    wsum_b[wid] = ib;
  }
  __syncthreads();
  if (wid == 0) {                            // kScanThreads / 32 == 32 warp sums
    const int32_t oa = wsum_a[lane], ob = wsum_b[lane];
    int32_t xa = oa, xb = ob;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int32_t ya = __shfl_up_sync(0xffffffffu, xa, o);
      const int32_t yb = __shfl_up_sync(0xffffffffu, xb, o);
      if (lane >= o) {
        xa += ya;
        xb += yb;
      }
    }
    wsum_a[lane] = xa - oa;                  // sums of the warps before this one
    wsum_b[lane] = xb - ob;
  }
  __syncthreads();
  ia += wsum_a[wid];
  ib += wsum_b[wid];
  if (tid < E) {
    p.offsets[tid + 1] = ia;
    p.padded_offsets[tid + 1] = ib;
  }
  if (tid == 0) {
    p.offsets[0] = 0;
    p.padded_offsets[0] = 0;
  }
  if (p.zero_pad_rows != nullptr) {
    // a warp per group: its at most 127 padding rows in four 32-wide steps
    scan_a[tid] = v;                         // count of group tid
    scan_b[tid] = ib;                        // padded end of group tid
    __syncthreads();
    for (int g = wid; g < E; g += kScanThreads / 32) {
      const int64_t end = scan_b[g];
      const int32_t cnt = scan_a[g];
      const int64_t start = end - (((int64_t)cnt + 127) / 128) * 128;
      const int64_t stop = end < p.rows_cap ? end : p.rows_cap;
      for (int64_t r = start + cnt + lane; r < stop; r += 32) p.zero_pad_rows[r] = 0.0f;
    }
  }
}

__global__ void k_route_rank(const PermuteParams p) {
  const int64_t n = p.T * p.k;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int e = __ldg(p.topk_idx + i);
    const int32_t lr = __ldg(p.local_rank + i);
    if (e < 0 || e >= p.E || lr < 0) continue;
    const int64_t t = i / p.k;
    const int64_t r = (int64_t)__ldg(p.offsets + e) +
                      __ldg(p.block_counts + (t / kRankTokens) * p.E + e) + lr;
    if (r < 0 || r >= n) continue;
    p.perm[r] = (int32_t)i;
    p.inv_perm[i] = (int32_t)r;
  }
}

}  // namespace

int64_t permute_blocks(int64_t T) { return (T + kRankTokens - 1) / kRankTokens; }

cudaError_t launch_route_count(const PermuteParams &p, cudaStream_t s) {
  const int64_t nblk = permute_blocks(p.T);
  if (nblk == 0) return cudaSuccess;
  const size_t smem = (size_t)8 * p.E * sizeof(uint32_t);
  if (p.logits == nullptr) {
    k_route_count<0><<<(unsigned)nblk, kRankTokens, smem, s>>>(p);
  } else {
    if (p.topk_idx != p.topk_idx_out || p.k > p.E || p.k > 32) return cudaErrorInvalidValue;
    if (p.E <= 32) k_route_count<1><<<(unsigned)nblk, kRankTokens, smem, s>>>(p);
    else if (p.E <= 64) k_route_count<2><<<(unsigned)nblk, kRankTokens, smem, s>>>(p);
    else if (p.E <= 128) k_route_count<4><<<(unsigned)nblk, kRankTokens, smem, s>>>(p);
    else if (p.E <= 256) k_route_count<8><<<(unsigned)nblk, kRankTokens, smem, s>>>(p);
    else if (p.E <= 512) k_route_count<16><<<(unsigned)nblk, kRankTokens, smem, s>>>(p);
    else k_route_count<32><<<(unsigned)nblk, kRankTokens, smem, s>>>(p);
  }
  return cudaGetLastError();
}

cudaError_t launch_route_scan(const PermuteParams &p, cudaStream_t s) {
  k_route_scan<<<1, kScanThreads, 0, s>>>(p, permute_blocks(p.T));
  return cudaGetLastError();
}

cudaError_t launch_route_rank(const PermuteParams &p, cudaStream_t s) {
  const int64_t n = p.T * p.k;
  if (n == 0) return cudaSuccess;
  int64_t blocks = (n + 255) / 256;
  if (blocks > 4096) blocks = 4096;
  k_route_rank<<<(unsigned)blocks, 256, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace nvfp4moe
