// Warp-wide top-k of one token's router logits (shared by the standalone
// router and the fused router + routing-histogram kernel).
//
// The rule (the pages give none; Qwen3-MoE style): the k experts with the
// largest logits, ties to the lower expert id, slots in descending order,
// weights = softmax renormalised over the chosen k.  The choice compares the
// FP32 logits exactly, so it is bit-reproducible; only the weights carry
// rounding (expf and one division).  Lane l holds logits l, l+32, ...; each of
// the k rounds is a warp arg-best under the strict order (larger logit, then
// lower id), so every lane agrees on the winner whatever the reduction order.
#pragma once

#include <climits>

#include "common.cuh"

namespace nvfp4moe {

// (va, ia) ranks before (vb, ib): larger logit first, then lower expert id
__device__ __forceinline__ bool topk_ranks_before(float va, int ia, float vb, int ib) {
  return va > vb || (va == vb && ia < ib);
}

// The whole warp calls this for one token's logits row.  Lane j < k returns
// the expert of slot j in my_id and its weight in my_w.  NE: logits per lane,
// E <= 32 * NE; 1 <= k <= min(E, 32).
template <int NE>
__device__ __forceinline__ void warp_topk(const float *__restrict__ row, int E, int k, int lane, int &my_id,
                                          float &my_w) {
  float v[NE];
  uint32_t taken = 0;   // bit i: expert i*32 + lane already chosen (or beyond E)
#pragma unroll
  for (int i = 0; i < NE; ++i) {
    const int e = i * 32 + lane;
    v[i] = e < E ? __ldg(row + e) : 0.0f;
    if (e >= E) taken |= 1u << i;
  }
  my_id = 0;
  float my_v = 0.0f;
  for (int j = 0; j < k; ++j) {
    float bv = 0.0f;
    int bi = INT_MAX;   // INT_MAX: this lane has nothing left
#pragma unroll
    for (int i = 0; i < NE; ++i) {
      const int e = i * 32 + lane;
      if (!((taken >> i) & 1u) && (bi == INT_MAX || topk_ranks_before(v[i], e, bv, bi))) {
        bv = v[i];
        bi = e;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (oi != INT_MAX && (bi == INT_MAX || topk_ranks_before(ov, oi, bv, bi))) {
        bv = ov;
        bi = oi;
      }
    }
    // k <= E, so a winner exists; its owner marks it taken
    if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
    if (lane == j) {
      my_id = bi;
      my_v = bv;
    }
  }
  // weights: exp(l_j - l_max) over the chosen, normalised; the sum is a fixed
  // butterfly, so the result depends on nothing but the logits
  const float m = __shfl_sync(0xffffffffu, my_v, 0);
  const float z = lane < k ? expf(my_v - m) : 0.0f;
  float s = z;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  my_w = __fdiv_rn(z, s);
}

}  // namespace nvfp4moe
