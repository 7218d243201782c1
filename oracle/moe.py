"""Token-to-expert permutation, grouped GEMM, SwiGLU + requantize, combine and
the whole W4A4 MoE expert layer -- CPU oracle (test infrastructure only).

Source passages
  * news.hamidun.com (Arabic / Russian editions), section "diagnostics,
    alignment and fast kernels": grouped GEMMs matter for MoE models such as
    Qwen3-30B-A3B whose work is split over many experts, and their overhead is
    why naive FP4 can lose to BF16.
  * www.aib.vote "miniTE report, NVFP4 RL stability", paragraph 4: contiguous
    data layout, device-side metadata, amax reuse, grouped matrix
    multiplication and operator fusion in the token-wise NVFP4 path.
  * The same pages' strict-alignment mode (learner and rollout compute one
    policy, log-prob gap about 1e-8): results must not depend on how tokens are
    batched, which is why strict mode uses per-token scales.

Readings taken where the pages are silent:
  R8   Rows are ordered by (expert, token, slot); each expert's group starts at
       a multiple of 128 rows in the padded layout.
  R9   GEMM: out[r, n] = sum_k x_hat_a[r, k] * x_hat_w[e(r), n, k] in fp64,
       then one rounding to the output type.
  R10  The fused gate_up weight holds the gate rows 0..I-1 and the up rows
       I..2I-1 of one [2I][H] matrix per expert, quantized as one tensor.
  R11  SwiGLU h = silu(g) * u with silu(g) = g / (1 + exp(-g)) in fp64, rounded
       once to BF16; the requantize input is that BF16 h.
  R12  Down-projection rows are BF16; y[t] = BF16( sum_j w[t,j] * D[t,j] ) with
       the sum in fp64 in slot order.
  R15  Top-k routing from FP32 router logits: the k experts with the largest
       logits (softmax is monotone, so these are the k most probable; ties
       go to the lower expert id), slots in descending logit order, and the
       weights are the softmax renormalised over the chosen k (Qwen3-MoE
       style), in fp64.
"""
from __future__ import annotations

import numpy as np

from . import nvfp4

GROUP_ALIGN = 128


def route_topk(logits: np.ndarray, k: int):
    """R15: top-k experts per token from router logits [T][E] (FP32 values).

    The choice is exact -- a comparison of the logits themselves, lower expert
    id first on equal logits -- and the weights are
    w_j = exp(l_j - l_max) / sum_{i in top-k} exp(l_i - l_max) in fp64.
    Returns idx int32 [T][k] and w float64 [T][k]."""
    logits = np.asarray(logits, dtype=np.float64)
    T, E = logits.shape
    if not 1 <= k <= E:
        raise ValueError("need 1 <= k <= E")
    idx = np.empty((T, k), dtype=np.int32)
    w = np.empty((T, k), dtype=np.float64)
    ids = np.arange(E)
    for t in range(T):
        # descending logit, ascending id on ties: lexsort sorts by its last key first
        order = np.lexsort((ids, -logits[t]))[:k]
        idx[t] = order
        z = np.exp(logits[t, order] - logits[t, order[0]])
        w[t] = z / z.sum()
    return idx, w


def permutation(topk_idx: np.ndarray, num_experts: int):
    """R8: stable order of the T*k routed rows by (expert, token, slot).

    Returns offsets[E+1], padded_offsets[E+1], perm[R] (perm[r] = t*k + j) and
    inv_perm[T][k] (inv_perm[t][j] = r).  r is the unpadded sorted position;
    the padded position of the same row is r - offsets[e] + padded_offsets[e].
    """
    topk_idx = np.asarray(topk_idx, dtype=np.int64)
    T, k = topk_idx.shape
    flat = topk_idx.reshape(-1)
    if flat.size and (flat.min() < 0 or flat.max() >= num_experts):
        raise ValueError("expert index out of range")
    counts = np.bincount(flat, minlength=num_experts)
    offsets = np.zeros(num_experts + 1, dtype=np.int64)
    offsets[1:] = np.cumsum(counts)
    padded = np.zeros(num_experts + 1, dtype=np.int64)
    padded[1:] = np.cumsum((counts + GROUP_ALIGN - 1) // GROUP_ALIGN * GROUP_ALIGN)
    # flat index t*k + j already orders (token, slot); a stable sort by expert
    # keeps that order inside each group.
    perm = np.argsort(flat, kind="stable")
    inv = np.empty_like(perm)
    inv[perm] = np.arange(perm.size)
    return {
        "offsets": offsets.astype(np.int32),
        "padded_offsets": padded.astype(np.int32),
        "perm": perm.astype(np.int32),
        "inv_perm": inv.reshape(T, k).astype(np.int32),
        "counts": counts.astype(np.int32),
    }


def padded_rows(perm_info) -> np.ndarray:
    """Padded row index of every sorted row r (length R)."""
    off = perm_info["offsets"].astype(np.int64)
    pad = perm_info["padded_offsets"].astype(np.int64)
    E = len(off) - 1
    expert_of_r = np.repeat(np.arange(E), np.diff(off))
    r = np.arange(off[-1])
    return r - off[expert_of_r] + pad[expert_of_r]


def expert_of_rows(offsets: np.ndarray) -> np.ndarray:
    off = np.asarray(offsets, dtype=np.int64)
    return np.repeat(np.arange(len(off) - 1), np.diff(off))


def grouped_gemm(a_hat: np.ndarray, offsets: np.ndarray, w_hat_of_expert) -> np.ndarray:
    """R9: per expert e, rows offsets[e]..offsets[e+1] of a_hat times W_e^T, fp64.

    w_hat_of_expert(e) returns the dequantized [N][K] weight of expert e.
    Returns fp64 [R][N].
    """
    off = np.asarray(offsets, dtype=np.int64)
    R = int(off[-1])
    out = None
    for e in range(len(off) - 1):
        lo, hi = int(off[e]), int(off[e + 1])
        if hi == lo:
            continue
        w = w_hat_of_expert(e)
        if out is None:
            out = np.zeros((R, w.shape[0]), dtype=np.float64)
        out[lo:hi] = a_hat[lo:hi] @ w.T
    if out is None:
        out = np.zeros((R, 0), dtype=np.float64)
    return out


def grouped_gemm_abs(a_hat: np.ndarray, offsets: np.ndarray, w_hat_of_expert) -> np.ndarray:
    """sum_k |a_k * w_k| for every output element: the scale of the GEMM
    tolerance bound |err| <= 1e-5 * sum_k |a_k w_k| + 1e-6."""
    return grouped_gemm(np.abs(a_hat), offsets, lambda e: np.abs(w_hat_of_expert(e)))


def silu(g: np.ndarray) -> np.ndarray:
    """silu(g) = g / (1 + exp(-g)) in fp64 (R11)."""
    g = np.asarray(g, dtype=np.float64)
    with np.errstate(over="ignore"):
        return g / (1.0 + np.exp(-g))


def swiglu(gate_up: np.ndarray, inter: int) -> np.ndarray:
    """R10/R11: h = silu(gate) * up, fp64, from [R][2I] (gate | up)."""
    g = gate_up[:, :inter]
    u = gate_up[:, inter:2 * inter]
    return silu(g) * u


def combine(d_rows_bf16: np.ndarray, inv_perm: np.ndarray, topk_w: np.ndarray) -> np.ndarray:
    """R12: y[t] = BF16( sum_j w[t,j] * D[inv_perm[t,j]] ), fp64 sum in slot order."""
    T, k = inv_perm.shape
    acc = np.zeros((T, d_rows_bf16.shape[1]), dtype=np.float64)
    w = np.asarray(topk_w, dtype=np.float32).astype(np.float64)
    for j in range(k):
        acc += w[:, j:j + 1] * d_rows_bf16[inv_perm[:, j]].astype(np.float64)
    return nvfp4.round_to_bf16(acc)


class QuantWeights:
    """Per-expert NVFP4 weights: each expert's [N][K] matrix is one tensor
    (one S_dec per expert, R10)."""

    def __init__(self, w: np.ndarray):
        """w: [E][N][K] float32 holding BF16 values."""
        self.E, self.N, self.K = w.shape
        self.q, self.sf, self.s_dec, self.amax = [], [], [], []
        for e in range(self.E):
            r = nvfp4.quantize(w[e], per_token=False)
            self.q.append(r["q"])
            self.sf.append(r["sf"])
            self.s_dec.append(r["s_dec"][0])
            self.amax.append(r["amax"][0])
        self.s_dec = np.array(self.s_dec, dtype=np.float32)
        self.amax = np.array(self.amax, dtype=np.float32)
        self._cache = {}

    def dequant(self, e: int) -> np.ndarray:
        if e not in self._cache:
            self._cache[e] = nvfp4.dequantize(self.q[e], self.sf[e], self.s_dec[e:e + 1])
        return self._cache[e]


def expert_layer(x: np.ndarray, topk_idx: np.ndarray, topk_w: np.ndarray,
                 w_gate_up: QuantWeights, w_down: QuantWeights, per_token: bool):
    """The W4A4 MoE expert layer, end to end, in the pages' order:

      1. quantize x once per token (amax reused for all k copies)
      2. permute rows to the contiguous (expert, token, slot) layout
      3. gate_up grouped GEMM (fp64 on dequantized operands)
      4. SwiGLU, BF16 h, requantize h (per tensor over all routed rows, or per
         row in per-token mode)
      5. down grouped GEMM -> BF16 rows D
      6. weighted combine in slot order -> BF16 y

    Returns a dict with every intermediate so that tests can compare stage by
    stage.
    """
    T, H = x.shape
    E = w_gate_up.E
    inter = w_gate_up.N // 2
    qx = nvfp4.quantize(x, per_token=per_token)
    x_hat = nvfp4.dequantize(qx["q"], qx["sf"], qx["s_dec"])
    p = permutation(topk_idx, E)
    k = topk_idx.shape[1]
    tok_of_row = p["perm"] // k
    a_hat = x_hat[tok_of_row]
    gu = grouped_gemm(a_hat, p["offsets"], w_gate_up.dequant)
    h = nvfp4.round_to_bf16(swiglu(gu, inter))
    qh = nvfp4.quantize(h, per_token=per_token)
    h_hat = nvfp4.dequantize(qh["q"], qh["sf"], qh["s_dec"])
    d = nvfp4.round_to_bf16(grouped_gemm(h_hat, p["offsets"], w_down.dequant))
    y = combine(d, p["inv_perm"], topk_w)
    return {"qx": qx, "perm": p, "gate_up": gu, "h": h, "qh": qh, "d": d, "y": y}
