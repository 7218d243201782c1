"""Comparison helpers shared by the GPU parity tests.

Tolerances (benchmark spec of the problem):
  * codes, scales, amax, S_dec, offsets and permutation: bit-exact;
  * a GEMM output in FP32: |gpu - exact| <= 1e-5 * sum_k |a_k w_k| + 1e-6;
  * a BF16 output: within one BF16 ulp of the exact value rounded to BF16,
    or -- where the FP32 bound itself spans more than one ulp (tiny outputs
    near cancellation) -- within that bound plus the BF16 half-ulp.
"""
from __future__ import annotations

import numpy as np
import torch

from oracle import moe, nvfp4

REL = 1e-5
ABS = 1e-6


def gemm_bound(sum_abs: np.ndarray) -> np.ndarray:
    return REL * sum_abs + ABS


def check_f32(gpu: np.ndarray, exact: np.ndarray, sum_abs: np.ndarray, what: str):
    err = np.abs(gpu.astype(np.float64) - exact)
    bound = gemm_bound(sum_abs)
    bad = err > bound
    assert not bad.any(), (f"{what}: {int(bad.sum())} of {bad.size} outside 1e-5*sum|aw|+1e-6; "
                           f"worst err/bound {float((err / bound).max()):.3g}")
    return float((err / np.maximum(sum_abs, 1e-30)).max())


def check_bf16(gpu: np.ndarray, exact: np.ndarray, extra_bound: np.ndarray, what: str):
    """gpu: float32 values of BF16 results; exact: fp64 reference before
    rounding; extra_bound: propagated FP32 error bound of the GPU's value."""
    gpu = gpu.astype(np.float64)
    ref = nvfp4.round_to_bf16(exact).astype(np.float64)
    ulp = nvfp4.bf16_ulp(ref)
    d = np.abs(gpu - ref)
    ok = (d <= ulp) | (np.abs(gpu - exact) <= extra_bound + 0.5 * nvfp4.bf16_ulp(gpu))
    assert ok.all(), (f"{what}: {int((~ok).sum())} of {ok.size} BF16 values off; "
                      f"worst |d|/ulp {float((d / ulp).max()):.3g}")


def to_np(t: torch.Tensor) -> np.ndarray:
    if t.dtype == torch.bfloat16:
        return t.float().cpu().numpy()
    return t.cpu().numpy()


def undo_gate_up_interleave(rows: np.ndarray, n: int) -> np.ndarray:
    """Kernel row order of a fused gate_up weight -> natural order (gate 0..I-1, up I..2I-1)."""
    half = n // 2
    idx = np.empty(n, dtype=np.int64)
    for j in range(half):
        idx[j] = (j // 128) * 256 + (j % 128)
        idx[half + j] = (j // 128) * 256 + 128 + (j % 128)
    return rows[idx]


def sf_rowmajor(flat: torch.Tensor, rows: int, K: int) -> np.ndarray:
    from nvfp4_moe_grouped_token_b200 import ops
    return ops.sf_mma_to_rowmajor(flat.cpu(), rows, K).numpy()


def check_weights_exact(prep, w_cpu: torch.Tensor, gate_up: bool, experts=None):
    """Prepared GPU weights == oracle quantization of each expert's matrix."""
    E, N, K = w_cpu.shape
    q = prep.q.cpu().numpy()
    sf = prep.sf.cpu()
    s_dec = prep.s_dec.cpu().numpy()
    for e in (range(E) if experts is None else experts):
        r = nvfp4.quantize(w_cpu[e].float().numpy(), per_token=False)
        qe = q[e]
        sfe = ops_rowmajor_expert(sf, e, N, K)
        if gate_up:
            qe = undo_gate_up_interleave(qe, N)
            sfe = undo_gate_up_interleave(sfe, N)
        assert np.array_equal(qe, r["q"]), f"weight codes expert {e}"
        assert np.array_equal(sfe, r["sf"]), f"weight scales expert {e}"
        assert s_dec[e] == r["s_dec"][0], f"weight S_dec expert {e}"


def ops_rowmajor_expert(sf_flat_cpu: torch.Tensor, e: int, N: int, K: int) -> np.ndarray:
    per = N * K // 16
    return sf_rowmajor(sf_flat_cpu[e * per:(e + 1) * per], N, K)


def dequant_weights(prep, e: int, gate_up: bool) -> np.ndarray:
    """Oracle dequantization of one expert from the GPU's (bit-exact) weights,
    in natural row order."""
    N, K = prep.N, prep.K
    q = prep.q[e].cpu().numpy()
    sf = ops_rowmajor_expert(prep.sf.cpu(), e, N, K)
    if gate_up:
        q = undo_gate_up_interleave(q, N)
        sf = undo_gate_up_interleave(sf, N)
    return nvfp4.dequantize(q, sf, prep.s_dec[e:e + 1].cpu().numpy())


def swiglu_bound(g, u, tg, tu):
    """Bound on |silu(g')u' - silu(g)u| for |g'-g| <= tg, |u'-u| <= tu
    (|silu'| <= 1.1), plus FP32 epilogue rounding (a few ulps of h)."""
    s = np.abs(moe.silu(g))
    h = np.abs(s * u)
    return 1.1 * tg * (np.abs(u) + tu) + (s + 1.1 * tg) * tu + 8 * 2.0 ** -24 * h + 1e-30
