"""Pins of the oracle's permutation, grouped GEMM, SwiGLU and combine:
brute force on tiny inputs, exact rational arithmetic, textbook values and
invariants."""
import math
from fractions import Fraction

import numpy as np
import pytest
import torch

from oracle import moe, nvfp4
from nvfp4_moe_grouped_token_b200 import workloads


def _bf16(a):
    return torch.from_numpy(np.asarray(a, np.float32)).to(torch.bfloat16).float().numpy()


# --------------------------------------------------------- permutation ----

@pytest.mark.parametrize("T,k,E", [(1, 1, 1), (7, 2, 4), (33, 3, 5), (64, 8, 128), (200, 4, 9)])
def test_permutation_brute_force(T, k, E):
    rng = np.random.default_rng(T * 100 + E)
    idx = np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32)
    p = moe.permutation(idx, E)
    rows = sorted(((int(idx[t, j]), t, j) for t in range(T) for j in range(k)))
    assert [t * k + j for _, t, j in rows] == list(p["perm"])
    for r, (e, t, j) in enumerate(rows):
        assert p["inv_perm"][t, j] == r
    counts = [sum(1 for e, _, _ in rows if e == x) for x in range(E)]
    assert list(p["counts"]) == counts
    assert list(p["offsets"]) == [0] + list(np.cumsum(counts))
    pad = [0]
    for c in counts:
        pad.append(pad[-1] + (c + 127) // 128 * 128)
    assert list(p["padded_offsets"]) == pad


def test_permutation_invariants_large():
    cfg = workloads.CONFIGS["moe30b"]
    idx, _ = workloads.routing(workloads.scaled(cfg, T=2048))
    p = moe.permutation(idx.numpy(), cfg.E)
    R = 2048 * cfg.k
    perm, inv = p["perm"], p["inv_perm"].reshape(-1)
    assert np.array_equal(perm[inv], np.arange(R)) and np.array_equal(inv[perm], np.arange(R))
    assert np.all(np.diff(p["offsets"]) >= 0) and p["offsets"][-1] == R
    assert np.all(p["padded_offsets"] % 128 == 0)
    e_of = moe.expert_of_rows(p["offsets"])
    assert np.array_equal(idx.numpy().reshape(-1)[perm], e_of)
    for e in range(cfg.E):
        seg = perm[p["offsets"][e]:p["offsets"][e + 1]]
        assert np.all(np.diff(seg) > 0)
    pr = moe.padded_rows(p)
    assert np.all(np.diff(pr) > 0)


def test_permutation_rejects_bad_index():
    with pytest.raises(ValueError):
        moe.permutation(np.array([[0, 5]], np.int32), 4)


# -------------------------------------------------------------- GEMM ----

def _exact_value(code, sf, s_dec):
    mag = [Fraction(0), Fraction(1, 2), Fraction(1), Fraction(3, 2), Fraction(2), Fraction(3), Fraction(4), Fraction(6)][code & 7]
    e, m = sf >> 3, sf & 7
    scale = Fraction(m, 2 ** 9) if e == 0 else (1 + Fraction(m, 8)) * Fraction(2) ** (e - 7)
    v = mag * scale * Fraction(float(s_dec))
    return -v if code & 8 else v


@pytest.mark.parametrize("M,N,K", [(3, 5, 16), (4, 7, 64), (9, 3, 128)])
def test_gemm_exact_rationals(M, N, K):
    """Dequantize + GEMM in exact rationals from the codes, compared with the
    oracle's fp64 path: the fp64 result must be the exact sum rounded (within
    the fp64 summation error, K ulps)."""
    rng = np.random.default_rng(M * N * K)
    a = _bf16(rng.normal(size=(M, K)))
    w = _bf16(rng.normal(0, 0.02, size=(N, K)))
    qa = nvfp4.quantize(a, per_token=True)
    qw = nvfp4.quantize(w, per_token=False)
    got = moe.grouped_gemm(nvfp4.dequantize(qa["q"], qa["sf"], qa["s_dec"]), np.array([0, M]),
                           lambda e: nvfp4.dequantize(qw["q"], qw["sf"], qw["s_dec"]))
    ca, cw = nvfp4.unpack_nibbles(qa["q"]), nvfp4.unpack_nibbles(qw["q"])
    for i in range(M):
        for n in range(N):
            s = Fraction(0)
            sabs = Fraction(0)
            for kk in range(K):
                va = _exact_value(int(ca[i, kk]), int(qa["sf"][i, kk // 16]), qa["s_dec"][i])
                vw = _exact_value(int(cw[n, kk]), int(qw["sf"][n, kk // 16]), qw["s_dec"][0])
                s += va * vw
                sabs += abs(va * vw)
            assert abs(Fraction(got[i, n]) - s) <= sabs * K * Fraction(2) ** -52


def test_grouped_equals_dense_for_one_expert():
    rng = np.random.default_rng(31)
    a = rng.normal(size=(37, 64))
    w = rng.normal(size=(24, 64))
    g = moe.grouped_gemm(a, np.array([0, 37]), lambda e: w)
    assert np.array_equal(g, a @ w.T)


def test_grouped_gemm_uses_each_experts_weight():
    rng = np.random.default_rng(37)
    a = rng.normal(size=(10, 32))
    ws = [rng.normal(size=(6, 32)) for _ in range(3)]
    off = np.array([0, 4, 4, 10])                # expert 1 is empty
    g = moe.grouped_gemm(a, off, lambda e: ws[e])
    assert np.allclose(g[:4], a[:4] @ ws[0].T, rtol=0, atol=1e-12)
    assert np.allclose(g[4:], a[4:] @ ws[2].T, rtol=0, atol=1e-12)


# ----------------------------------------------------------- SwiGLU ----

def test_silu_textbook_values():
    g = np.array([0.0, 1.0, -1.0, 20.0, -40.0, 800.0, -800.0])
    s = moe.silu(g)
    assert s[0] == 0.0
    assert abs(s[1] - 0.7310585786300049) < 1e-15        # 1 / (1 + e^-1)
    assert abs(s[2] - (-0.2689414213699951)) < 1e-15     # -1 / (1 + e)
    assert abs(s[3] - 20.0) < 1e-7
    assert abs(s[4]) < 1e-15
    assert s[5] == 800.0 and s[6] == 0.0 or abs(s[6]) < 1e-300


def test_silu_against_math_exp():
    xs = np.linspace(-30, 30, 1001)
    ref = np.array([x / (1 + math.exp(-x)) for x in xs])
    assert np.max(np.abs(moe.silu(xs) - ref)) < 1e-13


def test_swiglu_splits_gate_and_up():
    gu = np.array([[1.0, 2.0, 10.0, 100.0]])
    h = moe.swiglu(gu, 2)
    assert np.allclose(h, [[moe.silu(1.0) * 10.0, moe.silu(2.0) * 100.0]], rtol=1e-15)


# ----------------------------------------------------------- combine ----

def test_combine_single_slot_unit_weight_is_identity():
    rng = np.random.default_rng(41)
    d = _bf16(rng.normal(size=(12, 40)))
    inv = np.arange(12).reshape(12, 1)
    y = moe.combine(d, inv, np.ones((12, 1), np.float32))
    assert np.array_equal(y, d)


def test_combine_is_weighted_sum():
    d = _bf16(np.array([[1.0, 2.0], [3.0, -4.0], [0.5, 0.25]]))
    inv = np.array([[2, 0], [1, 2]])
    w = np.array([[0.5, 0.25], [1.0, 2.0]], np.float32)
    y = moe.combine(d, inv, w)
    assert np.array_equal(y, np.array([[0.5, 0.625], [4.0, -3.5]], np.float32))


def test_combine_slot_order_irrelevant_in_fp64_for_exact_sums():
    rng = np.random.default_rng(43)
    d = _bf16(rng.integers(-8, 8, size=(8, 16)).astype(np.float32))
    inv = np.array([[0, 1, 2], [3, 4, 5]])
    w = np.array([[0.5, 0.25, 0.125], [1, 2, 4]], np.float32)
    a = moe.combine(d, inv, w)
    b = moe.combine(d, inv[:, ::-1], w[:, ::-1])
    assert np.array_equal(a, b)


# ------------------------------------------------------------- layer ----

def test_layer_tiny_end_to_end_consistency():
    """The layer helper equals the composition of its stages, and with a
    single expert and k=1 it is the dense two-GEMM MLP."""
    cfg = workloads.LayerConfig("t", T=20, H=64, I=32, E=1, k=1, seed=9, routing="identity")
    inp = workloads.layer_inputs(cfg)
    x = inp["x"].float().numpy()
    wgu = moe.QuantWeights(inp["w_gate_up"].float().numpy())
    wdn = moe.QuantWeights(inp["w_down"].float().numpy())
    out = moe.expert_layer(x, inp["topk_idx"].numpy(), inp["topk_w"].numpy(), wgu, wdn, per_token=True)
    qx = nvfp4.quantize(x, per_token=True)
    xh = nvfp4.dequantize(qx["q"], qx["sf"], qx["s_dec"])
    gu = xh @ wgu.dequant(0).T
    h = nvfp4.round_to_bf16(moe.silu(gu[:, :32]) * gu[:, 32:])
    assert np.array_equal(out["h"], h)
    qh = nvfp4.quantize(h, per_token=True)
    d = nvfp4.round_to_bf16(nvfp4.dequantize(qh["q"], qh["sf"], qh["s_dec"]) @ wdn.dequant(0).T)
    assert np.array_equal(out["y"], d)
