"""The plain C++ oracle (oracle/nvfp4_oracle.cpp) on the CPU.

Pinned to things other than itself: exhaustive brute force over every BF16
bit pattern for the element and scale codecs, the hand-worked golden examples
under tests/golden/, exact rational GEMMs, a brute-force sort, and a
per-token brute-force formulation of the whole multi-expert layer that uses no
permutation at all.  It is also compared with the numpy oracle (a second,
separately written opinion): bit for bit on every integer result, within fp64
rounding on the GEMMs."""
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

from oracle import cpp, moe, nvfp4

HERE = os.path.dirname(os.path.abspath(__file__))

E2M1_GRID = [Fraction(0), Fraction(1, 2), Fraction(1), Fraction(3, 2), Fraction(2), Fraction(3), Fraction(4),
             Fraction(6)]


def all_bf16_values() -> np.ndarray:
    bits = np.arange(1 << 16, dtype=np.uint32) << 16
    v = bits.view(np.float32)
    return v[np.isfinite(v)]


def brute_nearest_even(a: Fraction, grid) -> int:
    """Index of the nearest grid value (exact rationals), ties to the even
    index, saturating at the top."""
    if a >= grid[-1]:
        return len(grid) - 1
    d = [abs(a - g) for g in grid]
    best = min(d)
    cands = [i for i, x in enumerate(d) if x == best]
    return cands[0] if len(cands) == 1 else [i for i in cands if i % 2 == 0][0]


def test_e2m1_every_bf16_pattern_against_brute_force():
    v = all_bf16_values()
    got = cpp.e2m1_encode(v)
    # group by magnitude: the brute force on the distinct magnitudes
    mags = np.unique(np.abs(v))
    want_mag = {float(m): brute_nearest_even(Fraction(float(m)), E2M1_GRID) for m in mags}
    want = np.array([want_mag[float(abs(x))] | (8 if np.signbit(x) else 0) for x in v], dtype=np.uint8)
    assert np.array_equal(got, want)
    assert np.array_equal(got, nvfp4.e2m1_encode(v))


def test_ue4m3_every_nonnegative_bf16_pattern_against_brute_force():
    v = all_bf16_values()
    v = v[(v >= 0) & ~np.signbit(v)]
    grid = [Fraction(m, 512) if e == 0 else Fraction(8 + m, 8) * Fraction(2) ** (e - 7)
            for e in range(16) for m in range(8)][:127]
    assert grid[-1] == 448
    got = cpp.ue4m3_encode(v)
    want = np.array([brute_nearest_even(Fraction(float(x)), grid) for x in v], dtype=np.uint8)
    assert np.array_equal(got, want)
    assert np.array_equal(got, nvfp4.ue4m3_encode(v))
    # and the independent library cast agrees below saturation
    t = torch.from_numpy(v[v <= 448])
    lib = t.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(cpp.ue4m3_encode(v[v <= 448]), lib)


def test_codes_round_trip():
    assert np.array_equal(cpp.e2m1_encode(cpp.e2m1_decode(np.arange(16))), np.arange(16))
    assert np.array_equal(cpp.ue4m3_encode(cpp.ue4m3_decode(np.arange(127))), np.arange(127))


def test_round_to_bf16_against_torch_and_numpy():
    rng = np.random.default_rng(3)
    f = np.concatenate([rng.standard_normal(200000) * 10.0 ** rng.integers(-40, 38, 200000),
                        [0.0, -0.0, 1e-45, 3.3895e38, 3.3897e38]]).astype(np.float32)
    want = torch.from_numpy(f).to(torch.bfloat16).float().numpy()
    ok = np.isfinite(want)
    assert np.array_equal(cpp.round_to_bf16(f.astype(np.float64))[ok], want[ok])
    d = rng.standard_normal(100000) * 10.0 ** rng.integers(-30, 30, 100000)
    assert np.array_equal(cpp.round_to_bf16(d), nvfp4.round_to_bf16(d))


def _golden(name):
    meta = {}
    rows = {}
    with open(os.path.join(HERE, "golden", name)) as f:
        for line in f:
            if line.startswith("#") or ":" not in line:
                continue
            key, val = line.split(":", 1)
            if key in ("x", "codes"):
                rows.setdefault(key, []).append([float(t) for t in val.split()])
            else:
                meta[key] = val.split()
    return rows, meta


def test_worked_quantization_example():
    rows, meta = _golden("quantize_worked_example.txt")
    x = np.array(rows["x"], dtype=np.float32).reshape(1, -1)
    codes = np.array(rows["codes"], dtype=np.uint8).reshape(-1)
    for per_token in (False, True):
        r = cpp.quantize(x, per_token)
        assert np.array_equal(nvfp4.unpack_nibbles(r["q"]).reshape(-1), codes)
        assert r["sf"].reshape(-1).tolist() == [int(t) for t in meta["sf"]]
        assert r["q"][0, :8].tolist() == [int(t, 16) for t in meta["q_block0_hex"]]
        assert r["amax"][0] == float(meta["amax"][0])


def test_global_scale_reading_golden():
    """R4 at an amax where 1/(2688/amax) and amax/2688 differ in binary32."""
    _, m = _golden("global_scale_reading.txt")
    amax = np.float32(int(m["amax_num"][0]) / int(m["amax_den"][0]))
    s_enc = math.ldexp(int(m["s_enc_mantissa"][0]), int(m["s_enc_exp2"][0]))
    s_dec = math.ldexp(int(m["s_dec_mantissa"][0]), int(m["s_dec_exp2"][0]))
    other = math.ldexp(int(m["other_reading_mantissa"][0]), int(m["other_reading_exp2"][0]))
    assert s_dec != other
    for mod in (cpp, nvfp4):
        enc, dec = mod.global_scales(np.array([amax], np.float32))
        assert float(enc[0]) == s_enc and float(dec[0]) == s_dec, mod.__name__
    # the quantizer stores that S_dec
    x = np.zeros((1, 16), np.float32)
    x[0, 3] = amax
    assert float(cpp.quantize(x, True)["s_dec"][0]) == s_dec


def _hard_inputs(rng, M, K):
    x = rng.standard_normal((M, K)).astype(np.float32)
    x[0] = 0.0                                        # all-zero row
    x[1, :16] = 1e-30                                 # block scale underflows
    if M > 2:
        x[2] *= 1e30                                  # huge values
    if M > 3:
        x[3, ::7] = -x[3, ::7]
    return nvfp4.round_to_bf16(x)


@pytest.mark.parametrize("shape", [(7, 64), (33, 256), (5, 1024)])
@pytest.mark.parametrize("per_token", [False, True])
def test_quantize_matches_numpy_oracle(shape, per_token):
    rng = np.random.default_rng(shape[0] * 100 + shape[1])
    x = _hard_inputs(rng, *shape)
    a = cpp.quantize(x, per_token)
    b = nvfp4.quantize(x, per_token)
    for key in ("q", "sf", "s_dec", "amax"):
        assert np.array_equal(a[key], b[key]), key
    # amax reuse: a given amax is used as is
    amax = np.full(shape[0] if per_token else 1, 3.0, np.float32)
    a = cpp.quantize(x, per_token, amax_in=amax)
    b = nvfp4.quantize(x, per_token, amax_in=amax)
    for key in ("q", "sf", "s_dec", "amax"):
        assert np.array_equal(a[key], b[key]), key
    assert np.array_equal(cpp.dequantize(a["q"], a["sf"], a["s_dec"]),
                          nvfp4.dequantize(b["q"], b["sf"], b["s_dec"]))


def test_permutation_against_sorted():
    rng = np.random.default_rng(11)
    T, k, E = 300, 4, 17
    idx = np.stack([rng.choice(E, k, replace=False) for _ in range(T)]).astype(np.int32)
    p = cpp.permutation(idx, E)
    order = sorted(range(T * k), key=lambda r: (idx.reshape(-1)[r], r // k, r % k))
    assert p["perm"].tolist() == order
    inv = p["inv_perm"].reshape(-1)
    assert np.array_equal(p["perm"][inv], np.arange(T * k))
    counts = np.bincount(idx.reshape(-1), minlength=E)
    assert np.array_equal(np.diff(p["offsets"]), counts)
    assert np.array_equal(np.diff(p["padded_offsets"]), (counts + 127) // 128 * 128)
    q = moe.permutation(idx, E)
    for key in ("offsets", "padded_offsets", "perm", "inv_perm"):
        assert np.array_equal(p[key], q[key]), key


def test_gemm_against_exact_rationals():
    rng = np.random.default_rng(5)
    R, N, K = 6, 5, 48
    qa = cpp.quantize(nvfp4.round_to_bf16(rng.standard_normal((R, K))), True)
    qw = cpp.quantize(nvfp4.round_to_bf16(rng.standard_normal((N, K)) * 0.02), False)
    a = cpp.dequantize(qa["q"], qa["sf"], qa["s_dec"])
    w = cpp.dequantize(qw["q"], qw["sf"], qw["s_dec"])
    out, ab = cpp.gemm_rows(a, w, with_abs=True)
    for r in range(R):
        for n in range(N):
            exact = sum(Fraction(float(a[r, c])) * Fraction(float(w[n, c])) for c in range(K))
            assert abs(Fraction(float(out[r, n])) - exact) <= Fraction(K) * Fraction(2) ** -52 * Fraction(float(ab[r, n]))
            assert ab[r, n] == pytest.approx(sum(abs(float(a[r, c]) * float(w[n, c])) for c in range(K)), rel=1e-14)
    assert np.allclose(out, a @ w.T, rtol=1e-13, atol=1e-300)


def test_swiglu_and_combine_match_numpy():
    rng = np.random.default_rng(9)
    gu = rng.standard_normal((40, 64)) * 5
    # two libm exp implementations: equal to within a few fp64 ulps
    a, b = cpp.swiglu(gu, 32), moe.swiglu(gu, 32)
    assert np.all(np.abs(a - b) <= 1e-15 * np.abs(b))
    g = np.array([[0.0, 50.0, -50.0, 1.0, 1.0, 1.0, 1.0, 2.0]])
    h = cpp.swiglu(g, 4)[0]
    assert h[0] == 0.0 and h[1] == 50.0 and abs(h[2]) < 1e-19
    assert h[3] == pytest.approx(2.0 / (1.0 + math.exp(-1.0)), rel=1e-15)
    T, k, H = 30, 3, 64
    d = nvfp4.round_to_bf16(rng.standard_normal((T * k, H)))
    inv = rng.permutation(T * k).reshape(T, k).astype(np.int32)
    w = rng.random((T, k)).astype(np.float32)
    assert np.array_equal(cpp.combine(d, inv, w), moe.combine(d, inv, w))


def _brute_force_layer(x, idx, topk_w, w_gu, w_dn, per_token):
    """The layer per routed (token, slot), with no permutation: quantize x,
    dequantize, one exactly rounded dot product (math.fsum) per output,
    SwiGLU, BF16, requantize, down, BF16, then the weighted sum over slots in
    slot order.  Per-tensor scales need the amax over every row first."""
    T, H = x.shape
    k = idx.shape[1]
    I = w_gu.shape[1] // 2
    qx = cpp.quantize(x, per_token)
    xh = cpp.dequantize(qx["q"], qx["sf"], qx["s_dec"])

    def wq(w):
        q = cpp.quantize(w, False)
        return cpp.dequantize(q["q"], q["sf"], q["s_dec"])

    wgu = [wq(w_gu[e]) for e in range(w_gu.shape[0])]
    wdn = [wq(w_dn[e]) for e in range(w_dn.shape[0])]
    h = {}
    for t in range(T):
        for j in range(k):
            e = int(idx[t, j])
            g = np.array([math.fsum(xh[t] * wgu[e][n]) for n in range(2 * I)])
            h[t, j] = nvfp4.round_to_bf16(g[:I] / (1.0 + np.exp(-g[:I])) * g[I:])
    amax_all = max(float(np.abs(v).max()) for v in h.values())
    y = np.zeros((T, H), np.float32)
    for t in range(T):
        acc = np.zeros(H)
        for j in range(k):
            e = int(idx[t, j])
            row = h[t, j].reshape(1, -1).astype(np.float32)
            qh = cpp.quantize(row, per_token, amax_in=None if per_token else np.array([amax_all], np.float32))
            hh = cpp.dequantize(qh["q"], qh["sf"], qh["s_dec"])[0]
            dvals = nvfp4.round_to_bf16(np.array([math.fsum(hh * wdn[e][n]) for n in range(H)]))
            acc = acc + float(topk_w[t, j]) * dvals.astype(np.float64)
        y[t] = nvfp4.round_to_bf16(acc)
    return y, h


@pytest.mark.parametrize("per_token", [True, False])
def test_expert_layer_against_per_token_brute_force(per_token):
    """A multi-expert, top-3 layer (8 experts, two of them empty) computed by
    the oracle's permuted grouped path and by the brute force above must agree
    exactly: a wrong token gather, group boundary, gate/up split or combine
    index fails this."""
    rng = np.random.default_rng(21 + per_token)
    T, H, I, E, k = 14, 64, 48, 8, 3
    x = nvfp4.round_to_bf16(rng.standard_normal((T, H)))
    idx = np.stack([rng.choice(6, k, replace=False) for _ in range(T)]).astype(np.int32)   # experts 6, 7 empty
    tw = rng.random((T, k)).astype(np.float32)
    w_gu = nvfp4.round_to_bf16(rng.standard_normal((E, 2 * I, H)) * 0.05)
    w_dn = nvfp4.round_to_bf16(rng.standard_normal((E, H, I)) * 0.05)
    out = cpp.expert_layer(x, idx, tw, w_gu, w_dn, per_token)
    y_bf, h_bf = _brute_force_layer(x, idx, tw, w_gu, w_dn, per_token)
    # h rows in sorted order
    for pos, r in enumerate(out["perm"]):
        assert np.array_equal(out["h"][pos], h_bf[r // k, r % k]), pos
    assert np.array_equal(out["y"], y_bf)


def test_expert_layer_matches_numpy_oracle():
    rng = np.random.default_rng(31)
    T, H, I, E, k = 40, 64, 64, 6, 2
    x = nvfp4.round_to_bf16(rng.standard_normal((T, H)))
    idx = np.stack([rng.choice(E, k, replace=False) for _ in range(T)]).astype(np.int32)
    tw = rng.random((T, k)).astype(np.float32)
    w_gu = nvfp4.round_to_bf16(rng.standard_normal((E, 2 * I, H)) * 0.05)
    w_dn = nvfp4.round_to_bf16(rng.standard_normal((E, H, I)) * 0.05)
    for per_token in (True, False):
        a = cpp.expert_layer(x, idx, tw, w_gu, w_dn, per_token)
        b = moe.expert_layer(x, idx, tw, moe.QuantWeights(w_gu), moe.QuantWeights(w_dn), per_token)
        assert np.array_equal(a["x_q"], b["qx"]["q"]) and np.array_equal(a["x_sf"], b["qx"]["sf"])
        assert np.array_equal(a["perm"], b["perm"]["perm"])
        # fp64 sums in a different order: BF16 results agree but for values
        # within a few fp64 ulps of a BF16 tie
        assert np.mean(a["h"] != b["h"]) < 1e-3
        assert np.mean(a["y"] != b["y"]) < 1e-3
        ulp = nvfp4.bf16_ulp(b["y"])
        assert np.all(np.abs(a["y"] - b["y"]) <= ulp)


def test_backward_against_autograd_and_numpy_oracle():
    """R16 in C++ against float64 torch autograd of the unquantized layer
    written per routed row (no permutation), and against the numpy oracle."""
    from oracle import backward
    rng = np.random.default_rng(41)
    T, H, I, E, k = 10, 32, 16, 5, 2
    x = nvfp4.round_to_bf16(rng.standard_normal((T, H)))
    idx = np.stack([rng.choice(4, k, replace=False) for _ in range(T)]).astype(np.int32)   # expert 4 empty
    tw = rng.random((T, k)).astype(np.float32)
    w_gu = nvfp4.round_to_bf16(rng.standard_normal((E, 2 * I, H)) * 0.2)
    w_dn = nvfp4.round_to_bf16(rng.standard_normal((E, H, I)) * 0.2)
    dy = nvfp4.round_to_bf16(rng.standard_normal((T, H)))
    got = cpp.expert_layer_backward(x, idx, tw, w_gu, w_dn, dy)

    xt = torch.tensor(x, dtype=torch.float64, requires_grad=True)
    wt = torch.tensor(tw, dtype=torch.float64, requires_grad=True)
    gut = torch.tensor(w_gu, dtype=torch.float64, requires_grad=True)
    dnt = torch.tensor(w_dn, dtype=torch.float64, requires_grad=True)
    y = torch.zeros(T, H, dtype=torch.float64)
    for t in range(T):
        for j in range(k):
            e = int(idx[t, j])
            g_u = gut[e] @ xt[t]
            h = torch.nn.functional.silu(g_u[:I]) * g_u[I:]
            y[t] = y[t] + wt[t, j] * (dnt[e] @ h)
    (y * torch.tensor(dy, dtype=torch.float64)).sum().backward()
    for key, ref in (("dx", xt.grad), ("dw", wt.grad), ("dw_gate_up", gut.grad), ("dw_down", dnt.grad)):
        assert np.allclose(got[key], ref.numpy(), rtol=1e-10, atol=1e-12), key
    ref_np = backward.expert_layer_backward(x, idx, tw, w_gu, w_dn, dy)
    for key in ("dx", "dw", "dw_gate_up", "dw_down"):
        assert np.allclose(got[key], ref_np[key], rtol=1e-12, atol=1e-14), key
    assert np.all(got["dw_gate_up"][4] == 0) and np.all(got["dw_down"][4] == 0)


def test_swiglu_backward_closed_form():
    g = np.array([[0.0, 2.0, -3.0, 5.0, 0.5, 1.0]])   # I = 3: gate 0, 2, -3; up 5, .5, 1
    dhp = np.array([[1.0, -2.0, 0.25]])
    dgu, h = cpp.swiglu_backward(g, dhp, np.array([0.5]))
    for i in range(3):
        gg, u, dh = g[0, i], g[0, 3 + i], 0.5 * dhp[0, i]
        s = 1.0 / (1.0 + math.exp(-gg))
        assert dgu[0, i] == pytest.approx(dh * u * (s + gg * s * (1 - s)), rel=1e-14, abs=1e-300)
        assert dgu[0, 3 + i] == pytest.approx(dh * gg * s, rel=1e-14, abs=1e-300)
        assert h[0, i] == pytest.approx(gg * s * u, rel=1e-14, abs=1e-300)
    assert dgu[0, 0] == 0.5 * 1.0 * 5.0 * 0.5     # silu'(0) = 1/2


def test_w4a16_layer_against_per_token_brute_force():
    """R19 (BF16 activations, NVFP4 weights): the oracle's permuted grouped
    path against a per-(token, slot) brute force with exactly rounded dot
    products, and against the W4A4 layer's weight quantization (the same
    dequantized weights)."""
    rng = np.random.default_rng(61)
    T, H, I, E, k = 12, 64, 48, 6, 2
    x = nvfp4.round_to_bf16(rng.standard_normal((T, H)))
    idx = np.stack([rng.choice(5, k, replace=False) for _ in range(T)]).astype(np.int32)   # expert 5 empty
    tw = rng.random((T, k)).astype(np.float32)
    w_gu = nvfp4.round_to_bf16(rng.standard_normal((E, 2 * I, H)) * 0.05)
    w_dn = nvfp4.round_to_bf16(rng.standard_normal((E, H, I)) * 0.05)
    out = cpp.expert_layer_w4a16(x, idx, tw, w_gu, w_dn)

    def wq(w):
        q = cpp.quantize(w, False)
        return cpp.dequantize(q["q"], q["sf"], q["s_dec"])

    wgu = [wq(w_gu[e]) for e in range(E)]
    wdn = [wq(w_dn[e]) for e in range(E)]
    y = np.zeros((T, H), np.float32)
    for t in range(T):
        acc = np.zeros(H)
        for j in range(k):
            e = int(idx[t, j])
            g = np.array([math.fsum(x[t].astype(np.float64) * wgu[e][n]) for n in range(2 * I)])
            h = nvfp4.round_to_bf16(g[:I] / (1.0 + np.exp(-g[:I])) * g[I:]).astype(np.float64)
            pos = int(out["inv_perm"][t, j])
            assert np.array_equal(out["h"][pos], h.astype(np.float32)), (t, j)
            d = nvfp4.round_to_bf16(np.array([math.fsum(h * wdn[e][n]) for n in range(H)]))
            assert np.array_equal(out["d"][pos], d), (t, j)
            acc = acc + float(tw[t, j]) * d.astype(np.float64)
        y[t] = nvfp4.round_to_bf16(acc)
    assert np.array_equal(out["y"], y)


def test_mxfp8_hand_derived_codes():
    """R17 on hand-derived values.  Block amax 1.9: s = floor(log2 1.9) - 8 =
    -8 (E8M0 code 119), so elements are scaled by 256:
      1.9   -> 486.4 > 448: saturates to 448 = E4M3 (e 15, m 6) = 0x7E
      0.3   -> 76.8: binade [64, 128) in steps of 8, nearest 80 = (e 13, m 2) = 0x6A
      -0.001 -> -0.256: binade [0.25, 0.5) in steps of 1/32, nearest 0.25 = (e 5, m 0), sign -> 0xA8
      1.0   -> 256 = (e 15, m 0) = 0x78
      -1e-6 -> -2.56e-4 < half the least subnormal 2^-9: -0 = 0x80
    An all-zero block takes s = -127 (code 0) and +0 codes."""
    x = np.zeros((1, 64), np.float32)
    x[0, :5] = [1.9, 0.3, -0.001, 1.0, -1e-6]
    codes, scales = cpp.mxfp8_quantize(x)
    assert list(codes[0, :5]) == [0x7E, 0x6A, 0xA8, 0x78, 0x80]
    assert not codes[0, 5:32].any() and not codes[0, 32:].any()
    assert list(scales[0]) == [119, 0]
    back = cpp.mxfp8_dequantize(codes, scales)
    assert list(back[0, :5]) == [448 / 256, 80 / 256, -0.25 / 256, 1.0, 0.0]
    assert math.copysign(1.0, back[0, 4]) == -1.0


def test_mxfp8_matches_the_numpy_reading():
    """The C++ and numpy statements of R17 agree code for code, on normal
    data, wide dynamic range, BF16 subnormals and all-zero blocks (the numpy
    one is pinned on its own in test_oracle_mxfp8.py)."""
    from oracle import mxfp8
    rng = np.random.default_rng(71)
    x = rng.standard_normal((64, 256)) * np.exp2(rng.integers(-30, 30, (64, 1)))
    x[3] = 0.0
    x[5, :32] = rng.standard_normal(32) * 2.0 ** -130
    x[7, 7] = 3e38
    x = nvfp4.round_to_bf16(x).astype(np.float32)
    c1, s1 = cpp.mxfp8_quantize(x)
    c2, s2 = mxfp8.quantize(x)
    assert np.array_equal(c1, c2) and np.array_equal(s1, s2)
    assert np.array_equal(cpp.mxfp8_dequantize(c1, s1), mxfp8.dequantize(c2, s2))


def test_w4a8_layer_against_per_token_brute_force():
    """R20 (NVFP4 weights, MXFP8 x and h): the grouped path against a
    per-(token, slot) loop with exactly rounded dot products."""
    rng = np.random.default_rng(62)
    T, H, I, E, k = 10, 64, 64, 5, 2
    x = nvfp4.round_to_bf16(rng.standard_normal((T, H)))
    idx = np.stack([rng.choice(4, k, replace=False) for _ in range(T)]).astype(np.int32)   # expert 4 empty
    tw = rng.random((T, k)).astype(np.float32)
    w_gu = nvfp4.round_to_bf16(rng.standard_normal((E, 2 * I, H)) * 0.05)
    w_dn = nvfp4.round_to_bf16(rng.standard_normal((E, H, I)) * 0.05)
    out = cpp.expert_layer_w4a8(x, idx, tw, w_gu, w_dn)

    def wq(w):
        q = cpp.quantize(w, False)
        return cpp.dequantize(q["q"], q["sf"], q["s_dec"])

    def qdq(v):
        return cpp.mxfp8_dequantize(*cpp.mxfp8_quantize(np.asarray(v, np.float32)[None, :]))[0]

    y = np.zeros((T, H), np.float32)
    for t in range(T):
        xq = qdq(x[t])
        acc = np.zeros(H)
        for j in range(k):
            e = int(idx[t, j])
            wgu, wdn = wq(w_gu[e]), wq(w_dn[e])
            g = np.array([math.fsum(xq * wgu[n]) for n in range(2 * I)])
            h = nvfp4.round_to_bf16(g[:I] / (1.0 + np.exp(-g[:I])) * g[I:])
            pos = int(out["inv_perm"][t, j])
            assert np.array_equal(out["h"][pos], h.astype(np.float32)), (t, j)
            hq = qdq(h)
            d = nvfp4.round_to_bf16(np.array([math.fsum(hq * wdn[n]) for n in range(H)]))
            assert np.array_equal(out["d"][pos], d), (t, j)
            acc = acc + float(tw[t, j]) * d.astype(np.float64)
        y[t] = nvfp4.round_to_bf16(acc)
    assert np.array_equal(out["y"], y)
