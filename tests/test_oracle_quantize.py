"""Pins of the oracle's NVFP4 quantizer: a hand-worked example, closed forms
(power-of-two scale invariance, sign symmetry, zero tensor), the block-scale
definition recomputed in exact rationals, and the error bound of the format."""
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

from oracle import nvfp4

HERE = os.path.dirname(os.path.abspath(__file__))


def _bf16(a):
    return torch.from_numpy(np.asarray(a, np.float32)).to(torch.bfloat16).float().numpy()


def _load_golden():
    rows = {"x": [], "codes": []}
    meta = {}
    with open(os.path.join(HERE, "golden", "quantize_worked_example.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, val = line.split(":", 1)
            if key in rows:
                rows[key].append([float(v) for v in val.split()])
            else:
                meta[key] = val.split()
    return rows, meta


@pytest.mark.parametrize("per_token", [False, True])
def test_worked_example(per_token):
    rows, meta = _load_golden()
    x = np.array([sum(rows["x"], [])], np.float32)
    x[0, 8] = np.float32(-0.0)
    x[0, 24] = np.float32(-0.0)
    assert nvfp4.is_bf16_exact(x)
    r = nvfp4.quantize(x, per_token=per_token)
    codes = nvfp4.unpack_nibbles(r["q"])[0]
    assert list(codes) == [int(c) for c in sum(rows["codes"], [])]
    assert list(r["sf"][0]) == [int(v) for v in meta["sf"]]
    assert [f"{b:02x}" for b in r["q"][0, :8]] == meta["q_block0_hex"]
    assert float(r["amax"][0]) == float(meta["amax"][0])
    s_enc, s_dec = nvfp4.global_scales(r["amax"])
    assert float(s_enc[0]) == float(meta["s_enc"][0])
    assert r["s_dec"][0] == np.float32(1.0) / np.float32(448.0)


def test_zero_tensor():
    r = nvfp4.quantize(np.zeros((3, 64), np.float32), per_token=False)
    assert r["amax"][0] == 0 and r["s_dec"][0] == 1.0
    assert not r["q"].any() and not r["sf"].any()


def test_all_zero_block_in_live_tensor():
    x = _bf16(np.random.default_rng(0).normal(size=(2, 64)))
    x[1, 16:32] = 0
    r = nvfp4.quantize(x, per_token=True)
    assert r["sf"][1, 1] == 0
    assert not nvfp4.unpack_nibbles(r["q"])[1, 16:32].any()


@pytest.mark.parametrize("per_token", [False, True])
@pytest.mark.parametrize("m", [-20, -3, 1, 7, 30])
def test_power_of_two_scale_invariance(per_token, m):
    """x * 2^m: every step of R4-R6 scales exactly, so codes and sf are equal
    and S_dec scales by exactly 2^m (away from over/underflow)."""
    rng = np.random.default_rng(5)
    x = _bf16(rng.normal(size=(8, 128)))
    a = nvfp4.quantize(x, per_token)
    b = nvfp4.quantize((x * np.float32(2.0 ** m)).astype(np.float32), per_token)
    assert np.array_equal(a["q"], b["q"]) and np.array_equal(a["sf"], b["sf"])
    assert np.array_equal(b["s_dec"], (a["s_dec"] * np.float32(2.0 ** m)).astype(np.float32))


def test_sign_symmetry():
    rng = np.random.default_rng(9)
    x = _bf16(rng.normal(size=(16, 256)))
    a = nvfp4.unpack_nibbles(nvfp4.quantize(x, False)["q"])
    b = nvfp4.unpack_nibbles(nvfp4.quantize(-x, False)["q"])
    assert np.array_equal(a ^ 8, b)


def test_block_scale_definition_in_exact_rationals():
    """sf is the UE4M3 value nearest (ties even) to fl32(fl32(bamax/6) * S_enc),
    recomputed here with Fractions and an explicit search of all 127 codes."""
    rng = np.random.default_rng(13)
    x = _bf16(rng.normal(size=(4, 256)) * np.exp2(rng.integers(-8, 8, size=(4, 1))))
    r = nvfp4.quantize(x, per_token=True)
    s_enc, _ = nvfp4.global_scales(r["amax"])
    grid = [Fraction(float(v)) for v in nvfp4.UE4M3_VALUES]
    for i in range(4):
        for b in range(16):
            bamax = np.float32(np.abs(x[i, 16 * b:16 * b + 16]).max())
            t = Fraction(float(np.float32(np.float32(bamax / np.float32(6)) * s_enc[i])))
            if t >= 448:
                want = 126
            else:
                d = [abs(t - g) for g in grid]
                best = min(d)
                c = [j for j, v in enumerate(d) if v == best]
                want = c[0] if len(c) == 1 else [j for j in c if j % 2 == 0][0]
            assert r["sf"][i, b] == want


def test_block_with_amax_has_full_scale():
    """The block holding the tensor amax maps to sf = 448 (6 * 448 * S_dec ~ amax)."""
    rng = np.random.default_rng(17)
    x = _bf16(rng.normal(size=(32, 512)))
    r = nvfp4.quantize(x, per_token=False)
    i, j = np.unravel_index(np.argmax(np.abs(x)), x.shape)
    assert nvfp4.ue4m3_decode(r["sf"][i, j // 16]) == 448.0
    xh = nvfp4.dequantize(r["q"], r["sf"], r["s_dec"])
    assert abs(abs(xh[i, j]) - abs(x[i, j])) <= abs(x[i, j]) * 2 ** -20


@pytest.mark.parametrize("per_token", [False, True])
def test_dequantize_error_bound(per_token):
    """|x_hat - x| <= (half the widest E2M1 gap, 1.0) * sf * S_dec, plus the
    overshoot when sf rounded down (y up to 6 * 17/16 saturating to 6)."""
    rng = np.random.default_rng(19)
    x = _bf16(rng.normal(size=(64, 256)) * np.exp2(rng.integers(-4, 4, size=(64, 1))))
    r = nvfp4.quantize(x, per_token)
    xh = nvfp4.dequantize(r["q"], r["sf"], r["s_dec"])
    step = np.repeat(nvfp4.ue4m3_decode(r["sf"]), 16, axis=1) * r["s_dec"].astype(np.float64).reshape(-1, 1)
    assert np.all(np.abs(xh - x) <= 1.0 * step + 1e-30)
    # and the reconstruction is close in relative terms over the tensor
    assert np.linalg.norm(xh - x) / np.linalg.norm(x) < 0.12


def test_per_token_rows_are_independent():
    rng = np.random.default_rng(23)
    x = _bf16(rng.normal(size=(10, 128)))
    full = nvfp4.quantize(x, per_token=True)
    for i in range(10):
        one = nvfp4.quantize(x[i:i + 1], per_token=True)
        assert np.array_equal(one["q"][0], full["q"][i]) and np.array_equal(one["sf"][0], full["sf"][i])
        assert one["s_dec"][0] == full["s_dec"][i]


def test_amax_reuse_equals_recompute():
    rng = np.random.default_rng(29)
    x = _bf16(rng.normal(size=(16, 64)))
    a = nvfp4.quantize(x, per_token=False)
    b = nvfp4.quantize(x, per_token=False, amax_in=a["amax"])
    assert all(np.array_equal(a[k], b[k]) for k in ("q", "sf", "s_dec"))


def test_global_scale_overflow_clamps():
    s_enc, s_dec = nvfp4.global_scales(np.array([1e-38, 0.0], np.float32))
    assert s_enc[0] == np.finfo(np.float32).max and s_enc[1] == 1.0
    assert s_dec[0] == np.float32(1) / np.finfo(np.float32).max
