"""Pins of the oracle's number formats against things other than the oracle:
the format definitions (round trips, the midpoint table), a library routine
(torch's float8_e4m3fn cast, torch's bfloat16 cast), and brute force."""
import math
from fractions import Fraction

import numpy as np
import pytest
import torch

from oracle import nvfp4

pytestmark = pytest.mark.filterwarnings("ignore")


def test_e2m1_all_codes_round_trip():
    codes = np.arange(16, dtype=np.uint8)
    vals = nvfp4.e2m1_decode(codes)
    # -0 must be given as a negative zero to come back as 0x8
    y = np.where(codes == 8, np.float32(-0.0), vals.astype(np.float32))
    assert np.array_equal(nvfp4.e2m1_encode(y), codes)


def test_e2m1_value_set_is_the_format_definition():
    # E2M1: 1 sign, 2 exponent (bias 1), 1 mantissa bit; subnormal at e=0.
    vals = []
    for e in range(4):
        for m in range(2):
            vals.append(m * 0.5 if e == 0 else (1 + m / 2) * 2.0 ** (e - 1))
    assert vals == list(nvfp4.E2M1_MAGNITUDES)


@pytest.mark.parametrize("y,code", [
    (0.25, 0), (0.75, 2), (1.25, 2), (1.75, 4), (2.5, 4), (3.5, 6), (5.0, 6),
    (0.2499, 0), (0.2501, 1), (5.01, 7), (6.0, 7), (7.0, 7), (1e30, 7),
    (-0.25, 8), (-5.0, 14), (-100.0, 15), (-0.1, 8), (0.0, 0),
])
def test_e2m1_midpoints_and_saturation(y, code):
    assert int(nvfp4.e2m1_encode(np.array([y], np.float32))[0]) == code


def test_e2m1_brute_force_nearest_even():
    rng = np.random.default_rng(7)
    y = np.concatenate([rng.uniform(-7, 7, 20000), rng.normal(0, 2, 20000)]).astype(np.float32)
    got = nvfp4.e2m1_encode(y)
    for yi, gi in zip(y[:4000], got[:4000]):
        a = Fraction(float(abs(yi)))
        grid = [Fraction(0), Fraction(1, 2), Fraction(1), Fraction(3, 2), Fraction(2), Fraction(3), Fraction(4), Fraction(6)]
        dist = [abs(a - g) for g in grid]
        best = min(dist)
        cands = [i for i, d in enumerate(dist) if d == best]
        idx = cands[0] if len(cands) == 1 else [c for c in cands if c % 2 == 0][0]
        want = idx | (8 if math.copysign(1.0, float(yi)) < 0 else 0)
        assert int(gi) == want, (float(yi), int(gi), want)


def test_ue4m3_all_codes_round_trip():
    codes = np.arange(127, dtype=np.uint8)
    vals = nvfp4.ue4m3_decode(codes).astype(np.float32)
    assert np.array_equal(nvfp4.ue4m3_encode(vals), codes)


def test_ue4m3_matches_torch_float8_e4m3fn_cast():
    """torch's CPU cast to float8_e4m3fn rounds to nearest even; in the finite
    range [0, 448] it must agree with the oracle bit for bit."""
    rng = np.random.default_rng(11)
    v = np.concatenate([
        rng.uniform(0, 448, 200000),
        np.exp2(rng.uniform(-12, 9, 200000)),
        nvfp4.UE4M3_VALUES,                                   # exact codes
        (nvfp4.UE4M3_VALUES[1:] + nvfp4.UE4M3_VALUES[:-1]) / 2,  # exact midpoints
    ]).astype(np.float32)
    v = v[v <= 448]
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(nvfp4.ue4m3_encode(v), ref)


def test_ue4m3_saturates():
    v = np.array([448, 449, 463.9, 464, 1000, 3.4e38], np.float32)
    assert np.all(nvfp4.ue4m3_encode(v) == 126)


def test_ue4m3_subnormals_and_underflow():
    v = np.array([2.0 ** -9, 2.0 ** -10, 1.5 * 2.0 ** -10, 2.0 ** -11, 7 * 2.0 ** -9, 2.0 ** -6], np.float32)
    assert list(nvfp4.ue4m3_encode(v)) == [1, 0, 1, 0, 7, 8]


def test_bf16_rounding_matches_torch_on_fp32_inputs():
    rng = np.random.default_rng(3)
    v = np.concatenate([rng.normal(0, 1, 100000), rng.normal(0, 1e-30, 1000),
                        np.exp2(rng.uniform(-140, 120, 10000))]).astype(np.float32)
    # exact ties: bf16 value + half its ulp
    b = torch.from_numpy(v[:1000]).to(torch.bfloat16).float().numpy()
    ties = (b.astype(np.float64) + nvfp4.bf16_ulp(b) / 2).astype(np.float32)
    v = np.concatenate([v, ties])
    ref = torch.from_numpy(v).to(torch.bfloat16).float().numpy()
    assert np.array_equal(nvfp4.round_to_bf16(v.astype(np.float64)), ref)


def test_bf16_rounding_is_direct_from_fp64():
    # 1 + 2^-8 + 2^-30 is above the BF16 midpoint 1 + 2^-8: must round up,
    # although a detour through fp32 would land on the tie and round down.
    v = np.array([1 + 2.0 ** -8 + 2.0 ** -30], np.float64)
    assert nvfp4.round_to_bf16(v)[0] == np.float32(1 + 2.0 ** -7)


def test_nibble_packing_low_first():
    codes = np.arange(16, dtype=np.uint8).reshape(1, 16)
    q = nvfp4.pack_nibbles(codes)
    assert list(q[0]) == [0x10, 0x32, 0x54, 0x76, 0x98, 0xBA, 0xDC, 0xFE]
    assert np.array_equal(nvfp4.unpack_nibbles(q), codes)
