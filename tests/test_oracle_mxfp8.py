"""Pins of the MXFP8 oracle (reading R17) against facts outside its code:
torch's float8_e4m3fn cast for the element rounding, exact power-of-two
scales from the binary exponent, the error bound of a 3-bit mantissa, and the
special cases (zero blocks, values already on the grid, saturation)."""
import numpy as np
import torch

from oracle import mxfp8


def _bf16(shape, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(shape, generator=g) * scale).to(torch.bfloat16).float().numpy().astype(np.float64)


def test_scales_are_powers_of_two_putting_the_block_max_in_256_512():
    x = _bf16((64, 256), 1) * np.exp2(np.random.default_rng(0).integers(-20, 20, size=(64, 1)))
    _, sc = mxfp8.quantize(x)
    s = sc.astype(np.int64) - 127
    amax = np.abs(x.reshape(64, 8, 32)).max(axis=2)
    ratio = amax / np.ldexp(1.0, s)
    assert np.all((ratio >= 256) & (ratio < 512))


def test_elements_round_like_torch_float8_e4m3fn_inside_the_range():
    x = _bf16((32, 512), 2, scale=3.0)
    codes, sc = mxfp8.quantize(x)
    s = sc.astype(np.int64) - 127
    v = x.reshape(32, 16, 32) / np.ldexp(1.0, s)[:, :, None]
    inside = np.abs(v) <= 448
    ref = torch.tensor(v[inside]).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(codes.reshape(32, 16, 32)[inside], ref)


def test_saturation_above_448():
    # a block whose max scales to 480 (2^8 <= 480 < 2^9) saturates to 448
    x = np.zeros((1, 32))
    x[0, 0] = 480.0
    x[0, 1] = -470.0
    codes, sc = mxfp8.quantize(x)
    assert sc[0, 0] == 127                         # s = 0
    deq = mxfp8.dequantize(codes, sc)
    assert deq[0, 0] == 448.0 and deq[0, 1] == -448.0


def test_relative_error_of_normal_elements_is_at_most_half_an_ulp():
    x = _bf16((16, 1024), 3)
    codes, sc = mxfp8.quantize(x)
    deq = mxfp8.dequantize(codes, sc)
    s = np.repeat(sc.astype(np.int64) - 127, 32, axis=1)
    normal = np.abs(x) >= np.ldexp(2.0 ** -6, s)            # E4M3 normals start at 2^-6
    not_sat = np.abs(x) <= np.ldexp(448.0, s)
    m = normal & not_sat
    assert np.all(np.abs(deq[m] - x[m]) <= 2.0 ** -4 * np.abs(x[m]))


def test_grid_values_and_zero_blocks_round_trip_exactly():
    grid = np.array([0.0, 2.0 ** -9, 0.015625, 1.0, 1.125, 240.0, 256.0, 448.0, -3.5, -448.0])
    x = np.zeros((2, 64))
    x[0, :len(grid)] = grid                          # block max 448 -> s = 0
    codes, sc = mxfp8.quantize(x)
    deq = mxfp8.dequantize(codes, sc)
    assert np.array_equal(deq[0, :len(grid)], grid)
    assert sc[1, 0] == 0 and sc[1, 1] == 0 and not codes[1].any()   # all-zero blocks: s = -127, +0 codes


def test_negative_values_that_round_to_zero_keep_the_sign():
    x = np.zeros((1, 32))
    x[0, 0] = 448.0
    x[0, 1] = -2.0 ** -11                            # below half the smallest subnormal at s = 0
    codes, _ = mxfp8.quantize(x)
    assert codes[0, 1] == 0x80


def test_mxfp4_scales_put_the_block_max_in_4_8_and_round_to_the_e2m1_grid():
    w = _bf16((32, 256), 5, scale=0.02)
    codes, sc = mxfp8.quantize_mxfp4(w)
    s = sc.astype(np.int64) - 127
    amax = np.abs(w.reshape(32, 8, 32)).max(axis=2)
    ratio = amax / np.ldexp(1.0, s)
    assert np.all((ratio >= 4) & (ratio < 8))
    deq = mxfp8.dequantize_mxfp4(codes, sc)
    # brute force: every element is the nearest point of the scaled E2M1 grid (saturating at 6)
    grid = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
    v = np.abs(w.reshape(32, 8, 32) / np.ldexp(1.0, s)[:, :, None]).reshape(-1)
    got = np.abs(deq.reshape(32, 8, 32) / np.ldexp(1.0, s)[:, :, None]).reshape(-1)
    dist = np.abs(v[:, None] - grid[None, :])
    best = dist.min(axis=1)
    assert np.all(np.abs(got - v) <= best + 1e-12)
    assert np.all(got <= 6.0)


def test_mxfp4_saturates_and_keeps_zero_blocks():
    w = np.zeros((2, 32))
    w[0, 0] = 7.5                                     # 4 <= 7.5 < 8 at s = 0 -> saturates to 6
    codes, sc = mxfp8.quantize_mxfp4(w)
    assert sc[0, 0] == 127 and mxfp8.dequantize_mxfp4(codes, sc)[0, 0] == 6.0
    assert sc[1, 0] == 0 and not codes[1].any()
