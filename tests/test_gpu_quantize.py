"""GPU quantizer and codec parity: bit-exact against the C++ CPU oracle,
including exhaustive sweeps of the hardware E2M1 / UE4M3 conversions over
every finite binary32 bit pattern."""
import numpy as np
import pytest
import torch

from oracle import cpp
from nvfp4_moe_grouped_token_b200 import ops

from _parity import sf_rowmajor

pytestmark = pytest.mark.gpu


def _x(M, K, seed, kind="normal"):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(M, K, generator=g)
    if kind == "wide":
        x *= torch.exp2(torch.randint(-30, 30, (M, 1), generator=g).float())
    elif kind == "outliers":
        ch = torch.randperm(K, generator=g)[: max(1, K // 1000)]
        x[:, ch] *= 30
    elif kind == "zeros":
        x[::3] = 0
        x[:, 16:32] = 0
        x[1, :] = 1e-38          # underflowing blocks: sf rounds to 0
    return x.to(torch.bfloat16)


def _gpu_quant(x_cpu, per_token, sf_mma=False, amax_in=None):
    x = x_cpu.cuda()
    M, K = x.shape
    rows = (M + 127) // 128 * 128 if sf_mma else M
    q = torch.full((M, K // 2), 0xAA, dtype=torch.uint8, device="cuda")
    sf = torch.full((rows * K // 16,), 0xAA, dtype=torch.uint8, device="cuda")
    n_s = M if per_token else 1
    s_dec = torch.empty(n_s, dtype=torch.float32, device="cuda")
    amax_out = torch.empty(n_s, dtype=torch.float32, device="cuda")
    flags = (ops.SCALE_PER_TOKEN if per_token else 0) | (ops.SF_MMA_LAYOUT if sf_mma else 0)
    ain = None if amax_in is None else torch.as_tensor(amax_in, dtype=torch.float32).cuda()
    ops.nvfp4_quantize(x, q, sf, s_dec, flags, amax_in=ain, amax_out=amax_out)
    torch.cuda.synchronize()
    sfn = sf_rowmajor(sf, M, K) if sf_mma else sf.cpu().numpy().reshape(M, K // 16)
    return q.cpu().numpy(), sfn, s_dec.cpu().numpy(), amax_out.cpu().numpy()


SHAPES = [(1, 64), (5, 64), (37, 256), (300, 768), (129, 2048), (64, 2560), (1000, 4096), (16, 9728)]


@pytest.mark.parametrize("M,K", SHAPES)
@pytest.mark.parametrize("per_token", [False, True])
def test_quantize_bit_exact(M, K, per_token):
    x = _x(M, K, seed=M * 7 + K)
    q, sf, s_dec, amax = _gpu_quant(x, per_token)
    r = cpp.quantize(x.float().numpy(), per_token)
    assert np.array_equal(amax, r["amax"])
    assert np.array_equal(s_dec, r["s_dec"])
    assert np.array_equal(sf, r["sf"])
    assert np.array_equal(q, r["q"])


@pytest.mark.parametrize("kind", ["wide", "outliers", "zeros"])
@pytest.mark.parametrize("per_token", [False, True])
def test_quantize_hard_inputs(kind, per_token):
    x = _x(200, 512, seed=3, kind=kind)
    q, sf, s_dec, amax = _gpu_quant(x, per_token)
    r = cpp.quantize(x.float().numpy(), per_token)
    assert np.array_equal(s_dec, r["s_dec"]) and np.array_equal(sf, r["sf"]) and np.array_equal(q, r["q"])


@pytest.mark.parametrize("per_token", [False, True])
def test_quantize_mma_layout_and_amax_reuse(per_token):
    x = _x(333, 1024, seed=5)
    ref = cpp.quantize(x.float().numpy(), per_token)
    q, sf, s_dec, amax = _gpu_quant(x, per_token, sf_mma=True)
    assert np.array_equal(sf, ref["sf"]) and np.array_equal(q, ref["q"])
    # amax reuse: the given amax is used as is (here: twice the true one)
    a2 = ref["amax"] * np.float32(2)
    q2, sf2, s2, amax2 = _gpu_quant(x, per_token, amax_in=a2)
    r2 = cpp.quantize(x.float().numpy(), per_token, amax_in=a2)
    assert np.array_equal(amax2, a2)
    assert np.array_equal(q2, r2["q"]) and np.array_equal(sf2, r2["sf"]) and np.array_equal(s2, r2["s_dec"])


def _neighbourhoods(points, span=64):
    """All fp32 values within `span` ulps of each point."""
    p = np.asarray(points, np.float32).view(np.int32).astype(np.int64)
    offs = np.arange(-span, span + 1)
    bits = (p[:, None] + offs[None, :]).reshape(-1)
    bits = bits[(bits >= 0) & (bits < 0x7F800000)]
    return bits.astype(np.int32).view(np.float32)


def test_e2m1_hardware_rounding_matches_definition():
    g = cpp.e2m1_decode(np.arange(8))
    mids = (g[1:] + g[:-1]) / 2
    pts = np.concatenate([g, mids, [6.5, 7.0, 100.0, 1e-30, 2.0 ** -126]])
    y = _neighbourhoods(pts[pts > 0])
    rng = np.random.default_rng(1)
    rnd = rng.integers(0, 0x7F800000, size=1 << 22, dtype=np.int64).astype(np.int32).view(np.float32)
    y = np.concatenate([y, rnd, [0.0]]).astype(np.float32)
    y = np.concatenate([y, -y])
    codes = torch.empty(y.size, dtype=torch.uint8, device="cuda")
    ops.nvfp4moe_encode_e2m1(torch.from_numpy(y).cuda(), codes)
    got = codes.cpu().numpy()
    want = cpp.e2m1_encode(y)
    bad = got != want
    assert not bad.any(), list(zip(y[bad][:8], got[bad][:8], want[bad][:8]))


def test_ue4m3_hardware_rounding_matches_definition():
    g = cpp.ue4m3_decode(np.arange(127))
    mids = (g[1:] + g[:-1]) / 2
    pts = np.concatenate([g[1:], mids, [448.0, 464.0, 480.0, 1e4, 2.0 ** -10]])
    v = _neighbourhoods(pts)
    rng = np.random.default_rng(2)
    rnd = rng.integers(0, 0x7F800000, size=1 << 22, dtype=np.int64).astype(np.int32).view(np.float32)
    v = np.concatenate([v, rnd, [0.0]]).astype(np.float32)
    codes = torch.empty(v.size, dtype=torch.uint8, device="cuda")
    ops.nvfp4moe_encode_ue4m3(torch.from_numpy(v).cuda(), codes)
    got = codes.cpu().numpy()
    want = cpp.ue4m3_encode(v)
    bad = got != want
    assert not bad.any(), list(zip(v[bad][:8], got[bad][:8], want[bad][:8]))


CHUNK = 1 << 26


def _sweep(lo, hi, encode_gpu, encode_cpu):
    """GPU codes of every binary32 pattern in [lo, hi) against the oracle's,
    chunk by chunk (the oracle builds its inputs from the same bit range)."""
    for start in range(lo, hi, CHUNK):
        n = min(CHUNK, hi - start)
        bits = torch.arange(start, start + n, dtype=torch.int64, device="cuda")
        vals = (bits - (1 << 32) * (bits >= (1 << 31))).to(torch.int32).view(torch.float32)
        codes = torch.empty(n, dtype=torch.uint8, device="cuda")
        encode_gpu(vals, codes)
        got = codes.cpu().numpy()
        want = encode_cpu(start, n)
        if not np.array_equal(got, want):
            bad = np.nonzero(got != want)[0][:8]
            raise AssertionError([(hex(start + int(i)), int(got[i]), int(want[i])) for i in bad])
        del bits, vals, codes


def test_e2m1_exhaustive_all_finite_fp32():
    """cvt.rn.satfinite.e2m1x2.f32 on all 2^32 - 2^24 finite patterns (both
    signs) equals the definition (round to nearest even, saturate at 6, sign
    kept on -0)."""
    _sweep(0, 0x7F800000, ops.nvfp4moe_encode_e2m1, cpp.e2m1_encode_bits)
    _sweep(0x80000000, 0xFF800000, ops.nvfp4moe_encode_e2m1, cpp.e2m1_encode_bits)


def test_ue4m3_exhaustive_all_nonnegative_finite_fp32():
    """cvt.rn.satfinite.e4m3x2.f32 on every non-negative finite pattern (the
    quantizer only converts non-negative block scales) equals UE4M3 round to
    nearest even saturating at 448."""
    _sweep(0, 0x7F800000, ops.nvfp4moe_encode_ue4m3, cpp.ue4m3_encode_bits)


def test_empty_is_noop():
    x = torch.empty(0, 64, dtype=torch.bfloat16, device="cuda")
    t = torch.empty(0, dtype=torch.uint8, device="cuda")
    f = torch.empty(1, dtype=torch.float32, device="cuda")
    ops.nvfp4_quantize(x, t, t, f, 0, amax_out=f)
