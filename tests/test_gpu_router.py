"""Top-k routing from router logits on the GPU against the oracle's router
(reading R15): expert ids bit-exact, weights within a tolerance derived from
the FP32 arithmetic, and the routed result feeding the permutation."""
import numpy as np
import pytest
import torch

from oracle import cpp
from nvfp4_moe_grouped_token_b200 import ops

pytestmark = pytest.mark.gpu

# Weight tolerance, relative: expf is within 2 ulp (2^-22); l_j - l_max is one
# FP32 subtraction (|error| <= 2^-24 * 16 for the N(0,1)-sized logits used
# here, about 1e-6 relative after exp); the sum over at most 32 slots is 5
# butterfly roundings and the division one more: about 2e-6 in all, 4e-6 with
# margin.
W_RTOL = 4e-6


def _logits(T, E, seed, ties=False):
    g = torch.Generator().manual_seed(seed)
    lg = torch.randn(T, E, generator=g, dtype=torch.float32)
    if ties:   # many exact ties: values on a 0.25 grid
        lg = torch.round(lg * 4) / 4
    return lg


def _route_gpu(lg, k):
    T, E = lg.shape
    idx = torch.full((T, k), -7, dtype=torch.int32, device="cuda")
    w = torch.full((T, k), float("nan"), dtype=torch.float32, device="cuda")
    ops.moe_route_topk(lg.cuda(), k, idx, w)
    torch.cuda.synchronize()
    return idx.cpu().numpy(), w.cpu().numpy()


def _check(lg, k):
    idx, w = _route_gpu(lg, k)
    ref_idx, ref_w = cpp.route_topk(lg.numpy(), k)
    assert np.array_equal(idx, ref_idx)
    err = np.abs(w.astype(np.float64) - ref_w)
    assert np.all(err <= W_RTOL * ref_w + 1e-38), float((err / ref_w).max())


@pytest.mark.parametrize("T,E,k", [(5000, 128, 8), (777, 16, 4), (300, 1, 1), (257, 33, 1),
                                   (200, 1000, 32), (129, 64, 32), (64, 256, 8), (64, 512, 16)])
def test_route_topk_matches_oracle(T, E, k):
    _check(_logits(T, E, seed=E * 31 + k), k)


def test_route_topk_ties_go_to_the_lower_id():
    _check(_logits(2000, 128, seed=9, ties=True), 8)
    idx, w = _route_gpu(torch.zeros(5, 128), 8)
    assert np.array_equal(idx, np.tile(np.arange(8), (5, 1)))
    assert np.allclose(w, 1 / 8, rtol=0, atol=1e-7)


def test_route_topk_empty_is_noop():
    idx = torch.full((0, 8), -7, dtype=torch.int32, device="cuda")
    w = torch.zeros(0, 8, dtype=torch.float32, device="cuda")
    ops.moe_route_topk(torch.zeros(0, 128, device="cuda"), 8, idx, w)
    torch.cuda.synchronize()


def test_routed_tokens_permute_like_the_oracle():
    """Logits -> device top-k -> device permutation, against the oracle's
    top-k and permutation of the same logits (16384 tokens, 128 experts, top-8)."""
    T, E, k = 16384, 128, 8
    lg = _logits(T, E, seed=11)
    idx = torch.empty(T, k, dtype=torch.int32, device="cuda")
    w = torch.empty(T, k, dtype=torch.float32, device="cuda")
    ops.moe_route_topk(lg.cuda(), k, idx, w)
    off = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    pad = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    perm = torch.empty(T * k, dtype=torch.int32, device="cuda")
    inv = torch.empty(T, k, dtype=torch.int32, device="cuda")
    ws = torch.zeros(ops.moe_permute_workspace_size(T, k, E), dtype=torch.uint8, device="cuda")
    ops.moe_permute(idx, E, off, pad, perm, inv, ws)
    assert ops.device_status(ws) == 0
    ref_idx, _ = cpp.route_topk(lg.numpy(), k)
    info = cpp.permutation(ref_idx, E)
    assert np.array_equal(off.cpu().numpy(), info["offsets"])
    assert np.array_equal(perm.cpu().numpy(), info["perm"])
    assert np.array_equal(inv.cpu().numpy(), info["inv_perm"])
    # the routing kernel's time at this shape (reported, not asserted)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    lgd = lg.cuda()
    for _ in range(3):
        ops.moe_route_topk(lgd, k, idx, w)
    e0.record()
    for _ in range(20):
        ops.moe_route_topk(lgd, k, idx, w)
    e1.record()
    torch.cuda.synchronize()
    us = e0.elapsed_time(e1) / 20 * 1e3
    print(f"moe_route_topk T={T} E={E} k={k}: {us:.1f} us per call "
          f"({T * E * 4 / (us * 1e-6) / 1e9:.0f} GB/s of logits)")


def _route_permute(lg, k):
    T, E = lg.shape
    idx = torch.full((T, k), -7, dtype=torch.int32, device="cuda")
    w = torch.full((T, k), float("nan"), dtype=torch.float32, device="cuda")
    off = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    pad = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    perm = torch.empty(T * k, dtype=torch.int32, device="cuda")
    inv = torch.empty(T, k, dtype=torch.int32, device="cuda")
    ws = torch.zeros(ops.moe_permute_workspace_size(T, k, E), dtype=torch.uint8, device="cuda")
    ops.moe_route_permute(lg.cuda(), k, idx, w, off, pad, perm, inv, ws)
    assert ops.device_status(ws) == 0
    return [t.cpu().numpy() for t in (idx, w, off, pad, perm, inv)]


@pytest.mark.parametrize("T,E,k", [(16384, 128, 8), (1000, 16, 4), (333, 1000, 32), (257, 33, 1), (130, 256, 8)])
def test_fused_route_permute_matches_oracle(T, E, k):
    """Router top-k folded into the routing-histogram kernel: ids and the
    whole permutation bit-exact against the oracle's router + permutation,
    weights within the router tolerance and bitwise equal to the standalone
    router kernel's (the same arithmetic)."""
    lg = _logits(T, E, seed=T + E + k, ties=(E == 128))
    idx, w, off, pad, perm, inv = _route_permute(lg, k)
    ref_idx, ref_w = cpp.route_topk(lg.numpy(), k)
    assert np.array_equal(idx, ref_idx)
    assert np.all(np.abs(w.astype(np.float64) - ref_w) <= W_RTOL * ref_w + 1e-38)
    idx2, w2 = _route_gpu(lg, k)
    assert np.array_equal(w.view(np.int32), w2.view(np.int32))
    info = cpp.permutation(ref_idx, E)
    for name, got in (("offsets", off), ("padded_offsets", pad), ("perm", perm), ("inv_perm", inv)):
        assert np.array_equal(got, info[name]), name


def test_layer_from_logits_equals_layer_with_routed_inputs():
    """moe_expert_layer_from_logits routes inside the layer's histogram
    kernel; its output is bitwise that of moe_expert_layer fed the same
    routing (which the standalone router produces)."""
    from nvfp4_moe_grouped_token_b200 import workloads
    cfg = workloads.LayerConfig("logits_layer", T=2000, H=512, I=256, E=16, k=4, seed=31)
    inp = workloads.layer_inputs(cfg)
    lg = _logits(cfg.T, cfg.E, seed=3).cuda()
    wgu = ops.nvfp4_prepare_weights(inp["w_gate_up"].cuda(), gate_up=True)
    wdn = ops.nvfp4_prepare_weights(inp["w_down"].cuda(), gate_up=False)
    x = inp["x"].cuda()
    for flags in (ops.STRICT, 0):
        ws = torch.zeros(ops.moe_expert_layer_workspace_size(cfg.T, cfg.H, cfg.I, cfg.E, cfg.k, flags),
                         dtype=torch.uint8, device="cuda")
        idx = torch.empty(cfg.T, cfg.k, dtype=torch.int32, device="cuda")
        w = torch.empty(cfg.T, cfg.k, dtype=torch.float32, device="cuda")
        y1 = torch.empty(cfg.T, cfg.H, dtype=torch.bfloat16, device="cuda")
        ops.moe_expert_layer_from_logits(x, lg, wgu, wdn, idx, w, y1, ws, flags)
        assert ops.device_status(ws) == 0
        idx2 = torch.empty_like(idx)
        w2 = torch.empty_like(w)
        ops.moe_route_topk(lg, cfg.k, idx2, w2)
        assert torch.equal(idx, idx2) and torch.equal(w.view(torch.int32), w2.view(torch.int32))
        y2 = torch.empty_like(y1)
        ops.moe_expert_layer(x, idx2, w2, wgu, wdn, y2, ws, flags)
        assert ops.device_status(ws) == 0
        assert torch.equal(y1.view(torch.int16), y2.view(torch.int16)), flags


# ------------------------------------------------------------ router GEMM --

def _router_inputs(T, H, E, seed):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(T, H, generator=g).to(torch.bfloat16)
    w = (torch.randn(E, H, generator=g) * 0.02).to(torch.bfloat16)
    return x, w


@pytest.mark.parametrize("T,H,E", [(300, 256, 32), (129, 512, 128), (1000, 2048, 288), (64, 64, 1024)])
def test_router_logits_match_oracle(T, H, E):
    """logits = x W_r^T on the tensor cores against the oracle's exactly
    rounded fp64 product, within 1e-5 * sum|x w| + 1e-6 (FP32 output).
    Ragged T (tile rows past T read as zeros), E above 256 (a partial second
    tile of weight rows) and H down to one K-step."""
    x, w = _router_inputs(T, H, E, seed=T + E)
    logits = torch.full((T, E), float("nan"), dtype=torch.float32, device="cuda")
    ws = ops.moe_router_logits(x.cuda(), w.cuda(), logits)
    assert ops.device_status(ws) == 0
    ex, sa = cpp.gemm_rows(x.float().numpy().astype(np.float64), w.float().numpy().astype(np.float64), with_abs=True)
    got = logits.cpu().numpy().astype(np.float64)
    assert np.all(np.abs(got - ex) <= 1e-5 * sa + 1e-6), float(np.max(np.abs(got - ex) / (1e-5 * sa + 1e-6)))


def test_router_logits_moe30b_shape_then_routing():
    """The Qwen3-30B-A3B router (T = 16384, H = 2048, E = 128), sampled rows
    checked against the oracle; then routing from the GPU's logits matches
    the oracle's router on the same logits (ids exact)."""
    T, H, E, k = 16384, 2048, 128, 8
    x, w = _router_inputs(T, H, E, seed=3)
    logits = torch.empty(T, E, dtype=torch.float32, device="cuda")
    ws = ops.moe_router_logits(x.cuda(), w.cuda(), logits)
    assert ops.device_status(ws) == 0
    rows = np.arange(7, T, 509)
    ex, sa = cpp.gemm_rows(x[rows].float().numpy().astype(np.float64), w.float().numpy().astype(np.float64),
                           with_abs=True)
    got = logits.cpu().numpy()
    assert np.all(np.abs(got[rows] - ex) <= 1e-5 * sa + 1e-6)
    idx, wt = _route_gpu(logits.cpu(), k)
    ref_idx, ref_w = cpp.route_topk(got, k)
    assert np.array_equal(idx, ref_idx)
    assert np.allclose(wt, ref_w, rtol=W_RTOL, atol=0)


def test_router_logits_rejects_bad_shapes():
    x, w = _router_inputs(16, 64, 48, seed=1)
    logits = torch.empty(16, 48, dtype=torch.float32, device="cuda")
    with pytest.raises(ops.NVFP4Error):        # E % 32 != 0
        ops.moe_router_logits(x.cuda(), w.cuda(), logits)
