"""The whole W4A4 MoE expert layer on the GPU, checked stage by stage
(teacher-forced: each stage is recomputed by the oracle from the GPU's own
previous-stage output), plus the strict-mode batch-invariance check."""
import numpy as np
import pytest
import torch

from oracle import cpp
from nvfp4_moe_grouped_token_b200 import ops, workloads

from _parity import (bf16_ulp, check_bf16, check_weights_exact, dequant_weights, expert_of_rows, gemm_bound,
                     padded_rows, swiglu_bound)

pytestmark = pytest.mark.gpu


class Layer:
    def __init__(self, cfg, flags):
        self.cfg = cfg
        self.flags = flags
        self.per_token = bool(flags & (ops.SCALE_PER_TOKEN | ops.STRICT))
        self.inp = workloads.layer_inputs(cfg)
        self.wgu = ops.nvfp4_prepare_weights(self.inp["w_gate_up"].cuda(), gate_up=True)
        self.wdn = ops.nvfp4_prepare_weights(self.inp["w_down"].cuda(), gate_up=False)
        T, H, I, E, k = cfg.T, cfg.H, cfg.I, cfg.E, cfg.k
        self.ws = torch.zeros(ops.moe_expert_layer_workspace_size(T, H, I, E, k, flags),
                              dtype=torch.uint8, device="cuda")
        self.y = torch.empty(T, H, dtype=torch.bfloat16, device="cuda")
        self.x = self.inp["x"].cuda()
        self.idx = self.inp["topk_idx"].cuda()
        self.w = self.inp["topk_w"].cuda()

    def run(self, keep_h=True):
        # KEEP_H leaves h readable for the stage-by-stage checks; the outputs
        # do not depend on it (test_keep_h_does_not_change_outputs)
        flags = self.flags | (ops.KEEP_H if keep_h else 0)
        ops.moe_expert_layer(self.x, self.idx, self.w, self.wgu, self.wdn, self.y, self.ws, flags)
        assert ops.device_status(self.ws) == 0
        c = self.cfg
        self.v = ops.layer_views(self.ws, c.T, c.H, c.I, c.E, c.k, self.flags)

    def check(self, sample_tokens=None, check_weights=True):
        c = self.cfg
        T, H, I, E, k = c.T, c.H, c.I, c.E, c.k
        v = self.v
        x = self.inp["x"].float().numpy()
        idx = self.inp["topk_idx"].numpy()
        if check_weights:
            check_weights_exact(self.wgu, self.inp["w_gate_up"], True, experts=range(min(E, 3)))
            check_weights_exact(self.wdn, self.inp["w_down"], False, experts=range(min(E, 3)))
        # 1-2. permutation (exact, all rows)
        info = cpp.permutation(idx, E)
        for key in ("offsets", "padded_offsets", "perm"):
            assert np.array_equal(v[key].cpu().numpy(), info[key]), key
        assert np.array_equal(v["inv_perm"].cpu().numpy(), info["inv_perm"])
        prow = padded_rows(info)
        tok = info["perm"] // k
        e_of = expert_of_rows(info["offsets"])
        # rows under test
        if sample_tokens is None:
            rows = np.arange(T * k)
            toks = np.arange(T)
        else:
            toks = np.asarray(sample_tokens)
            rows = np.sort(info["inv_perm"][toks].reshape(-1))
        pr = prow[rows]
        cap = v["rows_cap"]
        # 3. x quantized once per token, scattered (exact)
        qx = cpp.quantize(x, self.per_token)
        xq = v["x_q"].cpu().numpy()
        xsf = ops.sf_kstep_to_rowmajor(v["x_sf"].cpu(), cap, H).numpy()
        assert np.array_equal(xq[pr], qx["q"][tok[rows]])
        assert np.array_equal(xsf[pr], qx["sf"][tok[rows]])
        sd_want = qx["s_dec"][tok[rows]] if self.per_token else np.full(len(rows), qx["s_dec"][0])
        assert np.array_equal(v["x_sdec"].cpu().numpy()[pr], sd_want)
        # 4. gate_up + SwiGLU -> h (tolerance, teacher-forced from the exact codes)
        xh = cpp.dequantize(qx["q"], qx["sf"], qx["s_dec"])
        a = xh[tok[rows]]
        g = np.empty((len(rows), 2 * I))
        gs = np.empty_like(g)
        d_exact = np.empty((len(rows), H))
        d_abs = np.empty_like(d_exact)
        h_gpu_all = v["h"].float().cpu().numpy()
        h_gpu = h_gpu_all[pr]
        for e in np.unique(e_of[rows]):
            m = e_of[rows] == e
            we = dequant_weights(self.wgu, int(e), gate_up=True)
            g[m], gs[m] = cpp.gemm_rows(a[m], we, with_abs=True)
        h_exact = cpp.swiglu(g, I)
        tg, tu = gemm_bound(gs[:, :I]), gemm_bound(gs[:, I:])
        check_bf16(h_gpu, h_exact, swiglu_bound(g[:, :I], g[:, I:], tg, tu), "h")
        # 5. requant of the GPU's h, amax reused from the epilogue (exact)
        if self.per_token:
            qh = cpp.quantize(h_gpu, True)
        else:
            valid_h = h_gpu_all[prow]                     # every routed row
            amax = np.abs(valid_h).max()
            qh = cpp.quantize(h_gpu, False, amax_in=np.array([amax], np.float32))
        hq = v["h_q"].cpu().numpy()
        hsf = ops.sf_kstep_to_rowmajor(v["h_sf"].cpu(), cap, I).numpy()
        assert np.array_equal(hq[pr], qh["q"])
        assert np.array_equal(hsf[pr], qh["sf"])
        hsd = v["h_sdec"].cpu().numpy()[pr]
        assert np.array_equal(hsd, qh["s_dec"] if self.per_token else np.full(len(rows), qh["s_dec"][0]))
        # 6. down GEMM from the GPU's h codes -> D (tolerance)
        hh = cpp.dequantize(qh["q"], qh["sf"], qh["s_dec"])
        for e in np.unique(e_of[rows]):
            m = e_of[rows] == e
            we = dequant_weights(self.wdn, int(e), gate_up=False)
            d_exact[m], d_abs[m] = cpp.gemm_rows(hh[m], we, with_abs=True)
        d_gpu = v["d"].float().cpu().numpy()[rows]
        check_bf16(d_gpu, d_exact, gemm_bound(d_abs), "D")
        # 7. combine from the GPU's D (fp32 sum of k terms vs fp64: one BF16 ulp)
        d_all = v["d"].float().cpu().numpy()
        inv = info["inv_perm"][toks]
        wts = self.inp["topk_w"].numpy()[toks].astype(np.float64)
        y_exact = np.zeros((len(toks), H))
        for j in range(k):
            y_exact += wts[:, j:j + 1] * d_all[inv[:, j]]
        y_gpu = self.y.float().cpu().numpy()[toks]
        bound = 1e-6 * (np.abs(wts)[:, :, None] * np.abs(d_all[inv])).sum(axis=1) + 1e-30
        check_bf16(y_gpu, y_exact, bound, "y")


SMALL = workloads.LayerConfig("small", T=300, H=256, I=256, E=8, k=2, seed=21)


@pytest.mark.parametrize("flags", [0, ops.SCALE_PER_TOKEN, ops.STRICT, ops.STRICT | ops.FUSED_REQUANT])
def test_small_layer_all_rows(flags):
    L = Layer(SMALL, flags)
    L.run()
    L.check()


def test_small_layer_wide_row_scales():
    """Rows of x scaled by 2^-20 .. 2^20 (the per-token scales follow them):
    G reaches far below -64, where e^-g would overflow the fast division in
    a plain g / (1 + e^-g); h must still be within tolerance of the exact
    silu(g) u, which is a BF16 number down to g ~ -100."""
    L = Layer(SMALL, ops.STRICT)
    g = torch.Generator().manual_seed(12)
    sc = torch.exp2(torch.randint(-20, 21, (SMALL.T, 1), generator=g).float())
    L.inp["x"] = (L.inp["x"].float() * sc).to(torch.bfloat16)
    L.x = L.inp["x"].cuda()
    L.run()
    L.check(check_weights=False)


def test_small_layer_end_to_end_against_full_oracle():
    L = Layer(SMALL, ops.STRICT)
    L.run()
    x = L.inp["x"].float().numpy()
    ref = cpp.expert_layer(x, L.inp["topk_idx"].numpy(), L.inp["topk_w"].numpy(),
                           L.inp["w_gate_up"].float().numpy(), L.inp["w_down"].float().numpy(), per_token=True)
    y = L.y.float().cpu().numpy()
    rel = np.linalg.norm(y - ref["y"]) / np.linalg.norm(ref["y"])
    # not teacher-forced: requant code flips near rounding boundaries are expected
    print(f"end-to-end relative L2 difference vs oracle: {rel:.3g}")
    assert rel < 2e-2


@pytest.mark.parametrize("cfg_name", ["small", "moe30b", "dense4b"])
def test_fused_requant_matches_the_separate_pass(cfg_name):
    """NVFP4MOE_FUSED_REQUANT requantizes h inside the gate_up GEMM (m-tile-
    major tile order, worker warps); without KEEP_H it also drops h's cache
    lines.  Codes, scales, S_dec, D and y must be bitwise those of the
    separate requantization pass, and h itself with KEEP_H."""
    cfg = {"small": SMALL, "moe30b": workloads.CONFIGS["moe30b"], "dense4b": workloads.CONFIGS["dense4b"]}[cfg_name]
    L = Layer(cfg, ops.STRICT)
    L.run(keep_h=True)
    keys = ("h_q", "h_sf", "h_sdec", "d", "h_amax", "h")
    ref = {key: L.v[key].clone() for key in keys}
    y_ref = L.y.clone()
    for extra in (ops.FUSED_REQUANT | ops.KEEP_H, ops.FUSED_REQUANT):
        L.ws.zero_()
        L.y.zero_()
        L.flags = ops.STRICT | extra
        L.run(keep_h=False)
        for key in keys:
            if key == "h" and not extra & ops.KEEP_H:
                continue
            assert torch.equal(L.v[key].view(torch.uint8), ref[key].view(torch.uint8)), (key, extra)
        assert torch.equal(L.y.view(torch.int16), y_ref.view(torch.int16)), extra


@pytest.mark.parametrize("cfg_name", ["small", "moe30b"])
def test_fast_combine_matches_the_ordered_sum(cfg_name):
    """NVFP4MOE_FAST_COMBINE (non-strict): the down GEMM adds w * D (FP32)
    straight into y's FP32 accumulator.  Against the ordered path's BF16 D:
    |y_fast - sum_j w_j D_j| <= sum_j |w_j| ulp(D_j)/2 (D's BF16 rounding the
    fast path skips) + the FP32 sum's error + half a BF16 ulp of y."""
    cfg = SMALL if cfg_name == "small" else workloads.CONFIGS["moe30b"]
    L = Layer(cfg, ops.SCALE_PER_TOKEN)
    L.run()
    d = L.v["d"].float().cpu().numpy().astype(np.float64)
    inv = L.v["inv_perm"].cpu().numpy()
    wts = L.inp["topk_w"].numpy().astype(np.float64)
    ref = np.zeros((cfg.T, cfg.H))
    slack = np.zeros_like(ref)
    for j in range(cfg.k):
        dj = d[inv[:, j]]
        ref += wts[:, j:j + 1] * dj
        slack += np.abs(wts[:, j:j + 1]) * (0.5 * bf16_ulp(dj) + cfg.k * 2.0 ** -23 * np.abs(dj))
    ops.moe_expert_layer(L.x, L.idx, L.w, L.wgu, L.wdn, L.y, L.ws, ops.SCALE_PER_TOKEN | ops.FAST_COMBINE)
    assert ops.device_status(L.ws) == 0
    y = L.y.float().cpu().numpy().astype(np.float64)
    err = np.abs(y - ref)
    bound = slack + 0.5 * bf16_ulp(y) + 1e-30
    assert np.all(err <= bound), float((err / bound).max())
    with pytest.raises(ops.NVFP4Error):
        ops.moe_expert_layer(L.x, L.idx, L.w, L.wgu, L.wdn, L.y, L.ws, ops.STRICT | ops.FAST_COMBINE)


def test_moe30b_layer_sampled():
    cfg = workloads.CONFIGS["moe30b"]
    L = Layer(cfg, 0)
    L.run()
    L.check(sample_tokens=np.arange(0, cfg.T, 509), check_weights=False)


def test_moe30b_skew_layer_sampled():
    """65536 tokens with Zipf-skewed routing (several empty experts, a few
    experts above 5 % of the rows), per-token scaling as in the bench."""
    cfg = workloads.CONFIGS["moe30b_skew"]
    L = Layer(cfg, ops.SCALE_PER_TOKEN)
    L.run()
    counts = np.diff(L.v["offsets"].cpu().numpy())
    assert (counts == 0).sum() >= 5 and counts.max() > 0.05 * cfg.T * cfg.k
    L.check(sample_tokens=np.arange(0, cfg.T, 1021), check_weights=False)


def test_dense4b_layer_sampled():
    cfg = workloads.CONFIGS["dense4b"]
    L = Layer(cfg, ops.SCALE_PER_TOKEN)
    L.run()
    L.check(sample_tokens=np.arange(0, cfg.T, 1021), check_weights=False)


def test_strict_batch_invariance():
    """Each token's BF16 output is bitwise identical whether the 4096 tokens
    run as one batch, as batches of 1, 7 and 64, or in a shuffled order."""
    cfg = workloads.CONFIGS["strict"]
    L = Layer(cfg, ops.STRICT)
    L.run()
    full = L.y.clone()
    T = cfg.T

    def run_subset(tok_idx):
        n = len(tok_idx)
        y = torch.empty(n, cfg.H, dtype=torch.bfloat16, device="cuda")
        ops.moe_expert_layer(L.x[tok_idx], L.idx[tok_idx], L.w[tok_idx], L.wgu, L.wdn, y, L.ws, ops.STRICT)
        return y

    for bs in (1, 7, 64):
        out = torch.empty_like(full)
        for s in range(0, T, bs):
            sl = torch.arange(s, min(s + bs, T), device="cuda")
            out[sl] = run_subset(sl)
        assert torch.equal(out.view(torch.int16), full.view(torch.int16)), f"batch size {bs}"
    order = torch.randperm(T, generator=torch.Generator().manual_seed(5)).cuda()
    shuffled = run_subset(order)
    assert torch.equal(shuffled.view(torch.int16), full[order].view(torch.int16)), "shuffled order"
    assert ops.device_status(L.ws) == 0


def test_layer_replays_from_a_cuda_graph():
    """The layer makes no host synchronization and no allocation, so a call
    captures into a CUDA graph; replays with new inputs copied into the same
    buffers give bitwise the eagerly launched outputs."""
    cfg = SMALL
    L = Layer(cfg, ops.SCALE_PER_TOKEN)
    L.run(keep_h=False)                        # first call: one-time kernel set-up outside capture
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        ops.moe_expert_layer(L.x, L.idx, L.w, L.wgu, L.wdn, L.y, L.ws, L.flags)
    gen = torch.Generator().manual_seed(31)
    for _ in range(2):
        x2 = torch.randn(cfg.T, cfg.H, generator=gen).to(torch.bfloat16)
        keys = torch.rand(cfg.T, cfg.E, generator=gen)
        idx2 = torch.argsort(keys, dim=1)[:, :cfg.k].to(torch.int32).contiguous()
        w2 = torch.softmax(torch.randn(cfg.T, cfg.k, generator=gen), dim=1).float()
        L.x.copy_(x2)
        L.idx.copy_(idx2)
        L.w.copy_(w2)
        g.replay()
        torch.cuda.synchronize()
        y_graph = L.y.clone()
        y_eager = torch.empty_like(L.y)
        ops.moe_expert_layer(L.x, L.idx, L.w, L.wgu, L.wdn, y_eager, L.ws, L.flags)
        torch.cuda.synchronize()
        assert ops.device_status(L.ws) == 0
        assert torch.equal(y_graph.view(torch.int16), y_eager.view(torch.int16))
    del g


def test_moe30b_exact_stages_every_row():
    """The bit-exact stages on every routed row of the Qwen3-30B-A3B-shaped
    layer (per-token scaling, as benched): the x codes, scales and S_dec
    scattered to all 131072 rows, and the requantization of the GPU's h (amax
    from the epilogue) on all of them."""
    cfg = workloads.CONFIGS["moe30b"]
    L = Layer(cfg, ops.SCALE_PER_TOKEN)
    L.run()
    T, H, I, k = cfg.T, cfg.H, cfg.I, cfg.k
    v = L.v
    info = cpp.permutation(L.inp["topk_idx"].numpy(), cfg.E)
    for key in ("offsets", "padded_offsets", "perm"):
        assert np.array_equal(v[key].cpu().numpy(), info[key]), key
    prow = padded_rows(info)
    tok = info["perm"] // k
    cap = v["rows_cap"]
    qx = cpp.quantize(L.inp["x"].float().numpy(), True)
    xq = v["x_q"].cpu().numpy()[prow]
    xsf = ops.sf_kstep_to_rowmajor(v["x_sf"].cpu(), cap, H).numpy()[prow]
    assert np.array_equal(xq, qx["q"][tok])
    assert np.array_equal(xsf, qx["sf"][tok])
    assert np.array_equal(v["x_sdec"].cpu().numpy()[prow], qx["s_dec"][tok])
    h = v["h"].float().cpu().numpy()[prow]
    qh = cpp.quantize(h, True)
    assert np.array_equal(v["h_q"].cpu().numpy()[prow], qh["q"])
    assert np.array_equal(ops.sf_kstep_to_rowmajor(v["h_sf"].cpu(), cap, I).numpy()[prow], qh["sf"])
    assert np.array_equal(v["h_sdec"].cpu().numpy()[prow], qh["s_dec"])
