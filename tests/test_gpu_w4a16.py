"""The W4A16 MoE expert layer on the GPU: BF16 activations, the same NVFP4
weights as the W4A4 layer (converted to BF16 tile by tile inside the GEMM).

Stage by stage and teacher-forced against the C++ oracle: each GPU stage is
recomputed from the GPU's own previous-stage output with the stated
GEMM tolerance (1e-5 * sum|a w| + 1e-6 in FP32, then one BF16 ulp); the
permutation and the gathered rows are exact.  The whole layer is also
compared with the oracle's W4A16 layer (R19)."""
import numpy as np
import pytest
import torch

from oracle import cpp
from nvfp4_moe_grouped_token_b200 import ops, workloads

from _parity import check_bf16, dequant_weights, expert_of_rows, gemm_bound, padded_rows, swiglu_bound

pytestmark = pytest.mark.gpu


class W4:
    def __init__(self, cfg, inp=None):
        self.cfg = cfg
        self.inp = inp if inp is not None else workloads.layer_inputs(cfg)
        self.wgu = ops.nvfp4_prepare_weights(self.inp["w_gate_up"].cuda(), gate_up=True)
        self.wdn = ops.nvfp4_prepare_weights(self.inp["w_down"].cuda(), gate_up=False)
        T, H, I, E, k = cfg.T, cfg.H, cfg.I, cfg.E, cfg.k
        self.ws = torch.zeros(ops.moe_expert_layer_w4a16_workspace_size(T, H, I, E, k), dtype=torch.uint8,
                              device="cuda")
        self.y = torch.empty(T, H, dtype=torch.bfloat16, device="cuda")
        self.x = self.inp["x"].cuda()
        self.idx = self.inp["topk_idx"].cuda()
        self.w = self.inp["topk_w"].cuda()

    def run(self):
        ops.moe_expert_layer_w4a16(self.x, self.idx, self.w, self.wgu, self.wdn, self.y, self.ws)
        assert ops.device_status(self.ws) == 0
        c = self.cfg
        self.v = ops.w4a16_views(self.ws, c.T, c.H, c.I, c.E, c.k)

    def check(self, sample_tokens=None):
        c = self.cfg
        T, H, I, E, k = c.T, c.H, c.I, c.E, c.k
        v = self.v
        x = self.inp["x"].float().numpy().astype(np.float64)
        idx = self.inp["topk_idx"].numpy()
        info = cpp.permutation(idx, E)
        for key in ("offsets", "padded_offsets", "perm"):
            assert np.array_equal(v[key].cpu().numpy(), info[key]), key
        assert np.array_equal(v["inv_perm"].cpu().numpy(), info["inv_perm"])
        prow = padded_rows(info)
        tok = info["perm"] // k
        e_of = expert_of_rows(info["offsets"])
        if sample_tokens is None:
            rows = np.arange(T * k)
            toks = np.arange(T)
        else:
            toks = np.asarray(sample_tokens)
            rows = np.sort(info["inv_perm"][toks].reshape(-1))
        pr = prow[rows]
        # gathered rows of x (exact), zero padding rows
        xr = v["x_rows"].float().cpu().numpy()
        assert np.array_equal(xr[pr], x[tok[rows]])
        used = int(info["padded_offsets"][-1])
        pad_rows = np.setdiff1d(np.arange(used), prow)
        assert not xr[pad_rows].any()
        # gate_up with the dequantized NVFP4 weights + SwiGLU -> h
        h_all = v["h"].float().cpu().numpy()
        assert not h_all[pad_rows].any(), "padding rows of h"
        h_gpu = h_all[pr].astype(np.float64)
        g = np.empty((len(rows), 2 * I))
        gs = np.empty_like(g)
        d_exact = np.empty((len(rows), H))
        d_abs = np.empty_like(d_exact)
        for e in np.unique(e_of[rows]):
            m = e_of[rows] == e
            g[m], gs[m] = cpp.gemm_rows(x[tok[rows[m]]], dequant_weights(self.wgu, int(e), gate_up=True),
                                        with_abs=True)
        h_exact = cpp.swiglu(g, I)
        tg, tu = gemm_bound(gs[:, :I]), gemm_bound(gs[:, I:])
        check_bf16(h_gpu, h_exact, swiglu_bound(g[:, :I], g[:, I:], tg, tu), "h (W4A16)")
        # down from the GPU's h -> D
        for e in np.unique(e_of[rows]):
            m = e_of[rows] == e
            d_exact[m], d_abs[m] = cpp.gemm_rows(h_gpu[m], dequant_weights(self.wdn, int(e), gate_up=False),
                                                 with_abs=True)
        d_all = v["d"].float().cpu().numpy()
        check_bf16(d_all[rows], d_exact, gemm_bound(d_abs), "D (W4A16)")
        # slot-ordered combine from the GPU's D
        inv = info["inv_perm"][toks]
        wts = self.inp["topk_w"].numpy()[toks].astype(np.float64)
        y_exact = np.zeros((len(toks), H))
        for j in range(k):
            y_exact += wts[:, j:j + 1] * d_all[inv[:, j]]
        bound = 1e-6 * (np.abs(wts)[:, :, None] * np.abs(d_all[inv])).sum(axis=1) + 1e-30
        check_bf16(self.y.float().cpu().numpy()[toks], y_exact, bound, "y (W4A16)")


SMALL = workloads.LayerConfig("small_w4a16", T=300, H=256, I=256, E=8, k=2, seed=31)


def test_w4a16_small_all_rows_and_against_the_oracle_layer():
    L = W4(SMALL)
    L.run()
    L.check()
    i = L.inp
    ref = cpp.expert_layer_w4a16(i["x"].float().numpy(), i["topk_idx"].numpy(), i["topk_w"].numpy(),
                                 i["w_gate_up"].float().numpy(), i["w_down"].float().numpy())
    y = L.y.float().cpu().numpy()
    rel = np.linalg.norm(y - ref["y"]) / np.linalg.norm(ref["y"])
    # not teacher-forced: h may sit one BF16 ulp away where G is near a rounding boundary
    print(f"W4A16 end-to-end relative L2 difference vs oracle: {rel:.3g}")
    assert rel < 1e-2


def test_w4a16_ragged_groups_and_empty_experts():
    """Experts 6..11 receive no rows; group sizes are ragged; H and I span
    several 256-column tiles and K-steps."""
    cfg = workloads.LayerConfig("ragged_w4a16", T=333, H=512, I=512, E=12, k=3, seed=32)
    inp = workloads.layer_inputs(cfg)
    g = torch.Generator().manual_seed(6)
    keys = torch.rand(cfg.T, 6, generator=g)
    inp["topk_idx"] = torch.argsort(keys, dim=1)[:, :cfg.k].to(torch.int32).contiguous()
    L = W4(cfg, inp)
    L.run()
    L.check()


def test_w4a16_rejects_flags_and_unprepared_gate_up():
    L = W4(SMALL)
    with pytest.raises(ops.NVFP4Error):
        ops.moe_expert_layer_w4a16(L.x, L.idx, L.w, L.wgu, L.wdn, L.y, L.ws, flags=ops.STRICT)
    with pytest.raises(ops.NVFP4Error):
        ops.moe_expert_layer_w4a16(L.x, L.idx, L.w, L.wdn, L.wdn, L.y, L.ws)


def test_w4a16_moe30b_sampled():
    cfg = workloads.CONFIGS["moe30b"]
    L = W4(cfg)
    L.run()
    L.check(sample_tokens=np.arange(0, cfg.T, 997))


def test_w4a16_dense4b_sampled():
    cfg = workloads.CONFIGS["dense4b"]
    L = W4(cfg)
    L.run()
    L.check(sample_tokens=np.arange(5, cfg.T, 1531))


def test_w4a16_is_deterministic():
    L = W4(SMALL)
    L.run()
    y0 = L.y.clone()
    L.ws.zero_()
    L.run()
    assert torch.equal(L.y.view(torch.int16), y0.view(torch.int16))


def test_w4a16_subnormal_block_scales():
    """One weight of 2000 per matrix beside N(0, 0.02) weights: most blocks'
    UE4M3 scales are subnormal (m * 2^-9).  The converter decodes a scale as
    BF16 bits (a BF16 subnormal for these) and multiplies it in BF16; the
    products must still be exactly code * scale."""
    cfg = workloads.LayerConfig("subnormal_w4a16", T=200, H=256, I=256, E=2, k=1, seed=33)
    inp = workloads.layer_inputs(cfg)
    for key in ("w_gate_up", "w_down"):
        w = inp[key].clone()
        w[:, 0, 0] = 2000.0
        inp[key] = w
    L = W4(cfg, inp)
    for prep in (L.wgu, L.wdn):
        sf = prep.sf.cpu().numpy()
        sub = (((sf >> 3) & 0xF) == 0) & ((sf & 7) != 0)
        assert sub.mean() > 0.5, sub.mean()
    L.run()
    L.check()
