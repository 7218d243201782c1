"""The W4A8 MoE expert layer on the GPU: MXFP8 activations (x and h), the
W4A4 layer's NVFP4 weights, products on the BF16 tensor cores (MXFP8 values
are exact in BF16).

Teacher-forced against the C++ oracle: the MXFP8 quantize-dequantize of x
and of the GPU's own BF16 h are bit-exact; h before its requantization, D and
y are within the stated GEMM tolerance (1e-5 * sum|a w| + 1e-6 in FP32,
then one BF16 ulp).  The whole layer is also compared with the oracle's W4A8
layer (R20)."""
import numpy as np
import pytest
import torch

from oracle import cpp
from nvfp4_moe_grouped_token_b200 import ops, workloads

from _parity import check_bf16, dequant_weights, expert_of_rows, gemm_bound, padded_rows, swiglu_bound

pytestmark = pytest.mark.gpu


def qdq(v: np.ndarray) -> np.ndarray:
    """Oracle MXFP8 quantize-dequantize of rows (R17)."""
    return cpp.mxfp8_dequantize(*cpp.mxfp8_quantize(np.ascontiguousarray(v, dtype=np.float32)))


class W4A8:
    def __init__(self, cfg, inp=None, flags=ops.KEEP_H):
        self.cfg = cfg
        self.flags = flags
        self.inp = inp if inp is not None else workloads.layer_inputs(cfg)
        self.wgu = ops.nvfp4_prepare_weights(self.inp["w_gate_up"].cuda(), gate_up=True)
        self.wdn = ops.nvfp4_prepare_weights(self.inp["w_down"].cuda(), gate_up=False)
        T, H, I, E, k = cfg.T, cfg.H, cfg.I, cfg.E, cfg.k
        self.ws = torch.zeros(ops.moe_expert_layer_w4a8_workspace_size(T, H, I, E, k, flags), dtype=torch.uint8,
                              device="cuda")
        self.y = torch.empty(T, H, dtype=torch.bfloat16, device="cuda")
        self.x = self.inp["x"].cuda()
        self.idx = self.inp["topk_idx"].cuda()
        self.w = self.inp["topk_w"].cuda()

    def run(self):
        ops.moe_expert_layer_w4a8(self.x, self.idx, self.w, self.wgu, self.wdn, self.y, self.ws, self.flags)
        assert ops.device_status(self.ws) == 0
        c = self.cfg
        self.v = ops.w4a16_views(self.ws, c.T, c.H, c.I, c.E, c.k, self.flags, w4a8=True)

    def check(self, sample_tokens=None):
        c = self.cfg
        T, H, I, E, k = c.T, c.H, c.I, c.E, c.k
        v = self.v
        x = self.inp["x"].float().numpy()
        info = cpp.permutation(self.inp["topk_idx"].numpy(), E)
        for key in ("offsets", "padded_offsets", "perm"):
            assert np.array_equal(v[key].cpu().numpy(), info[key]), key
        prow = padded_rows(info)
        tok = info["perm"] // k
        e_of = expert_of_rows(info["offsets"])
        if sample_tokens is None:
            rows, toks = np.arange(T * k), np.arange(T)
        else:
            toks = np.asarray(sample_tokens)
            rows = np.sort(info["inv_perm"][toks].reshape(-1))
        pr = prow[rows]
        # x rows: MXFP8 quantize-dequantize of each token (exact), zero padding rows
        xq = qdq(x)
        xr = v["x_rows"].float().cpu().numpy()
        assert np.array_equal(xr[pr], xq[tok[rows]].astype(np.float32))
        pad_rows = np.setdiff1d(np.arange(int(info["padded_offsets"][-1])), prow)
        assert not xr[pad_rows].any()
        # h before its requantization (tolerance, from the exact G)
        g = np.empty((len(rows), 2 * I))
        gs = np.empty_like(g)
        for e in np.unique(e_of[rows]):
            m = e_of[rows] == e
            g[m], gs[m] = cpp.gemm_rows(xq[tok[rows[m]]], dequant_weights(self.wgu, int(e), gate_up=True),
                                        with_abs=True)
        h_pre = v["h_pre"].float().cpu().numpy()[pr]
        check_bf16(h_pre, cpp.swiglu(g, I), swiglu_bound(g[:, :I], g[:, I:], gemm_bound(gs[:, :I]),
                                                         gemm_bound(gs[:, I:])), "h before MXFP8 (W4A8)")
        # h's MXFP8 requantization, from the GPU's own BF16 h (exact)
        h = v["h"].float().cpu().numpy()
        assert np.array_equal(h[pr], qdq(h_pre).astype(np.float32)), "MXFP8 h"
        assert not h[pad_rows].any()
        # down from the GPU's h -> D, then the slot-ordered combine
        d_exact = np.empty((len(rows), H))
        d_abs = np.empty_like(d_exact)
        for e in np.unique(e_of[rows]):
            m = e_of[rows] == e
            d_exact[m], d_abs[m] = cpp.gemm_rows(h[pr[m]].astype(np.float64),
                                                 dequant_weights(self.wdn, int(e), gate_up=False), with_abs=True)
        d_all = v["d"].float().cpu().numpy()
        check_bf16(d_all[rows], d_exact, gemm_bound(d_abs), "D (W4A8)")
        inv = info["inv_perm"][toks]
        wts = self.inp["topk_w"].numpy()[toks].astype(np.float64)
        y_exact = np.zeros((len(toks), H))
        for j in range(k):
            y_exact += wts[:, j:j + 1] * d_all[inv[:, j]]
        bound = 1e-6 * (np.abs(wts)[:, :, None] * np.abs(d_all[inv])).sum(axis=1) + 1e-30
        check_bf16(self.y.float().cpu().numpy()[toks], y_exact, bound, "y (W4A8)")


SMALL = workloads.LayerConfig("small_w4a8", T=300, H=256, I=256, E=8, k=2, seed=41)


def hard_inputs(cfg):
    """Activations that exercise MXFP8's edges: rows scaled by 2^-20 .. 2^20
    (block scales far from 1; wider ranges make G so large that the SwiGLU
    check downstream measures only its FP32 bound), all-zero blocks, tiny
    negatives that quantize to -0, and blocks whose amax lands above 448
    after scaling (saturation)."""
    inp = workloads.layer_inputs(cfg)
    x = inp["x"].float()
    g = torch.Generator().manual_seed(9)
    x = x * torch.exp2(torch.randint(-20, 21, (cfg.T, 1), generator=g).float())
    x[::7, :32] = 0.0
    x[1::5, 5] = -1e-30 * x[1::5, 6].abs().clamp_min(1e-3)
    x[2::9, 40] = 1.9 * x[2::9, 32:64].abs().amax(dim=1)
    inp["x"] = x.to(torch.bfloat16)
    return inp


def test_w4a8_small_hard_inputs_all_rows():
    L = W4A8(SMALL, hard_inputs(SMALL))
    L.run()
    L.check()


def test_w4a8_small_against_the_oracle_layer_and_keep_h_changes_nothing():
    L = W4A8(SMALL)
    L.run()
    L.check()
    i = L.inp
    ref = cpp.expert_layer_w4a8(i["x"].float().numpy(), i["topk_idx"].numpy(), i["topk_w"].numpy(),
                                i["w_gate_up"].float().numpy(), i["w_down"].float().numpy())
    y = L.y.float().cpu().numpy()
    rel = np.linalg.norm(y - ref["y"]) / np.linalg.norm(ref["y"])
    # not teacher-forced: an MXFP8 code of h can flip where h sits on a rounding boundary
    print(f"W4A8 end-to-end relative L2 difference vs oracle: {rel:.3g}")
    assert rel < 2e-2
    y0 = L.y.clone()
    M = W4A8(SMALL, L.inp, flags=0)
    M.run()
    assert torch.equal(M.y.view(torch.int16), y0.view(torch.int16))


def test_w4a8_ragged_groups_and_empty_experts():
    cfg = workloads.LayerConfig("ragged_w4a8", T=333, H=512, I=512, E=12, k=3, seed=42)
    inp = workloads.layer_inputs(cfg)
    g = torch.Generator().manual_seed(8)
    keys = torch.rand(cfg.T, 6, generator=g)
    inp["topk_idx"] = torch.argsort(keys, dim=1)[:, :cfg.k].to(torch.int32).contiguous()
    L = W4A8(cfg, inp)
    L.run()
    L.check()


def test_w4a8_moe30b_sampled():
    cfg = workloads.CONFIGS["moe30b"]
    L = W4A8(cfg)
    L.run()
    L.check(sample_tokens=np.arange(3, cfg.T, 997))


def test_w4a8_rejects_other_flags():
    L = W4A8(SMALL)
    with pytest.raises(ops.NVFP4Error):
        ops.moe_expert_layer_w4a8(L.x, L.idx, L.w, L.wgu, L.wdn, L.y, L.ws, ops.STRICT)
