"""Backward of the MoE expert layer in the BF16-backward mode on the GPU.

Stage by stage and teacher-forced: each GPU stage is recomputed by the C++
oracle from the GPU's own stored inputs (BF16 rows, G, dG, w*h, dh'), with the
stated GEMM tolerance |err| <= 1e-5 * sum|a b| + 1e-6 in FP32 and one
BF16 ulp for BF16 outputs; the elementwise SwiGLU backward with a bound derived
from its FP32 arithmetic.  End to end, the gradients are compared with the
oracle's exact fp64 gradient of the unquantized layer (R16); BF16 storage of
the intermediates bounds that difference, which is reported and capped."""
import numpy as np
import pytest
import torch

from oracle import cpp
from nvfp4_moe_grouped_token_b200 import ops, workloads

from _parity import bf16_ulp, check_bf16, check_f32, expert_of_rows, gemm_bound, padded_rows

pytestmark = pytest.mark.gpu


def _f64(t):
    return t.float().cpu().numpy().astype(np.float64)


class Bwd:
    def __init__(self, cfg, flags=ops.BWD_KEEP_DH, dy_seed=77):
        self.cfg = cfg
        self.flags = flags
        inp = workloads.layer_inputs(cfg)
        self.inp = inp
        T, H, I, E, k = cfg.T, cfg.H, cfg.I, cfg.E, cfg.k
        g = torch.Generator().manual_seed(dy_seed)
        self.dy = torch.randn(T, H, generator=g).to(torch.bfloat16)
        dev = "cuda"
        self.d = {key: inp[key].to(dev) for key in ("x", "topk_idx", "topk_w", "w_gate_up", "w_down")}
        self.dy_d = self.dy.to(dev)
        self.ws = torch.zeros(ops.moe_expert_layer_backward_workspace_size(T, H, I, E, k, flags), dtype=torch.uint8,
                              device=dev)
        self.dx = torch.empty(T, H, dtype=torch.bfloat16, device=dev)
        self.dtw = torch.empty(T, k, dtype=torch.float32, device=dev)
        self.dwgu_f = torch.empty(E, 2 * I, H, dtype=torch.float32, device=dev)
        self.dwgu_b = torch.empty(E, 2 * I, H, dtype=torch.bfloat16, device=dev)
        self.dwdn_f = torch.empty(E, H, I, dtype=torch.float32, device=dev)
        self.dwdn_b = torch.empty(E, H, I, dtype=torch.bfloat16, device=dev)

    def run(self):
        d = self.d
        ops.moe_expert_layer_backward(d["x"], d["topk_idx"], d["topk_w"], d["w_gate_up"], d["w_down"], self.dy_d,
                                      self.dx, self.dtw, self.ws, dw_gate_up_bf16=self.dwgu_b,
                                      dw_gate_up_f32=self.dwgu_f, dw_down_bf16=self.dwdn_b, dw_down_f32=self.dwdn_f,
                                      flags=self.flags)
        assert ops.device_status(self.ws) == 0
        c = self.cfg
        self.v = ops.backward_views(self.ws, c.T, c.H, c.I, c.E, c.k, self.flags)

    def check(self, sample_tokens=None, experts=None):
        c = self.cfg
        T, H, I, E, k = c.T, c.H, c.I, c.E, c.k
        v = self.v
        x = self.inp["x"].float().numpy()
        idx = self.inp["topk_idx"].numpy()
        tw = self.inp["topk_w"].numpy()
        dy = self.dy.float().numpy()
        wgu = self.inp["w_gate_up"].float().numpy().astype(np.float64)
        wdn = self.inp["w_down"].float().numpy().astype(np.float64)
        info = cpp.permutation(idx, E)
        for key in ("offsets", "padded_offsets", "perm"):
            assert np.array_equal(v[key].cpu().numpy(), info[key]), key
        prow_all = padded_rows(info)
        tok_all = info["perm"] // k
        e_all = expert_of_rows(info["offsets"])
        if sample_tokens is None:
            rows = np.arange(T * k)
            toks = np.arange(T)
        else:
            toks = np.asarray(sample_tokens)
            rows = np.sort(info["inv_perm"][toks].reshape(-1))
        pr, tok, e_of = prow_all[rows], tok_all[rows], e_all[rows]

        # gather (exact): rows of x and dy, row weights, zero padding rows
        xr = _f64(v["x_rows"])
        dyr = _f64(v["dy_rows"])
        wr = v["w_rows"].cpu().numpy().astype(np.float64)
        assert np.array_equal(xr[pr], x[tok]) and np.array_equal(dyr[pr], dy[tok])
        assert np.array_equal(wr[pr], tw.reshape(-1)[info["perm"][rows]].astype(np.float64))
        used = int(info["padded_offsets"][-1])
        pad_rows = np.setdiff1d(np.arange(used), prow_all)
        assert not xr[pad_rows].any() and not dyr[pad_rows].any() and not wr[pad_rows].any()

        G = _f64(v["g"])
        dh = v["dh"].cpu().numpy().astype(np.float64)
        dG = _f64(v["dg"])
        hw = _f64(v["hw"])
        dxr = _f64(v["dx_rows"])
        for e in np.unique(e_of):
            m = e_of == e
            # G = x_rows W_gu^T (BF16 out)
            ex, sa = cpp.gemm_rows(xr[pr[m]], wgu[e], with_abs=True)
            check_bf16(G[pr[m]], ex, gemm_bound(sa), "G")
            # dh' = dy_rows W_dn (FP32, kept)
            ex, sa = cpp.gemm_rows(dyr[pr[m]], wdn[e].T, with_abs=True)
            check_f32(dh[pr[m]], ex, sa, "dh'")
            # dx rows = dG W_gu (BF16 out, compact rows)
            ex, sa = cpp.gemm_rows(dG[pr[m]], wgu[e].T, with_abs=True)
            check_bf16(dxr[rows[m]], ex, gemm_bound(sa), "dx rows")

        # SwiGLU backward from the GPU's G and dh' (FP32 arithmetic on the GPU)
        dgu_ex, h_ex = cpp.swiglu_backward(G[pr], dh[pr], wr[pr])
        check_bf16(dG[pr], dgu_ex, 1e-5 * np.abs(dgu_ex) + 1e-30, "dG")
        w_col = wr[pr][:, None]
        bound_hw = np.abs(w_col) * bf16_ulp(h_ex) + bf16_ulp(hw[pr]) + 1e-6 * np.abs(w_col * h_ex)
        assert np.all(np.abs(hw[pr] - w_col * h_ex) <= bound_hw), "w*h"
        part = v["dw_part"].cpu().numpy().astype(np.float64)[pr]
        prod = dh[pr] * h_ex
        want = prod.reshape(len(pr), I // 128, 128).sum(axis=2)
        slack = (np.abs(dh[pr]) * bf16_ulp(h_ex)).reshape(len(pr), I // 128, 128).sum(axis=2)
        fp32 = 128 * 2.0 ** -23 * np.abs(prod).reshape(len(pr), I // 128, 128).sum(axis=2)
        assert np.all(np.abs(part - want) <= slack + fp32 + 1e-30), "<dh', h> partials"

        # d topk_w: the row's partials summed in order (FP32)
        dtw = self.dtw.cpu().numpy().astype(np.float64)
        allpart = v["dw_part"].cpu().numpy().astype(np.float64)
        for t in toks:
            for j in range(k):
                p = prow_all[info["inv_perm"][t, j]]
                s = allpart[p].sum()
                assert abs(dtw[t, j] - s) <= I // 128 * 2.0 ** -23 * np.abs(allpart[p]).sum() + 1e-30
        # dx[t] = sum_j dx_rows[inv_perm[t][j]] (FP32 sum in slot order, BF16)
        dx = _f64(self.dx)
        s = np.zeros((len(toks), H))
        sa = np.zeros((len(toks), H))
        for j in range(k):
            s += dxr[info["inv_perm"][toks, j]]
            sa += np.abs(dxr[info["inv_perm"][toks, j]])
        check_bf16(dx[toks], s, k * 2.0 ** -23 * sa + 1e-30, "dx")

        # weight gradients: per expert, K over the group's rows
        off = info["offsets"]
        pad = info["padded_offsets"]
        dwgu = self.dwgu_f.cpu().numpy()
        dwdn = self.dwdn_f.cpu().numpy()
        for e in (range(E) if experts is None else experts):
            lo, hi = int(pad[e]), int(pad[e] + off[e + 1] - off[e])
            if hi == lo:
                assert not dwgu[e].any() and not dwdn[e].any(), f"empty expert {e}"
                continue
            ex, sa = cpp.gemm_rows(dyr[lo:hi].T, hw[lo:hi].T, with_abs=True)
            check_f32(dwdn[e], ex, sa, f"dW_down[{e}]")
            ex, sa = cpp.gemm_rows(dG[lo:hi].T, xr[lo:hi].T, with_abs=True)
            check_f32(dwgu[e], ex, sa, f"dW_gate_up[{e}]")
        # the BF16 outputs are the FP32 ones rounded once
        assert torch.equal(self.dwgu_f.to(torch.bfloat16).view(torch.int16), self.dwgu_b.view(torch.int16))
        assert torch.equal(self.dwdn_f.to(torch.bfloat16).view(torch.int16), self.dwdn_b.view(torch.int16))

    def end_to_end(self):
        """Against the exact fp64 gradient of the unquantized layer (R16)."""
        i = self.inp
        ref = cpp.expert_layer_backward(i["x"].float().numpy(), i["topk_idx"].numpy(), i["topk_w"].numpy(),
                                        i["w_gate_up"].float().numpy(), i["w_down"].float().numpy(),
                                        self.dy.float().numpy())
        got = {"dx": _f64(self.dx), "dw": self.dtw.cpu().numpy().astype(np.float64),
               "dw_gate_up": self.dwgu_f.cpu().numpy().astype(np.float64),
               "dw_down": self.dwdn_f.cpu().numpy().astype(np.float64)}
        rel = {key: float(np.linalg.norm(got[key] - ref[key]) / np.linalg.norm(ref[key])) for key in ref}
        print("backward relative L2 vs exact fp64 gradient:", rel)
        for key, r in rel.items():
            assert r < 2e-2, (key, r)
        return rel


SMALL = workloads.LayerConfig("small_bwd", T=300, H=256, I=256, E=8, k=2, seed=23)


def test_backward_small_all_rows():
    b = Bwd(SMALL)
    b.run()
    b.check()
    b.end_to_end()


def test_backward_with_empty_experts_and_ragged_groups():
    """Experts 5..9 receive no rows (their weight gradients are zero); group
    sizes are ragged (not multiples of 64 or 128)."""
    cfg = workloads.LayerConfig("ragged_bwd", T=333, H=512, I=256, E=10, k=3, seed=24)
    b = Bwd(cfg)
    g = torch.Generator().manual_seed(5)
    keys = torch.rand(cfg.T, 5, generator=g)
    b.inp["topk_idx"] = torch.argsort(keys, dim=1)[:, :cfg.k].to(torch.int32).contiguous()
    b.d["topk_idx"] = b.inp["topk_idx"].cuda()
    b.run()
    b.check()
    b.end_to_end()


def test_backward_wide_row_scales():
    """Rows of x scaled by 2^-20 .. 2^20: G reaches far below -64, where the
    sigmoid's e^-g overflows binary32; dG, w*h and the <dh', h> partials must
    still match the exact SwiGLU backward of the GPU's own G."""
    b = Bwd(SMALL)
    g = torch.Generator().manual_seed(13)
    sc = torch.exp2(torch.randint(-20, 21, (SMALL.T, 1), generator=g).float())
    b.inp["x"] = (b.inp["x"].float() * sc).to(torch.bfloat16)
    b.d["x"] = b.inp["x"].cuda()
    b.run()
    b.check()


def test_backward_without_keep_dh_matches():
    """The debug copy of dh' changes nothing else."""
    a = Bwd(SMALL)
    a.run()
    b = Bwd(SMALL, flags=0)
    b.run()
    for name in ("dx", "dtw", "dwgu_f", "dwdn_f"):
        assert torch.equal(getattr(a, name).view(torch.int32 if getattr(a, name).dtype == torch.float32 else
                                                 torch.int16),
                           getattr(b, name).view(torch.int32 if getattr(b, name).dtype == torch.float32 else
                                                 torch.int16)), name


def test_backward_moe30b_sampled():
    cfg = workloads.CONFIGS["moe30b"]
    b = Bwd(cfg)
    b.run()
    b.check(sample_tokens=np.arange(0, cfg.T, 1021), experts=[0, 77])
