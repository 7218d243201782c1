"""Backward of the MoE expert layer -- CPU oracle (test infrastructure only).

Source passage: www.aib.vote "miniTE report, NVFP4 RL stability",
paragraph 1: besides the full NVFP4 path the report times a mode that runs the
forward in NVFP4 and the backward in BF16 (about 1.33-1.37x over BF16 for the
full training update on 8xB300).  The pages give no formulas for it.

Reading taken where the pages are silent:
  R16  BF16-backward mode: the backward is the exact gradient of the layer
       y[t] = sum_j w[t,j] * down_e(silu(gate_e(x[t])) * up_e(x[t])),
       e = topk_idx[t,j], computed on the BF16 operands (x, the BF16 weights
       and the forward's h) with every quantizer of the forward treated as
       the identity (straight-through).  All of it is fp64 here; the routing
       (topk_idx) is not differentiated, the routing weights are.

The layer gradients, for one routed row r = (t, j) of expert e, with
G = [g | u] = x W_gu,e^T, h = silu(g) u and D = h W_dn,e^T:
  dD       = w[t,j] dy[t]                      (combine)
  dw[t,j]  = <dy[t], D>
  dh       = dD W_dn,e             dW_dn,e += dD^T h     (down: dgrad, wgrad)
  dg       = dh u silu'(g),  du = dh silu(g)             (SwiGLU)
  dx[t]   += [dg | du] W_gu,e      dW_gu,e += [dg | du]^T x[t]   (gate_up)
with silu'(g) = s (1 + g (1 - s)), s = 1 / (1 + exp(-g)).
"""
from __future__ import annotations

import numpy as np

from . import moe


def sigmoid(g: np.ndarray) -> np.ndarray:
    g = np.asarray(g, dtype=np.float64)
    with np.errstate(over="ignore"):
        return 1.0 / (1.0 + np.exp(-g))


def silu_grad(g: np.ndarray) -> np.ndarray:
    """d silu(g) / dg = s (1 + g (1 - s)), s = sigmoid(g)."""
    s = sigmoid(g)
    return s * (1.0 + np.asarray(g, dtype=np.float64) * (1.0 - s))


def expert_layer_forward_exact(x, topk_idx, topk_w, w_gate_up, w_down):
    """The layer without quantization, fp64: the function R16 differentiates.
    x [T][H], topk_idx [T][k], topk_w [T][k], w_gate_up [E][2I][H], w_down [E][H][I].
    Returns y [T][H] and the per-row intermediates (rows in the sorted order of
    moe.permutation)."""
    x = np.asarray(x, dtype=np.float64)
    wgu = np.asarray(w_gate_up, dtype=np.float64)
    wdn = np.asarray(w_down, dtype=np.float64)
    T, k = topk_idx.shape
    E, N2, H = wgu.shape
    inter = N2 // 2
    info = moe.permutation(np.asarray(topk_idx), E)
    tok = info["perm"] // k
    slot = info["perm"] % k
    off = info["offsets"]
    a = x[tok]
    gu = moe.grouped_gemm(a, off, lambda e: wgu[e])
    h = moe.swiglu(gu, inter)
    d = moe.grouped_gemm(h, off, lambda e: wdn[e])
    w_rows = np.asarray(topk_w, dtype=np.float64)[tok, slot]
    y = np.zeros((T, H), dtype=np.float64)
    np.add.at(y, tok, w_rows[:, None] * d)
    return y, {"info": info, "tok": tok, "slot": slot, "gu": gu, "h": h, "d": d, "w_rows": w_rows}


def expert_layer_backward(x, topk_idx, topk_w, w_gate_up, w_down, dy):
    """R16: gradients of sum(dy * y) with respect to x, topk_w, w_gate_up and
    w_down, in fp64.  Returns dict dx [T][H], dw [T][k], dw_gate_up
    [E][2I][H], dw_down [E][H][I]."""
    x = np.asarray(x, dtype=np.float64)
    dy = np.asarray(dy, dtype=np.float64)
    wgu = np.asarray(w_gate_up, dtype=np.float64)
    wdn = np.asarray(w_down, dtype=np.float64)
    T, k = topk_idx.shape
    E, N2, H = wgu.shape
    inter = N2 // 2
    _, f = expert_layer_forward_exact(x, topk_idx, topk_w, wgu, wdn)
    tok, slot, off = f["tok"], f["slot"], f["info"]["offsets"]
    g, u = f["gu"][:, :inter], f["gu"][:, inter:]
    # combine
    d_d = f["w_rows"][:, None] * dy[tok]
    d_w = np.zeros((T, k), dtype=np.float64)
    d_w[tok, slot] = np.einsum("rh,rh->r", dy[tok], f["d"])
    # down: dgrad per expert, wgrad per expert
    d_h = moe.grouped_gemm(d_d, off, lambda e: wdn[e].T)
    dw_down = np.zeros_like(wdn)
    for e in range(E):
        lo, hi = int(off[e]), int(off[e + 1])
        if hi > lo:
            dw_down[e] = d_d[lo:hi].T @ f["h"][lo:hi]
    # SwiGLU
    d_g = d_h * u * silu_grad(g)
    d_u = d_h * moe.silu(g)
    d_gu = np.concatenate([d_g, d_u], axis=1)
    # gate_up: dgrad to the routed rows, summed back to tokens; wgrad per expert
    dx_rows = moe.grouped_gemm(d_gu, off, lambda e: wgu[e].T)
    dx = np.zeros((T, H), dtype=np.float64)
    np.add.at(dx, tok, dx_rows)
    dw_gate_up = np.zeros_like(wgu)
    a = x[tok]
    for e in range(E):
        lo, hi = int(off[e]), int(off[e + 1])
        if hi > lo:
            dw_gate_up[e] = d_gu[lo:hi].T @ a[lo:hi]
    return {"dx": dx, "dw": d_w, "dw_gate_up": dw_gate_up, "dw_down": dw_down}
