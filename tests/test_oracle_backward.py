"""Pins of the backward oracle (reading R16: the BF16-backward mode, the
quantizers treated as the identity).  Its gradients are checked against
torch.autograd in float64 on an independent formulation of the layer (a loop
over tokens and slots: no permutation, no grouped GEMM) and against central
finite differences of the oracle's own exact forward."""
import numpy as np
import torch

from oracle import backward, moe


def _problem(T=7, H=16, I=8, E=4, k=2, seed=0):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((T, H))
    wgu = rng.standard_normal((E, 2 * I, H)) * 0.3
    wdn = rng.standard_normal((E, H, I)) * 0.3
    idx = np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32)
    w = rng.random((T, k))
    w = w / w.sum(axis=1, keepdims=True)
    dy = rng.standard_normal((T, H))
    return x, idx, w, wgu, wdn, dy


def _torch_grads(x, idx, w, wgu, wdn, dy):
    X = torch.tensor(x, dtype=torch.float64, requires_grad=True)
    W = torch.tensor(w, dtype=torch.float64, requires_grad=True)
    GU = torch.tensor(wgu, dtype=torch.float64, requires_grad=True)
    DN = torch.tensor(wdn, dtype=torch.float64, requires_grad=True)
    inter = wgu.shape[1] // 2
    ys = []
    for t in range(x.shape[0]):
        yt = torch.zeros(x.shape[1], dtype=torch.float64)
        for j in range(idx.shape[1]):
            e = int(idx[t, j])
            gu = GU[e] @ X[t]
            h = torch.nn.functional.silu(gu[:inter]) * gu[inter:]
            yt = yt + W[t, j] * (DN[e] @ h)
        ys.append(yt)
    y = torch.stack(ys)
    (y * torch.tensor(dy, dtype=torch.float64)).sum().backward()
    return y.detach().numpy(), {"dx": X.grad.numpy(), "dw": W.grad.numpy(), "dw_gate_up": GU.grad.numpy(),
                                "dw_down": DN.grad.numpy()}


def test_forward_exact_matches_an_independent_formulation():
    x, idx, w, wgu, wdn, dy = _problem()
    y, _ = backward.expert_layer_forward_exact(x, idx, w, wgu, wdn)
    y_ref, _ = _torch_grads(x, idx, w, wgu, wdn, dy)
    assert np.allclose(y, y_ref, rtol=1e-12, atol=1e-12)


def test_gradients_match_autograd():
    for seed, (T, H, I, E, k) in enumerate([(7, 16, 8, 4, 2), (12, 8, 4, 6, 3), (5, 32, 16, 1, 1)]):
        x, idx, w, wgu, wdn, dy = _problem(T, H, I, E, k, seed)
        got = backward.expert_layer_backward(x, idx, w, wgu, wdn, dy)
        _, ref = _torch_grads(x, idx, w, wgu, wdn, dy)
        for key in ("dx", "dw", "dw_gate_up", "dw_down"):
            assert np.allclose(got[key], ref[key], rtol=1e-10, atol=1e-12), key


def test_gradients_match_central_differences():
    x, idx, w, wgu, wdn, dy = _problem(T=4, H=6, I=3, E=3, k=2, seed=7)
    got = backward.expert_layer_backward(x, idx, w, wgu, wdn, dy)

    def loss(x_, w_, gu_, dn_):
        y, _ = backward.expert_layer_forward_exact(x_, idx, w_, gu_, dn_)
        return float((y * dy).sum())

    eps = 1e-6
    rng = np.random.default_rng(1)
    for name, arr, grad in (("x", x, got["dx"]), ("w", w, got["dw"]), ("gu", wgu, got["dw_gate_up"]),
                            ("dn", wdn, got["dw_down"])):
        for _ in range(6):
            pos = tuple(rng.integers(0, s) for s in arr.shape)
            plus, minus = arr.copy(), arr.copy()
            plus[pos] += eps
            minus[pos] -= eps
            args_p = {"x": x, "w": w, "gu": wgu, "dn": wdn}
            args_m = dict(args_p)
            args_p[name], args_m[name] = plus, minus
            fd = (loss(args_p["x"], args_p["w"], args_p["gu"], args_p["dn"]) -
                  loss(args_m["x"], args_m["w"], args_m["gu"], args_m["dn"])) / (2 * eps)
            assert abs(fd - grad[pos]) <= 1e-6 * max(1.0, abs(fd)), (name, pos, fd, grad[pos])


def test_unrouted_expert_gets_zero_weight_gradient():
    x, idx, w, wgu, wdn, dy = _problem(T=6, H=8, I=4, E=5, k=2, seed=3)
    idx = np.where(idx == 4, 0, idx).astype(np.int32)     # expert 4 receives no token
    idx[:, 1] = np.where(idx[:, 1] == idx[:, 0], (idx[:, 0] + 1) % 4, idx[:, 1])
    got = backward.expert_layer_backward(x, idx, w, wgu, wdn, dy)
    assert not got["dw_gate_up"][4].any() and not got["dw_down"][4].any()
    assert got["dw_gate_up"][:4].any()


def test_silu_grad_closed_form_points():
    # silu'(0) = 1/2; silu' -> 1 for large g and -> 0 for very negative g
    assert backward.silu_grad(np.array([0.0]))[0] == 0.5
    assert abs(backward.silu_grad(np.array([40.0]))[0] - 1.0) < 1e-12
    assert abs(backward.silu_grad(np.array([-40.0]))[0]) < 1e-12
    g = np.linspace(-5, 5, 11)
    fd = (moe.silu(g + 1e-6) - moe.silu(g - 1e-6)) / 2e-6
    assert np.allclose(backward.silu_grad(g), fd, rtol=1e-7, atol=1e-9)
