"""GPU permutation parity: offsets, padded offsets, perm and inv_perm are
bit-exact with the oracle; bad routing is reported, never written out of
bounds."""
import numpy as np
import pytest
import torch

from oracle import cpp
from nvfp4_moe_grouped_token_b200 import ops, workloads

pytestmark = pytest.mark.gpu


def _gpu_permute(idx_cpu, E):
    T, k = idx_cpu.shape
    idx = idx_cpu.cuda()
    off = torch.full((E + 1,), -1, dtype=torch.int32, device="cuda")
    pad = torch.full((E + 1,), -1, dtype=torch.int32, device="cuda")
    perm = torch.full((max(T * k, 1),), -1, dtype=torch.int32, device="cuda")
    inv = torch.full((T, k), -1, dtype=torch.int32, device="cuda")
    ws = torch.zeros(ops.moe_permute_workspace_size(T, k, E), dtype=torch.uint8, device="cuda")
    ops.moe_permute(idx, E, off, pad, perm, inv, ws)
    st = ops.device_status(ws)
    return off.cpu().numpy(), pad.cpu().numpy(), perm.cpu().numpy()[: T * k], inv.cpu().numpy(), st


def _check(idx_cpu, E):
    off, pad, perm, inv, st = _gpu_permute(idx_cpu, E)
    assert st == 0
    r = cpp.permutation(idx_cpu.numpy(), E)
    assert np.array_equal(off, r["offsets"])
    assert np.array_equal(pad, r["padded_offsets"])
    assert np.array_equal(perm, r["perm"])
    assert np.array_equal(inv, r["inv_perm"])
    return r


@pytest.mark.parametrize("name", ["toy", "moe30b", "moe30b_skew", "strict"])
def test_permute_configs(name):
    cfg = workloads.CONFIGS[name]
    idx, _ = workloads.routing(cfg)
    r = _check(idx, cfg.E)
    if name == "moe30b_skew":
        share = r["counts"] / r["counts"].sum()
        empty = int((r["counts"] == 0).sum())
        assert share.max() > 0.05 and 5 <= empty <= 20, (share.max(), empty)


@pytest.mark.parametrize("T,k,E", [(1, 1, 1), (1, 8, 128), (7, 3, 5), (129, 2, 1024), (300, 4, 300),
                                   (4096, 1, 1), (1000, 32, 40)])
def test_permute_edge_shapes(T, k, E):
    rng = np.random.default_rng(T + k + E)
    idx = np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32)
    _check(torch.from_numpy(idx), E)


def test_permute_empty_experts_and_skew():
    T, k, E = 2000, 2, 64
    idx = torch.stack([torch.zeros(T, dtype=torch.int32), torch.full((T,), 63, dtype=torch.int32)], 1)
    idx[::5, 1] = 17
    r = _check(idx, E)
    assert (r["counts"] == 0).sum() == 61


def test_permute_reports_bad_and_duplicate_experts():
    T, k, E = 64, 2, 8
    idx = torch.randint(0, E, (T, k), dtype=torch.int32)
    idx[:, 1] = (idx[:, 0] + 1) % E
    idx[3, 1] = 99          # out of range
    _, _, _, _, st = _gpu_permute(idx, E)
    assert st == ops.ERR_DEVICE_CHECK
    idx[3, 1] = idx[3, 0]   # duplicate
    _, _, _, _, st = _gpu_permute(idx, E)
    assert st == ops.ERR_DEVICE_CHECK
    idx[3, 1] = (idx[3, 0] + 1) % E
    _, _, _, _, st = _gpu_permute(idx, E)
    assert st == 0


def test_permute_zero_tokens():
    off, pad, perm, inv, st = _gpu_permute(torch.zeros(0, 2, dtype=torch.int32), 4)
    assert st == 0 and not off.any() and not pad.any()
