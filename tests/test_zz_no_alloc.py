"""moe_permute_noalloc: the permutation for callers that cannot provide
scratch memory (their memory planner owns all device memory, or allocation
is not allowed where they run).  Its scratch is a static device array of the
library.  Checked through the C-ABI against moe_permute, which uses a caller
workspace: offsets, padded offsets, perm and inv_perm must be identical, on
two calls in a row with different routing (the array keeps the previous
call's contents).  This file is collected last on purpose."""
import numpy as np
import pytest
import torch

from nvfp4_moe_grouped_token_b200 import ops, workloads

pytestmark = pytest.mark.gpu


def _outputs(T, k, E):
    return (torch.full((E + 1,), -1, dtype=torch.int32, device="cuda"),
            torch.full((E + 1,), -1, dtype=torch.int32, device="cuda"),
            torch.full((T * k,), -1, dtype=torch.int32, device="cuda"),
            torch.full((T, k), -1, dtype=torch.int32, device="cuda"))


def _with_workspace(idx, E):
    T, k = idx.shape
    off, pad, perm, inv = _outputs(T, k, E)
    ws = torch.zeros(ops.moe_permute_workspace_size(T, k, E), dtype=torch.uint8, device="cuda")
    ops.moe_permute(idx, E, off, pad, perm, inv, ws)
    assert ops.device_status(ws) == ops.OK
    return [t.cpu().numpy() for t in (off, pad, perm, inv)]


def _without_workspace(idx, E):
    T, k = idx.shape
    off, pad, perm, inv = _outputs(T, k, E)
    ops.moe_permute_noalloc(idx, E, off, pad, perm, inv)
    torch.cuda.synchronize()
    return [t.cpu().numpy() for t in (off, pad, perm, inv)]


def test_noalloc_permute_matches_workspace_version_twice():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    cfg = workloads.CONFIGS["moe30b"]                     # T*k = 131072: the array's full capacity
    idx1, _ = workloads.routing(cfg)
    idx2, _ = workloads.routing(workloads.scaled(cfg, T=3000, seed=77))
    for idx, E in ((idx1, cfg.E), (idx2, cfg.E)):
        idx = idx.cuda()
        want = _with_workspace(idx, E)
        got = _without_workspace(idx, E)
        for w, g in zip(want, got):
            assert np.array_equal(w, g)


def test_noalloc_permute_rejects_sizes_beyond_its_array():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    idx = torch.zeros(131072 // 8 + 1, 8, dtype=torch.int32, device="cuda")
    off, pad, perm, inv = _outputs(idx.shape[0], 8, 128)
    with pytest.raises(ops.NVFP4Error):
        ops.moe_permute_noalloc(idx, 128, off, pad, perm, inv)
