"""Expert parallelism on the GPU: G ranks, each owning E/G experts, with the
rows exchanged in NVFP4.  One GPU stands in for the G ranks (the exchanges
are device copies in the order the all-to-alls deliver them; no kernel waits
on another rank), and a one-rank NCCL group runs the collective path itself.

The layer with per-token (strict) scaling is batch invariant, so every rank's
y must equal, bit for bit, the single-GPU strict layer's y for the same
tokens: the codes, each row's GEMM and each combine are the same."""
import os
import socket

import numpy as np
import pytest
import torch

from nvfp4_moe_grouped_token_b200 import ep, ops, workloads

pytestmark = pytest.mark.gpu


def _strict_layer(inp, wgu, wdn, cfg):
    ws = torch.zeros(ops.moe_expert_layer_workspace_size(cfg.T, cfg.H, cfg.I, cfg.E, cfg.k, ops.STRICT),
                     dtype=torch.uint8, device="cuda")
    y = torch.empty(cfg.T, cfg.H, dtype=torch.bfloat16, device="cuda")
    ops.moe_expert_layer(inp["x"].cuda(), inp["topk_idx"].cuda(), inp["topk_w"].cuda(), wgu, wdn, y, ws, ops.STRICT)
    assert ops.device_status(ws) == 0
    return y


def _run_local(cfg, inp, G, bounds):
    wgu = ops.nvfp4_prepare_weights(inp["w_gate_up"].cuda(), gate_up=True)
    wdn = ops.nvfp4_prepare_weights(inp["w_down"].cuda(), gate_up=False)
    y_ref = _strict_layer(inp, wgu, wdn, cfg)
    xs, idxs, tws, ys = [], [], [], []
    for g in range(G):
        lo, hi = bounds[g], bounds[g + 1]
        xs.append(inp["x"][lo:hi].contiguous().cuda())
        idxs.append(inp["topk_idx"][lo:hi].contiguous().cuda())
        tws.append(inp["topk_w"][lo:hi].contiguous().cuda())
        ys.append(torch.full((hi - lo, cfg.H), float("nan"), dtype=torch.bfloat16, device="cuda"))
    rc = ep.moe_expert_layer_ep_local(xs, idxs, tws, [ep.local_weights(wgu, g, G) for g in range(G)],
                                      [ep.local_weights(wdn, g, G) for g in range(G)], ys, cfg.E)
    assert rc == ops.OK
    y_ep = torch.cat(ys)
    assert torch.equal(y_ep.view(torch.int16), y_ref.view(torch.int16))


CFG = workloads.LayerConfig("ep_small", T=333, H=512, I=256, E=8, k=2, seed=51)


@pytest.mark.parametrize("G,bounds", [(1, [0, 333]), (2, [0, 100, 333]), (4, [0, 90, 90, 200, 333])])
def test_ep_equals_the_strict_layer(G, bounds):
    """Ragged token splits; with G = 4 one rank has no tokens."""
    _run_local(CFG, workloads.layer_inputs(CFG), G, bounds)


def test_ep_rank_without_rows():
    """Routing to experts 0-3 only: with G = 2 the second rank's experts get
    no rows (it receives nothing and returns nothing)."""
    inp = workloads.layer_inputs(CFG)
    g = torch.Generator().manual_seed(4)
    keys = torch.rand(CFG.T, 4, generator=g)
    inp["topk_idx"] = torch.argsort(keys, dim=1)[:, :CFG.k].to(torch.int32).contiguous()
    _run_local(CFG, inp, 2, [0, 150, 333])


def test_ep_moe30b_four_ranks():
    """The Qwen3-30B-A3B-shaped layer over 4 ranks (32 experts each)."""
    cfg = workloads.CONFIGS["moe30b"]
    T = cfg.T
    _run_local(cfg, workloads.layer_inputs(cfg), 4, [0, T // 4, T // 2, 3 * T // 4, T])


def test_ep_through_a_one_rank_nccl_group():
    """moe_expert_layer_ep with a real NCCL process group of one rank: the
    counts and rows go through all_to_all_single."""
    import torch.distributed as dist

    cfg = CFG
    inp = workloads.layer_inputs(cfg)
    wgu = ops.nvfp4_prepare_weights(inp["w_gate_up"].cuda(), gate_up=True)
    wdn = ops.nvfp4_prepare_weights(inp["w_down"].cuda(), gate_up=False)
    y_ref = _strict_layer(inp, wgu, wdn, cfg)
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                            device_id=torch.device("cuda", 0))
    try:
        y = torch.empty(cfg.T, cfg.H, dtype=torch.bfloat16, device="cuda")
        rc = ep.moe_expert_layer_ep(inp["x"].cuda(), inp["topk_idx"].cuda(), inp["topk_w"].cuda(), wgu, wdn, y,
                                    cfg.E)
        torch.cuda.synchronize()
        assert rc == ops.OK
        assert torch.equal(y.view(torch.int16), y_ref.view(torch.int16))
    finally:
        dist.destroy_process_group()


def test_ep_arrange_rejects_a_short_layout():
    """rows_cap below moe_ep_rows_cap is refused before any launch."""
    counts = torch.tensor([[3, 0], [1, 2]], dtype=torch.int32, device="cuda")
    rows = 6
    cap = ops.moe_ep_rows_cap(rows, 2)
    H = 256
    q = torch.zeros(rows, H // 2, dtype=torch.uint8, device="cuda")
    sf = torch.zeros(rows, H // 16, dtype=torch.uint8, device="cuda")
    sd = torch.zeros(rows, dtype=torch.float32, device="cuda")
    short = cap - 128
    qa = torch.empty(short, H // 2, dtype=torch.uint8, device="cuda")
    sfa = torch.empty(short * H // 16, dtype=torch.uint8, device="cuda")
    sda = torch.empty(short, dtype=torch.float32, device="cuda")
    off = torch.empty(3, dtype=torch.int32, device="cuda")
    pad = torch.empty(3, dtype=torch.int32, device="cuda")
    ws = torch.empty(ops.moe_ep_arrange_workspace_size(2, 2), dtype=torch.uint8, device="cuda")
    with pytest.raises(ops.NVFP4Error):
        ops.moe_ep_arrange(q, sf, sd, counts, 2, 2, H, short, qa, sfa, sda, off, pad, ws)
