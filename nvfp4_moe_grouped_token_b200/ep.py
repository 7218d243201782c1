"""Expert parallelism for the NVFP4 MoE expert layer.

G ranks each own E / G consecutive experts (expert e lives on rank e // El).
Every step that touches the data runs in the library on the GPU:

  source       moe_ep_dispatch_pack: routing metadata, and each token
               quantized once (per-token NVFP4) into its k rows in compact
               (expert, token, slot) order, so the rows for rank g are one
               contiguous range;
  exchange     the [G][El] row counts, then the rows (codes, row-major scales,
               row S_dec), arriving source-major;
  destination  moe_ep_arrange (padded grouped layout), moe_ep_experts
               (gate_up + SwiGLU, requantization, down), moe_ep_return (D rows
               in received order);
  exchange     D rows back along the reverse splits;
  source       moe_combine in slot order with the dispatch's inv_perm.

The results equal moe_expert_layer with NVFP4MOE_STRICT bit for bit, whatever
G: each token's codes, each row's products and each combine are the same.
This module only sizes buffers, computes the exchange splits (one read of the
[E + 1] offsets back to the host) and runs the exchanges: NCCL all-to-alls in
`moe_expert_layer_ep`, or plain copies between the ranks one process drives
in `moe_expert_layer_ep_local` (one GPU standing in for G).
"""
from __future__ import annotations

import torch

from . import ops


def _empty(shape, dtype, device):
    return torch.empty(shape, dtype=dtype, device=device)


def dispatch(x, topk_idx, E: int, G: int) -> dict:
    """Source side: the rows to send, grouped by destination rank."""
    if E % G:
        raise ValueError("E must be a multiple of the number of ranks")
    T, H = x.shape
    k = topk_idx.shape[1]
    dev = x.device
    R = T * k
    out = {
        "q": _empty((R, H // 2), torch.uint8, dev),
        "sf": _empty((R, H // 16), torch.uint8, dev),
        "sdec": _empty((R,), torch.float32, dev),
        "offsets": _empty((E + 1,), torch.int32, dev),
        "inv_perm": _empty((T, k), torch.int32, dev),
        "ws": _empty((ops.moe_ep_dispatch_workspace_size(T, E, k),), torch.uint8, dev),
    }
    ops.moe_ep_dispatch_pack(x, topk_idx, E, out["q"], out["sf"], out["sdec"], out["offsets"], out["inv_perm"],
                             out["ws"])
    off = out["offsets"].cpu().to(torch.int64)          # the exchange needs its splits on the host
    El = E // G
    counts = (off[1:] - off[:-1]).view(G, El)            # [destination][local expert]
    out["counts"] = counts.to(torch.int32)
    out["splits"] = counts.sum(dim=1).tolist()
    return out


def destination(q_recv, sf_recv, sdec_recv, counts_recv, w_gate_up, w_down) -> dict:
    """Destination side: the local experts on the received rows.  counts_recv
    [G][El] (host) holds the rows from each source per local expert; returns
    the D rows in received order (`d_send`) plus the workspaces."""
    G, El = counts_recv.shape
    H = w_down.N
    I = w_down.K
    dev = q_recv.device
    rows_recv = int(counts_recv.sum())
    cap = ops.moe_ep_rows_cap(rows_recv, El)
    st = {
        "counts": counts_recv.to(device=dev, dtype=torch.int32).contiguous(),
        "q_a": _empty((cap, H // 2), torch.uint8, dev),
        "sf_a": _empty((cap * H // 16,), torch.uint8, dev),
        "sdec_a": _empty((cap,), torch.float32, dev),
        "offsets": _empty((El + 1,), torch.int32, dev),
        "padded": _empty((El + 1,), torch.int32, dev),
        "ws_arrange": _empty((ops.moe_ep_arrange_workspace_size(G, El),), torch.uint8, dev),
        "ws_experts": _empty((ops.moe_ep_experts_workspace_size(cap, H, I),), torch.uint8, dev),
        "d": _empty((rows_recv, H), torch.bfloat16, dev),
        "d_send": _empty((rows_recv, H), torch.bfloat16, dev),
        "rows_cap": cap,
    }
    if rows_recv == 0:                                   # no rows for this rank's experts
        st["ws_arrange"].zero_()
        st["ws_experts"].zero_()
        return st
    ops.moe_ep_arrange(q_recv, sf_recv, sdec_recv, st["counts"], G, El, H, cap, st["q_a"], st["sf_a"], st["sdec_a"],
                       st["offsets"], st["padded"], st["ws_arrange"])
    ops.moe_ep_experts(st["q_a"], st["sf_a"], st["sdec_a"], st["offsets"], st["padded"], cap, w_gate_up, w_down,
                       st["d"], st["ws_experts"])
    ops.moe_ep_return(st["d"], G, El, st["d_send"], st["ws_arrange"])
    return st


def device_status(src: dict, dst: dict) -> int:
    """The first device-side error of a rank's steps (0 if none)."""
    for ws in (src["ws"], dst["ws_arrange"], dst["ws_experts"]):
        rc = ops.device_status(ws)
        if rc != ops.OK:
            return rc
    return ops.OK


# ------------------------------------------------------------- exchanges --

def exchange_counts(counts_send, group=None):
    """[G][El] counts (this rank's rows per destination and local expert) ->
    [G][El] received (rows from each source per local expert), on the host."""
    import torch.distributed as dist

    dev = counts_send.device if dist.get_backend(group) != "nccl" else torch.device("cuda", torch.cuda.current_device())
    send = counts_send.to(device=dev, dtype=torch.int32).contiguous()
    recv = torch.empty_like(send)
    dist.all_to_all_single(recv, send, group=group)
    return recv.cpu()


def exchange_rows(t, send_splits, recv_splits, group=None):
    """Rows of t sent to each rank along send_splits; the received rows,
    source-major, along recv_splits."""
    import torch.distributed as dist

    out = torch.empty((int(sum(recv_splits)),) + tuple(t.shape[1:]), dtype=t.dtype, device=t.device)
    dist.all_to_all_single(out, t.contiguous(), [int(v) for v in recv_splits], [int(v) for v in send_splits],
                           group=group)
    return out


def moe_expert_layer_ep(x, topk_idx, topk_w, w_gate_up, w_down, y, E: int, group=None) -> int:
    """The layer across the ranks of `group` (torch.distributed, NCCL): this
    rank's tokens x / topk_idx / topk_w (global expert ids) in, y out; its
    weights w_gate_up / w_down hold experts [rank El, (rank + 1) El).
    Returns the first device-side error of this rank's steps (0 if none)."""
    import torch.distributed as dist

    G = dist.get_world_size(group)
    src = dispatch(x, topk_idx, E, G)
    counts_recv = exchange_counts(src["counts"], group)
    recv_splits = counts_recv.sum(dim=1).tolist()
    q = exchange_rows(src["q"], src["splits"], recv_splits, group)
    sf = exchange_rows(src["sf"], src["splits"], recv_splits, group)
    sd = exchange_rows(src["sdec"], src["splits"], recv_splits, group)
    dst = destination(q, sf, sd, counts_recv, w_gate_up, w_down)
    d_recv = exchange_rows(dst["d_send"], recv_splits, src["splits"], group)
    if x.shape[0] > 0:
        ops.moe_combine(d_recv, src["inv_perm"], topk_w, y)
    return device_status(src, dst)


def moe_expert_layer_ep_local(xs, topk_idxs, topk_ws, w_gate_ups, w_downs, ys, E: int) -> int:
    """G ranks driven by one process on one GPU: rank g's inputs are xs[g],
    topk_idxs[g], topk_ws[g], its local weights w_gate_ups[g], w_downs[g], its
    output ys[g].  The exchanges are device copies between the ranks'
    buffers, in the order the all-to-alls deliver them; every other step is
    the one moe_expert_layer_ep runs."""
    G = len(xs)
    srcs = [dispatch(xs[g], topk_idxs[g], E, G) for g in range(G)]
    dsts = []
    for g in range(G):
        counts_recv = torch.stack([srcs[s]["counts"][g] for s in range(G)])
        lo = [sum(srcs[s]["splits"][:g]) for s in range(G)]
        take = lambda key: torch.cat([srcs[s][key][lo[s]:lo[s] + srcs[s]["splits"][g]] for s in range(G)])
        dsts.append(destination(take("q"), take("sf"), take("sdec"), counts_recv, w_gate_ups[g], w_downs[g]))
    for s in range(G):
        parts = []
        for g in range(G):
            recv = torch.stack([srcs[q]["counts"][g] for q in range(G)]).sum(dim=1).tolist()
            lo = sum(recv[:s])
            parts.append(dsts[g]["d_send"][lo:lo + recv[s]])
        if xs[s].shape[0] > 0:
            ops.moe_combine(torch.cat(parts), srcs[s]["inv_perm"], topk_ws[s], ys[s])
    for g in range(G):
        rc = device_status(srcs[g], dsts[g])
        if rc != ops.OK:
            return rc
    return ops.OK


def local_weights(prep: "ops.NVFP4Weights", g: int, G: int) -> "ops.NVFP4Weights":
    """Rank g's experts of globally prepared weights (each expert is
    quantized on its own, so a slice equals preparing the slice)."""
    return prep.experts(g * (prep.E // G), (g + 1) * (prep.E // G))
