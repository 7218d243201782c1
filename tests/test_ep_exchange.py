"""The expert-parallel exchanges (nvfp4_moe_grouped_token_b200.ep), checked
with world_size 2 over gloo on CPU: the [G][El] counts arrive transposed
(rows from each source), rows travel along the splits and arrive
source-major, and the reverse exchange brings every row back to where it was
sent from, in its original order.  The splits are built exactly as the
source side builds them from its compact expert offsets."""
import os
import socket

import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    from nvfp4_moe_grouped_token_b200 import ep
    E, El = 6, 3
    # this rank's rows per (destination, local expert): deliberately uneven, one empty pair
    counts = torch.tensor([[2, 0, 1], [1, 3, 0]], dtype=torch.int32) + rank
    splits = counts.sum(dim=1).tolist()
    R = int(counts.sum())
    # row payload: (source rank, row index) in two columns of a uint8 "codes" tensor
    rows = torch.stack([torch.full((R,), rank, dtype=torch.uint8), torch.arange(R, dtype=torch.uint8)], dim=1)
    counts_recv = ep.exchange_counts(counts)
    recv_splits = counts_recv.sum(dim=1).tolist()
    got = ep.exchange_rows(rows, splits, recv_splits)
    back = ep.exchange_rows(got, recv_splits, splits)
    out[rank] = {"counts": counts.tolist(), "counts_recv": counts_recv.tolist(), "got": got.tolist(),
                 "back_equal": torch.equal(back, rows), "E": E, "El": El}
    dist.destroy_process_group()


def test_two_rank_exchange_counts_rows_and_return():
    world = 2
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
        res = dict(out)
    for g in range(world):
        # counts received by rank g: row s = what source s sends to g
        assert res[g]["counts_recv"] == [res[s]["counts"][g] for s in range(world)]
        # rows received by g: source-major, each source's slice for g in its order
        want = []
        for s in range(world):
            c = res[s]["counts"]
            lo = sum(sum(row) for row in c[:g])
            want += [[s, i] for i in range(lo, lo + sum(c[g]))]
        assert res[g]["got"] == want
        assert res[g]["back_equal"]
