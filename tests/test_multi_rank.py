"""The multi-GPU path is data-parallel replicas (no data-path collective):
its host logic -- per-rank token shards, max-over-ranks timing, whole-job
throughput -- checked with world_size 2 over gloo on CPU."""
import os
import socket

import pytest
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
    import bench
    from nvfp4_moe_grouped_token_b200 import workloads
    base = workloads.scaled(workloads.CONFIGS["moe30b"], T=64)
    cfg = bench.rank_config(base, rank, world)
    x = workloads.activations(cfg)
    idx, _ = workloads.routing(cfg)
    my_ms = 1.0 + rank                       # rank 1 is the slow one
    ms = bench.max_over_ranks(my_ms, world)
    x = x.float()
    gathered = [torch.zeros_like(x) for _ in range(world)]
    dist.all_gather(gathered, x)
    out[rank] = {
        "seed": cfg.seed,
        "ms": ms,
        "value": bench.job_throughput(cfg.T, world, ms),
        "distinct": not torch.equal(gathered[0], gathered[1]),
        "shape_same": cfg.T == base.T and cfg.H == base.H and cfg.E == base.E,
        "idx_ok": bool((idx >= 0).all() and (idx < cfg.E).all()),
    }
    dist.destroy_process_group()


def test_two_rank_replicas_shard_tokens_and_take_max_time():
    world = 2
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
        res = dict(out)
    assert res[0]["seed"] != res[1]["seed"]
    assert res[0]["distinct"] and res[1]["distinct"]
    assert res[0]["shape_same"] and res[1]["shape_same"] and res[0]["idx_ok"]
    assert res[0]["ms"] == res[1]["ms"] == 2.0                    # max over ranks
    assert res[0]["value"] == pytest.approx(2 * 64 / 2e-3)        # all ranks' tokens / slowest time


def test_single_rank_is_identity():
    import bench
    from nvfp4_moe_grouped_token_b200 import workloads
    cfg = workloads.CONFIGS["toy"]
    assert bench.rank_config(cfg, 0, 1) is cfg
    assert bench.max_over_ranks(3.5, 1) == 3.5
