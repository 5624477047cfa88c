"""Host logic of the multi-GPU benchmark path (independent replicas, one process
per GPU) on CPU ranks: world size 2 over gloo on 127.0.0.1."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import datetime
    import sys

    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        per_rank_ms = [120.0, 175.5][rank]
        mx = bench.reduce_max(per_rank_ms)
        out[rank] = (mx, bench.whole_job_ms_per_layer(mx, steps=5, world=world))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_reduce_max_and_whole_job_rate_over_two_gloo_ranks():
    port = _free_port()
    with mp.get_context("spawn").Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_worker, args=(2, port, out), nprocs=2, join=True)
        res = dict(out)
    assert res[0] == res[1]
    mx, per_layer = res[0]
    assert mx == pytest.approx(175.5)
    assert per_layer == pytest.approx(175.5 / (5 * 2))


def test_single_process_is_identity():
    import bench

    assert bench.reduce_max(3.25) == 3.25
    assert bench.whole_job_ms_per_layer(100.0, 4, 1) == 25.0


def _shard_worker(rank, world, port, out):
    import datetime
    import sys

    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        (qa, qb), (ka, kb) = bench.shard_heads(32, 8, world, rank)
        t = torch.tensor([qa, qb, ka, kb], dtype=torch.int64)
        allt = [torch.zeros(4, dtype=torch.int64) for _ in range(world)]
        dist.all_gather(allt, t)
        mx = bench.reduce_max([80.0, 95.0][rank])
        out[rank] = ([x.tolist() for x in allt], bench.whole_job_ms_per_layer(mx, steps=5, world=world, sharded=True))
    finally:
        dist.destroy_process_group()


def test_head_sharding_covers_every_head_once_over_two_gloo_ranks():
    port = _free_port()
    with mp.get_context("spawn").Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_shard_worker, args=(2, port, out), nprocs=2, join=True)
        res = dict(out)
    ranges, per_layer = res[0]
    assert res[1][0] == ranges
    q_heads = [h for qa, qb, _, _ in ranges for h in range(qa, qb)]
    kv_heads = [g for _, _, ka, kb in ranges for g in range(ka, kb)]
    assert q_heads == list(range(32)) and kv_heads == list(range(8))
    for qa, qb, ka, kb in ranges:  # each rank's query heads read only its own KV heads
        assert all(ka <= h // 4 < kb for h in range(qa, qb))
    assert per_layer == pytest.approx(95.0 / 5)


def test_head_sharding_rejects_uneven_split():
    import bench

    with pytest.raises(ValueError):
        bench.shard_heads(40, 8, 3, 0)
    assert bench.shard_heads(40, 8, 8, 7) == ((35, 40), (7, 8))
