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
