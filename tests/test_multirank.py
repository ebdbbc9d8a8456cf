"""Host-side logic of the multi-GPU bench path, on world_size-2 gloo ranks (CPU).

Heads are independent, so bench.py runs one copy of the workload per rank with
no collective on the data path; the only cross-rank steps are the timing
barrier and the max-over-ranks reduction, tested here without a GPU.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port),
                      RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w, r, local = bench.dist_env()
        assert (w, r, local) == (world, rank, rank)
        bench.barrier(world)
        ms = 10.0 + rank  # rank 1 is the slow one
        worst = bench.max_over_ranks(ms, world, device="cpu")
        out[rank] = (worst, bench.whole_job_tflops(5.5e12, world, worst))
    finally:
        dist.destroy_process_group()


def test_two_rank_timing_is_max_over_ranks():
    world, port = 2, _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    assert res[0] == res[1]
    worst, value = res[0]
    assert worst == pytest.approx(11.0)
    assert value == pytest.approx(2 * 5.5e12 / 11e-3 / 1e12)


def test_single_rank_defaults(monkeypatch):
    for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    assert bench.dist_env() == (1, 0, 0)
    assert bench.max_over_ranks(3.0, 1) == 3.0
    assert bench.whole_job_tflops(1e12, 1, 1.0) == pytest.approx(1000.0)
