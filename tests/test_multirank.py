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


def test_head_ranges_cover_every_head_once():
    from causal_softmax_attention_b200.shard import head_range
    for BH in (1, 3, 4, 7, 32, 33):
        for world in (1, 2, 3, 4, 8):
            seen = []
            for r in range(world):
                s, e = head_range(BH, world, r)
                assert 0 <= s <= e <= BH
                assert e - s <= -(-BH // world)
                seen.extend(range(s, e))
            assert seen == list(range(BH)), (BH, world)


def _gather_worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from causal_softmax_attention_b200.shard import gather_heads, head_block, head_range
        B, H, N, d = 2, 3, 5, 4
        full = torch.arange(B * H * N * d, dtype=torch.float32).reshape(B, H, N, d)
        mine = torch.full_like(full, -1.0)
        s, e = head_range(B * H, world, rank)
        head_block(mine, s, e).copy_(head_block(full, s, e))  # this rank's "result"
        got = gather_heads(mine, world, rank)
        q.put((rank, bool(torch.equal(got, full)), (s, e)))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_gather_heads_reassembles_the_blocks(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_gather_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert all(ok for _, ok, _ in res), res


def test_backward_shard_hands_each_rank_its_block(monkeypatch):
    # the views passed to attn_bwd: [1, heads of the rank, N, d] starting at
    # the rank's first head, for every tensor (no GPU: attn_bwd is recorded)
    import causal_softmax_attention_b200 as csa
    from causal_softmax_attention_b200 import shard
    calls = []
    monkeypatch.setattr(csa, "attn_bwd", lambda *a, **k: calls.append(a))
    B, H, N, d = 2, 3, 4, 8
    ts = [torch.randn(B, H, N, d) for _ in range(5)] + [torch.randn(B, H, N)] + \
         [torch.zeros(B, H, N, d) for _ in range(3)]
    for world in (1, 2, 4, 8):
        for rank in range(world):
            calls.clear()
            s, e = shard.backward_shard(*ts, "ws", world, rank)
            if e == s:
                assert not calls
                continue
            (args,) = calls
            for t, blk in zip(ts, args[:9]):
                assert blk.shape == (1, e - s) + tuple(t.shape[2:])
                assert blk.data_ptr() == t.reshape(B * H, *t.shape[2:])[s].data_ptr()
            assert args[9] == "ws"


@pytest.mark.parametrize("argv", [["--layout", "bnhd", "--block-mask", "causal"],
                                  ["--block-mask", "causal", "--config", "c1"],
                                  ["--block-mask", "diagonal"],
                                  ["--warmup", "2"]])
def test_bench_rejects_contradictory_flags_before_any_gpu_work(argv):
    import subprocess
    import sys
    r = subprocess.run([sys.executable, os.path.join(os.path.dirname(bench.__file__), "bench.py"),
                        *argv], capture_output=True, text=True, timeout=120)
    assert r.returncode == 2 and "Traceback" not in r.stderr, r.stderr[-500:]
