"""Multi-rank host logic of bench.py on CPU: gloo, world size 2.

Each rank runs its own canvases (replicas, no collective on the data path);
the only collectives are the barrier and the max-over-ranks reduction of the
timed region, and the whole-job value counts every rank's steps over the
slowest rank's time.
"""
import os
import socket

import pytest
import torch.multiprocessing as mp

from parity import reduce_partials_local


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    import datetime

    import torch.distributed as dist

    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        dist.barrier()
        ms = 10.0 + 5.0 * rank                      # the second rank is slower
        slowest = bench.max_over_ranks(ms, dist, "cpu")
        q.put((rank, slowest, bench.whole_job_rate(100, world, slowest)))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_the_slowest_time():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    assert [r[1] for r in res] == [15.0, 15.0]
    assert res[0][2] == pytest.approx(200 / 0.015)


def test_single_process_needs_no_group():
    import bench
    assert bench.max_over_ranks(3.5) == 3.5
    assert bench.whole_job_rate(10, 1, 20.0) == pytest.approx(500.0)


# --- vocabulary-parallel exchange: one sum and one max all-reduce ------------------
C_X, D_X = 4, 8


def _partials(rank):
    import torch

    import uniform_state_text_b200 as dg
    buf = torch.zeros((4 * (2 * C_X + C_X * D_X) + 16 * C_X) // 8, dtype=torch.int64)
    f, k = dg.partials_views(buf, C_X, D_X)
    f.copy_(torch.arange(f.numel(), dtype=torch.float32) * (rank + 1) + 0.25 * rank)
    # unsigned keys, some with the top bit set; rank 1 wins rows 0 and 3
    vals = [[0x8000000000000005, 7], [0x7FFFFFFF00000000, 9], [3, 0xC000000000000000], [1, 2]]
    if rank == 1:
        vals = [[0x8000000000000006, 6], [0x7FFFFFFE00000000, 1], [2, 0xBFFFFFFFFFFFFFFF], [5, 2]]
    flat = [v for row in vals for v in row]
    k.copy_(torch.tensor([v - (1 << 64) if v >= 1 << 63 else v for v in flat], dtype=torch.int64))
    return buf


def _exchange_rank(rank, world, port, q):
    import datetime

    import torch.distributed as dist

    import uniform_state_text_b200 as dg
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        buf = _partials(rank)
        dg.allreduce_partials(buf, C_X, D_X)
        q.put((rank, buf.tolist()))
    finally:
        dist.destroy_process_group()


def test_vocab_parallel_exchange_two_gloo_ranks():
    import torch

    import uniform_state_text_b200 as dg
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_exchange_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = dict(q.get(timeout=10) for _ in range(world))
    assert res[0] == res[1]                       # every rank holds the same result
    got = torch.tensor(res[0], dtype=torch.int64)
    f, k = dg.partials_views(got, C_X, D_X)
    f0, _ = dg.partials_views(_partials(0), C_X, D_X)
    f1, _ = dg.partials_views(_partials(1), C_X, D_X)
    assert torch.equal(f, f0 + f1)
    want = [0x8000000000000006, 7, 0x7FFFFFFF00000000, 9, 3, 0xC000000000000000, 5, 2]
    assert [v % (1 << 64) for v in k.tolist()] == want
    # the single-process helper gives the same buffers
    a, b = _partials(0), _partials(1)
    reduce_partials_local([a, b], C_X, D_X)
    assert torch.equal(a, got) and torch.equal(b, got)


# --- bench.py --parallel vocab: the per-step orchestration on two gloo ranks ---------
class _FakeShard:
    """Stands in for a vocabulary-shard Denoiser: its partial step writes this
    rank's partial row results, its finish records what the exchange left."""

    def __init__(self, rank):
        self.rank = rank
        self.calls = []
        self.seen = None

    def step_partial(self, buf):
        self.calls.append("partial")
        buf.copy_(_partials(self.rank))

    def step_finish(self, buf):
        self.calls.append("finish")
        self.seen = buf.clone()


def _vocab_loop_rank(rank, world, port, q):
    import datetime

    import torch
    import torch.distributed as dist

    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        den = _FakeShard(rank)
        buf = torch.zeros_like(_partials(0))
        for _ in range(2):
            bench.vocab_parallel_loop(den, buf, C_X, D_X)
        q.put((rank, den.calls, den.seen.tolist()))
    finally:
        dist.destroy_process_group()


def test_vocab_parallel_bench_loop_two_gloo_ranks():
    """Each step: the shard's partial step, the exchange, then the finish, on every
    rank; the finish sees the reduction of both ranks' partials."""
    import torch

    import uniform_state_text_b200 as dg
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_vocab_loop_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = {r: (calls, seen) for r, calls, seen in (q.get(timeout=10) for _ in range(world))}
    for r in range(world):
        assert res[r][0] == ["partial", "finish"] * 2
    assert res[0][1] == res[1][1]
    a, b = _partials(0), _partials(1)
    reduce_partials_local([a, b], C_X, D_X)
    assert torch.equal(torch.tensor(res[0][1], dtype=torch.int64), a)


def test_strong_scaling_rate():
    import bench
    assert bench.shared_canvas_rate(100, 50.0) == pytest.approx(2000.0)
