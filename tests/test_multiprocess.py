"""The N > 1 plumbing of bench.py (replicas, no exchange step) on CPU: two gloo ranks.

Each rank runs its own replica; the process group only carries the barriers around the
timed region and the max over ranks of the timings. The workload seeds differ per rank.
"""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp

import bench
from sparse_mixed_precision_b200.synth import WORKLOADS, generate


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    import torch.distributed as dist
    ws, r, _ = bench.dist_setup("gloo")
    try:
        assert (ws, r) == (world, rank)
        bench.barrier(ws)
        ms = bench.max_over_ranks(10.0 + 5.0 * rank, ws)          # rank 1 is the slowest
        w = WORKLOADS["tiny"]
        q, _, _ = generate(w, device="cpu", seed=w.seed + rank)
        digest = float(q.float().sum())
        out.put((rank, ms, digest))
        bench.barrier(ws)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_max_timing_and_distinct_replicas():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(world):
        rank, ms, digest = out.get(timeout=120)
        res[rank] = (ms, digest)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert res[0][0] == res[1][0] == 15.0                         # max over ranks
    assert res[0][1] != res[1][1]                                 # each rank its own replica
    w = WORKLOADS["wan720"]
    # weak scaling: N ranks complete N calls in the slowest rank's time
    assert bench.job_throughput(w, 2, 20.0) == pytest.approx(2 * bench.job_throughput(w, 1, 20.0))


def _seqpar_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    import torch.distributed as dist
    from sparse_mixed_precision_b200.seqpar import heads_to_seq, seq_to_heads
    dist.init_process_group("gloo")
    try:
        g = torch.Generator().manual_seed(7)
        B, T, H, d = 2, 12, 6, 8
        x = torch.randn(B, T, H, d, generator=g).to(torch.bfloat16)   # the same on every rank
        Tl, Hl = T // world, H // world
        local = x[:, rank * Tl:(rank + 1) * Tl].contiguous()
        y = seq_to_heads(local)
        ok1 = torch.equal(y, x[:, :, rank * Hl:(rank + 1) * Hl])
        back = heads_to_seq(y)
        ok2 = torch.equal(back, local)
        out.put((rank, ok1, ok2))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_sequence_to_head_exchange_round_trip(world):
    port = _free_port()
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    procs = [ctx.Process(target=_seqpar_main, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    res = [out.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert all(ok1 and ok2 for _, ok1, ok2 in res), res
