"""Multi-rank host logic of bench.py on CPU with the gloo backend (world size 2).

On more than one GPU every rank runs its own independent layer (the path has
no exchange step), so the only cross-rank operations are the barrier and the
max-over-ranks of the device-timed step; these run here on gloo, and the
per-rank inputs are checked to be distinct problems.
"""

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from long_context_tsa_b200 import inputs as I


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # Rank r pretends its step took (10 + r) ms and its attention (3 - r) ms.
        got = bench.max_over_ranks([10.0 + rank, 3.0 - rank], dist)
        w = I.custom(Hq=4, Hkv=2, L=64, D=64, dtype="bf16", W=8, sigma=0.5)
        qq, _, _ = I.make_qkv(w, seed=bench.rank_seed(rank))
        first = qq.float().flatten()[:8]
        gathered = [torch.zeros_like(first) for _ in range(world)]
        dist.all_gather(gathered, first)
        dist.barrier()
        q.put((rank, got, [g.tolist() for g in gathered]))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_distinct_problems_on_gloo():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, got, gathered in results:
        assert got == [11.0, 3.0]  # max over ranks, element by element
        assert gathered[0] != gathered[1]  # each rank runs its own seeded layer


def test_job_throughput_counts_every_rank():
    assert bench.job_tokens_per_s(1, 131072, 2.0) == pytest.approx(65_536_000.0)
    assert bench.job_tokens_per_s(4, 131072, 2.0) == pytest.approx(4 * 65_536_000.0)
    assert bench.max_over_ranks([1.5, 2.5]) == [1.5, 2.5]  # single process: identity
