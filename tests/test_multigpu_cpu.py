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


def _kv_worker(rank, world, port, q):
    # Each rank runs the oracle on its own KV-group slice of one layer; rank 0
    # gathers the slices and compares them with the whole layer, bit for bit.
    import numpy as np

    from long_context_tsa_b200 import shard
    from oracle import tsa_oracle as O

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = I.custom(Hq=8, Hkv=4, L=96, D=16, dtype="f32", W=8, sigma=1.0)
        qq, kk, vv = I.make_qkv(w, seed=5)
        budgets = [20, 33, 7, 96]
        g0, g1 = shard.kv_group_range(rank, world, w.Hkv)
        qs, ks, vs = shard.kv_group_slice(qq, kk, vv, g0, g1)
        bs = shard.slice_budgets(budgets, w.B, w.Hkv, g0, g1)
        sc, perm, out = O.forward(qs.numpy(), ks.numpy(), vs.numpy(), w.W, bs)
        parts = [torch.from_numpy(sc.copy()), torch.from_numpy(perm.copy()), torch.from_numpy(out.copy())]
        gathered = []
        for t in parts:
            lst = [torch.zeros_like(t) for _ in range(world)]
            dist.all_gather(lst, t)
            gathered.append(lst)
        ok = None
        if rank == 0:
            fs, fp, fo = O.forward(qq.numpy(), kk.numpy(), vv.numpy(), w.W, budgets)
            ok = (np.array_equal(torch.cat(gathered[0], 1).numpy(), fs)
                  and np.array_equal(torch.cat(gathered[1], 1).numpy(), fp)
                  and np.array_equal(torch.cat(gathered[2], 1).numpy(), fo))
        dist.barrier()
        q.put((rank, (g0, g1), ok))
    finally:
        dist.destroy_process_group()


def test_kv_group_partition_reproduces_the_layer_on_gloo():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_kv_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[1] for r in results] == [(0, 2), (2, 4)]
    assert results[0][2] is True


def test_kv_group_ranges_cover_every_group_once():
    from long_context_tsa_b200 import shard

    for Hkv in (1, 3, 8, 13):
        for world in (1, 2, 3, 8):
            if world > Hkv:
                continue
            rs = [shard.kv_group_range(r, world, Hkv) for r in range(world)]
            assert rs[0][0] == 0 and rs[-1][1] == Hkv
            assert all(a[1] == b[0] for a, b in zip(rs, rs[1:]))
            assert all(g1 > g0 for g0, g1 in rs)
    assert shard.slice_budgets([1, 2, 3, 4, 5, 6], 2, 3, 1, 3) == [2, 3, 5, 6]
