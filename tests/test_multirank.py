"""Multi-rank host logic on CPU (gloo, world size 2).

The path partitions into independent (request, KV group, query block) rows with
no exchange step, so ranks never trade data: each processes its own share and
only the timing is reduced (max over ranks). These tests run the oracle on
shards in two processes and check that the shards reproduce the one-process
result, and that the benchmark's reduction and whole-job value are right.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _case():
    rng = np.random.default_rng(42)
    L, hq, hkv, d, B = 96, 8, 4, 16, 16
    Q = rng.standard_normal((L, hq, d))
    K = rng.standard_normal((L, hkv, d))
    V = rng.standard_normal((L, hkv, d))
    u = rng.standard_normal(d)
    u /= np.linalg.norm(u)
    Q += 3 * u
    K[32:48] += 3 * u
    return Q, K, V, B


def _worker(rank, world, port, out_q):
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import oracle
        import bench
        Q, K, V, B = _case()
        G = Q.shape[1] // K.shape[1]
        # this rank's KV groups (and their query heads) only
        groups = [g for g in range(K.shape[1]) if g % world == rank]
        heads = [h for g in groups for h in range(g * G, (g + 1) * G)]
        res = oracle.flashprefill(Q[:, heads], K[:, groups], V[:, groups], B, 0.2, 16, 32)
        mine = {g: [l.tolist() for l in res["lists"][k]] for k, g in enumerate(groups)}
        outs = {h: res["O"][:, k] for k, h in enumerate(heads)}
        # timing reduction: each rank reports different times; every rank must see the max
        vals = [10.0 + rank, 1.0 + 2 * rank, 5.0 - rank]
        red = bench.max_over_ranks(vals, dist, "cpu")
        gathered = [None] * world
        dist.all_gather_object(gathered, (mine, outs, red))
        if rank == 0:
            out_q.put(gathered)
    finally:
        dist.destroy_process_group()


def _run(world=2):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    try:
        got = q.get(timeout=240)
    finally:
        for p in procs:
            p.join(timeout=60)
    for p in procs:
        assert p.exitcode == 0
    return got


@pytest.fixture(scope="module")
def two_ranks():
    return _run(2)


def test_shards_reproduce_the_single_process_result(two_ranks):
    import oracle
    Q, K, V, B = _case()
    full = oracle.flashprefill(Q, K, V, B, 0.2, 16, 32)
    lists, outs = {}, {}
    for mine, o, _ in two_ranks:
        assert not (set(mine) & set(lists)), "a KV group was processed twice"
        lists.update(mine)
        outs.update(o)
    assert sorted(lists) == list(range(K.shape[1]))
    for g, rows in lists.items():
        assert rows == [l.tolist() for l in full["lists"][g]]
    for h, o in outs.items():
        np.testing.assert_allclose(o, full["O"][:, h], rtol=0, atol=1e-12)


def test_timing_reduction_is_max_over_ranks(two_ranks):
    for _, _, red in two_ranks:
        assert red == [11.0, 3.0, 5.0]


def test_weak_scaling_value():
    import bench
    # every rank runs one layer of F flops; the job takes the slowest rank's time
    assert bench.weak_value(4, 2e12, 10.0) == pytest.approx(4 * 2e12 / 1e-2 / 1e12)
