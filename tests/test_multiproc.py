"""The N > 1 host logic on CPU with gloo, world size 2 (no GPU).

The forward shards as independent problems (no data-path collective).  These tests check
the share assignment, the max-over-ranks timing reduction, and that a tensor split by rows
across ranks yields exactly the whole tensor's absmean scale when the ranks' integer
partial sums are all-reduced (the exact fixed-point sum makes the exchange order-free)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from sparse_linear_layers_absmean_b200 import dist as sbn_dist


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import oracle
        import workloads
        out = {}
        w, r, _ = sbn_dist.env_world()
        out["env"] = (w, r)
        # shares of the 130 linears of the training-step workload
        out["share"] = sbn_dist.shard_range(130, world, rank)
        out["max"] = sbn_dist.max_over_ranks(float(rank + 1) * 1.5)
        # row-sharded absmean: integer partials all-reduced == whole tensor
        W = workloads.masters(96, 320, seed=7)
        b, e = sbn_dist.shard_range(96, world, rank)
        S_part, _, _, _ = oracle.weight_gamma(np.ascontiguousarray(W[b:e]), 0.0)
        t = torch.tensor([S_part], dtype=torch.int64)
        dist.all_reduce(t)
        S_full, gamma_full, _, _ = oracle.weight_gamma(W, 0.0)
        n = W.size
        gamma_sharded = np.float32(float(t.item()) / (float(n) * 16777216.0))
        out["S"] = (int(t.item()), S_full)
        out["gamma"] = (float(gamma_sharded), float(gamma_full))
        # the benchmark's per-rank workload: each rank runs one replica of the 32-layer stack
        # on its own seeded tensors; the reductions of its timing go through dist
        import bench
        out["stack"] = bench.stack_layers(rank)
        out["sum"] = sbn_dist.sum_over_ranks(float(rank + 1))
        w, r, l = sbn_dist.init("gloo")  # already joined: returns the environment's view
        out["init"] = (w, r, l)
        sbn_dist.barrier()
        q.put((rank, out))
    finally:
        dist.destroy_process_group()


@pytest.fixture(scope="module")
def results():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=180) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    return res


def test_env_and_shares(results):
    assert results[0]["env"] == (2, 0) and results[1]["env"] == (2, 1)
    s0, s1 = results[0]["share"], results[1]["share"]
    assert s0[0] == 0 and s0[1] == s1[0] and s1[1] == 130
    assert abs((s0[1] - s0[0]) - (s1[1] - s1[0])) <= 1


def test_max_over_ranks(results):
    assert results[0]["max"] == results[1]["max"] == 3.0


def test_row_sharded_gamma_is_exact(results):
    for r in (0, 1):
        S_red, S_full = results[r]["S"]
        assert S_red == S_full
        g_sh, g_full = results[r]["gamma"]
        assert g_sh == g_full


def test_bench_rank_replicas(results):
    """Both ranks run the same 160 layer shapes (weak scaling: one stack replica per GPU) on
    disjoint seeded tensors."""
    a, b = results[0]["stack"], results[1]["stack"]
    assert len(a) == len(b) == 160
    assert [x[:4] for x in a] == [x[:4] for x in b]
    assert not set(x[4] for x in a) & set(x[4] for x in b)
    assert results[0]["sum"] == results[1]["sum"] == 3.0
    assert results[0]["init"] == (2, 0, 0) and results[1]["init"] == (2, 1, 1)


@pytest.mark.parametrize("n,world", [(0, 1), (1, 3), (7, 2), (130, 8), (5, 5)])
def test_shard_range_partitions(n, world):
    seen = []
    for r in range(world):
        b, e = sbn_dist.shard_range(n, world, r)
        seen.extend(range(b, e))
    assert seen == list(range(n))
