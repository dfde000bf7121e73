"""The multi-GPU host logic on two CPU ranks (gloo, 127.0.0.1): every rank
gets a different workload of the same shape, the job time is the slowest
rank's, and the throughput counts both ranks' units. No GPU needed."""
import os
import socket

import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from sparse_fp4_kv_b200.ranks import job_throughput, max_over_ranks, rank_recipe
        from sparse_fp4_kv_b200.workloads import RECIPES
        base = RECIPES["tiny_full"]
        r = rank_recipe(base, rank, world)
        q = r.q(0).flatten()[:64].float()
        # a fixed fake per-rank time, rank 1 the slower
        t = max_over_ranks(10.0 + 5.0 * rank)
        value, ms = job_throughput(r.nq * r.layers, world, t, steps=5)
        out[rank] = (r.seed, q.tolist(), t, value, ms, tuple(r.seq_lens()))
    finally:
        dist.destroy_process_group()


def test_two_ranks_distinct_inputs_and_max_time():
    world, port = 2, _free_port()
    out = mp.get_context("spawn").Manager().dict()
    mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
    (s0, q0, t0, v0, ms0, l0), (s1, q1, t1, v1, ms1, l1) = out[0], out[1]
    assert s0 != s1 and q0 != q1          # different sequences per rank
    assert l0 == l1                        # same shape
    assert t0 == t1 == 15.0                # the slowest rank's time, on every rank
    assert v0 == v1 and ms0 == ms1 == 3.0
    from sparse_fp4_kv_b200.workloads import RECIPES
    r = RECIPES["tiny_full"]
    assert abs(v0 - r.nq * r.layers * world / 3e-3) < 1e-6


def test_single_process_is_identity():
    from sparse_fp4_kv_b200.ranks import max_over_ranks, rank_recipe
    from sparse_fp4_kv_b200.workloads import RECIPES
    base = RECIPES["tiny_full"]
    assert rank_recipe(base, 0, 1) is base
    assert max_over_ranks(3.5) == 3.5
