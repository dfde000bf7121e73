"""Entry-range sharded decode of one sequence, host logic on CPU: the shard
ranges, and the sharded decoder (local Full, key exchange, selection from the
union, Reindex over the owned pool ids, attention partials with the window on
the first shard, log-sum-exp merge) run with the oracle standing in for the
library calls, against the unsharded oracle decode. Two and three gloo ranks
(uneven ranges) for the exchange through torch.distributed; several shards in
one process for more world sizes, an empty shard and a Full layer without a
pool."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle_ops
from helpers import attn_excess
from oracle import stack as ostack
from sparse_fp4_kv_b200.sharded import DistGroup, EntryShard, LocalGroup, ShardedDecoder, local_ids, shard_ranges
from sparse_fp4_kv_b200.workloads import Recipe

# one sequence: Full with a pool, Reindex, Reuse, Reindex (a small 1M-entry-like layer mix)
SMALL = Recipe("sharded_small", seed=11, batch=1, q_per_seq=1, modes="FRUR", hi=8, di=128, k=128, p=512, h=16,
               w=48, n=3000)


def test_shard_ranges_cover_and_align():
    for n, world in [(3000, 2), (300, 4), (1 << 20, 8), (129, 3), (1, 2)]:
        rs = shard_ranges(n, world)
        assert len(rs) == world
        assert sum(c for _, c in rs) == n
        off = 0
        for o, c in rs:
            assert o == off and c >= 0 and o % 128 == 0 or c == 0
            off += c
    assert shard_ranges(300, 4) == [(0, 128), (128, 128), (256, 44), (300, 0)]


def test_local_ids():
    g = torch.tensor([[5, 130, -1, 127, 128, 300]], dtype=torch.int32)
    assert local_ids(g, 128, 100).tolist() == [[-1, 2, -1, -1, 0, -1]]
    assert local_ids(g, 0, 128).tolist() == [[5, -1, -1, 127, -1, -1]]


def _expected(recipe):
    return ostack.run(recipe, [0])


def _check(recipe, exp, topk, pool, o, lse, what):
    for l, (mode, _) in enumerate(ostack.schedule(recipe.modes)):
        want = exp["topk"][l][0]
        got = np.asarray(topk[l])
        assert sorted(got[got >= 0].tolist()) == sorted(want[want >= 0].tolist()), f"{what} layer {l} topk"
        assert (got < 0).sum() == (want < 0).sum()
        if mode == "full" and recipe.p > 0:
            wp, gp = exp["pool"][l][0], np.asarray(pool[l])
            assert sorted(gp[gp >= 0].tolist()) == sorted(wp[wp >= 0].tolist()), f"{what} layer {l} pool"
        assert attn_excess(np.asarray(o[l], np.float64), exp["o"][l][0]) <= 1.0, f"{what} layer {l} o"
        np.testing.assert_allclose(np.asarray(lse[l]), exp["lse"][l][0], atol=1e-4, rtol=0, err_msg=what)


def _run_local(recipe, world):
    shards = [EntryShard(recipe, off, n, "cpu", ops=oracle_ops) for off, n in shard_ranges(recipe.n, world)]
    dec = ShardedDecoder(recipe, shards, LocalGroup(world))
    dec.step()
    topk = [dec.topk_of(l)[0].numpy() for l in range(recipe.layers)]
    pool = [dec.pool[l][0].numpy() if dec.pool[l] is not None else None for l in range(recipe.layers)]
    o = [dec.o[l][0].float().numpy() for l in range(recipe.layers)]
    lse = [dec.lse[l][0].numpy() for l in range(recipe.layers)]
    return topk, pool, o, lse


@pytest.mark.parametrize("world", [1, 3])
def test_local_shards_match_unsharded_oracle(world):
    _check(SMALL, _expected(SMALL), *_run_local(SMALL, world), f"world {world}")


def test_empty_shard_and_full_without_pool():
    r = SMALL.scaled(name="sharded_tiny", n=300, modes="FU", p=0, k=96)
    _check(r, _expected(r), *_run_local(r, 4), "world 4, n 300")


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        off, n = shard_ranges(SMALL.n, world)[rank]
        dec = ShardedDecoder(SMALL, [EntryShard(SMALL, off, n, "cpu", ops=oracle_ops)], DistGroup())
        dec.step()
        L = SMALL.layers
        out[rank] = ([dec.topk_of(l)[0].tolist() for l in range(L)],
                     [dec.pool[l][0].tolist() if dec.pool[l] is not None else None for l in range(L)],
                     [dec.o[l][0].float().tolist() for l in range(L)],
                     [dec.lse[l][0].tolist() for l in range(L)])
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_gloo_ranks_match_unsharded_oracle(world):
    port = _free_port()
    out = mp.get_context("spawn").Manager().dict()
    mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
    exp = _expected(SMALL)
    for rank in range(world):
        _check(SMALL, exp, *out[rank], f"rank {rank} of {world}")
        assert out[rank][0] == out[0][0]   # every rank holds the same selection
