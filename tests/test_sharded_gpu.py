"""Entry-range sharded decode of one sequence on the GPU: the shards run one
after another on one device (no kernel waits for another shard), exchanging
through stacked tensors, with the library's calls (local Full, csa2_score_ids
with the shard's id offset, csa2_select_keys over the union of all shards'
keys, csa2_sparse_attn_partial per shard, csa2_attn_merge). Checked against
the unsharded oracle decode: Top-K and pool ids bit-exact as sets, attention
within the attention tolerance, lse within 1e-3. Sizes: a 20000-entry
sequence over 2 and 3 shards; 300 entries over 4 shards (one empty, a Full
layer without a pool); the 1M-entry hierarchical workload over 2, 4 and 8
shards. Also csa2_select_keys alone against a sort of the same keys, with key
sets that fit shared memory and ones that do not."""
import numpy as np
import pytest
import torch

from helpers import attn_excess, device_status_clean
from oracle import stack as ostack
from sparse_fp4_kv_b200.workloads import RECIPES, Recipe

pytestmark = pytest.mark.gpu

MID = Recipe("sharded_mid", seed=12, batch=1, q_per_seq=1, modes="FRUR", hi=8, di=128, k=512, p=2048, h=64, w=256,
             n=20000)


@pytest.fixture(scope="module")
def built():
    from sparse_fp4_kv_b200 import build
    build.build()


def _run(recipe, world, dev):
    from sparse_fp4_kv_b200.sharded import EntryShard, LocalGroup, ShardedDecoder, shard_ranges
    shards = [EntryShard(recipe, off, n, dev) for off, n in shard_ranges(recipe.n, world)]
    dec = ShardedDecoder(recipe, shards, LocalGroup(world))
    dec.step()
    torch.cuda.synchronize()
    assert device_status_clean()
    return dec


def _check(recipe, dec, exp, attn_layers, what):
    for l, (mode, _) in enumerate(ostack.schedule(recipe.modes)):
        want = exp["topk"][l][0]
        got = dec.topk_of(l)[0].cpu().numpy()
        assert sorted(got[got >= 0].tolist()) == sorted(want[want >= 0].tolist()), f"{what} layer {l} topk"
        assert (got < 0).sum() == (want < 0).sum(), f"{what} layer {l} topk padding"
        if mode == "full" and recipe.p > 0:
            wp, gp = exp["pool"][l][0], dec.pool[l][0].cpu().numpy()
            assert sorted(gp[gp >= 0].tolist()) == sorted(wp[wp >= 0].tolist()), f"{what} layer {l} pool"
        if l in attn_layers:
            go = dec.o[l][0].float().cpu().numpy()
            assert attn_excess(go, exp["o"][l][0]) <= 1.0, f"{what} layer {l}: {np.abs(go - exp['o'][l][0]).max()}"
            np.testing.assert_allclose(dec.lse[l][0].cpu().numpy(), exp["lse"][l][0], atol=1e-3, rtol=0,
                                       err_msg=f"{what} layer {l} lse")


@pytest.mark.parametrize("world", [2, 3])
def test_sharded_mid(built, cuda_device, world):
    exp = ostack.run(MID, [0])
    _check(MID, _run(MID, world, cuda_device), exp, range(MID.layers), f"world {world}")


def test_sharded_empty_shard_no_pool(built, cuda_device):
    r = MID.scaled(name="sharded_tiny", n=300, modes="FU", p=0, k=96, h=32, w=40)
    exp = ostack.run(r, [0])
    _check(r, _run(r, 4, cuda_device), exp, range(r.layers), "world 4, n 300")


@pytest.fixture(scope="module")
def hier1m_expected():
    return ostack.run(RECIPES["hier1m"], [0])


@pytest.mark.parametrize("world", [2, 4, 8])
def test_sharded_hier1m(built, cuda_device, hier1m_expected, world):
    # 2 shards: 16384 gathered keys per select (shared memory); 4 and 8: 32768
    # and 65536 (keys re-read from L2)
    r = RECIPES["hier1m"]
    _check(r, _run(r, world, cuda_device), hier1m_expected, [0, 1], f"hier1m world {world}")


@pytest.mark.parametrize("m", [5000, 100000])
def test_select_keys_against_sorted_keys(built, cuda_device, m):
    """csa2_select_keys = the ids of the k largest keys (numpy sort of the
    same keys), with heavy ties in the score half and empty slots."""
    from sparse_fp4_kv_b200 import binding as B
    rng = np.random.default_rng(m)
    nq, k = 3, 2048
    hi = rng.integers(0x80000000, 0x80000000 + 64, (nq, m), dtype=np.uint64)    # few distinct scores
    ids = np.stack([rng.permutation(1 << 24)[:m] for _ in range(nq)]).astype(np.uint64)
    keys = (hi << np.uint64(32)) | (~ids & np.uint64(0xFFFFFFFF))
    keys[:, ::7] = 0                                                            # empty slots
    dev_keys = torch.from_numpy(keys.view(np.int64)).to(cuda_device)
    out = torch.empty((nq, k), dtype=torch.int32, device=cuda_device)
    B.csa2_select_keys(dev_keys, k, out)
    torch.cuda.synchronize()
    assert device_status_clean()
    got = out.cpu().numpy()
    for qi in range(nq):
        live = np.sort(keys[qi][keys[qi] != 0])[::-1][:k]
        want = (~live & np.uint64(0xFFFFFFFF)).astype(np.int64)
        assert sorted(got[qi].tolist()) == sorted(want.tolist()), f"query {qi}"
