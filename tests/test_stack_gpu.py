"""Whole decode steps (append -> indexer modes -> attention per layer) of the
five workloads, at reduced sizes, against the oracle's own step: Top-k sets
exact, attention within 2e-3. The tiny Full workload runs at its full size.
Also checks the Reuse invariant (a Reuse layer's output equals its source's
when the queries coincide) on the GPU path."""
import numpy as np
import pytest
import torch

import oracle.stack as ostack
from helpers import attn_excess, compare_ids, device_status_clean
from sparse_fp4_kv_b200.workloads import RECIPES

pytestmark = pytest.mark.gpu

SMALL = {
    "tiny_full": RECIPES["tiny_full"],
    "stack20": RECIPES["stack20"].scaled(batch=2, n=3001, k=256, p=512, w=64),
    "hier1m": RECIPES["hier1m"].scaled(n=20000, k=256, p=1024, w=130),
    "paged64": RECIPES["paged64"].scaled(batch=4, n_range=(300, 5000), k=256, w=64),
    "chunk512": RECIPES["chunk512"].scaled(q_per_seq=64, cap=8192, prefill=6144, append=2048, k=256, w=32,
                                           swa_rows=95),
}


@pytest.fixture(scope="module")
def built():
    from sparse_fp4_kv_b200 import build
    build.build()


def _compare(dec, ref, recipe):
    for l, (mode, src) in enumerate(dec.schedule):
        g_topk = dec.topk_of(l).cpu().numpy()
        g_o = dec.o[l].float().cpu().numpy()
        g_lse = dec.lse[l].cpu().numpy()
        for qi, want in ref["topk"][l].items():
            compare_ids(g_topk[qi], want, f"layer {l} ({mode}) q{qi}")
            if mode == "full" and recipe.p > 0:
                compare_ids(dec.pool[l].cpu().numpy()[qi], ref["pool"][l][qi], f"pool layer {l} q{qi}")
            err = np.abs(g_o[qi] - ref["o"][l][qi]).max()
            assert attn_excess(g_o[qi], ref["o"][l][qi]) <= 1.0, f"layer {l} q{qi}: {err}"
            fin = np.isfinite(ref["lse"][l][qi])
            np.testing.assert_allclose(g_lse[qi][fin], ref["lse"][l][qi][fin], atol=1e-3, rtol=0)


@pytest.mark.parametrize("name", list(SMALL))
def test_step_matches_oracle(built, cuda_device, name):
    from sparse_fp4_kv_b200.stack import Csa2Decoder
    recipe = SMALL[name]
    dec = Csa2Decoder(recipe, cuda_device)
    dec.step()
    torch.cuda.synchronize()
    assert device_status_clean()
    seqs = list(range(recipe.batch))
    queries = None
    if recipe.chunked:
        queries = {0, 1, recipe.q_per_seq // 2, recipe.q_per_seq - 1}
    ref = ostack.run(recipe, seqs, queries=queries)
    _compare(dec, ref, recipe)
    # appended rows: the step's append wrote what the oracle's quantiser writes
    if recipe.chunked:
        oc = ostack.SeqCache(recipe, 0)
        rows = dec.physical_rows(0, torch.arange(recipe.prefill, recipe.prefill + recipe.append,
                                                 device=cuda_device))
        np.testing.assert_array_equal(dec.codes[rows].cpu().numpy(), oc.codes[recipe.prefill:])
        np.testing.assert_array_equal(dec.scales[rows].cpu().numpy(), oc.scales[recipe.prefill:])


def test_reuse_source_full_variant(built, cuda_device):
    from sparse_fp4_kv_b200.stack import Csa2Decoder
    recipe = SMALL["stack20"]
    dec = Csa2Decoder(recipe, cuda_device, reuse_from="full")
    dec.step()
    torch.cuda.synchronize()
    ref = ostack.run(recipe, [0, 1], reuse_from="full", layers=[6, 9, 16])
    for l in (6, 9, 16):
        assert dec.schedule[l] == ("reuse", 0 if l < 10 else 10)
        for qi, want in ref["topk"][l].items():
            compare_ids(dec.topk_of(l).cpu().numpy()[qi], want, f"layer {l}")
            assert attn_excess(dec.o[l].float().cpu().numpy()[qi], ref["o"][l][qi]) <= 1.0


def test_reuse_layer_reproduces_source_output(built, cuda_device):
    from sparse_fp4_kv_b200.stack import Csa2Decoder
    recipe = SMALL["stack20"]
    dec = Csa2Decoder(recipe, cuda_device)
    # give Reuse layer 3 the query and window of its source layer 0
    dec.q[3].copy_(dec.q[0])
    dec.swa[3].copy_(dec.swa[0])
    dec.step()
    torch.cuda.synchronize()
    assert torch.equal(dec.o[3], dec.o[0])
    assert torch.equal(dec.lse[3], dec.lse[0])


@pytest.mark.parametrize("reuse_from", ["previous", "full"])
def test_one_cache_per_full_layer(built, cuda_device, reuse_from):
    # the reading in which every Full layer generates its own global KV: two
    # caches for stack20's two Full layers; Reindex and Reuse layers read their
    # source's cache
    from sparse_fp4_kv_b200.stack import Csa2Decoder
    recipe = SMALL["stack20"].scaled(cache_per_full=True)
    dec = Csa2Decoder(recipe, cuda_device, reuse_from=reuse_from)
    assert len(dec.kvs) == 2 and dec.cache_of[:10] == [0] * 10 and dec.cache_of[10:] == [1] * 10
    dec.step()
    torch.cuda.synchronize()
    assert device_status_clean()
    ref = ostack.run(recipe, [0, 1], reuse_from=reuse_from)
    _compare(dec, ref, recipe)
    # the two caches really differ (different rows drawn for each)
    assert not torch.equal(dec.kvs[0].codes, dec.kvs[1].codes)
