"""The four benchmark workloads at their full sizes (stack20: 8 x 64K entries,
20 layers; hier1m: one 1M-entry sequence, Full + 3 Reindex; paged64: 64
ragged sequences in 64-entry pages; chunk512: 512 causal queries after a
32K-row append), run by the same decoder and library calls the benchmark
times, and checked against the oracle: the appended rows' codes and scales;
every query of layer 0 (16 queries spread over the chunked workload's 512),
its Top-K / pool ids (bit-exact as sets) and attention output (within the
attention tolerance); in later layers, the ids of the same queries in every
indexer layer and the attention of a few of them in a Reindex and a Reuse
layer. The oracle works on a contiguous host copy of each checked
sequence's cache rows."""
import math

import numpy as np
import pytest
import torch

import oracle
from helpers import attn_excess, bf16_bits, compare_ids, device_status_clean

pytestmark = pytest.mark.gpu

# workload -> (queries checked in layer 0 and in every indexer layer,
#              queries whose attention is checked in the later layers listed)
SAMPLES = {
    "stack20": (list(range(8)), [0, 5], [5, 6, 19]),   # 5: Reindex, 6 and 19: Reuse
    "hier1m": ([0], [0], [1, 2, 3]),                   # Reindex layers
    "paged64": (list(range(64)), [0, 37, 63], [1, 3]),  # Reuse layers
    "chunk512": ([0, 31, 63, 100, 127, 160, 200, 255, 256, 300, 341, 383, 400, 450, 480, 511], [], []),
}


@pytest.fixture(scope="module")
def built():
    from sparse_fp4_kv_b200 import build
    build.build()


def _seq_cache(dec, b, n):
    """Contiguous host copy of sequence b's first n cache rows (logical order)."""
    pos = torch.arange(n, dtype=torch.int64, device=dec.device)
    rows = dec.physical_rows(b, pos)
    return dec.codes[rows].cpu().numpy(), dec.scales[rows].cpu().numpy(), dec.kidx[rows].cpu().numpy()


@pytest.mark.parametrize("name", list(SAMPLES))
def test_fullsize_sampled(built, cuda_device, name):
    from sparse_fp4_kv_b200.stack import Csa2Decoder
    from sparse_fp4_kv_b200.workloads import RECIPES
    r = RECIPES[name]
    dec = Csa2Decoder(r, cuda_device)
    dec.step()
    torch.cuda.synchronize()
    assert device_status_clean()
    queries, late_queries, late_layers = SAMPLES[name]
    lens = dec.lens.numpy()
    q_limit = dec.q_limit.cpu().numpy() if dec.q_limit is not None else None

    # appended rows: codes and scales equal the oracle's quantisation
    xs = dec.x_new[:: max(1, dec.x_new.shape[0] // 64)][:64]
    idx = np.arange(0, dec.x_new.shape[0], max(1, dec.x_new.shape[0] // 64))[:64]
    want_c, want_s = oracle.quantize_rows(bf16_bits(xs))
    rows = dec.physical_rows(0, dec.x_pos[idx]) if r.chunked else None
    for j, i in enumerate(idx):
        b = int(dec.x_seq[i])
        row = int(dec.physical_rows(b, dec.x_pos[i:i + 1])[0]) if rows is None else int(rows[j])
        assert np.array_equal(dec.codes[row].cpu().numpy(), want_c[j]), f"codes of appended row {i}"
        assert np.array_equal(dec.scales[row].cpu().numpy(), want_s[j]), f"scales of appended row {i}"

    scale = 1.0 / math.sqrt(512.0)
    cache = {}

    def seq(b):
        if b not in cache:
            if len(cache) > 2:
                cache.clear()  # bound host memory: sequences are checked in order
            cache[b] = _seq_cache(dec, b, int(lens[b]))
        return cache[b]

    def check_attention(l, qi, b, codes, scales):
        n_b = int(lens[b])
        pt = np.zeros(1, np.int32)
        topk = dec.topk_of(l)[qi].cpu().numpy()
        wb, we = int(dec.swa_begin[qi]), int(dec.swa_end[qi])
        swa = dec.swa[l][b].cpu().numpy()[wb:we] if we > wb else None
        oo, ol = oracle.sparse_attn(bf16_bits(dec.q[l][qi]), codes, scales, pt, n_b, topk, swa, scale)
        go = dec.o[l][qi].float().cpu().numpy()
        assert attn_excess(go, oo) <= 1.0, f"{name} layer {l} q{qi}: {np.abs(go - oo).max()}"
        gl = dec.lse[l][qi].cpu().numpy()
        fin = np.isfinite(ol)
        assert np.all(np.isfinite(gl) == fin)
        np.testing.assert_allclose(gl[fin], ol[fin], atol=1e-3, rtol=0)

    for qi in queries:
        b = qi // r.q_per_seq
        n_b = int(lens[b])
        codes, scales, kidx = seq(b)
        pt = np.zeros(1, np.int32)
        lim = int(q_limit[qi]) if q_limit is not None else n_b
        for l, (mode, src) in enumerate(dec.schedule):
            qidx = dec.qidx[l][qi].cpu().numpy()
            w = dec.w[l][qi].cpu().numpy()
            if mode == "full":
                ot, op = oracle.index_full(qidx, w, kidx, pt, n_b, lim, r.k, r.p)
                compare_ids(dec.topk[l][qi].cpu().numpy(), ot, f"{name} layer {l} topk q{qi}")
                if r.p > 0:
                    compare_ids(dec.pool[l][qi].cpu().numpy(), op, f"{name} layer {l} pool q{qi}")
            elif mode == "reindex":
                pool = dec.pool[src][qi].cpu().numpy()
                want = oracle.index_reindex(qidx, w, kidx, pt, n_b, pool, r.k)
                compare_ids(dec.topk[l][qi].cpu().numpy(), want, f"{name} layer {l} reindex q{qi}")
        check_attention(0, qi, b, codes, scales)
        if qi in late_queries:
            for l in late_layers:
                check_attention(l, qi, b, codes, scales)
