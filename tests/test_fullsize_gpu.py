"""The four benchmark workloads at their full sizes (stack20: 8 x 64K entries,
20 layers; hier1m: one 1M-entry sequence, Full + 3 Reindex; paged64: 64
ragged sequences in 64-entry pages; chunk512: 512 causal queries after a
32K-row append), run by the same decoder and library calls the benchmark
times, and checked against the oracle on sampled outputs: the appended rows'
codes and scales, the Top-K / pool ids of sampled queries in every indexer
layer (bit-exact as sets), and the attention outputs of sampled queries in
the first layers (within the attention tolerance). The oracle works on a
contiguous host copy of the sampled sequence's cache rows."""
import math

import numpy as np
import pytest
import torch

import oracle
from helpers import attn_excess, bf16_bits, compare_ids, device_status_clean

pytestmark = pytest.mark.gpu

# workload -> (sampled queries, number of leading layers whose attention is checked)
SAMPLES = {
    "stack20": ([0, 5], 6),
    "hier1m": ([0], 2),
    "paged64": ([0, 63], 1),
    "chunk512": ([0, 511], 1),
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
    queries, attn_layers = SAMPLES[name]
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

    cache = {}
    scale = 1.0 / math.sqrt(512.0)
    for qi in queries:
        b = qi // r.q_per_seq
        n_b = int(lens[b])
        if b not in cache:
            cache[b] = _seq_cache(dec, b, n_b)
        codes, scales, kidx = cache[b]
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
            if l < attn_layers:
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
