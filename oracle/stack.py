"""Oracle decode step over a workload recipe (TEST INFRASTRUCTURE).

Builds each requested sequence's cache on the host with the oracle's own
quantiser (rows drawn from the shared seeded generator), applies the static
mode schedule with its own source resolution, and runs the oracle's Full,
Reindex and attention functions query by query. Only tests/, the smoke check
and bench.py's CPU-baseline leg use it.

Mode schedule (DeepSeek V4.1-Flash Cuts KV Cache by 437x, paragraph "CSA2
assigns each layer one of three static operating modes"; DeepSeek V4.1 Flash
Architecture Breakdown, section "How does the cache compress along three
dimensions at once?"): a Reindex layer re-scores the pool of the most recent
Full layer; a Reuse layer takes the Top-k of the most recent layer that
produced one (Reuse takes over earlier indices as they are), or, in the variant
reuse_from='full', of the most recent Full layer. With one global cache per
Full layer (the reading in which a Full layer generates its own global KV), a
Full layer scores and attends over its own cache, a Reindex layer over its
source Full layer's, a Reuse layer over its source layer's.
"""
import math

import numpy as np
import torch

from . import append_fp4, index_full, index_reindex, quantize_rows, sparse_attn


def schedule(modes, reuse_from="previous"):
    res = []
    last_full = None
    last_producer = None
    for layer, m in enumerate(modes):
        if m == "F":
            res.append(("full", None))
            last_full = layer
            last_producer = layer
        elif m == "R":
            res.append(("reindex", last_full))
            last_producer = layer
        else:
            res.append(("reuse", last_producer if reuse_from == "previous" else last_full))
    return res


def bf16_bits(t):
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


class SeqCache:
    """One sequence's logical cache (identity page table) built by the oracle;
    `cache` selects the cache of the per-Full-layer variant (0: shared)."""

    def __init__(self, recipe, b, cache=0):
        lens = recipe.seq_lens()
        self.n = int(lens[b])
        rows = []
        if recipe.chunked:
            rows.append(recipe.latent_rows(b, 0, recipe.prefill, cache=cache))
            rows.append(recipe.latent_rows(b, recipe.prefill, self.n, cache=cache))
        else:
            rows.append(recipe.latent_rows(b, 0, self.n, cache=cache))
        x = bf16_bits(torch.cat(rows))
        cap = max(self.n, 1)
        self.codes = np.zeros((cap, 256), np.uint8)
        self.scales = np.zeros((cap, 32), np.uint8)
        append_fp4(x, np.zeros(self.n, np.int32), np.arange(self.n, dtype=np.int64),
                   np.zeros((1, 1), np.int32), cap, self.codes, self.scales)
        self.kidx = recipe.kidx_rows(b, 0, self.n, cache=cache).numpy()
        self.page_table = np.zeros(1, np.int32)
        self.page_size = cap


def run(recipe, seqs, reuse_from="previous", layers=None, queries=None, attention=True):
    """Oracle results for the given sequences: dict with per-layer dicts
    topk[l][qi], pool[l][qi], o[l][qi] (f64 [h, 512]) and lse[l][qi]."""
    sched = schedule(recipe.modes, reuse_from)
    layers = range(recipe.layers) if layers is None else layers
    last = max(layers) if len(layers) else -1
    out = {"topk": {}, "pool": {}, "o": {}, "lse": {}}
    ql = recipe.q_limit()
    wb, we = recipe.swa_window()
    scale = 1.0 / math.sqrt(512.0)
    # which cache every layer reads: one shared, or one per Full layer (a Full
    # layer reads its own, Reindex its source Full layer's, Reuse its source's)
    cache_of, fulls = [], 0
    for layer, (mode, src) in enumerate(sched):
        if not recipe.cache_per_full:
            cache_of.append(0)
        elif mode == "full":
            cache_of.append(fulls)
            fulls += 1
        else:
            cache_of.append(cache_of[src])
    for b in seqs:
        caches = {}
        qis = [b * recipe.q_per_seq + j for j in range(recipe.q_per_seq)]
        if queries is not None:
            qis = [qi for qi in qis if qi in queries]
        for layer in range(last + 1):
            mode, src = sched[layer]
            if cache_of[layer] not in caches:
                caches[cache_of[layer]] = SeqCache(recipe, b, cache_of[layer])
            c = caches[cache_of[layer]]
            qidx = recipe.qidx(layer).numpy()
            w = recipe.weights(layer).numpy()
            need_attn = attention and layer in layers
            if need_attn:
                q = recipe.q(layer, rows=qis)
                swa = recipe.swa(layer, seqs=[b])[0].numpy()
            for j, qi in enumerate(qis):
                if mode == "full":
                    lim = int(ql[qi]) if ql is not None else c.n
                    tk, pl = index_full(qidx[qi], w[qi], c.kidx, c.page_table, c.page_size, lim, recipe.k,
                                        recipe.p)
                    out["topk"].setdefault(layer, {})[qi] = tk
                    out["pool"].setdefault(layer, {})[qi] = pl
                elif mode == "reindex":
                    tk = index_reindex(qidx[qi], w[qi], c.kidx, c.page_table, c.page_size,
                                       out["pool"][src][qi], recipe.k)
                    out["topk"].setdefault(layer, {})[qi] = tk
                else:
                    out["topk"].setdefault(layer, {})[qi] = out["topk"][src][qi]
                if need_attn:
                    win = swa[int(wb[qi]):int(we[qi])]
                    o, lse = sparse_attn(bf16_bits(q[j]), c.codes, c.scales, c.page_table, c.page_size,
                                         out["topk"][layer][qi], win, scale)
                    out["o"].setdefault(layer, {})[qi] = o
                    out["lse"].setdefault(layer, {})[qi] = lse
    return out
