"""GPU decode step of a workload: the shared cache, the per-layer inputs and
outputs, and the layer loop that applies the static mode schedule.

DeepSeek V4.1-Flash Cuts KV Cache by 437x (ainewsfeed.tech), paragraph "CSA2
assigns each layer one of three static operating modes": Full layers index the
whole context, Reindex layers re-score the pool a Full layer built, Reuse
layers skip indexing and take earlier indices as they are. All layers attend
over one shared global KV cache (paragraph "CSA2 tackles storage").

Every compute step is a call into libcsa2.so through binding.py; torch only
provides device memory and the stream.
"""
import math

import torch

from . import binding as B
from .workloads import Recipe, cache_of_layers, resolve_schedule


class Csa2Decoder:
    """Holds everything one step of `recipe` touches, resident on `device`."""

    def __init__(self, recipe: Recipe, device, reuse_from="previous", build_chunk=65536):
        self.r = r = recipe
        self.device = device = torch.device(device)
        self.schedule = resolve_schedule(r.modes, reuse_from)
        # global KV caches: one shared by all layers, or one per Full layer
        self.cache_of = cache_of_layers(r.modes, self.schedule, r.cache_per_full)
        ps, pt, rows_cap = r.layout()
        self.page_size = ps
        lens = r.seq_lens()
        self.lens = lens
        self.n_max = int(lens.max())
        self.page_table = pt.to(device)
        self.seq_len = lens.to(torch.int32).to(device)
        self.kvs = []
        for c in range(r.caches()):
            self.kvs.append(B.KvCache(torch.zeros((rows_cap, 256), dtype=torch.uint8, device=device),
                                      torch.zeros((rows_cap, 32), dtype=torch.uint8, device=device),
                                      torch.zeros((rows_cap, r.di), dtype=torch.uint8, device=device),
                                      self.page_table, self.seq_len, ps))
        # cache 0 (the shared cache, or the first Full layer's)
        self.kv = self.kvs[0]
        self.codes, self.scales, self.kidx = self.kv.codes, self.kv.scales, self.kv.kidx

        # ---- cache contents present before the step --------------------------------
        present = [r.prefill if r.chunked else int(l) for l in lens.tolist()]
        for c, kv in enumerate(self.kvs):
            for b in range(r.batch):
                for t0 in range(0, present[b], build_chunk):
                    t1 = min(present[b], t0 + build_chunk)
                    self._write_rows(kv, c, b, t0, t1, r.latent_rows(b, t0, t1, device, cache=c))
            if r.chunked:
                # indexer keys of the rows the step appends (the key append itself
                # is not part of this path; the keys are inputs of the Full layer)
                for t0 in range(r.prefill, r.prefill + r.append, build_chunk):
                    t1 = min(r.prefill + r.append, t0 + build_chunk)
                    pos = torch.arange(t0, t1, dtype=torch.int64, device=device)
                    kv.kidx[self.physical_rows(0, pos)] = r.kidx_rows(0, t0, t1, device, cache=c)

        # ---- step inputs -----------------------------------------------------------
        self.x_news = []
        for c in range(len(self.kvs)):
            if r.chunked:
                total = r.prefill + r.append
                self.x_news.append(r.latent_rows(0, r.prefill, total, device, cache=c).contiguous())
            else:
                # the decoded token of each sequence: its last position
                rows = [r.latent_rows(b, int(lens[b]) - 1, int(lens[b]), device, cache=c) for b in range(r.batch)]
                self.x_news.append(torch.cat(rows).contiguous())
        self.x_new = self.x_news[0]
        if r.chunked:
            self.x_seq = torch.zeros(r.append, dtype=torch.int32, device=device)
            self.x_pos = torch.arange(r.prefill, r.prefill + r.append, dtype=torch.int64, device=device)
        else:
            self.x_seq = torch.arange(r.batch, dtype=torch.int32, device=device)
            self.x_pos = (lens - 1).to(torch.int64).to(device)
        ql = r.q_limit()
        self.q_limit = ql.to(device) if ql is not None else None
        wb, we = r.swa_window()
        self.swa_begin, self.swa_end = wb.to(device), we.to(device)
        self.q = [r.q(l, device).contiguous() for l in range(r.layers)]
        self.qidx = [r.qidx(l, device).contiguous() for l in range(r.layers)]
        self.w = [r.weights(l, device).contiguous() for l in range(r.layers)]
        self.swa = [r.swa(l, device).contiguous() for l in range(r.layers)]
        self.scale = 1.0 / math.sqrt(512.0)

        # ---- outputs and workspaces -------------------------------------------------
        nq = r.nq
        self.o = [torch.empty((nq, r.h, 512), dtype=torch.bfloat16, device=device) for _ in range(r.layers)]
        self.lse = [torch.empty((nq, r.h), dtype=torch.float32, device=device) for _ in range(r.layers)]
        self.topk = [None] * r.layers
        self.pool = [None] * r.layers
        for l, (mode, src) in enumerate(self.schedule):
            if mode in ("full", "reindex"):
                self.topk[l] = torch.empty((nq, r.k), dtype=torch.int32, device=device)
            if mode == "full" and r.p > 0:
                self.pool[l] = torch.empty((nq, r.p), dtype=torch.int32, device=device)
        self.ws_full = B.workspace(B.csa2_index_full_workspace_size(nq, self.n_max), device)
        self.ws_reindex = B.workspace(B.csa2_index_reindex_workspace_size(nq, max(r.p, 1)), device)
        self.ws_attn = B.workspace(B.csa2_sparse_attn_workspace_size(nq, r.h, r.k, r.w), device)
        torch.cuda.synchronize(device)

    def _write_rows(self, kv, c, b, t0, t1, x):
        """Quantise + append latent rows (kernel) and store their indexer keys."""
        n = t1 - t0
        seq = torch.full((n,), b, dtype=torch.int32, device=self.device)
        pos = torch.arange(t0, t1, dtype=torch.int64, device=self.device)
        B.csa2_append_fp4(x.contiguous(), seq, pos, kv)
        rows = self.physical_rows(b, pos)
        kv.kidx[rows] = self.r.kidx_rows(b, t0, t1, self.device, cache=c)

    def physical_rows(self, b, pos):
        ps = self.page_size
        return self.page_table[b, pos // ps].to(torch.int64) * ps + pos % ps

    def topk_of(self, layer):
        mode, src = self.schedule[layer]
        return self.topk[layer] if mode != "reuse" else self.topk_of(src)

    # ---- one step -------------------------------------------------------------------
    def append(self, stream=None):
        for x, kv in zip(self.x_news, self.kvs):
            B.csa2_append_fp4(x, self.x_seq, self.x_pos, kv, stream)

    def layer(self, l, stream=None, before_attention=None):
        """Layer l on `stream`: its indexer call (Full or Reindex; none for
        Reuse), then attention. before_attention, if given, is called between
        the two (e.g. to make the stream wait for q alone, which only the
        attention reads)."""
        r = self.r
        mode, src = self.schedule[l]
        kv = self.kvs[self.cache_of[l]]
        if mode == "full":
            B.csa2_index_full(self.qidx[l], self.w[l], r.q_per_seq, self.q_limit, self.n_max, kv, r.k,
                              r.p if self.pool[l] is not None else 0, self.topk[l], self.pool[l], self.ws_full,
                              stream)
        elif mode == "reindex":
            B.csa2_index_reindex(self.qidx[l], self.w[l], r.q_per_seq, self.pool[src], kv, r.k, self.topk[l],
                                 self.ws_reindex, stream)
        if before_attention is not None:
            before_attention()
        B.csa2_sparse_attn_decode(self.q[l], r.q_per_seq, kv, self.topk_of(l), self.swa[l],
                                  self.swa[l].shape[1], self.swa_begin, self.swa_end, r.w, self.scale, self.o[l],
                                  self.lse[l], self.ws_attn, stream)

    def step(self, stream=None):
        self.append(stream)
        for l in range(self.r.layers):
            self.layer(l, stream)
