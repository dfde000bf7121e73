"""One long sequence decoded with its entries split across ranks by entry
range (the 1M-entry contexts of the pages: DeepSeek V4.1-Flash Cuts KV Cache
by 437x, paragraph "CSA2 tackles storage"; DeepSeek V4.1 Flash Architecture
Breakdown, section "How does the cache compress along three dimensions at
once?").

Rank r holds entries [off_r, off_r + n_r) of the sequence in its own cache
and runs every kernel on its shard; each layer has one exchange step:
  Full     local Top-P (Top-K without a pool) -> 64-bit keys (score, ~global
           id) of those candidates -> all-gather -> every rank selects the
           same global pool and Top-K from the union (the global Top-P of the
           sequence is contained in the union of the local Top-Ps, and the id
           in the key keeps ties in ascending id order);
  Reindex  each rank scores the pool ids it owns -> all-gather -> select;
  Reuse    nothing;
  attention each rank attends over the selected ids it owns (rank 0 also
           over the window) into a normalised f32 partial with its
           log-sum-exp -> all-gather -> merge by log-sum-exp weights.
Every compute step is a library call; the exchange is a torch.distributed
all-gather (NCCL between GPUs). `LocalGroup` runs all shards in one process,
one after another, for single-GPU use and tests.

Limits: the all-gathered keys of one query (world x pool size for Full with a
pool and for Reindex, world x Top-K for Full without one) must not exceed
the 2^20 keys csa2_select_keys takes; entry offsets stay below 2^31.
"""
import math

import torch

from .workloads import resolve_schedule


def shard_ranges(n, world, align=128):
    """[(offset, count)] of `world` contiguous entry ranges covering n entries;
    offsets are multiples of `align` (the last range takes the rest)."""
    per = -(-n // world)
    per = -(-per // align) * align
    out, off = [], 0
    for r in range(world):
        cnt = max(0, min(n, off + per) - off)
        out.append((off, cnt))
        off += cnt
    return out


def local_ids(global_ids, off, n):
    """Global ids -> ids local to the range [off, off + n); others -> -1."""
    loc = global_ids - off
    return torch.where((global_ids >= 0) & (loc >= 0) & (loc < n), loc, torch.full_like(loc, -1)).to(torch.int32)


class LocalGroup:
    """All ranks' shards in this process: the gather stacks their tensors."""

    def __init__(self, world):
        self.world = world

    def gather(self, per_shard):
        assert len(per_shard) == self.world
        return torch.stack(per_shard)


class DistGroup:
    """One shard per process: the gather is a torch.distributed all-gather
    (into one tensor with NCCL, through a list with gloo)."""

    def __init__(self):
        import torch.distributed as dist
        self.dist = dist
        self.world = dist.get_world_size()
        self.nccl = dist.get_backend() == "nccl"

    def gather(self, per_shard):
        (mine,) = per_shard
        mine = mine.contiguous()
        if self.nccl:
            out = torch.empty((self.world,) + tuple(mine.shape), dtype=mine.dtype, device=mine.device)
            self.dist.all_gather_into_tensor(out, mine)
            return out
        parts = [torch.empty_like(mine) for _ in range(self.world)]
        self.dist.all_gather(parts, mine)
        return torch.stack(parts)


class EntryShard:
    """Rank r's part of one sequence: entries [off, off + n) in its own cache.
    `ops` holds the library calls (default: the binding of the CUDA library)."""

    def __init__(self, recipe, off, n, device, build_chunk=65536, ops=None):
        assert recipe.batch == 1, "one sequence"
        if ops is None:
            from . import binding as ops
        self.r, self.off, self.n, self.device = recipe, off, n, torch.device(device)
        self.ops = ops
        cap = max(128, -(-n // 128) * 128)
        self.cap = cap
        z = lambda *shape: torch.zeros(shape, dtype=torch.uint8, device=self.device)
        self.kv = ops.KvCache(z(cap, 256), z(cap, 32), z(cap, recipe.di),
                            torch.zeros((1, 1), dtype=torch.int32, device=self.device),
                            torch.full((1,), n, dtype=torch.int32, device=self.device), cap)
        for t0 in range(0, n, build_chunk):
            t1 = min(n, t0 + build_chunk)
            x = recipe.latent_rows(0, off + t0, off + t1, self.device).contiguous()
            pos = torch.arange(t0, t1, dtype=torch.int64, device=self.device)
            ops.csa2_append_fp4(x, torch.zeros(t1 - t0, dtype=torch.int32, device=self.device), pos, self.kv)
            self.kv.kidx[t0:t1] = recipe.kidx_rows(0, off + t0, off + t1, self.device)


class ShardedDecoder:
    """The layers of `recipe` (one sequence) over `shards` (one per rank held by
    this process; all of them for LocalGroup, one for DistGroup)."""

    def __init__(self, recipe, shards, group, reuse_from="previous"):
        self.r, self.shards, self.group = recipe, shards, group
        self.ops = B = shards[0].ops
        self.schedule = resolve_schedule(recipe.modes, reuse_from)
        dev = shards[0].device
        r = recipe
        self.q = [r.q(l, dev).contiguous() for l in range(r.layers)]
        self.qidx = [r.qidx(l, dev).contiguous() for l in range(r.layers)]
        self.w = [r.weights(l, dev).contiguous() for l in range(r.layers)]
        self.swa = [r.swa(l, dev).contiguous() for l in range(r.layers)]
        wb, we = r.swa_window()
        self.swa_begin, self.swa_end = wb.to(dev), we.to(dev)
        self.scale = 1.0 / math.sqrt(512.0)
        nq = r.nq
        self.topk = [None] * r.layers
        self.pool = [None] * r.layers
        self.o = [torch.empty((nq, r.h, 512), dtype=torch.bfloat16, device=dev) for _ in range(r.layers)]
        self.lse = [torch.empty((nq, r.h), dtype=torch.float32, device=dev) for _ in range(r.layers)]
        self.ws_full = [B.workspace(B.csa2_index_full_workspace_size(nq, s.n), dev) for s in shards]
        # the first shard attends with the window, the others without (their own split plans)
        self.ws_attn = B.workspace(max(B.csa2_sparse_attn_workspace_size(nq, r.h, r.k, r.w),
                                       B.csa2_sparse_attn_workspace_size(nq, r.h, r.k, 0)), dev)

    def topk_of(self, layer):
        mode, src = self.schedule[layer]
        return self.topk[layer] if mode != "reuse" else self.topk_of(src)

    def _gather_keys(self, per_shard):
        """[nq][m] keys per local shard -> [nq][world * m] keys of all ranks."""
        g = self.group.gather(per_shard)
        return g.permute(1, 0, 2).reshape(g.shape[1], -1).contiguous()

    def _select(self, keys, k):
        ids = torch.empty((keys.shape[0], k), dtype=torch.int32, device=keys.device)
        self.ops.csa2_select_keys(keys, k, ids)
        return ids

    def layer(self, l):
        B = self.ops
        r, (mode, src) = self.r, self.schedule[l]
        nq, dev = r.nq, self.shards[0].device
        if mode == "full":
            m = r.p if r.p > 0 else r.k
            keys = []
            for s, ws in zip(self.shards, self.ws_full):
                if s.n == 0:
                    keys.append(torch.zeros((nq, m), dtype=torch.int64, device=dev))
                    continue
                loc_k = torch.empty((nq, r.k), dtype=torch.int32, device=dev)
                loc_p = torch.empty((nq, r.p), dtype=torch.int32, device=dev) if r.p > 0 else None
                B.csa2_index_full(self.qidx[l], self.w[l], r.q_per_seq, None, s.n, s.kv, r.k, r.p, loc_k, loc_p, ws)
                cand = loc_p if loc_p is not None else loc_k
                kk = torch.empty((nq, m), dtype=torch.int64, device=dev)
                B.csa2_score_ids(self.qidx[l], self.w[l], r.q_per_seq, cand, s.kv, s.off, kk)
                keys.append(kk)
            allk = self._gather_keys(keys)
            self.topk[l] = self._select(allk, r.k)
            if r.p > 0:
                self.pool[l] = self._select(allk, r.p)
        elif mode == "reindex":
            pool = self.pool[src]
            keys = []
            for s in self.shards:
                kk = torch.zeros((nq, pool.shape[1]), dtype=torch.int64, device=dev)
                if s.n > 0:
                    B.csa2_score_ids(self.qidx[l], self.w[l], r.q_per_seq, local_ids(pool, s.off, s.n), s.kv, s.off,
                                     kk)
                keys.append(kk)
            self.topk[l] = self._select(self._gather_keys(keys), r.k)
        # attention: partial over the ids each rank owns (rank 0 also over the window)
        topk = self.topk_of(l)
        parts, lses = [], []
        for s in self.shards:
            o = torch.empty((nq, r.h, 512), dtype=torch.float32, device=dev)
            lse = torch.empty((nq, r.h), dtype=torch.float32, device=dev)
            first = s.off == 0
            B.csa2_sparse_attn_partial(self.q[l], r.q_per_seq, s.kv, local_ids(topk, s.off, s.n),
                                       self.swa[l] if first else None, self.swa[l].shape[1],
                                       self.swa_begin if first else None, self.swa_end if first else None,
                                       r.w if first else 0, self.scale, o, lse, self.ws_attn)
            parts.append(o)
            lses.append(lse)
        op, lp = self.group.gather(parts), self.group.gather(lses)
        B.csa2_attn_merge(op.contiguous(), lp.contiguous(), self.o[l], self.lse[l])

    def step(self):
        for l in range(self.r.layers):
            self.layer(l)
