"""Workload recipes: shapes, mode schedules and seeded synthetic inputs of
the five decode workloads the path is measured and checked on.

A recipe only says which numbers go where; values come from synth.py's
counter-based generator, so any row of any tensor can be drawn on the host
(for the oracle) or on the GPU (for the kernels) with identical bits. Nothing
here quantises, scores, selects or attends.

Workloads (names used by tests and bench.py):
  tiny_full  1 sequence, 1 query, N = 4096 entries, one Full layer,
             indexer 4 x 64, Top-K 512, 16 heads, window 128.
  stack20    20-layer decoder step, 8 sequences x 1 query, N = 65536 each,
             Full at layers 0 and 10, Reindex at 5 and 15 (pool 4096),
             Reuse elsewhere, Top-K 2048, 64 heads, window 512.
  hier1m     1 sequence, N = 1,048,576, Full (indexer 8 x 128, pool 8192)
             then 3 Reindex layers, Top-K 2048, 64 heads, window 1024.
  paged64    64 sequences, lengths uniform on [16384, 262144], 64-entry
             pages under a shuffled page table, Full + 3 Reuse, Top-K 2048,
             32 heads, window 512.
  chunk512   append 32768 rows (1% of values x20) to a 256K-entry cache
             holding 229376 rows, then 512 causal queries at positions
             261632..262143: Full (Top-K 2048) + attention with 32 heads over
             a 256-row window ending at the query.
Value distributions: latent rows and queries discretised N(0, 1) in bf16,
indexer keys and queries integers uniform on [-8, 8] stored as E4M3, head
weights integers uniform on [1, 4], window rows N(0, 1) rounded to E4M3.
"""
from dataclasses import dataclass, field, replace
import math

import torch

from . import synth

# value streams (the stream id of synth's generator)
S_LATENT, S_KIDX, S_LEN, S_PERM, S_APPEND, S_OUTLIER = 1, 2, 3, 4, 5, 6
S_QIDX, S_W, S_Q, S_SWA = 100, 200, 300, 400
T_STRIDE = 1 << 22  # counter stride between sequences (max entries per sequence)
S_CACHE = 1000       # stream offset between the caches of the per-Full-layer variant


@dataclass(frozen=True)
class Recipe:
    name: str
    seed: int
    batch: int
    q_per_seq: int
    modes: str               # one letter per layer: F(ull), R(eindex), U(se = Reuse)
    hi: int
    di: int
    k: int
    p: int                   # pool size built by Full layers (0 = none)
    h: int
    w: int                   # window rows per query
    n: int = 0               # entries per sequence (fixed-length workloads)
    n_range: tuple = None    # (lo, hi) inclusive, drawn per sequence
    page_size: int = 0       # 0 = one contiguous page per sequence
    cap: int = 0             # per-sequence capacity (0 = rounded-up length)
    prefill: int = 0         # rows present before the append (chunk512)
    append: int = 0          # rows appended in the step (chunk512)
    outlier_p: float = 0.0
    outlier_mul: float = 1.0
    swa_rows: int = 0        # window buffer rows per sequence (0 = w)
    chunked: bool = False    # queries at the last q_per_seq positions, causal
    cache_per_full: bool = False  # every Full layer has its own global KV (cache c = c-th Full layer)
    extra: dict = field(default_factory=dict)

    # ---- sizes ----------------------------------------------------------------
    @property
    def nq(self):
        return self.batch * self.q_per_seq

    @property
    def layers(self):
        return len(self.modes)

    def seq_lens(self):
        if self.n_range is not None:
            lo, hi = self.n_range
            return synth.uniform_int(self.seed, S_LEN, 0, self.batch, lo, hi)
        total = self.prefill + self.append if self.chunked else self.n
        return torch.full((self.batch,), total, dtype=torch.int64)

    def layout(self):
        """(page_size, page_table int32 [batch, max_pages], rows_cap)."""
        lens = self.seq_lens()
        if self.page_size == 0:
            cap = self.cap or int(math.ceil(int(lens.max()) / 128) * 128)
            pt = torch.arange(self.batch, dtype=torch.int32).view(self.batch, 1)
            return cap, pt, cap * self.batch
        ps = self.page_size
        npages = [(int(l) + ps - 1) // ps for l in lens.tolist()]
        total = sum(npages)
        perm = synth.permutation(self.seed, S_PERM, total)
        max_pages = max(npages)
        pt = torch.zeros((self.batch, max_pages), dtype=torch.int32)
        off = 0
        for b, c in enumerate(npages):
            pt[b, :c] = perm[off:off + c]
            off += c
        return ps, pt, total * ps

    def window_rows(self):
        return self.swa_rows or self.w

    # ---- values ---------------------------------------------------------------
    def latent_rows(self, b, t0, t1, device="cpu", cache=0):
        """bf16 [t1 - t0, 512]: latent rows of sequence b at positions t0..t1-1
        of cache `cache` (appended rows of the chunked workload carry the
        outliers). Cache 0 is the shared cache; with cache_per_full, cache c
        belongs to the c-th Full layer and draws from its own streams."""
        off = S_CACHE * cache
        if self.chunked and t1 > self.prefill:
            assert t0 >= self.prefill, "split prefill/append ranges"
            c0 = ((b * T_STRIDE) + (t0 - self.prefill)) * 512
            return synth.normal_bf16(self.seed, S_APPEND + off, c0, (t1 - t0) * 512, device,
                                     outlier_p=self.outlier_p, outlier_mul=self.outlier_mul,
                                     outlier_stream=S_OUTLIER + off).view(t1 - t0, 512)
        c0 = (b * T_STRIDE + t0) * 512
        return synth.normal_bf16(self.seed, S_LATENT + off, c0, (t1 - t0) * 512, device).view(t1 - t0, 512)

    def kidx_rows(self, b, t0, t1, device="cpu", cache=0):
        c0 = (b * T_STRIDE + t0) * self.di
        return synth.int_e4m3(self.seed, S_KIDX + S_CACHE * cache, c0, (t1 - t0) * self.di,
                              device=device).view(t1 - t0, self.di)

    def caches(self):
        """Number of global KV caches: 1 (shared by all layers) or one per Full layer."""
        return max(1, self.modes.count("F")) if self.cache_per_full else 1

    def qidx(self, layer, device="cpu"):
        n = self.nq * self.hi * self.di
        return synth.int_e4m3(self.seed, S_QIDX + layer, 0, n, device=device).view(self.nq, self.hi, self.di)

    def weights(self, layer, device="cpu"):
        v = synth.uniform_int(self.seed, S_W + layer, 0, self.nq * self.hi, 1, 4, device)
        return v.to(torch.float32).view(self.nq, self.hi)

    def q(self, layer, device="cpu", rows=None):
        """bf16 [nq, h, 512] (or only the query rows listed in `rows`)."""
        per = self.h * 512
        if rows is None:
            return synth.normal_bf16(self.seed, S_Q + layer, 0, self.nq * per, device).view(self.nq, self.h, 512)
        out = [synth.normal_bf16(self.seed, S_Q + layer, r * per, per, device).view(self.h, 512) for r in rows]
        return torch.stack(out)

    def swa(self, layer, device="cpu", seqs=None):
        """uint8 E4M3 [batch, window_rows, 512] window buffer of one layer."""
        seqs = range(self.batch) if seqs is None else seqs
        per = self.window_rows() * 512
        out = [synth.normal_e4m3(self.seed, S_SWA + layer, b * per, per, device).view(self.window_rows(), 512)
               for b in seqs]
        return torch.stack(out)

    def swa_window(self):
        """(begin, end) int32 [nq]: each query's window rows in its buffer."""
        if self.chunked:
            j = torch.arange(self.q_per_seq, dtype=torch.int32).repeat(self.batch)
            return j, j + self.w
        z = torch.zeros(self.nq, dtype=torch.int32)
        return z, z + self.w

    def q_limit(self):
        """int32 [nq] visible entries per query (chunked: causal), or None."""
        if not self.chunked:
            return None
        total = self.prefill + self.append
        first = total - self.q_per_seq
        j = torch.arange(self.q_per_seq, dtype=torch.int32).repeat(self.batch)
        return first + j + 1

    def scaled(self, **kw):
        return replace(self, **kw)


RECIPES = {
    "tiny_full": Recipe("tiny_full", seed=0, batch=1, q_per_seq=1, modes="F", hi=4, di=64, k=512, p=0, h=16,
                        w=128, n=4096),
    "stack20": Recipe("stack20", seed=1, batch=8, q_per_seq=1, modes="FUUUURUUUUFUUUURUUUU", hi=4, di=64, k=2048,
                      p=4096, h=64, w=512, n=65536),
    "hier1m": Recipe("hier1m", seed=2, batch=1, q_per_seq=1, modes="FRRR", hi=8, di=128, k=2048, p=8192, h=64,
                     w=1024, n=1048576),
    "paged64": Recipe("paged64", seed=3, batch=64, q_per_seq=1, modes="FUUU", hi=4, di=64, k=2048, p=0, h=32,
                      w=512, n_range=(16384, 262144), page_size=64),
    "chunk512": Recipe("chunk512", seed=4, batch=1, q_per_seq=512, modes="F", hi=4, di=64, k=2048, p=0, h=32,
                       w=256, cap=262144, prefill=229376, append=32768, outlier_p=0.01, outlier_mul=20.0,
                       swa_rows=767, chunked=True),
}


def cache_of_layers(modes, schedule, per_full):
    """Cache index read by every layer: 0 for all layers with one shared cache;
    with one cache per Full layer, a Full layer reads its own, a Reindex layer
    its source Full layer's, a Reuse layer its source layer's."""
    if not per_full:
        return [0] * len(modes)
    out, fulls = [], 0
    for layer, (mode, src) in enumerate(schedule):
        if mode == "full":
            out.append(fulls)
            fulls += 1
        else:
            out.append(out[src])
    return out


def resolve_schedule(modes, reuse_from="previous"):
    """[(mode, source_layer)] for a mode string. Reindex re-scores the pool of
    the most recent Full layer. Reuse takes the Top-k of the most recent layer
    that produced one (reuse_from='previous': Reuse takes over the earlier
    indices as they are) or of the most recent Full layer (reuse_from='full')."""
    out, last_full, last_idx = [], None, None
    for layer, m in enumerate(modes):
        if m == "F":
            out.append(("full", -1))
            last_full = last_idx = layer
        elif m == "R":
            if last_full is None:
                raise ValueError("Reindex layer before any Full layer")
            out.append(("reindex", last_full))
            last_idx = layer
        elif m == "U":
            if last_idx is None:
                raise ValueError("Reuse layer before any index-producing layer")
            out.append(("reuse", last_idx if reuse_from == "previous" else last_full))
        else:
            raise ValueError(f"unknown mode {m!r}")
    return out
