"""Benchmark of the CSA2 decode hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload all|NAME]
    python bench.py --impl reference ...      # the CPU oracle, same metric

A step is one decode step of a workload through the C-ABI: FP4 append of the
step's new rows, then every layer of the static mode schedule (Full /
Reindex indexer where scheduled, Reuse otherwise) followed by sparse + window
attention. Every workload of the benchmark set is measured (tiny_full,
stack20, hier1m, paged64, chunk512; --workload picks one); the JSON line
carries one record per workload under "configs", and its headline fields are
those of the largest single-GPU workload, paged64 (64 paged sequences of
16K-256K entries, Full + 3 Reuse layers, 32 heads).

Metric: decode query-steps per second per layer = sequences * queries *
layers / step time, with the achieved HBM bandwidth of the step's
algorithmic bytes. Timing: each workload's step is captured once in a CUDA
graph; each of the K timed steps is preceded by an L2 flush (256 MiB written,
then another 256 MiB read, so no dirty line is left to write back) and
bracketed by CUDA events on the launching stream; a barrier and a device
synchronize bracket each workload's timed loop; the reported time is the max
over ranks. Multi-GPU runs give every rank its own independent sequences
(weak scaling, no collective on the data path).
"""
import argparse
import datetime
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "CSA2 decode query-steps/s per layer; achieved HBM TB/s vs ~8 TB/s peak"
UNIT = "query-steps/s/layer"
WORKLOADS = ("tiny_full", "stack20", "hier1m", "paged64", "chunk512")
HEADLINE = "paged64"  # the largest workload that fits one GPU


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="all", help="one workload, or 'all' (the default)")
    ap.add_argument("--headline", default=HEADLINE, help="workload whose record fills the headline fields")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-sharded", action="store_true", help="skip the entry-range sharded side measurement")
    ap.add_argument("--no-side", action="store_true",
                    help="skip every side measurement (appends, sharded decode, attention variants)")
    return ap.parse_args()


# ---------------------------------------------------------------------------
# algorithmic work (what the method must move / compute)
# ---------------------------------------------------------------------------
def call_costs(recipe, lens, schedule):
    """[(kind, layer, bytes, flops, tc)] of the step's C-ABI calls in order:
    algorithmic bytes (inputs read once, outputs written once) and flops; tc
    names the tensor-core type of the flops ('fp8' indexer products, 'f16'
    attention products, None)."""
    nq, h, d = recipe.nq, recipe.h, 512
    n_vis = [int(l) for l in lens.tolist()]
    out = []
    rows_app = recipe.append if recipe.chunked else recipe.batch
    out.append(("append", -1, rows_app * (d * 2 + d // 2 + d // 16), 0.0, None))
    ql = recipe.q_limit()
    for l, (mode, src) in enumerate(schedule):
        if mode == "full":
            # keys of a sequence are read once for all its queries (the widest
            # visible range); every query scores each visible key
            b = f = 0.0
            seq_n = {}
            for qi in range(nq):
                n = int(ql[qi]) if ql is not None else n_vis[qi // recipe.q_per_seq]
                sq = qi // recipe.q_per_seq
                seq_n[sq] = max(seq_n.get(sq, 0), n)
                b += 4 * (recipe.k + recipe.p) + recipe.hi * (recipe.di + 4)
                f += 2.0 * recipe.hi * recipe.di * n
            b += sum(seq_n.values()) * recipe.di
            out.append(("full", l, b, f, "fp8"))
        elif mode == "reindex":
            out.append(("reindex", l, nq * recipe.p * (recipe.di + 4) + nq * recipe.k * 4,
                        2.0 * nq * recipe.hi * recipe.di * recipe.p, "fp8"))
        a_by = nq * (recipe.k * (d // 2 + d // 16 + 4) + recipe.w * d + 2 * 2 * h * d)
        a_fl = 4.0 * nq * h * (recipe.k + recipe.w) * d
        out.append(("attention", l, a_by, a_fl, "f16"))
    return out


def call_roof_us(by, fl, tc, hbm_gbs, peaks_tf):
    """max(bytes / HBM peak, flops / tensor peak of the call's type), in us,
    and which of the two bounds it."""
    t_b = by / (hbm_gbs * 1e9) * 1e6
    t_f = fl / (peaks_tf[tc] * 1e12) * 1e6 if tc else 0.0
    return (t_b, "hbm") if t_b >= t_f else (t_f, "tensor")


def time_append_chunk512(B, dev, hbm_gbs, reps=20):
    """The 32,768-row FP4 append of the chunked-prefill workload (a 256K-entry
    cache), timed on its own: CUDA events around each call, L2 flushed before
    each."""
    import torch
    from sparse_fp4_kv_b200.workloads import RECIPES
    r = RECIPES["chunk512"]
    cap, n = r.cap, r.append
    codes = torch.zeros((cap, 256), dtype=torch.uint8, device=dev)
    scales = torch.zeros((cap, 32), dtype=torch.uint8, device=dev)
    kidx = torch.zeros((cap, r.di), dtype=torch.uint8, device=dev)
    pt = torch.zeros((1, 1), dtype=torch.int32, device=dev)
    sl = torch.full((1,), cap, dtype=torch.int32, device=dev)
    kv = B.KvCache(codes, scales, kidx, pt, sl, cap)
    x = r.latent_rows(0, r.prefill, r.prefill + n, dev).contiguous()
    seq = torch.zeros(n, dtype=torch.int32, device=dev)
    pos = torch.arange(r.prefill, r.prefill + n, dtype=torch.int64, device=dev)
    flush = L2Flush(dev)
    stream = torch.cuda.Stream(dev)
    for _ in range(3):
        B.csa2_append_fp4(x, seq, pos, kv)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        B.csa2_append_fp4(x, seq, pos, kv, stream)
    res = {}
    for mode, run in (("eager", lambda: B.csa2_append_fp4(x, seq, pos, kv, stream)), ("graph", g.replay)):
        ts = []
        for i in range(reps):
            with torch.cuda.stream(stream):
                flush.fill_(i & 0xFF)
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                run()
                e1.record(stream)
            e1.synchronize()
            ts.append(e0.elapsed_time(e1) * 1e3)
        ts.sort()
        res[mode] = ts[len(ts) // 2]
    del g
    by = n * (512 * 2 + 256 + 32)
    us = res["graph"]
    return {"rows": n, "us_median_graph": us, "us_median_eager": res["eager"], "algorithmic_bytes": by,
            "achieved_gbs": by / (us * 1e-6) / 1e9, "peak_gbs": hbm_gbs, "frac": by / (us * 1e-6) / 1e9 / hbm_gbs,
            "note": "bf16 rows in, FP4 codes + E4M3 scales out, 256K-entry cache; CUDA events around the call, "
                    "replayed from a CUDA graph (frac) and eager (launch included), median of %d, L2 flushed "
                    "before each" % reps}


def time_append_e4m3(B, dev, hbm_gbs, reps=20):
    """The FP8 appends at chunked-prefill size: 32,768 window rows (512 values)
    into a ring of 32,768 slots, and 32,768 indexer keys (64 values) into a
    256K-entry key array; CUDA events around each call, L2 flushed before each."""
    import torch
    from sparse_fp4_kv_b200 import synth
    n, ring, cap, di = 32768, 32768, 262144, 64
    flush = L2Flush(dev)
    xw = synth.normal_bf16(11, 1, 0, n * 512).view(n, 512).to(dev)
    xk = synth.normal_bf16(11, 2, 0, n * di).view(n, di).to(dev)
    swa = torch.zeros((1, ring, 512), dtype=torch.uint8, device=dev)
    codes = torch.zeros((cap, 256), dtype=torch.uint8, device=dev)
    scales = torch.zeros((cap, 32), dtype=torch.uint8, device=dev)
    kidx = torch.zeros((cap, di), dtype=torch.uint8, device=dev)
    kv = B.KvCache(codes, scales, kidx, torch.zeros((1, 1), dtype=torch.int32, device=dev),
                   torch.full((1,), cap, dtype=torch.int32, device=dev), cap)
    seq = torch.zeros(n, dtype=torch.int32, device=dev)
    pos = torch.arange(cap - n, cap, dtype=torch.int64, device=dev)
    stream = torch.cuda.Stream(dev)
    out = {}
    for name, call, by in (("window", lambda s: B.csa2_append_swa_e4m3(xw, seq, pos, swa, s), n * 512 * 3),
                           ("keys", lambda s: B.csa2_append_kidx_e4m3(xk, seq, pos, kv, s), n * di * 3)):
        for _ in range(3):
            call(stream)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            call(stream)
        res = {}
        for mode, run in (("eager", lambda: call(stream)), ("graph", g.replay)):
            ts = []
            for i in range(reps):
                with torch.cuda.stream(stream):
                    flush.fill_(i & 0xFF)
                    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                    e0.record(stream)
                    run()
                    e1.record(stream)
                e1.synchronize()
                ts.append(e0.elapsed_time(e1) * 1e3)
            ts.sort()
            res[mode] = ts[len(ts) // 2]
        del g
        us = res["graph"]
        out[name] = {"rows": n, "us_median_graph": us, "us_median_eager": res["eager"], "algorithmic_bytes": by,
                     "achieved_gbs": by / (us * 1e-6) / 1e9, "frac": by / (us * 1e-6) / 1e9 / hbm_gbs}
    out["note"] = ("bf16 in, E4M3 out; CUDA events around the call, replayed from a CUDA graph (frac) and eager "
                   "(launch included), median of %d, L2 flushed before each" % reps)
    return out


def time_attn_variants(B, dec, reps=30):
    """One attention layer of the benchmark step (layer 0's queries, Top-K and
    window) through the exact call and through the NVFP4 variant (q rounded to
    NVFP4 for the scores, FP4 block-scaled products on the selected entries);
    CUDA events around each call (kernel + merge), L2 flushed before each,
    median of `reps`."""
    import torch
    r = dec.r
    dev = dec.device
    flush = L2Flush(dev)
    topk = dec.topk_of(0)
    o = torch.empty_like(dec.o[0])
    lse = torch.empty_like(dec.lse[0])
    ws_nv = B.workspace(B.csa2_sparse_attn_nvfp4_workspace_size(r.nq, r.h, r.k, r.w), dev)
    args = (dec.q[0], r.q_per_seq, dec.kv, topk, dec.swa[0], dec.swa[0].shape[1], dec.swa_begin, dec.swa_end, r.w,
            dec.scale, o, lse)
    calls = {"exact": lambda: B.csa2_sparse_attn_decode(*args, dec.ws_attn),
             "nvfp4": lambda: B.csa2_sparse_attn_decode_nvfp4(*args, ws_nv)}
    out = {}
    stream = torch.cuda.Stream(device=dev)
    for name, call in calls.items():
        for _ in range(3):
            call()
        torch.cuda.synchronize()
        # the call captured in a CUDA graph, as in the decode step
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            call()
        for mode, run in (("eager", call), ("graph", g.replay)):
            ts = []
            for i in range(reps):
                with torch.cuda.stream(stream):
                    flush.fill_(i & 0xFF)
                    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                    e0.record(stream)
                    run()
                    e1.record(stream)
                e1.synchronize()
                ts.append(e0.elapsed_time(e1) * 1e3)
            ts.sort()
            out[f"{name}_{mode}_us"] = ts[len(ts) // 2]
        del g
    if B.csa2_device_status() != 0:
        raise RuntimeError("device error in the attention variants")
    out["speedup_graph"] = out["exact_graph_us"] / out["nvfp4_graph_us"]
    out["note"] = (f"{r.name} layer 0: {r.nq} queries x {r.h} heads, Top-K {r.k} + window {r.w}; events around "
                   f"each call (exact: attention + merge kernels; nvfp4: q quantisation + attention + merge), eager "
                   f"and replayed from a CUDA graph, median of {reps} after an L2 flush")
    return out


def time_sharded_hier1m(dev, world=2, reps=5):
    """The 1M-entry sequence split by entry range into `world` shards, all on
    this GPU one after another (local Full, key exchange, select, Reindex,
    attention partials, merge); CUDA events around each step, L2 flushed
    before each. One rank of a real split runs one shard's share of the
    kernels plus the all-gathers whose sizes are given."""
    import torch
    from sparse_fp4_kv_b200.sharded import EntryShard, LocalGroup, ShardedDecoder, shard_ranges
    from sparse_fp4_kv_b200.workloads import RECIPES
    r = RECIPES["hier1m"]
    shards = [EntryShard(r, off, n, dev) for off, n in shard_ranges(r.n, world)]
    dec = ShardedDecoder(r, shards, LocalGroup(world))
    flush = L2Flush(dev)
    for _ in range(2):
        dec.step()
    ts = []
    for i in range(reps):
        flush.fill_(i & 0xFF)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        dec.step()
        e1.record()
        e1.synchronize()
        ts.append(e0.elapsed_time(e1))
    ts.sort()
    ms = ts[len(ts) // 2]
    keys = sum((r.p if r.p else r.k) * 8 for m, _ in dec.schedule if m in ("full", "reindex")) * r.nq
    parts = r.layers * r.nq * r.h * (512 + 1) * 4
    del dec, shards
    return {"workload": "hier1m", "shards": world, "ms_per_step_all_shards_one_gpu": ms,
            "bytes_sent_per_rank_per_step": keys + parts,
            "note": f"shards run sequentially on one GPU; median of {reps} steps (no append in the step)"}


class L2Flush:
    """Clears the 126 MB L2 between timed iterations: fill_() writes a
    256 MiB buffer, then reads a second 256 MiB buffer, so the timed kernels
    find neither their inputs nor the flush's dirty lines in L2 (the write-back
    of those would otherwise land inside the timed region)."""

    def __init__(self, dev):
        import torch
        self.w = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
        self.r = torch.zeros(64 << 20, dtype=torch.int32, device=dev)

    def fill_(self, v):
        self.w.fill_(v)
        self.r.sum()


def peaks():
    """Roofline denominators: the measured copy bandwidth and cuBLAS
    bf16 rates of this machine's B200s (MEASURED_PEAKS.json), else the fallback
    figures of the same pool."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        return {"hbm_gbs": float(j.get("hbm_gbs", 6650.0)), "bf16_tflops": float(j.get("bf16_tflops", 1590.0)),
                "bf16_tflops_sustained": float(j.get("bf16_tflops_sustained", 1400.0)), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def measure_tc_probe(dev):
    """Tensor-core rates of this library's own instruction forms (tcgen05.mma
    kind::f16 and kind::f8f6f4, M = 128, every SM, CUDA events around the
    grid): TF/s per (kind, N)."""
    import ctypes
    import torch
    lib = ctypes.CDLL(os.path.join(ROOT, "sparse_fp4_kv_b200", "libcsa2_peak.so"))
    lib.peak_tcgen05.restype = ctypes.c_float
    lib.peak_tcgen05.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_void_p]
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    stream = torch.cuda.current_stream(dev).cuda_stream
    iters = 1 << 15
    out = {}
    for kind, name, kk in ((0, "f16", 16), (1, "fp8_e4m3", 32)):
        for n in (64, 256):
            ms = min(lib.peak_tcgen05(kind, n, iters, stream) for _ in range(3))
            if ms > 0:
                out[f"{name}_n{n}_tflops"] = 2.0 * 128 * n * kk * iters * sms / (ms * 1e-3) / 1e12
    out["note"] = ("one CTA per SM issuing tcgen05.mma (M = 128, operands in shared memory) back to back; "
                   f"{iters} instructions per SM, CUDA events around the grid")
    return out


def code_of(src):
    """C++/CUDA source without comments, trailing blanks and empty lines (what the
    compiler sees), so that comment edits do not count as kernel changes."""
    out, i, n = [], 0, len(src)
    while i < n:
        if src.startswith("//", i):
            j = src.find("\n", i)
            i = n if j < 0 else j
        elif src.startswith("/*", i):
            j = src.find("*/", i + 2)
            i = n if j < 0 else j + 2
        elif src[i] == '"':
            j = i + 1
            while j < n and src[j] != '"':
                j += 2 if src[j] == "\\" else 1
            out.append(src[i:j + 1])
            i = j + 1
        else:
            out.append(src[i])
            i += 1
    return "\n".join(ln.rstrip() for ln in "".join(out).split("\n") if ln.strip())


def kernel_source_hash(csrc=None):
    csrc = csrc or os.path.join(ROOT, "sparse_fp4_kv_b200", "csrc")
    h = hashlib.sha256()
    for fn in sorted(os.listdir(csrc)):
        with open(os.path.join(csrc, fn), encoding="utf-8") as f:
            h.update(code_of(f.read()).encode())
    return h.hexdigest()[:16]


def recorded_traffic(kernel, workload):
    """Per-launch DRAM bytes of `kernel` from a committed ncu summary, if it was
    taken on the current kernel sources."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        j = json.load(f)
    e = j.get(f"{kernel}:{workload}")
    if not e or e.get("source_hash") != kernel_source_hash():
        return None
    return e.get("dram_bytes_per_launch")


# ---------------------------------------------------------------------------
# clocks sampler
# ---------------------------------------------------------------------------
class Clocks:
    """SM clock, power and throttle reasons of this rank's GPU, read through
    NVML by a thread every 2 ms (reading only: no setting is touched).
    summary() describes the samples taken between the last mark(0) and
    mark(1) (a timed region)."""
    PERIOD_S = 0.002

    def __init__(self, device):
        self.device = device
        self.window = [None, None]
        self.rows = []  # (perf_counter time, sm MHz, max MHz, power W, reasons)
        self.thread = None
        self.stop_flag = False
        self.error = None

    def _nvml_handle(self):
        """NVML handle of this process's CUDA device: by UUID (NVML does not
        follow CUDA_VISIBLE_DEVICES), else by index."""
        import pynvml
        import torch
        pynvml.nvmlInit()
        try:
            uuid = str(torch.cuda.get_device_properties(self.device).uuid)
            return pynvml.nvmlDeviceGetHandleByUUID(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
        except Exception:
            return pynvml.nvmlDeviceGetHandleByIndex(int(self.device.index or 0))

    def start(self):
        try:
            import threading
            import pynvml
            h = self._nvml_handle()
            bits = {"hw_slowdown": pynvml.nvmlClocksEventReasonHwSlowdown,
                    "hw_thermal_slowdown": pynvml.nvmlClocksEventReasonHwThermalSlowdown,
                    "sw_thermal_slowdown": pynvml.nvmlClocksEventReasonSwThermalSlowdown,
                    "sw_power_cap": pynvml.nvmlClocksEventReasonSwPowerCap}
            max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM))

            def loop():
                while not self.stop_flag:
                    t = time.perf_counter()
                    try:
                        sm = float(pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM))
                        pw = pynvml.nvmlDeviceGetPowerUsage(h) / 1000.0
                        rs = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
                        self.rows.append((t, sm, max_mhz, pw, [n for n, b in bits.items() if rs & b]))
                    except Exception:
                        pass
                    time.sleep(self.PERIOD_S)

            self.thread = threading.Thread(target=loop, daemon=True)
            self.thread.start()
        except Exception as e:  # no NVML: the record says so
            self.thread = None
            self.error = str(e)[:80]

    def mark(self, which):
        self.window[which] = time.perf_counter()

    def summary(self):
        if self.thread is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [f"no clock source ({self.error})"]}
        t0, t1 = self.window
        inside = [r for r in list(self.rows) if t0 is not None and t1 is not None and t0 <= r[0] <= t1]
        reasons = sorted({n for r in inside for n in r[4]})
        return {"sm_mhz": statistics.median(r[1] for r in inside) if inside else None,
                "sm_max_mhz": max(r[2] for r in inside) if inside else None, "reasons": reasons,
                "samples_in_timed_region": len(inside),
                "power_w_median": statistics.median(r[3] for r in inside) if inside else None,
                "source": "NVML every 2 ms"}

    def stop(self):
        self.stop_flag = True
        if self.thread is not None:
            self.thread.join(timeout=5)


# ---------------------------------------------------------------------------
# CPU oracle (cpu_baseline leg and --impl reference)
# ---------------------------------------------------------------------------
def oracle_sample(recipe, layers, seq=0, queries=None):
    """Time the oracle's step for one sequence over `layers` and the listed
    queries of that sequence (all of them by default); cache build and input
    generation are excluded. Returns (seconds, query-layers processed)."""
    import numpy as np
    import torch
    import oracle
    import oracle.stack as ostack
    sched = ostack.schedule(recipe.modes)
    cache = ostack.SeqCache(recipe, seq)
    js = list(range(recipe.q_per_seq)) if queries is None else list(queries)
    qis = [seq * recipe.q_per_seq + j for j in js]
    inputs = {}
    for l in layers:
        inputs[l] = (recipe.qidx(l).numpy(), recipe.weights(l).numpy(), recipe.q(l, rows=qis),
                     recipe.swa(l, seqs=[seq])[0].numpy())
    wb, we = recipe.swa_window()
    ql = recipe.q_limit()
    scale = 1.0 / math.sqrt(512.0)
    topk, pool = {}, {}
    t0 = time.perf_counter()
    for l in layers:
        mode, src = sched[l]
        qidx, w, q, swa = inputs[l]
        for j, qi in enumerate(qis):
            if mode == "full":
                lim = int(ql[qi]) if ql is not None else cache.n
                topk[(l, qi)], pool[(l, qi)] = oracle.index_full(qidx[qi], w[qi], cache.kidx, cache.page_table,
                                                                 cache.page_size, lim, recipe.k, recipe.p)
            elif mode == "reindex":
                topk[(l, qi)] = oracle.index_reindex(qidx[qi], w[qi], cache.kidx, cache.page_table, cache.page_size,
                                                     pool[(src, qi)], recipe.k)
            else:
                topk[(l, qi)] = topk[(src, qi)]
            oracle.sparse_attn(ostack.bf16_bits(q[j]), cache.codes, cache.scales, cache.page_table, cache.page_size,
                               topk[(l, qi)], swa[int(wb[qi]):int(we[qi])], scale)
    return time.perf_counter() - t0, len(qis) * len(layers)


# Bounded oracle samples of each workload (a few seconds of single-threaded
# CPU work each): (sequence, queries of it or None for all), layers = all.
CPU_SAMPLE = {"tiny_full": (0, None), "stack20": (0, None), "hier1m": (0, None), "paged64": (0, None),
              "chunk512": (0, [0, 511])}


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return None


def _oracle_worker(job):
    recipe, seq, queries, layers = job
    return oracle_sample(recipe, layers, seq, queries)


def oracle_all_cores(recipe, layers, procs):
    """The oracle on independent units at once, one spawned process each (no
    GPU): sequences 0..procs-1, or queries of sequence 0 for a one-sequence
    workload. Units of all processes over the longest process's time."""
    import multiprocessing as mp
    if recipe.batch >= procs:
        jobs = [(recipe, s, [0] if recipe.q_per_seq > 1 else None, layers) for s in range(procs)]
        what = f"sequences 0..{procs - 1}"
    else:
        jobs = [(recipe, 0, [j], layers) for j in range(procs)]
        what = f"queries 0..{procs - 1} of sequence 0"
    with mp.get_context("spawn").Pool(procs) as pool:
        res = pool.map(_oracle_worker, jobs)
    dt = max(r[0] for r in res)
    n = sum(r[1] for r in res)
    return {"value": n / dt, "unit": UNIT, "cores": procs,
            "sample": f"{what}, layers {layers[0]}..{layers[-1]}, one process each ({dt:.1f} s)"}


def cpu_baseline(recipe):
    layers = list(range(recipe.layers))
    seq, queries = CPU_SAMPLE.get(recipe.name, (0, None))
    dt, n = oracle_sample(recipe, layers, seq, queries)
    nq = recipe.q_per_seq if queries is None else len(queries)
    rec = {"value": n / dt, "unit": UNIT, "cores": 1, "kind": "oracle",
           "sample": f"sequence {seq} ({nq} quer{'y' if nq == 1 else 'ies'}), layers {layers[0]}..{layers[-1]} of "
                     f"{recipe.name}, single-threaded C oracle ({dt:.1f} s)",
           "cpu_model": cpu_model(), "nproc": os.cpu_count()}
    units = recipe.batch if recipe.batch > 1 else recipe.q_per_seq
    procs = max(1, min(os.cpu_count() or 1, 8, units))
    if procs > 1:
        rec["all_cores"] = oracle_all_cores(recipe, layers, procs)
    return rec


def run_reference(args):
    from sparse_fp4_kv_b200.workloads import RECIPES
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    name = args.headline if args.workload == "all" else args.workload
    recipe = RECIPES[name]
    layers = list(range(recipe.layers))
    seq, queries = CPU_SAMPLE.get(recipe.name, (0, None))
    times = []
    n_units = 0
    for i in range(args.warmup + args.steps):
        dt, n_units = oracle_sample(recipe, layers, seq, queries)
        if i >= args.warmup:
            times.append(dt)
    total = sum(times)
    value = n_units * len(times) / total
    nq = recipe.q_per_seq if queries is None else len(queries)
    sample = (f"sequence {seq} of {recipe.name} ({nq} quer{'y' if nq == 1 else 'ies'}), layers "
              f"{layers[0]}..{layers[-1]} ({recipe.modes}), single-threaded C oracle, per step")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / len(times),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": recipe.name, "sample_layers": layers},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------
def graph_kernel_nodes(g):
    """Kernel nodes of a captured CUDA graph (the library's kernels: the step
    graph holds nothing else), counted through the driver API, or None if the
    graph cannot be inspected."""
    import ctypes
    try:
        cuda = ctypes.CDLL("libcuda.so.1")
        cuda.cuGraphGetNodes.restype = ctypes.c_int
        cuda.cuGraphGetNodes.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.POINTER(ctypes.c_size_t)]
        cuda.cuGraphNodeGetType.restype = ctypes.c_int
        cuda.cuGraphNodeGetType.argtypes = [ctypes.c_void_p, ctypes.POINTER(ctypes.c_int)]
        h = ctypes.c_void_p(int(g.raw_cuda_graph()))
        n = ctypes.c_size_t(0)
        if cuda.cuGraphGetNodes(h, None, ctypes.byref(n)) != 0:
            return None
        nodes = (ctypes.c_void_p * max(1, n.value))()
        if cuda.cuGraphGetNodes(h, nodes, ctypes.byref(n)) != 0:
            return None
        kernels = 0
        for i in range(n.value):
            t = ctypes.c_int(-1)
            if cuda.cuGraphNodeGetType(ctypes.c_void_p(nodes[i]), ctypes.byref(t)) != 0:
                return None
            kernels += t.value == 0  # CU_GRAPH_NODE_TYPE_KERNEL
        return kernels
    except Exception:
        return None


def issue_call(dec, kind, l, s):
    """One C-ABI call of the step on stream s."""
    from sparse_fp4_kv_b200 import binding as B
    r = dec.r
    if kind == "append":
        dec.append(s)
    elif kind == "full":
        B.csa2_index_full(dec.qidx[l], dec.w[l], r.q_per_seq, dec.q_limit, dec.n_max, dec.kv, r.k,
                          r.p if dec.pool[l] is not None else 0, dec.topk[l], dec.pool[l], dec.ws_full, s)
    elif kind == "reindex":
        src = dec.schedule[l][1]
        B.csa2_index_reindex(dec.qidx[l], dec.w[l], r.q_per_seq, dec.pool[src], dec.kv, r.k, dec.topk[l],
                             dec.ws_reindex, s)
    else:
        B.csa2_sparse_attn_decode(dec.q[l], r.q_per_seq, dec.kv, dec.topk_of(l), dec.swa[l], dec.swa[l].shape[1],
                                  dec.swa_begin, dec.swa_end, r.w, dec.scale, dec.o[l], dec.lse[l], dec.ws_attn, s)


def graph_times_us(g, stream, flush, n):
    """n replays of graph g, each after an L2 flush, CUDA events on the stream."""
    import torch
    st = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
    en = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
    out = []
    for i in range(n):
        with torch.cuda.stream(stream):
            flush.fill_(i & 0xFF)
            st[i].record(stream)
            g.replay()
            en[i].record(stream)
        en[i].synchronize()
        out.append(st[i].elapsed_time(en[i]) * 1e3)
    return out


def bench_workload(name, args, world, rank, dev, stream, flush, clocks, pk):
    """One workload: the timed step (value, ms_per_step), the per-call
    breakdown, the roofline of its dominant call, e2e and the CPU oracle."""
    import torch
    import torch.distributed as dist
    from cuda.bindings import driver as cu
    from sparse_fp4_kv_b200 import binding as B
    from sparse_fp4_kv_b200.ranks import job_throughput, max_over_ranks, rank_recipe
    from sparse_fp4_kv_b200.stack import Csa2Decoder
    from sparse_fp4_kv_b200.workloads import RECIPES

    recipe = rank_recipe(RECIPES[name], rank, world)
    dec = Csa2Decoder(recipe, dev)
    costs = call_costs(recipe, dec.lens, dec.schedule)
    by = sum(c[2] for c in costs)
    fl = sum(c[3] for c in costs)
    calls = [(c[0], c[1]) for c in costs]

    # eager warm-up (first calls set kernel attributes), then the step graph
    with torch.cuda.stream(stream):
        dec.step(stream)
    stream.synchronize()
    if B.csa2_device_status(stream) != 0:
        raise RuntimeError(f"{name}: device error during warm-up")
    graph = torch.cuda.CUDAGraph(keep_graph=True)
    with torch.cuda.graph(graph, stream=stream):
        dec.step(stream)
    graph.instantiate()
    stream.synchronize()
    launches = graph_kernel_nodes(graph)

    for _ in range(args.warmup):
        graph_times_us(graph, stream, flush, 1)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    clocks.mark(0)
    per_step = graph_times_us(graph, stream, flush, args.steps)
    torch.cuda.synchronize(dev)
    clocks.mark(1)
    if world > 1:
        dist.barrier()
    clk = clocks.summary()
    if B.csa2_device_status(stream) != 0:
        raise RuntimeError(f"{name}: device error during the timed steps")
    total_ms = max_over_ranks(sum(per_step) * 1e-3, dev)
    value, ms = job_throughput(recipe.nq * recipe.layers, world, total_ms, args.steps)

    # per-call breakdown: external events around every call of a second graph
    def new_event():
        err, ev = cu.cuEventCreate(cu.CUevent_flags.CU_EVENT_DEFAULT)
        assert err == cu.CUresult.CUDA_SUCCESS
        return ev
    ev_pairs = [(new_event(), new_event()) for _ in calls]
    ext = cu.CUevent_record_flags.CU_EVENT_RECORD_EXTERNAL
    graph_ev = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph_ev, stream=stream):
        h = cu.CUstream(stream.cuda_stream)
        for (kind, l), (e0, e1) in zip(calls, ev_pairs):
            cu.cuEventRecordWithFlags(e0, h, ext)
            issue_call(dec, kind, l, stream)
            cu.cuEventRecordWithFlags(e1, h, ext)
    stream.synchronize()
    per_call = {}
    for _ in range(max(3, min(args.steps, 20))):
        graph_times_us(graph_ev, stream, flush, 1)
        for (kind, l), (a, b) in zip(calls, ev_pairs):
            err, t = cu.cuEventElapsedTime(a, b)
            per_call.setdefault(kind, []).append(t * 1e3)
    n_rep = max(3, min(args.steps, 20))
    calls_per_step = {k: sum(1 for c in calls if c[0] == k) for k in per_call}
    breakdown = {k: statistics.mean(v) for k, v in per_call.items()}
    share = {k: breakdown[k] * calls_per_step[k] for k in breakdown}
    for e0, e1 in ev_pairs:
        cu.cuEventDestroy(e0)
        cu.cuEventDestroy(e1)
    del graph_ev

    # roofline of the dominant call: that call alone in a graph, L2 flushed
    # before each replay, CUDA events around it
    peaks_tf = {"f16": pk["bf16_tflops"], "fp8": pk["fp8_tflops"]}
    dom = max(share, key=share.get)
    dom_call = next(c for c in costs if c[0] == dom)
    g1 = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g1, stream=stream):
        issue_call(dec, dom, dom_call[1], stream)
    stream.synchronize()
    t1 = graph_times_us(g1, stream, flush, max(args.steps, 10))
    del g1
    launch_us = statistics.median(t1)
    _, bound = call_roof_us(dom_call[2], dom_call[3], dom_call[4], pk["hbm_gbs"], peaks_tf)
    kernel_of = {"attention": f"k_attn_decode<{recipe.h}>", "full": "k_index_full", "reindex": "k_reindex",
                 "append": "k_append_fp4"}
    if bound == "hbm":
        achieved, peak, unit = dom_call[2] / (launch_us * 1e-6) / 1e9, pk["hbm_gbs"], "GB/s"
        peak_src = f"{pk['source']} HBM copy bandwidth (burst)"
    else:
        tc = dom_call[4]
        achieved, peak, unit = dom_call[3] / (launch_us * 1e-6) / 1e12, peaks_tf[tc], "TFLOP/s"
        peak_src = (f"{pk['source']} bf16 dense (burst; f16 runs at the bf16 rate)" if tc == "f16"
                    else "fp8 e4m3 dense measured by this bench's own tcgen05 kind::f8f6f4 loop")
    roofline = {"bound": bound, "kernel": kernel_of[dom], "call": dom, "achieved": achieved, "peak": peak,
                "unit": unit, "frac": achieved / peak, "peak_source": peak_src, "launch_us": launch_us,
                "launch_note": "median CUDA-event time of the call alone (its kernels) replayed from a graph, "
                               "L2 flushed before each replay",
                "bytes_per_launch": dom_call[2], "flops_per_launch": dom_call[3],
                "traffic": recorded_traffic(kernel_of[dom], name)}

    # the whole step against its roofline (sum over calls of their bound)
    t_roof = sum(call_roof_us(c[2], c[3], c[4], pk["hbm_gbs"], peaks_tf)[0] for c in costs)
    step_rl = {"t_roof_us": t_roof, "step_us": ms * 1e3, "frac": t_roof / (ms * 1e3),
               "peaks": f"{pk['source']}: {pk['hbm_gbs']} GB/s HBM, {pk['bf16_tflops']} TF/s bf16 burst, "
                        f"{pk['fp8_tflops']:.0f} TF/s fp8 (own tcgen05 loop)"}

    rec = {"value": value, "unit": UNIT, "ms_per_step": ms, "steps": args.steps, "warmup": args.warmup,
           "config": {"workload": name, "batch": recipe.batch, "queries_per_seq": recipe.q_per_seq,
                      "layers": recipe.layers, "modes": recipe.modes, "entries_max": int(dec.n_max),
                      "entries_total": int(dec.lens.sum()), "topk": recipe.k, "pool": recipe.p, "heads": recipe.h,
                      "window": recipe.w, "indexer": f"{recipe.hi}x{recipe.di}",
                      "l2": "before every timed step 256 MiB written, then another 256 MiB read (inputs and dirty lines out of L2)", "graph": "one CUDA graph per step"},
           "hbm_tbs": by / (ms * 1e-3) / 1e12, "algorithmic_bytes_per_step": by, "algorithmic_flops_per_step": fl,
           "roofline": roofline, "step_roofline": step_rl,
           "breakdown_us_per_call": breakdown, "calls_per_step": calls_per_step,
           "breakdown_note": "CUDA-event durations of each C-ABI call in a separately captured, instrumented "
                             f"replay of the same step ({n_rep} replays; event nodes between calls prevent "
                             "launch overlap)",
           "gpu_launches": (launches * args.steps) if launches is not None else None,
           "gpu_launches_per_step": launches, "clocks": clk}
    if not args.no_e2e:
        rec["e2e"] = run_e2e(args, dec, stream, flush, world=world, dev=dev)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rec["cpu_baseline"] = cpu_baseline(recipe)
    extra = {}
    if world == 1 and not args.no_side and name != "tiny_full":
        extra["attention_nvfp4"] = time_attn_variants(B, dec)
    del graph
    del dec
    torch.cuda.empty_cache()
    return rec, extra


def run_ours(args):
    import torch
    import torch.distributed as dist

    from sparse_fp4_kv_b200 import build
    build.build()
    from sparse_fp4_kv_b200 import binding as B  # noqa: F401  (fails loudly without the library)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    stream = torch.cuda.Stream(dev)
    flush = L2Flush(dev)

    pk = peaks()
    probe = measure_tc_probe(dev)
    pk["fp8_tflops"] = probe.get("fp8_e4m3_n256_tflops", 2.0 * pk["bf16_tflops"])
    names = list(WORKLOADS) if args.workload == "all" else [args.workload]
    headline = args.headline if args.headline in names else names[0]
    clocks = Clocks(dev)
    clocks.start()
    time.sleep(0.05)
    records, extra = {}, {}
    for name in names:
        rec, ex = bench_workload(name, args, world, rank, dev, stream, flush, clocks, pk)
        records[name] = rec
        for key, val in ex.items():
            extra.setdefault(key, {})[name] = val
    clocks.stop()

    side = world == 1 and not args.no_side
    hbm = pk["hbm_gbs"]
    if side:
        extra["append_chunk512"] = time_append_chunk512(B, dev, hbm)
        extra["append_e4m3"] = time_append_e4m3(B, dev, hbm)
        if not args.no_sharded:
            extra["sharded_hier1m"] = time_sharded_hier1m(dev)
    h = records[headline]
    line = {
        "metric": METRIC, "value": h["value"], "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": h["ms_per_step"], "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f16+e4m3 tensor-core, f32 accumulate", "data": "synthetic",
        "config": dict(h["config"], parallelism=f"dp{world} (independent sequences)"),
        "hbm_tbs": h["hbm_tbs"], "roofline": h["roofline"], "step_roofline": h["step_roofline"],
        "gpu_launches": h["gpu_launches"], "clocks": h["clocks"],
        "breakdown_us_per_call": h["breakdown_us_per_call"],
    }
    if "e2e" in h:
        line["e2e"] = h["e2e"]
    if "cpu_baseline" in h:
        line["cpu_baseline"] = h["cpu_baseline"]
    line["peaks"] = {"hbm_gbs": hbm, "bf16_tflops": pk["bf16_tflops"], "source": pk["source"],
                     "fp8_tflops": pk["fp8_tflops"], "tc_probe": probe}
    line["configs"] = records
    line.update(extra)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def run_e2e(args, dec, stream, flush, world, dev):
    """Same metric through the C-ABI with host buffers: every step copies its
    inputs (new latent rows, per-layer queries, indexer queries and weights)
    from pinned host memory to the device and reads every layer's output back.
    The step is one CUDA graph on three streams: the input copies run in layer
    order on one copy stream (per layer the indexer inputs, then q), layer l's
    indexer call waits only for its indexer inputs and its attention for q as
    well, and layer l's output is copied back on a second copy stream as soon as
    the layer is done, so the transfers overlap the compute of other layers."""
    import torch
    r = dec.r
    L = r.layers
    # each layer's indexer inputs (qidx, w) packed into one pinned host buffer
    # and one device buffer (256-byte aligned parts; the decoder's tensors
    # become views of it for the measurement), its q in another: the indexer
    # call waits only for the small pack, the attention for q as well
    saved = (list(dec.q), list(dec.qidx), list(dec.w))

    def pack(parts):
        offs, tot = [], 0
        for t in parts:
            offs.append(tot)
            tot += (t.numel() * t.element_size() + 255) // 256 * 256
        dbuf = torch.empty(tot, dtype=torch.uint8, device=dev)
        hbuf = torch.empty(tot, dtype=torch.uint8, pin_memory=True)
        views = []
        for t, o in zip(parts, offs):
            nb = t.numel() * t.element_size()
            hbuf[o:o + nb].copy_(t.contiguous().view(-1).cpu().view(torch.uint8))
            views.append(dbuf[o:o + nb].view(t.dtype).view(t.shape))
        return dbuf, hbuf, views

    packs, hosts = [], []  # per layer: [indexer pack, q pack]
    for l in range(L):
        di, hi, (dec.qidx[l], dec.w[l]) = pack([dec.qidx[l], dec.w[l]])
        dq, hq, (dec.q[l],) = pack([dec.q[l]])
        packs.append((di, dq))
        hosts.append((hi, hq))
    host_x = dec.x_new.cpu().pin_memory()
    host_out = [torch.empty(o.shape, dtype=o.dtype, pin_memory=True) for o in dec.o]
    h2d = host_x.numel() * host_x.element_size() + sum(hi.numel() + hq.numel() for hi, hq in hosts)
    d2h = sum(t.numel() * t.element_size() for t in host_out)
    s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    ev_x = torch.cuda.Event()
    ev_in = [torch.cuda.Event() for _ in range(L)]
    ev_q = [torch.cuda.Event() for _ in range(L)]
    ev_done = [torch.cuda.Event() for _ in range(L)]
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        s_in.wait_stream(stream)
        s_out.wait_stream(stream)
        with torch.cuda.stream(s_in):
            dec.x_new.copy_(host_x, non_blocking=True)
            ev_x.record(s_in)
            for l in range(L):
                packs[l][0].copy_(hosts[l][0], non_blocking=True)
                ev_in[l].record(s_in)
                packs[l][1].copy_(hosts[l][1], non_blocking=True)
                ev_q[l].record(s_in)
        stream.wait_event(ev_x)
        dec.append(stream)
        for l in range(L):
            stream.wait_event(ev_in[l])
            dec.layer(l, stream, before_attention=lambda l=l: stream.wait_event(ev_q[l]))
            ev_done[l].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_done[l])
                host_out[l].copy_(dec.o[l], non_blocking=True)
        stream.wait_stream(s_in)
        stream.wait_stream(s_out)
    stream.synchronize()
    times = []
    for i in range(args.warmup + args.steps):
        st, en = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            flush.fill_(i & 0xFF)
            st.record(stream)
            g.replay()
            en.record(stream)
        en.synchronize()
        if i >= args.warmup:
            times.append(st.elapsed_time(en))
    total = sum(times)
    if world > 1:
        import torch.distributed as dist
        t = torch.tensor([total], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        total = float(t.item())
    ms = total / len(times)
    # the copied-back outputs are the device outputs of the last replay
    torch.cuda.synchronize(dev)
    for h_t, o in zip(host_out, dec.o):
        if not torch.equal(h_t, o.cpu()):
            raise RuntimeError("e2e: host output differs from the device output")
    del g
    dec.q, dec.qidx, dec.w = saved
    return {"value": r.nq * r.layers * world / (ms * 1e-3), "unit": UNIT, "ms_per_step": ms,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "note": "one CUDA graph per step: each layer's inputs copied in layer order on a copy stream as two "
                    "copies (qidx and w packed, then q), the layer's indexer call waits for the first, its "
                    "attention for q as well, each layer's output copied back as soon as it is done"}


def main():
    import faulthandler
    faulthandler.enable()  # a crash in native code prints the Python stack
    args = parse()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
