"""Benchmark of the CSA2 decode hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload stack20]
    python bench.py --impl reference ...      # the CPU oracle, same metric

A step is one decode step of the workload through the C-ABI: FP4 append of
the new token of every sequence, then every layer of the static mode schedule
(Full / Reindex indexer where scheduled, Reuse otherwise) followed by sparse +
window attention. Default workload: the 20-layer decoder stack, 8 sequences
x 1 query, 65536 FP4 entries each (Full at 0 and 10, Reindex at 5 and 15,
Reuse elsewhere, Top-K 2048, 64 heads, window 512).

Metric: decode query-steps per second per layer = batch * queries * layers /
step time, with the achieved HBM bandwidth of the step's algorithmic bytes.
Timing: the step is captured once in a CUDA graph; each of the K timed steps
is preceded by a 256 MiB L2 flush and bracketed by CUDA events on the
launching stream; a barrier and a device synchronize bracket the whole timed
loop; the reported time is the max over ranks. Multi-GPU runs give every rank
its own independent batch of sequences (weak scaling, no collective on the
data path).
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


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="stack20")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-sharded", action="store_true", help="skip the entry-range sharded side measurement")
    ap.add_argument("--no-side", action="store_true",
                    help="skip every side measurement (appends, sharded decode, attention variants)")
    return ap.parse_args()


# ---------------------------------------------------------------------------
# algorithmic work (what the method must move / compute)
# ---------------------------------------------------------------------------
def algorithmic(recipe, lens, schedule):
    """(bytes, flops) of one step, and (bytes, flops) of one attention launch."""
    nq, h, d = recipe.nq, recipe.h, 512
    n_vis = [int(l) for l in lens.tolist()]
    by = fl = 0.0
    rows_app = recipe.append if recipe.chunked else recipe.batch
    by += rows_app * (d * 2 + d // 2 + d // 16)
    attn_by = attn_fl = 0.0
    for mode, src in schedule:
        if mode == "full":
            for qi in range(nq):
                n = n_vis[qi // recipe.q_per_seq]
                by += n * recipe.di
                fl += 2.0 * recipe.hi * recipe.di * n
        elif mode == "reindex":
            by += nq * recipe.p * (recipe.di + 4)
            fl += 2.0 * nq * recipe.hi * recipe.di * recipe.p
        rows = recipe.k + recipe.w
        a_by = nq * (recipe.k * (d // 2 + d // 16 + 4) + recipe.w * d + 2 * 2 * h * d)
        a_fl = 4.0 * nq * h * rows * d
        by += a_by
        fl += a_fl
        attn_by, attn_fl = a_by, a_fl
    return by, fl, attn_by, attn_fl


def step_roofline_us(recipe, lens, schedule, hbm_gbs, tc_tflops):
    """t_roof of one step in microseconds: the sum over the step's kernels of
    max(algorithmic bytes / HBM peak, flops / tensor peak); the indexer's
    FP8 products are counted at twice the bf16 peak."""
    nq, h, d = recipe.nq, recipe.h, 512
    n_vis = [int(l) for l in lens.tolist()]
    bw, tc = hbm_gbs * 1e9, tc_tflops * 1e12
    rows_app = recipe.append if recipe.chunked else recipe.batch
    t = rows_app * (d * 2 + d // 2 + d // 16) / bw
    parts = {"append": t}
    for mode, src in schedule:
        if mode == "full":
            b = f = 0.0
            for qi in range(nq):
                n = n_vis[qi // recipe.q_per_seq]
                b += n * recipe.di
                f += 2.0 * recipe.hi * recipe.di * n
            parts["full"] = parts.get("full", 0.0) + max(b / bw, f / (2 * tc))
        elif mode == "reindex":
            b = nq * recipe.p * (recipe.di + 4)
            f = 2.0 * nq * recipe.hi * recipe.di * recipe.p
            parts["reindex"] = parts.get("reindex", 0.0) + max(b / bw, f / (2 * tc))
        a_by = nq * (recipe.k * (d // 2 + d // 16 + 4) + recipe.w * d + 2 * 2 * h * d)
        a_fl = 4.0 * nq * h * (recipe.k + recipe.w) * d
        parts["attention"] = parts.get("attention", 0.0) + max(a_by / bw, a_fl / tc)
    return sum(parts.values()) * 1e6, {k: v * 1e6 for k, v in parts.items()}


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
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    for _ in range(3):
        B.csa2_append_fp4(x, seq, pos, kv)
    ts = []
    for i in range(reps):
        flush.fill_(i & 0xFF)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        B.csa2_append_fp4(x, seq, pos, kv)
        e1.record()
        e1.synchronize()
        ts.append(e0.elapsed_time(e1) * 1e3)
    ts.sort()
    us = ts[len(ts) // 2]
    by = n * (512 * 2 + 256 + 32)
    return {"rows": n, "us_median": us, "algorithmic_bytes": by, "achieved_gbs": by / (us * 1e-6) / 1e9,
            "peak_gbs": hbm_gbs, "frac": by / (us * 1e-6) / 1e9 / hbm_gbs,
            "note": "bf16 rows in, FP4 codes + E4M3 scales out, 256K-entry cache; CUDA events around the call "
                    "(launch included), median of %d after an L2 flush" % reps}


def time_append_e4m3(B, dev, hbm_gbs, reps=20):
    """The FP8 appends at chunked-prefill size: 32,768 window rows (512 values)
    into a ring of 32,768 slots, and 32,768 indexer keys (64 values) into a
    256K-entry key array; CUDA events around each call, L2 flushed before each."""
    import torch
    from sparse_fp4_kv_b200 import synth
    n, ring, cap, di = 32768, 32768, 262144, 64
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
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
    out = {}
    for name, call, by in (("window", lambda: B.csa2_append_swa_e4m3(xw, seq, pos, swa), n * 512 * 3),
                           ("keys", lambda: B.csa2_append_kidx_e4m3(xk, seq, pos, kv), n * di * 3)):
        for _ in range(3):
            call()
        ts = []
        for i in range(reps):
            flush.fill_(i & 0xFF)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            call()
            e1.record()
            e1.synchronize()
            ts.append(e0.elapsed_time(e1) * 1e3)
        ts.sort()
        us = ts[len(ts) // 2]
        out[name] = {"rows": n, "us_median": us, "algorithmic_bytes": by,
                     "achieved_gbs": by / (us * 1e-6) / 1e9, "frac": by / (us * 1e-6) / 1e9 / hbm_gbs}
    out["note"] = "bf16 in, E4M3 out; events around the call (launch included), median of %d after an L2 flush" % reps
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
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
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
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
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


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        return j.get("hbm_gbs", 6650.0), j.get("bf16_tflops", 1590.0), j.get("bf16_tflops_sustained", 1400.0), \
            "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


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
    """nvidia-smi samples every 50 ms; only the samples taken between mark()
    calls (the timed region) are summarised."""
    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.window = [None, None]

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def mark(self, which):
        self.window[which] = datetime.datetime.now()

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        out, _ = self.proc.communicate(timeout=10)
        rows = []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 10:
                continue
            try:
                ts = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f")
                rows.append((ts, float(parts[2]), float(parts[3]),
                             [n for n, v in zip(names, parts[6:10]) if v.lower() == "active"]))
            except ValueError:
                continue
        t0, t1 = self.window
        inside = [r for r in rows if t0 is not None and t1 is not None and t0 <= r[0] <= t1]
        use = inside if inside else rows
        reasons = sorted({n for r in use for n in r[3]})
        return {"sm_mhz": statistics.median(r[1] for r in use) if use else None,
                "sm_max_mhz": max(r[2] for r in use) if use else None, "reasons": reasons,
                "samples": len(use), "samples_in_timed_region": len(inside),
                "power_w_note": "50 ms nvidia-smi sampling"}


# ---------------------------------------------------------------------------
# CPU oracle (cpu_baseline leg and --impl reference)
# ---------------------------------------------------------------------------
def oracle_sample(recipe, layers, seq=0):
    """Time the oracle's step for one sequence over `layers` (cache build and
    input generation excluded). Returns (seconds, query-layers processed)."""
    import numpy as np
    import torch
    import oracle
    import oracle.stack as ostack
    sched = ostack.schedule(recipe.modes)
    cache = ostack.SeqCache(recipe, seq)
    qis = [seq * recipe.q_per_seq + j for j in range(recipe.q_per_seq)]
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


def reference_layers(recipe):
    """Layers of the bounded oracle sample: from layer 0 up to the first
    Reindex layer (so every mode is exercised), capped at 6."""
    modes = recipe.modes
    end = modes.find("R")
    end = len(modes) if end < 0 else end + 1
    return list(range(min(end, 6)))


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
    recipe, seq, layers = job
    return oracle_sample(recipe, layers, seq)


def oracle_all_cores(recipe, layers):
    """The oracle on independent sequences at once, one process each (spawned,
    no GPU), up to one per core: units of all processes over the longest
    process's compute time."""
    import multiprocessing as mp
    procs = max(1, min(os.cpu_count() or 1, recipe.batch))
    with mp.get_context("spawn").Pool(procs) as pool:
        res = pool.map(_oracle_worker, [(recipe, s, layers) for s in range(procs)])
    dt = max(r[0] for r in res)
    n = sum(r[1] for r in res)
    return {"value": n / dt, "unit": UNIT, "cores": procs,
            "sample": f"sequences 0..{procs - 1}, layers {layers[0]}..{layers[-1]}, one process per sequence "
                      f"({dt:.1f} s)"}


def run_reference(args):
    from sparse_fp4_kv_b200.workloads import RECIPES
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    recipe = RECIPES[args.workload]
    layers = reference_layers(recipe)
    times = []
    n_units = 0
    for i in range(args.warmup + args.steps):
        dt, n_units = oracle_sample(recipe, layers)
        if i >= args.warmup:
            times.append(dt)
    total = sum(times)
    value = n_units * len(times) / total
    sample = (f"sequence 0 of {recipe.name}, layers {layers[0]}..{layers[-1]} "
              f"({''.join(recipe.modes[l] for l in layers)}), {recipe.q_per_seq} quer"
              f"{'y' if recipe.q_per_seq == 1 else 'ies'}, single-threaded C oracle")
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
def run_ours(args):
    import torch
    import torch.distributed as dist
    from cuda.bindings import driver as cu

    from sparse_fp4_kv_b200 import build
    build.build()
    from sparse_fp4_kv_b200 import binding as B
    from sparse_fp4_kv_b200.stack import Csa2Decoder
    from sparse_fp4_kv_b200.workloads import RECIPES

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)

    from sparse_fp4_kv_b200.ranks import job_throughput, max_over_ranks, rank_recipe
    base = RECIPES[args.workload]
    recipe = rank_recipe(base, rank, world)
    dec = Csa2Decoder(recipe, dev)
    by, fl, attn_by, attn_fl = algorithmic(recipe, dec.lens, dec.schedule)

    stream = torch.cuda.Stream(dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    # external timing events around every attention launch inside the graph
    def new_event():
        err, ev = cu.cuEventCreate(cu.CUevent_flags.CU_EVENT_DEFAULT)
        assert err == cu.CUresult.CUDA_SUCCESS
        return ev

    # external timing events around every C-ABI call inside the graph: the
    # attention call of every layer (the roofline kernel) and the others
    # for the per-call breakdown
    calls = [("append", None)]
    for l, (mode, _) in enumerate(dec.schedule):
        if mode in ("full", "reindex"):
            calls.append((mode, l))
        calls.append(("attention", l))
    ev_pairs = [(new_event(), new_event()) for _ in calls]
    ext = cu.CUevent_record_flags.CU_EVENT_RECORD_EXTERNAL

    def step_with_events(s):
        h = cu.CUstream(s.cuda_stream)
        r = dec.r
        for (kind, l), (e0, e1) in zip(calls, ev_pairs):
            cu.cuEventRecordWithFlags(e0, h, ext)
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
                B.csa2_sparse_attn_decode(dec.q[l], r.q_per_seq, dec.kv, dec.topk_of(l), dec.swa[l],
                                          dec.swa[l].shape[1], dec.swa_begin, dec.swa_end, r.w, dec.scale, dec.o[l],
                                          dec.lse[l], dec.ws_attn, s)
            cu.cuEventRecordWithFlags(e1, h, ext)

    # eager warm-up (first calls set kernel attributes), then capture two
    # graphs of the step: the plain one that is timed, and one with external
    # timing events around every call (event nodes sit between the kernels
    # and stop programmatic launch overlap, so it only feeds the per-call
    # breakdown and the roofline kernel's duration)
    with torch.cuda.stream(stream):
        step_with_events(stream)
    stream.synchronize()
    if B.csa2_device_status(stream) != 0:
        raise RuntimeError("device error during warm-up")
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        dec.step(stream)
    stream.synchronize()
    graph_ev = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph_ev, stream=stream):
        step_with_events(stream)
    stream.synchronize()

    def timed_steps(g, n, record):
        st = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
        en = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
        per_step, attn = [], {}
        for i in range(n):
            with torch.cuda.stream(stream):
                flush.fill_(i & 0xFF)
                st[i].record(stream)
                g.replay()
                en[i].record(stream)
            en[i].synchronize()
            per_step.append(st[i].elapsed_time(en[i]))
            if record:
                for (kind, _), (a, b) in zip(calls, ev_pairs):
                    err, ms = cu.cuEventElapsedTime(a, b)
                    attn.setdefault(kind, []).append(ms)
        return per_step, attn

    launches_per_step = count_launches(dec, recipe)
    for _ in range(args.warmup):
        timed_steps(graph, 1, False)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    clocks = Clocks(local)
    clocks.start()
    time.sleep(0.2)  # the sampler is running
    clocks.mark(0)
    per_step, _ = timed_steps(graph, args.steps, False)
    torch.cuda.synchronize(dev)
    clocks.mark(1)
    if world > 1:
        dist.barrier()
    clk = clocks.stop()
    # instrumented replays right after the timed loop: per-call durations
    _, attn = timed_steps(graph_ev, args.steps, True)
    if B.csa2_device_status(stream) != 0:
        raise RuntimeError("device error during the timed steps")
    total_ms = max_over_ranks(sum(per_step), dev)
    value, ms = job_throughput(recipe.nq * recipe.layers, world, total_ms, args.steps)

    # e2e: host buffers in pinned memory, copies inside the timed region
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(args, dec, stream, flush, world=world, dev=dev)

    hbm_gbs, bf16_burst, bf16_sust, peak_kind = peaks()
    t_roof, t_parts = step_roofline_us(recipe, dec.lens, dec.schedule, hbm_gbs, bf16_sust)
    step_rl = {"t_roof_us": t_roof, "parts_us": t_parts, "step_us": ms * 1e3, "frac": t_roof / (ms * 1e3),
               "peaks": f"{peak_kind}: {hbm_gbs} GB/s HBM, {bf16_sust} TF/s bf16 sustained (FP8 at 2x)"}
    side = world == 1 and not args.no_side
    append_c4 = time_append_chunk512(B, dev, hbm_gbs) if side else None
    append_f8 = time_append_e4m3(B, dev, hbm_gbs) if side else None
    sharded = time_sharded_hier1m(dev) if side and not args.no_sharded else None
    attn_nv = time_attn_variants(B, dec) if side and recipe.h == 64 else None
    breakdown = {k: 1e3 * statistics.mean(v) for k, v in attn.items()}
    attn_ms = statistics.mean(attn["attention"]) if attn else float("nan")
    achieved_tf = attn_fl / (attn_ms * 1e-3) / 1e12
    kernel = f"k_sparse_attn<{recipe.h}>"
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f16+e4m3 tensor-core, f32 accumulate", "data": "synthetic",
        "config": {"workload": recipe.name, "batch": recipe.batch, "queries_per_seq": recipe.q_per_seq,
                   "layers": recipe.layers, "modes": recipe.modes, "entries": int(dec.n_max),
                   "topk": recipe.k, "pool": recipe.p, "heads": recipe.h, "window": recipe.w,
                   "indexer": f"{recipe.hi}x{recipe.di}", "l2": "256 MiB flush before every timed step",
                   "graph": "one CUDA graph per step", "parallelism": f"dp{world} (independent sequences)"},
        "hbm_tbs": by / (ms * 1e-3) / 1e12,
        "algorithmic_bytes_per_step": by, "algorithmic_flops_per_step": fl,
        "roofline": {"bound": "tensor", "kernel": kernel, "achieved": achieved_tf, "peak": bf16_sust,
                     "unit": "TFLOP/s", "frac": achieved_tf / bf16_sust,
                     "peak_source": f"{peak_kind} bf16 dense sustained (f16 runs at the bf16 rate)",
                     "launch_us": attn_ms * 1e3, "launch_note": "event-timed attention call (attention kernel + "
                     "split combine) in the instrumented replay", "flops_per_launch": attn_fl, "bytes_per_launch": attn_by,
                     "hbm_frac": attn_by / (attn_ms * 1e-3) / (hbm_gbs * 1e9),
                     "traffic": recorded_traffic(kernel, recipe.name)},
        "step_roofline": step_rl,
        "append_chunk512": append_c4,
        "append_e4m3": append_f8,
        "sharded_hier1m": sharded,
        "attention_nvfp4": attn_nv,
        "breakdown_us_per_call": breakdown,
        "breakdown_note": "CUDA-event durations of each C-ABI call in a separately captured, instrumented replay "
                          "of the same step (event nodes between calls prevent launch overlap)",
        "breakdown_calls_per_step": {k: len(v) // args.steps for k, v in attn.items()},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clk,
    }
    if e2e is not None:
        line["e2e"] = e2e
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        layers = list(range(recipe.layers))
        dt, n = oracle_sample(recipe, layers)
        line["cpu_baseline"] = {
            "value": n / dt, "unit": UNIT, "cores": 1, "kind": "oracle",
            "sample": f"sequence 0, layers {layers[0]}..{layers[-1]} of {recipe.name}, single-threaded C oracle "
                      f"({dt:.1f} s)", "cpu_model": cpu_model(), "nproc": os.cpu_count(),
            "all_cores": oracle_all_cores(recipe, layers)}
    if rank == 0:
        print(json.dumps(line), flush=True)
    del graph, graph_ev
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def count_launches(dec, recipe):
    """Kernels of this library launched by one step (the memset of the Full
    layer's histograms is a runtime call, not counted)."""
    from sparse_fp4_kv_b200 import binding as B
    n = 1  # append
    for mode, _ in dec.schedule:
        if mode == "full":
            n += 5
        elif mode == "reindex":
            n += 2
        n += 1 + (1 if B.csa2_sparse_attn_workspace_size(recipe.nq, recipe.h, recipe.k, recipe.w) > 0 else 0)
    return n


def run_e2e(args, dec, stream, flush, world, dev):
    """Same metric through the C-ABI with host buffers: every step copies its
    inputs (new latent rows, per-layer queries, indexer queries and weights)
    from pinned host memory to the device and reads every layer's output back.
    The step is one CUDA graph on three streams: the input copies run in layer
    order on one copy stream, layer l waits only for its own inputs, and layer
    l's output is copied back on a second copy stream as soon as the layer is
    done, so the transfers overlap the compute of other layers."""
    import torch
    r = dec.r
    L = r.layers
    # each layer's inputs (q, qidx, w) packed into one pinned host buffer and
    # one device buffer (256-byte aligned parts; the decoder's tensors become
    # views of it for the measurement), so a layer takes one copy
    saved = (list(dec.q), list(dec.qidx), list(dec.w))
    packs, hosts = [], []
    for l in range(L):
        parts = [dec.q[l], dec.qidx[l], dec.w[l]]
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
        dec.q[l], dec.qidx[l], dec.w[l] = views
        packs.append(dbuf)
        hosts.append(hbuf)
    host_x = dec.x_new.cpu().pin_memory()
    host_out = [torch.empty(o.shape, dtype=o.dtype, pin_memory=True) for o in dec.o]
    h2d = host_x.numel() * host_x.element_size() + sum(h.numel() for h in hosts)
    d2h = sum(t.numel() * t.element_size() for t in host_out)
    s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    ev_x = torch.cuda.Event()
    ev_in = [torch.cuda.Event() for _ in range(L)]
    ev_done = [torch.cuda.Event() for _ in range(L)]
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        s_in.wait_stream(stream)
        s_out.wait_stream(stream)
        with torch.cuda.stream(s_in):
            dec.x_new.copy_(host_x, non_blocking=True)
            ev_x.record(s_in)
            for l in range(L):
                packs[l].copy_(hosts[l], non_blocking=True)
                ev_in[l].record(s_in)
        stream.wait_event(ev_x)
        dec.append(stream)
        for l in range(L):
            stream.wait_event(ev_in[l])
            dec.layer(l, stream)
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
            "note": "one CUDA graph per step: each layer's inputs (q, qidx, w packed, one copy) copied in layer "
                    "order on a copy stream, each layer waits for its own inputs, each layer's output copied back "
                    "as soon as it is done"}


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
