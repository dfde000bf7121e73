"""Host-side arithmetic of the benchmark, on the CPU: the algorithmic bytes
and flops of every call of a decode step (the numerators of every roofline
fraction the benchmark prints), the choice of the bound, and the source hash
that decides whether a recorded ncu traffic figure still belongs to the
kernels. The expected values are written out from the data layout: an FP4
entry is 512 / 2 code bytes + 512 / 16 E4M3 scale bytes, a window row 512
E4M3 bytes, a selected id 4 bytes, q and o bf16 rows of 512 values, an
indexer key di E4M3 bytes, and a Full call reads each sequence's keys once
however many of its queries score them."""
import shutil

import pytest

import bench
from sparse_fp4_kv_b200.workloads import RECIPES, resolve_schedule

D = 512
FP4_ENTRY = D // 2 + D // 16  # 288 bytes: codes + scales
ROW_IN = D * 2                # one bf16 latent row


def _costs(name):
    r = RECIPES[name]
    return r, bench.call_costs(r, r.seq_lens(), resolve_schedule(r.modes))


def test_paged64_step_costs():
    r, costs = _costs("paged64")
    lens = [int(x) for x in r.seq_lens().tolist()]
    assert [c[0] for c in costs] == ["append", "full", "attention", "attention", "attention", "attention"]
    # the step appends one row per sequence
    assert costs[0][2] == 64 * (ROW_IN + FP4_ENTRY)
    # Full: each sequence's keys once, per query its Top-K ids out (no pool),
    # its 4 indexer heads' q (64 E4M3 bytes) and weight (4 bytes) in
    _, _, by, fl, tc = costs[1]
    assert tc == "fp8"
    assert by == 64 * (4 * 2048 + 4 * (64 + 4)) + 64 * sum(lens)
    assert fl == sum(2.0 * 4 * 64 * n for n in lens)
    # attention, every layer: 2048 selected entries (288 B + a 4-byte id),
    # 512 window rows, q in and o out, 32 heads
    for kind, _, by, fl, tc in costs[2:]:
        assert by == 64 * (2048 * (FP4_ENTRY + 4) + 512 * D + 2 * 32 * ROW_IN) == 59244544
        assert fl == 2 * 2 * 64 * 32 * (2048 + 512) * D == 10737418240
        assert tc == "f16"


def test_stack20_full_and_reindex_costs():
    r, costs = _costs("stack20")
    kinds = [c[0] for c in costs]
    assert kinds.count("full") == 2 and kinds.count("reindex") == 2 and kinds.count("attention") == 20
    full = [c for c in costs if c[0] == "full"]
    for _, layer, by, fl, _ in full:
        assert layer in (0, 10)
        # Top-K and pool ids out, 8 sequences of 65536 keys of 64 bytes
        assert by == 8 * (4 * (2048 + 4096) + 4 * (64 + 4)) + 8 * 65536 * 64
        assert fl == 8 * 2.0 * 4 * 64 * 65536
    for _, layer, by, fl, _ in (c for c in costs if c[0] == "reindex"):
        assert layer in (5, 15)
        # each pool id read with its key, Top-K ids out
        assert by == 8 * 4096 * (64 + 4) + 8 * 2048 * 4
        assert fl == 2.0 * 8 * 4 * 64 * 4096
    att = [c for c in costs if c[0] == "attention"]
    assert all(c[2] == 8 * (2048 * (FP4_ENTRY + 4) + 512 * D + 2 * 64 * ROW_IN) for c in att)


def test_chunk512_counts_the_shared_keys_once():
    r, costs = _costs("chunk512")
    assert costs[0][0] == "append" and costs[0][2] == 32768 * (ROW_IN + FP4_ENTRY) == 42991616
    _, _, by, fl, _ = costs[1]
    # 512 causal queries at positions 261632 .. 262143 see 261633 .. 262144
    # entries; the one sequence's 262144 keys are read once
    assert by == 512 * (4 * 2048 + 4 * (64 + 4)) + 262144 * 64
    seen = 512 * 261633 + 511 * 512 // 2
    assert fl == 2.0 * 4 * 64 * seen == 68652498944
    _, _, by, fl, _ = costs[2]
    assert by == 512 * (2048 * (FP4_ENTRY + 4) + 256 * D + 2 * 32 * ROW_IN)
    assert fl == 4.0 * 512 * 32 * (2048 + 256) * D


def test_roof_takes_the_slower_bound():
    peaks = {"f16": 1000.0, "fp8": 2000.0}
    # 6.65 MB at 6650 GB/s is 1 us; 1e10 f16 flops at 1000 TF/s is 10 us
    t, bound = bench.call_roof_us(6.65e6, 1e10, "f16", 6650.0, peaks)
    assert bound == "tensor" and t == pytest.approx(10.0)
    t, bound = bench.call_roof_us(6.65e7, 1e10, "fp8", 6650.0, peaks)
    assert bound == "hbm" and t == pytest.approx(10.0)
    t, bound = bench.call_roof_us(6.65e6, 0.0, None, 6650.0, peaks)
    assert bound == "hbm" and t == pytest.approx(1.0)


def test_source_hash_ignores_comments_only(tmp_path):
    src = tmp_path / "csrc"
    shutil.copytree(bench.os.path.join(bench.ROOT, "sparse_fp4_kv_b200", "csrc"), src)
    h0 = bench.kernel_source_hash(str(src))
    assert h0 == bench.kernel_source_hash()
    f = src / "append.cuh"
    text = f.read_text()
    f.write_text("// a comment line\n" + text.replace("namespace csa2 {", "namespace csa2 { /* inline */", 1) + "\n\n")
    assert bench.kernel_source_hash(str(src)) == h0
    f.write_text(text.replace("constexpr int kAppendRing = 4;", "constexpr int kAppendRing = 5;", 1))
    assert bench.kernel_source_hash(str(src)) != h0
    # a string literal keeps its comment-like contents
    assert bench.code_of('x = "a // b"; // gone') == 'x = "a // b";'
