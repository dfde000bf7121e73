"""Sparse + window attention kernel against the oracle (f64): outputs within
2e-3 max-abs (bf16 out), log-sum-exp within 1e-3. Covers 16/32/64 heads,
ragged tile counts, -1 ids, empty windows, paged caches, single-split and
split-and-combine launches, and the degenerate empty set."""
import math

import numpy as np
import pytest
import torch

import oracle
from helpers import attn_excess, bf16_bits, device_status_clean, kv_from_numpy, paged_layout
from sparse_fp4_kv_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def B():
    from sparse_fp4_kv_b200 import build
    build.build()
    from sparse_fp4_kv_b200 import binding
    return binding


def _cache(rng, lens, ps, seed):
    pt, cap = paged_layout(rng, lens, ps)
    x = synth.normal_bf16(seed, 1, 0, cap * 512).view(cap, 512)
    codes, scales = oracle.quantize_rows(bf16_bits(x))
    return pt, cap, codes, scales


def _run(B, dev, lens, ps, h, k, w, q_per_seq=1, seed=0, neg_frac=0.05, swa_rows=None, uniform=False):
    rng = np.random.default_rng(seed)
    pt, cap, codes, scales = _cache(rng, lens, ps, seed)
    if uniform:
        codes[:] = codes[0]
        scales[:] = scales[0]
    nb = len(lens)
    nq = nb * q_per_seq
    topk = np.full((nq, k), -1, np.int32)
    for qi in range(nq):
        n = lens[qi // q_per_seq]
        m = min(k, n)
        ids = rng.permutation(n)[:m].astype(np.int32)
        ids[rng.random(m) < neg_frac] = -1
        topk[qi, :m] = ids
        topk[qi] = rng.permutation(topk[qi])
    swa_rows = swa_rows or max(w, 1)
    swa = synth.normal_e4m3(seed, 4, 0, nb * swa_rows * 512).view(nb, swa_rows, 512).numpy()
    if uniform:
        swa[:] = 0
    begin = rng.integers(0, swa_rows - w + 1, nq).astype(np.int32)
    end = (begin + w).astype(np.int32)
    q = synth.normal_bf16(seed, 3, 0, nq * h * 512).view(nq, h, 512)
    scale = 1.0 / math.sqrt(512)
    kv = kv_from_numpy(codes, scales, None, pt, lens, ps, dev)
    o = torch.full((nq, h, 512), float("nan"), dtype=torch.bfloat16, device=dev)
    lse = torch.full((nq, h), float("nan"), dtype=torch.float32, device=dev)
    ws = B.workspace(B.csa2_sparse_attn_workspace_size(nq, h, k, w), dev)
    d = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dev)
    B.csa2_sparse_attn_decode(q.to(dev), q_per_seq, kv, d(topk) if k > 0 else None, d(swa), swa_rows, d(begin),
                              d(end), w, scale, o, lse, ws)
    torch.cuda.synchronize()
    assert device_status_clean()
    go = o.float().cpu().numpy()
    gl = lse.cpu().numpy()
    worst = 0.0
    for qi in range(nq):
        b = qi // q_per_seq
        oo, ol = oracle.sparse_attn(bf16_bits(q[qi]), codes, scales, pt[b], ps, topk[qi],
                                    swa[b][begin[qi]:end[qi]] if w > 0 else None, scale)
        err = np.abs(go[qi] - oo).max()
        worst = max(worst, err)
        assert attn_excess(go[qi], oo) <= 1.0, f"q{qi}: max |o - oracle| = {err}"
        fin = np.isfinite(ol)
        assert np.all(np.isfinite(gl[qi]) == fin)
        np.testing.assert_allclose(gl[qi][fin], ol[fin], atol=1e-3, rtol=0)
    return go, gl, worst


@pytest.mark.parametrize("h", [16, 32, 64])
def test_heads_ragged_tiles(B, cuda_device, h):
    _run(B, cuda_device, [900, 1500], 64, h, 300, 77, seed=h)


def test_single_query_many_tiles_split(B, cuda_device):
    # one query, 20 tiles -> split across CTAs and merged
    _run(B, cuda_device, [70000], 128, 64, 2048, 512, seed=1)


@pytest.mark.parametrize("per", ["1", "3", "7", "12", "20", "40", "auto"])
def test_several_queries_split_ragged(B, cuda_device, monkeypatch, per):
    # several queries with ragged row counts, 32 and 16 heads, the tiles per
    # CTA fixed or chosen by the plan: 1, 3: every query split over several
    # CTAs; 7: CTAs that end one query and start the next (partial first and
    # last segments); 12: one whole query per CTA; 20, 40: CTAs holding whole
    # queries and parts of others, or every query (no merge)
    if per != "auto":
        monkeypatch.setenv("CSA2_ATTN_PER", per)
    _run(B, cuda_device, [9000, 5000, 3000], 64, 32, 1300, 200, seed=21)
    _run(B, cuda_device, [9000, 7000], 64, 16, 1800, 300, seed=22)
    _run(B, cuda_device, [4000, 4000, 4000, 4000], 64, 64, 1000, 120, seed=23)


def test_many_queries_single_split(B, cuda_device):
    # enough queries that each one runs in a single CTA
    _run(B, cuda_device, [600] * 4, 64, 32, 256, 33, q_per_seq=80, seed=2, swa_rows=160)


def test_no_window_and_window_only(B, cuda_device):
    _run(B, cuda_device, [500], 64, 64, 200, 0, seed=3)
    _run(B, cuda_device, [500], 64, 64, 0, 130, seed=4)


def test_empty_set_gives_zero(B, cuda_device):
    go, gl, _ = _run(B, cuda_device, [300], 64, 16, 64, 0, seed=5, neg_frac=1.0)
    assert np.all(go == 0) and np.all(np.isneginf(gl))


def test_identical_rows_return_that_row(B, cuda_device):
    go, _, _ = _run(B, cuda_device, [400], 64, 32, 256, 0, seed=6, uniform=True, neg_frac=0.0)
    v = go[0]
    assert np.allclose(v, v[0:1], atol=0)


def test_running_max_raised_in_later_tiles(B, cuda_device):
    # order each query's ids by ascending score so that every later tile
    # raises the per-head maximum by more than 2^8 (the O rescale path)
    rng = np.random.default_rng(21)
    lens, ps, h, k = [3000], 64, 64, 640
    pt, cap, codes, scales = _cache(rng, lens, ps, 21)
    q = synth.normal_bf16(21, 3, 0, h * 512).view(1, h, 512) * 4.0
    q = q.to(torch.bfloat16)
    ids = rng.permutation(lens[0])[:k].astype(np.int32)
    rows = [pt[0][t // ps] * ps + t % ps for t in ids]
    V = np.stack([oracle.dequant_row(codes[r], scales[r]) for r in rows])
    z = (q[0].double().numpy() @ V.T).max(axis=0)
    topk = ids[np.argsort(z)][None, :]
    kv = kv_from_numpy(codes, scales, None, pt, lens, ps, cuda_device)
    o = torch.empty((1, h, 512), dtype=torch.bfloat16, device=cuda_device)
    lse = torch.empty((1, h), dtype=torch.float32, device=cuda_device)
    ws = B.workspace(B.csa2_sparse_attn_workspace_size(1, h, k, 0), cuda_device)
    scale = 1.0 / math.sqrt(512)
    B.csa2_sparse_attn_decode(q.to(cuda_device), 1, kv, torch.from_numpy(topk).to(cuda_device), None, 0, None, None,
                              0, scale, o, lse, ws)
    torch.cuda.synchronize()
    assert device_status_clean()
    oo, ol = oracle.sparse_attn(bf16_bits(q[0]), codes, scales, pt[0], ps, topk[0], None, scale)
    s2 = (q[0].double().numpy() @ V[np.argsort(z)].T) * scale / math.log(2)
    tmax = [s2[:, t * 128:(t + 1) * 128].max(axis=1) for t in range(k // 128)]
    assert np.any(tmax[-1] > tmax[0] + 8), "case does not reach the rescale path"
    assert attn_excess(o.float().cpu().numpy()[0], oo) <= 1.0
    np.testing.assert_allclose(lse.cpu().numpy()[0], ol, atol=1e-3, rtol=0)


def test_window_longer_than_w_max_is_dropped(B, cuda_device):
    # a window of w_max + 5 rows (still inside its ring) breaks the call's
    # contract: the window is dropped, the device error word records it, and
    # the query attends its selected entries only
    rng = np.random.default_rng(31)
    lens, ps, h, k, w = [2000, 2000], 64, 32, 256, 100
    pt, cap, codes, scales = _cache(rng, lens, ps, 31)
    topk = np.stack([rng.permutation(2000)[:k].astype(np.int32) for _ in range(2)])
    swa_rows = 160
    swa = synth.normal_e4m3(31, 4, 0, 2 * swa_rows * 512).view(2, swa_rows, 512).numpy()
    begin = np.array([0, 10], np.int32)
    end = np.array([w, 10 + w + 5], np.int32)  # query 1: w_max + 5 rows
    q = synth.normal_bf16(31, 3, 0, 2 * h * 512).view(2, h, 512)
    scale = 1.0 / math.sqrt(512)
    kv = kv_from_numpy(codes, scales, None, pt, lens, ps, cuda_device)
    d = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(cuda_device)
    o = torch.full((2, h, 512), float("nan"), dtype=torch.bfloat16, device=cuda_device)
    lse = torch.full((2, h), float("nan"), dtype=torch.float32, device=cuda_device)
    ws = B.workspace(B.csa2_sparse_attn_workspace_size(2, h, k, w), cuda_device)
    B.csa2_sparse_attn_decode(q.to(cuda_device), 1, kv, d(topk), d(swa), swa_rows, d(begin), d(end), w, scale, o,
                              lse, ws)
    torch.cuda.synchronize()
    assert B.csa2_device_status() == 1  # CSA2_DEVERR_BAD_ROW
    go = o.float().cpu().numpy()
    o0, _ = oracle.sparse_attn(bf16_bits(q[0]), codes, scales, pt[0], ps, topk[0], swa[0][0:w], scale)
    o1, _ = oracle.sparse_attn(bf16_bits(q[1]), codes, scales, pt[1], ps, topk[1], None, scale)
    assert attn_excess(go[0], o0) <= 1.0
    assert attn_excess(go[1], o1) <= 1.0


def test_query_outside_f16_range_is_reported(B, cuda_device):
    # q is converted to f16 for the tensor-core products: a value whose
    # magnitude rounds beyond f16's largest finite value sets
    # CSA2_DEVERR_Q_RANGE; the other queries are unaffected
    rng = np.random.default_rng(32)
    lens, ps, h, k = [1500, 1500], 64, 16, 128
    pt, cap, codes, scales = _cache(rng, lens, ps, 32)
    topk = np.stack([rng.permutation(1500)[:k].astype(np.int32) for _ in range(2)])
    q = synth.normal_bf16(32, 3, 0, 2 * h * 512).view(2, h, 512).clone()
    q[1, 3, 17] = 70000.0
    scale = 1.0 / math.sqrt(512)
    kv = kv_from_numpy(codes, scales, None, pt, lens, ps, cuda_device)
    o = torch.full((2, h, 512), float("nan"), dtype=torch.bfloat16, device=cuda_device)
    lse = torch.full((2, h), float("nan"), dtype=torch.float32, device=cuda_device)
    ws = B.workspace(B.csa2_sparse_attn_workspace_size(2, h, k, 0), cuda_device)
    B.csa2_sparse_attn_decode(q.to(cuda_device), 1, kv, torch.from_numpy(topk).to(cuda_device), None, 0, None, None,
                              0, scale, o, lse, ws)
    torch.cuda.synchronize()
    assert B.csa2_device_status() == 8  # CSA2_DEVERR_Q_RANGE
    o0, _ = oracle.sparse_attn(bf16_bits(q[0]), codes, scales, pt[0], ps, topk[0], None, scale)
    assert attn_excess(o.float().cpu().numpy()[0], o0) <= 1.0


def test_merge_kernel_path(cuda_device):
    """Queries split over at most two CTAs are merged inside the attention kernel
    by the CTA that finishes their last part; wider splits by the merge
    kernel. This runs the attention tests again with the merge kernel for
    every split (CSA2_ATTN_MERGE=kernel, read per call; a separate process keeps
    the environment of this one)."""
    import os
    import subprocess
    import sys
    here = os.path.dirname(os.path.abspath(__file__))
    env = dict(os.environ, CSA2_ATTN_MERGE="kernel")
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-m", "gpu", "-p", "no:cacheprovider",
                        os.path.join(here, "test_attention_gpu.py"), "-k", "not merge_kernel_path"],
                       env=env, cwd=os.path.dirname(here), capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-2000:]
