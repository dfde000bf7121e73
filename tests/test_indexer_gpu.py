"""Full and Reindex indexer kernels against the oracle. Inputs are
small-integer E4M3 values, so every score is an exact integer in binary32
and the Top-k / pool id sets must match the oracle's exactly (ties broken
toward the lower id). Covers contiguous and shuffled-paged caches, di 64 and
128, 1..16 heads, ragged lengths, causal per-query limits, sequences shorter
than k, all-equal scores and the largest per-head dot products."""
import os

import numpy as np
import pytest
import torch

import oracle
from helpers import compare_ids, device_status_clean, int_e4m3_np, kv_from_numpy, paged_layout

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def B():
    from sparse_fp4_kv_b200 import build
    build.build()
    from sparse_fp4_kv_b200 import binding
    return binding


def _case(rng, lens, ps, di, hi, q_per_seq=1, kidx_fn=None, shuffle=True):
    pt, cap = paged_layout(rng, lens, ps, shuffle=shuffle)
    kidx = kidx_fn(cap, di) if kidx_fn else int_e4m3_np(rng, (cap, di))
    nq = len(lens) * q_per_seq
    qidx = int_e4m3_np(rng, (nq, hi, di))
    w = rng.integers(1, 5, (nq, hi)).astype(np.float32)
    codes = np.zeros((cap, 256), np.uint8)
    scales = np.zeros((cap, 32), np.uint8)
    return pt, cap, kidx, qidx, w, codes, scales


def _run_full(B, dev, lens, ps, di, hi, k, p, q_per_seq=1, q_limit=None, kidx_fn=None, seed=0, shuffle=True):
    rng = np.random.default_rng(seed)
    pt, cap, kidx, qidx, w, codes, scales = _case(rng, lens, ps, di, hi, q_per_seq, kidx_fn, shuffle)
    kv = kv_from_numpy(codes, scales, kidx, pt, lens, ps, dev)
    nq = qidx.shape[0]
    n_max = max(lens) if q_limit is None else int(max(q_limit))
    topk = torch.full((nq, k), -7, dtype=torch.int32, device=dev)
    pool = torch.full((nq, p), -7, dtype=torch.int32, device=dev) if p > 0 else None
    ws = B.workspace(B.csa2_index_full_workspace_size(nq, n_max), dev)
    ql = torch.from_numpy(np.asarray(q_limit, np.int32)).to(dev) if q_limit is not None else None
    B.csa2_index_full(torch.from_numpy(qidx).to(dev), torch.from_numpy(w).to(dev), q_per_seq, ql, n_max, kv, k, p,
                      topk, pool, ws)
    torch.cuda.synchronize()
    assert device_status_clean()
    g_topk = topk.cpu().numpy()
    g_pool = pool.cpu().numpy() if pool is not None else None
    # the multi-launch path leaves every score key in the workspace (offset 0);
    # the single-launch cluster path keeps them in shared memory
    multipass = os.environ.get("CSA2_FULL_PATH") == "multipass"
    keys = ws[: nq * ((max(n_max, 1) + 127) // 128 * 128) * 4].view(torch.int32).cpu().numpy().view(np.uint32)
    keys = keys.reshape(nq, -1)
    for qi in range(nq):
        b = qi // q_per_seq
        lim = lens[b] if q_limit is None else int(q_limit[qi])
        ot, op, osc = oracle.index_full(qidx[qi], w[qi], kidx, pt[b], ps, lim, k, p, want_scores=True)
        # scores: the kernel's ordered keys decode to the oracle's exact scores
        if multipass:
            u = keys[qi, :lim]
            f = np.where(u & 0x80000000, u & 0x7FFFFFFF, ~u).astype(np.uint32).view(np.float32)
            np.testing.assert_array_equal(f.astype(np.float64), osc, err_msg=f"scores q{qi}")
        compare_ids(g_topk[qi], ot, f"topk q{qi}")
        assert np.all(np.diff(g_topk[qi][g_topk[qi] >= 0]) > 0), "ascending ids"
        if p > 0:
            compare_ids(g_pool[qi], op, f"pool q{qi}")
            assert set(g_topk[qi][g_topk[qi] >= 0]) <= set(g_pool[qi][g_pool[qi] >= 0])
    return g_topk, g_pool, (pt, kidx, qidx, w, kv)


def test_full_contiguous_di64(B, cuda_device):
    _run_full(B, cuda_device, [4096 + 37], 4224, 64, 4, 512, 1024, shuffle=False)


def test_full_paged_ragged_batch(B, cuda_device):
    _run_full(B, cuda_device, [1000, 130, 2047, 64], 64, 64, 4, 100, 300)


def test_full_di128_eight_heads(B, cuda_device):
    _run_full(B, cuda_device, [5000, 3333], 128, 128, 8, 256, 700, seed=1)


def test_full_page32_and_head_extremes(B, cuda_device):
    _run_full(B, cuda_device, [777], 32, 64, 1, 50, 0, seed=2)
    _run_full(B, cuda_device, [900, 1200], 256, 128, 16, 64, 128, seed=3)


def test_full_short_sequences_pad(B, cuda_device):
    _run_full(B, cuda_device, [50, 1, 200], 64, 64, 4, 64, 128, seed=4)


def test_full_causal_queries(B, cuda_device):
    total = 3000
    q_limit = [total - 40 + j + 1 for j in range(40)]
    _run_full(B, cuda_device, [total], 3072, 64, 4, 200, 0, q_per_seq=40, q_limit=q_limit, seed=5,
              shuffle=False)


def test_full_empty_sequences_and_many_queries(B, cuda_device):
    # sequences without entries between others (a query that owns no tile),
    # and 400 causal queries of one sequence (the batched path by default, the
    # multi-launch path when it is forced)
    _run_full(B, cuda_device, [700, 0, 3000, 129, 0, 5000], 64, 64, 4, 100, 300, seed=16)
    total = 3000
    _run_full(B, cuda_device, [total], 3072, 64, 4, 150, 0, q_per_seq=400, q_limit=_causal(total, 400), seed=17,
              shuffle=False)


@pytest.mark.parametrize("csize", ["auto", "10", "12", "16"])
def test_full_long_sequences_ragged(B, cuda_device, monkeypatch, csize):
    # long enough that a query's entries are spread over 8 to 16 CTAs (the
    # cluster size chosen by the library, or fixed), with ragged tails
    if csize != "auto":
        monkeypatch.setenv("CSA2_FULL_CLUSTER", csize)
    _run_full(B, cuda_device, [40000 + 17, 33333], 40064, 64, 4, 2048, 4096, shuffle=False, seed=14)
    _run_full(B, cuda_device, [36000 + 5], 36096, 128, 8, 1000, 3000, shuffle=False, seed=15)


def test_full_all_ties_take_lowest_ids(B, cuda_device):
    same = lambda cap, di: np.full((cap, di), 0x38, np.uint8)  # every key = 1.0
    topk, pool, _ = _run_full(B, cuda_device, [2500], 64, 64, 4, 300, 900, kidx_fn=same, seed=6)
    assert list(topk[0]) == list(range(300))
    assert list(pool[0]) == list(range(900))


def test_full_largest_dot_products_exact(B, cuda_device):
    # |q_h . k| up to 64 * 64 (di 64) and 128 * 64 (di 128): accumulation must be exact
    def extreme(cap, di):
        rng = np.random.default_rng(7)
        v = np.where(rng.random((cap, di)) < 0.97, 8.0, -8.0).astype(np.float32)
        return torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    _run_full(B, cuda_device, [3000], 64, 64, 4, 333, 1000, kidx_fn=extreme, seed=7)
    _run_full(B, cuda_device, [3000], 64, 128, 8, 333, 1000, kidx_fn=extreme, seed=8)


@pytest.mark.parametrize("di,hi", [(64, 4), (128, 8)])
def test_reindex_matches_oracle(B, cuda_device, di, hi):
    lens = [3000, 1800]
    topk, pool, (pt, kidx, _, _, kv) = _run_full(B, cuda_device, lens, 64, di, hi, 200, 600, seed=9)
    rng = np.random.default_rng(10)
    nq = len(lens)
    qidx = int_e4m3_np(rng, (nq, hi, di))
    w = rng.integers(1, 5, (nq, hi)).astype(np.float32)
    # the Full layer's pool, shuffled, with -1 padding spread through it
    pools = np.full((nq, 700), -1, np.int32)
    for qi in range(nq):
        ids = pool[qi][pool[qi] >= 0]
        pos = rng.permutation(700)[: ids.size]
        pools[qi, pos] = rng.permutation(ids)
    out = torch.full((nq, 200), -7, dtype=torch.int32, device=cuda_device)
    ws = B.workspace(B.csa2_index_reindex_workspace_size(nq, 700), cuda_device)
    B.csa2_index_reindex(torch.from_numpy(qidx).to(cuda_device), torch.from_numpy(w).to(cuda_device), 1,
                         torch.from_numpy(pools).to(cuda_device), kv, 200, out, ws)
    torch.cuda.synchronize()
    assert device_status_clean()
    g = out.cpu().numpy()
    for qi in range(nq):
        want = oracle.index_reindex(qidx[qi], w[qi], kidx, pt[qi], 64, pools[qi], 200)
        compare_ids(g[qi], want, f"reindex q{qi}")


def test_reindex_with_every_entry_equals_full(B, cuda_device):
    n = 2000
    topk, _, (pt, kidx, qidx, w, kv) = _run_full(B, cuda_device, [n], 64, 64, 4, 150, 0, seed=11)
    rng = np.random.default_rng(12)
    allp = rng.permutation(n).astype(np.int32)[None, :]
    out = torch.empty((1, 150), dtype=torch.int32, device=cuda_device)
    ws = B.workspace(B.csa2_index_reindex_workspace_size(1, n), cuda_device)
    B.csa2_index_reindex(torch.from_numpy(qidx).to(cuda_device), torch.from_numpy(w).to(cuda_device), 1,
                         torch.from_numpy(allp).to(cuda_device), kv, 150, out, ws)
    torch.cuda.synchronize()
    assert sorted(out.cpu().numpy()[0]) == sorted(topk[0])


def test_reindex_ties_and_short_pool(B, cuda_device):
    n = 600
    same = lambda cap, di: np.full((cap, di), 0x38, np.uint8)
    _, _, (pt, kidx, qidx, w, kv) = _run_full(B, cuda_device, [n], 64, 64, 4, 10, 0, kidx_fn=same, seed=13)
    pool = np.array([[500, -1, 3, 77, 2, -1, 599, 4, 1, 0, 300]], np.int32)
    out = torch.empty((1, 6), dtype=torch.int32, device=cuda_device)
    ws = B.workspace(B.csa2_index_reindex_workspace_size(1, pool.shape[1]), cuda_device)
    B.csa2_index_reindex(torch.from_numpy(qidx).to(cuda_device), torch.from_numpy(w).to(cuda_device), 1,
                         torch.from_numpy(pool).to(cuda_device), kv, 6, out, ws)
    torch.cuda.synchronize()
    assert sorted(out.cpu().numpy()[0]) == [0, 1, 2, 3, 4, 77]
    out2 = torch.empty((1, 12), dtype=torch.int32, device=cuda_device)
    B.csa2_index_reindex(torch.from_numpy(qidx).to(cuda_device), torch.from_numpy(w).to(cuda_device), 1,
                         torch.from_numpy(pool).to(cuda_device), kv, 12, out2, ws)
    torch.cuda.synchronize()
    g = out2.cpu().numpy()[0]
    assert sorted(g[:9]) == sorted(pool[0][pool[0] >= 0]) and list(g[9:]) == [-1, -1, -1]


# ---- many queries of one sequence: the batched path (16 queries per key tile
# with up to 4 indexer heads, 8 with up to 8), chosen for 64 or more queries
# per sequence without a pool ----
def _causal(total, nqs, first=None):
    first = total - nqs if first is None else first
    return [min(total, first + j + 1) for j in range(nqs)]


def test_full_batched_causal_di64(B, cuda_device):
    total = 5000
    _run_full(B, cuda_device, [total], 5120, 64, 4, 300, 0, q_per_seq=64, q_limit=_causal(total, 64), seed=21,
              shuffle=False)


def test_full_batched_two_sequences_paged_di128(B, cuda_device):
    # two sequences of 64 queries each, eight indexer heads (8 queries per
    # tile), a shuffled 64-entry page table; each query sees all of its sequence
    _run_full(B, cuda_device, [3000, 2600], 64, 128, 8, 400, 0, q_per_seq=64, seed=22)


def test_full_batched_limits_below_k(B, cuda_device):
    # the first queries see fewer entries than k: all of them, then -1 padding
    total = 2000
    _run_full(B, cuda_device, [total], 2048, 64, 3, 500, 0, q_per_seq=128, q_limit=_causal(total, 128, first=100),
              seed=23, shuffle=False)


def test_full_batched_all_ties(B, cuda_device):
    same = lambda cap, di: np.full((cap, di), 0x38, np.uint8)  # every key = 1.0
    topk, _, _ = _run_full(B, cuda_device, [3000], 3072, 64, 4, 700, 0, q_per_seq=64, kidx_fn=same, seed=24,
                           shuffle=False)
    for qi in range(64):
        assert list(topk[qi]) == list(range(700))


def test_full_batched_largest_dot_products(B, cuda_device):
    def extreme(cap, di):
        rng = np.random.default_rng(25)
        v = np.where(rng.random((cap, di)) < 0.97, 8.0, -8.0).astype(np.float32)
        return torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    _run_full(B, cuda_device, [4000], 4096, 128, 8, 333, 0, q_per_seq=64, kidx_fn=extreme, seed=25, shuffle=False)


def test_full_batched_sample_misses_leave_it_to_the_exact_passes(B, cuda_device):
    # the batched path first samples every 32nd tile of 256 entries (entries
    # [8192 j, 8192 j + 256)) and takes the keys at or above a threshold from
    # that sample; here exactly those tiles hold the largest scores, so the
    # threshold leaves fewer than k candidates and the exact passes must take
    # over (the result is checked against the oracle as usual)
    total = 40000

    def sampled_high(cap, di):
        rng = np.random.default_rng(26)
        v = np.where(rng.random(di) < 0.5, 1.0, -1.0).astype(np.float32)
        t = np.arange(cap)
        high = (t % 8192) < 256
        mag = np.where(high, rng.choice([4.0, 6.0], cap), rng.choice([0.5, 1.0], cap)).astype(np.float32)
        x = mag[:, None] * v[None, :]
        return torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()

    _run_full(B, cuda_device, [total], 40960, 64, 4, 600, 0, q_per_seq=64, kidx_fn=sampled_high, seed=26,
              shuffle=False)
