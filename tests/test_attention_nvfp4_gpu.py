"""NVFP4 variant of the decode attention (csa2_sparse_attn_decode_nvfp4)
against its oracle: the exact attention with q rounded to NVFP4 by the
cache's block quantiser (oracle.sparse_attn_nvfp4). Same bar as the exact
kernel: outputs within 2e-3 max-abs (bf16 out), log-sum-exp within 1e-3.
Covers 64 heads, and 16 / 32 heads run as 64 with zero-padded q; tiles of selected entries only (block-scaled FP4
products) and the partial last entry tile plus the window (f16 path with the
rounded q), k below one tile, no window, window only, -1 ids, many queries,
the empty set and the running-maximum raise. Also records how far the
variant lands from the exact attention of the unrounded q."""
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


def _run(B, dev, lens, ps, h, k, w, q_per_seq=1, seed=0, neg_frac=0.05, swa_rows=None, q_mul=1.0):
    rng = np.random.default_rng(seed)
    pt, cap = paged_layout(rng, lens, ps)
    x = synth.normal_bf16(seed, 1, 0, cap * 512).view(cap, 512)
    codes, scales = oracle.quantize_rows(bf16_bits(x))
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
    begin = rng.integers(0, swa_rows - w + 1, nq).astype(np.int32)
    end = (begin + w).astype(np.int32)
    q = (synth.normal_bf16(seed, 3, 0, nq * h * 512).view(nq, h, 512) * q_mul).to(torch.bfloat16)
    scale = 1.0 / math.sqrt(512)
    kv = kv_from_numpy(codes, scales, None, pt, lens, ps, dev)
    o = torch.full((nq, h, 512), float("nan"), dtype=torch.bfloat16, device=dev)
    lse = torch.full((nq, h), float("nan"), dtype=torch.float32, device=dev)
    ws = B.workspace(B.csa2_sparse_attn_nvfp4_workspace_size(nq, h, k, w), dev)
    d = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dev)
    B.csa2_sparse_attn_decode_nvfp4(q.to(dev), q_per_seq, kv, d(topk) if k > 0 else None, d(swa), swa_rows,
                                    d(begin), d(end), w, scale, o, lse, ws)
    torch.cuda.synchronize()
    assert device_status_clean()
    go = o.float().cpu().numpy()
    gl = lse.cpu().numpy()
    dev_exact = 0.0
    for qi in range(nq):
        b = qi // q_per_seq
        win = swa[b][begin[qi]:end[qi]] if w > 0 else None
        oo, ol = oracle.sparse_attn_nvfp4(bf16_bits(q[qi]), codes, scales, pt[b], ps, topk[qi], win, scale)
        err = np.abs(go[qi] - oo).max()
        assert attn_excess(go[qi], oo) <= 1.0, f"q{qi}: max |o - oracle| = {err}"
        fin = np.isfinite(ol)
        assert np.all(np.isfinite(gl[qi]) == fin)
        np.testing.assert_allclose(gl[qi][fin], ol[fin], atol=1e-3, rtol=0)
        if qi < 2:
            oe, _ = oracle.sparse_attn(bf16_bits(q[qi]), codes, scales, pt[b], ps, topk[qi], win, scale)
            dev_exact = max(dev_exact, float(np.abs(go[qi] - oe).max()))
    return go, gl, dev_exact


def test_ragged_tiles(B, cuda_device):
    _run(B, cuda_device, [900, 1500], 64, 64, 300, 77, seed=32)


def test_single_query_many_tiles(B, cuda_device):
    # 16 tiles of selected entries (FP4 products) + 4 window tiles (f16 path)
    _, _, dev_exact = _run(B, cuda_device, [70000], 128, 64, 2048, 512, seed=1)
    print(f"max |o_nvfp4 - o_exact(unrounded q)| = {dev_exact:.4f}")
    assert dev_exact > 0.0


def test_several_queries_ragged(B, cuda_device):
    _run(B, cuda_device, [9000, 5000, 3000], 64, 64, 1300, 200, seed=21)
    _run(B, cuda_device, [9000, 7000], 64, 64, 1800, 300, seed=22)


def test_many_queries(B, cuda_device):
    _run(B, cuda_device, [600] * 4, 64, 64, 256, 33, q_per_seq=40, seed=2, swa_rows=160)


def test_no_window_window_only_and_short_k(B, cuda_device):
    _run(B, cuda_device, [500], 64, 64, 256, 0, seed=3)
    _run(B, cuda_device, [500], 64, 64, 0, 130, seed=4)
    _run(B, cuda_device, [500], 64, 64, 100, 50, seed=5)


def test_empty_set_gives_zero(B, cuda_device):
    go, gl, _ = _run(B, cuda_device, [300], 64, 64, 256, 0, seed=6, neg_frac=1.0)
    assert np.all(go == 0) and np.all(np.isneginf(gl))


def test_large_scores_raise_running_max(B, cuda_device):
    # q x 8: scores spread over far more than 2^8 in base 2, so later tiles
    # raise the running maximum (rescale of O) on the FP4 path too
    _run(B, cuda_device, [20000], 64, 64, 1024, 0, seed=7, q_mul=8.0)


@pytest.mark.parametrize("h", [16, 32])
def test_fewer_heads_run_padded_to_64(B, cuda_device, h):
    # 16 and 32 heads run as a 64-head call with q padded by zero heads (the
    # block-scaled products keep the shape whose scale-factor layout is
    # validated); the padded heads' outputs are dropped
    _run(B, cuda_device, [9000, 5000], 64, h, 1300, 200, seed=40 + h)
    _run(B, cuda_device, [600] * 3, 64, h, 256, 33, q_per_seq=8, seed=50 + h, swa_rows=160)
