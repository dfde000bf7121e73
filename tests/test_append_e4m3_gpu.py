"""FP8 appends (window rows into per-sequence rings, indexer keys into the
paged key array) against the oracle, bit-exact: every bf16 bit pattern,
ring wrap-around, shuffled pages, di 64 and 128, bad destinations; and the
attention kernel reading a window that wraps around the end of its ring."""
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


def _all_patterns(rows, width):
    bits = np.arange(rows * width, dtype=np.int64) % 65536
    return bits.astype(np.uint16).reshape(rows, width)


def test_window_append_every_bf16_pattern(B, cuda_device):
    rng = np.random.default_rng(41)
    batch, ring = 2, 64
    x = _all_patterns(128, 512)                    # all 65536 bf16 patterns
    # 128 distinct (sequence, slot) pairs; positions wrap the ring several times
    pairs = rng.permutation(batch * ring)
    seq = (pairs // ring).astype(np.int32)
    pos = (pairs % ring + ring * rng.integers(0, 20, pairs.size)).astype(np.int64)
    swa = np.full((batch, ring, 512), 0xAA, np.uint8)
    want = swa.copy()
    oracle.append_swa_e4m3(x, seq, pos, want)
    d = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(cuda_device)
    g = d(swa)
    B.csa2_append_swa_e4m3(d(x.view(np.int16)).view(torch.bfloat16), d(seq), d(pos), g)
    torch.cuda.synchronize()
    assert device_status_clean()
    np.testing.assert_array_equal(g.cpu().numpy(), want)


@pytest.mark.parametrize("di", [64, 128])
def test_key_append_paged(B, cuda_device, di):
    rng = np.random.default_rng(42 + di)
    lens, ps = [3000, 1700, 2222], 64
    pt, cap = paged_layout(rng, lens, ps)
    kidx = rng.integers(0, 256, (cap, di)).astype(np.uint8)
    codes = np.zeros((cap, 256), np.uint8)
    scales = np.zeros((cap, 32), np.uint8)
    kv = kv_from_numpy(codes, scales, kidx, pt, lens, ps, cuda_device)
    # 600 distinct (sequence, position) pairs
    cand = np.array([(b, t) for b, n in enumerate(lens) for t in range(n)])
    pick = cand[rng.permutation(len(cand))[:600]]
    seq, pos = pick[:, 0].astype(np.int32), pick[:, 1].astype(np.int64)
    x = synth.normal_bf16(7, di, 0, 600 * di).view(600, di)
    want = kidx.copy()
    oracle.append_kidx_e4m3(bf16_bits(x), seq, pos, pt, ps, want)
    d = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(cuda_device)
    B.csa2_append_kidx_e4m3(x.to(cuda_device), d(seq), d(pos), kv)
    torch.cuda.synchronize()
    assert device_status_clean()
    np.testing.assert_array_equal(kv.kidx.cpu().numpy(), want)


def test_bad_destinations_set_the_error_word(B, cuda_device):
    batch, ring = 2, 16
    x = synth.normal_bf16(8, 0, 0, 4 * 512).view(4, 512).to(cuda_device)
    swa = torch.zeros((batch, ring, 512), dtype=torch.uint8, device=cuda_device)
    seq = torch.tensor([0, 5, 1, -1], dtype=torch.int32, device=cuda_device)
    pos = torch.tensor([3, 3, -2, 4], dtype=torch.int64, device=cuda_device)
    B.csa2_append_swa_e4m3(x, seq, pos, swa)
    torch.cuda.synchronize()
    assert B.csa2_device_status() != 0             # rows 1, 2, 3 are skipped and reported
    assert B.csa2_device_status() == 0             # reading clears it
    got = swa.cpu().numpy()
    want = np.zeros_like(got)
    oracle.append_swa_e4m3(bf16_bits(x[:1]), np.array([0], np.int32), np.array([3], np.int64), want)
    np.testing.assert_array_equal(got, want)


def test_attention_window_wraps_around_the_ring(B, cuda_device):
    rng = np.random.default_rng(43)
    lens, ps, h, k, ring = [5000, 4000], 64, 32, 700, 300
    pt, cap = paged_layout(rng, lens, ps)
    xr = synth.normal_bf16(9, 1, 0, cap * 512).view(cap, 512)
    codes, scales = oracle.quantize_rows(bf16_bits(xr))
    kv = kv_from_numpy(codes, scales, None, pt, lens, ps, cuda_device)
    nq = len(lens)
    topk = np.stack([rng.permutation(n)[:k] for n in lens]).astype(np.int32)
    swa = synth.normal_e4m3(9, 4, 0, nq * ring * 512).view(nq, ring, 512).numpy()
    begin = np.array([250, 120], np.int32)          # query 0 wraps: 250..299, then 0..149
    end = np.array([450, 320], np.int32)            # query 1 wraps: 120..299, then 0..19
    w = 200
    q = synth.normal_bf16(9, 3, 0, nq * h * 512).view(nq, h, 512)
    d = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(cuda_device)
    o = torch.empty((nq, h, 512), dtype=torch.bfloat16, device=cuda_device)
    lse = torch.empty((nq, h), dtype=torch.float32, device=cuda_device)
    ws = B.workspace(B.csa2_sparse_attn_workspace_size(nq, h, k, w), cuda_device)
    scale = 1.0 / math.sqrt(512)
    B.csa2_sparse_attn_decode(q.to(cuda_device), 1, kv, d(topk), d(swa), ring, d(begin), d(end), w, scale, o, lse,
                              ws)
    torch.cuda.synchronize()
    assert device_status_clean()
    for qi in range(nq):
        rows = swa[qi][(begin[qi] + np.arange(end[qi] - begin[qi])) % ring]
        oo, ol = oracle.sparse_attn(bf16_bits(q[qi]), codes, scales, pt[qi], ps, topk[qi], rows, scale)
        go = o[qi].float().cpu().numpy()
        assert attn_excess(go, oo) <= 1.0, f"q{qi}: {np.abs(go - oo).max()}"
        np.testing.assert_allclose(lse[qi].cpu().numpy(), ol, atol=1e-3, rtol=0)
