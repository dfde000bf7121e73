"""Shared helpers of the GPU parity tests: building small caches on both
sides from the same seeded inputs and comparing id lists."""
import numpy as np
import torch

import oracle
from sparse_fp4_kv_b200 import synth

ATTN_TOL = 2e-3  # max |o_gpu - o_oracle| where |o| <= 0.5 (bf16 output)


def attn_excess(o_gpu, o_ref):
    """Largest ratio of an output's error to its bound over the outputs; <= 1
    passes. Where |o_ref| <= 0.5 the bound is the acceptance bar 2e-3 on
    |o_gpu - o_ref| (meaningful for the N(0,1) workloads, where |o| stays far
    below 0.5). Above 0.5 half a bf16 ulp of the output alone can exceed
    2e-3, so there the kernel's bf16 value must lie within one bf16 ulp of the
    bf16 rounding of the oracle's value: the kernel's own error may only move
    the rounding to a neighbouring bf16 value."""
    o_gpu = np.asarray(o_gpu, np.float64)
    o_ref = np.asarray(o_ref, np.float64)
    a = np.abs(o_ref)
    big = a > 0.5
    ratio = np.abs(o_gpu - o_ref) / ATTN_TOL
    if big.any():
        rb = torch.from_numpy(o_ref[big]).to(torch.bfloat16).double().numpy()
        ulp = np.exp2(np.floor(np.log2(np.abs(rb))) - 7.0)
        ratio[big] = np.abs(o_gpu[big] - rb) / ulp
    return float(ratio.max()) if ratio.size else 0.0


def bf16_bits(t):
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def int_e4m3_np(rng, shape, lo=-8, hi=8):
    v = rng.integers(lo, hi + 1, size=shape).astype(np.float32)
    return torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def paged_layout(rng, lens, ps, shuffle=True, spare_pages=3):
    """Page table [batch, max_pages] over a pool of physical pages."""
    npages = [max(1, (int(l) + ps - 1) // ps) for l in lens]
    total = sum(npages) + spare_pages
    perm = rng.permutation(total) if shuffle else np.arange(total)
    pt = np.full((len(lens), max(npages)), -1, np.int32)
    off = 0
    for b, c in enumerate(npages):
        pt[b, :c] = perm[off:off + c]
        off += c
    return pt, total * ps


def compare_ids(gpu_row, oracle_row, what=""):
    """GPU lists are in ascending id order then -1; oracle lists are in score
    order then -1. Same multiset of ids and same padding length required."""
    g = np.asarray(gpu_row)
    o = np.asarray(oracle_row)
    assert g.shape == o.shape, what
    ng = int((g >= 0).sum())
    no = int((o >= 0).sum())
    assert ng == no, f"{what}: {ng} ids vs {no}"
    assert np.all(g[ng:] == -1), f"{what}: padding"
    np.testing.assert_array_equal(np.sort(g[:ng]), np.sort(o[:no]), err_msg=what)


def kv_from_numpy(codes, scales, kidx, page_table, seq_len, ps, device):
    from sparse_fp4_kv_b200 import binding as B
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(device)
    return B.KvCache(t(codes), t(scales), t(kidx) if kidx is not None else None, t(page_table),
                     t(np.asarray(seq_len, np.int32)), ps)


def device_status_clean():
    from sparse_fp4_kv_b200 import binding as B
    return B.csa2_device_status() == 0


def normal_bf16_rows(seed, stream, n, d=512):
    return synth.normal_bf16(seed, stream, 0, n * d).view(n, d)
