"""The allocation-free decode attention entry point (fixed device scratch in
place of a caller workspace) against the regular entry point, through the
C-ABI, on two calls in a row with different inputs (the second call must not
see anything the first left in the shared scratch). Both entry points launch
the same kernels with the same split plan, only the partials' address
differs, so o and lse must be bit-identical. Also checks that a launch whose
partials would not fit the fixed scratch is refused on the host before
anything is launched (the refused call gets real, small device buffers, so
even a regression of the refusal could not touch memory outside them)."""
import math

import numpy as np
import pytest
import torch

import oracle
from helpers import bf16_bits, device_status_clean, kv_from_numpy, paged_layout
from sparse_fp4_kv_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def B():
    from sparse_fp4_kv_b200 import build
    build.build()
    from sparse_fp4_kv_b200 import binding
    return binding


def _inputs(dev, lens, ps, h, k, w, seed):
    rng = np.random.default_rng(seed)
    pt, cap = paged_layout(rng, lens, ps)
    x = synth.normal_bf16(seed, 1, 0, cap * 512).view(cap, 512)
    codes, scales = oracle.quantize_rows(bf16_bits(x))
    nq = len(lens)
    topk = np.full((nq, k), -1, np.int32)
    for qi in range(nq):
        m = min(k, lens[qi])
        topk[qi, :m] = rng.permutation(lens[qi])[:m]
        topk[qi] = rng.permutation(topk[qi])
    swa_rows = w + 37
    swa = synth.normal_e4m3(seed, 4, 0, nq * swa_rows * 512).view(nq, swa_rows, 512)
    begin = rng.integers(0, swa_rows - w + 1, nq).astype(np.int32)
    end = (begin + w).astype(np.int32)
    q = synth.normal_bf16(seed, 3, 0, nq * h * 512).view(nq, h, 512)
    kv = kv_from_numpy(codes, scales, None, pt, lens, ps, dev)
    d = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dev)
    return dict(q=q.to(dev), kv=kv, topk=d(topk), swa=swa.to(dev), swa_rows=swa_rows, begin=d(begin), end=d(end))


def _outputs(dev, nq, h):
    o = torch.full((nq, h, 512), float("nan"), dtype=torch.bfloat16, device=dev)
    lse = torch.full((nq, h), float("nan"), dtype=torch.float32, device=dev)
    return o, lse


def test_static_scratch_matches_workspace_path_twice(B, cuda_device):
    lens, ps, h, k, w = [3000, 2500, 4096, 1800], 64, 64, 1024, 256
    nq = len(lens)
    need = B.csa2_sparse_attn_workspace_size(nq, h, k, w)
    # the case splits every query, so the partials really go through the scratch
    assert 0 < need <= B.CSA2_ATTN_STATIC_SCRATCH_BYTES
    scale = 1.0 / math.sqrt(512)
    for call, seed in enumerate((21, 22)):
        I = _inputs(cuda_device, lens, ps, h, k, w, seed)
        o_ref, lse_ref = _outputs(cuda_device, nq, h)
        ws = B.workspace(need, cuda_device)
        B.csa2_sparse_attn_decode(I["q"], 1, I["kv"], I["topk"], I["swa"], I["swa_rows"], I["begin"], I["end"], w,
                                  scale, o_ref, lse_ref, ws)
        o, lse = _outputs(cuda_device, nq, h)
        B.csa2_sparse_attn_decode_static(I["q"], 1, I["kv"], I["topk"], I["swa"], I["swa_rows"], I["begin"],
                                         I["end"], w, scale, o, lse)
        torch.cuda.synchronize()
        assert device_status_clean()
        assert torch.isfinite(o.float()).all(), f"call {call}: non-finite output"
        assert torch.equal(o, o_ref), f"call {call}: o differs from the workspace path"
        assert torch.equal(lse, lse_ref), f"call {call}: lse differs from the workspace path"


def test_static_scratch_refuses_oversized_launch(B, cuda_device):
    # find a launch whose split partials exceed the fixed scratch; the call is
    # refused on the host (status 3) before any pointer is used
    h, k = 64, 4096
    big = None
    for nq in (8, 16, 24, 32, 48, 64, 96, 128):
        if B.csa2_sparse_attn_workspace_size(nq, h, k, 0) > B.CSA2_ATTN_STATIC_SCRATCH_BYTES:
            big = nq
            break
    assert big is not None
    dev = cuda_device
    # a real, small cache of one 128-row page per sequence, every Top-k id
    # empty (-1) and no window: a kernel launched by mistake would read and
    # write only inside these buffers
    rows = 128
    kv = B.KvCache(torch.zeros((big * rows, 256), dtype=torch.uint8, device=dev),
                   torch.zeros((big * rows, 32), dtype=torch.uint8, device=dev), None,
                   torch.arange(big, dtype=torch.int32, device=dev).view(big, 1),
                   torch.full((big,), rows, dtype=torch.int32, device=dev), rows)
    q = torch.zeros((big, h, 512), dtype=torch.bfloat16, device=dev)
    topk = torch.full((big, k), -1, dtype=torch.int32, device=dev)
    o = torch.zeros((big, h, 512), dtype=torch.bfloat16, device=dev)
    st = B._lib.csa2_sparse_attn_decode_static(q.data_ptr(), big, 1, h, kv.desc, topk.data_ptr(), k, None, 0,
                                               None, None, 0, 0.05, o.data_ptr(), None,
                                               torch.cuda.current_stream().cuda_stream)
    assert st == 3
    assert B.csa2_status_string(st) == "workspace missing or too small"
    torch.cuda.synchronize()
    assert device_status_clean()
