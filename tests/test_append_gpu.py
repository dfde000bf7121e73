"""FP4 quantise + append kernel against the oracle: codes and scales must be
bit-exact. Inputs cover every bf16 bit pattern (NaN, Inf, subnormals),
blocks built around exact rounding midpoints at many scales, N(0,1) rows
with x20 outliers, and paged placement."""
import numpy as np
import pytest
import torch

import oracle
from helpers import bf16_bits, device_status_clean, paged_layout

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def B():
    from sparse_fp4_kv_b200 import build
    build.build()
    from sparse_fp4_kv_b200 import binding
    return binding


def _run_append(B, x_bf16, seq, pos, page_table, rows_cap, ps, device):
    codes = torch.zeros((rows_cap, 256), dtype=torch.uint8, device=device)
    scales = torch.zeros((rows_cap, 32), dtype=torch.uint8, device=device)
    pt = torch.from_numpy(page_table).to(device)
    seq_len = torch.zeros(page_table.shape[0], dtype=torch.int32, device=device)
    kv = B.KvCache(codes, scales, None, pt, seq_len, ps)
    B.csa2_append_fp4(x_bf16.to(device).contiguous(), torch.from_numpy(seq).to(device),
                      torch.from_numpy(pos).to(device), kv)
    torch.cuda.synchronize()
    return codes.cpu().numpy(), scales.cpu().numpy()


def _check_rows(B, x_bf16, device, ps=None):
    n = x_bf16.shape[0]
    ps = ps or 128 * ((n + 127) // 128)
    rng = np.random.default_rng(n)
    pt, cap = paged_layout(rng, [n], ps)
    seq = np.zeros(n, np.int32)
    pos = np.arange(n, dtype=np.int64)
    codes, scales = _run_append(B, x_bf16, seq, pos, pt, cap, ps, device)
    oc = np.zeros((cap, 256), np.uint8)
    osc = np.zeros((cap, 32), np.uint8)
    oracle.append_fp4(bf16_bits(x_bf16), seq, pos, pt, ps, oc, osc)
    bad_s = np.argwhere(scales != osc)
    assert bad_s.size == 0, f"scale mismatch at {bad_s[:5]}"
    bad_c = np.argwhere(codes != oc)
    assert bad_c.size == 0, f"code mismatch at {bad_c[:5]}"
    assert device_status_clean()


def test_every_bf16_pattern(B, cuda_device):
    # all 65536 patterns, 16 consecutive patterns per block, 128 rows
    bits = torch.arange(65536, dtype=torch.int32).to(torch.int16)
    x = bits.view(torch.bfloat16).view(128, 512)
    _check_rows(B, x, cuda_device)
    # the same patterns with each block's amax set by a leading element at
    # several scales, so every pattern is also rounded against finite scales
    rows = []
    for amax in [6.0, 1.0, 0.1, 448.0, 6 * 448.0, 1e-3, 3.0e4]:
        xb = x.clone().view(-1, 16)
        xb[:, 0] = amax
        keep = torch.isfinite(xb).all(dim=1) & (xb.float().abs().amax(dim=1) <= amax)
        rows.append(xb[keep])
    y = torch.cat(rows)
    y = y[: (y.shape[0] // 32) * 32].reshape(-1, 512)
    _check_rows(B, y, cuda_device)


def test_midpoints_at_many_scales(B, cuda_device):
    # blocks whose values sit on, just above and just below x/value(s)
    # midpoints of the E2M1 grid, for scales across the E4M3 range
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])
    rows = []
    for e in range(-9, 9):
        for m in range(8):
            s = (1 + m / 8) * 2.0 ** e
            if s > 448:
                continue
            vals = np.concatenate([[6 * s], mids * s, np.nextafter(mids * s, 0), np.nextafter(mids * s, 99)])
            vals = vals[:16]
            vals = np.concatenate([vals, np.zeros(16 - vals.size)])
            sign = np.where(np.arange(16) % 3 == 0, -1.0, 1.0)
            sign[0] = 1.0
            rows.append(vals * sign)
    blocks = torch.tensor(np.array(rows), dtype=torch.float32).to(torch.bfloat16)
    nb = blocks.shape[0]
    pad = (-nb) % 32
    blocks = torch.cat([blocks, torch.zeros((pad, 16), dtype=torch.bfloat16)])
    _check_rows(B, blocks.reshape(-1, 512), cuda_device)


def test_normal_rows_with_outliers_paged(B, cuda_device):
    from sparse_fp4_kv_b200 import synth
    n = 3000
    x = synth.normal_bf16(4, 5, 0, n * 512, outlier_p=0.01, outlier_mul=20.0, outlier_stream=6).view(n, 512)
    x[7] = 0.0
    x[8] = x[8] * 1e-4
    _check_rows(B, x, cuda_device, ps=64)


@pytest.mark.parametrize("n", [1, 17, 4097, 131073])
def test_ragged_row_counts(B, cuda_device, n):
    # row counts that leave warps of the grid without rows or with one row
    # fewer than others; 131073 rows give every warp of a full one-wave grid
    # (148 SMs x 3 CTAs x 8 warps) more than one group of 32 rows. Rows nobody
    # writes must stay zero
    from sparse_fp4_kv_b200 import synth
    x = synth.normal_bf16(12, 3, 0, n * 512, outlier_p=0.01, outlier_mul=20.0, outlier_stream=6).view(n, 512)
    _check_rows(B, x, cuda_device, ps=64)


def test_scattered_positions_and_bad_rows(B, cuda_device):
    rng = np.random.default_rng(3)
    ps = 32
    lens = [100, 70, 300]
    pt, cap = paged_layout(rng, lens, ps)
    n = 50
    seq = rng.integers(0, 3, n).astype(np.int32)
    pos = np.array([rng.integers(0, lens[s]) for s in seq], np.int64)
    _, idx = np.unique(seq.astype(np.int64) * 1000 + pos, return_index=True)  # distinct targets
    seq, pos = seq[idx], pos[idx]
    from sparse_fp4_kv_b200 import synth
    x = synth.normal_bf16(9, 1, 0, len(seq) * 512).view(len(seq), 512)
    codes, scales = _run_append(B, x, seq, pos, pt, cap, ps, cuda_device)
    oc = np.zeros((cap, 256), np.uint8)
    osc = np.zeros((cap, 32), np.uint8)
    oracle.append_fp4(bf16_bits(x), seq, pos, pt, ps, oc, osc)
    np.testing.assert_array_equal(codes, oc)
    np.testing.assert_array_equal(scales, osc)
    assert device_status_clean()
    # a position beyond the page table is skipped and reported
    seq2 = np.array([0, 1], np.int32)
    pos2 = np.array([5, pt.shape[1] * ps + 3], np.int64)
    codes2, _ = _run_append(B, x[:2], seq2, pos2, pt, cap, ps, cuda_device)
    from sparse_fp4_kv_b200 import binding
    assert binding.csa2_device_status() & 1
    row0 = pt[0, 0] * ps + 5
    oc2 = np.zeros((1, 256), np.uint8)
    oracle.append_fp4(bf16_bits(x[:1]), np.zeros(1, np.int32), np.zeros(1, np.int64), np.zeros((1, 1), np.int32),
                      1, oc2, np.zeros((1, 32), np.uint8))
    np.testing.assert_array_equal(codes2[row0], oc2[0])
    assert codes2.sum() == oc2.sum()
