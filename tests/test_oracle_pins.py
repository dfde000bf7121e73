"""Pins for the CPU oracle: every oracle function is checked here against
something other than itself -- printed format definitions (tests/golden/),
hand-derived worked examples, a library routine (torch's float8 conversion
and softmax/matmul), brute force on small inputs, and invariants the
method fixes. No GPU is used."""
import math
import os

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden_lines(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return [ln.strip() for ln in f if ln.strip() and not ln.startswith("#")]


def _bf16_bits(vals):
    t = torch.tensor(vals, dtype=torch.float32).to(torch.bfloat16)
    return t.view(torch.int16).numpy().astype(np.uint16)


# ---------------------------------------------------------------------------
# Number formats
# ---------------------------------------------------------------------------

def test_e2m1_decode_matches_ocp_table():
    for ln in _golden_lines("e2m1_codes.txt"):
        code, val = ln.split()
        got = oracle.e2m1_value(int(code))
        assert got == float(val) and math.copysign(1, got) == math.copysign(1, float(val)), ln


def test_e4m3_decode_landmarks():
    for ln in _golden_lines("e4m3_points.txt"):
        byte, val = ln.split()
        got = oracle.e4m3_value(int(byte, 16))
        if val == "nan":
            assert math.isnan(got)
        else:
            assert got == float(val) and math.copysign(1, got) == math.copysign(1, float(val))


def test_e4m3_decode_all_codes_match_torch():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    for c in range(256):
        got = oracle.e4m3_value(c)
        if math.isnan(ref[c]):
            assert math.isnan(got)
        else:
            assert got == ref[c] and math.copysign(1, got) == math.copysign(1, ref[c]), c


def _e4m3_table():
    vals = np.array([oracle.e4m3_value(c) for c in range(0x7F)], np.float64)  # 0..448
    return vals


def _brute_round(x, grid, maxval):
    """Nearest grid point by exhaustive distance; exact ties go to the even
    index (= even mantissa, since grid index = code for non-negative codes);
    |x| >= maxval saturates. Returns codes for |x| and the sign separately."""
    a = np.abs(x.astype(np.float64))
    out = np.empty(a.shape, np.int64)
    for s in range(0, a.size, 20000):
        blk = a[s:s + 20000]
        dist = np.abs(blk[:, None] - grid[None, :])
        dmin = dist.min(axis=1, keepdims=True)
        cand = dist == dmin
        idx = np.arange(grid.size)[None, :]
        even = cand & (idx % 2 == 0)
        pick = np.where(even.any(axis=1), np.argmax(even, axis=1), np.argmax(cand, axis=1))
        out[s:s + 20000] = pick
    out[a >= maxval] = grid.size - 1
    return out


def _e4m3_sample(rng):
    grid = _e4m3_table()
    mids = (grid[1:] + grid[:-1]) / 2
    m32 = mids.astype(np.float32)
    xs = [grid, mids, np.nextafter(m32, np.float32(np.inf)), np.nextafter(m32, np.float32(0)),
          np.exp2(rng.uniform(-14, 10, 30000)), rng.uniform(0, 500, 30000),
          np.array([0.0, 2 ** -10, 2 ** -11, 448, 460, 464, 464.0001, 480, 1e30, np.float32(3e38)])]
    x = np.concatenate([np.asarray(v, np.float64) for v in xs]).astype(np.float32)
    return np.concatenate([x, -x])


def test_e4m3_encode_brute_force():
    rng = np.random.default_rng(1)
    x = _e4m3_sample(rng)
    grid = _e4m3_table()
    want = _brute_round(x, grid, 448.0)
    got = np.array([oracle.e4m3_rne_sat(v) for v in x])
    sign = np.signbit(x).astype(np.int64) << 7
    np.testing.assert_array_equal(got, want | sign)


def test_e4m3_encode_matches_torch_in_range():
    rng = np.random.default_rng(2)
    x = _e4m3_sample(rng)
    x = x[np.abs(x) < 464]  # torch turns larger magnitudes into NaN; the oracle saturates
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle.e4m3_rne_sat(v) for v in x])
    np.testing.assert_array_equal(got, ref)


def test_e4m3_encode_saturates():
    for v in [448.0, 464.0, 470.0, 1e6, float("inf")]:
        assert oracle.e4m3_rne_sat(v) == 0x7E
        assert oracle.e4m3_rne_sat(-v) == 0xFE
    assert oracle.e4m3_rne_sat(float("nan")) & 0x7F == 0x7F


def test_e2m1_encode_brute_force():
    grid = np.array([oracle.e2m1_value(c) for c in range(8)])
    assert list(grid) == [0, 0.5, 1, 1.5, 2, 3, 4, 6]
    rng = np.random.default_rng(3)
    mids = (grid[1:] + grid[:-1]) / 2
    m32 = mids.astype(np.float32)
    x = np.concatenate([
        np.arange(-8 * 1024, 8 * 1024 + 1) / 1024.0, mids,
        np.nextafter(m32, np.float32(np.inf)), np.nextafter(m32, np.float32(0)),
        rng.uniform(-7, 7, 20000), [1e-30, 6.0, 6.5, 1e30, float("inf")]]).astype(np.float32)
    x = np.concatenate([x, -x])
    want = _brute_round(x, grid, 6.0)
    sign = np.signbit(x).astype(np.int64) << 3
    got = np.array([oracle.e2m1_rne_sat(v) for v in x])
    np.testing.assert_array_equal(got, want | sign)


def test_e2m1_encode_ties_listed():
    # midpoints of the grid and where they go (even mantissa)
    cases = {0.25: 0, 0.75: 2, 1.25: 2, 1.75: 4, 2.5: 4, 3.5: 6, 5.0: 6, -0.1: 8, -5.0: 14}
    for y, c in cases.items():
        assert oracle.e2m1_rne_sat(y) == c, y


# ---------------------------------------------------------------------------
# Quantiser
# ---------------------------------------------------------------------------

def test_quantize_worked_examples():
    lines = _golden_lines("quant_block_worked.txt")
    assert len(lines) % 4 == 0
    for i in range(0, len(lines), 4):
        x = [float(v) for v in lines[i].split(":")[1].split()]
        scale = int(lines[i + 1].split(":")[1], 16)
        packed = [int(v, 16) for v in lines[i + 3].split(":")[1].split()]
        codes, scales = oracle.quantize_rows(_bf16_bits(x)[None, :])
        assert scales[0, 0] == scale, (x, scales)
        assert list(codes[0]) == packed, (x, [hex(v) for v in codes[0]])


def _spacing(y):
    a = np.abs(y)
    return np.where(a < 2, 0.5, np.where(a < 4, 1.0, 2.0))


def test_quantize_invariants_random_rows():
    rng = np.random.default_rng(4)
    x = rng.standard_normal((64, 512)).astype(np.float32)
    x[::7] *= 20.0
    x[3, 16:32] = 0.0
    bits = _bf16_bits(x)
    xb = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).float().numpy()
    codes, scales = oracle.quantize_rows(bits)
    e2m1 = np.array([oracle.e2m1_value(c) for c in range(16)])
    for r in range(64):
        blocks = xb[r].reshape(32, 16)
        amax = np.abs(blocks).max(axis=1).astype(np.float32)
        t = (amax / np.float32(6.0)).astype(np.float32)
        want_scale = torch.from_numpy(t).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
        np.testing.assert_array_equal(scales[r], want_scale)
        sval = torch.from_numpy(scales[r]).view(torch.float8_e4m3fn).double().numpy()
        c = np.stack([codes[r] & 15, codes[r] >> 4], axis=1).reshape(32, 16)
        v = e2m1[c] * sval[:, None]
        y = blocks / np.where(sval == 0, 1, sval)[:, None]
        ok = np.abs(y) <= 6
        err = np.abs(blocks - v)
        bound = 0.5 * _spacing(y) * sval[:, None]
        assert np.all(err[ok] <= bound[ok] + 0)
        assert np.all(np.abs(v[~ok]) == 6 * np.broadcast_to(sval[:, None], v.shape)[~ok])
    assert np.all(codes[3, 8:16] == 0) and scales[3, 1] == 0


def test_quantize_inf_saturates():
    x = np.zeros(16, np.float32)
    x[0] = np.inf
    x[1] = -np.inf
    x[2] = 100.0
    codes, scales = oracle.quantize_rows(_bf16_bits(x)[None, :])
    assert scales[0, 0] == 0x7E
    assert codes[0, 0] == (7 | (15 << 4))
    assert codes[0, 1] & 15 == 0  # 100/448 < 0.25


def test_physical_row_worked():
    pt = np.array([3, 0, 2], np.int32)
    assert oracle.physical_row(pt, 4, 0) == 12
    assert oracle.physical_row(pt, 4, 3) == 15
    assert oracle.physical_row(pt, 4, 5) == 1
    assert oracle.physical_row(pt, 4, 11) == 11


def test_append_places_rows_through_page_table():
    rng = np.random.default_rng(5)
    d, ps = 32, 4
    page_table = np.array([[2, 0], [1, 3]], np.int32)
    x = rng.standard_normal((3, d)).astype(np.float32)
    bits = _bf16_bits(x)
    codes = np.zeros((16, d // 2), np.uint8)
    scales = np.zeros((16, d // 16), np.uint8)
    seq = np.array([0, 1, 0], np.int32)
    pos = np.array([5, 2, 0], np.int64)
    oracle.append_fp4(bits, seq, pos, page_table, ps, codes, scales)
    want_c, want_s = oracle.quantize_rows(bits)
    for i, row in enumerate([0 * 4 + 1, 1 * 4 + 2, 2 * 4 + 0]):
        np.testing.assert_array_equal(codes[row], want_c[i])
        np.testing.assert_array_equal(scales[row], want_s[i])
    touched = {1, 6, 8}
    for r in range(16):
        if r not in touched:
            assert not codes[r].any() and not scales[r].any()


# ---------------------------------------------------------------------------
# Indexer and Top-k
# ---------------------------------------------------------------------------

def _int_e4m3(vals):
    return torch.tensor(vals, dtype=torch.float32).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def test_index_score_worked():
    lines = _golden_lines("index_score_worked.txt")
    q = _int_e4m3([float(v) for v in lines[0].split(":")[1].split()]).reshape(2, 4)
    w = np.array([float(v) for v in lines[1].split(":")[1].split()], np.float32)
    for ln in lines[2:]:
        lhs, rhs = ln.split(":")[1].split("=")
        k = _int_e4m3([float(v) for v in lhs.split()])
        got = oracle.index_score(q, w, k)
        assert got == float(rhs) and math.copysign(1, got) == 1.0, ln


def test_index_score_single_head_is_relu_dot():
    rng = np.random.default_rng(6)
    for _ in range(50):
        qv = rng.integers(-8, 9, 64)
        kv = rng.integers(-8, 9, 64)
        got = oracle.index_score(_int_e4m3(qv)[None, :], np.ones(1, np.float32), _int_e4m3(kv))
        assert got == max(0, int(np.dot(qv, kv)))


def test_select_topk_brute_force_with_ties():
    rng = np.random.default_rng(7)
    for trial in range(300):
        n = int(rng.integers(0, 64))
        k = int(rng.integers(1, 70))
        s = rng.integers(0, 4, n).astype(np.float64)  # heavy ties
        ids = rng.permutation(1000)[:n].astype(np.int32)
        got, m = oracle.select_topk(s, ids, k)
        order = sorted(range(n), key=lambda i: (-s[i], ids[i]))
        want = [int(ids[i]) for i in order[:k]] + [-1] * max(0, k - n)
        assert list(got) == want
        assert m == min(k, n)


def test_select_topk_all_equal_takes_lowest_ids():
    s = np.zeros(100)
    ids = np.arange(100, dtype=np.int32)[::-1].copy()
    got, _ = oracle.select_topk(s, ids, 10)
    assert list(got) == list(range(10))


def _small_cache(rng, rows, di, d=32):
    kidx = _int_e4m3(rng.integers(-8, 9, rows * di)).reshape(rows, di)
    return kidx


def test_index_full_matches_sorted_scores_paged():
    rng = np.random.default_rng(8)
    hi, di, ps = 3, 16, 8
    page_table = rng.permutation(12).astype(np.int32)
    kidx = _small_cache(rng, 96, di)
    q = _int_e4m3(rng.integers(-8, 9, hi * di)).reshape(hi, di)
    w = rng.integers(1, 5, hi).astype(np.float32)
    n_vis = 90
    topk, pool, sc = oracle.index_full(q, w, kidx, page_table, ps, n_vis, 10, 25, want_scores=True)
    for t in range(n_vis):
        row = page_table[t // ps] * ps + t % ps
        assert sc[t] == oracle.index_score(q, w, kidx[row])
    order = sorted(range(n_vis), key=lambda t: (-sc[t], t))
    assert list(topk) == order[:10]
    assert list(pool) == order[:25]
    assert set(topk) <= set(pool)


def test_reindex_with_full_pool_reproduces_full():
    rng = np.random.default_rng(9)
    hi, di, ps = 4, 32, 16
    page_table = np.arange(8, dtype=np.int32)
    kidx = _small_cache(rng, 128, di)
    q = _int_e4m3(rng.integers(-8, 9, hi * di)).reshape(hi, di)
    w = rng.integers(1, 5, hi).astype(np.float32)
    topk, pool = oracle.index_full(q, w, kidx, page_table, ps, 128, 12, 40)
    # pool = every entry -> Reindex equals Full
    allpool = rng.permutation(128).astype(np.int32)
    assert sorted(oracle.index_reindex(q, w, kidx, page_table, ps, allpool, 12)) == sorted(topk)
    # the Full layer's own pool with the same query -> same Top-k (P >= K)
    assert sorted(oracle.index_reindex(q, w, kidx, page_table, ps, pool, 12)) == sorted(topk)
    # padding entries are ignored
    padded = np.concatenate([pool, -np.ones(9, np.int32)])
    assert sorted(oracle.index_reindex(q, w, kidx, page_table, ps, padded, 12)) == sorted(topk)


def test_index_full_short_sequence_pads():
    rng = np.random.default_rng(10)
    kidx = _small_cache(rng, 16, 16)
    q = _int_e4m3(rng.integers(-8, 9, 16)).reshape(1, 16)
    w = np.ones(1, np.float32)
    topk, pool = oracle.index_full(q, w, kidx, np.arange(1, dtype=np.int32), 16, 5, 8, 10)
    assert sorted(topk[:5]) == [0, 1, 2, 3, 4] and list(topk[5:]) == [-1, -1, -1]
    assert list(pool[5:]) == [-1] * 5


# ---------------------------------------------------------------------------
# Attention
# ---------------------------------------------------------------------------

def _e2m1_golden():
    return np.array([float(ln.split()[1]) for ln in _golden_lines("e2m1_codes.txt")])


def _dequant_indep(codes, scales):
    """FP4 rows -> float64 with the golden E2M1 table and torch's E4M3 decode."""
    tab = _e2m1_golden()
    c = np.stack([codes & 15, codes >> 4], axis=-1).reshape(codes.shape[0], -1)
    s = torch.from_numpy(scales).view(torch.float8_e4m3fn).double().numpy()
    return tab[c] * np.repeat(s, 16, axis=1)


def test_attention_worked_closed_form():
    lines = _golden_lines("attention_worked.txt")
    want = {ln.split(":")[0]: float(ln.split(":")[1]) for ln in lines}
    d = 16
    q = np.zeros((1, d), np.float32)
    q[0, 0] = 2.0
    swa = np.zeros((2, d), np.uint8)
    swa[0, 0] = 0x38
    swa[1, 1] = 0x38
    o, lse = oracle.sparse_attn(_bf16_bits(q), np.zeros((1, 8), np.uint8), np.zeros((1, 1), np.uint8),
                                np.zeros(1, np.int32), 1, np.zeros(0, np.int32), swa, 0.5)
    assert abs(o[0, 0] - want["o0"]) < 1e-15
    assert abs(o[0, 1] - want["o1"]) < 1e-15
    assert np.all(o[0, 2:] == 0)
    assert abs(lse[0] - want["lse"]) < 1e-15


def _attn_case(rng, n_rows=40, d=64, h=4, k=24, nw=7, ps=8):
    x = rng.standard_normal((n_rows, d)).astype(np.float32)
    codes, scales = oracle.quantize_rows(_bf16_bits(x))
    page_table = rng.permutation(n_rows // ps).astype(np.int32)
    topk = rng.permutation(n_rows)[:k].astype(np.int32)
    swa = torch.from_numpy(rng.standard_normal((nw, d)).astype(np.float32)).to(
        torch.float8_e4m3fn).view(torch.uint8).numpy()
    q = _bf16_bits(rng.standard_normal((h, d)).astype(np.float32))
    return q, codes, scales, page_table, topk, swa


def test_attention_matches_torch_dense_softmax():
    rng = np.random.default_rng(11)
    d = 64
    q, codes, scales, pt, topk, swa = _attn_case(rng, d=d)
    topk[3] = -1
    scale = 1.0 / math.sqrt(d)
    o, lse = oracle.sparse_attn(q, codes, scales, pt, 8, topk, swa, scale)
    # independent dense reference: gather the rows by hand, dequantise with the
    # golden table and torch's float8 decode, then torch softmax + matmul
    ps = 8
    rows = [pt[t // ps] * ps + t % ps for t in topk if t >= 0]
    V = np.concatenate([_dequant_indep(codes[rows], scales[rows]),
                        torch.from_numpy(swa).view(torch.float8_e4m3fn).double().numpy()])
    Q = torch.from_numpy(q.view(np.int16)).view(torch.bfloat16).double()
    Vt = torch.from_numpy(V)
    z = scale * Q @ Vt.T
    ref = torch.softmax(z, dim=-1) @ Vt
    np.testing.assert_allclose(o, ref.numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, torch.logsumexp(z, dim=-1).numpy(), rtol=0, atol=1e-12)
    # the softmax weights implied by lse sum to one
    assert np.allclose(torch.exp(z - torch.from_numpy(lse)[:, None]).sum(-1).numpy(), 1.0, atol=1e-12)


def test_attention_all_rows_equal_gives_that_row():
    rng = np.random.default_rng(12)
    d = 32
    x = np.tile(rng.standard_normal((1, d)).astype(np.float32), (16, 1))
    codes, scales = oracle.quantize_rows(_bf16_bits(x))
    u = _dequant_indep(codes[:1], scales[:1])[0]
    q = _bf16_bits(rng.standard_normal((3, d)).astype(np.float32))
    o, _ = oracle.sparse_attn(q, codes, scales, np.arange(1, dtype=np.int32), 16,
                              np.arange(16, dtype=np.int32), None, 0.3)
    np.testing.assert_allclose(o, np.tile(u, (3, 1)), atol=1e-14)


def test_attention_single_entry_and_empty():
    rng = np.random.default_rng(13)
    q, codes, scales, pt, topk, swa = _attn_case(rng)
    one = np.array([-1, 17, -1], np.int32)
    o, lse = oracle.sparse_attn(q, codes, scales, pt, 8, one, None, 0.125)
    row = pt[17 // 8] * 8 + 17 % 8
    v = _dequant_indep(codes[row:row + 1], scales[row:row + 1])[0]
    np.testing.assert_allclose(o, np.tile(v, (q.shape[0], 1)), atol=1e-14)
    o, lse = oracle.sparse_attn(q, codes, scales, pt, 8, -np.ones(4, np.int32), None, 0.125)
    assert np.all(o == 0) and np.all(np.isneginf(lse))


def test_attention_padding_and_order_do_not_matter():
    rng = np.random.default_rng(14)
    q, codes, scales, pt, topk, swa = _attn_case(rng)
    o1, l1 = oracle.sparse_attn(q, codes, scales, pt, 8, topk, swa, 0.2)
    perm = np.concatenate([rng.permutation(topk), -np.ones(5, np.int32)]).astype(np.int32)
    o2, l2 = oracle.sparse_attn(q, codes, scales, pt, 8, perm, swa, 0.2)
    np.testing.assert_allclose(o1, o2, atol=1e-13)
    np.testing.assert_allclose(l1, l2, atol=1e-13)


# ---- NVFP4 variant of the attention ------------------------------------------

def test_nvfp4_round_is_independent_dequant_of_quantiser_and_idempotent():
    rng = np.random.default_rng(15)
    q = _bf16_bits((rng.standard_normal((6, 512)) * np.exp(rng.uniform(-4, 4, (6, 1)))).astype(np.float32))
    r = oracle.nvfp4_round(q)
    codes, scales = oracle.quantize_rows(q)
    want = _bf16_bits(_dequant_indep(codes, scales).astype(np.float32))
    np.testing.assert_array_equal(r, want)
    np.testing.assert_array_equal(oracle.nvfp4_round(r), r)       # already NVFP4 values stay put
    assert np.any(r != q)


def test_attention_nvfp4_is_dense_softmax_of_rounded_q():
    rng = np.random.default_rng(16)
    d = 64
    q, codes, scales, pt, topk, swa = _attn_case(rng, d=d)
    scale = 1.0 / math.sqrt(d)
    o, lse = oracle.sparse_attn_nvfp4(q, codes, scales, pt, 8, topk, swa, scale)
    # independent: q rounded with the independent dequantisation of its codes,
    # rows gathered and dequantised by hand, torch softmax + matmul
    qc, qs = oracle.quantize_rows(q)
    Qh = torch.from_numpy(_dequant_indep(qc, qs))
    rows = [pt[t // 8] * 8 + t % 8 for t in topk if t >= 0]
    V = torch.from_numpy(np.concatenate([_dequant_indep(codes[rows], scales[rows]),
                                         torch.from_numpy(swa).view(torch.float8_e4m3fn).double().numpy()]))
    z = scale * Qh @ V.T
    np.testing.assert_allclose(o, (torch.softmax(z, dim=-1) @ V).numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, torch.logsumexp(z, dim=-1).numpy(), rtol=0, atol=1e-12)
    # the quantised q changes the result; a q that is already NVFP4 does not
    o_exact, _ = oracle.sparse_attn(q, codes, scales, pt, 8, topk, swa, scale)
    assert np.abs(o - o_exact).max() > 1e-4
    qn = oracle.nvfp4_round(q)
    o1, l1 = oracle.sparse_attn_nvfp4(qn, codes, scales, pt, 8, topk, swa, scale)
    o2, l2 = oracle.sparse_attn(qn, codes, scales, pt, 8, topk, swa, scale)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(l1, l2)


# ---- FP8 appends (window rows, indexer keys) --------------------------------

def _all_bf16():
    return np.arange(65536, dtype=np.uint32).astype(np.uint16)


def test_e4m3_row_matches_torch_cast_in_range_and_saturates():
    bits = _all_bf16()
    got = oracle.e4m3_row(bits)
    x = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).float()
    a = x.abs()
    finite = torch.isfinite(x)
    # inside the representable range torch's (non-saturating) cast is the RNE reference
    inside = finite & (a < 464.0)
    ref = x[inside].to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(got[inside.numpy()], ref)
    # saturation: |x| >= 464 (incl. infinities) -> +-448
    sat = (~torch.isnan(x)) & (a >= 464.0)
    sign = (bits >> 15).astype(np.uint8)
    np.testing.assert_array_equal(got[sat.numpy()], (0x7E | (sign << 7))[sat.numpy()])
    # NaN keeps its sign and becomes 0x7F
    nan = torch.isnan(x).numpy()
    np.testing.assert_array_equal(got[nan], (0x7F | (sign << 7))[nan])


def test_e4m3_row_worked_example():
    x = np.array([1.0, -2.5, 448.0, 500.0, 0.0, 0.001953125, 3.3, -0.0], np.float32)
    got = oracle.e4m3_row(_bf16_bits(x[None, :])[0])
    # 1 = 0x38; -2.5 = 1|1000|010; 448 = 0x7E; 500 saturates; 0; 2^-9 = smallest subnormal;
    # bf16(3.3) = 3.296875 -> 3.25 = 0|1000|101; -0 keeps its sign
    assert [int(v) for v in got] == [0x38, 0xC2, 0x7E, 0x7E, 0x00, 0x01, 0x45, 0x80]


def test_append_swa_ring_slots():
    rng = np.random.default_rng(31)
    ring, b = 7, 3
    swa = np.full((b, ring, 512), 0xAA, np.uint8)
    seq = np.array([0, 2, 2, 1], np.int32)
    pos = np.array([3, 6, 7, 15], np.int64)         # 7 wraps to slot 0, 15 to slot 1
    x = _bf16_bits(rng.standard_normal((4, 512)).astype(np.float32))
    oracle.append_swa_e4m3(x, seq, pos, swa)
    want = np.full_like(swa, 0xAA)
    for i in range(4):
        want[seq[i], pos[i] % ring] = oracle.e4m3_row(x[i])
    np.testing.assert_array_equal(swa, want)


def test_append_kidx_paged():
    rng = np.random.default_rng(32)
    ps, di = 4, 64
    pt = np.array([[5, 2, 7], [0, 3, 6]], np.int32)
    kidx = np.zeros((8 * ps, di), np.uint8)
    seq = np.array([0, 1, 0], np.int32)
    pos = np.array([5, 9, 11], np.int64)             # rows 2*4+1, 6*4+1, 7*4+3
    x = _bf16_bits(rng.standard_normal((3, di)).astype(np.float32))
    oracle.append_kidx_e4m3(x, seq, pos, pt, ps, kidx)
    want = np.zeros_like(kidx)
    for i, row in enumerate([9, 25, 31]):
        want[row] = oracle.e4m3_row(x[i])
    np.testing.assert_array_equal(kidx, want)
