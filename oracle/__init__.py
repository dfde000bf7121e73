"""ctypes front end of the plain CPU oracle (oracle/csa2_oracle.c).

TEST INFRASTRUCTURE. Only tests/, the smoke check in __graft_entry__.py and
the CPU-baseline leg of bench.py may import this package. The CUDA library
and its Python binding never import it, and it imports nothing from them.

Each function wraps one C function of the oracle and works on numpy arrays.
Loops over independent (sequence, query) units stay in Python; the inner
arithmetic is the C definition.
"""
import ctypes
import os

import numpy as np

from . import build as _build

_LIB = None


def lib():
    """Load (building if needed) the oracle library."""
    global _LIB
    if _LIB is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        c_u8p = ctypes.POINTER(ctypes.c_uint8)
        c_u16p = ctypes.POINTER(ctypes.c_uint16)
        c_i32p = ctypes.POINTER(ctypes.c_int32)
        c_i64p = ctypes.POINTER(ctypes.c_int64)
        c_f32p = ctypes.POINTER(ctypes.c_float)
        c_f64p = ctypes.POINTER(ctypes.c_double)
        i32, i64 = ctypes.c_int32, ctypes.c_int64
        sig = {
            "orc_e2m1_value": (ctypes.c_double, [ctypes.c_uint32]),
            "orc_e4m3_value": (ctypes.c_double, [ctypes.c_uint32]),
            "orc_e4m3_rne_sat": (ctypes.c_uint32, [ctypes.c_float]),
            "orc_e2m1_rne_sat": (ctypes.c_uint32, [ctypes.c_float]),
            "orc_quantize_block16": (None, [c_u16p, c_u8p, c_u8p]),
            "orc_quantize_row": (None, [c_u16p, i32, c_u8p, c_u8p]),
            "orc_physical_row": (i64, [c_i32p, i32, i64]),
            "orc_append_fp4": (None, [c_u16p, i32, i32, c_i32p, c_i64p, c_i32p, i32, i32,
                                      c_u8p, c_u8p]),
            "orc_index_score": (ctypes.c_double, [c_u8p, c_f32p, i32, i32, c_u8p]),
            "orc_select_topk": (i32, [c_f64p, c_i32p, i64, i32, c_i32p]),
            "orc_index_full": (None, [c_u8p, c_f32p, i32, i32, c_u8p, c_i32p, i32, i64, i32, i32,
                                      c_i32p, c_i32p, c_f64p]),
            "orc_index_reindex": (None, [c_u8p, c_f32p, i32, i32, c_u8p, c_i32p, i32, c_i32p,
                                         i32, i32, c_i32p]),
            "orc_sparse_attn": (None, [c_u16p, i32, i32, c_u8p, c_u8p, c_i32p, i32, c_i32p, i32,
                                       c_u8p, i32, ctypes.c_double, c_f64p, c_f64p]),
            "orc_dequant_row": (None, [c_u8p, c_u8p, i32, c_f64p]),
            "orc_e4m3_row": (None, [c_u16p, i32, c_u8p]),
            "orc_append_swa_e4m3": (None, [c_u16p, i32, c_i32p, c_i64p, i64, c_u8p]),
            "orc_append_kidx_e4m3": (None, [c_u16p, i32, i32, c_i32p, c_i64p, c_i32p, i32, i32, c_u8p]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _LIB = L
    return _LIB


def _p(a, ctype):
    """Pointer to the data of a C-contiguous numpy array (None passes NULL)."""
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data_as(ctypes.POINTER(ctype))


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


# ---- number formats -------------------------------------------------------

def e2m1_value(code):
    return lib().orc_e2m1_value(int(code))


def e4m3_value(byte):
    return lib().orc_e4m3_value(int(byte))


def e4m3_rne_sat(x):
    return lib().orc_e4m3_rne_sat(float(np.float32(x)))


def e2m1_rne_sat(y):
    return lib().orc_e2m1_rne_sat(float(np.float32(y)))


# ---- quantiser / cache ----------------------------------------------------

def quantize_rows(x_bf16_bits):
    """x: uint16 [n, d] raw bf16 bits -> (codes uint8 [n, d/2], scales uint8 [n, d/16])."""
    x = _c(x_bf16_bits, np.uint16)
    n, d = x.shape
    codes = np.zeros((n, d // 2), np.uint8)
    scales = np.zeros((n, d // 16), np.uint8)
    L = lib()
    for i in range(n):
        L.orc_quantize_row(_p(x[i], ctypes.c_uint16), d, _p(codes[i], ctypes.c_uint8),
                           _p(scales[i], ctypes.c_uint8))
    return codes, scales


def physical_row(page_table_seq, page_size, t):
    pt = _c(page_table_seq, np.int32)
    return lib().orc_physical_row(_p(pt, ctypes.c_int32), int(page_size), int(t))


def append_fp4(x_bf16_bits, seq, pos, page_table, page_size, codes, scales):
    """Quantise rows of x and store them in the (paged) cache arrays in place."""
    x = _c(x_bf16_bits, np.uint16)
    n, d = x.shape
    seq = _c(seq, np.int32)
    pos = _c(pos, np.int64)
    pt = _c(page_table, np.int32)
    assert codes.dtype == np.uint8 and scales.dtype == np.uint8
    assert codes.flags["C_CONTIGUOUS"] and scales.flags["C_CONTIGUOUS"]
    lib().orc_append_fp4(_p(x, ctypes.c_uint16), n, d, _p(seq, ctypes.c_int32),
                         _p(pos, ctypes.c_int64), _p(pt, ctypes.c_int32), pt.shape[1],
                         int(page_size), _p(codes, ctypes.c_uint8), _p(scales, ctypes.c_uint8))


def e4m3_row(x_bf16_bits):
    """bf16 bits [width] -> E4M3 codes [width] (RNE, saturating, no scale)."""
    x = _c(x_bf16_bits, np.uint16).reshape(-1)
    out = np.zeros(x.shape[0], np.uint8)
    lib().orc_e4m3_row(_p(x, ctypes.c_uint16), x.shape[0], _p(out, ctypes.c_uint8))
    return out


def append_swa_e4m3(x_bf16_bits, seq, pos, swa):
    """Window rows into the ring buffer swa [batch][ring_rows][512] in place."""
    x = _c(x_bf16_bits, np.uint16)
    n = x.shape[0]
    seq = _c(seq, np.int32)
    pos = _c(pos, np.int64)
    assert swa.dtype == np.uint8 and swa.flags["C_CONTIGUOUS"] and swa.shape[2] == 512
    lib().orc_append_swa_e4m3(_p(x, ctypes.c_uint16), n, _p(seq, ctypes.c_int32), _p(pos, ctypes.c_int64),
                              swa.shape[1], _p(swa, ctypes.c_uint8))


def append_kidx_e4m3(x_bf16_bits, seq, pos, page_table, page_size, kidx):
    """Indexer keys into the (paged) key array kidx [rows][di] in place."""
    x = _c(x_bf16_bits, np.uint16)
    n, di = x.shape
    seq = _c(seq, np.int32)
    pos = _c(pos, np.int64)
    pt = _c(page_table, np.int32)
    assert kidx.dtype == np.uint8 and kidx.flags["C_CONTIGUOUS"] and kidx.shape[1] == di
    lib().orc_append_kidx_e4m3(_p(x, ctypes.c_uint16), n, di, _p(seq, ctypes.c_int32), _p(pos, ctypes.c_int64),
                               _p(pt, ctypes.c_int32), pt.shape[1], int(page_size), _p(kidx, ctypes.c_uint8))


def dequant_row(codes_row, scales_row):
    c = _c(codes_row, np.uint8)
    s = _c(scales_row, np.uint8)
    d = c.shape[0] * 2
    out = np.zeros(d, np.float64)
    lib().orc_dequant_row(_p(c, ctypes.c_uint8), _p(s, ctypes.c_uint8), d,
                          _p(out, ctypes.c_double))
    return out


# ---- indexer ----------------------------------------------------------------

def index_score(q, w, k_row):
    q = _c(q, np.uint8)
    hi, di = q.shape
    w = _c(w, np.float32)
    k_row = _c(k_row, np.uint8)
    return lib().orc_index_score(_p(q, ctypes.c_uint8), _p(w, ctypes.c_float), hi, di,
                                 _p(k_row, ctypes.c_uint8))


def select_topk(scores, ids, k):
    s = _c(scores, np.float64)
    i = _c(ids, np.int32)
    out = np.full(k, -1, np.int32)
    m = lib().orc_select_topk(_p(s, ctypes.c_double), _p(i, ctypes.c_int32), s.shape[0], int(k),
                              _p(out, ctypes.c_int32))
    return out, m


def index_full(qidx, w, kidx, page_table_seq, page_size, n_visible, k, p, want_scores=False):
    """One query: qidx uint8 [hi, di], w float32 [hi], kidx uint8 [rows, di]."""
    q = _c(qidx, np.uint8)
    hi, di = q.shape
    w = _c(w, np.float32)
    kx = _c(kidx, np.uint8)
    pt = _c(page_table_seq, np.int32)
    topk = np.full(k, -1, np.int32)
    pool = np.full(max(p, 1), -1, np.int32)
    sc = np.zeros(max(int(n_visible), 1), np.float64) if want_scores else None
    lib().orc_index_full(_p(q, ctypes.c_uint8), _p(w, ctypes.c_float), hi, di,
                         _p(kx, ctypes.c_uint8), _p(pt, ctypes.c_int32), int(page_size),
                         int(n_visible), int(k), int(p), _p(topk, ctypes.c_int32),
                         _p(pool, ctypes.c_int32) if p > 0 else None,
                         _p(sc, ctypes.c_double) if sc is not None else None)
    res = (topk, pool[:p] if p > 0 else None)
    if want_scores:
        res = res + (sc[: int(n_visible)],)
    return res


def index_reindex(qidx, w, kidx, page_table_seq, page_size, pool, k):
    q = _c(qidx, np.uint8)
    hi, di = q.shape
    w = _c(w, np.float32)
    kx = _c(kidx, np.uint8)
    pt = _c(page_table_seq, np.int32)
    pl = _c(pool, np.int32)
    topk = np.full(k, -1, np.int32)
    lib().orc_index_reindex(_p(q, ctypes.c_uint8), _p(w, ctypes.c_float), hi, di,
                            _p(kx, ctypes.c_uint8), _p(pt, ctypes.c_int32), int(page_size),
                            _p(pl, ctypes.c_int32), pl.shape[0], int(k), _p(topk, ctypes.c_int32))
    return topk


# ---- attention --------------------------------------------------------------

def sparse_attn(q_bf16_bits, codes, scales, page_table_seq, page_size, topk, swa_rows,
                softmax_scale):
    """One query: q uint16 [h, d]; swa_rows uint8 [nw, d]. Returns (o [h, d], lse [h]) in f64."""
    q = _c(q_bf16_bits, np.uint16)
    h, d = q.shape
    c = _c(codes, np.uint8)
    s = _c(scales, np.uint8)
    pt = _c(page_table_seq, np.int32)
    tk = _c(topk, np.int32)
    sw = _c(swa_rows, np.uint8).reshape(-1, d) if swa_rows is not None else np.zeros((0, d), np.uint8)
    o = np.zeros((h, d), np.float64)
    lse = np.zeros(h, np.float64)
    lib().orc_sparse_attn(_p(q, ctypes.c_uint16), h, d, _p(c, ctypes.c_uint8),
                          _p(s, ctypes.c_uint8), _p(pt, ctypes.c_int32), int(page_size),
                          _p(tk, ctypes.c_int32), tk.shape[0],
                          _p(sw, ctypes.c_uint8) if sw.shape[0] else None, sw.shape[0],
                          float(softmax_scale), _p(o, ctypes.c_double), _p(lse, ctypes.c_double))
    return o, lse


def nvfp4_round(x_bf16_bits):
    """Rows of bf16 bits [n, d] -> bf16 bits of their NVFP4 quantise-then-
    dequantise (the block quantiser above, then code value x scale value).
    Every such value has at most 6 significant bits and lies in
    [2^-10, 2688], so it is exact in bf16."""
    x = _c(x_bf16_bits, np.uint16)
    codes, scales = quantize_rows(x)
    out = np.zeros_like(x)
    for i in range(x.shape[0]):
        v = dequant_row(codes[i], scales[i]).astype(np.float32)
        bits = v.view(np.uint32)
        assert np.all((bits & 0xFFFF) == 0), "NVFP4 value not exact in bf16"
        out[i] = (bits >> 16).astype(np.uint16)
    return out


def sparse_attn_nvfp4(q_bf16_bits, codes, scales, page_table_seq, page_size, topk, swa_rows, softmax_scale):
    """The NVFP4 variant of the decode attention: the scores of every row use
    q after NVFP4 quantisation (nvfp4_round); keys, values and softmax as in
    sparse_attn."""
    return sparse_attn(nvfp4_round(q_bf16_bits), codes, scales, page_table_seq, page_size, topk, swa_rows,
                       softmax_scale)
