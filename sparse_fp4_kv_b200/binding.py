"""Python binding of libcsa2.so: the C-ABI calls under the same names.

Argument marshalling only: torch tensors are turned into device pointers and
sizes, the caller's current CUDA stream is passed along, and a non-OK status
raises. Every step of the computation runs in the library's kernels; there is
no fallback of any kind. If the library is missing the import fails.
"""
import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libcsa2.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is not built; run `python -m sparse_fp4_kv_b200.build` (nvcc, sm_100a)")

_lib = ctypes.CDLL(LIB_PATH)

CSA2_D = 512
CSA2_ATTN_STATIC_SCRATCH_BYTES = 16 << 20
STATUS = {0: "ok", 1: "invalid argument", 2: "unsupported configuration",
          3: "workspace missing or too small", 4: "CUDA error", 5: "device-side error recorded"}


class Csa2Error(RuntimeError):
    def __init__(self, call, status):
        super().__init__(f"{call}: {STATUS.get(status, status)} (status {status})")
        self.status = status


class csa2_kv_desc(ctypes.Structure):
    _fields_ = [
        ("codes", ctypes.c_void_p),
        ("scales", ctypes.c_void_p),
        ("kidx", ctypes.c_void_p),
        ("page_table", ctypes.c_void_p),
        ("seq_len", ctypes.c_void_p),
        ("rows_cap", ctypes.c_int64),
        ("d", ctypes.c_int32),
        ("di", ctypes.c_int32),
        ("page_size", ctypes.c_int32),
        ("max_pages", ctypes.c_int32),
        ("batch", ctypes.c_int32),
        ("reserved", ctypes.c_int32),
    ]


_vp, _i32, _i64, _sz, _f32 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t, ctypes.c_float
_kvp = ctypes.POINTER(csa2_kv_desc)
_SIGS = {
    "csa2_append_fp4": (_i32, [_vp, _i32, _vp, _vp, _kvp, _vp]),
    "csa2_index_full": (_i32, [_vp, _vp, _i32, _i32, _i32, _vp, _i64, _kvp, _i32, _i32, _vp, _vp, _vp, _sz,
                               _vp]),
    "csa2_append_swa_e4m3": (_i32, [_vp, _i32, _vp, _vp, _vp, _i32, _i64, _vp]),
    "csa2_append_kidx_e4m3": (_i32, [_vp, _i32, _vp, _vp, _kvp, _vp]),
    "csa2_index_full_workspace_size": (_sz, [_i32, _i64]),
    "csa2_index_reindex": (_i32, [_vp, _vp, _i32, _i32, _i32, _vp, _i32, _kvp, _i32, _vp, _vp, _sz, _vp]),
    "csa2_index_reindex_workspace_size": (_sz, [_i32, _i32]),
    "csa2_sparse_attn_decode": (_i32, [_vp, _i32, _i32, _i32, _kvp, _vp, _i32, _vp, _i64, _vp, _vp, _i32,
                                       _f32, _vp, _vp, _vp, _sz, _vp]),
    "csa2_sparse_attn_workspace_size": (_sz, [_i32, _i32, _i32, _i32]),
    "csa2_sparse_attn_decode_nvfp4": (_i32, [_vp, _i32, _i32, _i32, _kvp, _vp, _i32, _vp, _i64, _vp, _vp, _i32,
                                             _f32, _vp, _vp, _vp, _sz, _vp]),
    "csa2_sparse_attn_nvfp4_workspace_size": (_sz, [_i32, _i32, _i32, _i32]),
    "csa2_sparse_attn_decode_static": (_i32, [_vp, _i32, _i32, _i32, _kvp, _vp, _i32, _vp, _i64, _vp, _vp, _i32,
                                              _f32, _vp, _vp, _vp]),
    "csa2_score_ids": (_i32, [_vp, _vp, _i32, _i32, _i32, _vp, _i32, _kvp, _i32, _vp, _vp]),
    "csa2_select_keys": (_i32, [_vp, _i32, _i32, _i32, _vp, _vp]),
    "csa2_sparse_attn_partial": (_i32, [_vp, _i32, _i32, _i32, _kvp, _vp, _i32, _vp, _i64, _vp, _vp, _i32,
                                        _f32, _vp, _vp, _vp, _sz, _vp]),
    "csa2_attn_merge": (_i32, [_vp, _vp, _i32, _i32, _i32, _vp, _vp, _vp]),
    "csa2_device_status": (_i32, [_vp, ctypes.POINTER(ctypes.c_uint32)]),
    "csa2_check_wait_timeout": (_i32, [ctypes.c_uint32, _vp]),
    "csa2_status_string": (ctypes.c_char_p, [_i32]),
    "csa2_version": (_i32, []),
}
for _name, (_res, _args) in _SIGS.items():
    _fn = getattr(_lib, _name)
    _fn.restype = _res
    _fn.argtypes = _args

EXPORTED = tuple(_SIGS)


def _ptr(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("device tensor expected")
    if not t.is_contiguous():
        raise ValueError("contiguous tensor expected")
    return t.data_ptr()


def _stream(stream):
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _check(call, st):
    if st != 0:
        raise Csa2Error(call, st)


class KvCache:
    """The shared global KV cache: torch tensors plus the C descriptor.

    codes [rows_cap, 256] u8, scales [rows_cap, 32] u8, kidx [rows_cap, di] u8,
    page_table [batch, max_pages] i32, seq_len [batch] i32 (all on the device).
    """

    def __init__(self, codes, scales, kidx, page_table, seq_len, page_size):
        self.codes, self.scales, self.kidx = codes, scales, kidx
        self.page_table, self.seq_len = page_table, seq_len
        self.page_size = int(page_size)
        d = ctypes.pointer(csa2_kv_desc())
        d.contents.codes = _ptr(codes)
        d.contents.scales = _ptr(scales)
        d.contents.kidx = _ptr(kidx) if kidx is not None else None
        d.contents.page_table = _ptr(page_table)
        d.contents.seq_len = _ptr(seq_len)
        d.contents.rows_cap = codes.shape[0]
        d.contents.d = CSA2_D
        d.contents.di = kidx.shape[1] if kidx is not None else 0
        d.contents.page_size = self.page_size
        d.contents.max_pages = page_table.shape[1]
        d.contents.batch = page_table.shape[0]
        self.desc = d

    @property
    def di(self):
        return self.desc.contents.di


def csa2_append_fp4(x_bf16, seq, pos, kv: KvCache, stream=None):
    n = x_bf16.shape[0] if x_bf16.dim() == 2 else 0
    _check("csa2_append_fp4", _lib.csa2_append_fp4(_ptr(x_bf16), n, _ptr(seq), _ptr(pos), kv.desc,
                                                   _stream(stream)))


def csa2_index_full_workspace_size(nq, n_max):
    return _lib.csa2_index_full_workspace_size(nq, n_max)


def csa2_index_full(qidx, w, q_per_seq, q_limit, n_max, kv: KvCache, k, p, topk, pool, ws, stream=None):
    nq, hi = qidx.shape[0], qidx.shape[1]
    _check("csa2_index_full", _lib.csa2_index_full(
        _ptr(qidx), _ptr(w), nq, q_per_seq, hi, _ptr(q_limit), int(n_max), kv.desc, k, p, _ptr(topk),
        _ptr(pool), _ptr(ws), ws.numel() * ws.element_size() if ws is not None else 0, _stream(stream)))


def csa2_index_reindex_workspace_size(nq, p):
    return _lib.csa2_index_reindex_workspace_size(nq, p)


def csa2_index_reindex(qidx, w, q_per_seq, pool, kv: KvCache, k, topk, ws, stream=None):
    nq, hi = qidx.shape[0], qidx.shape[1]
    p = pool.shape[1]
    _check("csa2_index_reindex", _lib.csa2_index_reindex(
        _ptr(qidx), _ptr(w), nq, q_per_seq, hi, _ptr(pool), p, kv.desc, k, _ptr(topk), _ptr(ws),
        ws.numel() * ws.element_size() if ws is not None else 0, _stream(stream)))


def csa2_sparse_attn_workspace_size(nq, h, k, w_max):
    return _lib.csa2_sparse_attn_workspace_size(nq, h, k, w_max)


def csa2_sparse_attn_decode(q_bf16, q_per_seq, kv: KvCache, topk, swa, swa_seq_stride, swa_begin, swa_end,
                            w_max, softmax_scale, o_bf16, lse, ws, stream=None):
    nq, h = q_bf16.shape[0], q_bf16.shape[1]
    k = topk.shape[1] if topk is not None else 0
    _check("csa2_sparse_attn_decode", _lib.csa2_sparse_attn_decode(
        _ptr(q_bf16), nq, q_per_seq, h, kv.desc, _ptr(topk), k, _ptr(swa), int(swa_seq_stride),
        _ptr(swa_begin), _ptr(swa_end), int(w_max), float(softmax_scale), _ptr(o_bf16), _ptr(lse),
        _ptr(ws), ws.numel() * ws.element_size() if ws is not None else 0, _stream(stream)))


def csa2_sparse_attn_decode_static(q_bf16, q_per_seq, kv: KvCache, topk, swa, swa_seq_stride, swa_begin, swa_end,
                                   w_max, softmax_scale, o_bf16, lse, stream=None):
    """csa2_sparse_attn_decode with the library's fixed device scratch
    (CSA2_ATTN_STATIC_SCRATCH_BYTES) in place of a caller workspace, for
    callers that cannot allocate device memory. Calls whose kernels can
    overlap on one device share that scratch and race."""
    nq, h = q_bf16.shape[0], q_bf16.shape[1]
    k = topk.shape[1] if topk is not None else 0
    _check("csa2_sparse_attn_decode_static", _lib.csa2_sparse_attn_decode_static(
        _ptr(q_bf16), nq, q_per_seq, h, kv.desc, _ptr(topk), k, _ptr(swa), int(swa_seq_stride),
        _ptr(swa_begin), _ptr(swa_end), int(w_max), float(softmax_scale), _ptr(o_bf16), _ptr(lse),
        _stream(stream)))


def csa2_sparse_attn_nvfp4_workspace_size(nq, h, k, w_max):
    return _lib.csa2_sparse_attn_nvfp4_workspace_size(nq, h, k, w_max)


def csa2_sparse_attn_decode_nvfp4(q_bf16, q_per_seq, kv: KvCache, topk, swa, swa_seq_stride, swa_begin, swa_end,
                                  w_max, softmax_scale, o_bf16, lse, ws, stream=None):
    """csa2_sparse_attn_decode with q quantised to NVFP4 for the scores (FP4
    block-scaled products on the selected entries); h = 64."""
    nq, h = q_bf16.shape[0], q_bf16.shape[1]
    k = topk.shape[1] if topk is not None else 0
    _check("csa2_sparse_attn_decode_nvfp4", _lib.csa2_sparse_attn_decode_nvfp4(
        _ptr(q_bf16), nq, q_per_seq, h, kv.desc, _ptr(topk), k, _ptr(swa), int(swa_seq_stride),
        _ptr(swa_begin), _ptr(swa_end), int(w_max), float(softmax_scale), _ptr(o_bf16), _ptr(lse),
        _ptr(ws), ws.numel() * ws.element_size() if ws is not None else 0, _stream(stream)))


def csa2_append_swa_e4m3(x_bf16, seq, pos, swa, stream=None):
    """Window rows x [n][512] into ring slots pos % ring_rows of swa [batch][ring_rows][512]."""
    _check("csa2_append_swa_e4m3", _lib.csa2_append_swa_e4m3(
        _ptr(x_bf16), x_bf16.shape[0], _ptr(seq), _ptr(pos), _ptr(swa), swa.shape[0], swa.shape[1],
        _stream(stream)))


def csa2_append_kidx_e4m3(x_bf16, seq, pos, kv: KvCache, stream=None):
    """Indexer keys x [n][di] into the physical rows of (seq, pos) of the key array."""
    _check("csa2_append_kidx_e4m3", _lib.csa2_append_kidx_e4m3(
        _ptr(x_bf16), x_bf16.shape[0], _ptr(seq), _ptr(pos), kv.desc, _stream(stream)))


def csa2_score_ids(qidx, w, q_per_seq, ids, kv: KvCache, id_offset, keys, stream=None):
    """Unique 64-bit keys (score key << 32 | ~(id + id_offset)) of ids [nq][m] (local to kv)."""
    nq, hi = qidx.shape[0], qidx.shape[1]
    _check("csa2_score_ids", _lib.csa2_score_ids(_ptr(qidx), _ptr(w), nq, q_per_seq, hi, _ptr(ids), ids.shape[1],
                                                 kv.desc, int(id_offset), _ptr(keys), _stream(stream)))


def csa2_select_keys(keys, k, ids, stream=None):
    """The ids carried by the k largest of each query's keys [nq][m] (padded with -1)."""
    _check("csa2_select_keys", _lib.csa2_select_keys(_ptr(keys), keys.shape[0], keys.shape[1], int(k), _ptr(ids),
                                                     _stream(stream)))


def csa2_sparse_attn_partial(q_bf16, q_per_seq, kv: KvCache, topk, swa, swa_seq_stride, swa_begin, swa_end,
                             w_max, softmax_scale, o_f32, lse, ws, stream=None):
    nq, h = q_bf16.shape[0], q_bf16.shape[1]
    k = topk.shape[1] if topk is not None else 0
    _check("csa2_sparse_attn_partial", _lib.csa2_sparse_attn_partial(
        _ptr(q_bf16), nq, q_per_seq, h, kv.desc, _ptr(topk), k, _ptr(swa), int(swa_seq_stride),
        _ptr(swa_begin), _ptr(swa_end), int(w_max), float(softmax_scale), _ptr(o_f32), _ptr(lse),
        _ptr(ws), ws.numel() * ws.element_size() if ws is not None else 0, _stream(stream)))


def csa2_attn_merge(o_parts, lse_parts, o_bf16, lse, stream=None):
    """Merge g partials o_parts [g][nq][h][512] f32, lse_parts [g][nq][h] into bf16 o and lse."""
    g, nq, h = o_parts.shape[0], o_parts.shape[1], o_parts.shape[2]
    _check("csa2_attn_merge", _lib.csa2_attn_merge(_ptr(o_parts), _ptr(lse_parts), g, nq, h, _ptr(o_bf16), _ptr(lse),
                                                   _stream(stream)))


def csa2_device_status(stream=None):
    code = ctypes.c_uint32(0)
    st = _lib.csa2_device_status(_stream(stream), ctypes.byref(code))
    if st not in (0, 5):
        raise Csa2Error("csa2_device_status", st)
    return code.value


def csa2_check_wait_timeout(limit_us, stream=None):
    """Launch the bounded-wait self-check (a wait that runs out after limit_us)."""
    _check("csa2_check_wait_timeout", _lib.csa2_check_wait_timeout(int(limit_us), _stream(stream)))


def csa2_status_string(status):
    return _lib.csa2_status_string(status).decode()


def csa2_version():
    return _lib.csa2_version()


def workspace(nbytes, device):
    """A device byte buffer (256-byte aligned by the caching allocator)."""
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)
