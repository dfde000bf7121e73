"""Host-side checks of the C-ABI library (no GPU needed): it loads, exports
every function include/csa2.h declares, and rejects bad arguments on the host
before anything is launched."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def binding():
    from sparse_fp4_kv_b200 import build
    build.build()
    from sparse_fp4_kv_b200 import binding as b
    return b


def _declared():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names |= set(re.findall(r"\b(csa2_\w+)\s*\(", src))
    return names


def test_exports_every_declared_symbol(binding):
    declared = _declared()
    assert {"csa2_append_fp4", "csa2_index_full", "csa2_index_reindex", "csa2_sparse_attn_decode"} <= declared
    lib = ctypes.CDLL(binding.LIB_PATH)
    for name in sorted(declared):
        assert hasattr(lib, name), name
    assert declared <= set(binding.EXPORTED)


def test_library_needs_no_cuda_runtime_at_load(binding):
    # statically linked runtime: the library must load on a host without GPU
    lib = ctypes.CDLL(binding.LIB_PATH)
    assert lib.csa2_version() == binding.csa2_version()


def test_status_strings(binding):
    for s in range(6):
        assert binding.csa2_status_string(s) == binding.STATUS[s]


def test_workspace_sizes_monotone(binding):
    a = binding.csa2_index_full_workspace_size(8, 65536)
    b = binding.csa2_index_full_workspace_size(8, 131072)
    assert 0 < a < b
    assert a >= 8 * 65536 * 4
    assert binding.csa2_index_full_workspace_size(0, 10) == 0
    assert binding.csa2_index_reindex_workspace_size(8, 4096) >= 8 * 4096 * 8
    assert binding.csa2_sparse_attn_workspace_size(0, 64, 2048, 512) == 0


def _desc(binding, **kw):
    d = binding.csa2_kv_desc()
    d.codes = kw.get("codes", 0x10000)
    d.scales = kw.get("scales", 0x20000)
    d.kidx = kw.get("kidx", 0x30000)
    d.page_table = kw.get("page_table", 0x40000)
    d.seq_len = kw.get("seq_len", 0x50000)
    d.rows_cap = kw.get("rows_cap", 4096)
    d.d = kw.get("d", 512)
    d.di = kw.get("di", 64)
    d.page_size = kw.get("page_size", 4096)
    d.max_pages = kw.get("max_pages", 1)
    d.batch = kw.get("batch", 1)
    return ctypes.pointer(d)


def test_host_validation_rejects_before_launch(binding):
    L = binding._lib
    # unsupported latent width
    assert L.csa2_append_fp4(0x1000, 4, 0x2000, 0x3000, _desc(binding, d=256), None) == 2
    # null descriptor
    assert L.csa2_append_fp4(0x1000, 4, 0x2000, 0x3000, None, None) == 1
    # misaligned input rows
    assert L.csa2_append_fp4(0x1001, 4, 0x2000, 0x3000, _desc(binding), None) == 1
    # n = 0 is a no-op
    assert L.csa2_append_fp4(0x1000, 0, 0x2000, 0x3000, _desc(binding), None) == 0
    # bad page size
    assert L.csa2_append_fp4(0x1000, 4, 0x2000, 0x3000, _desc(binding, page_size=48), None) == 2
    # Full: di unsupported, hi out of range, p < k, missing workspace
    args = lambda **kw: (0x1000, 0x2000, 1, 1, kw.get("hi", 4), None, 4096, _desc(binding, **kw.get("kv", {})),
                         kw.get("k", 8), kw.get("p", 0), 0x3000, kw.get("pool", None), kw.get("ws", None),
                         kw.get("wsb", 0), None)
    assert L.csa2_index_full(*args(kv={"di": 32})) == 2
    assert L.csa2_index_full(*args(hi=17)) == 2
    assert L.csa2_index_full(*args(p=4, pool=0x4000)) == 1
    assert L.csa2_index_full(*args()) == 3
    # pool pointer without pool size
    assert L.csa2_index_full(*args(pool=0x4000)) == 1
    # Reindex: pool too large
    assert L.csa2_index_reindex(0x1000, 0x2000, 1, 1, 4, 0x3000, 20000, _desc(binding), 8, 0x4000, 0x5000,
                                1 << 30, None) == 2
    # attention: unsupported head count, window without begin/end
    assert L.csa2_sparse_attn_decode(0x1000, 1, 1, 48, _desc(binding), 0x2000, 8, None, 0, None, None, 0, 0.1,
                                     0x3000, None, None, 0, None) == 2
    assert L.csa2_sparse_attn_decode(0x1000, 1, 1, 64, _desc(binding), 0x2000, 8, None, 0, None, None, 16, 0.1,
                                     0x3000, None, None, 0, None) == 1


def test_host_validation_of_shard_and_variant_calls(binding):
    L = binding._lib
    kv = _desc(binding)
    # NVFP4 attention: 16, 32 or 64 heads (16 and 32 padded to 64 in the
    # workspace, so they need one); a window size without window rows
    assert L.csa2_sparse_attn_decode_nvfp4(0x1000, 1, 1, 48, kv, 0x2000, 8, None, 0, None, None, 0, 0.1, 0x3000,
                                           None, None, 0, None) == 2
    assert L.csa2_sparse_attn_decode_nvfp4(0x1000, 1, 1, 32, kv, 0x2000, 8, None, 0, None, None, 0, 0.1, 0x3000,
                                           None, None, 0, None) == 3
    assert L.csa2_sparse_attn_decode_nvfp4(0x1000, 1, 1, 64, kv, 0x2000, 8, None, 0, None, None, 16, 0.1, 0x3000,
                                           None, None, 0, None) == 1
    assert binding.csa2_sparse_attn_nvfp4_workspace_size(1, 48, 256, 0) == 0
    assert binding.csa2_sparse_attn_nvfp4_workspace_size(1, 32, 256, 0) > \
        binding.csa2_sparse_attn_nvfp4_workspace_size(1, 64, 256, 0)
    # f32 partials need an lse output
    assert L.csa2_sparse_attn_partial(0x1000, 1, 1, 64, kv, 0x2000, 8, None, 0, None, None, 0, 0.1, 0x3000,
                                      None, None, 0, None) == 1
    # merge: head count, part count, alignment
    assert L.csa2_attn_merge(0x1000, 0x2000, 2, 1, 48, 0x3000, None, None) == 2
    assert L.csa2_attn_merge(0x1000, 0x2000, 0, 1, 64, 0x3000, None, None) == 1
    assert L.csa2_attn_merge(0x1004, 0x2000, 2, 1, 64, 0x3000, None, None) == 1
    # id scoring: indexer heads, empty id list, negative offset, unsupported key width
    assert L.csa2_score_ids(0x1000, 0x2000, 1, 1, 17, 0x3000, 8, kv, 0, 0x4000, None) == 2
    assert L.csa2_score_ids(0x1000, 0x2000, 1, 1, 4, 0x3000, 0, kv, 0, 0x4000, None) == 1
    assert L.csa2_score_ids(0x1000, 0x2000, 1, 1, 4, 0x3000, 8, kv, -1, 0x4000, None) == 1
    assert L.csa2_score_ids(0x1000, 0x2000, 1, 1, 4, 0x3000, 8, _desc(binding, di=32), 0, 0x4000, None) == 2
    # key selection: too many keys, k = 0, misaligned keys
    assert L.csa2_select_keys(0x1000, 1, (1 << 20) + 1, 8, 0x2000, None) == 2
    assert L.csa2_select_keys(0x1000, 1, 64, 0, 0x2000, None) == 1
    assert L.csa2_select_keys(0x1004, 1, 64, 8, 0x2000, None) == 1


def test_wait_selfcheck_limits_refused_on_host(binding):
    L = binding._lib
    assert L.csa2_check_wait_timeout(0, None) == 1
    assert L.csa2_check_wait_timeout(1000001, None) == 1
