"""CPU-side checks of the C ABI: the library loads, exports every symbol that
include/msa.h declares, sizes workspaces and rejects bad arguments on the host
before touching any device memory (no compute call is made here)."""
from __future__ import annotations

import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def capi():
    from block_sparse_gqa_idx_b200 import build

    build.build()
    from block_sparse_gqa_idx_b200 import _capi

    return _capi


def _header_symbols():
    with open(os.path.join(ROOT, "include", "msa.h")) as f:
        text = f.read()
    return set(re.findall(r"MSA_API\s+[\w\s\*]+?\b(msa_\w+)\s*\(", text))


def test_library_exports_every_declared_symbol(capi):
    declared = _header_symbols()
    assert declared == set(capi.EXPORTS)
    lib = ctypes.CDLL(capi.LIB_PATH)
    for name in declared:
        assert hasattr(lib, name), name
    assert "sm_100a" in capi.version()


def test_workspace_sizes(capi):
    d = capi.dims(131072, 32, 4, 128, 64, 128, 16)
    assert capi.index_topk_workspace_size(d) >= 16
    ws = capi.sparse_attn_fwd_workspace_size(d)
    # fp16 partials of every (query, group, slot) and head of one 131072-query
    # chunk: 131072*H_q*k*d_h*2 bytes, plus the inverse index
    assert ws >= 131072 * 32 * 16 * 128 * 2
    assert ws < 131072 * 32 * 16 * 128 * 2 * 1.2
    d1m = capi.dims(1 << 20, 32, 4, 128, 64, 128, 16)
    # the prefill works in query chunks: 1M needs about the same workspace
    assert capi.sparse_attn_fwd_workspace_size(d1m) < ws * 1.1
    dd = capi.decode_dims(64, 131328, 32, 4, 128, 64, 128, 16)
    assert capi.sparse_decode_workspace_size(dd) > 64 * 4 * 16 * 8 * 128 * 4


FAKE = ctypes.c_void_p(1 << 20)  # aligned, never dereferenced: validation fails first


@pytest.mark.parametrize("field,value,status", [
    ("H_q", 6, 1),       # H_q % H_kv != 0 -> invalid
    ("k", 0, 1),         # k < 1 -> invalid
    ("N", 0, 1),         # empty -> invalid
    ("B_k", 32, 2),      # block size without a kernel -> unsupported
    ("d_idx", 48, 2),    # index head dim without a kernel -> unsupported
    ("k", 33, 2),        # k above 32 -> unsupported
])
def test_index_topk_rejects_on_host(capi, field, value, status):
    d = capi.dims(4096, 8, 4, 128, 64, 128, 16)
    setattr(d, field, value)
    st = capi.LIB.msa_index_topk(ctypes.byref(d), FAKE, FAKE, FAKE, None, FAKE, 1 << 20, None)
    assert st == status


def test_misaligned_and_null_pointers_rejected(capi):
    d = capi.dims(4096, 8, 4, 128, 64, 128, 16)
    bad = ctypes.c_void_p((1 << 20) + 2)
    assert capi.LIB.msa_index_topk(ctypes.byref(d), bad, FAKE, FAKE, None, FAKE, 1 << 20, None) == 1
    assert capi.LIB.msa_index_topk(ctypes.byref(d), None, FAKE, FAKE, None, FAKE, 1 << 20, None) == 1
    # a misaligned score_out is rejected too
    assert capi.LIB.msa_index_topk(ctypes.byref(d), FAKE, FAKE, FAKE, bad, FAKE, 1 << 20, None) == 1
    assert capi.LIB.msa_sparse_attn_fwd(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, FAKE, None,
                                        None, 0, None) == 1
    # a too-small workspace is reported before anything is launched
    assert capi.LIB.msa_index_topk(ctypes.byref(d), FAKE, FAKE, FAKE, None, FAKE, 8, None) == 3
    d.d_h = 96
    assert capi.LIB.msa_sparse_attn_fwd(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE,
                                        1 << 40, None) == 2


def test_decode_rejects_on_host(capi):
    dd = capi.decode_dims(4, 1024, 32, 4, 128, 64, 128, 16)
    args = [FAKE] * 12
    dd.S = 0
    assert capi.LIB.msa_sparse_decode(ctypes.byref(dd), *args, 1 << 30, None) == 1
    dd.S = 4
    dd.H_q = 4 * 33  # G = 33 > the decode kernel's 16 query rows per MMA
    assert capi.LIB.msa_sparse_decode(ctypes.byref(dd), *args, 1 << 30, None) == 2


def test_selftest_rejects_bad_workspace_on_host(capi):
    assert capi.LIB.msa_selftest_bounded_wait(None, None) == 1
    assert capi.LIB.msa_selftest_bounded_wait(ctypes.c_void_p((1 << 20) + 4), None) == 1


def test_status_strings(capi):
    texts = {capi.LIB.msa_status_string(i).decode() for i in range(6)}
    assert len(texts) == 6


def test_index_lse_rejects_on_host(capi):
    d = capi.dims(4096, 8, 4, 128, 64, 128, 16)
    ws_ok = capi.LIB.msa_index_lse_workspace(ctypes.byref(d))
    assert ws_ok > 4096 * 4 * 16 * 4  # one fp32 LSE per (query, group, slot)
    assert capi.LIB.msa_index_lse(ctypes.byref(d), None, FAKE, FAKE, FAKE, FAKE, ws_ok, None) == 1
    assert capi.LIB.msa_index_lse(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, FAKE, 8, None) == 3
    d.d_idx = 48
    assert capi.LIB.msa_index_lse(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, FAKE, 1 << 40, None) == 2


@pytest.mark.parametrize("field,value,status", [
    ("H_kv", 0, 1),      # would divide by zero in the size computation
    ("H_q", 0, 1),
    ("d_h", -128, 2),    # negative sizes must not wrap into a huge size_t
    ("H_q", 30, 1),      # H_q % H_kv != 0
    ("S", 0, 1),
])
def test_decode_workspace_and_noalloc_validate_dims_first(capi, field, value, status):
    dd = capi.decode_dims(4, 1024, 32, 4, 128, 64, 128, 16)
    setattr(dd, field, value)
    # the size query answers 0 for dims the call would reject ...
    assert capi.LIB.msa_sparse_decode_workspace(ctypes.byref(dd)) == 0
    # ... and the no-workspace entry point reports the dims error itself,
    # not a scratch-size error, launching nothing
    assert capi.LIB.msa_sparse_decode_noalloc(ctypes.byref(dd), *([FAKE] * 11), None) == status


def test_prefill_workspace_queries_reject_bad_dims(capi):
    for field, value in (("H_kv", 0), ("H_q", 6), ("d_h", -64), ("k", 0), ("N", -5)):
        d = capi.dims(4096, 8, 4, 128, 64, 128, 16)
        setattr(d, field, value)
        assert capi.LIB.msa_sparse_attn_fwd_workspace(ctypes.byref(d)) == 0, field
    for field, value in (("H_kv", 0), ("d_idx", 48), ("B_k", 0)):
        d = capi.dims(4096, 8, 4, 128, 64, 128, 16)
        setattr(d, field, value)
        assert capi.LIB.msa_index_lse_workspace(ctypes.byref(d)) == 0, field


def test_varlen_rejects_bad_cu_seqlens_on_host(capi):
    """cu_seqlens must run from 0 to N without decreasing; the workspace
    queries return 0 and the calls INVALID_ARG, launching nothing."""
    FAKE = ctypes.c_void_p(1 << 20)
    d = capi.varlen_dims(3, 500, 8, 2, 64, 32, 64, 4)

    def cu(vals):
        return (ctypes.c_int64 * len(vals))(*vals)

    good = cu([0, 200, 200, 500])
    assert capi.LIB.msa_index_topk_varlen_workspace(ctypes.byref(d), good) > 0
    assert capi.LIB.msa_sparse_attn_fwd_varlen_workspace(ctypes.byref(d), good) > 0
    for bad in ([1, 200, 300, 500], [0, 300, 200, 500], [0, 200, 300, 499]):
        c = cu(bad)
        assert capi.LIB.msa_index_topk_varlen_workspace(ctypes.byref(d), c) == 0, bad
        assert capi.LIB.msa_sparse_attn_fwd_varlen_workspace(ctypes.byref(d), c) == 0, bad
        assert capi.LIB.msa_index_topk_varlen(ctypes.byref(d), c, FAKE, FAKE, FAKE, None, FAKE,
                                              1 << 30, None) == 1, bad
        assert capi.LIB.msa_sparse_attn_fwd_varlen(ctypes.byref(d), c, FAKE, FAKE, FAKE, FAKE,
                                                   FAKE, None, FAKE, 1 << 30, None) == 1, bad
    assert capi.LIB.msa_index_topk_varlen(ctypes.byref(d), None, FAKE, FAKE, FAKE, None, FAKE,
                                          1 << 30, None) == 1
    # a workspace below the query's size
    assert capi.LIB.msa_index_topk_varlen(ctypes.byref(d), good, FAKE, FAKE, FAKE, None, FAKE,
                                          8, None) == 3
    with pytest.raises(ValueError):
        capi._cu([0, 10, 20], 30)
