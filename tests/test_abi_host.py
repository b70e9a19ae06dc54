"""Host-side checks of the C ABI: the library loads, exports everything
include/fathom.h declares, and rejects bad arguments before any launch.
No GPU needed: every call here fails validation (or only sizes things)."""

import ctypes
import os
import re

import pytest

from bit_plane_kv_scan_b200 import build as fbuild
from bit_plane_kv_scan_b200 import fathom as F

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    fbuild.build()
    return F.lib()


def declared_functions():
    with open(os.path.join(ROOT, "include", "fathom.h")) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(fathom_[a-z_]+)\s*\(", text)))


def test_header_declares_the_hot_path():
    names = declared_functions()
    for want in ("fathom_pack_planes", "fathom_allocate", "fathom_scan_topk",
                 "fathom_scan_topk_batched", "fathom_scan_topk_workspace_size"):
        assert want in names


def test_every_declared_symbol_is_exported(L):
    names = declared_functions()
    assert names
    for name in names:
        assert hasattr(L, name), name
    assert sorted(F.EXPORTED) == names


def test_checked_build_exports_the_same_symbols():
    """The debug build (device bounds checks) is a drop-in for libfathom.so."""
    fbuild.build()
    assert os.path.exists(fbuild.LIB_CHECKED)
    C = ctypes.CDLL(fbuild.LIB_CHECKED)
    for name in declared_functions():
        assert hasattr(C, name), name


def test_check_device_status_rejects_a_host_workspace(L):
    buf = ctypes.create_string_buffer(256)
    assert L.fathom_check_device_status(None, None) == F.ERR_INVALID_ARGUMENT
    assert L.fathom_check_device_status(ctypes.addressof(buf), None) == F.ERR_INVALID_ARGUMENT


def test_plane_words(L):
    assert [L.fathom_plane_words(n) for n in (0, 1, 127, 128, 129, 1 << 20)] == \
        [0, 4, 4, 4, 8, 32768]
    assert L.fathom_planes_bytes(1 << 20, 128, 8) == 8 * 128 * 4 * 32768 * 4


def _status(call):
    return call


def test_pack_rejects_bad_shapes(L):
    assert L.fathom_pack_planes(None, 100, 33, 1, None, None) == F.ERR_UNSUPPORTED
    assert L.fathom_pack_planes(None, 100, 512, 1, None, None) == F.ERR_UNSUPPORTED
    assert L.fathom_pack_planes(None, -1, 128, 1, None, None) == F.ERR_INVALID_ARGUMENT
    assert L.fathom_pack_planes(None, 100, 128, 0, None, None) == F.ERR_INVALID_ARGUMENT
    # null codes
    assert L.fathom_pack_planes(None, 100, 128, 1, None, None) == F.ERR_INVALID_ARGUMENT
    assert b"codes" in L.fathom_last_error()
    # n = 0 is a no-op
    assert L.fathom_pack_planes(None, 0, 128, 1, None, None) == F.OK


def test_pack_rejects_host_pointers(L):
    buf = ctypes.create_string_buffer(4096)
    st = L.fathom_pack_planes(ctypes.addressof(buf), 32, 32, 1, ctypes.addressof(buf), None)
    assert st == F.ERR_INVALID_ARGUMENT
    assert b"device pointer" in L.fathom_last_error()


def test_allocate_rejects_bad_arguments(L):
    assert L.fathom_allocate(None, F.BF16, None, 32, 8, 100, 92, None, None) == F.ERR_UNSUPPORTED
    assert L.fathom_allocate(None, F.BF16, None, 30, 8, 128, 92, None, None) == F.ERR_INVALID_ARGUMENT
    assert L.fathom_allocate(None, F.BF16, None, 32, 8, 128, 513, None, None) == F.ERR_INVALID_ARGUMENT
    assert L.fathom_allocate(None, F.BF16, None, 32, 8, 128, -1, None, None) == F.ERR_INVALID_ARGUMENT
    assert L.fathom_allocate(None, 7, None, 32, 8, 128, 92, None, None) == F.ERR_INVALID_ARGUMENT
    assert L.fathom_allocate(None, F.BF16, None, 32, 8, 128, 92, None, None) == F.ERR_INVALID_ARGUMENT


def _args(**kw):
    a = dict(planes=None, planes_location=F.PLANES_DEVICE, qmin=None, qscale=None, q=None,
             q_dtype=F.BF16, alloc=None, n=1 << 20, d=128, h_q=32, h_kv=8, k=2048,
             out_idx=None, out_score=None, debug_scores=None, flags=0)
    a.update(kw)
    return F.ScanArgs(**a)


def test_append_rejects_bad_arguments(L):
    assert L.fathom_append_planes(None, 100, 1, 33, 1, None, None, None) == F.ERR_UNSUPPORTED
    assert L.fathom_append_planes(None, -1, 1, 128, 1, None, None, None) == F.ERR_INVALID_ARGUMENT
    assert L.fathom_append_planes(None, 100, -1, 128, 1, None, None, None) == F.ERR_INVALID_ARGUMENT
    assert L.fathom_append_planes(None, 100, 1, 128, 1, None, None, None) == F.ERR_INVALID_ARGUMENT
    assert b"planes_out" in L.fathom_last_error()
    assert L.fathom_append_planes(None, 0, 0, 128, 1, None, None, None) == F.OK


def test_allocate_uniform_rejects_bad_arguments(L):
    assert L.fathom_allocate_uniform(32, 100, 92, None, None) == F.ERR_UNSUPPORTED
    assert L.fathom_allocate_uniform(0, 128, 92, None, None) == F.ERR_INVALID_ARGUMENT
    assert L.fathom_allocate_uniform(32, 128, 513, None, None) == F.ERR_INVALID_ARGUMENT
    assert L.fathom_allocate_uniform(32, 128, -1, None, None) == F.ERR_INVALID_ARGUMENT
    assert L.fathom_allocate_uniform(32, 128, 136, None, None) == F.ERR_INVALID_ARGUMENT
    assert b"alloc" in L.fathom_last_error()


def test_sparse_attention_rejects_bad_arguments(L):
    def args(**kw):
        a = dict(q=None, q_dtype=F.BF16, k_rows=None, v_rows=None, idx=None, n=1000, d=128,
                 h_q=32, h_kv=8, k=64, softmax_scale=0.088, out=None, lse=None)
        a.update(kw)
        return ctypes.byref(F.AttentionArgs(**a))
    assert L.fathom_sparse_attention(None, None) == F.ERR_INVALID_ARGUMENT
    assert L.fathom_sparse_attention(args(d=100), None) == F.ERR_UNSUPPORTED
    assert L.fathom_sparse_attention(args(h_q=30), None) == F.ERR_INVALID_ARGUMENT
    assert L.fathom_sparse_attention(args(k=-1), None) == F.ERR_INVALID_ARGUMENT
    assert L.fathom_sparse_attention(args(n=-5), None) == F.ERR_INVALID_ARGUMENT
    assert L.fathom_sparse_attention(args(softmax_scale=float("inf")), None) == F.ERR_INVALID_ARGUMENT
    assert L.fathom_sparse_attention(args(q_dtype=9), None) == F.ERR_INVALID_ARGUMENT
    assert L.fathom_sparse_attention(args(kv_location=5), None) == F.ERR_INVALID_ARGUMENT
    assert b"kv_location" in L.fathom_last_error()
    assert L.fathom_sparse_attention(args(), None) == F.ERR_INVALID_ARGUMENT
    assert b"q" in L.fathom_last_error()


def test_scan_workspace_size_and_limits(L):
    ws = L.fathom_scan_topk_workspace_size(ctypes.byref(_args()))
    assert ws > 0 and ws % 256 == 0
    # candidate buffers dominate: 32 heads x capacity x 8 bytes
    assert ws >= 32 * 8 * 8 * 2048
    for bad in (dict(d=100), dict(h_q=24), dict(h_q=64), dict(k=0), dict(k=8193),
                dict(n=-1), dict(n=1 << 31), dict(q_dtype=9), dict(planes_location=5)):
        assert L.fathom_scan_topk_workspace_size(ctypes.byref(_args(**bad))) == 0, bad
    # G = 1 and G = 2 are supported
    assert L.fathom_scan_topk_workspace_size(ctypes.byref(_args(h_q=8))) > 0
    assert L.fathom_scan_topk_workspace_size(ctypes.byref(_args(h_q=16))) > 0
    # no sampling needs room for every key as a candidate
    big = L.fathom_scan_topk_workspace_size(ctypes.byref(_args(flags=F.FLAG_NO_SAMPLING)))
    assert big >= 32 * 8 * (1 << 20)


def test_token_group_arguments(L):
    """Per-token-group statistics: a positive multiple of the quantum, tensor-core
    scan only; the workspace grows by one plan per extra token group."""
    for tg in (-65536, 1000, 65537, 3 * 65536 + 1):
        a = _args(token_group=tg)
        assert L.fathom_scan_topk_workspace_size(ctypes.byref(a)) == 0
        assert L.fathom_scan_topk(ctypes.byref(a), None, 0, None) == F.ERR_INVALID_ARGUMENT
        assert b"token_group" in L.fathom_last_error()
    a = _args(token_group=65536, flags=F.FLAG_CUDA_CORES)
    assert L.fathom_scan_topk_workspace_size(ctypes.byref(a)) == 0
    assert L.fathom_scan_topk(ctypes.byref(a), None, 0, None) == F.ERR_UNSUPPORTED
    # past the token-group checks, the null pointers are what is rejected
    a = _args(token_group=65536)
    assert L.fathom_scan_topk(ctypes.byref(a), None, 0, None) == F.ERR_INVALID_ARGUMENT
    assert b"qmin" in L.fathom_last_error()
    base = L.fathom_scan_topk_workspace_size(ctypes.byref(_args()))
    for tg, groups in ((65536, 16), (1 << 20, 1), (1 << 21, 1), (3 * 65536, 6)):
        size = L.fathom_scan_topk_workspace_size(ctypes.byref(_args(token_group=tg)))
        assert size >= base and (size > base) == (groups > 1), (tg, size, base)


def test_scan_rejects_before_launch(L):
    assert L.fathom_scan_topk(None, None, 0, None) == F.ERR_INVALID_ARGUMENT
    assert L.fathom_scan_topk(ctypes.byref(_args(h_q=24)), None, 0, None) == F.ERR_UNSUPPORTED
    assert L.fathom_scan_topk(ctypes.byref(_args()), None, 0, None) == F.ERR_INVALID_ARGUMENT
    assert b"qmin" in L.fathom_last_error()


def test_batched_rejects_bad_arguments(L):
    a = F.BatchedArgs(sessions=None, num_sessions=0, n_max=1000, d=128, h_q=32, h_kv=8, k=1024,
                      q_dtype=F.BF16, planes_location=F.PLANES_DEVICE, flags=0)
    assert L.fathom_scan_topk_batched_workspace_size(ctypes.byref(a)) == 0
    assert L.fathom_scan_topk_batched(ctypes.byref(a), None, 0, None) == F.ERR_INVALID_ARGUMENT
    a.num_sessions = 32
    assert L.fathom_scan_topk_batched_workspace_size(ctypes.byref(a)) > 0
    assert L.fathom_scan_topk_batched(ctypes.byref(a), None, 0, None) == F.ERR_INVALID_ARGUMENT
    assert b"sessions" in L.fathom_last_error()


def test_report_rejects_null(L):
    assert L.fathom_scan_read_report(None, None, None) == F.ERR_INVALID_ARGUMENT


def test_merge_rejects_bad_arguments(L):
    offs = (ctypes.c_int64 * 2)(0, 100)
    m = L.fathom_merge_topk
    assert m(None, None, 0, offs, 8, 64, 64, None, None, None) == F.ERR_INVALID_ARGUMENT
    assert m(None, None, F.MAX_MERGE_PARTS + 1, offs, 8, 64, 64, None, None, None) == \
        F.ERR_INVALID_ARGUMENT
    assert m(None, None, 2, offs, 0, 64, 64, None, None, None) == F.ERR_INVALID_ARGUMENT
    assert m(None, None, 2, offs, 8, 0, 64, None, None, None) == F.ERR_INVALID_ARGUMENT
    assert m(None, None, 2, offs, 8, 64, 8193, None, None, None) == F.ERR_INVALID_ARGUMENT
    assert m(None, None, 2, None, 8, 64, 64, None, None, None) == F.ERR_INVALID_ARGUMENT
    bad = (ctypes.c_int64 * 2)(0, 1 << 31)
    assert m(None, None, 2, bad, 8, 64, 64, None, None, None) == F.ERR_INVALID_ARGUMENT
    assert b"offsets" in L.fathom_last_error()
    assert m(None, None, 2, offs, 8, 64, 64, None, None, None) == F.ERR_INVALID_ARGUMENT
    assert b"in_idx" in L.fathom_last_error()


def test_noalloc_report_rejects_null(L):
    assert L.fathom_scan_read_report_noalloc(None, None) == F.ERR_INVALID_ARGUMENT
    assert b"report" in L.fathom_last_error()
