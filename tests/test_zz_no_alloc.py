"""fathom_scan_topk_noalloc, the scan entry point for callers that cannot
allocate device memory (for example a plugin inside a serving process that
owns all device memory, or a decode loop that must not block on cudaMalloc).

It is called through the C ABI and must give the same top-k as
fathom_scan_topk with a caller workspace, on two calls in a row (the second
call finds the previous call's data in the shared scratch).  This file is
collected last so that a failure here leaves every other test already run.
"""

import ctypes

import numpy as np
import pytest
import torch

import synthkv
from parity import check_scores_at

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def F():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from bit_plane_kv_scan_b200 import build, fathom
    build.build()
    fathom.lib()
    return fathom


def _inputs(F, case, budget):
    dev = torch.device("cuda")
    planes = F.pack_planes(case.codes.to(dev))
    q = case.q_storage().to(dev)
    alloc = F.allocate(q, case.sigma.to(dev), budget)
    return planes, case.qmin.to(dev), case.qscale.to(dev), q, alloc


def test_noalloc_matches_workspace_entry_point(F):
    L = F.lib()
    case = synthkv.make_case(seed=31, n=150000, h_kv=2, h_q=8, d=128, q_dtype="bf16")
    k = 512
    planes, qmin, qscale, q, alloc = _inputs(F, case, 92)
    ref_idx, ref_sc = F.scan_topk(planes, qmin, qscale, q, alloc, k, case.n)
    torch.cuda.synchronize()
    ref_rep = F.read_report()
    ref_idx, ref_sc = ref_idx.cpu().numpy(), ref_sc.cpu().numpy()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call in range(2):
        idx = torch.full((8, k), -7, dtype=torch.int32, device="cuda")
        sc = torch.full((8, k), 7.0, dtype=torch.float32, device="cuda")
        args = F.scan_args(planes, qmin, qscale, q, alloc, k, case.n, idx, sc)
        st = L.fathom_scan_topk_noalloc(ctypes.byref(args), stream)
        assert st == F.OK, L.fathom_last_error()
        torch.cuda.synchronize()
        got_i, got_s = idx.cpu().numpy(), sc.cpu().numpy()
        np.testing.assert_array_equal(got_i, ref_idx, err_msg="call %d" % call)
        # the status block in the scratch: the same report as the workspace's
        rep = F.ScanReport()
        st = L.fathom_scan_read_report_noalloc(ctypes.byref(rep), stream)
        assert st == F.OK, L.fathom_last_error()
        assert rep.union_planes == ref_rep.union_planes, "call %d" % call
        assert rep.device_faults == 0 and rep.fallback_heads == ref_rep.fallback_heads
        for h in range(8):
            check_scores_at(got_s[h], ref_sc[h], 0.0, "call %d head %d" % (call, h))


def test_noalloc_rejects_sizes_beyond_its_scratch(F):
    L = F.lib()
    args = F.ScanArgs(planes=None, planes_location=F.PLANES_DEVICE, qmin=None, qscale=None,
                      q=None, q_dtype=F.BF16, alloc=None, n=(1 << 31) - 1, d=128, h_q=32,
                      h_kv=8, k=8192, out_idx=None, out_score=None, debug_scores=None, flags=0)
    assert L.fathom_scan_topk_workspace_size(ctypes.byref(args)) > F.NOALLOC_SCRATCH_BYTES
    st = L.fathom_scan_topk_noalloc(ctypes.byref(args), None)
    assert st == F.ERR_WORKSPACE_TOO_SMALL
    assert b"scratch" in L.fathom_last_error()
