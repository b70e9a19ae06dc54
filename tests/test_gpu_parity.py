"""Parity of the CUDA scan (through the C ABI) with the CPU oracle.

Rules and tolerances: tests/parity.py.  Small cases compare every output;
the full-size workloads (131k, 1M, 32 ragged sessions, host-resident planes)
run in the launch configuration the benchmark times and compare every
allocation, the full top-k of a subset of heads against the oracle's
brute force, and every returned score against the oracle's score at that
index.
"""

import numpy as np
import pytest
import torch

import oracle
import synthkv
from parity import (check_dense, check_scores_at, check_topk, check_topk_sampled,
                    fixed_point_bound, score_scale)

pytestmark = pytest.mark.gpu

F = None


@pytest.fixture(scope="module", autouse=True)
def _lib():
    global F
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import bit_plane_kv_scan_b200 as fb
    from bit_plane_kv_scan_b200 import build
    build.build()
    F = fb
    F.lib()
    yield


def _np(t):
    return t.detach().cpu().numpy()


def _planes_np(planes):
    return _np(planes).view(np.uint32)


def run_gpu(case, budget, k, flags=0, debug=False, host_mapped=False, uniform=False):
    dev = torch.device("cuda")
    codes = case.codes.to(dev)
    planes = F.pack_planes(codes)
    if host_mapped:
        hp = torch.empty(planes.shape, dtype=planes.dtype, pin_memory=True)
        hp.copy_(planes)
        planes_used = hp
    else:
        planes_used = planes
    q = case.q_storage().to(dev)
    sigma = case.sigma.to(dev)
    if uniform:
        alloc = F.allocate_uniform(case.h_q, case.d, budget, device=dev)
    else:
        alloc = F.allocate(q, sigma, budget)
    out = F.scan_topk(planes_used, case.qmin.to(dev), case.qscale.to(dev), q, alloc, k, case.n,
                      debug_scores=debug, flags=flags, host_mapped=host_mapped)
    torch.cuda.synchronize()
    return planes, alloc, out


def oracle_head(case_np, h, t_h):
    codes, qmin, qscale, q = case_np
    G = q.shape[0] // codes.shape[0]
    g = h // G
    return oracle.scores_from_codes(codes[g], qmin[g], qscale[g], q[h], t_h)


def case_np(case):
    return (_np(case.codes), _np(case.qmin), _np(case.qscale), _np(case.q).astype(np.float64))


# ------------------------------------------------------------------ pack --

@pytest.mark.parametrize("n,d,h_kv", [(1, 32, 1), (31, 64, 2), (4096, 128, 1), (4097, 128, 2),
                                      (33333, 256, 1), (100000, 96, 3), (5000, 160, 2),
                                      (1025, 192, 1), (70000, 224, 1)])
def test_pack_bit_exact(n, d, h_kv):
    rng = np.random.default_rng(n + d)
    codes = rng.integers(0, 256, size=(h_kv, n, d // 2), dtype=np.uint8)
    planes = F.pack_planes(torch.from_numpy(codes).cuda())
    torch.cuda.synchronize()
    np.testing.assert_array_equal(_planes_np(planes), oracle.pack_planes(codes))


def test_pack_full_size_1m():
    case = synthkv.make_case(seed=2, n=1 << 20, h_kv=8, h_q=32, device="cuda", keep_keys=False)
    planes = F.pack_planes(case.codes)
    torch.cuda.synchronize()
    got = _planes_np(planes)
    codes = _np(case.codes)
    # the oracle packs two KV heads in full; the rest are checked on sampled words
    for g in (0, 7):
        np.testing.assert_array_equal(got[g:g + 1], oracle.pack_planes(codes[g:g + 1]))
    rng = np.random.default_rng(0)
    for g in range(8):
        for w in rng.integers(0, got.shape[-1], 16):
            sl = codes[g:g + 1, 32 * w:32 * w + 32]
            ref = oracle.pack_planes(sl)[0, :, :, 0]
            np.testing.assert_array_equal(got[g, :, :, w], ref)


# -------------------------------------------------------------- allocate --

def _alloc_cases():
    rng = np.random.default_rng(42)
    out = []
    for d in (32, 128, 256):
        q = rng.normal(size=(8, d)) * np.exp(rng.normal(size=(8, d)))
        sigma = np.exp(rng.uniform(np.log(0.1), np.log(10), size=(2, d)))
        out.append(("random_d%d" % d, q, sigma))
    d = 128
    q = np.zeros((4, d))
    q[0, ::7] = 1.0                     # many equal weights
    q[1, :] = 2.0 ** rng.integers(-4, 4, d)  # weights that tie across channels after 4^-tau
    q[2, :5] = [1, -1, 2, -2, 0.5]      # mostly zero weights
    q[3, :] = 1.0                       # all equal
    out.append(("ties", q, np.ones((1, d))))
    return out


@pytest.mark.parametrize("name,q,sigma", _alloc_cases(), ids=lambda x: x if isinstance(x, str) else "")
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_allocate_bit_exact(name, q, sigma, dtype):
    d = q.shape[1]
    qt = torch.from_numpy(q).to(dtype)
    qd = qt.float().numpy().astype(np.float64)  # the exact values the library sees
    sig = torch.from_numpy(sigma).float()
    for B in sorted(x for x in {0, 1, 5, 68, 92, 136, 4 * d - 1, 4 * d} if x <= 4 * d):
        got = _np(F.allocate(qt.cuda(), sig.cuda(), B))
        want = oracle.allocate_heads(qd, sig.numpy().astype(np.float64), B)
        np.testing.assert_array_equal(got, want, err_msg="%s B=%d" % (name, B))


# ------------------------------------------------------------ small scans --

def _want_alloc(case, cn, budget, uniform):
    if uniform:
        return oracle.allocate_uniform(case.h_q, case.d, budget)
    return oracle.allocate_heads(cn[3], _np(case.sigma), budget)


def _tol(flags, q_h, qmin_g, qscale_g, t_h):
    """Score tolerance of one head (tests/parity.py): the paths that
    accumulate fp32 products (the CUDA-core scan and the exact single-block
    fallback) take the S_h / 8 floor; the tensor-core path takes the bare
    1e-5 and, for a score so close to 0 that 1e-5 of it is below the
    fixed-point resolution, its exact fixed-point bound B Delta_h / 2."""
    if flags & (F.FLAG_CUDA_CORES | F.FLAG_FORCE_FALLBACK):
        return dict(floor=score_scale(q_h, qmin_g, qscale_g) / 8.0)
    return dict(abs_tol=fixed_point_bound(q_h, qscale_g, t_h))


def _full_check(case, budget, k, flags=0, what="", uniform=False):
    planes, alloc, (idx, sc, dbg) = run_gpu(case, budget, k, flags=flags, debug=True,
                                            uniform=uniform)
    cn = case_np(case)
    want_alloc = _want_alloc(case, cn, budget, uniform)
    np.testing.assert_array_equal(_np(alloc), want_alloc)
    np.testing.assert_array_equal(_planes_np(planes), oracle.pack_planes(cn[0]))
    G = case.group
    idx, sc, dbg = _np(idx), _np(sc), _np(dbg)
    for h in range(case.h_q):
        g = h // G
        ref = oracle_head(cn, h, want_alloc[h])
        scale = score_scale(cn[3][h], cn[1][g], cn[2][g])
        check_dense(dbg[h], ref, scale, "%s head %d" % (what, h))
        check_topk(idx[h], sc[h], ref, k, what="%s head %d" % (what, h),
                   **_tol(flags, cn[3][h], cn[1][g], cn[2][g], want_alloc[h]))


@pytest.mark.parametrize("h_q,d,B", [(1, 32, 0), (4, 64, 100), (32, 128, 92), (32, 128, 136),
                                     (3, 96, 200), (7, 256, 1024)])
def test_allocate_uniform_bit_exact(h_q, d, B):
    got = F.allocate_uniform(h_q, d, B)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(_np(got), oracle.allocate_uniform(h_q, d, B))


@pytest.mark.parametrize("B", [68, 136])
@pytest.mark.parametrize("cuda_cores", [False, True])
def test_uniform_read_scan(B, cuda_cores):
    """The scan over a query-independent allocation, dense scores and top-k
    against the oracle (both scan kernels)."""
    case = synthkv.make_case(seed=11 + B, n=20000, h_kv=2, h_q=8, d=128, q_dtype="bf16")
    _full_check(case, B, 64, flags=F.FLAG_CUDA_CORES if cuda_cores else 0,
                what="uniform B=%d cc=%d" % (B, cuda_cores), uniform=True)


def test_tiny_4k_config():
    """The tiny single-head workload: n=4096, d=128, fp32 query, B=92, k=64."""
    c = synthkv.CONFIGS["tiny_4k"]
    case = synthkv.make_case(c["seed"], c["n"], c["h_kv"], c["h_q"], c["d"], c["q_dtype"])
    _full_check(case, 92, 64, what="tiny_4k")


@pytest.mark.parametrize("n", [1, 33, 4095, 4097, 12345])
@pytest.mark.parametrize("G", [1, 2, 4])
def test_ragged_n_and_groups(n, G):
    case = synthkv.make_case(seed=100 + n + G, n=n, h_kv=2, h_q=2 * G, d=128, q_dtype="bf16")
    for B, k in ((92, 7), (17, 100)):
        _full_check(case, B, k, what="n=%d G=%d B=%d k=%d" % (n, G, B, k))


@pytest.mark.parametrize("d", [32, 64, 256])
def test_other_widths(d):
    case = synthkv.make_case(seed=d, n=5000, h_kv=1, h_q=4, d=d, q_dtype="bf16")
    _full_check(case, d // 2, 33, what="d=%d" % d)


@pytest.mark.parametrize("B", [0, 1, 512])
def test_degenerate_budgets(B):
    """B = 0: every score is the per-query constant and the top-k is the first
    k indices; B = 4d: the full 4-bit dequantised dot product."""
    case = synthkv.make_case(seed=7, n=3000, h_kv=1, h_q=4, d=128, q_dtype="bf16")
    _full_check(case, B, 50, what="B=%d" % B)
    if B == 0:
        _, _, (idx, sc) = run_gpu(case, 0, 50)
        assert (_np(idx) == np.arange(50)[None, :]).all()


@pytest.mark.parametrize("cuda_cores", [False, True])
def test_empty_union_on_a_stale_workspace(cuda_cores):
    """B = 0 (every union prefix empty) on a workspace that holds no plan of
    this call: first a scan at another d fills it, then a fresh workspace is
    filled with 0xFF bytes.  Both must give the oracle's answer (the scan may
    read nothing outside the planes of this call)."""
    flags = F.FLAG_CUDA_CORES if cuda_cores else 0
    dev = torch.device("cuda")
    other = synthkv.make_case(seed=41, n=9000, h_kv=2, h_q=8, d=256, q_dtype="bf16")
    run_gpu(other, 700, 40, flags=flags)
    case = synthkv.make_case(seed=42, n=7000, h_kv=2, h_q=8, d=128, q_dtype="bf16")
    for fill in (None, 0xFF):
        ws = None
        if fill is not None:
            ws = F.Workspace(dev)
            ws.buf = torch.full((64 << 20,), fill, dtype=torch.uint8, device=dev)
        q = case.q_storage().to(dev)
        alloc = F.allocate(q, case.sigma.to(dev), 0)
        planes = F.pack_planes(case.codes.to(dev))
        idx, sc, dbg = F.scan_topk(planes, case.qmin.to(dev), case.qscale.to(dev), q, alloc, 50,
                                   case.n, debug_scores=True, flags=flags, workspace=ws)
        torch.cuda.synchronize()
        rep = F.read_report(ws)
        assert rep.device_faults == 0 and rep.union_planes == 0
        cn = case_np(case)
        for h in range(case.h_q):
            g = h // case.group
            ref = oracle_head(cn, h, np.zeros(case.d, dtype=np.uint8))
            scale = score_scale(cn[3][h], cn[1][g], cn[2][g])
            check_dense(_np(dbg)[h], ref, scale, "B=0 fill=%s head %d" % (fill, h))
            check_topk(_np(idx)[h], _np(sc)[h], ref, 50, what="B=0 fill=%s head %d" % (fill, h),
                       **_tol(flags, cn[3][h], cn[1][g], cn[2][g], np.zeros(case.d, np.uint8)))
            assert (_np(idx)[h] == np.arange(50)).all()


@pytest.mark.parametrize("cuda_cores", [False, True])
def test_batched_descriptor_beyond_n_max(cuda_cores):
    """A session descriptor whose n exceeds the n_max the workspace was sized
    for is scanned as empty and reported as a device fault; the other
    sessions are unaffected."""
    import ctypes
    flags = F.FLAG_CUDA_CORES if cuda_cores else 0
    dev = torch.device("cuda")
    cases = [synthkv.make_case(seed=50 + i, n=n, h_kv=1, h_q=4, d=128, q_dtype="bf16")
             for i, n in enumerate((6000, 3000))]
    descs = []
    for c in cases:
        q = c.q_storage().to(dev)
        descs.append(dict(planes=F.pack_planes(c.codes.to(dev)), qmin=c.qmin.to(dev),
                          qscale=c.qscale.to(dev), q=q, alloc=F.allocate(q, c.sigma.to(dev), 92),
                          n=c.n))
    scan = F.BatchedScan(descs, 64, 128, 4, 1, torch.bfloat16, flags=flags, device=dev)
    scan.args.n_max = 4000  # session 0 (n = 6000) is beyond the bound
    L = F.lib()
    need = L.fathom_scan_topk_batched_workspace_size(ctypes.byref(scan.args))
    ws = F.Workspace(dev)
    buf = ws.get(need)
    st = L.fathom_scan_topk_batched(ctypes.byref(scan.args), ctypes.c_void_p(buf.data_ptr()), need,
                                    ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == F.OK, L.fathom_last_error()
    torch.cuda.synchronize()
    rep = F.ScanReport()
    st = L.fathom_scan_read_report(ctypes.c_void_p(buf.data_ptr()), ctypes.byref(rep), None)
    assert st == F.ERR_DEVICE_CHECK and rep.device_faults == 1
    assert L.fathom_check_device_status(ctypes.c_void_p(buf.data_ptr()), None) == F.ERR_DEVICE_CHECK
    i0, s0 = scan.outs[0]
    assert (_np(i0) == -1).all() and np.isneginf(_np(s0)).all()
    c = cases[1]
    cn = case_np(c)
    want = oracle.allocate_heads(cn[3], _np(c.sigma), 92)
    i1, s1 = _np(scan.outs[1][0]), _np(scan.outs[1][1])
    for h in range(4):
        ref = oracle_head(cn, h, want[h])
        check_topk(i1[h], s1[h], ref, 64, what="session 1 head %d" % h,
                   **_tol(flags, cn[3][h], cn[1][0], cn[2][0], want[h]))


def test_k_larger_than_n_and_empty():
    case = synthkv.make_case(seed=8, n=40, h_kv=1, h_q=4, d=128, q_dtype="bf16")
    _full_check(case, 92, 64, what="k>n")
    empty = synthkv.make_case(seed=9, n=0 + 1, h_kv=1, h_q=4, d=128, q_dtype="bf16")
    dev = torch.device("cuda")
    q = empty.q_storage().to(dev)
    alloc = F.allocate(q, empty.sigma.to(dev), 92)
    planes = torch.zeros((1, 128, 4, 4), dtype=torch.int32, device=dev)
    idx, sc = F.scan_topk(planes, empty.qmin.to(dev), empty.qscale.to(dev), q, alloc, 5, 0)
    torch.cuda.synchronize()
    assert (_np(idx) == -1).all() and np.isneginf(_np(sc)).all()


@pytest.mark.parametrize("cuda_cores", [False, True])
def test_largest_k(cuda_cores):
    """k = FATHOM_MAX_K (8192), the merge's largest output and sort."""
    case = synthkv.make_case(seed=17, n=100000, h_kv=1, h_q=4, d=128, q_dtype="bf16")
    _full_check(case, 92, 8192, flags=F.FLAG_CUDA_CORES if cuda_cores else 0, what="k=8192")


@pytest.mark.parametrize("cuda_cores", [False, True])
def test_report_counts_and_workspace_reuse(cuda_cores):
    """The report's union-plane count is the sum over KV heads of every
    channel's largest prefix in its query-head group (the bytes the scan
    reads, in plane rows), and a second scan on the same workspace reports
    its own counts: the status, counters and thresholds are cleared by the
    scan itself, with no memset."""
    case = synthkv.make_case(seed=23, n=40000, h_kv=2, h_q=8, d=128, q_dtype="bf16")
    G = case.h_q // case.h_kv
    base = F.FLAG_CUDA_CORES if cuda_cores else 0
    for budget, extra in ((92, F.FLAG_FORCE_FALLBACK), (136, 0), (92, 0)):
        _, alloc, (idx, sc) = run_gpu(case, budget, 64, flags=base | extra)
        rep = F.read_report()
        t = _np(alloc).astype(np.int64).reshape(case.h_kv, G, case.d)
        assert rep.union_planes == int(t.max(axis=1).sum())
        assert rep.fallback_heads == (case.h_q if extra else 0)
        assert rep.device_faults == 0
        assert 64 <= rep.max_candidates


def test_sampled_threshold_path_and_fallbacks():
    """n large enough that the sampled threshold is used (k=64 samples from
    n >= 8192); the forced fallback and the no-sampling path must give the
    same answer."""
    case = synthkv.make_case(seed=21, n=40000, h_kv=2, h_q=8, d=128, q_dtype="bf16")
    _full_check(case, 92, 64, what="sampled")
    _, _, base = run_gpu(case, 92, 64)
    rep = F.read_report()
    assert rep.fallback_heads == 0
    _full_check(case, 92, 64, flags=F.FLAG_FORCE_FALLBACK, what="fallback")
    _, _, forced = run_gpu(case, 92, 64, flags=F.FLAG_FORCE_FALLBACK)
    rep = F.read_report()
    assert rep.fallback_heads == 8
    _full_check(case, 92, 64, flags=F.FLAG_NO_SAMPLING, what="no-sampling")
    _, _, nos = run_gpu(case, 92, 64, flags=F.FLAG_NO_SAMPLING)
    np.testing.assert_array_equal(_np(base[0]), _np(nos[0]))
    np.testing.assert_array_equal(_np(base[1]), _np(nos[1]))


def test_fallback_with_compaction():
    """Forced fallback on a context long enough that the single-block stream
    compacts its candidate buffer several times."""
    case = synthkv.make_case(seed=22, n=300000, h_kv=1, h_q=4, d=128, q_dtype="bf16")
    _, alloc, (idx, sc) = run_gpu(case, 92, 1000, flags=F.FLAG_FORCE_FALLBACK)
    cn = case_np(case)
    for h in range(4):
        ref = oracle_head(cn, h, _np(alloc)[h])
        check_topk(_np(idx)[h], _np(sc)[h], ref, 1000, what="fallback head %d" % h,
                   **_tol(F.FLAG_FORCE_FALLBACK, cn[3][h], cn[1][0], cn[2][0], _np(alloc)[h]))


# --------------------------------------------------- CUDA-core scan kernel --
# (the default scan is the tcgen05 kernel; the CUDA-core kernel is the
# second implementation behind FLAG_CUDA_CORES)

@pytest.mark.parametrize("n,G,B,k", [(4096, 1, 92, 64), (4097, 4, 92, 7), (12345, 2, 17, 100),
                                     (40000, 4, 136, 64), (3000, 4, 0, 50), (3000, 4, 512, 50)])
def test_cuda_core_scan(n, G, B, k):
    """The CUDA-core (fp32 FMA) form of the scan gives the oracle's answer."""
    case = synthkv.make_case(seed=300 + n + G, n=n, h_kv=2, h_q=2 * G, d=128, q_dtype="bf16")
    _full_check(case, B, k, flags=F.FLAG_CUDA_CORES, what="cc n=%d G=%d B=%d" % (n, G, B))


@pytest.mark.parametrize("d", [32, 256])
def test_cuda_core_scan_widths(d):
    case = synthkv.make_case(seed=d + 1, n=5000, h_kv=1, h_q=4, d=d, q_dtype="bf16")
    _full_check(case, d // 2, 33, flags=F.FLAG_CUDA_CORES, what="cc d=%d" % d)


def test_cuda_core_scan_layer_131k(layer_131k):
    _check_config(layer_131k, 92, 2048, heads_full={0, 13, 26, 31}, what="cc 131k",
                  flags=F.FLAG_CUDA_CORES)


# ------------------------------------------------------ full-size configs --

def _check_config(case, budget, k, heads_full, what, host_mapped=False, flags=0, uniform=False):
    _, alloc, (idx, sc) = run_gpu(case, budget, k, host_mapped=host_mapped, flags=flags,
                                  uniform=uniform)
    cn = case_np(case)
    want_alloc = _want_alloc(case, cn, budget, uniform)
    got_alloc = _np(alloc)
    np.testing.assert_array_equal(got_alloc, want_alloc)
    idx, sc = _np(idx), _np(sc)
    G = case.group
    for h in range(case.h_q):
        g = h // G
        kk = min(k, case.n)
        ref_at = oracle.scores_at(cn[0][g], cn[1][g], cn[2][g], cn[3][h], want_alloc[h],
                                  idx[h, :kk].astype(np.int64))
        tol = _tol(flags, cn[3][h], cn[1][g], cn[2][g], want_alloc[h])
        check_topk_sampled(idx[h], sc[h], ref_at, k, case.n, what="%s head %d" % (what, h), **tol)
        if h in heads_full:
            ref = oracle_head(cn, h, want_alloc[h])
            check_topk(idx[h], sc[h], ref, k, what="%s head %d" % (what, h), **tol)
    return idx, sc


@pytest.fixture(scope="module")
def layer_131k():
    c = synthkv.CONFIGS["qwen3_8b_layer_131k"]
    return synthkv.make_case(c["seed"], c["n"], c["h_kv"], c["h_q"], c["d"], c["q_dtype"],
                             device="cuda", keep_keys=False)


@pytest.mark.parametrize("B", [68, 92, 136])
def test_qwen3_8b_layer_131k(layer_131k, B):
    _check_config(layer_131k, B, 2048, heads_full=set(range(32)), what="131k B=%d" % B)


@pytest.fixture(scope="module")
def decode_1m():
    c = synthkv.CONFIGS["decode_1m"]
    return synthkv.make_case(c["seed"], c["n"], c["h_kv"], c["h_q"], c["d"], c["q_dtype"],
                             device="cuda", keep_keys=False)


@pytest.mark.parametrize("B", [92, 136])
def test_decode_1m(decode_1m, B):
    # B = 92 (the benchmarked step): full brute force on every query head;
    # B = 136: on one query head of every KV head; sampled checks on all
    heads = set(range(32)) if B == 92 else {0, 5, 10, 15, 16, 21, 26, 31}
    _check_config(decode_1m, B, 2048, heads_full=heads, what="1M B=%d" % B)
    rep = F.read_report()
    assert rep.fallback_heads == 0


def test_decode_1m_uniform_136(decode_1m):
    """The fixed-depth comparison read: 136 bits per key, the same for every
    query head, on the 1M-token step."""
    _check_config(decode_1m, 136, 2048, heads_full={0, 31}, what="1M uniform 136", uniform=True)
    rep = F.read_report()
    assert rep.fallback_heads == 0
    assert rep.union_planes == 8 * 136  # a GQA group's union is one head's read


def test_decode_1m_cuda_cores(decode_1m):
    """The CUDA-core scan on the 1M-token step."""
    _check_config(decode_1m, 92, 2048, heads_full={0, 21}, what="cc 1M",
                  flags=F.FLAG_CUDA_CORES)
    rep = F.read_report()
    assert rep.fallback_heads == 0
    assert rep.device_faults == 0


def test_host_resident_1m_budget_sweep():
    """Planes in pinned host memory: same results as device-resident planes,
    and oracle-checked, for every budget of the sweep."""
    c = synthkv.CONFIGS["host_resident_1m"]
    case = synthkv.make_case(c["seed"], c["n"], c["h_kv"], c["h_q"], c["d"], c["q_dtype"],
                             device="cuda", keep_keys=False)
    for B in c["budgets"]:
        # full brute force on one query head of every KV head, for every budget
        idx_h, sc_h = _check_config(case, B, 2048, heads_full={3, 4, 9, 14, 19, 20, 25, 30},
                                    what="host B=%d" % B, host_mapped=True)
        _, _, (idx_d, sc_d) = run_gpu(case, B, 2048)
        np.testing.assert_array_equal(idx_h, _np(idx_d))
        np.testing.assert_array_equal(sc_h, _np(sc_d))
    # the CUDA-core scan reads host-resident planes too
    idx_h, sc_h = _check_config(case, 92, 2048, heads_full={3, 30}, what="cc host B=92",
                                host_mapped=True, flags=F.FLAG_CUDA_CORES)
    _, _, (idx_d, sc_d) = run_gpu(case, 92, 2048, flags=F.FLAG_CUDA_CORES)
    np.testing.assert_array_equal(idx_h, _np(idx_d))
    np.testing.assert_array_equal(sc_h, _np(sc_d))


@pytest.mark.parametrize("cuda_cores", [False, True])
def test_ragged_32_sessions_batched(cuda_cores):
    flags = F.FLAG_CUDA_CORES if cuda_cores else 0
    c = synthkv.CONFIGS["ragged_32_sessions"]
    sessions = synthkv.make_ragged(c["seed"], c["sessions"], c["n_lo"], c["n_hi"], c["h_kv"],
                                   c["h_q"], c["d"], c["q_dtype"], device="cuda")
    dev = torch.device("cuda")
    k, B = c["k"], 92
    # one allocation launch for every session's query heads
    q_all = torch.cat([s.q_storage() for s in sessions]).to(dev)
    sig_all = torch.cat([s.sigma for s in sessions]).to(dev)
    alloc_all = F.allocate(q_all, sig_all, B)
    descs = []
    for i, s in enumerate(sessions):
        descs.append(dict(planes=F.pack_planes(s.codes), qmin=s.qmin, qscale=s.qscale,
                          q=q_all[i * 32:(i + 1) * 32], alloc=alloc_all[i * 32:(i + 1) * 32],
                          n=s.n))
    outs = F.scan_topk_batched(descs, k, 128, 32, 8, torch.bfloat16, flags=flags)
    torch.cuda.synchronize()
    assert F.read_report().device_faults == 0
    want_alloc = oracle.allocate_heads(_np(q_all.float()).astype(np.float64), _np(sig_all), B)
    np.testing.assert_array_equal(_np(alloc_all), want_alloc)
    for i, s in enumerate(sessions):
        cn = case_np(s)
        idx, sc = _np(outs[i][0]), _np(outs[i][1])
        for h in range(32):
            g = h // 4
            t_h = want_alloc[i * 32 + h]
            ref_at = oracle.scores_at(cn[0][g], cn[1][g], cn[2][g], cn[3][h], t_h,
                                      idx[h, :min(k, s.n)].astype(np.int64))
            tol = _tol(flags, cn[3][h], cn[1][g], cn[2][g], t_h)
            check_topk_sampled(idx[h], sc[h], ref_at, k, s.n, what="session %d head %d" % (i, h),
                               **tol)
            if i in (0, 13, 31) and h in (0, 9, 18, 27):
                ref = oracle_head(cn, h, t_h)
                check_topk(idx[h], sc[h], ref, k, what="session %d head %d" % (i, h), **tol)


# ------------------------------------------------------ sparse attention --

def _bf16_rows(shape, seed, dev):
    g = torch.Generator(device=dev).manual_seed(seed)
    return torch.randn(shape, generator=g, device=dev, dtype=torch.float32).to(torch.bfloat16)


def _attention_ref(q, K, V, idx, scale, h_kv):
    """The oracle on the gathered rows only (the full K/V need not fit on the host)."""
    q = q.float().cpu().numpy().astype(np.float64)
    idx = idx.cpu().numpy()
    h_q, d = q.shape
    n = K.shape[1]
    G = h_q // h_kv
    out = np.zeros((h_q, d))
    lse = np.zeros(h_q)
    for h in range(h_q):
        keep = (idx[h] >= 0) & (idx[h] < n)
        rows = torch.from_numpy(idx[h][keep].astype(np.int64)).to(K.device)
        Ks = K[h // G].index_select(0, rows).float().cpu().numpy()[None]
        Vs = V[h // G].index_select(0, rows).float().cpu().numpy()[None]
        sub = np.arange(len(rows), dtype=np.int32)[None]
        o, l = oracle.sparse_attention(q[h:h + 1], Ks, Vs, sub, scale)
        out[h], lse[h] = o[0], l[0]
    return out, lse


def _check_attention(out, lse, ref_o, ref_l, V, what):
    out, lse = _np(out).astype(np.float64), _np(lse).astype(np.float64)
    vmax = max(1.0, float(V.float().abs().max()))
    err = np.abs(out - ref_o).max()
    assert err <= 2e-5 * vmax, "%s: |o - oracle| = %g" % (what, err)
    fin = np.isfinite(ref_l)
    assert (np.isneginf(lse) == ~fin).all(), what
    lerr = np.abs(lse[fin] - ref_l[fin]) / np.maximum(1.0, np.abs(ref_l[fin]))
    assert lerr.size == 0 or lerr.max() <= 2e-5, "%s: lse error %g" % (what, lerr.max())


@pytest.mark.parametrize("n,h_kv,G,d,k,qd", [(5000, 2, 4, 128, 64, "bf16"), (3000, 1, 1, 32, 300, "f32"),
                                            (2000, 2, 2, 256, 100, "bf16"), (700, 1, 4, 96, 1000, "bf16"),
                                            (4000, 1, 2, 160, 257, "f32")])
def test_sparse_attention_random_rows(n, h_kv, G, d, k, qd):
    """Random selections with -1 padding, out-of-range entries and an empty head."""
    dev = torch.device("cuda")
    h_q = h_kv * G
    rng = np.random.default_rng(n + d)
    K = _bf16_rows((h_kv, n, d), n, dev)
    V = _bf16_rows((h_kv, n, d), n + 1, dev)
    q = torch.from_numpy(rng.normal(size=(h_q, d)).astype(np.float32))
    q = (q.to(torch.bfloat16) if qd == "bf16" else q).to(dev)
    idx = rng.integers(0, n, size=(h_q, k)).astype(np.int32)
    idx[0, k // 2:] = -1
    if h_q > 1:
        idx[1, 0] = n + 7
        idx[h_q - 1, :] = -1
    idx = torch.from_numpy(idx).to(dev)
    scale = 1.0 / np.sqrt(d)
    out, lse = F.sparse_attention(q, K, V, idx, scale)
    torch.cuda.synchronize()
    # the oracle on the whole K/V and the raw entries (it skips those outside [0, n))
    ref_o, ref_l = oracle.sparse_attention(_np(q.float()).astype(np.float64),
                                           _np(K.float()), _np(V.float()), _np(idx), scale)
    _check_attention(out, lse, ref_o, ref_l, V, "n=%d d=%d k=%d" % (n, d, k))


def _dequant_rows(codes, qmin, qscale):
    """Key rows m_c + s_c u from 4-bit codes [h_kv, n, d/2] (low nibble =
    even channel), in fp64 from the fp32 statistics."""
    c = np.asarray(codes)
    u = np.empty(c.shape[:-1] + (2 * c.shape[-1],), dtype=np.float64)
    u[..., 0::2] = c & 15
    u[..., 1::2] = c >> 4
    m = np.asarray(qmin, dtype=np.float64)[:, None, :]
    s = np.asarray(qscale, dtype=np.float64)[:, None, :]
    return m + s * u


@pytest.mark.parametrize("host_mapped", [False, True])
@pytest.mark.parametrize("n,h_kv,G,d,k,qd", [(5000, 2, 4, 128, 64, "bf16"), (3000, 1, 1, 32, 300, "f32"),
                                            (2000, 2, 2, 256, 100, "bf16"), (700, 1, 4, 96, 1000, "bf16"),
                                            (4000, 1, 2, 160, 257, "f32")])
def test_sparse_attention_4bit_keys_and_host_rows(n, h_kv, G, d, k, qd, host_mapped):
    """Keys gathered as 4-bit codes and dequantised in the gather, bf16
    values; with host_mapped the codes and values sit in pinned host memory
    and only the selected rows cross the host link.  Also bf16 key rows from
    host memory."""
    dev = torch.device("cuda")
    h_q = h_kv * G
    rng = np.random.default_rng(3 * n + d)
    codes = torch.from_numpy(rng.integers(0, 256, size=(h_kv, n, d // 2), dtype=np.uint8))
    qmin = torch.from_numpy(rng.normal(size=(h_kv, d)).astype(np.float32))
    qscale = torch.from_numpy(np.exp(rng.uniform(-3, 0, size=(h_kv, d))).astype(np.float32))
    Kb = _bf16_rows((h_kv, n, d), n + 5, dev)
    V = _bf16_rows((h_kv, n, d), n + 6, dev)
    q = torch.from_numpy(rng.normal(size=(h_q, d)).astype(np.float32))
    q = (q.to(torch.bfloat16) if qd == "bf16" else q).to(dev)
    idx = rng.integers(0, n, size=(h_q, k)).astype(np.int32)
    idx[0, k // 3:] = -1
    if h_q > 1:
        idx[1, 0] = n
        idx[h_q - 1, :] = -1
    idx_t = torch.from_numpy(idx).to(dev)
    scale = 1.0 / np.sqrt(d)
    if host_mapped:
        codes_u = codes.pin_memory()
        V_u = V.cpu().pin_memory()
        Kb_u = Kb.cpu().pin_memory()
    else:
        codes_u, V_u, Kb_u = codes.to(dev), V, Kb
    out, lse = F.sparse_attention(q, None, V_u, idx_t, scale, k_codes=codes_u,
                                  k_qmin=qmin.to(dev), k_qscale=qscale.to(dev),
                                  host_mapped=host_mapped)
    torch.cuda.synchronize()
    Kd = _dequant_rows(codes.numpy(), qmin.numpy(), qscale.numpy())
    ref_o, ref_l = oracle.sparse_attention(_np(q.float()).astype(np.float64), Kd,
                                           _np(V.float()), idx, scale)
    _check_attention(out, lse, ref_o, ref_l, V, "4-bit keys n=%d d=%d host=%d" % (n, d, host_mapped))
    if host_mapped:
        out2, lse2 = F.sparse_attention(q, Kb_u, V_u, idx_t, scale, host_mapped=True)
        torch.cuda.synchronize()
        ref_o2, ref_l2 = oracle.sparse_attention(_np(q.float()).astype(np.float64),
                                                 _np(Kb.float()), _np(V.float()), idx, scale)
        _check_attention(out2, lse2, ref_o2, ref_l2, V, "host bf16 keys n=%d d=%d" % (n, d))


def test_sparse_attention_after_the_scan(decode_1m):
    """The step after the 1M-token scan: attention over each head's top-2048."""
    dev = torch.device("cuda")
    _, _, (idx, _) = run_gpu(decode_1m, 92, 2048)
    n, d = decode_1m.n, decode_1m.d
    K = _bf16_rows((decode_1m.h_kv, n, d), 21, dev)
    V = _bf16_rows((decode_1m.h_kv, n, d), 22, dev)
    q = decode_1m.q_storage().to(dev)
    out, lse = F.sparse_attention(q, K, V, idx)
    torch.cuda.synchronize()
    ref_o, ref_l = _attention_ref(q, K, V, idx, 1.0 / np.sqrt(d), decode_1m.h_kv)
    _check_attention(out, lse, ref_o, ref_l, V, "1M top-2048")
    del K, V


# ----------------------------------------------------------------- append --

@pytest.mark.parametrize("n,m,d,h_kv", [(0, 1, 128, 1), (1, 1, 128, 2), (31, 1, 64, 1), (32, 1, 128, 1),
                                        (127, 1, 128, 2), (128, 1, 128, 1), (1000, 37, 256, 1),
                                        (4096, 200, 32, 3), (5000, 1, 96, 2), (777, 0, 128, 1)])
def test_append_equals_packing_everything(n, m, d, h_kv):
    """Appending m decoded tokens to a packed store of n gives the store of
    all n + m tokens, bit for bit (in place while the row length holds)."""
    rng = np.random.default_rng(n * 7 + m + d)
    codes = rng.integers(0, 256, size=(h_kv, n + m, d // 2), dtype=np.uint8)
    dev = torch.device("cuda")
    old = torch.from_numpy(np.ascontiguousarray(codes[:, :n])).to(dev)
    new = torch.from_numpy(np.ascontiguousarray(codes[:, n:])).to(dev)
    planes = F.pack_planes(old) if n > 0 else torch.empty((h_kv, d, 4, 0), dtype=torch.int32,
                                                           device=dev)
    got = F.append_planes(planes, n, new)
    torch.cuda.synchronize()
    if F.plane_words(n + m) == F.plane_words(n) and n > 0:
        assert got.data_ptr() == planes.data_ptr()
    np.testing.assert_array_equal(_planes_np(got), oracle.pack_planes(codes))


def test_append_token_by_token():
    """A store grown one token at a time equals one packed at once."""
    case = synthkv.make_case(seed=31, n=300, h_kv=1, h_q=4, d=128, q_dtype="bf16")
    dev = torch.device("cuda")
    codes = case.codes.to(dev)
    planes = F.pack_planes(codes[:, :250].contiguous())
    for i in range(250, 300):
        planes = F.append_planes(planes, i, codes[:, i:i + 1].contiguous())
    torch.cuda.synchronize()
    np.testing.assert_array_equal(_planes_np(planes), oracle.pack_planes(_np(case.codes)))


# ------------------------------------------- per-token-group statistics --

def _group_tol(flags, q_h, qmin_gg, qscale_gg, t_h):
    """_tol with the worst token group's bound (each group has its own Delta_h
    and score scale)."""
    if flags & (F.FLAG_CUDA_CORES | F.FLAG_FORCE_FALLBACK):
        return dict(floor=max(score_scale(q_h, m, s) for m, s in zip(qmin_gg, qscale_gg)) / 8.0)
    return dict(abs_tol=max(fixed_point_bound(q_h, s, t_h) for s in qscale_gg))


@pytest.mark.parametrize("n,tg,k,flags", [(200003, 65536, 256, 0), (131072, 131072, 100, 0),
                                          (70000, 65536, 1024, 0), (150001, 65536, 64, 2),
                                          (140000, 65536, 300, 1), (65536, 65536 * 4, 50, 0)])
def test_token_group_statistics(n, tg, k, flags):
    """The quantiser variant with (m, s) per run of tg keys: dense scores and the
    top-k of every head against the oracle's grouped scores (ragged last group,
    one group spanning the context, forced fallback, no sampling)."""
    case = synthkv.make_case(seed=70 + n % 97, n=n, h_kv=2, h_q=8, d=128, q_dtype="bf16",
                             token_group=tg)
    dev = torch.device("cuda")
    q = case.q_storage().to(dev)
    alloc = F.allocate(q, case.sigma.to(dev), 92)
    planes = F.pack_planes(case.codes.to(dev))
    idx, sc, dbg = F.scan_topk(planes, case.qmin.to(dev), case.qscale.to(dev), q, alloc, k, n,
                               flags=flags, debug_scores=True, token_group=tg)
    torch.cuda.synchronize()
    assert F.read_report().device_faults == 0
    codes, qmin, qscale = _np(case.codes), _np(case.qmin), _np(case.qscale)
    qd = _np(case.q).astype(np.float64)
    want = oracle.allocate_heads(qd, _np(case.sigma), 92)
    np.testing.assert_array_equal(_np(alloc), want)
    for h in range(8):
        g = h // 4
        ref = oracle.scores_from_codes_grouped(codes[g], qmin[g], qscale[g], qd[h], want[h], tg)
        scale = max(score_scale(qd[h], m, s) for m, s in zip(qmin[g], qscale[g]))
        check_dense(_np(dbg)[h], ref, scale, "tg=%d head %d" % (tg, h))
        check_topk(_np(idx)[h], _np(sc)[h], ref, k, what="tg=%d flags=%d head %d" % (tg, flags, h),
                   **_group_tol(flags, qd[h], qmin[g], qscale[g], want[h]))


@pytest.mark.parametrize("d", [64, 256])
def test_token_groups_host_mapped_planes(d):
    """Token groups with the planes in pinned host memory: the same answer as
    from device memory, and the oracle's top-k."""
    n, tg, k = 140000, 65536, 100
    case = synthkv.make_case(seed=91, n=n, h_kv=1, h_q=4, d=d, q_dtype="bf16", token_group=tg)
    dev = torch.device("cuda")
    q = case.q_storage().to(dev)
    alloc = F.allocate(q, case.sigma.to(dev), 92)
    planes = F.pack_planes(case.codes.to(dev))
    hp = torch.empty(planes.shape, dtype=planes.dtype, pin_memory=True)
    hp.copy_(planes)
    qmin, qscale = case.qmin.to(dev), case.qscale.to(dev)
    i0, s0 = F.scan_topk(planes, qmin, qscale, q, alloc, k, n, token_group=tg)
    i1, s1 = F.scan_topk(hp, qmin, qscale, q, alloc, k, n, token_group=tg, host_mapped=True)
    torch.cuda.synchronize()
    assert torch.equal(i0, i1) and torch.equal(s0, s1)
    codes, m, s = _np(case.codes), _np(case.qmin), _np(case.qscale)
    qd = _np(case.q).astype(np.float64)
    want = oracle.allocate_heads(qd, _np(case.sigma), 92)
    for h in range(4):
        ref = oracle.scores_from_codes_grouped(codes[0], m[0], s[0], qd[h], want[h], tg)
        check_topk(_np(i1)[h], _np(s1)[h], ref, k, what="host tg d=%d head %d" % (d, h),
                   **_group_tol(0, qd[h], m[0], s[0], want[h]))


def test_token_groups_with_shared_statistics_change_nothing():
    """Every token group holding the context's (m, s): the same top-k, bit for
    bit, as the per-channel scan (the plans are equal; only the segments split)."""
    n, tg, k = 300000, 65536, 500
    case = synthkv.make_case(seed=88, n=n, h_kv=2, h_q=8, d=128, q_dtype="bf16")
    dev = torch.device("cuda")
    q = case.q_storage().to(dev)
    alloc = F.allocate(q, case.sigma.to(dev), 92)
    planes = F.pack_planes(case.codes.to(dev))
    qmin, qscale = case.qmin.to(dev), case.qscale.to(dev)
    groups = (n + tg - 1) // tg
    qmin_g = qmin[:, None, :].expand(2, groups, 128).contiguous()
    qscale_g = qscale[:, None, :].expand(2, groups, 128).contiguous()
    i0, s0 = F.scan_topk(planes, qmin, qscale, q, alloc, k, n)
    i1, s1 = F.scan_topk(planes, qmin_g, qscale_g, q, alloc, k, n, token_group=tg)
    torch.cuda.synchronize()
    assert torch.equal(i0, i1) and torch.equal(s0, s1)


# ---------------------------------------------------- token-range sharding --

@pytest.mark.parametrize("cuts,k", [((0, 3000, 9000), 50), ((0, 1, 4096, 4097, 20000), 300),
                                    ((0, 20000), 64), ((0, 6000, 12000, 18000, 20000), 2000)])
def test_token_range_shards_merge_to_the_unsplit_topk(cuts, k):
    """The scan split into token ranges (as sharded_scan_topk splits it over
    GPUs, here all on one device): each range packed and scanned on its own,
    the lists merged by fathom_merge_topk, equals the oracle's top-k of the
    whole context."""
    dev = torch.device("cuda")
    n = cuts[-1]
    case = synthkv.make_case(seed=70 + len(cuts), n=n, h_kv=2, h_q=8, d=128, q_dtype="bf16")
    q = case.q_storage().to(dev)
    alloc = F.allocate(q, case.sigma.to(dev), 92)
    codes = case.codes.to(dev)
    idx_parts, sc_parts = [], []
    for lo, hi in zip(cuts[:-1], cuts[1:]):
        planes = F.pack_planes(codes[:, lo:hi].contiguous())
        i, s = F.scan_topk(planes, case.qmin.to(dev), case.qscale.to(dev), q, alloc, k, hi - lo)
        idx_parts.append(i)
        sc_parts.append(s)
    mi, ms = F.merge_topk(torch.stack(idx_parts), torch.stack(sc_parts), list(cuts[:-1]), k)
    torch.cuda.synchronize()
    cn = case_np(case)
    want = oracle.allocate_heads(cn[3], _np(case.sigma), 92)
    for h in range(case.h_q):
        ref = oracle_head(cn, h, want[h])
        check_topk(_np(mi)[h], _np(ms)[h], ref, k, what="shards %s head %d" % (cuts, h),
                   **_tol(0, cn[3][h], cn[1][h // 4], cn[2][h // 4], want[h]))


def test_merge_topk_hand_lists():
    """Hand-made partial lists: equal scores go to the lower global index,
    padding is skipped, and fewer entries than k leave -1 / -inf."""
    dev = torch.device("cuda")
    idx = torch.tensor([[[2, 0, -1]], [[1, 0, -1]]], dtype=torch.int32, device=dev)
    sc = torch.tensor([[[5.0, 3.0, -np.inf]], [[5.0, 4.0, -np.inf]]], dtype=torch.float32,
                      device=dev)
    mi, ms = F.merge_topk(idx, sc, [0, 10], 5)
    torch.cuda.synchronize()
    assert _np(mi)[0].tolist() == [2, 11, 10, 0, -1]
    assert _np(ms)[0][:4].tolist() == [5.0, 5.0, 4.0, 3.0] and np.isneginf(_np(ms)[0][4])
