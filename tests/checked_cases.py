"""Small scans run on the checked build (libfathom_checked.so: device bounds
checks on every plane-row, sample and candidate index the kernels use).
Run as a script with FATHOM_LIB=checked; exits non-zero on a failure.  Each
case must give the oracle's answer and record no device fault."""

import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
sys.path.insert(0, os.path.join(ROOT, "tests"))

import numpy as np  # noqa: E402
import torch  # noqa: E402

import oracle  # noqa: E402
import synthkv  # noqa: E402
from parity import check_topk, fixed_point_bound, score_scale  # noqa: E402


def run():
    import bit_plane_kv_scan_b200 as F
    from bit_plane_kv_scan_b200 import fathom
    assert fathom.LIB_PATH.endswith("libfathom_checked.so"), fathom.LIB_PATH
    F.lib()
    dev = torch.device("cuda")
    cases = [(4096, 1, 92, 64, 0), (4097, 4, 92, 7, 0), (12345, 2, 17, 100, 0), (40000, 4, 92, 64, 0),
             (3000, 4, 0, 50, 0), (3000, 4, 512, 50, 0), (40000, 4, 136, 64, F.FLAG_CUDA_CORES),
             (5000, 2, 92, 33, F.FLAG_CUDA_CORES), (40000, 4, 92, 64, F.FLAG_FORCE_FALLBACK),
             (20000, 4, 92, 64, F.FLAG_NO_SAMPLING)]
    # tiny contexts and the narrowest channel count as well (n = 33, 64, 4096 at d = 32)
    cases = [(n, G, B, k, flags, 128) for n, G, B, k, flags in cases] + \
        [(33, 1, 17, 5, 0, 32), (64, 2, 92, 10, 0, 32), (4096, 4, 64, 50, 0, 32),
         (64, 2, 92, 10, F.FLAG_CUDA_CORES, 32)]
    for n, G, B, k, flags, d in cases:
        case = synthkv.make_case(seed=900 + n + G, n=n, h_kv=2, h_q=2 * G, d=d, q_dtype="bf16")
        q = case.q_storage().to(dev)
        alloc = F.allocate(q, case.sigma.to(dev), B)
        planes = F.pack_planes(case.codes.to(dev))
        idx, sc = F.scan_topk(planes, case.qmin.to(dev), case.qscale.to(dev), q, alloc, k, n,
                              flags=flags)
        torch.cuda.synchronize()
        F.check_device_status()  # raises on a recorded device fault
        rep = F.read_report()
        assert rep.device_faults == 0
        codes, qd = case.codes.numpy(), case.q.numpy().astype(np.float64)
        want = oracle.allocate_heads(qd, case.sigma.numpy(), B)
        for h in range(case.h_q):
            g = h // G
            m, s = case.qmin.numpy()[g], case.qscale.numpy()[g]
            ref = oracle.scores_from_codes(codes[g], m, s, qd[h], want[h])
            if flags & (F.FLAG_CUDA_CORES | F.FLAG_FORCE_FALLBACK):
                tol = dict(floor=score_scale(qd[h], m, s) / 8.0)
            else:
                tol = dict(abs_tol=fixed_point_bound(qd[h], s, want[h]))
            check_topk(idx.cpu().numpy()[h], sc.cpu().numpy()[h], ref, k,
                       what="checked n=%d G=%d B=%d flags=%d head %d" % (n, G, B, flags, h), **tol)
        print("ok n=%d G=%d B=%d k=%d flags=%d" % (n, G, B, k, flags))
    # per-token-group statistics: plans per token group, segments split at
    # group boundaries, and the exact fallback walking the groups
    for n, tg, k, flags in ((140001, 65536, 64, 0), (140001, 65536, 64, F.FLAG_FORCE_FALLBACK)):
        case = synthkv.make_case(seed=977, n=n, h_kv=2, h_q=8, d=128, q_dtype="bf16",
                                 token_group=tg)
        q = case.q_storage().to(dev)
        alloc = F.allocate(q, case.sigma.to(dev), 92)
        planes = F.pack_planes(case.codes.to(dev))
        idx, sc = F.scan_topk(planes, case.qmin.to(dev), case.qscale.to(dev), q, alloc, k, n,
                              flags=flags, token_group=tg)
        torch.cuda.synchronize()
        F.check_device_status()
        codes, qd = case.codes.numpy(), case.q.numpy().astype(np.float64)
        want = oracle.allocate_heads(qd, case.sigma.numpy(), 92)
        for h in range(8):
            g = h // 4
            m, s = case.qmin.numpy()[g], case.qscale.numpy()[g]
            ref = oracle.scores_from_codes_grouped(codes[g], m, s, qd[h], want[h], tg)
            if flags & F.FLAG_FORCE_FALLBACK:
                tol = dict(floor=max(score_scale(qd[h], a, b) for a, b in zip(m, s)) / 8.0)
            else:
                tol = dict(abs_tol=max(fixed_point_bound(qd[h], b, want[h]) for b in s))
            check_topk(idx.cpu().numpy()[h], sc.cpu().numpy()[h], ref, k,
                       what="checked token groups flags=%d head %d" % (flags, h), **tol)
        print("ok token_group=%d n=%d flags=%d" % (tg, n, flags))
    # the batched launch over ragged sessions
    sessions = [synthkv.make_case(seed=950 + i, n=n, h_kv=2, h_q=8, d=128, q_dtype="bf16")
                for i, n in enumerate((9000, 20001, 3333))]
    descs = []
    for s in sessions:
        q = s.q_storage().to(dev)
        descs.append(dict(planes=F.pack_planes(s.codes.to(dev)), qmin=s.qmin.to(dev),
                          qscale=s.qscale.to(dev), q=q, alloc=F.allocate(q, s.sigma.to(dev), 92),
                          n=s.n))
    outs = F.scan_topk_batched(descs, 50, 128, 8, 2, torch.bfloat16)
    torch.cuda.synchronize()
    assert F.read_report().device_faults == 0
    for i, s in enumerate(sessions):
        qd = s.q.numpy().astype(np.float64)
        want = oracle.allocate_heads(qd, s.sigma.numpy(), 92)
        for h in range(8):
            g = h // 4
            ref = oracle.scores_from_codes(s.codes.numpy()[g], s.qmin.numpy()[g],
                                           s.qscale.numpy()[g], qd[h], want[h])
            check_topk(outs[i][0].cpu().numpy()[h], outs[i][1].cpu().numpy()[h], ref, 50,
                       what="checked batched session %d head %d" % (i, h),
                       abs_tol=fixed_point_bound(qd[h], s.qscale.numpy()[g], want[h]))
    print("ok batched")
    return 0


if __name__ == "__main__":
    sys.exit(run())
