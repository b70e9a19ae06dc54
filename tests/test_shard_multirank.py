"""Token-range sharding (the scan split over GPUs by ranges of the context),
host side, on CPU with two gloo ranks.

Each rank takes a contiguous range of one context's keys and computes that
range's top-k (here with the oracle, in local indices); gather_parts, the
collective step of bit_plane_kv_scan_b200.sharded_scan_topk, brings every
rank's lists and key count to every rank; merging them must give the
oracle's top-k of the whole context.  The merge itself is the oracle's
top-k over the gathered candidates placed at their global indices (the
CUDA merge, fathom_merge_topk, is checked against the same rule on the GPU).
"""

import os
import socket
import sys

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _case():
    import synthkv
    return synthkv.make_case(seed=61, n=9000, h_kv=2, h_q=8, d=64, q_dtype="bf16")


def _oracle_scores(case, t):
    import oracle
    codes = case.codes.numpy()
    q = case.q.numpy().astype(np.float64)
    G = case.h_q // case.h_kv
    return [oracle.scores_from_codes(codes[h // G], case.qmin.numpy()[h // G],
                                     case.qscale.numpy()[h // G], q[h], t[h])
            for h in range(case.h_q)]


def merge_with_oracle(idx_parts, sc_parts, offsets, n_total, k):
    """The oracle rule for merging partial lists: every gathered candidate at
    its global index in a dense score row (-inf elsewhere), then the oracle's
    top-k (score desc, index asc), -1 past the gathered entries."""
    import oracle
    parts, h_q, _ = idx_parts.shape
    out_i = np.zeros((h_q, k), dtype=np.int32)
    out_s = np.zeros((h_q, k), dtype=np.float64)
    for h in range(h_q):
        row = np.full(n_total, -np.inf)
        for p in range(parts):
            li = idx_parts[p, h]
            keep = li >= 0
            row[offsets[p] + li[keep]] = sc_parts[p, h][keep]
        out_i[h], out_s[h] = oracle.topk(row, k)
        out_i[h][np.isneginf(out_s[h])] = -1  # past the gathered entries
    return out_i, out_s


def _worker(rank, world, port, k, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import oracle
        from bit_plane_kv_scan_b200.fathom import gather_parts
        case = _case()
        oracle.build()
        t = oracle.allocate_heads(case.q.numpy().astype(np.float64), case.sigma.numpy(), 40)
        scores = _oracle_scores(case, t)
        # uneven ranges: rank 0 takes 3000 keys, rank 1 the other 6000
        cut = [0, 3000, case.n][:world + 1] if world == 2 else None
        lo, hi = cut[rank], cut[rank + 1]
        idx = np.zeros((case.h_q, k), dtype=np.int32)
        sc = np.zeros((case.h_q, k), dtype=np.float32)
        for h in range(case.h_q):
            li, ls = oracle.topk(scores[h][lo:hi], k)
            idx[h], sc[h] = li, ls.astype(np.float32)
        ip, sp, offsets = gather_parts(torch.from_numpy(idx), torch.from_numpy(sc), hi - lo)
        mi, ms = merge_with_oracle(ip.numpy(), sp.numpy().astype(np.float64), offsets, case.n, k)
        results[rank] = (offsets, mi.tolist(), ms.tolist())
    finally:
        dist.destroy_process_group()


def test_two_rank_token_sharding_equals_the_unsplit_topk():
    import oracle
    oracle.build()
    world, k = 2, 50
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        results = m.dict()
        procs = [ctx.Process(target=_worker, args=(r, world, port, k, results))
                 for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(300)
            assert p.exitcode == 0
        res = dict(results)
    case = _case()
    t = oracle.allocate_heads(case.q.numpy().astype(np.float64), case.sigma.numpy(), 40)
    scores = _oracle_scores(case, t)
    for r in range(world):
        offsets, mi, ms = res[r]
        assert offsets == [0, 3000]
        for h in range(case.h_q):
            want_i, want_s = oracle.topk(scores[h], k)
            # the partial lists carry fp32 scores: the same keys, in the same
            # order, unless two keys' fp32 scores tie
            np.testing.assert_array_equal(np.sort(mi[h]), np.sort(want_i))
            np.testing.assert_allclose(ms[h], want_s, rtol=1e-6)


def test_merge_rule_on_hand_lists():
    """Two ranges' lists by hand: ties by score go to the lower global index,
    padding is ignored, and fewer entries than k leave -1."""
    import oracle
    oracle.build()
    idx = np.array([[[2, 0, -1]], [[1, 0, -1]]], dtype=np.int32)     # [parts=2][h=1][3]
    sc = np.array([[[5.0, 3.0, -np.inf]], [[5.0, 4.0, -np.inf]]])
    mi, ms = merge_with_oracle(idx, sc, [0, 10], 20, 5)
    assert mi[0].tolist() == [2, 11, 10, 0, -1]
    assert ms[0][:4].tolist() == [5.0, 5.0, 4.0, 3.0] and np.isneginf(ms[0][4])
