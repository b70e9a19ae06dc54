"""Design check (CPU, oracle scores): how many candidates each threshold rule
lets through on the 1M-key decode workload, for one KV head and its 4 query
heads (B = 92, k = 2048).

  * two-pass (what the library does): score every 64th 256-key sector first,
    take the r-th best sampled score as tau (r = max(16, ceil(k / 32))), then
    keep every key whose score reaches tau;
  * single pass, running threshold: each CTA of the persistent scan keeps the
    k best scores it has seen and publishes its k-th best; a key is kept when
    it reaches the largest published value so far.  Simulated here in the
    scan's own partition (contiguous runs of about 55 tiles of 1024 keys per
    CTA, about 19 CTAs per KV head), optimistically: every CTA sees every
    other CTA's latest value at once.

Both rules keep the exact top-k (tau never exceeds the k-th best score).  The
running threshold cannot be set before a CTA has seen k keys, so each CTA's
first two tiles pass whole; it lets through several times the two-pass
candidates, which the merge then has to rank.
"""

import os
import sys

import numpy as np

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

import oracle  # noqa: E402
import synthkv  # noqa: E402

TILE = 1024
SECTOR = 256
STRIDE = 64


def _two_pass(scores, k):
    n = scores.shape[0]
    sectors = (n + SECTOR - 1) // SECTOR
    picked = np.concatenate([scores[j * SECTOR:min(n, (j + 1) * SECTOR)]
                             for j in range(0, sectors, STRIDE)])
    r = max(16, (k + 31) // 32)
    tau = np.sort(picked)[::-1][r - 1]
    return int((scores >= tau).sum()), tau


def _running(scores, k, ctas):
    n = scores.shape[0]
    tiles = (n + TILE - 1) // TILE
    bounds = np.linspace(0, tiles, ctas + 1).round().astype(int)
    seen = [np.empty(0) for _ in range(ctas)]
    tau = -np.inf
    passed = 0
    for step in range(int(np.diff(bounds).max())):
        kth = []
        for c in range(ctas):
            t = bounds[c] + step
            if t >= bounds[c + 1]:
                continue
            keys = scores[t * TILE:min(n, (t + 1) * TILE)]
            passed += int((keys >= tau).sum())
            seen[c] = np.concatenate([seen[c], keys])
            if seen[c].size > k:
                seen[c] = np.partition(seen[c], seen[c].size - k)[-k:]
            if seen[c].size >= k:
                kth.append(seen[c].min())
        if kth:
            tau = max(tau, max(kth))
    return passed


def test_two_pass_threshold_admits_fewer_candidates_than_a_running_one():
    n, k, budget = 1 << 20, 2048, 92
    case = synthkv.make_case(2, n, 1, 4, 128, "bf16", device="cpu", keep_keys=False)
    codes = case.codes.numpy()
    q = case.q_storage().float().numpy().astype(np.float64)
    alloc = oracle.allocate_heads(q, case.sigma.numpy(), budget)
    ctas = round(1024 / (8192 / 148))  # the 1M step's tiles per CTA, per KV head
    for h in range(4):
        s = oracle.scores_from_codes(codes[0], case.qmin.numpy()[0], case.qscale.numpy()[0],
                                     q[h], alloc[h])
        kth = np.sort(s)[::-1][k - 1]
        two, tau = _two_pass(s, k)
        run = _running(s, k, ctas)
        print("head %d: two-pass %d candidates, running threshold %d (k = %d)" % (h, two, run, k))
        assert tau <= kth and two >= k  # the sampled threshold keeps the top-k here
        assert run >= 3 * two
