"""Comparison rules between the CUDA scan and the CPU oracle.

Tolerances (stated here once, used by every parity test):
  * plane words and bit allocations: bit-exact;
  * a returned top-k score: |s_gpu - s_ref| <= 1e-5 |s_ref| (the bare
    relative bound of the contract: fp32 scores against the fp64 oracle).
    The tensor-core scan sums the plane bits exactly in int32 against
    fixed-point weights X = round(W / Delta_h), Delta_h = 2^(e - 30) with
    8 max_c |q_c s_c| < 2^e, forms C_h + Delta_h sum X b in fp64 and rounds
    once to fp32: |s_gpu - s_ref| <= B Delta_h / 2 + 2^-24 |s_ref| exactly
    (B planes read, each weight off by at most Delta_h / 2).  Its checks pass
    abs_tol = B Delta_h / 2 (fixed_point_bound), which exceeds 1e-5 |s_ref|
    only for a score within ~1e-7 S_h of zero (S_h below);
    The CUDA-core scan accumulates d + 1 fp32 terms whose running value
    reaches ~2 S_h (S_h = sum_c |q_c| max(|m_c|, |m_c + 15 s_c|) bounds every
    score of head h): an absolute error of order sqrt(d) 2^-24 2 S_h.  Its
    checks may pass floor=S_h/8, i.e. |err| <= 1e-5 max(|s_ref|, S_h / 8),
    which matters only for a returned score below S_h / 8;
  * every score of a dense (debug) dump: |s_gpu - s_ref| <= 1e-5 S_h (a bare
    relative bound is ill-posed for scores near 0, where the parts cancel);
  * top-k sets: identical except for keys whose oracle score lies within
    1e-5 max(|s_k|, floor) of the oracle's k-th score s_k (where more than one
    set is correct); the returned list is sorted by score descending, equal
    fp32 scores by index ascending, and indices are distinct and in range.
"""

import numpy as np

REL = 1e-5


def score_scale(q_h, qmin_g, qscale_g) -> float:
    q = np.abs(np.asarray(q_h, dtype=np.float64))
    m = np.asarray(qmin_g, dtype=np.float64)
    s = np.asarray(qscale_g, dtype=np.float64)
    return float(np.sum(q * np.maximum(np.abs(m), np.abs(m + 15.0 * s))))


def fixed_point_bound(q_h, qscale_g, t_h) -> float:
    """B Delta_h / 2: the largest error the tensor-core scan's fixed-point
    weights can put into a score of head h (B = sum_c t_c planes read, each
    weight W = q_c s_c 2^(3-j) rounded to a multiple of Delta_h)."""
    import math
    q = np.asarray(q_h, dtype=np.float64)
    s = np.asarray(qscale_g, dtype=np.float64)
    t = np.asarray(t_h)
    w = np.abs(q * s)[t > 0]
    if w.size == 0 or w.max() == 0.0:
        return 0.0
    _, e = math.frexp(8.0 * float(w.max()))  # 8 max|q s| < 2^e
    return float(t.sum()) * math.ldexp(1.0, e - 30) / 2.0


def score_tol(ref, floor=0.0, abs_tol=0.0):
    ref = np.abs(np.asarray(ref, dtype=np.float64))
    return np.maximum(REL * np.maximum(ref, floor), abs_tol + 2.0 ** -23 * ref)


def check_scores_at(gpu_scores, ref_scores, floor=0.0, what="", abs_tol=0.0):
    """Returned scores against the oracle's at the same keys; returns the
    largest bare relative error |s - s_ref| / |s_ref|."""
    g = np.asarray(gpu_scores, dtype=np.float64)
    r = np.asarray(ref_scores, dtype=np.float64)
    err = np.abs(g - r)
    tol = score_tol(r, floor, abs_tol)
    bad = np.nonzero(err > tol)[0]
    assert bad.size == 0, "%s: %d scores off, worst |err|=%g at ref=%g (tol %g)" % (
        what, bad.size, err[bad].max(), r[bad[np.argmax(err[bad])]], tol[bad].min())
    return float((err / np.maximum(np.abs(r), 1e-300)).max()) if r.size else 0.0


def check_dense(gpu_scores, ref_scores, scale, what=""):
    g = np.asarray(gpu_scores, dtype=np.float64)
    r = np.asarray(ref_scores, dtype=np.float64)
    err = np.abs(g - r).max() if r.size else 0.0
    assert err <= REL * scale, "%s: dense scores off by %g > %g" % (what, err, REL * scale)
    return err / scale if scale else 0.0


def check_topk(idx, sc, ref_scores, k, floor=0.0, what="", abs_tol=0.0):
    """idx/sc: the GPU's k results for one head; ref_scores: oracle scores of
    all n keys.  Returns the largest bare relative error of the returned scores."""
    idx = np.asarray(idx).astype(np.int64)
    sc = np.asarray(sc, dtype=np.float32)
    ref = np.asarray(ref_scores, dtype=np.float64)
    n = ref.shape[0]
    kk = min(k, n)
    assert (idx[kk:] == -1).all() and np.isneginf(sc[kk:]).all(), what + ": padding"
    gi, gs = idx[:kk], sc[:kk]
    assert (gi >= 0).all() and (gi < n).all(), what + ": index out of range"
    assert np.unique(gi).size == kk, what + ": repeated index"
    # order: score desc, then index asc among equal scores
    assert (np.diff(gs.astype(np.float64)) <= 0).all(), what + ": not sorted by score"
    eq = gs[1:] == gs[:-1]
    assert (gi[1:][eq] > gi[:-1][eq]).all(), what + ": equal scores not by index"
    if kk == 0:
        return 0.0
    rel = check_scores_at(gs, ref[gi], floor, what, abs_tol)
    order = np.lexsort((np.arange(n), -ref))
    ref_k = ref[order[kk - 1]]
    band = max(REL * max(abs(ref_k), floor), 2.0 * (abs_tol + 2.0 ** -23 * abs(ref_k)))
    want = set(order[:kk].tolist())
    got = set(gi.tolist())
    for i in got ^ want:
        assert abs(ref[i] - ref_k) <= band, "%s: key %d (ref %.9g) differs from the oracle set " \
            "outside the near-tie band around the k-th score %.9g" % (what, i, ref[i], ref_k)
    return rel


def check_topk_sampled(idx, sc, ref_at, k, n, floor=0.0, what="", abs_tol=0.0):
    """Checks that need no full oracle scan: structure, and the returned scores
    against oracle scores at the returned indices (ref_at[i] for i < min(k, n))."""
    idx = np.asarray(idx).astype(np.int64)
    sc = np.asarray(sc, dtype=np.float32)
    kk = min(k, n)
    assert (idx[kk:] == -1).all(), what
    gi, gs = idx[:kk], sc[:kk]
    assert (gi >= 0).all() and (gi < n).all() and np.unique(gi).size == kk, what
    assert (np.diff(gs.astype(np.float64)) <= 0).all(), what
    return check_scores_at(gs, ref_at, floor, what, abs_tol)
