"""Comparison rules between the CUDA scan and the CPU oracle.

Tolerances (stated here once, used by every parity test):
  * plane words and bit allocations: bit-exact;
  * a score: |s_gpu - s_ref| <= 1e-5 max(|s_ref|, S_h / 8) (fp32 accumulation
    against fp64), where S_h = sum_c |q_c| max(|m_c|, |m_c + 15 s_c|) bounds
    every score of head h.  A bare relative bound is ill-posed for scores
    near 0: an fp32 sum of d + 1 terms whose running value reaches ~2 S_h
    carries an absolute rounding error of order sqrt(d) 2^-24 2 S_h
    (~1.4e-6 S_h at d = 128, ~3e-7 S_h observed), so below |s_ref| = S_h / 8
    the bound stays at 1.25e-6 S_h;
  * every score of a dense (debug) dump: |s_gpu - s_ref| <= 1e-5 S_h;
  * top-k sets: identical except for keys whose oracle score lies within
    1e-5 max(|s_k|, S_h / 8) of the oracle's k-th score s_k (where more than
    one set is correct); the returned list is sorted by score descending, equal fp32
    scores by index ascending, and indices are distinct and in range.
"""

import numpy as np

REL = 1e-5


def score_scale(q_h, qmin_g, qscale_g) -> float:
    q = np.abs(np.asarray(q_h, dtype=np.float64))
    m = np.asarray(qmin_g, dtype=np.float64)
    s = np.asarray(qscale_g, dtype=np.float64)
    return float(np.sum(q * np.maximum(np.abs(m), np.abs(m + 15.0 * s))))


def score_tol(ref, scale):
    ref = np.abs(np.asarray(ref, dtype=np.float64))
    return REL * np.maximum(ref, scale / 8.0)


def check_scores_at(gpu_scores, ref_scores, scale, what=""):
    g = np.asarray(gpu_scores, dtype=np.float64)
    r = np.asarray(ref_scores, dtype=np.float64)
    err = np.abs(g - r)
    tol = score_tol(r, scale)
    bad = np.nonzero(err > tol)[0]
    assert bad.size == 0, "%s: %d scores off, worst |err|=%g at ref=%g (tol %g)" % (
        what, bad.size, err[bad].max(), r[bad[np.argmax(err[bad])]], tol[bad].min())
    return float((err / np.maximum(np.abs(r), 1e-30)).max()) if r.size else 0.0


def check_dense(gpu_scores, ref_scores, scale, what=""):
    g = np.asarray(gpu_scores, dtype=np.float64)
    r = np.asarray(ref_scores, dtype=np.float64)
    err = np.abs(g - r).max() if r.size else 0.0
    assert err <= REL * scale, "%s: dense scores off by %g > %g" % (what, err, REL * scale)
    return err / scale if scale else 0.0


def check_topk(idx, sc, ref_scores, k, scale, what=""):
    """idx/sc: the GPU's k results for one head; ref_scores: oracle scores of all n keys."""
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
        return
    check_scores_at(gs, ref[gi], scale, what)
    order = np.lexsort((np.arange(n), -ref))
    ref_k = ref[order[kk - 1]]
    band = REL * max(abs(ref_k), scale / 8.0)
    want = set(order[:kk].tolist())
    got = set(gi.tolist())
    for i in got ^ want:
        assert abs(ref[i] - ref_k) <= band, "%s: key %d (ref %.9g) differs from the oracle set " \
            "outside the near-tie band around the k-th score %.9g" % (what, i, ref[i], ref_k)


def check_topk_sampled(idx, sc, ref_at, k, n, scale, what=""):
    """Checks that need no full oracle scan: structure, and the returned scores
    against oracle scores at the returned indices (ref_at[i] for i < min(k, n))."""
    idx = np.asarray(idx).astype(np.int64)
    sc = np.asarray(sc, dtype=np.float32)
    kk = min(k, n)
    assert (idx[kk:] == -1).all(), what
    gi, gs = idx[:kk], sc[:kk]
    assert (gi >= 0).all() and (gi < n).all() and np.unique(gi).size == kk, what
    assert (np.diff(gs.astype(np.float64)) <= 0).all(), what
    check_scores_at(gs, ref_at, scale, what)
