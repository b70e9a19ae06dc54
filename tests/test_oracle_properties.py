"""Property checks of the oracle on random inputs (hypothesis), beside the
hand-picked pins of test_oracle_pins.py: many exact ties in the allocation's
slot values, random token-group layouts, and top-k over heavily tied scores.
Each property is stated from its definition, independently of the oracle's
code."""

import os
import sys

import numpy as np
from hypothesis import given, settings, strategies as st

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

import oracle  # noqa: E402

SETTINGS = settings(max_examples=60, deadline=None)


@SETTINGS
@given(st.data())
def test_allocation_is_the_b_best_slots_with_ties_by_slot_order(data):
    """Reverse water-filling as slot selection: channel c offers slots (c, tau)
    worth w_c 4^-tau; the B best are taken, equal values by lower 4c + tau."""
    d = data.draw(st.sampled_from([8, 16, 32]))
    # values from a small set, so that slot values tie often (w = q^2 sigma^2
    # and 4^-tau scale by powers of two)
    q = np.array(data.draw(st.lists(st.sampled_from([0.0, 0.5, -1.0, 1.0, 2.0, -2.0]),
                                    min_size=d, max_size=d)), dtype=np.float64)
    sigma = np.array(data.draw(st.lists(st.sampled_from([0.0, 0.5, 1.0, 2.0]),
                                        min_size=d, max_size=d)), dtype=np.float32)
    B = data.draw(st.integers(0, 4 * d))
    t = oracle.allocate(q, sigma, B).astype(int)
    w = (q * q) * (sigma.astype(np.float64) ** 2)
    slots = sorted(((w[c] * 4.0 ** -tau, -(4 * c + tau)) for c in range(d) for tau in range(4)),
                   reverse=True)  # value desc, then slot index asc
    taken = {-s for _, s in slots[:B]}
    want = np.zeros(d, dtype=int)
    for s in taken:
        want[s // 4] += 1
    # the B best slots hold each channel's first slots (values fall with tau),
    # so counting them per channel gives the allocation
    assert sorted(taken) == sorted(4 * c + tau for c in range(d) for tau in range(want[c]))
    np.testing.assert_array_equal(t, want)


@SETTINGS
@given(st.data())
def test_grouped_scores_by_definition(data):
    """Key i's score uses its own token group's (m, s): the cell-centre
    reconstruction summed over channels, for random layouts and allocations."""
    d = data.draw(st.sampled_from([2, 4, 8]))
    n = data.draw(st.integers(1, 150))
    tg = data.draw(st.integers(1, 64))
    groups = (n + tg - 1) // tg
    rng = np.random.default_rng(data.draw(st.integers(0, 2**31 - 1)))
    u = rng.integers(0, 16, size=(n, d)).astype(np.uint8)
    codes = (u[:, 0::2] | (u[:, 1::2] << 4)).astype(np.uint8)
    m = rng.normal(size=(groups, d)).astype(np.float32)
    s = rng.uniform(0.0, 2.0, size=(groups, d)).astype(np.float32)
    q = rng.normal(size=d)
    t = rng.integers(0, 5, size=d).astype(np.uint8)
    got = oracle.scores_from_codes_grouped(codes, m, s, q, t, tg)
    cell = 2.0 ** (4 - t.astype(np.float64))
    v = (u.astype(np.int64) >> (4 - t.astype(np.int64))).astype(np.float64)
    g = np.arange(n) // tg
    deq = m[g].astype(np.float64) + s[g].astype(np.float64) * (cell * v + (cell - 1.0) / 2.0)
    want = deq @ q
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-12 * max(1.0, np.abs(want).max()))


@SETTINGS
@given(st.lists(st.sampled_from([-1.5, 0.0, 0.25, 2.0, 7.0]), min_size=0, max_size=200),
       st.integers(1, 64))
def test_topk_over_tied_scores(scores, k):
    """Score descending, equal scores by index ascending; -1 / -inf padding."""
    sc = np.array(scores, dtype=np.float64)
    idx, val = oracle.topk(sc, k)
    order = sorted(range(len(scores)), key=lambda i: (-scores[i], i))[:k]
    kk = len(order)
    assert list(idx[:kk]) == order
    np.testing.assert_array_equal(val[:kk], sc[order])
    assert (idx[kk:] == -1).all() and np.isneginf(val[kk:]).all()
