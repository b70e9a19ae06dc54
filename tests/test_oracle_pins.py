"""Pins of the CPU oracle to what the Fathom pages and mathematics fix.

Nothing here compares the oracle with itself: each check ties it to an input
it must reproduce, a closed form, a hand-worked example, brute force, or a
library routine (numpy matmul / lexsort).

Sources: "Fathom Makes KV-Cache Scans Query-Adaptive for Long-Context
Decoding" (cctest.ai), method paragraphs 2-3; arXiv 2609.17652, abstract.
"""

import itertools
import math
from fractions import Fraction

import numpy as np
import pytest

import oracle
import synthkv


@pytest.fixture(scope="module")
def tiny():
    """A 4096-token, one-head case with its fp32 keys kept."""
    return synthkv.make_case(seed=0, n=4096, h_kv=1, h_q=1, d=128, q_dtype="f32",
                             keep_keys=True)


@pytest.fixture(scope="module")
def small_gqa():
    """A ragged-length GQA case: 2 KV heads, 8 query heads, n not a multiple of 32."""
    return synthkv.make_case(seed=11, n=1000, h_kv=2, h_q=8, d=64, q_dtype="bf16",
                             keep_keys=True)


def _unpack_codes(codes):
    codes = np.asarray(codes)
    u = np.empty(codes.shape[:-1] + (2 * codes.shape[-1],), dtype=np.uint8)
    u[..., 0::2] = codes & 15
    u[..., 1::2] = codes >> 4
    return u


# ---------------------------------------------------------------- packing --

def test_hand_example_planes(golden):
    ex = golden["scan"]
    codes = np.array(ex["codes_bytes"], dtype=np.uint8).reshape(1, ex["n"], ex["d"] // 2)
    planes = oracle.pack_planes(codes)
    assert planes.shape == (1, 2, 4, 4)
    np.testing.assert_array_equal(planes.reshape(8, 4), np.array(ex["planes_words"]))


@pytest.mark.parametrize("n", [1, 31, 32, 33, 127, 128, 129, 1000])
def test_pack_roundtrip_and_padding(n):
    rng = np.random.default_rng(n)
    u = rng.integers(0, 16, size=(2, n, 16), dtype=np.uint8)
    planes = oracle.pack_planes(synthkv.pack_nibbles(__import__("torch").from_numpy(u)).numpy())
    W = oracle.plane_words(n)
    assert W == ((n + 127) // 128) * 4 and W * 32 >= n and W % 4 == 0
    # all four planes give back the codes exactly
    np.testing.assert_array_equal(oracle.prefix_values(planes, n, 4), u)
    # every t-prefix is the code's top t bits
    for t in range(5):
        np.testing.assert_array_equal(oracle.prefix_values(planes, n, t), u >> (4 - t))
    # bits past the last token are zero
    bits = np.unpackbits(planes.view(np.uint8), bitorder="little").reshape(2, 16, 4, W * 32)
    assert not bits[..., n:].any()


def test_prefix_is_the_t_bit_quantiser(tiny):
    """A t-plane prefix equals the t-bit min-max quantiser of the real key:
    Q_t(k) = floor(((k - m)/s + 1/2) / 2^(4-t)) (method paragraph 2)."""
    planes = oracle.pack_planes(tiny.codes.numpy())
    k = tiny.keys.numpy()[0].astype(np.float64)
    m = tiny.qmin.numpy()[0].astype(np.float64)
    s = tiny.qscale.numpy()[0].astype(np.float64)
    x = (k - m) / s
    for t in range(1, 5):
        q_t = np.clip(np.floor((x + 0.5) / 2.0 ** (4 - t)), 0, 2 ** t - 1)
        v = oracle.prefix_values(planes, tiny.n, t)[0]
        assert (v == q_t).all(), t


def test_prefix_quantiser_in_exact_rationals(tiny):
    """Same identity with (k - m)/s taken exactly, on a sample: count the keys
    where float rounding moves a cell boundary (expected none)."""
    planes = oracle.pack_planes(tiny.codes.numpy())
    rng = np.random.default_rng(5)
    ii = rng.integers(0, tiny.n, 1500)
    cc = rng.integers(0, tiny.d, 1500)
    k = tiny.keys.numpy()[0]
    m = tiny.qmin.numpy()[0]
    s = tiny.qscale.numpy()[0]
    disagree = 0
    for t in (1, 2, 3, 4):
        v = oracle.prefix_values(planes, tiny.n, t)[0]
        for i, c in zip(ii, cc):
            x = (Fraction(float(k[i, c])) - Fraction(float(m[c]))) / Fraction(float(s[c]))
            q_t = math.floor((x + Fraction(1, 2)) / 2 ** (4 - t))
            q_t = min(max(q_t, 0), 2 ** t - 1)
            disagree += int(q_t != v[i, c])
    assert disagree == 0


def test_dequant_is_cell_centre():
    """deq_t(v) is the mean of the 4-bit reconstructions m + s*u over the
    codes u whose top t bits are v; t = 4 is m + s*u, t = 0 is m + 7.5 s."""
    m, s = -1.25, 0.375
    for t in range(5):
        cell = 2 ** (4 - t)
        for v in range(2 ** t):
            us = range(v * cell, (v + 1) * cell)
            mean = sum(m + s * u for u in us) / cell
            assert oracle.dequant_prefix(m, s, t, v) == pytest.approx(mean, rel=0, abs=1e-15)
    assert oracle.dequant_prefix(m, s, 4, 9) == m + 9 * s
    assert oracle.dequant_prefix(m, s, 0, 0) == m + 7.5 * s


# ------------------------------------------------------------- allocation --

def test_hand_example_allocation(golden):
    ex = golden["allocation"]
    for B, want in ex["t_by_budget"].items():
        got = oracle.allocate(ex["q"], ex["sigma"], int(B))
        assert got.tolist() == want, B


def _w(q, sigma):
    return (np.asarray(q, np.float64) ** 2) * (np.asarray(sigma, np.float64) ** 2)


def _rand_head(rng, d):
    q = rng.normal(size=d)
    sigma = np.exp(rng.uniform(math.log(0.1), math.log(10), size=d))
    return q, sigma


@pytest.mark.parametrize("B", [0, 1, 5, 68, 92, 136, 255, 256, 511, 512])
def test_allocation_budget_range_and_exchange_optimality(B):
    rng = np.random.default_rng(B)
    for _ in range(5):
        q, sigma = _rand_head(rng, 128)
        t = oracle.allocate(q, sigma, B).astype(int)
        assert t.sum() == B and t.min() >= 0 and t.max() <= 4
        w = _w(q, sigma)
        # no bit can move from c to c' and lower sum_c w_c 4^-t_c
        give = np.where(t > 0, w * 4.0 ** (-(t - 1)), np.inf)   # what c's last bit buys
        take = np.where(t < 4, w * 4.0 ** (-t), -np.inf)        # what c' next bit would buy
        assert give.min() >= take.max()


def test_allocation_extremes():
    rng = np.random.default_rng(1)
    q, sigma = _rand_head(rng, 128)
    assert (oracle.allocate(q, sigma, 0) == 0).all()
    assert (oracle.allocate(q, sigma, 512) == 4).all()


def test_allocation_zero_weights_take_leftover_bits_in_channel_order():
    q = np.zeros(8)
    q[[2, 5]] = [1.0, -3.0]
    sigma = np.ones(8)
    t = oracle.allocate(q, sigma, 13)
    # 8 bits fill channels 5 and 2; the other 5 go to the zero channels in
    # (channel, tau) order: channel 0 takes 4, channel 1 takes 1.
    assert t.tolist() == [4, 1, 4, 0, 0, 4, 0, 0]


def test_allocation_brute_force_d8():
    """For d = 8 enumerate all 5^8 allocations; the oracle's reaches the
    minimum of sum_c w_c 4^-t_c at every budget 0..32."""
    rng = np.random.default_rng(7)
    allt = np.array(list(itertools.product(range(5), repeat=8)), dtype=np.int64)
    sums = allt.sum(1)
    for trial in range(6):
        q, sigma = _rand_head(rng, 8)
        if trial == 5:  # exact ties between channels
            q = np.array([1, 1, 2, 0.5, 1, 4, 0.25, 2.0])
            sigma = np.ones(8)
        w = _w(q, sigma)
        obj = (w[None, :] * 4.0 ** (-allt)).sum(1)
        for B in range(33):
            best = obj[sums == B].min()
            t = oracle.allocate(q, sigma, B).astype(np.int64)
            assert t.sum() == B
            got = (w * 4.0 ** (-t)).sum()
            assert got <= best * (1 + 1e-12) + 1e-300, (trial, B)


def _theta_star(w, B):
    """Water level of the closed form: sum_c clip(log2(w_c/theta)/2, 0, 4) = B."""
    lo, hi = math.log2(w.min()) - 10, math.log2(w.max()) + 1
    for _ in range(200):
        mid = (lo + hi) / 2
        tot = np.clip(0.5 * (np.log2(w) - mid), 0, 4).sum()
        lo, hi = (mid, hi) if tot > B else (lo, mid)
    return (lo + hi) / 2


@pytest.mark.parametrize("B", [17, 68, 92, 136, 300])
def test_allocation_matches_closed_form_water_filling(B):
    """t_c is floor or ceil of b_c = clip(log2(w_c/theta*)/2, 0, 4), and is
    exactly the largest-remainder rounding of b (ties to the lower channel)."""
    rng = np.random.default_rng(100 + B)
    for _ in range(5):
        q, sigma = _rand_head(rng, 128)
        w = _w(q, sigma)
        lt = _theta_star(w, B)
        b = np.clip(0.5 * (np.log2(w) - lt), 0, 4)
        # KKT of the continuous problem
        inner = (b > 1e-9) & (b < 4 - 1e-9)
        assert np.allclose(np.log2(w[inner]) - 2 * b[inner], lt, atol=1e-6)
        assert (np.log2(w[b <= 1e-9]) <= lt + 1e-6).all()
        assert (np.log2(w[b >= 4 - 1e-9]) - 8 >= lt - 1e-6).all()
        t = oracle.allocate(q, sigma, B).astype(int)
        fl = np.floor(b + 1e-9).astype(int)
        assert ((t == fl) | (t == np.ceil(b - 1e-9).astype(int))).all()
        R = B - fl.sum()
        frac = b - fl
        order = sorted(range(128), key=lambda c: (-frac[c], c))
        lr = fl.copy()
        lr[order[:R]] += 1
        assert (t == lr).all()


# ------------------------------------------------------------------ scores --

@pytest.mark.parametrize("d", [8, 32, 128])
def test_uniform_allocation_is_water_filling_with_equal_importance(d):
    """The fixed-depth read: for every budget it equals the C oracle's
    water-filling allocation when every channel has the same importance
    (the slot order then takes every channel's first slot, lower channels
    first, then every second slot, ...), sums to B and varies by at most one
    plane between channels."""
    ones = np.ones(d)
    budgets = range(0, 4 * d + 1) if d <= 32 else [0, 1, 68, 92, 127, 128, 129, 136, 300, 511, 512]
    for B in budgets:
        t = oracle.allocate_uniform(3, d, B)
        assert t.shape == (3, d) and t.dtype == np.uint8
        assert (t == t[0]).all()
        np.testing.assert_array_equal(t[0], oracle.allocate(ones, ones, B))
        assert int(t[0].sum()) == B
        assert int(t[0].max()) - int(t[0].min()) <= 1
        assert t[0].max() <= 4


def _attention_loops(q, k_rows, v_rows, idx, scale):
    """Tiny-case brute force with scalar loops and math.exp (no max shift)."""
    import math
    h_q, d = len(q), len(q[0])
    G = h_q // len(k_rows)
    out, lse = [], []
    for h in range(h_q):
        rows = [int(i) for i in idx[h] if 0 <= i < len(k_rows[0])]
        if not rows:
            out.append([0.0] * d)
            lse.append(-math.inf)
            continue
        e = []
        for i in rows:
            dot = 0.0
            for c in range(d):
                dot += float(q[h][c]) * float(k_rows[h // G][i][c])
            e.append(math.exp(dot * scale))
        z = sum(e)
        out.append([sum(e[j] * float(v_rows[h // G][rows[j]][c]) for j in range(len(rows))) / z
                    for c in range(d)])
        lse.append(math.log(z))
    return np.array(out), np.array(lse)


def test_sparse_attention_pins():
    """The attention over the selected rows, against scalar-loop brute force,
    closed forms (q = 0 averages the selected values and gives log of their
    count; one selected row returns it), permutation invariance and the
    skipped -1 entries."""
    rng = np.random.default_rng(5)
    h_q, h_kv, n, d, k = 4, 2, 40, 8, 6
    q = rng.normal(size=(h_q, d))
    K = rng.normal(size=(h_kv, n, d))
    V = rng.normal(size=(h_kv, n, d))
    idx = np.stack([rng.choice(n, size=k, replace=False) for _ in range(h_q)]).astype(np.int32)
    idx[1, 4:] = -1
    idx[3, :] = -1
    scale = 0.3
    o, lse = oracle.sparse_attention(q, K, V, idx, scale)
    bo, blse = _attention_loops(q, K, V, idx, scale)
    np.testing.assert_allclose(o, bo, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(lse[:3], blse[:3], rtol=1e-12)
    assert np.isneginf(lse[3]) and (o[3] == 0).all()
    # q = 0: uniform weights
    o0, l0 = oracle.sparse_attention(np.zeros_like(q), K, V, idx, scale)
    for h in range(3):
        sel = idx[h][idx[h] >= 0]
        np.testing.assert_allclose(o0[h], V[h // 2][sel].mean(axis=0), rtol=1e-12, atol=1e-14)
        assert abs(l0[h] - np.log(len(sel))) < 1e-12
    # one selected row
    one = np.full((h_q, k), -1, dtype=np.int32)
    one[:, 0] = 7
    o1, l1 = oracle.sparse_attention(q, K, V, one, scale)
    for h in range(h_q):
        np.testing.assert_allclose(o1[h], V[h // 2][7], rtol=1e-12)
        assert abs(l1[h] - scale * float(q[h] @ K[h // 2][7])) < 1e-12
    # the order of the selected rows does not matter
    perm = idx[:, ::-1].copy()
    op, lp = oracle.sparse_attention(q, K, V, perm, scale)
    np.testing.assert_allclose(op, o, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(lp[:3], lse[:3], rtol=1e-12)
    # entries at or past n select nothing, like the -1 padding
    far = idx.copy()
    far[1, 4] = n
    far[1, 5] = n + 7
    far[3, :2] = [2 * n, n]
    of, lf = oracle.sparse_attention(q, K, V, far, scale)
    bf, blf = _attention_loops(q, K, V, far, scale)
    np.testing.assert_allclose(of, o, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(of, bf, rtol=1e-12, atol=1e-12)
    assert np.isneginf(lf[3]) and np.isneginf(blf[3])


def test_hand_example_scores_and_topk(golden):
    ex = golden["scan"]
    codes = np.array(ex["codes_bytes"], dtype=np.uint8).reshape(ex["n"], 1)
    args = (np.array(ex["qmin"], np.float32), np.array(ex["qscale"], np.float32),
            np.array(ex["q"]), np.array(ex["alloc"], np.uint8))
    s = oracle.scores_from_codes(codes, *args)
    np.testing.assert_array_equal(s, ex["scores"])
    planes = np.array(ex["planes_words"], dtype=np.uint32).reshape(2, 4, 4)
    np.testing.assert_array_equal(oracle.scores_from_planes(planes, ex["n"], *args), ex["scores"])
    idx, val = oracle.topk(s, 2)
    assert idx.tolist() == ex["top2_idx"] and val.tolist() == ex["top2_score"]
    idx, val = oracle.topk(s, 5)
    assert idx.tolist() == ex["top5_idx"] and np.isneginf(val[3:]).all()


def _score_scale(q, m, s):
    return np.sum(np.abs(q) * np.maximum(np.abs(m), np.abs(m + 15 * s)))


def test_full_budget_is_the_4bit_dequantised_matmul(small_gqa):
    """B = 4d reads every plane: the score is q . (m + s u), a plain matmul."""
    case = small_gqa
    u = _unpack_codes(case.codes.numpy()).astype(np.float64)
    q = case.q.numpy().astype(np.float64)
    G = case.group
    for h in range(case.h_q):
        g = h // G
        m = case.qmin.numpy()[g].astype(np.float64)
        s = case.qscale.numpy()[g].astype(np.float64)
        t = oracle.allocate(q[h], case.sigma.numpy()[g], 4 * case.d)
        assert (t == 4).all()
        got = oracle.scores_from_codes(case.codes.numpy()[g], case.qmin.numpy()[g],
                                       case.qscale.numpy()[g], q[h], t)
        want = (m[None, :] + s[None, :] * u[g]) @ q[h]
        np.testing.assert_allclose(got, want, rtol=0, atol=1e-12 * _score_scale(q[h], m, s))


def test_zero_budget_is_constant_and_topk_is_first_indices(small_gqa):
    case = small_gqa
    q = case.q.numpy().astype(np.float64)
    m = case.qmin.numpy()[0].astype(np.float64)
    s = case.qscale.numpy()[0].astype(np.float64)
    t = oracle.allocate(q[0], case.sigma.numpy()[0], 0)
    got = oracle.scores_from_codes(case.codes.numpy()[0], case.qmin.numpy()[0],
                                   case.qscale.numpy()[0], q[0], t)
    const = np.sum(q[0] * (m + 7.5 * s))
    np.testing.assert_allclose(got, const, rtol=0, atol=1e-12 * _score_scale(q[0], m, s))
    # equal scores: ties go to the lower index
    idx, _ = oracle.topk(np.full(case.n, const), 10)
    assert idx.tolist() == list(range(10))


@pytest.mark.parametrize("B", [1, 37, 92, 136, 200])
def test_codes_and_planes_formulations_agree(small_gqa, B):
    case = small_gqa
    planes = oracle.pack_planes(case.codes.numpy())
    q = case.q.numpy().astype(np.float64)
    G = case.group
    for h in (0, 5):
        g = h // G
        t = oracle.allocate(q[h], case.sigma.numpy()[g], B)
        a = oracle.scores_from_codes(case.codes.numpy()[g], case.qmin.numpy()[g],
                                     case.qscale.numpy()[g], q[h], t)
        b = oracle.scores_from_planes(planes[g], case.n, case.qmin.numpy()[g],
                                      case.qscale.numpy()[g], q[h], t)
        scale = _score_scale(q[h], case.qmin.numpy()[g].astype(np.float64),
                             case.qscale.numpy()[g].astype(np.float64))
        np.testing.assert_allclose(a, b, rtol=0, atol=1e-12 * scale)


def test_error_against_exact_keys_falls_with_budget(tiny):
    """More bits per key bring the scan's score closer to the exact dot
    product with the fp32 keys."""
    q = tiny.q.numpy()[0].astype(np.float64)
    exact = tiny.keys.numpy()[0].astype(np.float64) @ q
    mse = []
    for B in (0, 32, 92, 256, 512):
        t = oracle.allocate(q, tiny.sigma.numpy()[0], B)
        s = oracle.scores_from_codes(tiny.codes.numpy()[0], tiny.qmin.numpy()[0],
                                     tiny.qscale.numpy()[0], q, t)
        mse.append(np.mean((s - exact) ** 2))
    assert all(a > b for a, b in zip(mse, mse[1:])), mse


def test_scores_at_matches_full_scores(small_gqa):
    case = small_gqa
    q = case.q.numpy().astype(np.float64)
    t = oracle.allocate(q[3], case.sigma.numpy()[0], 92)
    full = oracle.scores_from_codes(case.codes.numpy()[0], case.qmin.numpy()[0],
                                    case.qscale.numpy()[0], q[3], t)
    idx = np.array([0, 999, 17, 500, 17], dtype=np.int64)
    part = oracle.scores_at(case.codes.numpy()[0], case.qmin.numpy()[0],
                            case.qscale.numpy()[0], q[3], t, idx)
    np.testing.assert_array_equal(part, full[idx])


# ------------------------------------------- per-token-group statistics --

def _grouped_brute_force(u, m, s, q, t, token_group):
    """Scalar loops straight from the cell-centre reconstruction, each key with
    its own group's (m, s): u [n][d] codes, m/s [groups][d]."""
    n, d = u.shape
    out = np.zeros(n)
    for i in range(n):
        g = i // token_group
        acc = 0.0
        for c in range(d):
            tc = int(t[c])
            v = int(u[i, c]) >> (4 - tc)
            w = 2.0 ** (4 - tc)
            acc += q[c] * (float(m[g, c]) + float(s[g, c]) * (w * v + (w - 1.0) / 2.0))
        out[i] = acc
    return out


def test_grouped_scores_brute_force():
    """Key i must use group i // token_group's statistics: an off-by-one group,
    a transposed (group, channel) index or a shared row all fail here."""
    rng = np.random.default_rng(7)
    n, d, tg = 300, 8, 128
    u = rng.integers(0, 16, size=(n, d)).astype(np.uint8)
    codes = (u[:, 0::2] | (u[:, 1::2] << 4)).astype(np.uint8)
    groups = (n + tg - 1) // tg
    m = rng.normal(size=(groups, d)).astype(np.float32)
    s = rng.uniform(0.05, 2.0, size=(groups, d)).astype(np.float32)
    q = rng.normal(size=d)
    for t in (np.array([4, 3, 2, 1, 0, 4, 1, 2]), np.full(d, 4), np.zeros(d, dtype=int)):
        got = oracle.scores_from_codes_grouped(codes, m, s, q, t.astype(np.uint8), tg)
        want = _grouped_brute_force(u, m, s, q, t, tg)
        np.testing.assert_allclose(got, want, rtol=0, atol=1e-12 * np.abs(want).max())
        idx = np.array([0, 127, 128, 255, 256, 299, 5], dtype=np.int64)
        np.testing.assert_array_equal(
            oracle.scores_at_grouped(codes, m, s, q, t.astype(np.uint8), idx, tg), got[idx])


def test_grouped_scores_reduce_to_per_channel(small_gqa):
    """Every group holding the context's statistics, or one group spanning the
    context, gives the per-channel scores."""
    case = small_gqa
    q = case.q.numpy().astype(np.float64)
    t = oracle.allocate(q[2], case.sigma.numpy()[0], 92)
    codes, m, s = case.codes.numpy()[0], case.qmin.numpy()[0], case.qscale.numpy()[0]
    full = oracle.scores_from_codes(codes, m, s, q[2], t)
    for tg in (64, 333, 1000, 4096):
        groups = (case.n + tg - 1) // tg
        got = oracle.scores_from_codes_grouped(codes, np.tile(m, (groups, 1)),
                                               np.tile(s, (groups, 1)), q[2], t, tg)
        np.testing.assert_array_equal(got, full)


def test_grouped_quantiser_fixture_matches_per_range_statistics():
    """synthkv's grouped variant: each run of token_group keys carries the
    min/max statistics of its own keys, and its codes reconstruct them."""
    tg = 512
    case = synthkv.make_case(seed=12, n=1300, h_kv=1, h_q=1, d=32, q_dtype="f32",
                             keep_keys=True, token_group=tg)
    k = case.keys.numpy()[0].astype(np.float64)
    assert case.qmin.shape == (1, 3, 32)
    u = _unpack_codes(case.codes.numpy()[0])
    for j in range(3):
        kk = k[j * tg:(j + 1) * tg]
        np.testing.assert_array_equal(case.qmin.numpy()[0, j], kk.min(0).astype(np.float32))
        rec = case.qmin.numpy()[0, j].astype(np.float64) + \
            case.qscale.numpy()[0, j].astype(np.float64) * u[j * tg:(j + 1) * tg]
        assert np.all(np.abs(rec - kk) <= case.qscale.numpy()[0, j] * 0.5 + 1e-5)


# ------------------------------------------------------------------- top-k --

def test_topk_brute_force_with_ties():
    rng = np.random.default_rng(3)
    for n in (1, 2, 7, 64, 333):
        s = rng.integers(-5, 5, size=n).astype(np.float64)  # many exact ties
        for k in (1, 3, n, n + 4):
            idx, val = oracle.topk(s, k)
            want = sorted(range(n), key=lambda i: (-s[i], i))[:k]
            assert idx[:min(k, n)].tolist() == want
            assert (idx[n:] == -1).all() and np.isneginf(val[n:]).all()
            np.testing.assert_array_equal(val[:min(k, n)], s[want])


def test_topk_matches_numpy_lexsort(tiny):
    q = tiny.q.numpy()[0].astype(np.float64)
    t = oracle.allocate(q, tiny.sigma.numpy()[0], 92)
    s = oracle.scores_from_codes(tiny.codes.numpy()[0], tiny.qmin.numpy()[0],
                                 tiny.qscale.numpy()[0], q, t)
    idx, val = oracle.topk(s, 64)
    order = np.lexsort((np.arange(tiny.n), -s))[:64]
    np.testing.assert_array_equal(idx, order)
    np.testing.assert_array_equal(val, s[order])
