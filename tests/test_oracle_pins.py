"""Pins of the fp64 oracle against what the pages and the mathematics fix (no GPU).

Each test compares the oracle with something other than itself: hand-derived worked
examples (tests/golden/), a library softmax, brute force over tiny inputs, and the special
cases the method statement fixes (q == p accepts every position, a disjoint one-hot draft is
rejected at position 0, temperature 0 is exact argmax matching, a one-child-per-node trie is
the linear sampler). Source of the rule: review page of arXiv 2609.04010, section 3.3.
"""
import itertools
import math

import numpy as np
import pytest
import scipy.special

import oracle
from goldens import load, nums, rows


# ---------------------------------------------------------------- worked examples


@pytest.mark.parametrize("case", load("rows.txt"), ids=lambda c: c["name"])
def test_golden_rows(case):
    probs, band = oracle.row_dist(nums(case["logits"]), _f(case["T"]), _f(case["top_p"]))
    np.testing.assert_allclose(probs, nums(case["probs"]), rtol=0, atol=1e-12)


@pytest.mark.parametrize("case", load("cdf.txt"), ids=lambda c: c["name"])
def test_golden_cdf(case):
    w = nums(case["weights"])
    for item in case["cases"].split(";"):
        u, y = item.split("->")
        got, _ = oracle.inverse_cdf(w, float(u))
        assert got == int(y), (u, got, y)


@pytest.mark.parametrize("case", load("linear.txt"), ids=lambda c: c["name"])
def test_golden_linear(case):
    tgt, drf = rows(case["target"]), rows(case["draft"])
    K, V = drf.shape
    r = oracle.verify_linear(tgt[None], drf[None], np.array(nums(case["tokens"]), np.int32)[None],
                             np.array(nums(case["u_accept"]))[None], np.array(nums(case["u_resid"]))[None],
                             [_f(case["T"])], [_f(case["top_p"])])
    assert r["accept_len"][0] == int(_f(case["expect_len"]))
    assert r["tokens"][0].tolist() == [int(x) for x in nums(case["expect_tokens"])]
    np.testing.assert_allclose(r["p"][0], nums(case["expect_p"]), atol=1e-12)
    np.testing.assert_allclose(r["q"][0], nums(case["expect_q"]), atol=1e-12)


@pytest.mark.parametrize("case", load("tree.txt"), ids=lambda c: c["name"])
def test_golden_tree(case):
    tgt, drf = rows(case["target"]), rows(case["draft"])
    n = tgt.shape[0]
    md = int(case["max_depth"])
    r = oracle.verify_tree(tgt, drf, [0, n], np.array(nums(case["parent"]), np.int32),
                           np.array(nums(case["tokens"]), np.int32), nums(case["u_accept"]), nums(case["u_resid"]),
                           [_f(case["T"])], [_f(case["top_p"])], md)
    assert r["accept_len"][0] == int(_f(case["expect_len"]))
    assert r["path"][0].tolist() == [int(x) for x in nums(case["expect_path"])]
    assert r["tokens"][0].tolist() == [int(x) for x in nums(case["expect_tokens"])]


def _f(s):
    return nums(s)[0]


# ---------------------------------------------------------------- closed forms / library routines


@pytest.mark.parametrize("T", [0.3, 0.7, 1.0, 2.5])
def test_softmax_matches_library(T):
    rng = np.random.default_rng(5)
    for _ in range(20):
        l = rng.normal(0, 4, size=int(rng.integers(1, 300)))
        l[rng.random(l.size) < 0.05] = -np.inf
        if not np.isfinite(l).any():
            l[0] = 0.0
        p, band = oracle.row_dist(l, T, 1.0)
        np.testing.assert_allclose(p, scipy.special.softmax(l / T), rtol=1e-12, atol=1e-300)
        assert band == math.inf


def test_bad_rows_rejected():
    assert oracle.row_dist([0.0, np.nan], 1.0)[0] is None
    assert oracle.row_dist([0.0, np.inf], 1.0)[0] is None
    assert oracle.row_dist([-np.inf, -np.inf], 1.0)[0] is None
    assert oracle.row_dist([0.0, 1.0], -1.0)[0] is None


def _topp_brute(l, T, top_p):
    """Every candidate threshold t among the row's values; keep the largest whose
    tie-inclusive tail probability reaches top_p."""
    p = scipy.special.softmax(l / T)
    best = -np.inf
    for t in np.unique(l):
        if p[l >= t].sum() >= top_p:
            best = max(best, t)
    keep = l >= best
    out = np.where(keep, p, 0.0)
    return out / out.sum()


def test_topp_brute_force_with_ties():
    rng = np.random.default_rng(7)
    checked = 0
    for _ in range(400):
        V = int(rng.integers(1, 9))
        l = rng.choice([-1.0, 0.0, 0.5, 1.0, 2.0, -np.inf], size=V)
        if not np.isfinite(l).any():
            continue
        T = float(rng.choice([0.5, 1.0, 3.0]))
        top_p = float(rng.choice([0.1, 0.33, 0.5, 0.77, 0.9, 0.999]))
        p, band = oracle.row_dist(l, T, top_p)
        if band < 1e-9:  # a threshold exactly on a tail boundary is rounding-sensitive
            continue
        np.testing.assert_allclose(p, _topp_brute(l, T, top_p), atol=1e-12)
        checked += 1
    assert checked > 300


def test_topp_one_is_identity_and_tiny_keeps_max():
    l = np.array([0.3, -1.0, 2.0, 2.0, 0.0])
    np.testing.assert_allclose(oracle.row_dist(l, 1.0, 1.0)[0], scipy.special.softmax(l))
    p = oracle.row_dist(l, 1.0, 1e-9)[0]
    np.testing.assert_allclose(p, [0, 0, 0.5, 0.5, 0])  # both tied maxima survive


def _topk_topp_brute(l, T, top_k, top_p):
    """Top-k by enumeration (every token whose value is at least the k-th of the sorted row),
    then, on that renormalised set, the largest candidate threshold whose tie-inclusive tail
    reaches top_p (every candidate tried)."""
    V = l.size
    p = scipy.special.softmax(l / T)
    if 0 < top_k < V:
        kth = sorted(l.tolist(), reverse=True)[top_k - 1]
        p = np.where(l >= kth, p, 0.0)
        p = p / p.sum()
    if top_p < 1.0:
        best = -np.inf
        for t in np.unique(l[p > 0]):
            if p[l >= t].sum() >= top_p:
                best = max(best, t)
        p = np.where(l >= best, p, 0.0)
        p = p / p.sum()
    return p


def test_topk_brute_force_with_ties():
    """Top-k then top-p (the reading for the README's --top-k), against enumeration on tiny
    rows with forced ties and -inf entries, over every k from off to beyond V."""
    rng = np.random.default_rng(11)
    checked = 0
    for _ in range(600):
        V = int(rng.integers(1, 9))
        l = rng.choice([-1.0, 0.0, 0.5, 1.0, 2.0, -np.inf], size=V)
        if not np.isfinite(l).any():
            continue
        T = float(rng.choice([0.5, 1.0, 3.0]))
        k = int(rng.integers(0, V + 2))
        top_p = float(rng.choice([1.0, 0.33, 0.6, 0.9]))
        p, band = oracle.row_dist(l, T, top_p, k)
        if top_p < 1.0 and band < 1e-9:  # a threshold exactly on a tail boundary
            continue
        np.testing.assert_allclose(p, _topk_topp_brute(l, T, k, top_p), atol=1e-12)
        checked += 1
    assert checked > 450


def test_topk_special_cases_and_order():
    l = np.array([0.3, -1.0, 2.0, 2.0, 0.0])
    off = oracle.row_dist(l, 1.0, 0.9)[0]
    for k in (0, -3, 5, 9):  # off, and k >= V
        np.testing.assert_allclose(oracle.row_dist(l, 1.0, 0.9, k)[0], off)
    np.testing.assert_allclose(oracle.row_dist(l, 1.0, 1.0, 1)[0], [0, 0, 0.5, 0.5, 0])  # tied maxima stay
    np.testing.assert_allclose(oracle.row_dist(l, 0.0, 1.0, 3)[0], [0, 0, 1, 0, 0])  # greedy: k is a no-op
    # the order: top-p acts on the renormalised top-k set. With logits (2, 1, 0.5, 0), k = 3
    # and top_p = 0.85, top-k first keeps (2, 1, 0.5) with shares (0.628, 0.231, 0.140), and
    # top-p then stops after two tokens; top-p first would keep three.
    e = math.e
    np.testing.assert_allclose(oracle.row_dist([2.0, 1.0, 0.5, 0.0], 1.0, 0.85, 3)[0],
                               [e * e / (e * e + e), e / (e * e + e), 0, 0], atol=1e-15)


def test_topk_reaches_the_samplers():
    """sample_draft draws from the top-k distribution, and q == p still accepts every position
    with top-k on both rows."""
    rng = np.random.default_rng(3)
    V, K = 40, 3
    d = rng.normal(size=(K, V)) * 2.0
    u = np.array([0.1, 0.5, 0.93])
    s = oracle.sample_draft(d, [1.0] * K, [0.9] * K, u, row_req=np.arange(K), top_k=[5] * K)
    for i in range(K):
        r, _ = oracle.row_dist(d[i], 1.0, 0.9, 5)
        assert s["tokens"][i] == oracle.inverse_cdf(r, u[i])[0]
        assert abs(s["q"][i] - r[s["tokens"][i]]) < 1e-15
    t = rng.normal(size=(1, K + 1, V))
    x = np.array([[int(np.argmax(t[0, i])) for i in range(K)]])  # tokens inside every top-k set
    out = oracle.verify_linear(t, t[:, :K], x, np.full((1, K), 0.999), np.full((1, K + 1), 0.5), [1.0], [1.0],
                               top_k=[4])
    assert out["accept_len"][0] == K


def test_inverse_cdf_exhaustive_grid():
    """Over a fine uniform grid, the fraction of u mapped to token v equals r(v)/Z exactly
    (dyadic weights, midpoint grid)."""
    rng = np.random.default_rng(3)
    G = 1 << 12
    u = (np.arange(G) + 0.5) / G
    for _ in range(30):
        V = int(rng.integers(1, 9))
        w = rng.integers(0, 5, size=V).astype(np.float64)
        if w.sum() == 0:
            w[0] = 1
        w = w / w.sum()
        w = np.round(w * 64) / 64  # dyadic
        if w.sum() == 0:
            continue
        counts = np.zeros(V)
        for x in u:
            y, _ = oracle.inverse_cdf(w, x)
            counts[y] += 1
        np.testing.assert_allclose(counts / G, w / w.sum(), atol=1.5 / G)
        assert (counts[w == 0] == 0).all()


# ---------------------------------------------------------------- special cases of the rule


def _rand_rows(rng, B, n, V, scale=2.0):
    return rng.normal(0, scale, size=(B, n, V))


def test_q_equals_p_accepts_every_position():
    rng = np.random.default_rng(11)
    B, K, V = 50, 5, 40
    tgt = _rand_rows(rng, B, K + 1, V)
    drf = tgt[:, :K].copy()
    x = rng.integers(0, V, size=(B, K))
    ua = rng.random((B, K))
    ur = rng.random((B, K + 1))
    for T, tp in [(1.0, 1.0), (0.7, 0.9), (1.3, 0.5)]:
        r = oracle.verify_linear(tgt, drf, x, ua, ur, [T] * B, [tp] * B)
        # a token outside the top-p set has p = q = 0 and is rejected (u * 0 < 0 fails);
        # everywhere else p/q = 1 > u
        for b in range(B):
            keep = r["q"][b] > 0
            j = int(np.argmin(keep)) if not keep.all() else K
            assert r["accept_len"][b] == j
            assert r["tokens"][b, :j].tolist() == x[b, :j].tolist()
            if j == K:  # bonus token drawn from the last verifier row with u_resid[b, K]
                pK, _ = oracle.row_dist(tgt[b, K], T, tp)
                assert r["tokens"][b, K] == int(np.searchsorted(np.cumsum(pK), ur[b, K] * pK.sum(), side="right"))
            np.testing.assert_allclose(r["p"][b], r["q"][b])


def test_disjoint_one_hot_draft_rejects_at_zero():
    rng = np.random.default_rng(12)
    B, K, V = 40, 3, 16
    tgt = _rand_rows(rng, B, K + 1, V)
    drf = np.full((B, K, V), -np.inf)
    x = np.zeros((B, K), np.int64)
    for b in range(B):
        for i in range(K):
            x[b, i] = rng.integers(0, V)
            drf[b, i, x[b, i]] = 0.0
            tgt[b, i, x[b, i]] = -np.inf  # p(x) = 0: disjoint supports
    ur = rng.random((B, K + 1))
    r = oracle.verify_linear(tgt, drf, x, rng.random((B, K)), ur, [1.0] * B, [1.0] * B)
    assert (r["accept_len"] == 0).all()
    for b in range(B):
        # residual max(0, p - q) = p_0 because the supports are disjoint
        p0 = scipy.special.softmax(tgt[b, 0])
        want = int(np.searchsorted(np.cumsum(p0), ur[b, 0] * p0.sum(), side="right"))
        assert r["tokens"][b, 0] == want
        assert (r["tokens"][b, 1:] == -1).all()


def test_temperature_zero_is_argmax_match_brute_force():
    """All rows over a small value set with V = 3, K = 1: accepted iff the draft token is the
    verifier argmax (lowest index), and the emitted token is always the verifier argmax."""
    vals = [0.0, 1.0, 2.0]
    cases = list(itertools.product(vals, repeat=3))
    for lt in cases:
        for lq in cases[::5]:
            for x in range(3):
                tgt = np.array([[lt, (2.0, 0.0, 1.0)]])
                drf = np.array([[lq]])
                r = oracle.verify_linear(tgt, drf, [[x]], [[0.5]], [[0.5, 0.5]], [0.0], [0.9])
                a = int(np.argmax(lt))
                if x == a:
                    assert r["accept_len"][0] == 1 and r["tokens"][0].tolist() == [x, 0]
                else:
                    assert r["accept_len"][0] == 0 and r["tokens"][0].tolist() == [a, -1]


def _chain_tree(tgt, drf, x, ua, ur):
    """Lay a linear block out as a one-child-per-node trie."""
    B, K1, V = tgt.shape
    K = K1 - 1
    N = B * (K + 1)
    t_rows = tgt.reshape(N, V)
    d_rows = np.concatenate([drf, np.zeros((B, 1, V))], axis=1).reshape(N, V)
    parent = np.tile(np.arange(-1, K), B).astype(np.int32)
    tok = np.zeros((B, K + 1), np.int32)
    tok[:, 1:] = x
    uacc = np.zeros((B, K + 1))
    uacc[:, 1:] = ua
    return t_rows, d_rows, np.arange(0, N + 1, K + 1), parent, tok.reshape(-1), uacc.reshape(-1), ur.reshape(-1)


@pytest.mark.parametrize("T,tp", [(1.0, 1.0), (0.7, 0.9), (0.0, 1.0)])
def test_branching_one_tree_equals_linear(T, tp):
    rng = np.random.default_rng(13)
    B, K, V = 60, 4, 12
    tgt = _rand_rows(rng, B, K + 1, V, 1.5)
    drf = tgt[:, :K] + rng.normal(0, 1.0, size=(B, K, V))
    x = rng.integers(0, V, size=(B, K))
    ua, ur = rng.random((B, K)), rng.random((B, K + 1))
    lin = oracle.verify_linear(tgt, drf, x, ua, ur, [T] * B, [tp] * B)
    tr = oracle.verify_tree(*_chain_tree(tgt, drf, x, ua, ur), [T] * B, [tp] * B, K)
    assert (lin["accept_len"] == tr["accept_len"]).all()
    assert (lin["tokens"] == tr["tokens"]).all()
    for b in range(B):
        j = lin["accept_len"][b]
        assert tr["path"][b, :j].tolist() == list(range(1, j + 1))


def test_topp_at_or_below_zero_keeps_the_maximum_value():
    """top_p <= 0 is met by the maximum's value alone (its ties kept), like a tiny top_p; NaN
    and values >= 1 leave the row unfiltered."""
    l = np.array([0.5, 2.0, -1.0, 2.0, 1.5])
    for tp in (0.0, -0.5, 1e-9):
        p, _ = oracle.row_dist(l, 1.0, tp)
        assert np.array_equal(p, np.array([0.0, 0.5, 0.0, 0.5, 0.0]))
    full, _ = oracle.row_dist(l, 1.0, 1.0)
    assert np.allclose(full, np.exp(l - l.max()) / np.exp(l - l.max()).sum(), rtol=0, atol=1e-15)
    for tp in (float("nan"), 1.0, 3.0):
        assert np.array_equal(oracle.row_dist(l, 1.0, tp)[0], full)
