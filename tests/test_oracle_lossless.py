"""Losslessness pins of the oracle (no GPU).

The review page of arXiv 2609.04010 (section 1, executive summary, and section 7.1) states
what the rejection correction guarantees: the emitted tokens follow the verifier's (AR)
distribution exactly, whatever the drafter proposes. These tests check the oracle's
emitted-token law against that distribution, computed here with scipy's softmax and a
brute-force top-p, not with the oracle:

  * an exhaustive uniform grid over (u_draft, u_accept, u_resid) for one drafted position,
    with a rigorous discretisation bound;
  * multi-round generation on a tiny table language model (V = 3) up to L tokens, compared
    with the product of the verifier's conditionals by a chi-squared test at a fixed seed,
    for the linear sampler (K = 1, 2, 3) and the tree sampler (without-replacement children).
"""
import numpy as np
import pytest
import scipy.special
import scipy.stats

import oracle


def _dist(l, T, top_p, top_k=0):
    """Verifier distribution computed independently of the oracle (top-k by an explicit sort,
    then top-p over the renormalised top-k set)."""
    l = np.asarray(l, dtype=np.float64)
    if T == 0:
        out = np.zeros_like(l)
        out[int(np.argmax(l))] = 1.0
        return out
    p = scipy.special.softmax(l / T)
    if 0 < top_k < l.size:
        kth = np.sort(l)[::-1][top_k - 1]
        p = np.where(l >= kth, p, 0.0)
        p = p / p.sum()
    if top_p >= 1:
        return p
    best = -np.inf
    for t in np.unique(l):
        if p[l >= t].sum() >= top_p:
            best = max(best, t)
    out = np.where(l >= best, p, 0.0)
    return out / out.sum()


def test_exhaustive_grid_one_position():
    """First emitted token ~ p_0 and, after an acceptance, bonus ~ p_1.

    q_0 is dyadic in eighths, so an 8-point midpoint grid over u_draft reproduces it exactly;
    accept and residual grids of G points each perturb a probability by at most 1/G and 2/G.
    """
    q0 = np.array([1 / 2, 1 / 4, 1 / 8, 1 / 8])
    p0 = np.array([0.1, 0.45, 0.3, 0.15])
    p1 = np.array([0.25, 0.05, 0.5, 0.2])
    G, Gd = 256, 8
    ud = (np.arange(Gd) + 0.5) / Gd
    ug = (np.arange(G) + 0.5) / G
    UD, UA, UR = np.meshgrid(ud, ug, ug, indexing="ij")
    n = UD.size
    x = oracle.sample_draft(np.log(q0)[None].repeat(Gd, 0), [1.0] * Gd, [1.0] * Gd, ud)["tokens"]
    assert np.bincount(x, minlength=4).tolist() == [4, 2, 1, 1]
    X = np.repeat(x, G * G)
    tgt = np.broadcast_to(np.stack([np.log(p0), np.log(p1)])[None], (n, 2, 4))
    drf = np.broadcast_to(np.log(q0)[None, None], (n, 1, 4))
    ur = np.stack([UR.reshape(-1), UR.reshape(-1)], axis=1)
    r = oracle.verify_linear(tgt, drf, X[:, None], UA.reshape(-1, 1), ur, np.ones(n), np.ones(n))
    first = r["tokens"][:, 0]
    law = np.bincount(first, minlength=4) / n
    assert np.abs(law - p0).max() <= 1.0 / G + 2.0 / G
    acc = r["accept_len"] == 1
    bonus = np.bincount(r["tokens"][acc, 1], minlength=4) / acc.sum()
    assert np.abs(bonus - p1).max() <= 2.0 / G + 1e-12
    # the accepted fraction is sum_x q(x) min(1, p/q) = 1 - TV(p, q)
    assert abs(acc.mean() - (1 - 0.5 * np.abs(p0 - q0).sum())) <= 1.0 / G


class TableLM:
    """Next-token logits for every context of length < 8 over V tokens, seeded."""

    def __init__(self, V, seed, draft_noise=1.0):
        self.V = V
        self.base = V + 1
        n = self.base**8
        rng = np.random.default_rng(seed)
        self.P = rng.normal(0, 1.5, size=(n, V))
        self.Q = self.P + rng.normal(0, draft_noise, size=(n, V))

    def extend(self, code, length, tok):
        return code + (np.asarray(tok) + 1) * self.base ** np.asarray(length)

    def law(self, L, T, top_p, top_k=0):
        """Exact law of the first L tokens under the verifier."""
        out = {}

        def rec(prefix, code, prob):
            if len(prefix) == L:
                out[tuple(prefix)] = prob
                return
            d = _dist(self.P[code], T, top_p, top_k)
            for t in range(self.V):
                if d[t] > 0:
                    rec(prefix + [t], int(self.extend(code, len(prefix), t)), prob * d[t])

        rec([], 0, 1.0)
        return out


def _chi2_check(samples, law, V, L):
    idx = {k: i for i, k in enumerate(law)}
    obs = np.zeros(len(law))
    for row in samples:
        k = tuple(int(t) for t in row[:L])
        assert k in idx, "emitted a sequence of probability zero: %r" % (k,)
        obs[idx[k]] += 1
    exp = np.array(list(law.values())) * len(samples)
    big = exp >= 5
    o = np.append(obs[big], obs[~big].sum())
    e = np.append(exp[big], exp[~big].sum())
    if e[-1] == 0:
        o, e = o[:-1], e[:-1]
    stat, pval = scipy.stats.chisquare(o, e * o.sum() / e.sum())
    assert pval > 1e-3, (stat, pval)


@pytest.mark.parametrize("K,T,top_p,top_k", [(1, 1.0, 1.0, 0), (2, 1.0, 1.0, 0), (3, 0.8, 0.8, 0), (2, 1.3, 0.9, 0),
                                             (2, 1.0, 1.0, 2), (3, 1.2, 0.9, 2)])
def test_multiround_linear_matches_verifier_law(K, T, top_p, top_k):
    V, L, N = 3, 4, 40000
    lm = TableLM(V, seed=100 + K + 10 * top_k)
    rng = np.random.default_rng(200 + K + 10 * top_k)
    kk = np.full(N, top_k, np.int32) if top_k else None
    seq = np.full((N, L + K + 1), -1, np.int64)
    length = np.zeros(N, np.int64)
    code = np.zeros(N, np.int64)
    while (length < L).any():
        act = np.nonzero(length < L)[0]
        n = act.size
        c = [code[act]]
        x = np.zeros((n, K), np.int64)
        for i in range(K):
            s = oracle.sample_draft(lm.Q[c[-1]], np.full(n, T), np.full(n, top_p), rng.random(n),
                                    top_k=None if kk is None else kk[:n])
            x[:, i] = s["tokens"]
            c.append(lm.extend(c[-1], length[act] + i, x[:, i]))
        codes = np.stack(c, axis=1)  # [n, K+1]
        r = oracle.verify_linear(lm.P[codes], lm.Q[codes[:, :K]], x, rng.random((n, K)), rng.random((n, K + 1)),
                                 np.full(n, T), np.full(n, top_p), top_k=None if kk is None else kk[:n])
        assert (r["accept_len"] >= 0).all()
        for row, b in enumerate(act):
            j = r["accept_len"][row]
            for t in r["tokens"][row, : j + 1]:
                seq[b, length[b]] = t
                code[b] = lm.extend(code[b], length[b], t)
                length[b] += 1
    _chi2_check(seq, lm.law(L, T, top_p, top_k), V, L)


def test_multiround_tree_matches_verifier_law():
    """Binary trie of depth 2 per round; children drawn without replacement from q."""
    V, L, N, T = 3, 4, 30000, 1.0
    lm = TableLM(V, seed=300)
    rng = np.random.default_rng(301)
    parent = np.array([-1, 0, 0, 1, 1, 2, 2], np.int32)
    seq = np.full((N, L + 4), -1, np.int64)
    length = np.zeros(N, np.int64)
    code = np.zeros(N, np.int64)
    while (length < L).any():
        act = np.nonzero(length < L)[0]
        n = act.size
        codes = np.zeros((n, 7), np.int64)
        toks = np.zeros((n, 7), np.int64)
        codes[:, 0] = code[act]
        for node in range(1, 7):
            pa = parent[node]
            ql = lm.Q[codes[:, pa]].copy()
            for sib in range(1, node):  # earlier siblings' tokens are removed
                if parent[sib] == pa:
                    ql[np.arange(n), toks[:, sib]] = -np.inf
            toks[:, node] = oracle.sample_draft(ql, np.full(n, T), np.ones(n), rng.random(n))["tokens"]
            depth = 1 if pa == 0 else 2
            codes[:, node] = lm.extend(codes[:, pa], length[act] + depth - 1, toks[:, node])
        r = oracle.verify_tree(lm.P[codes].reshape(-1, V), lm.Q[codes].reshape(-1, V), np.arange(0, 7 * n + 1, 7),
                               np.tile(parent, n), toks.reshape(-1), rng.random(7 * n), rng.random(7 * n),
                               np.full(n, T), np.ones(n), 2)
        assert (r["accept_len"] >= 0).all()
        for row, b in enumerate(act):
            j = r["accept_len"][row]
            for t in r["tokens"][row, : j + 1]:
                seq[b, length[b]] = t
                code[b] = lm.extend(code[b], length[b], t)
                length[b] += 1
    _chi2_check(seq, lm.law(L, T, 1.0), V, L)


def test_multiround_tree_with_top_k_matches_verifier_law():
    """Binary trie of depth 2 per round under top-k 3 of V = 4: children drawn here (numpy,
    from the independently computed top-k draft distribution) without replacement, verified by
    the oracle with the same top-k; the emitted tokens follow the top-k verifier law."""
    V, L, N, T, k = 4, 3, 30000, 1.0, 3
    lm = TableLM(V, seed=700)
    rng = np.random.default_rng(701)
    parent = np.array([-1, 0, 0, 1, 1, 2, 2], np.int32)
    seq = np.full((N, L + 4), -1, np.int64)
    length = np.zeros(N, np.int64)
    code = np.zeros(N, np.int64)
    while (length < L).any():
        act = np.nonzero(length < L)[0]
        n = act.size
        codes = np.zeros((n, 7), np.int64)
        toks = np.zeros((n, 7), np.int64)
        codes[:, 0] = code[act]
        for node in range(1, 7):
            pa = parent[node]
            lq = lm.Q[codes[:, pa]] / T
            kth = np.sort(lm.Q[codes[:, pa]], axis=1)[:, V - k][:, None]  # top-k by an explicit sort
            q = np.where(lm.Q[codes[:, pa]] >= kth, np.exp(lq - lq.max(axis=1, keepdims=True)), 0.0)
            for sib in range(1, node):  # earlier siblings' tokens are removed
                if parent[sib] == pa:
                    q[np.arange(n), toks[:, sib]] = 0.0
            c = np.cumsum(q / q.sum(axis=1, keepdims=True), axis=1)
            toks[:, node] = np.minimum((c <= rng.random(n)[:, None]).sum(axis=1), V - 1)
            codes[:, node] = lm.extend(codes[:, pa], length[act] + (1 if pa == 0 else 2) - 1, toks[:, node])
        r = oracle.verify_tree(lm.P[codes].reshape(-1, V), lm.Q[codes].reshape(-1, V), np.arange(0, 7 * n + 1, 7),
                               np.tile(parent, n), toks.reshape(-1), rng.random(7 * n), rng.random(7 * n),
                               np.full(n, T), np.ones(n), 2, top_k=np.full(n, k, np.int32))
        assert (r["accept_len"] >= 0).all()
        for row, b in enumerate(act):
            j = r["accept_len"][row]
            for t in r["tokens"][row, : j + 1]:
                seq[b, length[b]] = t
                code[b] = lm.extend(code[b], length[b], t)
                length[b] += 1
    _chi2_check(seq, lm.law(L, T, 1.0, k), V, L)
