"""Pins of the tree sampler's candidate trie and of the two further tree rules (no GPU).

Review page of arXiv 2609.04010, section 3.4 ("Tree Sampler"): at every position of the block
take the top-K tokens, keep the V most probable prefixes, and verify them together. A trie
built that way is a deterministic function of the draft rows, so its children are checked by
rejection with point-mass proposals (oracle rule TREE_DETERMINISTIC); children drawn from q
independently are checked with q unchanged after a rejection (TREE_SAMPLED_WR). The pins:

  * the best-first construction equals a full enumeration of every candidate prefix, sorted
    (ties included), on tiny rows with forced ties, temperature 0 and top-p cuts;
  * structural invariants of the trie and its special cases (one candidate per position is the
    greedy chain, T = 0 is the argmax chain, a budget beyond the candidates keeps them all);
  * an exhaustive uniform grid shows the deterministic rule's first token follows p exactly
    (within the grid's discretisation bound), and the bonus after an accepted leaf follows
    that leaf's row;
  * multi-round generation on a table language model: tries built from draft marginals and
    verified with the deterministic rule, and tries of independently drawn children verified
    with the with-replacement rule, both emit the verifier's law (chi-squared, fixed seeds);
  * on single-child chains the with-replacement and without-replacement rules coincide.
"""
import functools
import itertools

import numpy as np
import pytest

import oracle
from test_oracle_lossless import TableLM, _chi2_check


def _brute_tree(draft, T, top_p, cand_k, n_prefixes, top_k=0):
    """Every prefix over the candidate lists, sorted: prefixes of one length by their logit sum
    (the same positions share their normalisers, so this is their probability order, exactly),
    then by rank path; prefixes of different lengths by probability, then the shorter first."""
    K, V = draft.shape
    q = [oracle.row_dist(draft[i], T, top_p, top_k)[0] for i in range(K)]
    cands = [sorted((v for v in range(V) if q[i][v] > 0), key=lambda v: (-q[i][v], v))[:cand_k] for i in range(K)]
    entries = []
    for L in range(1, K + 1):
        for ranks in itertools.product(*[range(len(cands[i])) for i in range(L)]):
            s, lsum = 1.0, 0.0
            for i, r in enumerate(ranks):
                s *= q[i][cands[i][r]]
                lsum += draft[i][cands[i][r]]
            entries.append((s, lsum, L, ranks))

    def order(a, b):
        (sa, la, da, ra), (sb, lb, db, rb) = a, b
        if da != db:
            return -1 if sa > sb or (sa == sb and da < db) else 1
        if la != lb:
            return -1 if la > lb else 1
        return -1 if ra < rb else (1 if ra > rb else 0)

    entries.sort(key=functools.cmp_to_key(order))
    return [(tuple(cands[i][r] for i, r in enumerate(ranks)), s) for s, _, L, ranks in entries[:n_prefixes]]


def _paths(tree):
    """Token path of every non-root node, in node order."""
    out, path = [], {0: ()}
    for i in range(1, len(tree["parent"])):
        path[i] = path[int(tree["parent"][i])] + (int(tree["tokens"][i]),)
        out.append(path[i])
    return out


def _tied_rows(rng, K, V):
    """Logits on a half-integer grid (many exact ties), some positions repeating a row."""
    d = rng.integers(-4, 5, size=(K, V)) / 2.0
    if K > 1 and rng.random() < 0.5:
        d[1] = d[0]
    return d


CASES = [(K, V, ck, n, T, tp) for K, V in ((1, 5), (2, 4), (3, 4), (4, 3)) for ck in (1, 2, 3, 6)
         for n in (1, 3, 7, 200) for T, tp in ((1.0, 1.0), (0.7, 0.8), (0.0, 1.0))]


@pytest.mark.parametrize("K,V,cand_k,n,T,top_p", CASES[::3])
def test_build_tree_equals_enumeration(K, V, cand_k, n, T, top_p):
    rng = np.random.default_rng(K * 1000 + V * 100 + cand_k * 10 + n)
    for trial in range(4):
        d = _tied_rows(rng, K, V) if trial % 2 == 0 else rng.normal(0, 1.5, size=(K, V))
        tree = oracle.build_tree(d, T, top_p, cand_k, n)
        want = _brute_tree(d, T, top_p, cand_k, n)
        assert _paths(tree) == [p for p, _ in want]
        assert np.array_equal(tree["score"][1:], np.array([s for _, s in want]))


def test_build_tree_ties_across_depths():
    """Exact ties between prefixes of different lengths: a position whose only candidate has
    q = 1 (the rest -inf) extends a prefix without lowering its probability, so the shorter
    prefixes must come first; equal rows at two positions tie prefixes of the same length."""
    ninf = -np.inf
    d = np.array([[0.0, 0.0, 0.0, ninf], [0.0, ninf, ninf, ninf], [0.0, 0.0, ninf, ninf], [1.0, 1.0, 0.0, 0.0]])
    for ck, n in ((3, 10), (2, 7), (4, 40), (1, 3)):
        tree = oracle.build_tree(d, 1.0, 1.0, ck, n)
        want = _brute_tree(d, 1.0, 1.0, ck, n)
        assert _paths(tree) == [p for p, _ in want]
        assert np.array_equal(tree["score"][1:], np.array([s for _, s in want]))
    # the first three kept prefixes are the single tokens (0.25 each) and then their q = 1
    # extensions, shorter first
    t = oracle.build_tree(d, 1.0, 1.0, 3, 6)
    assert _paths(t) == [(0,), (1,), (2,), (0, 0), (1, 0), (2, 0)]


def test_build_tree_exact_ties_of_equal_length():
    """Prefixes of one length whose logit sums are equal have equal probabilities whatever
    rounding their products carry: they follow the candidate ranks. Rows [2, 1, 0] and
    [1, 2, 0]: (0,0) and (1,1) both sum to 3, and (0,2), (1,0), (2,1) to 2."""
    d = np.array([[2.0, 1.0, 0.0], [1.0, 2.0, 0.0]])
    for T in (1.0, 0.7, 1.9):
        p = _paths(oracle.build_tree(d, T, 1.0, 3, 12))
        assert len(p) == 12
        assert p.index((0, 0)) < p.index((1, 1))
        assert p.index((0, 2)) < p.index((1, 0)) < p.index((2, 1))
        assert p.index((0, 1)) < p.index((0, 0))


def test_build_tree_with_top_k_control():
    rng = np.random.default_rng(7)
    for _ in range(6):
        d = _tied_rows(rng, 3, 6)
        tree = oracle.build_tree(d, 1.0, 0.9, 4, 20, top_k=2)
        assert _paths(tree) == [p for p, _ in _brute_tree(d, 1.0, 0.9, 4, 20, top_k=2)]


def test_build_tree_invariants_and_special_cases():
    rng = np.random.default_rng(11)
    K, V = 4, 6
    for _ in range(20):
        d = _tied_rows(rng, K, V)
        ck, n = int(rng.integers(1, 5)), int(rng.integers(1, 40))
        t = oracle.build_tree(d, 1.0, 1.0, ck, n)
        par, dep, sc = t["parent"], t["depth"], t["score"]
        assert par[0] == -1 and dep[0] == 0 and sc[0] == 1.0
        assert len(par) == 1 + min(n, sum(ck**L for L in range(1, K + 1)))
        for i in range(1, len(par)):
            assert 0 <= par[i] < i and dep[i] == dep[par[i]] + 1 <= K
            assert sc[i] <= sc[par[i]]
        # kept in decreasing probability (equal probabilities may differ in their last fp64 bit)
        assert (np.diff(sc[1:]) <= 1e-12 * sc[1:-1]).all()
        for i in range(len(par)):  # siblings carry distinct tokens
            kids = t["tokens"][par == i]
            assert len(set(kids.tolist())) == kids.size
    # one candidate per position: the chain of per-position argmaxes of q
    d = rng.normal(0, 2, size=(5, 9))
    t = oracle.build_tree(d, 0.8, 1.0, 1, 50)
    assert _paths(t)[-1] == tuple(int(np.argmax(r)) for r in d) and len(t["parent"]) == 6
    # temperature 0: a point mass per position, the same chain whatever cand_k is
    t0 = oracle.build_tree(d, 0.0, 1.0, 4, 50)
    assert _paths(t0) == _paths(t) and (t0["score"] == 1.0).all()
    # a budget beyond the candidates keeps every candidate prefix
    t = oracle.build_tree(d[:2], 1.0, 1.0, 3, 100)
    assert len(t["parent"]) == 1 + 3 + 9
    # no candidates, no budget, no positions
    assert len(oracle.build_tree(d, 1.0, 1.0, 0, 10)["parent"]) == 1
    assert len(oracle.build_tree(d, 1.0, 1.0, 3, 0)["parent"]) == 1
    assert len(oracle.build_tree(d[:0], 1.0, 1.0, 3, 10)["parent"]) == 1
    # a bad draft row is reported
    bad = d.copy()
    bad[2, 3] = np.nan
    assert oracle.build_tree(bad, 1.0, 1.0, 2, 10) is None


def test_deterministic_rule_exhaustive_grid():
    """Root p0 with fixed children (tokens 2, then 0): the first token follows p0 and the bonus
    after accepting the first child follows its row; each grid of G midpoints moves a branch
    probability by at most 1/G."""
    p0 = np.array([0.1, 0.45, 0.3, 0.15])
    p1 = np.array([0.25, 0.05, 0.5, 0.2])  # row at the child carrying token 2
    p2 = np.array([0.4, 0.3, 0.2, 0.1])  # row at the child carrying token 0
    G = 64
    g = (np.arange(G) + 0.5) / G
    A1, A2, R = (x.reshape(-1) for x in np.meshgrid(g, g, g, indexing="ij"))
    n = A1.size
    tgt = np.tile(np.log(np.stack([p0, p1, p2])), (n, 1))
    par = np.tile(np.array([-1, 0, 0], np.int32), n)
    tok = np.tile(np.array([-1, 2, 0], np.int32), n)
    ua = np.stack([np.zeros(n), A1, A2], 1).reshape(-1)
    ur = np.stack([R, R, R], 1).reshape(-1)
    r = oracle.verify_tree(tgt, np.full_like(tgt, np.nan), np.arange(0, 3 * n + 1, 3), par, tok, ua, ur,
                           np.ones(n), np.ones(n), 1, rule=oracle.TREE_DETERMINISTIC)
    assert (r["accept_len"] >= 0).all()  # the draft rows are not read under this rule
    first = r["tokens"][:, 0]
    assert np.abs(np.bincount(first, minlength=4) / n - p0).max() <= 3.0 / G
    acc1 = (r["accept_len"] == 1) & (r["path"][:, 0] == 1)
    assert abs(acc1.mean() - p0[2]) <= 1.0 / G  # accept probability r(t) = p0(2)
    bonus = np.bincount(r["tokens"][acc1, 1], minlength=4) / acc1.sum()
    assert np.abs(bonus - p1).max() <= 1.0 / G + 1e-12


def _apply(seq, length, code, lm, act, r):
    for row, b in enumerate(act):
        j = r["accept_len"][row]
        for t in r["tokens"][row, : j + 1]:
            seq[b, length[b]] = t
            code[b] = lm.extend(code[b], length[b], t)
            length[b] += 1


@pytest.mark.parametrize("top_k", [0, 2])
def test_multiround_deterministic_tree_matches_verifier_law(top_k):
    """Per round: draft marginals for K positions (the draft's next-token row, then its row
    after the draft's own argmax), the candidate trie over them, the deterministic rule; with
    top-k, the trie and the verification both use it and the law is the top-k verifier's."""
    V, L, N, T, K, ck, nv = 3, 4, 20000, 1.0, 2, 2, 4
    lm = TableLM(V, seed=500 + top_k)
    rng = np.random.default_rng(501 + top_k)
    seq = np.full((N, L + K + 1), -1, np.int64)
    length = np.zeros(N, np.int64)
    code = np.zeros(N, np.int64)
    while (length < L).any():
        act = np.nonzero(length < L)[0]
        n = act.size
        c0 = code[act]
        c1 = lm.extend(c0, length[act], np.argmax(lm.Q[c0], axis=1))
        offs, pars, toks, codes = [0], [], [], []
        for row in range(n):
            t = oracle.build_tree(np.stack([lm.Q[c0[row]], lm.Q[c1[row]]]), T, 1.0, ck, nv, top_k=top_k)
            m = len(t["parent"])
            nc = np.zeros(m, np.int64)
            nc[0] = c0[row]
            for i in range(1, m):
                nc[i] = lm.extend(nc[t["parent"][i]], length[act[row]] + t["depth"][i] - 1, t["tokens"][i])
            pars.append(t["parent"])
            toks.append(t["tokens"])
            codes.append(nc)
            offs.append(offs[-1] + m)
        codes = np.concatenate(codes)
        tok = np.concatenate(toks)
        tok[tok < 0] = 0
        r = oracle.verify_tree(lm.P[codes], lm.Q[codes], np.array(offs), np.concatenate(pars), tok,
                               rng.random(codes.size), rng.random(codes.size), np.full(n, T), np.ones(n), K,
                               top_k=np.full(n, top_k, np.int32), rule=oracle.TREE_DETERMINISTIC)
        assert (r["accept_len"] >= 0).all()
        _apply(seq, length, code, lm, act, r)
    _chi2_check(seq, lm.law(L, T, 1.0, top_k), V, L)


@pytest.mark.parametrize("top_k", [0, 2])
def test_multiround_with_replacement_tree_matches_verifier_law(top_k):
    """Binary trie of depth 2; every child drawn from its parent's q independently (siblings
    may repeat a token); the with-replacement rule, with and without top-k."""
    V, L, N, T = 3, 4, 20000, 1.0
    lm = TableLM(V, seed=600 + top_k, draft_noise=1.5)
    rng = np.random.default_rng(601 + top_k)
    kk = np.full(N, top_k, np.int32)
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
            toks[:, node] = oracle.sample_draft(lm.Q[codes[:, pa]], np.full(n, T), np.ones(n), rng.random(n),
                                                top_k=kk[:n])["tokens"]
            codes[:, node] = lm.extend(codes[:, pa], length[act] + (1 if pa == 0 else 2) - 1, toks[:, node])
        r = oracle.verify_tree(lm.P[codes].reshape(-1, V), lm.Q[codes].reshape(-1, V), np.arange(0, 7 * n + 1, 7),
                               np.tile(parent, n), toks.reshape(-1), rng.random(7 * n), rng.random(7 * n),
                               np.full(n, T), np.ones(n), 2, top_k=kk[:n], rule=oracle.TREE_SAMPLED_WR)
        assert (r["accept_len"] >= 0).all()
        _apply(seq, length, code, lm, act, r)
    _chi2_check(seq, lm.law(L, T, 1.0, top_k), V, L)


def test_rules_coincide_on_single_child_chains():
    rng = np.random.default_rng(21)
    B, D, V = 200, 4, 6
    n = D + 1
    tgt = rng.normal(0, 1.5, size=(B * n, V))
    drf = tgt + rng.normal(0, 1.0, size=tgt.shape)
    par = np.tile(np.arange(-1, D, dtype=np.int32), B)
    tok = rng.integers(0, V, size=B * n).astype(np.int32)
    ua, ur = rng.random(B * n), rng.random(B * n)
    args = (tgt, drf, np.arange(0, B * n + 1, n), par, tok, ua, ur, np.full(B, 0.9), np.full(B, 0.95), D)
    a = oracle.verify_tree(*args, rule=oracle.TREE_SAMPLED_WOR)
    b = oracle.verify_tree(*args, rule=oracle.TREE_SAMPLED_WR)
    for k in ("path", "tokens", "accept_len"):
        assert np.array_equal(a[k], b[k])
    with pytest.raises(ValueError):
        oracle.verify_tree(*args, rule=3)
