"""Comparison of CUDA-path outputs with the oracle's, honouring the agreed bands.

Integer results (accept lengths, token ids, tree paths) must be identical, except for a
request whose path holds a decision the oracle marks as within E_BAND (1e-6) of its
threshold: |u - p/q| (E1), a CDF edge against u (E2), or a top-p tail against top_p (E3).
Such requests are counted (by kind) and reported. One of them may differ only if the oracle
itself produces the CUDA path's result once the near-tied inputs are moved within the band:
the uniforms of the request, or its top_p, shifted by up to 2e-6 (see `Recheck`). Every
comparison also bounds the number of in-band requests (`band_limit`) and prints its counts.
Probabilities must agree to 1e-5 (entries behind a top-p near-tie are counted, not compared).
"""
import numpy as np

import oracle

E_BAND = 1e-6
P_TOL = 1e-5
SHIFTS = (-2e-6, -1e-6, 1e-6, 2e-6)
KIND_NAMES = {oracle.BAND_E1: "E1", oracle.BAND_E2: "E2", oracle.BAND_E3: "E3"}


def _np(x):
    """Host numpy view of an array or tensor (bf16 widened to fp32, which is exact)."""
    if hasattr(x, "detach"):
        x = x.detach().cpu()
        if str(x.dtype) == "torch.bfloat16":
            x = x.float()
        return x.numpy()
    return np.asarray(x)


def band_limit(n: int, V: int, draws: float = 1.0, cut_rows: float = 0.0) -> int:
    """Upper bound on the in-band requests among n. A draw over V tokens lands within 1e-6 of
    an edge of the drawn token's interval with probability about 2e-6 per token of support
    (the expectation of 2e-6 / p over the drawn token's probability p), so about 2e-6 V per
    draw; a top-p threshold is near a tail with probability below 1e-3 per cut row at these
    sizes. The bound is three times the expected count, plus 3."""
    rate = min(1.0, 2e-6 * V * draws + 1e-3 * cut_rows)
    return int(3 * rate * n + 3)


def _clip_u(u):
    return np.clip(u, 0.0, 1.0 - 2.0 ** -24)


class Recheck:
    """Outcomes of the oracle for one request with its near-tied inputs moved within the band:
    every uniform of the request shifted together, the accept and residual uniforms shifted
    separately, and top_p shifted, each by the offsets in SHIFTS."""

    def __init__(self, run):
        self.run = run  # run(b, shift_acc, shift_res, shift_p) -> the oracle's outcome

    def outcomes(self, b):
        out = set()
        for d in SHIFTS:
            for sa, sr, sp in ((d, d, 0.0), (d, 0.0, 0.0), (0.0, d, 0.0), (0.0, 0.0, d), (d, d, d)):
                out.add(self.run(b, sa, sr, sp))
        return out


def linear_recheck(tgt, drf, x, ua, ur, T, P, top_k=None):
    """Recheck for verify_linear inputs (host arrays or CPU tensors indexed by request)."""
    tgt, drf = _np(tgt), _np(drf)
    x, ua, ur, T, P = (np.asarray(_np(a)) for a in (x, ua, ur, T, P))
    tk = None if top_k is None else np.asarray(_np(top_k))

    def run(b, sa, sr, sp):
        r = oracle.verify_linear(tgt[b:b + 1].astype(np.float64), drf[b:b + 1].astype(np.float64), x[b:b + 1],
                                 _clip_u(ua[b:b + 1] + sa), _clip_u(ur[b:b + 1] + sr), T[b:b + 1],
                                 np.minimum(P[b:b + 1] + sp, 1.0) if P[b] < 1.0 else P[b:b + 1],
                                 top_k=None if tk is None else tk[b:b + 1])
        return int(r["accept_len"][0]), tuple(int(t) for t in r["tokens"][0])

    return Recheck(run)


def sample_recheck(drf_rows, T, P, u, row_req, top_k=None):
    """Recheck for sample_draft inputs: one draft row per index."""
    d = _np(drf_rows)
    u, rr, T, P = np.asarray(_np(u)).reshape(-1), np.asarray(row_req), np.asarray(_np(T)), np.asarray(_np(P))
    tk = None if top_k is None else np.asarray(_np(top_k))

    def run(i, sa, sr, sp):
        b = rr[i]
        r = oracle.sample_draft(d[i:i + 1].astype(np.float64), T[b:b + 1], np.minimum(P[b:b + 1] + sp, 1.0)
                                if P[b] < 1.0 else P[b:b + 1], _clip_u(u[i:i + 1] + sa), row_req=[0],
                                top_k=None if tk is None else tk[b:b + 1])
        return int(r["tokens"][0])

    return Recheck(run)


def tree_recheck(tgt, drf, offs, parent, tokens, ua, ur, T, P, max_depth, top_k=None, rule=oracle.TREE_SAMPLED_WOR):
    """Recheck for verify_tree inputs (nodes of request b are offs[b]:offs[b+1])."""
    tgt, drf = _np(tgt), _np(drf)
    offs, parent, tokens = np.asarray(_np(offs)), np.asarray(_np(parent)), np.asarray(_np(tokens))
    ua, ur, T, P = (np.asarray(_np(a)) for a in (ua, ur, T, P))
    tk = None if top_k is None else np.asarray(_np(top_k))

    def run(b, sa, sr, sp):
        s, e = int(offs[b]), int(offs[b + 1])
        r = oracle.verify_tree(tgt[s:e].astype(np.float64), drf[s:e].astype(np.float64), [0, e - s], parent[s:e],
                               tokens[s:e], _clip_u(ua[s:e] + sa), _clip_u(ur[s:e] + sr), T[b:b + 1],
                               np.minimum(P[b:b + 1] + sp, 1.0) if P[b] < 1.0 else P[b:b + 1], max_depth,
                               top_k=None if tk is None else tk[b:b + 1], rule=rule)
        return (int(r["accept_len"][0]), tuple(int(t) for t in r["tokens"][0]), tuple(int(t) for t in r["path"][0]))

    return Recheck(run)


def _kinds(ora, in_band):
    k = np.asarray(ora.get("band_kind", np.zeros(in_band.size, np.int32)))
    return {name: int((in_band & (k == code)).sum()) for code, name in KIND_NAMES.items()}


def _finish(label, n, in_band, differ, ora, limit, extra=None):
    rep = {"n": int(n), "in_band": int(in_band.sum()), "kinds": _kinds(ora, in_band),
           "differ_in_band": int(differ.sum())}
    if extra:
        rep.update(extra)
    print("parity %s: %s" % (label or "", rep))
    if limit is not None:
        assert rep["in_band"] <= limit, "%d in-band of %d exceeds the bound %d" % (rep["in_band"], n, limit)
    return rep


def _explain(differ, recheck, gpu_outcome, what):
    """Every in-band difference must be an outcome of the oracle within the band."""
    for b in np.nonzero(differ)[0]:
        assert recheck is not None, "%s %d differs in band and no recheck was given" % (what, b)
        got = gpu_outcome(b)
        ok = recheck.outcomes(int(b))
        assert got in ok, "%s %d: GPU outcome %s is not an oracle outcome within the band %s" % (what, b, got, ok)


def compare_linear(gpu: dict, ora: dict, check_pq: bool = True, recheck: Recheck = None, limit: int = None,
                   label: str = None) -> dict:
    g_len, o_len = _np(gpu["accept_len"]), ora["accept_len"]
    g_tok, o_tok = _np(gpu["tokens"]), ora["tokens"]
    band = ora["band"]
    in_band = band < E_BAND
    same = (g_len == o_len) & (g_tok == o_tok).all(axis=1)
    bad = ~same & ~in_band
    assert not bad.any(), "mismatch outside the bands at requests %s: gpu len %s tok %s / oracle len %s tok %s band %s" % (
        np.nonzero(bad)[0][:5], g_len[bad][:5], g_tok[bad][:3], o_len[bad][:5], o_tok[bad][:3], band[bad][:5])
    differ = ~same & in_band
    _explain(differ, recheck, lambda b: (int(g_len[b]), tuple(int(t) for t in g_tok[b])), "request")
    pq_skipped = 0
    if check_pq and gpu.get("p") is not None:
        gp, gq = _np(gpu["p"]), _np(gpu["q"])
        ok = ora["pq_band"] >= E_BAND
        pq_skipped = int((~ok).sum())
        dp = np.abs(gp - ora["p"])[ok]
        dq = np.abs(gq - ora["q"])[ok]
        assert dp.size == 0 or dp.max() <= P_TOL, dp.max()
        assert dq.size == 0 or dq.max() <= P_TOL, dq.max()
    rep = _finish(label, g_len.size, in_band, differ, ora, limit, {"pq_in_band": pq_skipped})
    rep["mean_accept"] = float(o_len[o_len >= 0].mean()) if (o_len >= 0).any() else float("nan")
    return rep


def compare_sample(g_tok, g_q, ora: dict, recheck: Recheck = None, limit: int = None, label: str = None) -> dict:
    g_tok, g_q = _np(g_tok).reshape(-1), _np(g_q).reshape(-1)
    o_tok, band = ora["tokens"], ora["band"]
    in_band = band < E_BAND
    same = g_tok == o_tok
    bad = ~same & ~in_band
    assert not bad.any(), "sample mismatch outside the bands at rows %s: gpu %s oracle %s band %s" % (
        np.nonzero(bad)[0][:5], g_tok[bad][:5], o_tok[bad][:5], band[bad][:5])
    differ = ~same & in_band
    _explain(differ, recheck, lambda i: int(g_tok[i]), "row")
    ok = same & (o_tok >= 0)
    dq = np.abs(g_q[ok] - ora["q"][ok])
    assert dq.size == 0 or dq.max() <= P_TOL, dq.max()
    return _finish(label, g_tok.size, in_band, differ, ora, limit)


def compare_tree(gpu: dict, ora: dict, recheck: Recheck = None, limit: int = None, label: str = None) -> dict:
    g_len, o_len = _np(gpu["accept_len"]), ora["accept_len"]
    g_tok, g_path = _np(gpu["tokens"]), _np(gpu["path"])
    same = (g_len == o_len) & (g_tok == ora["tokens"]).all(axis=1) & (g_path == ora["path"]).all(axis=1)
    in_band = ora["band"] < E_BAND
    bad = ~same & ~in_band
    assert not bad.any(), "tree mismatch outside the bands at requests %s: gpu %s / oracle %s" % (
        np.nonzero(bad)[0][:5], g_tok[bad][:3], ora["tokens"][bad][:3])
    differ = ~same & in_band
    _explain(differ, recheck, lambda b: (int(g_len[b]), tuple(int(t) for t in g_tok[b]),
                                         tuple(int(t) for t in g_path[b])), "trie")
    return _finish(label, g_len.size, in_band, differ, ora, limit)
