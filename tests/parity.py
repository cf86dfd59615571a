"""Comparison of CUDA-path outputs with the oracle's, honouring the agreed bands.

Integer results (accept lengths, token ids, tree paths) must be identical, except for a
request whose path holds a decision the oracle marks as within E_BAND (1e-6) of its
threshold: |u - p/q|, a CDF boundary against u, or a top-p tail against top_p. Such requests
are counted and reported, and only they may differ. Probabilities must agree to 1e-5.
"""
import numpy as np

E_BAND = 1e-6
P_TOL = 1e-5


def _np(x):
    return x.detach().cpu().numpy() if hasattr(x, "detach") else np.asarray(x)


def compare_linear(gpu: dict, ora: dict, check_pq: bool = True) -> dict:
    g_len, o_len = _np(gpu["accept_len"]), ora["accept_len"]
    g_tok, o_tok = _np(gpu["tokens"]), ora["tokens"]
    band = ora["band"]
    in_band = band < E_BAND
    same = (g_len == o_len) & (g_tok == o_tok).all(axis=1)
    bad = ~same & ~in_band
    assert not bad.any(), "mismatch outside the bands at requests %s: gpu len %s tok %s / oracle len %s tok %s band %s" % (
        np.nonzero(bad)[0][:5], g_len[bad][:5], g_tok[bad][:3], o_len[bad][:5], o_tok[bad][:3], band[bad][:5])
    if check_pq and gpu.get("p") is not None:
        gp, gq = _np(gpu["p"]), _np(gpu["q"])
        ok = ora["pq_band"] >= E_BAND
        dp = np.abs(gp - ora["p"])[ok]
        dq = np.abs(gq - ora["q"])[ok]
        assert dp.size == 0 or dp.max() <= P_TOL, dp.max()
        assert dq.size == 0 or dq.max() <= P_TOL, dq.max()
    return {"requests": int(g_len.size), "in_band": int(in_band.sum()), "differ_in_band": int((~same & in_band).sum()),
            "mean_accept": float(o_len[o_len >= 0].mean()) if (o_len >= 0).any() else float("nan")}


def compare_sample(g_tok, g_q, ora: dict) -> dict:
    g_tok, g_q = _np(g_tok).reshape(-1), _np(g_q).reshape(-1)
    o_tok, band = ora["tokens"], ora["band"]
    in_band = band < E_BAND
    same = g_tok == o_tok
    bad = ~same & ~in_band
    assert not bad.any(), "sample mismatch outside the bands at rows %s: gpu %s oracle %s band %s" % (
        np.nonzero(bad)[0][:5], g_tok[bad][:5], o_tok[bad][:5], band[bad][:5])
    ok = same & (o_tok >= 0)
    dq = np.abs(g_q[ok] - ora["q"][ok])
    assert dq.size == 0 or dq.max() <= P_TOL, dq.max()
    return {"rows": int(g_tok.size), "in_band": int(in_band.sum()), "differ_in_band": int((~same & in_band).sum())}


def compare_tree(gpu: dict, ora: dict) -> dict:
    g_len, o_len = _np(gpu["accept_len"]), ora["accept_len"]
    same = (g_len == o_len) & (_np(gpu["tokens"]) == ora["tokens"]).all(axis=1) & (
        _np(gpu["path"]) == ora["path"]).all(axis=1)
    in_band = ora["band"] < E_BAND
    bad = ~same & ~in_band
    assert not bad.any(), "tree mismatch outside the bands at requests %s: gpu %s / oracle %s" % (
        np.nonzero(bad)[0][:5], _np(gpu["tokens"])[bad][:3], ora["tokens"][bad][:3])
    return {"requests": int(g_len.size), "in_band": int(in_band.sum()), "differ_in_band": int((~same & in_band).sum())}
