"""Pins of the oracle's exception bands (no GPU).

The parity tests compare the CUDA path with the oracle exactly, except on requests whose path
holds a decision within 1e-6 of its boundary (the oracle's "band"): an accept test u against
p/q (E1), an inverse-CDF draw against the edges of the drawn token's interval (E2), a top-p
threshold against the tail masses (E3). Those requests are counted and reported, so a wrong
band would hide mismatches. These tests fix the bands by hand-derived values
(tests/golden/bands.txt), by edges placed a known distance from u, and by the kind of decision
each band names. Source of the decisions: review page of arXiv 2609.04010, section 3.3 (accept
with min(1, p/q), residual [p - q]_+, bonus draw) and the README's --top-p control.
"""
import math

import numpy as np
import pytest

import oracle
from goldens import load, nums, rows

BANDS = load("bands.txt")


def _kind(k):
    return [c for c in BANDS if c["kind"] == k]


def _f(s):
    return nums(s)[0]


def _close(got, want):
    if math.isinf(want):
        assert math.isinf(got), got
    else:
        assert abs(got - want) <= 1e-12, (got, want)


@pytest.mark.parametrize("case", _kind("cdf"), ids=lambda c: c["name"])
def test_cdf_band(case):
    y, band = oracle.inverse_cdf(nums(case["weights"]), _f(case["u"]))
    assert y == int(_f(case["expect_token"]))
    _close(band, _f(case["expect_band"]))


@pytest.mark.parametrize("case", _kind("row"), ids=lambda c: c["name"])
def test_topp_band(case):
    _, band = oracle.row_dist(nums(case["logits"]), _f(case["T"]), _f(case["top_p"]), int(_f(case["top_k"])))
    _close(band, _f(case["expect_band"]))


@pytest.mark.parametrize("case", _kind("sample"), ids=lambda c: c["name"])
def test_sample_band(case):
    r = oracle.sample_draft(np.array([nums(case["logits"])]), [_f(case["T"])], [_f(case["top_p"])], [_f(case["u"])])
    assert r["tokens"][0] == int(_f(case["expect_token"]))
    _close(r["band"][0], _f(case["expect_band"]))


@pytest.mark.parametrize("case", _kind("linear"), ids=lambda c: c["name"])
def test_linear_band(case):
    tgt, drf = rows(case["target"]), rows(case["draft"])
    r = oracle.verify_linear(tgt[None], drf[None], np.array(nums(case["tokens"]), np.int32)[None],
                             np.array(nums(case["u_accept"]))[None], np.array(nums(case["u_resid"]))[None],
                             [_f(case["T"])], [_f(case["top_p"])])
    assert r["accept_len"][0] == int(_f(case["expect_len"]))
    assert r["tokens"][0].tolist() == [int(x) for x in nums(case["expect_tokens"])]
    _close(r["band"][0], _f(case["expect_band"]))


@pytest.mark.parametrize("case", _kind("tree"), ids=lambda c: c["name"])
def test_tree_band(case):
    tgt, drf = rows(case["target"]), rows(case["draft"])
    n = tgt.shape[0]
    rule = {"deterministic": oracle.TREE_DETERMINISTIC}.get(case.get("rule"), oracle.TREE_SAMPLED_WOR)
    r = oracle.verify_tree(tgt, drf, [0, n], np.array(nums(case["parent"]), np.int32),
                           np.array(nums(case["tokens"]), np.int32), nums(case["u_accept"]), nums(case["u_resid"]),
                           [_f(case["T"])], [_f(case["top_p"])], int(case["max_depth"]), rule=rule)
    assert r["accept_len"][0] == int(_f(case["expect_len"]))
    assert r["path"][0].tolist() == [int(x) for x in nums(case["expect_path"])]
    assert r["tokens"][0].tolist() == [int(x) for x in nums(case["expect_tokens"])]
    _close(r["band"][0], _f(case["expect_band"]))


def test_band_kinds_name_the_closest_decision():
    """band_kind says which decision gives the band: the accept test (E1), a draw edge (E2), a
    top-p tail (E3)."""
    by_name = {c["name"]: c for c in BANDS}
    want = {"accept_then_bonus": oracle.BAND_E1, "bonus_edge_is_closest": oracle.BAND_E2,
            "reject_then_residual": oracle.BAND_E1, "residual_edge_is_closest": oracle.BAND_E2,
            "topp_threshold_is_closest": oracle.BAND_E3}
    for name, kind in want.items():
        c = by_name[name]
        tgt, drf = rows(c["target"]), rows(c["draft"])
        r = oracle.verify_linear(tgt[None], drf[None], np.array(nums(c["tokens"]), np.int32)[None],
                                 np.array(nums(c["u_accept"]))[None], np.array(nums(c["u_resid"]))[None],
                                 [_f(c["T"])], [_f(c["top_p"])])
        assert r["band_kind"][0] == kind, (name, r["band_kind"][0])
    for name, kind in {"draw_with_topp": oracle.BAND_E3, "draw_without_cut": oracle.BAND_E2}.items():
        c = by_name[name]
        r = oracle.sample_draft(np.array([nums(c["logits"])]), [_f(c["T"])], [_f(c["top_p"])], [_f(c["u"])])
        assert r["band_kind"][0] == kind, (name, r["band_kind"][0])
    for name, kind in {"reject_accept_bonus": oracle.BAND_E1, "leaf_draw_is_closest": oracle.BAND_E2}.items():
        c = by_name[name]
        tgt, drf = rows(c["target"]), rows(c["draft"])
        r = oracle.verify_tree(tgt, drf, [0, tgt.shape[0]], np.array(nums(c["parent"]), np.int32),
                               np.array(nums(c["tokens"]), np.int32), nums(c["u_accept"]), nums(c["u_resid"]),
                               [_f(c["T"])], [_f(c["top_p"])], int(c["max_depth"]))
        assert r["band_kind"][0] == kind, (name, r["band_kind"][0])


def test_draw_band_tracks_the_distance_to_every_edge():
    """Integer weights give exact CDF edges k/Z. For u placed d above an edge (and d below the
    next one) the band is exactly d, whatever the edge: 1e-7 is inside the 1e-6 band, 1e-3 is
    not. Zero weights add no edge."""
    rng = np.random.default_rng(11)
    for _ in range(40):
        V = int(rng.integers(2, 40))
        w = rng.integers(0, 5, size=V).astype(np.float64)
        w[rng.integers(0, V)] += 1.0
        Z = float(w.sum())
        edges = np.concatenate([[0.0], np.cumsum(w)]) / Z  # exact: small integers over Z
        for v in np.nonzero(w)[0]:
            lo, hi = edges[v], edges[v + 1]
            for d in (1e-7, 1e-3):
                if hi - lo <= 2 * d:
                    continue
                for u, want in ((lo + d, d), (hi - d, d)):
                    y, band = oracle.inverse_cdf(w, u)
                    assert y == v, (w, u, y, v)
                    assert abs(band - want) <= 1e-12, (w, u, band, want)
                    assert (band < oracle.E_BAND) == (d < oracle.E_BAND)


def test_ratio_band_tracks_u():
    """One position, p = (1/2, 1/2), q = (3/4, 1/4), x = 0 (p/q = 2/3); the bonus draw is kept
    far from its edges. The band is |u - 2/3| on both sides of the boundary."""
    tgt = np.array([[[0.0, 0.0], [math.log(4.0), 0.0]]])
    drf = np.array([[[math.log(3.0), 0.0]]])
    for d in (1e-7, 5e-7, 2e-6, 1e-3, 0.05):
        for sign in (-1, 1):
            u = 2.0 / 3.0 + sign * d
            r = oracle.verify_linear(tgt, drf, np.array([[0]], np.int32), np.array([[u]]),
                                     np.array([[0.5, 0.5 if sign < 0 else 0.6]]), [1.0], [1.0])
            assert r["accept_len"][0] == (1 if sign < 0 else 0)
            assert abs(r["band"][0] - d) <= 1e-12, (u, r["band"][0], d)
            assert r["band_kind"][0] == oracle.BAND_E1


def test_topp_band_tracks_top_p():
    """p = (0.6, 0.3, 0.1): the band of top_p = tail +- d is d, at both tails."""
    l = [math.log(6.0), math.log(3.0), 0.0]
    for tail in (0.6, 0.9):
        for d in (1e-7, 3e-4, 0.02):
            for sign in (-1, 1):
                _, band = oracle.row_dist(l, 1.0, tail + sign * d)
                assert abs(band - d) <= 1e-12, (tail, sign, d, band)
