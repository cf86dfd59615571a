"""Host logic of the parity comparison (no GPU): what an in-band difference must satisfy.

A request whose decision lies within 1e-6 of its boundary may come out differently in the
CUDA path only if the oracle gives that same outcome with the near-tied inputs moved within the
band. These tests feed hand-made "device" outputs to the comparison helpers.
"""
import math

import numpy as np
import pytest

import oracle
from parity import band_limit, compare_linear, compare_sample, linear_recheck, sample_recheck

# p_0 = (1/2, 1/2), q_0 = (3/4, 1/4), x = 0 (p/q = 2/3, accepted with u = 0.6); the bonus row
# p_1 = (4/5, 1/5) has its CDF edge at 4/5.
TGT = np.array([[[0.0, 0.0], [math.log(4.0), 0.0]]])
DRF = np.array([[[math.log(3.0), 0.0]]])
X = np.array([[0]], np.int32)
UA = np.array([[0.6]])


def _ora(ur):
    return oracle.verify_linear(TGT, DRF, X, UA, ur, [1.0], [1.0])


def _fake(len_, toks):
    return {"accept_len": np.array([len_], np.int32), "tokens": np.array([toks], np.int32)}


def test_in_band_difference_reproduced_within_the_band_passes():
    ur = np.array([[0.5, 0.8 - 5e-7]])  # the bonus draw 5e-7 below the edge: token 0, in band
    ora = _ora(ur)
    assert ora["tokens"][0].tolist() == [0, 0] and ora["band"][0] < 1e-6
    rc = linear_recheck(TGT, DRF, X, UA, ur, [1.0], [1.0])
    rep = compare_linear(_fake(1, [0, 1]), ora, check_pq=False, recheck=rc, limit=1)
    assert rep["in_band"] == 1 and rep["differ_in_band"] == 1 and rep["kinds"]["E2"] == 1


def test_in_band_difference_not_reproduced_fails():
    ur = np.array([[0.5, 0.8 - 5e-7]])
    ora = _ora(ur)
    rc = linear_recheck(TGT, DRF, X, UA, ur, [1.0], [1.0])
    with pytest.raises(AssertionError):  # a rejection is not an outcome within the band
        compare_linear(_fake(0, [1, -1]), ora, check_pq=False, recheck=rc)


def test_difference_outside_the_band_fails():
    ur = np.array([[0.5, 0.5]])
    ora = _ora(ur)
    assert ora["band"][0] > 1e-6
    with pytest.raises(AssertionError):
        compare_linear(_fake(1, [0, 1]), ora, check_pq=False, recheck=linear_recheck(TGT, DRF, X, UA, ur, [1.0], [1.0]))


def test_in_band_count_is_bounded():
    ur = np.array([[0.5, 0.8 - 5e-7]])
    ora = _ora(ur)
    with pytest.raises(AssertionError):
        compare_linear(_fake(1, [0, 0]), ora, check_pq=False, limit=0)


def test_sample_in_band_difference():
    d = np.array([[math.log(6.0), math.log(3.0), 0.0]])  # q = (0.6, 0.3, 0.1), edges 0.6, 0.9
    u = np.array([0.9 - 3e-7])
    ora = oracle.sample_draft(d, [1.0], [1.0], u)
    assert ora["tokens"][0] == 1 and ora["band"][0] < 1e-6
    rc = sample_recheck(d, [1.0], [1.0], u, [0])
    compare_sample(np.array([2]), np.array([0.1]), ora, recheck=rc, limit=1)
    with pytest.raises(AssertionError):
        compare_sample(np.array([0]), np.array([0.6]), ora, recheck=rc)


def test_band_limit_grows_with_the_support():
    assert band_limit(100, 8) == 3
    assert band_limit(100, 151936) > band_limit(100, 20000) > band_limit(100, 1000)
    assert band_limit(10, 151936, 1.0) <= 3 * 10 + 3
