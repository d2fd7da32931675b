"""Pins for the stateful Atop-N oracle (calibrated threshold reused across steps).

Each pin checks the oracle against something other than its own formula: the
algebraic identity that a step with tau calibrated on the same scores puts the
threshold exactly on the N-th score (for any tail), hand-computed thresholds,
shift invariance, the capacity rule, and the exact top-N / dense oracles.
"More Value per Key", §3.1 and App. C.1.
"""
import math

import numpy as np
import pytest

import oracle
from oracle import atopn_oracle as ao


def _tie_free(rng, L):
    # distinct scores with gaps well above float64 rounding
    return rng.permutation(L).astype(np.float64) * 1e-3 + rng.normal(0, 1e-6, L) + rng.normal(0, 1.5, 1)


@pytest.mark.parametrize("L,N", [(50, 7), (300, 100), (1000, 1), (64, 64)])
def test_calibrated_threshold_is_the_nth_score_for_any_tail(L, N):
    # t = m_hat + log(p_N * s_hat) and s_hat = exp(m - m_hat) * sum exp(z - m), so
    # t = m_hat + (z_N - m) + (m - m_hat) = z_N whatever the tail
    rng = np.random.default_rng(L + N)
    z = _tie_free(rng, L) * 3.0
    tau = ao.calibrate_tau(z, N)
    z_n = np.sort(z)[::-1][min(N, L) - 1]
    for tail in (1, 5, L // 2, L):
        assert abs(ao.step_threshold(z, tau, tail) - z_n) < 1e-9
        # a hair below: exactly the top-N positions, as the exact oracle selects them
        sel = ao.step_select(z, tau * (1 - 1e-7), tail, cap=2 * N)
        assert np.array_equal(sel, np.sort(oracle.top_n(z, N)))


def test_hand_computed_thresholds():
    # z = [0, ln 2, ln 3], tail 1: m_hat = ln 3, s_hat = (1 + 2 + 3) / 3 = 2
    z = np.array([0.0, math.log(2.0), math.log(3.0)])
    assert ao.step_threshold(z, 0.3, 1) == pytest.approx(math.log(1.8), abs=1e-12)
    assert ao.step_select(z, 0.3, 1, cap=6).tolist() == [1, 2]          # t = ln 1.8
    assert ao.step_select(z, 0.4, 1, cap=6).tolist() == [2]             # t = ln 2.4
    assert ao.step_select(z, 0.1, 1, cap=6).tolist() == [0, 1, 2]       # t = ln 0.6 < 0
    # tail 3 (the whole row): m_hat = ln 3 again, same thresholds
    assert ao.step_select(z, 0.3, 3, cap=6).tolist() == [1, 2]


def test_calibrate_tau_closed_form():
    # p = [1/4, 1/4, 1/2]: the 2nd largest probability is 1/4, the 1st 1/2
    z = np.array([0.0, 0.0, math.log(2.0)])
    assert ao.calibrate_tau(z, 2) == pytest.approx(0.25, abs=1e-15)
    assert ao.calibrate_tau(z, 1) == pytest.approx(0.5, abs=1e-15)
    assert ao.calibrate_tau(z, 10) == pytest.approx(0.25, abs=1e-15)   # N >= L: the smallest


def test_shift_invariance():
    rng = np.random.default_rng(3)
    z = _tie_free(rng, 500)
    for tau in (1e-4, 3e-3, 2e-2):
        a = ao.step_select(z, tau, 16, cap=400)
        b = ao.step_select(z + 7.25, tau, 16, cap=400)
        assert np.array_equal(a, b)


def test_capacity_keeps_the_lowest_positions():
    rng = np.random.default_rng(4)
    z = rng.normal(0, 1, 200)
    sel = ao.step_select(z, 1e-12, 8, cap=30)          # every entry passes
    assert sel.tolist() == list(range(30))


def test_step_with_everything_selected_is_dense_attention():
    rng = np.random.default_rng(5)
    d, L = 16, 40
    q = rng.normal(0, 1, d)
    k = rng.normal(0, 1, (L, d))
    v = rng.normal(0, 1, (L, d))
    out, idx, _ = ao.step_row(q, k, v, 1e-12, 4, cap=2 * L)
    assert idx.tolist() == list(range(L))
    z = k @ q / math.sqrt(d)
    p = np.exp(z - z.max())
    p /= p.sum()
    np.testing.assert_allclose(out, p @ v, rtol=0, atol=1e-12)
    # the exact oracle with N = L is the same dense attention
    ref = oracle.combine(z, v)
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)


def test_threshold_above_every_probability_selects_nothing():
    # the row's largest probability is 1/2 (z = [0, 0, ln 2]); tau = 0.6 is above it
    z = np.array([0.0, 0.0, math.log(2.0)])
    assert ao.step_select(z, 0.6, 1, cap=6).size == 0
    k = np.eye(3, 4) * 2.0
    q = np.array([0.0, 0.0, math.log(2.0), 0.0])
    out, idx, _ = ao.step_row(q, k, np.ones((3, 4)), 0.9, 1, cap=6)
    assert idx.size == 0 and np.all(out == 0.0)
