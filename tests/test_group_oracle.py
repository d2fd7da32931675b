"""Pins for the group-shared selection oracle (one position set per value head).

Each pin checks the oracle against something other than its own formula: the
per-head exact top-N and dense attention of ``oracle.saga_oracle`` (independent
code), a hand-computed two-head case, and invariants of the definition.
"""
import math

import numpy as np
import pytest

import oracle
from oracle import group_oracle as go


def _rows(seed, g_v, L, d):
    rng = np.random.default_rng(seed)
    return rng.normal(0, 1, (g_v, d)), rng.normal(0, 1, (L, d)), rng.normal(0, 1, (L, d))


@pytest.mark.parametrize("N", [1, 7, 64])
def test_group_of_one_head_is_the_exact_top_n(N):
    q, k, v = _rows(1, 1, 200, 16)
    out, idx = go.group_rows(q, k, v, N)
    z = oracle.scores(q[0], k)
    assert np.array_equal(idx, np.sort(oracle.top_n(z, N)))
    ref = oracle.combine(z[np.sort(oracle.top_n(z, N))], v[np.sort(oracle.top_n(z, N))])
    np.testing.assert_allclose(out[0], ref, rtol=0, atol=1e-12)


def test_group_of_identical_heads_is_each_heads_top_n():
    q1, k, v = _rows(2, 1, 150, 8)
    q = np.repeat(q1, 4, axis=0)
    out, idx = go.group_rows(q, k, v, 20)
    z = oracle.scores(q1[0], k)
    assert np.array_equal(idx, np.sort(oracle.top_n(z, 20)))
    assert np.allclose(out, out[0])


def test_per_head_shift_invariance():
    q, k, _ = _rows(3, 3, 300, 8)
    z = (q @ k.T) / math.sqrt(8)
    a = go.group_select(z, 40)
    b = go.group_select(z + np.array([[5.0], [-2.0], [30.0]]), 40)
    assert np.array_equal(a, b)


def test_hand_computed_two_heads():
    # z1 = [0, ln 2, 0] -> p1 = [1/4, 1/2, 1/4]; z2 = [ln 3, 0, 0] -> p2 = [3/5, 1/5, 1/5]
    # s = [0.85, 0.70, 0.45]: N = 1 keeps {0}, N = 2 keeps {0, 1}
    z = np.array([[0.0, math.log(2.0), 0.0], [math.log(3.0), 0.0, 0.0]])
    assert np.allclose(go.group_statistic(z), [0.85, 0.70, 0.45], atol=1e-15)
    assert go.group_select(z, 1).tolist() == [0]
    assert go.group_select(z, 2).tolist() == [0, 1]
    # outputs over I = {0, 1}: head 1 weights [1/3, 2/3], head 2 weights [3/4, 1/4];
    # keys chosen so that q . k / sqrt(d) reproduces z (d = 4, k_i = 2 e_i)
    k = np.eye(3, 4) * 2.0
    q = np.zeros((2, 4))
    q[0, :3] = z[0]
    q[1, :3] = z[1]
    v = np.array([[1.0, 0, 0, 0], [0, 1.0, 0, 0], [0, 0, 1.0, 0]])
    out, idx = go.group_rows(q, k, v, 2)
    assert idx.tolist() == [0, 1]
    np.testing.assert_allclose(out[0], [1 / 3, 2 / 3, 0, 0], atol=1e-15)
    np.testing.assert_allclose(out[1], [3 / 4, 1 / 4, 0, 0], atol=1e-15)


def test_everything_selected_is_dense_attention_per_head():
    q, k, v = _rows(5, 3, 40, 8)
    out, idx = go.group_rows(q, k, v, 100)
    assert idx.tolist() == list(range(40))
    for j in range(3):
        z = oracle.scores(q[j], k)
        np.testing.assert_allclose(out[j], oracle.combine(z, v), rtol=0, atol=1e-12)


def test_sets_are_nested_in_N():
    q, k, _ = _rows(6, 6, 500, 16)
    z = (q @ k.T) / 4.0
    prev = set()
    for N in (1, 5, 50, 200, 500):
        cur = set(go.group_select(z, N).tolist())
        assert prev <= cur and len(cur) == N
        prev = cur


def test_group_attn_uses_value_heads_and_ragged_rows():
    rng = np.random.default_rng(7)
    B, h_q, h_k, h_v, d, L = 2, 4, 1, 2, 8, 30
    q = rng.normal(0, 1, (B, h_q, d))
    k = rng.normal(0, 1, (B, h_k, L, d))
    v = rng.normal(0, 1, (B, h_v, L, d))
    lens = [30, 11]
    out, sets = go.group_attn(q, k, v, lens, h_q, h_k, h_v, 5)
    assert set(sets) == {(b, vh) for b in range(B) for vh in range(h_v)}
    for (b, vh), idx in sets.items():
        assert len(idx) == 5 and idx.max() < lens[b]
        heads = [2 * vh, 2 * vh + 1]
        o, i2 = go.group_rows(q[b, heads], k[b, 0, :lens[b]], v[b, vh, :lens[b]], 5)
        assert np.array_equal(i2, idx)
        np.testing.assert_allclose(out[b, heads], o, rtol=0, atol=1e-12)
