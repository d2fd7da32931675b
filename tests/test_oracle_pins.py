"""Pins for the CPU oracle: each check ties it to something other than itself.

Sources of truth, all independent of ``oracle/``: closed forms derived by hand
from the definitions ("More Value per Key: Asymmetric Sparse Attention for
Faster LLM Decoding", §2.1 Eq. (2), §2.5 Eq. (6), §3.1 Eq. (7), App. B
Eq. (29)); a pure-Python brute force; torch's float64
``scaled_dot_product_attention`` (dense attention, and dense attention with a
top-N mask chosen by ``torch.topk``); and invariants the definitions imply.
"""
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from bruteforce_ref import brute_row
from sparse_asymmetric_gqa_b200 import workload

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "closed_form_cases.json")


def _np(t):
    return t.float().numpy()


def _rand_case(seed, B, L, h_q, h_k, h_v, d, lens=None):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, h_q, d, generator=g).to(torch.bfloat16)
    k = torch.randn(B, h_k, L, d, generator=g).to(torch.bfloat16)
    v = torch.randn(B, h_v, L, d, generator=g).to(torch.bfloat16)
    if lens is None:
        lens = [L] * B
    return q, k, v, np.array(lens, dtype=np.int64)


def _expand(x, heads_out):
    """Block-expand cache heads so query head j sees head j // (h_q / h) (App. B Eq. (29))."""
    rep = heads_out // x.shape[1]
    return x.repeat_interleave(rep, dim=1)


# ---------------------------------------------------------------------------
# Closed forms (hand-derived, tests/golden/closed_form_cases.json)
# ---------------------------------------------------------------------------

def _eval_expr(s):
    return float(eval(s, {"__builtins__": {}},
                      {"sigmoid": lambda x: 1.0 / (1.0 + math.exp(-x)), "exp": math.exp}))


def _golden_cases():
    with open(GOLDEN) as f:
        return json.load(f)["cases"]


@pytest.mark.parametrize("case", _golden_cases(), ids=lambda c: c["name"])
def test_closed_form_cases(case):
    q = np.array(case["q"], dtype=np.float64)
    k = np.array(case["k"], dtype=np.float64)
    v = np.array(case["v"], dtype=np.float64)
    lens = np.array(case["seq_lens"])
    out, idx, _ = oracle.decode_attn(q, k, v, lens, case["h_q"], case["h_k"], case["h_v"], case["N"])
    for b in range(q.shape[0]):
        for j in range(case["h_q"]):
            assert list(idx[b][j]) == case["expected_idx"][b][j]
            want = np.array([_eval_expr(s) for s in case["expected_out"][b][j]])
            np.testing.assert_allclose(out[b, j], want, rtol=0, atol=1e-14)


# ---------------------------------------------------------------------------
# Brute force with exact ties
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("seed,L,d,N", [(1, 17, 8, 5), (2, 64, 8, 16), (3, 40, 4, 39),
                                         (4, 33, 8, 1), (5, 12, 8, 40)])
def test_bruteforce_with_ties(seed, L, d, N):
    rng = np.random.default_rng(seed)
    h_q, h_k, h_v = 4, 2, 1
    # small integers: many exactly equal scores, so the tie rule is exercised
    q = rng.integers(-2, 3, size=(1, h_q, d)).astype(np.float64)
    k = rng.integers(-2, 3, size=(1, h_k, L, d)).astype(np.float64)
    v = rng.standard_normal((1, h_v, L, d))
    lens = np.array([L])
    out, idx, zsel = oracle.decode_attn(q, k, v, lens, h_q, h_k, h_v, N)
    for j in range(h_q):
        kh = j // (h_q // h_k)
        vh = j // (h_q // h_v)
        b_out, b_idx, b_z = brute_row(q[0, j].tolist(), k[0, kh].tolist(), v[0, vh].tolist(), N)
        assert list(idx[0][j]) == b_idx
        np.testing.assert_allclose(zsel[0][j], b_z, rtol=0, atol=1e-12)
        np.testing.assert_allclose(out[0, j], b_out, rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------------------
# Library routines: dense attention, and dense attention under a top-N mask
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("shape", [(2, 96, 8, 2, 4, 16), (1, 130, 12, 1, 2, 32),
                                   (3, 50, 4, 4, 4, 8)])
def test_dense_equals_sdpa(shape):
    B, L, h_q, h_k, h_v, d = shape
    lens = [L - 7 * b for b in range(B)]
    q, k, v, lens = _rand_case(11, B, L, h_q, h_k, h_v, d, lens)
    out, idx, _ = oracle.decode_attn(_np(q), _np(k), _np(v), lens, h_q, h_k, h_v, N=L)
    for b in range(B):
        Lb = int(lens[b])
        qq = q[b:b + 1].double().unsqueeze(2)                      # [1, h_q, 1, d]
        kk = _expand(k[b:b + 1, :, :Lb].double(), h_q)             # [1, h_q, Lb, d]
        vv = _expand(v[b:b + 1, :, :Lb].double(), h_q)
        ref = F.scaled_dot_product_attention(qq, kk, vv)[0, :, 0]
        np.testing.assert_allclose(out[b], ref.numpy(), rtol=1e-12, atol=1e-12)
        for j in range(h_q):
            assert list(idx[b][j]) == list(range(Lb))


@pytest.mark.parametrize("N", [1, 7, 32, 100])
def test_topn_equals_masked_sdpa(N):
    B, L, h_q, h_k, h_v, d = 2, 160, 8, 2, 4, 16
    q, k, v, lens = _rand_case(23, B, L, h_q, h_k, h_v, d)
    out, idx, _ = oracle.decode_attn(_np(q), _np(k), _np(v), lens, h_q, h_k, h_v, N)
    qq = q.double().unsqueeze(2)
    kk = _expand(k.double(), h_q)
    vv = _expand(v.double(), h_q)
    logits = (qq @ kk.transpose(-1, -2))[:, :, 0] / math.sqrt(d)        # [B, h_q, L]
    top = torch.topk(logits, N, dim=-1).indices                         # random data: no ties
    mask = torch.zeros_like(logits, dtype=torch.bool).scatter_(-1, top, True)
    ref = F.scaled_dot_product_attention(qq, kk, vv, attn_mask=mask.unsqueeze(2))[:, :, 0]
    np.testing.assert_allclose(out, ref.numpy(), rtol=1e-12, atol=1e-12)
    for b in range(B):
        for j in range(h_q):
            assert list(idx[b][j]) == sorted(top[b, j].tolist())


# ---------------------------------------------------------------------------
# Invariants
# ---------------------------------------------------------------------------

def test_weights_sum_to_one_and_shift_invariance():
    rng = np.random.default_rng(5)
    for _ in range(20):
        z = rng.standard_normal(rng.integers(1, 300)) * rng.uniform(0.1, 30)
        p = oracle.softmax_selected(z)
        assert abs(p.sum() - 1.0) < 1e-12
        assert np.all(p >= 0)
        c = rng.uniform(-50, 50)
        np.testing.assert_allclose(oracle.softmax_selected(z + c), p, rtol=1e-10, atol=1e-15)


def test_asymmetric_equals_expanded_mha():
    """A SAGA layer equals an MHA layer whose heads are block-expanded copies."""
    B, L, h_q, h_k, h_v, d, N = 2, 200, 12, 1, 2, 16, 24
    q, k, v, lens = _rand_case(31, B, L, h_q, h_k, h_v, d, [200, 131])
    out, idx, _ = oracle.decode_attn(_np(q), _np(k), _np(v), lens, h_q, h_k, h_v, N)
    out2, idx2, _ = oracle.decode_attn(_np(q), _np(_expand(k, h_q)), _np(_expand(v, h_q)), lens,
                                       h_q, h_q, h_q, N)
    np.testing.assert_array_equal(out, out2)
    # and each MHA head is an independent single-head problem
    for j in range(h_q):
        o1, i1, _ = oracle.decode_attn(_np(q[:, j:j + 1]), _np(k), _np(v[:, j // 6:j // 6 + 1]),
                                       lens, 1, 1, 1, N)
        np.testing.assert_array_equal(o1[:, 0], out[:, j])


def test_nested_sets_in_N():
    rng = np.random.default_rng(7)
    z = np.round(rng.standard_normal(500), 1)   # rounding creates many ties
    prev = set()
    for N in range(1, 501, 13):
        cur = set(oracle.top_n(z, N).tolist())
        assert prev <= cur and len(cur) == N
        prev = cur


def test_nth_score_is_threshold():
    rng = np.random.default_rng(9)
    z = np.round(rng.standard_normal(300), 2)
    for N in (1, 5, 50, 299, 300, 400):
        t = oracle.nth_score(z, N)
        idx = oracle.top_n(z, N)
        n_b = min(N, 300)
        assert (z[idx] >= t).all()
        assert (z > t).sum() < n_b <= (z >= t).sum()


def test_planted_keys_selected_and_closed_form():
    """Tiny workload: 16 planted keys per query head equal 3 q_j, so each head's
    output is (to ~1e-5) the plain mean of V at its own planted positions."""
    spec = workload.TINY
    inp = workload.make_inputs(spec)
    q, k, v = _np(inp.q), _np(inp.k_cache), _np(inp.v_cache)
    lens = inp.seq_lens.numpy()
    out, idx, zsel = oracle.decode_attn(q, k, v, lens, spec.h_q, spec.h_k, spec.h_v, spec.N)
    by_head = {}
    for b, j, p in inp.planted:
        by_head.setdefault(j, []).append(p)
    assert len(by_head) == spec.h_q and all(len(p) == 16 for p in by_head.values())
    for j, pos in by_head.items():
        assert set(pos) <= set(idx[0][j].tolist())
        vh = j // spec.g_v
        mean_v = v[0, vh, sorted(pos)].astype(np.float64).mean(axis=0)
        np.testing.assert_allclose(out[0, j], mean_v, atol=1e-3)


def test_single_position_row():
    q, k, v, _ = _rand_case(3, 1, 8, 2, 1, 1, 8)
    out, idx, _ = oracle.decode_attn(_np(q), _np(k), _np(v), np.array([1]), 2, 1, 1, N=4)
    for j in range(2):
        assert list(idx[0][j]) == [0]
        np.testing.assert_array_equal(out[0, j], _np(v)[0, 0, 0].astype(np.float64))
