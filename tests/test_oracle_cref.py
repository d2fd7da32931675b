"""The plain C++ oracle (``oracle/decode_ref.cpp``) against the NumPy oracle.

Two independent implementations of the same definitions (scores, top-N with
ties to the lowest position, softmax over the selection, gathered P.V): index
sets must be identical and values equal to double rounding; one thread and
several threads must give bit-identical results.
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import cref


def _inputs(seed, B, L, lens, h_q, h_k, h_v, d, integer=False):
    g = torch.Generator().manual_seed(seed)
    if integer:   # small integers: many exact ties among the scores
        q = torch.randint(-2, 3, (B, h_q, d), generator=g).to(torch.bfloat16)
        k = torch.randint(-2, 3, (B, h_k, L, d), generator=g).to(torch.bfloat16)
    else:
        q = torch.randn(B, h_q, d, generator=g).to(torch.bfloat16)
        k = torch.randn(B, h_k, L, d, generator=g).to(torch.bfloat16)
    v = torch.randn(B, h_v, L, d, generator=g).to(torch.bfloat16)
    return q, k, v, np.array(lens, dtype=np.int32)


CASES = [
    # (B, L, lens, h_q, h_k, h_v, d, N, integer keys)
    (2, 300, [300, 117], 8, 2, 4, 16, 40, False),
    (1, 64, [64], 4, 1, 2, 8, 64, False),            # N = L: dense attention
    (2, 200, [200, 3], 6, 3, 2, 8, 10, True),         # exact ties, a row with L_b < N
    (3, 96, [96, 1, 50], 4, 4, 4, 16, 7, True),       # MHA
]


@pytest.mark.parametrize("case", CASES)
def test_cpp_oracle_matches_numpy_oracle(case):
    B, L, lens, h_q, h_k, h_v, d, N, integer = case
    q, k, v, lens = _inputs(sum(lens) + N, B, L, lens, h_q, h_k, h_v, d, integer)
    out, idx, logit = cref.decode(q, k, v, lens, h_q, h_k, h_v, N)
    ref, ref_idx, ref_z = oracle.decode_attn(q.float().numpy(), k.float().numpy(), v.float().numpy(),
                                             lens, h_q, h_k, h_v, N)
    for b in range(B):
        for j in range(h_q):
            n_b = min(N, int(lens[b]))
            assert idx[b, j, :n_b].tolist() == list(ref_idx[b][j]), (b, j)
            assert (idx[b, j, n_b:] == -1).all() and np.isneginf(logit[b, j, n_b:]).all()
            np.testing.assert_allclose(logit[b, j, :n_b], ref_z[b][j], rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-12)


def test_threads_do_not_change_results():
    q, k, v, lens = _inputs(5, 4, 500, [500, 250, 499, 1], 8, 1, 2, 32, 50)
    a = cref.decode(q, k, v, lens, 8, 1, 2, 50, threads=1)
    b = cref.decode(q, k, v, lens, 8, 1, 2, 50, threads=5)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)


def test_invalid_rows_are_zero_and_padding():
    q, k, v, _ = _inputs(6, 2, 40, [40, 40], 2, 1, 1, 8)
    out, idx, logit = cref.decode(q, k, v, np.array([0, 41], dtype=np.int32), 2, 1, 1, 5)
    assert (out == 0).all() and (idx == -1).all() and np.isneginf(logit).all()
