"""Pins for the oracle with keys narrower than values (the pages' key-dimension
variant, "More Value per Key" §5.2: (h_k, d_k) = (2, 32) keys beside wider values).

Queries and keys have d_k, values and the output d_v; the score scale is
1/sqrt(d_k) (Eq. (2) scales by the key width).
"""
import math

import numpy as np
import torch

import oracle


def _inputs(seed, B, L, h_q, h_k, h_v, d_k, d_v):
    rng = np.random.default_rng(seed)
    return (rng.normal(0, 1, (B, h_q, d_k)), rng.normal(0, 1, (B, h_k, L, d_k)),
            rng.normal(0, 1, (B, h_v, L, d_v)))


def test_dense_equals_sdpa_with_different_key_and_value_widths():
    B, L, h_q, h_k, h_v, d_k, d_v = 2, 48, 8, 2, 4, 32, 64
    q, k, v = _inputs(1, B, L, h_q, h_k, h_v, d_k, d_v)
    out, _, _ = oracle.decode_attn(q, k, v, [L, L], h_q, h_k, h_v, N=L)
    assert out.shape == (B, h_q, d_v)
    g, g_v = h_q // h_k, h_q // h_v
    kt = torch.tensor(k).repeat_interleave(g, dim=1)          # [B, h_q, L, d_k]
    vt = torch.tensor(v).repeat_interleave(g_v, dim=1)        # [B, h_q, L, d_v]
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.tensor(q)[:, :, None, :], kt, vt)[:, :, 0, :]
    np.testing.assert_allclose(out, ref.numpy(), rtol=0, atol=1e-12)


def test_scale_is_the_key_width():
    # zero-padding q and k from d_k to d_v leaves q.k unchanged; only a 1/sqrt(d_k)
    # scale gives the unpadded scores
    rng = np.random.default_rng(2)
    q, k = rng.normal(0, 1, 32), rng.normal(0, 1, (20, 32))
    qp, kp = np.pad(q, (0, 32)), np.pad(k, ((0, 0), (0, 32)))
    z = oracle.scores(q, k)
    zp = oracle.scores(qp, kp)
    np.testing.assert_allclose(z, zp * math.sqrt(64) / math.sqrt(32), rtol=1e-14)
    np.testing.assert_allclose(z, k @ q / math.sqrt(32), rtol=1e-14)


def test_sparse_rows_with_narrow_keys():
    B, L, h_q, h_k, h_v, d_k, d_v, N = 1, 200, 4, 2, 4, 32, 128, 17
    q, k, v = _inputs(3, B, L, h_q, h_k, h_v, d_k, d_v)
    out, idx, _ = oracle.decode_attn(q, k, v, [L], h_q, h_k, h_v, N)
    for j in range(h_q):
        z = k[0, j // 2] @ q[0, j] / math.sqrt(d_k)
        sel = np.sort(np.argsort(-z, kind="stable")[:N])
        assert list(idx[0][j]) == sel.tolist()
        p = np.exp(z[sel] - z[sel].max())
        p /= p.sum()
        np.testing.assert_allclose(out[0, j], p @ v[0, j, sel], rtol=0, atol=1e-12)
