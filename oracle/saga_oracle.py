"""CPU oracle for the SAGA + Atop-N single-token decode step.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import or run
this module.  The product path (the CUDA library and its Python binding) never
touches it and shares no code with it.

What it computes is the plain definition, in float64, written from
"More Value per Key: Asymmetric Sparse Attention for Faster LLM Decoding"
(Elata et al.), cited below as [MVK]:

* scores      z_i = q . k_i / sqrt(d_k) over every cached position, the current
                token included (d_k the query/key width; values may be wider,
                d_v, as in the pages' key-dimension variant, [MVK] §5.2)
                                                    [MVK] §2.1 Eq. (2), §2.2 Eq. (5)
* selection   i = TopN(z): the N largest entries of the score row of each query
              head; everything else is masked       [MVK] §2.5 Eq. (6)
* softmax     over the gathered (selected) logits only; padding slots get zero
              probability                           [MVK] §3.1 Eq. (7), App. C.1
* output      O = softmax(A[i]) V[i]               [MVK] §3.1 Eq. (7)
* heads       query head j reads key head floor(j / (h_q/h_k)) and value head
              floor(j / (h_q/h_v)): contiguous query blocks share a head, as in
              GQA and the block layout of the induced permutations
                                                    [MVK] §2.3, §3.2, App. B Eq. (29)

Readings where the pages are silent (each also listed in the design notes):

* Atop-N reuses a calibrated threshold across decode steps ([MVK] §3.1, App.
  C.1).  A single stateless call recomputes the exact N-th score every call,
  i.e. Atop-N with n = 1, which is exactly the top-N definition above.
* Ties at the N-th score are broken by the lowest position index; exactly
  N_b = min(N, L_b) positions are selected.
* Selection is on the scaled scores z (softmax is monotone, so a threshold in
  probability space and one in logit space select the same set, [MVK] App. C.1).
* L_b < N selects all L_b positions (dense attention); the remaining N - L_b
  output slots are padding (index -1, logit -inf).

Parity pins: every function here is pinned in ``tests/test_oracle_pins.py``
against closed forms, a pure-Python brute force, torch's float64
``scaled_dot_product_attention`` and structural invariants (and, for keys
narrower than values, in ``tests/test_oracle_dkdv.py``).  No function is
"parity unpinned".

Inputs are numpy arrays whose values are exactly representable in bf16 (the
tests convert torch bf16 tensors with ``.float().numpy()``); every step
computes in float64.
"""
from __future__ import annotations

import numpy as np


def head_maps(h_q: int, h_k: int, h_v: int):
    """Key and value head read by each query head ([MVK] §2.3, §3.2, App. B Eq. (29)).

    Query heads are split into h_k contiguous blocks of g = h_q/h_k heads that
    share one key head, and into h_v contiguous blocks of g_v = h_q/h_v heads
    that share one value head.
    """
    if h_q % h_k or h_q % h_v:
        raise ValueError("h_k and h_v must divide h_q")
    g, g_v = h_q // h_k, h_q // h_v
    key_head = [j // g for j in range(h_q)]
    value_head = [j // g_v for j in range(h_q)]
    return key_head, value_head


def scores(q_j: np.ndarray, keys: np.ndarray) -> np.ndarray:
    """Scaled scores of one query against L cached keys ([MVK] Eq. (2), Eq. (5)).

    q_j: [d]; keys: [L, d] (positions 0..L-1, the newest token last).
    Returns z: [L] float64 with z_i = (q_j . k_i) / sqrt(d).
    """
    q64 = np.asarray(q_j, dtype=np.float64)
    k64 = np.asarray(keys, dtype=np.float64)
    d = q64.shape[-1]
    return (k64 @ q64) / np.sqrt(d)


def top_n(z: np.ndarray, N: int) -> np.ndarray:
    """Indices of the N largest scores of one row ([MVK] §2.5 Eq. (6)).

    Ties are broken by the lowest index.  Returns min(N, L) positions in
    ascending position order.
    """
    z = np.asarray(z, dtype=np.float64)
    L = z.shape[0]
    n_b = min(N, L)
    # Order by (score descending, index ascending); keep the first n_b.
    order = np.lexsort((np.arange(L), -z))
    return np.sort(order[:n_b])


def nth_score(z: np.ndarray, N: int) -> float:
    """The N_b-th largest score of a row: the exact threshold of this call."""
    z = np.asarray(z, dtype=np.float64)
    n_b = min(N, z.shape[0])
    return float(np.sort(z)[::-1][n_b - 1])


def softmax_selected(z_sel: np.ndarray) -> np.ndarray:
    """Softmax over the gathered logits only ([MVK] §3.1 Eq. (7), App. C.1)."""
    z_sel = np.asarray(z_sel, dtype=np.float64)
    m = z_sel.max()
    e = np.exp(z_sel - m)
    return e / e.sum()


def gathered_pv(p: np.ndarray, v_rows: np.ndarray) -> np.ndarray:
    """Probability-weighted sum of the gathered value rows ([MVK] Eq. (7))."""
    return np.asarray(p, dtype=np.float64) @ np.asarray(v_rows, dtype=np.float64)


def decode_row(q, k_cache, v_cache, seq_lens, b: int, j: int,
               h_q: int, h_k: int, h_v: int, N: int):
    """One (batch row, query head) of the decode step.

    q: [B, h_q, d_k]; k_cache: [B, h_k, L_max, d_k]; v_cache: [B, h_v, L_max, d_v];
    seq_lens: [B] (positions 0..L_b-1 are valid, the current token at L_b-1).
    Returns (out [d_v] float64, idx [N_b] ascending, z_sel [N_b], z [L_b]).
    """
    key_head, value_head = head_maps(h_q, h_k, h_v)
    L_b = int(seq_lens[b])
    z = scores(q[b, j], k_cache[b, key_head[j], :L_b])
    idx = top_n(z, N)
    z_sel = z[idx]
    p = softmax_selected(z_sel)
    out = gathered_pv(p, v_cache[b, value_head[j], idx])
    return out, idx, z_sel, z


def decode_attn(q, k_cache, v_cache, seq_lens, h_q: int, h_k: int, h_v: int, N: int):
    """The whole decode step for every (b, j).

    Returns (out [B, h_q, d_v] float64, idx list-of-lists, z_sel list-of-lists).
    """
    B = q.shape[0]
    d_v = v_cache.shape[-1]          # the output has the value width (d_v may differ from d_k)
    out = np.zeros((B, h_q, d_v), dtype=np.float64)
    idx_all, zsel_all = [], []
    for b in range(B):
        idx_b, zsel_b = [], []
        for j in range(h_q):
            o, idx, z_sel, _ = decode_row(q, k_cache, v_cache, seq_lens, b, j,
                                          h_q, h_k, h_v, N)
            out[b, j] = o
            idx_b.append(idx)
            zsel_b.append(z_sel)
        idx_all.append(idx_b)
        zsel_all.append(zsel_b)
    return out, idx_all, zsel_all


def combine(z_sel: np.ndarray, v_rows: np.ndarray) -> np.ndarray:
    """Softmax over given selected logits, then the gathered P.V (Eq. (7))."""
    return gathered_pv(softmax_selected(z_sel), v_rows)
