"""CPU oracle for group-shared selection: one set of selected positions per value
head, shared by the query heads that read that value head.

TEST INFRASTRUCTURE ONLY.  Only ``tests/`` (and the bench's CPU legs) may import
or run this module; the CUDA library and its Python binding never touch it and
share no code with it.

Written from the GQA form of SparQ's position selection as the pages describe it
(the position step sums the attention scores of the g query heads of a group and
takes the top-k of the sum), applied to SAGA's decode step ("More Value per Key",
§3.1 Eq. (7), §3.2): the heads that share a value head fetch the same N value
rows, so the V gather reads N rows per value head.  In float64:

* per query head j of value-head group G_v = {j : floor(j / g_v) = v}, the
  attention probabilities over every cached position, p_j = softmax(z_j);
* the group statistic s_i = sum over j in G_v of p_j[i];
* the shared set I_v = the N_b = min(N, L_b) positions with the largest s (ties
  to the lowest position), listed in ascending order;
* per query head j in G_v: the softmax of its own logits z_j over I_v and the
  gathered P.V over value head v.

Readings where the pages leave the step open (also in the design notes):

* the group is the query heads of one value head (the rows whose V reads can be
  shared); SparQ groups by key head, where K and V heads coincide;
* the summed scores are exact softmax probabilities (SparQ sums the
  probabilities of its approximate scores; here the scores are exact);
* SparQ's local-window term and its mean-value reallocation step are not part
  of this method and are left out.

Parity pins (``tests/test_group_oracle.py``): a group of one head is the exact
top-N; a group of identical heads is each head's top-N; per-head shift
invariance; a hand-computed two-head case; N >= L_b is dense attention per head;
nested sets in N.
"""
from __future__ import annotations

import numpy as np


def _softmax(z: np.ndarray) -> np.ndarray:
    e = np.exp(z - z.max())
    return e / e.sum()


def group_statistic(z_rows: np.ndarray) -> np.ndarray:
    """s_i = sum_j softmax(z_j)_i over the rows of z_rows [g_v, L]."""
    z_rows = np.asarray(z_rows, dtype=np.float64)
    return np.sum([_softmax(z) for z in z_rows], axis=0)


def group_select(z_rows: np.ndarray, N: int) -> np.ndarray:
    """The shared set: the min(N, L) positions with the largest group statistic,
    ties to the lowest position, ascending."""
    s = group_statistic(z_rows)
    L = s.shape[0]
    order = np.lexsort((np.arange(L), -s))          # by -s, then by position
    return np.sort(order[:min(N, L)])


def group_rows(q_rows: np.ndarray, keys: np.ndarray, values: np.ndarray, N: int):
    """One value-head group whose query heads read the same key head: q_rows
    [g_v, d], keys [L, d], values [L, d] (``group_attn`` covers groups that span
    several key heads).  Returns (out [g_v, d], the shared positions)."""
    q = np.asarray(q_rows, dtype=np.float64)
    k = np.asarray(keys, dtype=np.float64)
    z_rows = (q @ k.T) / np.sqrt(q.shape[1])
    idx = group_select(z_rows, N)
    v = np.asarray(values, dtype=np.float64)[idx]
    out = np.stack([_softmax(z[idx]) @ v for z in z_rows])
    return out, idx


def group_attn(q, k_cache, v_cache, seq_lens, h_q: int, h_k: int, h_v: int, N: int):
    """All rows: (out [B, h_q, d], shared positions per (b, value head)).  Query head j
    reads key head floor(j / (h_q / h_k)) and value head floor(j / (h_q / h_v))."""
    B, _, d = q.shape
    g, g_v = h_q // h_k, h_q // h_v
    out = np.zeros((B, h_q, d))
    sets = {}
    for b in range(B):
        L = int(seq_lens[b])
        for vh in range(h_v):
            heads = list(range(vh * g_v, (vh + 1) * g_v))
            z_rows = np.stack([
                np.asarray(k_cache[b, j // g, :L], dtype=np.float64)
                @ np.asarray(q[b, j], dtype=np.float64) / np.sqrt(d) for j in heads])
            idx = group_select(z_rows, N)
            v = np.asarray(v_cache[b, vh, :L], dtype=np.float64)[idx]
            for r, j in enumerate(heads):
                out[b, j] = _softmax(z_rows[r][idx]) @ v
            sets[(b, vh)] = idx
    return out, sets
