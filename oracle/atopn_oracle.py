"""CPU oracle for stateful Atop-N: the calibrated probability threshold reused
across decode steps.

TEST INFRASTRUCTURE ONLY.  Only ``tests/`` (and the bench's CPU legs) may import
or run this module; the CUDA library and its Python binding never touch it and
share no code with it.

Written from "More Value per Key: Asymmetric Sparse Attention for Faster LLM
Decoding" (Elata et al.), cited as [MVK], §3.1 and App. C.1 (Atop-N attention),
in float64:

* calibration (the first decode step after prefill, then every n steps): the
  exact probabilities p = softmax(z) over every cached position, and per head
  the probability of the N-th largest entry, tau = p_(N)          [MVK] App. C.1
* a later step, with tau fixed: the max logit is approximated by m_hat, the
  largest logit over a small tail of positions; s_hat = sum_i exp(z_i - m_hat)
  over every position (one reduction pass); the logit threshold is
  t = m_hat + log(tau * s_hat), and every entry with z_i >= t is collected
  into a buffer of capacity 2N; the collected logits get a softmax and weight
  the gathered value rows                                          [MVK] App. C.1

Readings where the pages leave the step open (also in the design notes):

* the tail is the last ``tail`` positions of the row (the most recent tokens);
* when more than ``cap`` = 2N entries pass the threshold, the ``cap`` lowest
  positions are kept (the pages drop the excess in whatever order an atomic
  counter gives; a fixed rule makes the result reproducible);
* the collected positions are listed in ascending order; unused slots are
  padding (index -1, logit -inf);
* calibration with N >= L_b gives tau = the smallest probability (every
  position passes);
* a step where no entry reaches the threshold (tau above the row's largest
  probability) selects nothing and gives a zero output (a softmax over an
  all-padding buffer has no value; the zero row is the convention of the
  library's combine stage for a row with no valid entry).

Parity pins (``tests/test_atopn_oracle.py``): a step with tau calibrated on the
same scores selects exactly the top-N for any tail (t reduces to the N-th
score: the tail max cancels), hand-computed thresholds, shift invariance, the
capacity rule, and agreement with the exact top-N oracle.
"""
from __future__ import annotations

import numpy as np


def calibrate_tau(z: np.ndarray, N: int) -> float:
    """tau = softmax(z) at the N_b-th largest entry (N_b = min(N, len(z))) ([MVK] App. C.1)."""
    z = np.asarray(z, dtype=np.float64)
    m = z.max()
    e = np.exp(z - m)
    n_b = min(N, z.size)
    zn = np.sort(z)[::-1][n_b - 1]
    return float(np.exp(zn - m) / e.sum())


def tail_max(z: np.ndarray, tail: int) -> float:
    """m_hat: the largest logit over the last ``tail`` positions ([MVK] App. C.1)."""
    z = np.asarray(z, dtype=np.float64)
    return float(z[max(0, z.size - tail):].max())


def step_threshold(z: np.ndarray, tau: float, tail: int) -> float:
    """t = m_hat + log(tau * s_hat), s_hat = sum_i exp(z_i - m_hat) over every position."""
    z = np.asarray(z, dtype=np.float64)
    m_hat = tail_max(z, tail)
    s_hat = np.exp(z - m_hat).sum()
    return float(m_hat + np.log(tau * s_hat))


def step_select(z: np.ndarray, tau: float, tail: int, cap: int) -> np.ndarray:
    """Positions with z >= t, ascending, at most ``cap`` (the lowest ones kept)."""
    z = np.asarray(z, dtype=np.float64)
    t = step_threshold(z, tau, tail)
    return np.flatnonzero(z >= t)[:cap]


def step_row(q_j, keys, values, tau: float, tail: int, cap: int):
    """One (b, j) row of a step: (out [d], selected positions, their logits)."""
    d = q_j.shape[0]
    z = keys.astype(np.float64) @ q_j.astype(np.float64) / np.sqrt(d)
    idx = step_select(z, tau, tail, cap)
    z_sel = z[idx]
    if idx.size == 0:
        return np.zeros(values.shape[1]), idx, z_sel
    p = np.exp(z_sel - z_sel.max())
    p /= p.sum()
    out = p @ values[idx].astype(np.float64)
    return out, idx, z_sel


def calibrate_row(q_j, keys, N: int) -> float:
    d = q_j.shape[0]
    z = keys.astype(np.float64) @ q_j.astype(np.float64) / np.sqrt(d)
    return calibrate_tau(z, N)


def step_attn(q, k_cache, v_cache, seq_lens, h_q: int, h_k: int, h_v: int, tau,
              tail: int, cap: int):
    """All rows of a step: (out [B, h_q, d], index lists, logit lists); tau is [B, h_q]."""
    B, _, d = q.shape
    g, g_v = h_q // h_k, h_q // h_v
    out = np.zeros((B, h_q, d))
    idx_all, z_all = [], []
    for b in range(B):
        L = int(seq_lens[b])
        for j in range(h_q):
            o, idx, zs = step_row(q[b, j], k_cache[b, j // g, :L], v_cache[b, j // g_v, :L],
                                  float(tau[b][j]), tail, cap)
            out[b, j] = o
            idx_all.append(idx)
            z_all.append(zs)
    return out, idx_all, z_all
