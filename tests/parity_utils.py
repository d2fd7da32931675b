"""Shared checks for the GPU parity tests (the oracle side is ``oracle/``).

Matching rules for one (b, j) row:
* scores: |z_gpu - z_oracle| within the worst-case fp32 accumulation bound of
  a d-term dot product, 4 * d * 2^-24 * sum_t |q_t k_t| / sqrt(d) (4x slack
  for a truncating adder);
* selection: the GPU keeps exactly N_b = min(N, L_b) positions, ascending,
  padded with -1 / -inf; every position whose oracle (float64) score is more
  than BAND = 1e-5 above the oracle's N_b-th score is kept and every position
  more than BAND below it is not, so the GPU and oracle sets can differ only
  inside the band;
* output: per element |err| <= 2e-3, or |err| <= 1e-2 * |ref|, against the
  oracle's float64 output, both on the oracle's own selection and on the
  GPU's selection.
"""
import math

import numpy as np

import oracle

BAND = 1e-5
ATOL = 2e-3
RTOL = 1e-2


def to_np(t):
    return t.detach().float().cpu().numpy()


def assert_out_close(got, ref, what=""):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    err = np.abs(got - ref)
    ok = (err <= ATOL) | (err <= RTOL * np.abs(ref))
    if not ok.all():
        i = int(np.argmax(np.where(ok, 0, err)))
        raise AssertionError(f"{what}: {int((~ok).sum())} elements out of tolerance; worst at "
                             f"{np.unravel_index(i, err.shape)} got {got.flat[i]} ref {ref.flat[i]}")


def score_bound(q_row, k_rows):
    """Per-position worst-case bound on the fp32 score error."""
    q = np.asarray(q_row, dtype=np.float64)
    k = np.asarray(k_rows, dtype=np.float64)
    d = q.shape[0]
    return 4.0 * d * 2.0 ** -24 * (np.abs(k) @ np.abs(q)) / math.sqrt(d) + 1e-7


def check_row(gpu_idx, gpu_logit, gpu_out, q_row, k_rows, v_rows, N, what=""):
    """One (b, j) row against the oracle.  q_row [d]; k_rows / v_rows: the row's
    key / value head over its valid positions [L_b, d].  Returns the number of
    positions where the GPU and oracle selections differ (all inside the band)."""
    z_ref = oracle.scores(q_row, k_rows)
    L = z_ref.shape[0]
    n_b = min(N, L)
    gpu_idx = np.asarray(gpu_idx)
    gpu_logit = np.asarray(gpu_logit, dtype=np.float64)
    sel = gpu_idx[:n_b]
    assert (gpu_idx[n_b:] == -1).all(), f"{what}: padding"
    assert np.isneginf(gpu_logit[n_b:]).all(), f"{what}: logit padding"
    assert (np.diff(sel) > 0).all(), f"{what}: not strictly ascending"
    assert sel.min() >= 0 and sel.max() < L, f"{what}: index out of range"
    t = oracle.nth_score(z_ref, N)
    gpu_set = np.zeros(L, dtype=bool)
    gpu_set[sel] = True
    must = z_ref > t + BAND
    must_not = z_ref < t - BAND
    assert not (must & ~gpu_set).any(), f"{what}: missed {np.flatnonzero(must & ~gpu_set)[:5]}"
    assert not (must_not & gpu_set).any(), f"{what}: extra {np.flatnonzero(must_not & gpu_set)[:5]}"
    ref_idx = oracle.top_n(z_ref, N)
    ref_set = np.zeros(L, dtype=bool)
    ref_set[ref_idx] = True
    diff = np.flatnonzero(ref_set != gpu_set)
    assert (np.abs(z_ref[diff] - t) <= BAND).all(), f"{what}: set differs outside the band"
    bound = score_bound(q_row, np.asarray(k_rows)[sel])
    err = np.abs(gpu_logit[:n_b] - z_ref[sel])
    assert (err <= bound).all(), f"{what}: selected logits off by {err.max()} (bound {bound.min()})"
    out_ref = oracle.combine(z_ref[ref_idx], np.asarray(v_rows)[ref_idx])
    assert_out_close(gpu_out, out_ref, f"{what} out vs oracle")
    out_on_gpu_set = oracle.combine(z_ref[sel], np.asarray(v_rows)[sel])
    assert_out_close(gpu_out, out_on_gpu_set, f"{what} out vs oracle on GPU set")
    return len(diff)
