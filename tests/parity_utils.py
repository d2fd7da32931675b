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


# --------------------------------------------------------------------------- stateful Atop-N

TAIL = 32          # the oracle's tail for m_hat (the threshold does not depend on it)
EPS32 = 2.0 ** -24


def lse_error(q_row, k_rows, z_ref, extra=0.0):
    """The row's float64 log-sum-exp and a bound on the error of the GPU's fp32 one.

    The GPU sums exp(z - m_ref) of its fp32 scores, m_ref one of the row's
    sampled scores: d(LSE)/dz_i = p_i, so the scores' errors move it by at most
    sum_i p_i * bound_i; the fast exp is within 2 + 1.17 |x| ulp for an
    argument x (|x| <= the row's score range), the sums add at most 32 ulp
    relative (reduction depth < 32), and the fp32 values of magnitude |LSE| and
    |extra| combined with it a few ulp each."""
    m = z_ref.max()
    e = np.exp(z_ref - m)
    lse = m + math.log(e.sum())
    p = e / e.sum()
    spread = float(z_ref.max() - z_ref.min())
    err = (float(p @ score_bound(q_row, k_rows)) + (34 + 1.17 * spread) * EPS32 +
           8 * EPS32 * (abs(lse) + abs(extra)))
    return lse, err


def check_log_tau(gpu_log_tau, q_row, k_rows, N, what=""):
    """Calibration: log tau = z_(N_b) - logsumexp(z) of the row, against the oracle in
    float64; tolerance: the N-th score within BAND plus its fp32 bound, and the
    log-sum-exp's error bound."""
    z_ref = oracle.scores(q_row, k_rows)
    ref = math.log(oracle.calibrate_tau(z_ref, N))
    n_b = min(N, z_ref.shape[0])
    k = np.asarray(k_rows)
    near = np.flatnonzero(np.abs(z_ref - np.sort(z_ref)[::-1][n_b - 1]) <= BAND)
    _, err = lse_error(q_row, k_rows, z_ref, ref)
    tol = BAND + float(score_bound(q_row, k[near]).max()) + err
    assert abs(float(gpu_log_tau) - ref) <= tol, \
        f"{what}: log tau {float(gpu_log_tau)} vs oracle {ref} (tolerance {tol})"


def check_step_row(gpu_idx, gpu_logit, gpu_out, q_row, k_rows, v_rows, log_tau, N, what=""):
    """A step of stateful Atop-N against the oracle replaying the same tau.

    The oracle threshold is t = m_hat + log(tau * s_hat) in float64 with
    tau = exp(log_tau) (the GPU's state).  The GPU keeps the positions with
    z >= t in ascending order, at most 2N of them; a position may go either way
    when its oracle score lies within BAND + its fp32 score bound + the bound
    on the GPU threshold's error (its log-sum-exp, see lse_error) of t; the
    output is compared with the
    oracle's softmax and P.V over the GPU's kept set, and with the oracle's own
    step output when the two sets agree.  Returns the number of kept
    positions."""
    z_ref = oracle.scores(q_row, k_rows)
    L = z_ref.shape[0]
    cap = 2 * N
    tau = math.exp(float(log_tau))
    t = oracle.step_threshold(z_ref, tau, TAIL)
    gpu_idx = np.asarray(gpu_idx)
    gpu_logit = np.asarray(gpu_logit, dtype=np.float64)
    n = int((gpu_idx >= 0).sum())
    sel = gpu_idx[:n]
    assert (gpu_idx[n:] == -1).all(), f"{what}: padding"
    assert np.isneginf(gpu_logit[n:]).all(), f"{what}: logit padding"
    assert n <= cap
    if n:
        assert (np.diff(sel) > 0).all(), f"{what}: not strictly ascending"
        assert sel.min() >= 0 and sel.max() < L, f"{what}: index out of range"
    gpu_set = np.zeros(L, dtype=bool)
    gpu_set[sel] = True
    _, t_err = lse_error(q_row, k_rows, z_ref, abs(float(log_tau)) + abs(t))
    band = BAND + t_err + score_bound(q_row, k_rows)
    sure = z_ref > t + band
    maybe = np.abs(z_ref - t) <= band
    assert not (gpu_set & ~(sure | maybe)).any(), \
        f"{what}: kept below the threshold {np.flatnonzero(gpu_set & ~(sure | maybe))[:5]}"
    if (sure | maybe).sum() <= cap:
        assert not (sure & ~gpu_set).any(), f"{what}: missed {np.flatnonzero(sure & ~gpu_set)[:5]}"
    else:
        # capacity binds: the first 2N passing positions, so every sure position
        # before the last kept one is kept
        assert n == cap, f"{what}: {n} kept, capacity {cap} binds"
        early = sure & (np.arange(L) < sel[-1])
        assert not (early & ~gpu_set).any(), f"{what}: skipped {np.flatnonzero(early & ~gpu_set)[:5]}"
    if n:
        bound = score_bound(q_row, np.asarray(k_rows)[sel])
        err = np.abs(gpu_logit[:n] - z_ref[sel])
        assert (err <= bound).all(), f"{what}: kept logits off by {err.max()}"
        assert_out_close(gpu_out, oracle.combine(z_ref[sel], np.asarray(v_rows)[sel]),
                         f"{what} out vs oracle on the GPU's set")
    else:
        assert_out_close(gpu_out, np.zeros_like(np.asarray(gpu_out, dtype=np.float64)),
                         f"{what} empty selection")
    # the oracle's own step output, where its selection is the GPU's (with tau
    # calibrated on the same scores, t sits on a score, and one entry more or
    # less -- inside the band -- moves the output by its whole weight)
    out_ref, idx_ref, _ = oracle.step_row(np.asarray(q_row), np.asarray(k_rows),
                                          np.asarray(v_rows), tau, TAIL, cap)
    if np.array_equal(idx_ref, sel):
        assert_out_close(gpu_out, out_ref, f"{what} out vs oracle step")
    return n
