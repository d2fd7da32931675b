"""GPU parity of stateful Atop-N: the calibration call and later steps (through
the C ABI) against the oracle replaying the same tau ("More Value per Key",
App. C.1).

The state is the GPU's own log tau: the calibration is checked against the
oracle's log p_(N), and each step against the oracle's threshold
m_hat + log(tau * s_hat) for tau = exp(log tau), under the rules of
``parity_utils.check_step_row``.
"""
import numpy as np
import pytest
import torch

from parity_utils import (check_log_tau, check_row, check_step_row, to_np)
from sparse_asymmetric_gqa_b200 import SagaDecoder, SagaError, workload
from sparse_asymmetric_gqa_b200 import _lib

pytestmark = pytest.mark.gpu


def _dev(inp):
    return (inp.q.cuda(), inp.k_cache.cuda(), inp.v_cache.cuda(), inp.seq_lens.cuda())


def calibrate(dec, q, k, v, lens, N):
    B, h_q = q.shape[0], q.shape[1]
    idx = torch.empty(B, h_q, N, dtype=torch.int32, device="cuda")
    logit = torch.empty(B, h_q, N, dtype=torch.float32, device="cuda")
    out, log_tau = dec.atopn_calibrate(q, k, v, lens, N, sel_idx=idx, sel_logit=logit)
    return out, idx, logit, log_tau, dec.status()


def step(dec, q, k, v, lens, N, log_tau):
    B, h_q = q.shape[0], q.shape[1]
    idx = torch.empty(B, h_q, 2 * N, dtype=torch.int32, device="cuda")
    logit = torch.empty(B, h_q, 2 * N, dtype=torch.float32, device="cuda")
    out = dec.atopn_step(q, k, v, lens, N, log_tau, sel_idx=idx, sel_logit=logit)
    return out, idx, logit, dec.status()


def rows_of(inp, h_q, h_k, h_v, rows):
    """(b, j, q_row, k_rows, v_rows) over each row's valid positions."""
    q = to_np(inp.q)
    g, g_v = h_q // h_k, h_q // h_v
    lens = inp.seq_lens.tolist()
    for b, j in rows:
        L = lens[b]
        yield b, j, q[b, j], to_np(inp.k_cache[b, j // g, :L]), to_np(inp.v_cache[b, j // g_v, :L])


def check_calibration(inp, h_q, h_k, h_v, N, out, idx, logit, log_tau, rows):
    o, i, lg, lt = to_np(out), idx.cpu().numpy(), logit.cpu().numpy(), log_tau.cpu().numpy()
    for b, j, qr, kr, vr in rows_of(inp, h_q, h_k, h_v, rows):
        check_row(i[b, j], lg[b, j], o[b, j], qr, kr, vr, N, what=f"calibrate ({b},{j})")
        check_log_tau(lt[b, j], qr, kr, N, what=f"calibrate ({b},{j})")


def check_steps(inp, h_q, h_k, h_v, N, out, idx, logit, log_tau, rows):
    o, i, lg, lt = to_np(out), idx.cpu().numpy(), logit.cpu().numpy(), log_tau.cpu().numpy()
    return [check_step_row(i[b, j], lg[b, j], o[b, j], qr, kr, vr, lt[b, j], N,
                           what=f"step ({b},{j})")
            for b, j, qr, kr, vr in rows_of(inp, h_q, h_k, h_v, rows)]


def make_raw(seed, B, L_max, lens, h_q, h_k, h_v, d):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, h_q, d, generator=g).to(torch.bfloat16)
    k = torch.randn(B, h_k, L_max, d, generator=g).to(torch.bfloat16)
    v = torch.randn(B, h_v, L_max, d, generator=g).to(torch.bfloat16)
    return workload.DecodeInputs(q, k, v, torch.tensor(lens, dtype=torch.int32))


# --------------------------------------------------------------------------- calibration

def test_calibrate_tiny_planted_all_rows():
    spec = workload.TINY
    inp = workload.make_inputs(spec)
    dec = SagaDecoder(spec.batch, spec.seq_len, spec.h_q, spec.h_k, spec.h_v, spec.head_dim, spec.N)
    out, idx, logit, log_tau, st = calibrate(dec, *_dev(inp), spec.N)
    assert st & 0xFF == 0
    rows = [(0, j) for j in range(spec.h_q)]
    check_calibration(inp, spec.h_q, spec.h_k, spec.h_v, spec.N, out, idx, logit, log_tau, rows)
    # the calibration's output is the exact decode step's
    ref = dec.attn(*_dev(inp), spec.N)
    assert torch.equal(out, ref)


@pytest.mark.parametrize("case", [
    # (B, L_max, lens, h_q, h_k, h_v, d, N): long rows use the score pass's chunk
    # sums, rows of at most 8192 positions their complete candidate lists
    (2, 20000, [20000, 12345], 12, 1, 2, 128, 256),
    (3, 9000, [9000, 8192, 700], 8, 2, 4, 64, 64),
    (2, 4096, [4096, 37], 16, 1, 8, 64, 128),          # a row with L_b < N: tau = min probability
], ids=["long", "mixed", "short"])
def test_calibrate_then_step_same_inputs_selects_the_top_n(case):
    # With tau calibrated on the very same scores the step's threshold is the
    # N-th score (the reference cancels): the step selects the top N_b, up to
    # scores within the band of the threshold.
    B, L_max, lens, h_q, h_k, h_v, d, N = case
    inp = make_raw(21, B, L_max, lens, h_q, h_k, h_v, d)
    dec = SagaDecoder(B, L_max, h_q, h_k, h_v, d, N)
    dev = _dev(inp)
    out, idx, logit, log_tau, st = calibrate(dec, *dev, N)
    assert st & 0xFF == 0
    rows = [(b, j) for b in range(B) for j in range(h_q)]
    check_calibration(inp, h_q, h_k, h_v, N, out, idx, logit, log_tau, rows)
    s_out, s_idx, s_logit, st = step(dec, *dev, N, log_tau)
    assert st & 0xFF == 0
    kept = check_steps(inp, h_q, h_k, h_v, N, s_out, s_idx, s_logit, log_tau, rows)
    for (b, j), n in zip(rows, kept):
        n_b = min(N, lens[b])
        assert abs(n - n_b) <= 2, f"row ({b},{j}) kept {n} of {n_b}"


def test_step_with_a_wider_selection_than_calibrated():
    # tau of the N-th score, a step with 4N: the threshold is the calibrated
    # N-th score, well inside the candidates the step's bound (for 8N) keeps, so
    # the fast path runs with a threshold that is not the step's own N-th score.
    B, L, h_q, h_k, h_v, d, N = 2, 30000, 12, 1, 2, 128, 128
    inp = make_raw(38, B, L, [L, 26000], h_q, h_k, h_v, d)
    dec = SagaDecoder(B, L, h_q, h_k, h_v, d, 4 * N)
    dev = _dev(inp)
    _, log_tau = dec.atopn_calibrate(*dev, N)
    out, idx, logit, st = step(dec, *dev, 4 * N, log_tau)
    assert st == 0
    rows = [(b, j) for b in range(B) for j in range(h_q)]
    kept = check_steps(inp, h_q, h_k, h_v, 4 * N, out, idx, logit, log_tau, rows)
    assert all(abs(n - N) <= 2 for n in kept)


@pytest.mark.parametrize("drift", [0.05, 0.3])
def test_steps_with_drifting_queries_and_growing_rows(drift):
    # Decoding: tau from the first step, then three steps with new queries (the
    # old ones plus noise) over rows one position longer each time; planted
    # query-aligned keys as in the Qwen-shaped workload.  Rows whose threshold
    # moved below the sampled bound take the exact fallback; all must match.
    spec = workload.scaled(workload.QWEN_32K, batch=2, seq_len=24576, N=512, layers=1, seed=77)
    inp = workload.make_inputs(spec)
    B, H, d, N = spec.batch, spec.h_q, spec.head_dim, spec.N
    L0 = spec.seq_len - 8
    inp.seq_lens[:] = L0
    dec = SagaDecoder(B, spec.seq_len, H, spec.h_k, spec.h_v, d, N)
    q, k, v, lens = _dev(inp)
    out, idx, logit, log_tau, st = calibrate(dec, q, k, v, lens, N)
    assert st & 0xFF == 0
    g = torch.Generator().manual_seed(5)
    robust = 0
    for s in range(1, 4):
        inp.q = (inp.q.float() + drift * torch.randn(inp.q.shape, generator=g)).to(torch.bfloat16)
        inp.seq_lens[:] = L0 + s
        q, lens = inp.q.cuda(), inp.seq_lens.cuda()
        s_out, s_idx, s_logit, st = step(dec, q, k, v, lens, N, log_tau)
        assert st & 0xFF == 0
        robust += bool(st & _lib.SAGA_STATUS_INFO_ROBUST_PATH)
        rows = [(b, j) for b in range(B) for j in range(H)]
        kept = check_steps(inp, H, spec.h_k, spec.h_v, N, s_out, s_idx, s_logit, log_tau, rows)
        assert max(kept) > 0
    print(f"drift {drift}: {robust} of 3 steps had a row on the exact fallback")


def test_step_capacity_keeps_the_lowest_positions():
    # log tau = -200: every position passes; the step keeps the first 2N.  The
    # threshold lies far below the sampled bound, so the row is scored again.
    B, L, h_q, h_k, h_v, d, N = 1, 16384, 4, 1, 2, 64, 64
    inp = make_raw(31, B, L, [L], h_q, h_k, h_v, d)
    dec = SagaDecoder(B, L, h_q, h_k, h_v, d, N)
    log_tau = torch.full((B, h_q), -200.0, device="cuda")
    out, idx, logit, st = step(dec, *_dev(inp), N, log_tau)
    assert st & 0xFF == 0 and st & _lib.SAGA_STATUS_INFO_ROBUST_PATH
    assert (idx.cpu() == torch.arange(2 * N, dtype=torch.int32)).all()
    check_steps(inp, h_q, h_k, h_v, N, out, idx, logit, log_tau, [(0, j) for j in range(h_q)])


def test_step_nan_log_tau_takes_every_position():
    B, L, h_q, h_k, h_v, d, N = 1, 3000, 4, 1, 2, 128, 100
    inp = make_raw(32, B, L, [L], h_q, h_k, h_v, d)
    dec = SagaDecoder(B, L, h_q, h_k, h_v, d, N)
    log_tau = torch.full((B, h_q), float("nan"), device="cuda")
    out, idx, logit, st = step(dec, *_dev(inp), N, log_tau)
    assert st & 0xFF == 0
    assert (idx.cpu() == torch.arange(2 * N, dtype=torch.int32)).all()


def test_step_threshold_above_every_probability_selects_nothing():
    # tau > 1 puts t above logsumexp(z) >= max z: nothing passes, zero output
    B, L, h_q, h_k, h_v, d, N = 2, 10000, 4, 2, 4, 64, 32
    inp = make_raw(33, B, L, [L, 5000], h_q, h_k, h_v, d)
    dec = SagaDecoder(B, L, h_q, h_k, h_v, d, N)
    log_tau = torch.full((B, h_q), 0.5, device="cuda")
    out, idx, logit, st = step(dec, *_dev(inp), N, log_tau)
    assert st & 0xFF == 0
    assert (idx.cpu() == -1).all() and torch.isneginf(logit.cpu()).all()
    assert (out.cpu().float() == 0).all()


def test_exp_sums_out_of_range_fall_back_exactly():
    # One key far above every sampled score (z - m_ref > 64): the chunk sums
    # overflow by design, the row is scored again and its log-sum-exp taken
    # exactly; calibration and step still match the oracle.
    B, L, h_q, h_k, h_v, d, N = 1, 16384, 2, 1, 2, 128, 128
    inp = make_raw(34, B, L, [L], h_q, h_k, h_v, d)
    inp.q[0, 1] = inp.q[0, 0]
    p = 5000 + 17                                      # not a sampled position (L / 32 = 512)
    lpb = L // 32
    sampled = {32 * ((blk * lpb) // 32) + i for blk in range(32) for i in range(32)}
    assert p not in sampled
    inp.k_cache[0, 0, p] = (8.0 * inp.q[0, 0].float()).to(torch.bfloat16)   # z ~ 8 sqrt(d) ~ 90
    dec = SagaDecoder(B, L, h_q, h_k, h_v, d, N)
    dev = _dev(inp)
    out, idx, logit, log_tau, st = calibrate(dec, *dev, N)
    assert st & 0xFF == 0 and st & _lib.SAGA_STATUS_INFO_ROBUST_PATH
    rows = [(0, 0), (0, 1)]
    check_calibration(inp, h_q, h_k, h_v, N, out, idx, logit, log_tau, rows)
    s_out, s_idx, s_logit, st = step(dec, *dev, N, log_tau)
    assert st & 0xFF == 0
    check_steps(inp, h_q, h_k, h_v, N, s_out, s_idx, s_logit, log_tau, rows)


def test_bad_seq_lens_calibrate_and_step():
    B, L, h_q, h_k, h_v, d, N = 3, 1024, 4, 1, 2, 64, 64
    inp = make_raw(35, B, L, [0, 700, L + 5], h_q, h_k, h_v, d)
    dec = SagaDecoder(B, L, h_q, h_k, h_v, d, N)
    dev = _dev(inp)
    out, idx, logit, log_tau, st = calibrate(dec, *dev, N)
    assert st & _lib.SAGA_STATUS_BAD_SEQ_LEN
    lt = log_tau.cpu()
    assert torch.isneginf(lt[0]).all() and torch.isneginf(lt[2]).all()
    check_calibration(inp, h_q, h_k, h_v, N, out, idx, logit, log_tau, [(1, j) for j in range(h_q)])
    s_out, s_idx, s_logit, st = step(dec, *dev, N, log_tau)
    assert st & _lib.SAGA_STATUS_BAD_SEQ_LEN
    for b in (0, 2):
        assert (s_out[b].float() == 0).all() and (s_idx[b] == -1).all()
    check_steps(inp, h_q, h_k, h_v, N, s_out, s_idx, s_logit, log_tau, [(1, j) for j in range(h_q)])


def test_step_is_deterministic_and_launches_four_kernels():
    B, L, h_q, h_k, h_v, d, N = 2, 20000, 12, 1, 2, 128, 256
    inp = make_raw(36, B, L, [L, 15000], h_q, h_k, h_v, d)
    dec = SagaDecoder(B, L, h_q, h_k, h_v, d, N)
    dev = _dev(inp)
    _, log_tau = dec.atopn_calibrate(*dev, N)
    n0 = dec.launch_count()
    a = dec.atopn_step(*dev, N, log_tau)
    assert dec.launch_count() - n0 == 4          # sample, bound, score, top-N with P.V
    b = dec.atopn_step(*dev, N, log_tau)
    assert dec.status() & 0xFF == 0
    assert torch.equal(a, b)


def test_argument_checks():
    B, L, h_q, h_k, h_v, d = 1, 4096, 4, 1, 2, 64
    inp = make_raw(37, B, L, [L], h_q, h_k, h_v, d)
    dec = SagaDecoder(B, L, h_q, h_k, h_v, d, 4096)
    dev = _dev(inp)
    log_tau = torch.zeros(B, h_q, device="cuda")
    with pytest.raises(SagaError) as e:
        dec.atopn_step(*dev, 4096, log_tau)            # 2N beyond the candidate path
    assert e.value.code == _lib.SAGA_ERR_UNSUPPORTED
    rc = dec.lib.saga_atopn_step(dec._h, dev[0].data_ptr(), dev[1].data_ptr(), dev[2].data_ptr(),
                                 dev[3].data_ptr(), h_q, h_k, h_v, d, 16, None,
                                 torch.empty(B, h_q, d, dtype=torch.bfloat16, device="cuda").data_ptr(),
                                 None, None)
    assert rc == _lib.SAGA_ERR_INVALID_ARG             # no state


# --------------------------------------------------------------------------- full size

def test_full_size_qwen_calibrate_and_step_sampled_rows():
    spec = workload.QWEN_32K
    inp = workload.make_inputs(spec)
    dec = SagaDecoder(spec.batch, spec.seq_len, spec.h_q, spec.h_k, spec.h_v, spec.head_dim, spec.N)
    dev = _dev(inp)
    out, idx, logit, log_tau, st = calibrate(dec, *dev, spec.N)
    assert st & 0xFF == 0
    rng = np.random.default_rng(3)
    rows = sorted({(int(rng.integers(spec.batch)), int(rng.integers(spec.h_q))) for _ in range(6)}
                  | {(0, 0), (spec.batch - 1, spec.h_q - 1)})
    check_calibration(inp, spec.h_q, spec.h_k, spec.h_v, spec.N, out, idx, logit, log_tau, rows)
    s_out, s_idx, s_logit, st = step(dec, *dev, spec.N, log_tau)
    assert st == 0                                      # no row needed the fallback
    kept = check_steps(inp, spec.h_q, spec.h_k, spec.h_v, spec.N, s_out, s_idx, s_logit, log_tau, rows)
    assert all(abs(n - spec.N) <= 2 for n in kept)
    assert torch.isfinite(s_out.float()).all()
    assert torch.isfinite(log_tau).all()


@pytest.mark.parametrize("shift", [0.0, -1.5, 2.0])
def test_step_keeps_an_upper_set_of_its_own_scores(shift):
    # The step's compare, bit-exact against the GPU's own fp32 scores (the stage-wise
    # score pass computes them with the same arithmetic): its logits are those scores
    # exactly, and the kept positions are the first 2N in position order of
    # {i : z_i >= t} for one threshold t, so no position before the last kept one
    # with a score at or above the smallest kept score is left out.  log tau is
    # shifted (0: as calibrated; < 0 keeps more, hitting the 2N capacity; > 0 keeps
    # fewer), and rows below and above the candidate cap are both covered.  A long
    # row whose threshold falls below its sampled bound is scored again on CUDA
    # cores (INFO_ROBUST_PATH), with another summation order: the long rows of
    # such a call are not compared bit for bit.
    B, L, h_q, h_k, h_v, d, N = 2, 20000, 4, 1, 2, 128, 256
    lens = [L, 5000]
    inp = make_raw(71, B, L, lens, h_q, h_k, h_v, d)
    dec = SagaDecoder(B, L, h_q, h_k, h_v, d, N)
    dev = _dev(inp)
    _, _, _, log_tau, st = calibrate(dec, *dev, N)
    assert st & 0xFF == 0
    _, idx, logit, st = step(dec, *dev, N, log_tau + shift)
    assert st & 0xFF == 0
    rescored = bool(st & _lib.SAGA_STATUS_INFO_ROBUST_PATH)
    z = dec.score(dev[0], dev[1], dev[3]).cpu().numpy()
    idx, logit = idx.cpu().numpy(), logit.cpu().numpy()
    checked = 0
    for b in range(B):
        if rescored and lens[b] > 8192:
            continue
        for j in range(h_q):
            what = f"shift {shift} ({b},{j})"
            checked += 1
            kept = idx[b, j][idx[b, j] >= 0]
            n = kept.size
            assert (idx[b, j, n:] == -1).all(), f"{what}: padding"
            zr = z[b, j, :lens[b]]
            np.testing.assert_array_equal(logit[b, j, :n], zr[kept], err_msg=what)
            if n == 0:
                continue
            assert (np.diff(kept) > 0).all(), f"{what}: not ascending"
            t_min = zr[kept].min()
            left_out = np.ones(kept[-1] + 1, dtype=bool)
            left_out[kept] = False
            assert (zr[:kept[-1] + 1][left_out] < t_min).all(), f"{what}: a score >= the kept ones left out"
            if n < 2 * N:                               # below capacity: nothing after the last one either
                assert (zr[kept[-1] + 1:] < t_min).all(), f"{what}: a later score >= the kept ones left out"
    assert checked >= h_q
