"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle.

Every case draws seeded inputs on the CPU, runs the library on cuda:0 and
compares element by element with ``oracle/`` under the rules in
``parity_utils``.  Full-size workloads are checked on sampled rows (the oracle
computes them one by one) plus properties that hold for every row.
"""
import numpy as np
import pytest
import torch

import oracle
from parity_utils import assert_out_close, check_row, score_bound, to_np
from sparse_asymmetric_gqa_b200 import SagaDecoder, workload
from sparse_asymmetric_gqa_b200 import _lib

pytestmark = pytest.mark.gpu


def _dev(inp):
    return (inp.q.cuda(), inp.k_cache.cuda(), inp.v_cache.cuda(), inp.seq_lens.cuda())


def run_decode(dec, q, k, v, lens, N):
    B, h_q = q.shape[0], q.shape[1]
    idx = torch.empty(B, h_q, N, dtype=torch.int32, device="cuda")
    logit = torch.empty(B, h_q, N, dtype=torch.float32, device="cuda")
    out = dec.attn(q, k, v, lens, N, sel_idx=idx, sel_logit=logit)
    st = dec.status()
    return out, idx, logit, st


def check_rows(inp, h_q, h_k, h_v, N, out, idx, logit, rows):
    q = to_np(inp.q)
    k = inp.k_cache
    v = inp.v_cache
    lens = inp.seq_lens.tolist()
    out_n, idx_n, logit_n = to_np(out), idx.cpu().numpy(), logit.cpu().numpy()
    g, g_v = h_q // h_k, h_q // h_v
    band_swaps = 0
    for b, j in rows:
        L = lens[b]
        k_rows = to_np(k[b, j // g, :L])
        v_rows = to_np(v[b, j // g_v, :L])
        band_swaps += check_row(idx_n[b, j], logit_n[b, j], out_n[b, j], q[b, j], k_rows, v_rows,
                                N, what=f"(b={b}, j={j})")
    return band_swaps


def make_raw(seed, B, L_max, lens, h_q, h_k, h_v, d):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, h_q, d, generator=g).to(torch.bfloat16)
    k = torch.randn(B, h_k, L_max, d, generator=g).to(torch.bfloat16)
    v = torch.randn(B, h_v, L_max, d, generator=g).to(torch.bfloat16)
    return workload.DecodeInputs(q, k, v, torch.tensor(lens, dtype=torch.int32))


# --------------------------------------------------------------------------- workloads

def test_tiny_planted_all_rows():
    spec = workload.TINY
    inp = workload.make_inputs(spec)
    dec = SagaDecoder(spec.batch, spec.seq_len, spec.h_q, spec.h_k, spec.h_v, spec.head_dim, spec.N)
    out, idx, logit, st = run_decode(dec, *_dev(inp), spec.N)
    assert st == 0
    rows = [(0, j) for j in range(spec.h_q)]
    check_rows(inp, spec.h_q, spec.h_k, spec.h_v, spec.N, out, idx, logit, rows)
    # closed form: each head's output is the mean of V over its 16 planted keys
    for j in range(spec.h_q):
        pos = sorted(p for b, jj, p in inp.planted if jj == j)
        assert set(pos) <= set(idx[0, j].tolist())
        mean_v = to_np(inp.v_cache[0, j // spec.g_v, pos]).astype(np.float64).mean(0)
        assert_out_close(to_np(out[0, j]), mean_v, f"closed form head {j}")


def test_dense_llama_all_rows_equal_softmax_attention():
    spec = workload.DENSE_LLAMA
    inp = workload.make_inputs(spec)
    dec = SagaDecoder(spec.batch, spec.seq_len, spec.h_q, spec.h_k, spec.h_v, spec.head_dim, spec.N)
    out, idx, logit, st = run_decode(dec, *_dev(inp), spec.N)
    assert st == 0
    # N = L: every position selected, in order
    assert (idx.cpu() == torch.arange(spec.seq_len, dtype=torch.int32)).all()
    rows = [(b, j) for b in range(spec.batch) for j in range(spec.h_q)]
    check_rows(inp, spec.h_q, spec.h_k, spec.h_v, spec.N, out, idx, logit, rows)


@pytest.mark.parametrize("spec", [workload.QWEN_32K, workload.LLAMA_RAGGED], ids=lambda s: s.name)
def test_full_size_sampled_rows(spec):
    inp = workload.make_inputs(spec)
    dec = SagaDecoder(spec.batch, spec.seq_len, spec.h_q, spec.h_k, spec.h_v, spec.head_dim, spec.N)
    out, idx, logit, st = run_decode(dec, *_dev(inp), spec.N)
    assert st == 0
    rng = np.random.default_rng(1)
    rows = {(int(rng.integers(spec.batch)), int(rng.integers(spec.h_q))) for _ in range(10)}
    rows |= {(0, 0), (spec.batch - 1, spec.h_q - 1)}
    check_rows(inp, spec.h_q, spec.h_k, spec.h_v, spec.N, out, idx, logit, sorted(rows))
    # properties of every row: N_b ascending positions below L_b; planted keys kept
    idx_c = idx.cpu()
    lens = inp.seq_lens.tolist()
    for b in range(spec.batch):
        sel = idx_c[b]
        assert (sel[:, 1:] > sel[:, :-1]).all() and (sel[:, 0] >= 0).all()
        assert (sel[:, -1] < lens[b]).all()
    keep = {}
    for b, j, p in inp.planted:
        keep.setdefault((b, j), []).append(p)
    for (b, j), pos in keep.items():
        assert set(pos) <= set(idx_c[b, j].tolist()), f"planted keys of ({b}, {j}) not selected"
    assert torch.isfinite(out.float()).all()


SWEEP = {s.name: s for s in workload.sweep_specs()}
SWEEP_POINTS = ["qwen_sweep_b1_l128k_n2048", "qwen_sweep_b8_l32k_n1024",
                "qwen_sweep_b64_l8k_n512", "qwen_sweep_b64_l128k_n512"]


@pytest.mark.parametrize("name", SWEEP_POINTS)
def test_sweep_points_sampled_rows(name):
    # Corners of the long-context sweep (Qwen shapes, 1% planted keys), inputs drawn
    # on the device; rows of 128K positions fit the shared-memory candidate list.
    spec = SWEEP[name]
    inp = workload.make_inputs(spec, device="cuda")
    dec = SagaDecoder(spec.batch, spec.seq_len, spec.h_q, spec.h_k, spec.h_v, spec.head_dim, spec.N)
    out, idx, logit, st = run_decode(dec, inp.q, inp.k_cache, inp.v_cache, inp.seq_lens, spec.N)
    assert st & 0xFF == 0
    rng = np.random.default_rng(len(name))
    rows = {(int(rng.integers(spec.batch)), int(rng.integers(spec.h_q))) for _ in range(3)}
    rows |= {(0, 0), (spec.batch - 1, spec.h_q - 1)}
    check_rows(inp, spec.h_q, spec.h_k, spec.h_v, spec.N, out, idx, logit, sorted(rows))
    idx_c = idx.cpu()
    assert (idx_c[..., 1:] > idx_c[..., :-1]).all() and (idx_c[..., 0] >= 0).all()
    keep = {}
    for b, j, pos in inp.planted:
        keep.setdefault((b, j), []).append(pos)
    for (b, j), pos in keep.items():
        assert set(pos) <= set(idx_c[b, j].tolist()), f"planted keys of ({b}, {j}) not selected"
    assert torch.isfinite(out.float()).all()


# --------------------------------------------------------------------------- shapes and edges

SHAPES = [
    # (B, L_max, lens, h_q, h_k, h_v, d, N)
    (2, 1000, [1000, 617], 8, 2, 4, 64, 64),          # ragged, L not a multiple of 128
    (3, 300, [300, 1, 129], 4, 4, 4, 128, 32),        # MHA (g = 1), a 1-position row
    (1, 4096, [4096], 64, 1, 8, 64, 256),             # g = 64
    (2, 2048, [2048, 2000], 48, 1, 2, 128, 100),      # g = 48
    (2, 2048, [1500, 2048], 20, 1, 4, 64, 1499),      # g = 20, N_b = L_b - 1 and L_b = N + 1
    (4, 512, [512, 511, 100, 50], 12, 1, 2, 128, 256),  # rows with L_b < N (dense rows)
    (1, 70000, [70000], 12, 1, 2, 128, 2048),         # long row: many compaction chunks
    (2, 3000, [3000, 2999], 16, 2, 16, 64, 1),        # N = 1
    (64, 640, [640 - 7 * i for i in range(64)], 8, 1, 2, 128, 40),  # many rows
]


@pytest.mark.parametrize("shape", SHAPES, ids=[f"s{i}" for i in range(len(SHAPES))])
def test_shapes_all_rows(shape):
    B, L_max, lens, h_q, h_k, h_v, d, N = shape
    inp = make_raw(100 + B + L_max, B, L_max, lens, h_q, h_k, h_v, d)
    dec = SagaDecoder(B, L_max, h_q, h_k, h_v, d, N)
    out, idx, logit, st = run_decode(dec, *_dev(inp), N)
    assert st & 0xFF == 0
    rows = [(b, j) for b in range(B) for j in range(h_q)]
    check_rows(inp, h_q, h_k, h_v, N, out, idx, logit, rows)


def test_duplicate_keys_ties_go_to_lowest_index():
    B, L, h_q, h_k, h_v, d, N = 1, 2048, 8, 1, 2, 64, 300
    inp = make_raw(7, B, L, [L], h_q, h_k, h_v, d)
    # every key appears 4 times: scores come in groups of 4 exact ties
    base = inp.k_cache[:, :, :L // 4].clone()
    inp.k_cache[:, :, :] = base.repeat_interleave(4, dim=2)
    dec = SagaDecoder(B, L, h_q, h_k, h_v, d, N)
    q, k, v, lens = _dev(inp)
    out, idx, logit, st = run_decode(dec, q, k, v, lens, N)
    z_gpu = dec.score(q, k, lens)
    for j in range(h_q):
        z = z_gpu[0, j, :L].cpu().numpy().astype(np.float64)
        # on the GPU's own scores the selection is unique: compare bit-exactly
        assert idx[0, j].tolist() == oracle.top_n(z, N).tolist()
    check_rows(inp, h_q, h_k, h_v, N, out, idx, logit, [(0, j) for j in range(h_q)])


def test_all_equal_scores_take_lowest_positions():
    # row 0 is too long for the candidate buffer and too flat for the histogram:
    # it takes a whole-row path; row 1 fits the buffer directly
    B, L, h_q, h_k, h_v, d, N = 2, 20000, 4, 1, 1, 128, 777
    inp = make_raw(8, B, L, [L, 5000], h_q, h_k, h_v, d)
    inp.k_cache[:] = inp.k_cache[:, :, :1]            # one key everywhere: every score equal
    dec = SagaDecoder(B, L, h_q, h_k, h_v, d, N)
    out, idx, logit, st = run_decode(dec, *_dev(inp), N)
    assert st & (_lib.SAGA_STATUS_INFO_EXACT_FALLBACK | _lib.SAGA_STATUS_INFO_ROBUST_PATH)
    assert (idx.cpu() == torch.arange(N, dtype=torch.int32)).all()
    for b in range(B):
        mean_v = to_np(inp.v_cache[b, 0, :N]).astype(np.float64).mean(0)
        for j in range(h_q):
            assert_out_close(to_np(out[b, j]), mean_v, f"row ({b},{j})")


def test_bound_that_misses_rescores_the_row():
    # Adversarial for the sampled bound: query-aligned keys exactly at the 1024
    # sampled positions (32 blocks of 32 at 32 * floor(blk * (L / 32) / 32)),
    # small keys elsewhere, and N = 2048.  The bound lands among the planted
    # scores, fewer than N_b scores pass it, and the row must be scored again
    # and selected exactly (INFO_ROBUST_PATH).
    B, L, h_q, h_k, h_v, d, N = 1, 16384, 4, 1, 2, 64, 2048
    inp = make_raw(11, B, L, [L], h_q, h_k, h_v, d)
    inp.q[:] = inp.q[:, :1]                               # one query for all four heads
    inp.k_cache.mul_(0.1)
    lpb = L // 32
    sampled = [32 * ((blk * lpb) // 32) + i for blk in range(32) for i in range(32)]
    inp.k_cache[0, 0, sampled] = (3.0 * inp.q[0, 0].float()).to(torch.bfloat16)
    dec = SagaDecoder(B, L, h_q, h_k, h_v, d, N)
    out, idx, logit, st = run_decode(dec, *_dev(inp), N)
    assert st & _lib.SAGA_STATUS_INFO_ROBUST_PATH
    assert st & 0xFF == 0
    sel = set(idx[0, 0].tolist())
    assert set(sampled) <= sel                            # every planted key is selected
    check_rows(inp, h_q, h_k, h_v, N, out, idx, logit, [(0, j) for j in range(h_q)])


def test_bad_seq_lens_flagged_and_zeroed():
    B, L, h_q, h_k, h_v, d, N = 3, 1024, 4, 1, 2, 64, 64
    inp = make_raw(9, B, L, [0, 700, L + 5], h_q, h_k, h_v, d)
    dec = SagaDecoder(B, L, h_q, h_k, h_v, d, N)
    out, idx, logit, st = run_decode(dec, *_dev(inp), N)
    assert st & _lib.SAGA_STATUS_BAD_SEQ_LEN
    for b in (0, 2):
        assert (out[b].float() == 0).all()
        assert (idx[b] == -1).all()
    inp.seq_lens[:] = torch.tensor([1, 700, 1], dtype=torch.int32)
    check_rows(inp, h_q, h_k, h_v, N, out, idx, logit, [(1, j) for j in range(h_q)])
    assert dec.status() == 0        # status was cleared by the previous read


# --------------------------------------------------------------------------- stages alone

def test_score_stage_against_oracle():
    B, L, h_q, h_k, h_v, d = 2, 3000, 24, 2, 4, 128
    inp = make_raw(10, B, L, [3000, 1234], h_q, h_k, h_v, d)
    dec = SagaDecoder(B, L, h_q, h_k, h_v, d, 16)
    q, k, v, lens = _dev(inp)
    z = dec.score(q, k, lens).cpu().numpy()
    qn = to_np(inp.q)
    for b, Lb in enumerate([3000, 1234]):
        assert np.isnan(z[b, :, Lb:]).all()        # positions >= L_b untouched
        for j in range(h_q):
            k_rows = to_np(inp.k_cache[b, j // (h_q // h_k), :Lb])
            ref = oracle.scores(qn[b, j], k_rows)
            assert (np.abs(z[b, j, :Lb] - ref) <= score_bound(qn[b, j], k_rows)).all()


CRAFTED = {
    "two_valued": lambda rng, L: rng.choice([1.5, -2.0], size=L),
    "all_equal": lambda rng, L: np.full(L, 0.25),
    "ascending": lambda rng, L: np.linspace(-3, 3, L),
    "descending": lambda rng, L: np.linspace(5, -5, L),
    "signed_zeros": lambda rng, L: rng.choice([0.0, -0.0, 1.0, -1.0], size=L),
    "outliers": lambda rng, L: np.where(rng.random(L) < 0.001, 1e30, rng.standard_normal(L)),
    "all_negative": lambda rng, L: -np.abs(rng.standard_normal(L)) - 10,
    "tiny_range": lambda rng, L: 1.0 + rng.integers(0, 5, size=L) * 2.0 ** -23,
    "subnormal": lambda rng, L: rng.integers(-3, 4, size=L) * 1e-40,
    "normal": lambda rng, L: rng.standard_normal(L),
    "huge_range": lambda rng, L: rng.choice([-3e38, 3e38, 0.0, 1.0], size=L),
}


@pytest.mark.parametrize("kind", sorted(CRAFTED))
@pytest.mark.parametrize("N", [1, 100, 4999, 6000])
def test_select_stage_bit_exact(kind, N):
    B, h_q, L = 2, 3, 5000
    rng = np.random.default_rng(sum(map(ord, kind)) * 7919 + N)
    z = np.stack([np.stack([CRAFTED[kind](rng, L) for _ in range(h_q)]) for _ in range(B)])
    z32 = torch.from_numpy(z.astype(np.float32))
    dec = SagaDecoder(B, L, h_q, 1, 1, 64, N)
    lens = torch.tensor([L, L - 1234], dtype=torch.int32)
    idx, logit = dec.select(z32.cuda(), lens.cuda(), N)
    dec.status()
    z64 = z32.double().numpy()
    for b in range(B):
        Lb = int(lens[b])
        n_b = min(N, Lb)
        for j in range(h_q):
            want = oracle.top_n(z64[b, j, :Lb], N)
            got = idx[b, j].cpu().numpy()
            assert got[:n_b].tolist() == want.tolist(), f"{kind} ({b},{j})"
            assert (got[n_b:] == -1).all()
            np.testing.assert_array_equal(logit[b, j, :n_b].cpu().numpy(), z32[b, j, want].numpy())


def test_combine_stage_against_oracle():
    B, L, h_q, h_v, d, N = 2, 4000, 8, 2, 128, 333
    inp = make_raw(11, B, L, [4000, 2500], h_q, 1, h_v, d)
    rng = np.random.default_rng(3)
    idx = np.full((B, h_q, N), -1, dtype=np.int32)
    logit = np.full((B, h_q, N), -np.inf, dtype=np.float32)
    for b, Lb in enumerate([4000, 2500]):
        for j in range(h_q):
            n = N - 17 * j
            idx[b, j, :n] = np.sort(rng.choice(Lb, size=n, replace=False))
            logit[b, j, :n] = rng.standard_normal(n) * 3
    dec = SagaDecoder(B, L, h_q, 1, h_v, d, N)
    out = dec.combine(torch.from_numpy(idx).cuda(), torch.from_numpy(logit).cuda(),
                      inp.v_cache.cuda(), inp.seq_lens.cuda())
    assert dec.status() == 0
    for b in range(B):
        for j in range(h_q):
            valid = idx[b, j] >= 0
            ref = oracle.combine(logit[b, j, valid].astype(np.float64),
                                 to_np(inp.v_cache[b, j // (h_q // h_v), idx[b, j, valid]]))
            assert_out_close(to_np(out[b, j]), ref, f"({b},{j})")


def test_fused_selection_equals_stagewise():
    spec = workload.scaled(workload.QWEN_32K, batch=3, seq_len=20000)
    inp = workload.make_inputs(spec)
    dec = SagaDecoder(spec.batch, spec.seq_len, spec.h_q, spec.h_k, spec.h_v, spec.head_dim, spec.N)
    q, k, v, lens = _dev(inp)
    out, idx, logit, st = run_decode(dec, q, k, v, lens, spec.N)
    z = dec.score(q, k, lens)
    idx2, logit2 = dec.select(z, lens, spec.N)
    out2 = dec.combine(idx2, logit2, v, lens)
    assert torch.equal(idx, idx2) and torch.equal(logit, logit2)
    # same selection and weights; the fused P.V sums in another order, so the
    # two fp32 accumulations may round to neighbouring bf16 values
    torch.testing.assert_close(out.float(), out2.float(), atol=2e-3, rtol=1e-2)


# --------------------------------------------------------------------------- API behaviour

def test_deterministic_and_host_entry_point():
    spec = workload.scaled(workload.LLAMA_RAGGED, batch=4, seq_len=4096, ragged=(1000, 4096))
    inp = workload.make_inputs(spec)
    dec = SagaDecoder(spec.batch, spec.seq_len, spec.h_q, spec.h_k, spec.h_v, spec.head_dim, spec.N)
    q, k, v, lens = _dev(inp)
    a, ia, la, _ = run_decode(dec, q, k, v, lens, spec.N)
    b, ib, lb, _ = run_decode(dec, q, k, v, lens, spec.N)
    assert torch.equal(a, b) and torch.equal(ia, ib) and torch.equal(la, lb)
    q_h = inp.q.clone().pin_memory()
    l_h = inp.seq_lens.clone().pin_memory()
    o_h = torch.empty_like(inp.q).pin_memory()
    n0 = dec.launch_count()
    dec.attn_host(q_h, k, v, l_h, spec.N, o_h)
    assert dec.status() == 0
    assert dec.launch_count() - n0 == 4   # sample, bound, score, top-N with P.V
    assert torch.equal(o_h, a.cpu())


def test_batch_smaller_than_max():
    spec = workload.scaled(workload.TINY, batch=4)
    inp = workload.make_inputs(spec)
    dec = SagaDecoder(8, spec.seq_len, spec.h_q, spec.h_k, spec.h_v, spec.head_dim, spec.N)
    dec.set_batch(4)
    out, idx, logit, st = run_decode(dec, *_dev(inp), spec.N)
    assert st == 0
    check_rows(inp, spec.h_q, spec.h_k, spec.h_v, spec.N, out, idx, logit,
               [(b, j) for b in range(4) for j in range(0, spec.h_q, 3)])


def test_bounded_wait_runs_out_and_reports_timeout():
    # Failure detection without a fault: a pipeline wait with nothing to wait for
    # gives up after its limit, the status word says SAGA_STATUS_TIMEOUT, and the
    # handle keeps working (the next decode call is clean and correct).
    spec = workload.TINY
    inp = workload.make_inputs(spec)
    dec = SagaDecoder(spec.batch, spec.seq_len, spec.h_q, spec.h_k, spec.h_v, spec.head_dim, spec.N)
    dec.selftest_timeout()
    st = dec.status()
    assert st & _lib.SAGA_STATUS_TIMEOUT
    out, idx, logit, st = run_decode(dec, *_dev(inp), spec.N)
    assert st == 0
    check_rows(inp, spec.h_q, spec.h_k, spec.h_v, spec.N, out, idx, logit,
               [(0, j) for j in range(spec.h_q)])
