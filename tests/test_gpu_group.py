"""GPU parity of group-shared selection (``saga_group_attn``) against the oracle.

One set of positions per value head: the N_b largest s_i = sum over the group's
heads of softmax(z_j)_i (``oracle.group_oracle``).  Matching: positions whose
oracle s lies within a band of the oracle's N_b-th s may go either way, the band
being the fp32 error of s (the score bound and the log-sum-exp error of each
head, relative to s); each head's logits within the score bound; outputs against
the oracle's softmax and P.V over the GPU's set.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from oracle import group_oracle as go
from parity_utils import BAND, assert_out_close, lse_error, score_bound, to_np
from sparse_asymmetric_gqa_b200 import SagaDecoder, SagaError, workload
from sparse_asymmetric_gqa_b200 import _lib

pytestmark = pytest.mark.gpu


def make_raw(seed, B, L_max, lens, h_q, h_k, h_v, d):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, h_q, d, generator=g).to(torch.bfloat16)
    k = torch.randn(B, h_k, L_max, d, generator=g).to(torch.bfloat16)
    v = torch.randn(B, h_v, L_max, d, generator=g).to(torch.bfloat16)
    return workload.DecodeInputs(q, k, v, torch.tensor(lens, dtype=torch.int32))


def run_group(dec, inp, N):
    B, h_q = inp.q.shape[:2]
    h_v = inp.v_cache.shape[1]
    idx = torch.empty(B, h_v, N, dtype=torch.int32, device="cuda")
    stat = torch.empty(B, h_v, N, dtype=torch.float32, device="cuda")
    logit = torch.empty(B, h_q, N, dtype=torch.float32, device="cuda")
    out = dec.group_attn(inp.q.cuda(), inp.k_cache.cuda(), inp.v_cache.cuda(), inp.seq_lens.cuda(), N,
                         sel_idx=idx, sel_stat=stat, sel_logit=logit)
    return out, idx.cpu().numpy(), stat.cpu().numpy(), logit.cpu().numpy(), dec.status()


def check_group(inp, h_q, h_k, h_v, N, out, idx, stat, logit, groups):
    q = to_np(inp.q)
    g, g_v = h_q // h_k, h_q // h_v
    lens = inp.seq_lens.tolist()
    o = to_np(out)
    for b, vh in groups:
        L = lens[b]
        heads = list(range(vh * g_v, (vh + 1) * g_v))
        keys = [to_np(inp.k_cache[b, j // g, :L]) for j in heads]
        vals = to_np(inp.v_cache[b, vh, :L])
        z = np.stack([oracle.scores(q[b, j], keys[r]) for r, j in enumerate(heads)])
        s = go.group_statistic(z)
        n_b = min(N, L)
        sel = idx[b, vh]
        n = int((sel >= 0).sum())
        assert n == n_b and (sel[n:] == -1).all() and (np.diff(sel[:n]) > 0).all()
        sN = np.sort(s)[::-1][n_b - 1]
        err = max(lse_error(q[b, j], keys[r], z[r])[1] + float(score_bound(q[b, j], keys[r]).max())
                  for r, j in enumerate(heads))
        band = sN * (BAND + 2 * err) + 1e-30
        gpu = np.zeros(L, dtype=bool)
        gpu[sel[:n]] = True
        assert not ((s > sN + band) & ~gpu).any(), f"({b},{vh}) missed positions"
        assert not ((s < sN - band) & gpu).any(), f"({b},{vh}) extra positions"
        rel = np.abs(stat[b, vh, :n] - s[sel[:n]]) / np.maximum(s[sel[:n]], 1e-30)
        assert (rel <= BAND + 2 * err).all(), f"({b},{vh}) s off by {rel.max()}"
        for r, j in enumerate(heads):
            bound = score_bound(q[b, j], keys[r][sel[:n]])
            assert (np.abs(logit[b, j, :n] - z[r][sel[:n]]) <= bound).all()
            assert np.isneginf(logit[b, j, n:]).all()
            assert_out_close(o[b, j], oracle.combine(z[r][sel[:n]], vals[sel[:n]]), f"({b},{j}) out")


CASES = [
    # (B, L_max, lens, h_q, h_k, h_v, d, N, planted)
    (2, 20000, [20000, 15000], 12, 1, 2, 128, 256, True),    # Qwen heads, peaked rows
    (2, 16384, [16384, 9000], 8, 2, 4, 64, 128, False),      # flat rows: the check may send them back
    (2, 4096, [4096, 1000], 16, 1, 8, 64, 64, False),        # rows that keep every position
    (1, 12000, [12000], 4, 1, 4, 128, 100, False),           # g_v = 1: the per-head top-N
]


@pytest.mark.parametrize("case", CASES, ids=[f"c{i}" for i in range(len(CASES))])
def test_group_selection_against_oracle(case):
    B, L_max, lens, h_q, h_k, h_v, d, N, planted = case
    if planted:
        spec = workload.scaled(workload.QWEN_32K, batch=B, seq_len=L_max, N=N, layers=1, seed=91)
        inp = workload.make_inputs(spec)
        inp.seq_lens[:] = torch.tensor(lens, dtype=torch.int32)
    else:
        inp = make_raw(60 + N, B, L_max, lens, h_q, h_k, h_v, d)
    dec = SagaDecoder(B, L_max, h_q, h_k, h_v, d, N)
    out, idx, stat, logit, st = run_group(dec, inp, N)
    assert st & 0xFF == 0
    groups = [(b, vh) for b in range(B) for vh in range(h_v)]
    check_group(inp, h_q, h_k, h_v, N, out, idx, stat, logit, groups)


def test_group_of_one_head_selects_the_per_head_top_n():
    B, L, h_q, h_k, h_v, d, N = 1, 12000, 4, 1, 4, 128, 100
    inp = make_raw(70, B, L, [L], h_q, h_k, h_v, d)
    dec = SagaDecoder(B, L, h_q, h_k, h_v, d, N)
    out, idx, _, _, st = run_group(dec, inp, N)
    assert st & 0xFF == 0
    sel = torch.empty(B, h_q, N, dtype=torch.int32, device="cuda")
    ref = dec.attn(inp.q.cuda(), inp.k_cache.cuda(), inp.v_cache.cuda(), inp.seq_lens.cuda(), N,
                   sel_idx=sel)
    assert np.array_equal(idx, sel.cpu().numpy())
    assert_out_close(to_np(out), to_np(ref), "group of one vs per-head")


def test_group_unsupported_shapes():
    dec = SagaDecoder(1, 4096, 64, 1, 8, 64, 256)       # g = 64 > 32
    inp = make_raw(71, 1, 4096, [4096], 64, 1, 8, 64)
    with pytest.raises(SagaError) as e:
        dec.group_attn(inp.q.cuda(), inp.k_cache.cuda(), inp.v_cache.cuda(), inp.seq_lens.cuda(), 64)
    assert e.value.code == _lib.SAGA_ERR_UNSUPPORTED
