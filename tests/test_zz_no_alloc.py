"""saga_combine_noalloc against the oracle and against saga_combine.

saga_combine_noalloc is the softmax + gathered P.V step for callers that cannot allocate
device memory (a serving engine whose memory manager owns the whole device, a process under a
hard memory cap): it takes no handle and keeps its scratch in a fixed array inside the
library.  Here it is called through the C ABI twice in a row; each result is checked row by
row against the float64 oracle (oracle.combine over the same selection) and against the
handle-based saga_combine, with the parity tolerance of the other tests (|err| <= 2e-3 or
<= 1e-2 |ref|).  The entry point reports no device-side errors (there is no status word to
read), so the rows it must zero and the entries it must skip are checked directly.  The file
is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from parity_utils import assert_out_close, to_np
from sparse_asymmetric_gqa_b200 import SagaDecoder, _lib, load

pytestmark = pytest.mark.gpu


def _selection(seed, B, h_q, N, lens):
    rng = np.random.default_rng(seed)
    idx = np.full((B, h_q, N), -1, dtype=np.int32)
    logit = np.full((B, h_q, N), -np.inf, dtype=np.float32)
    for b, Lb in enumerate(lens):
        for j in range(h_q):
            n = min(N, Lb) - (5 * j) % 7
            idx[b, j, :n] = np.sort(rng.choice(Lb, size=n, replace=False))
            logit[b, j, :n] = rng.standard_normal(n) * 3
    return idx, logit


def _call_noalloc(lib, idx, logit, v, lens, out):
    B, h_q, N = idx.shape
    _, h_v, L_max, d = v.shape
    stream = torch.cuda.current_stream().cuda_stream
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    return lib.saga_combine_noalloc(p(idx), p(logit), p(v), p(lens), B, L_max, h_q, h_v, d, N,
                                    p(out), ctypes.c_void_p(stream))


def _oracle_rows(idx, logit, v, lens, g_v):
    """oracle.combine over the valid entries of every (b, j) selection row."""
    B, h_q, _ = idx.shape
    d = v.shape[-1]
    ref = np.zeros((B, h_q, d))
    for b in range(B):
        for j in range(h_q):
            keep = (idx[b, j] >= 0) & (idx[b, j] < lens[b])
            if keep.any():
                ref[b, j] = oracle.combine(logit[b, j][keep].astype(np.float64),
                                           v[b, j // g_v][idx[b, j][keep]])
    return ref


@pytest.mark.parametrize("shape", [
    # (B, L_max, lens, h_q, h_v, d, N)
    (4, 6000, [6000, 4100, 650, 5999], 12, 2, 128, 1024),
    (3, 3000, [3000, 700, 2999], 16, 8, 64, 3000),          # dense rows (N >= L_b)
])
def test_noalloc_matches_oracle_and_handle_path_on_two_calls(shape):
    B, L_max, lens, h_q, h_v, d, N = shape
    g = torch.Generator().manual_seed(11)
    v = torch.randn(B, h_v, L_max, d, generator=g).to(torch.bfloat16)
    v_np = v.float().numpy()
    v = v.cuda()
    seq = torch.tensor(lens, dtype=torch.int32).cuda()
    lib = load()
    dec = SagaDecoder(B, L_max, h_q, 1, h_v, d, N)
    for call in range(2):
        idx_np, logit_np = _selection(100 + call, B, h_q, N, lens)
        idx, logit = torch.from_numpy(idx_np).cuda(), torch.from_numpy(logit_np).cuda()
        out = torch.full((B, h_q, d), float("nan"), dtype=torch.bfloat16, device="cuda")
        assert _call_noalloc(lib, idx, logit, v, seq, out) == _lib.SAGA_OK
        torch.cuda.synchronize()
        got = to_np(out)
        assert_out_close(got, _oracle_rows(idx_np, logit_np, v_np, lens, h_q // h_v),
                         f"call {call} vs oracle")
        ref = dec.combine(idx, logit, v, seq)
        assert_out_close(got, to_np(ref), f"call {call} vs saga_combine")


def test_noalloc_zeros_bad_rows_and_skips_bad_indices():
    """A seq_len outside [1, L_max] zeroes its rows; an index >= the row's seq_len is skipped
    (the rest of the row is the oracle's softmax and P.V over the valid entries)."""
    B, L_max, h_q, h_v, d, N = 3, 2048, 4, 2, 128, 300
    lens = [2048, 0, 1500]                     # row 1 invalid
    g = torch.Generator().manual_seed(5)
    v = torch.randn(B, h_v, L_max, d, generator=g).to(torch.bfloat16)
    v_np = v.float().numpy()
    idx_np, logit_np = _selection(7, B, h_q, N, [2048, 2048, 1500])
    idx_np[2, 1, 3] = 1700                     # >= seq_lens[2]: skipped
    idx_np[2, 3, 0] = 1999
    lib = load()
    out = torch.full((B, h_q, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    seq = torch.tensor(lens, dtype=torch.int32).cuda()
    assert _call_noalloc(lib, torch.from_numpy(idx_np).cuda(), torch.from_numpy(logit_np).cuda(),
                         v.cuda(), seq, out) == _lib.SAGA_OK
    torch.cuda.synchronize()
    got = to_np(out)
    assert (got[1] == 0).all(), "rows of an invalid seq_len are zero"
    ref = _oracle_rows(idx_np, logit_np, v_np, [2048, 0, 1500], h_q // h_v)
    assert_out_close(got[0], ref[0], "valid row 0")
    assert_out_close(got[2], ref[2], "row 2 without its out-of-range entries")


def test_noalloc_rejects_problems_larger_than_its_scratch():
    lib = load()
    B, h_q, h_v, d, N, L_max = 64, 64, 8, 128, 8192, 8192     # 4096 rows x 32 chunks x 130 floats
    idx = torch.zeros(1, dtype=torch.int32, device="cuda")
    logit = torch.zeros(1, dtype=torch.float32, device="cuda")
    v = torch.zeros(1, dtype=torch.bfloat16, device="cuda")
    seq = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = torch.zeros(1, dtype=torch.bfloat16, device="cuda")
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    rc = lib.saga_combine_noalloc(p(idx), p(logit), p(v), p(seq), B, L_max, h_q, h_v, d, N, p(out),
                                  ctypes.c_void_p(0))
    assert rc == _lib.SAGA_ERR_SCRATCH_TOO_SMALL
    assert b"4 MiB" in lib.saga_decode_error_string(rc)
