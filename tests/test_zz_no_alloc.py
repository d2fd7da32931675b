"""saga_combine_noalloc against saga_combine.

saga_combine_noalloc is the softmax + gathered P.V step for callers that cannot allocate
device memory (a serving engine whose memory manager owns the whole device, a process under a
hard memory cap): it takes no handle and keeps its scratch in a fixed array inside the
library.  Here it is called through the C ABI twice in a row and each result is checked
against the handle-based saga_combine on the same selection, with the parity tolerance of the
other tests (|err| <= 2e-3 or <= 1e-2 |ref|).  The file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

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
    return torch.from_numpy(idx).cuda(), torch.from_numpy(logit).cuda()


def _call_noalloc(lib, idx, logit, v, lens, out):
    B, h_q, N = idx.shape
    _, h_v, L_max, d = v.shape
    stream = torch.cuda.current_stream().cuda_stream
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    return lib.saga_combine_noalloc(p(idx), p(logit), p(v), p(lens), B, L_max, h_q, h_v, d, N,
                                    p(out), ctypes.c_void_p(stream))


@pytest.mark.parametrize("shape", [
    # (B, L_max, lens, h_q, h_v, d, N)
    (4, 6000, [6000, 4100, 650, 5999], 12, 2, 128, 1024),
    (3, 3000, [3000, 700, 2999], 16, 8, 64, 3000),          # dense rows (N >= L_b)
])
def test_noalloc_matches_handle_path_on_two_calls(shape):
    B, L_max, lens, h_q, h_v, d, N = shape
    g = torch.Generator().manual_seed(11)
    v = torch.randn(B, h_v, L_max, d, generator=g).to(torch.bfloat16).cuda()
    seq = torch.tensor(lens, dtype=torch.int32).cuda()
    lib = load()
    dec = SagaDecoder(B, L_max, h_q, 1, h_v, d, N)
    for call in range(2):
        idx, logit = _selection(100 + call, B, h_q, N, lens)
        ref = dec.combine(idx, logit, v, seq)
        out = torch.full((B, h_q, d), float("nan"), dtype=torch.bfloat16, device="cuda")
        assert _call_noalloc(lib, idx, logit, v, seq, out) == _lib.SAGA_OK
        torch.cuda.synchronize()
        assert dec.status() == 0
        assert_out_close(to_np(out), to_np(ref), f"call {call}")


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
