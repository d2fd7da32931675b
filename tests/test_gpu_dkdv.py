"""Keys and values of different widths ("More Value per Key" §5.2) on the GPU.

A handle made with ``head_dim_v`` != ``head_dim`` scores with the key width
(scale 1/sqrt(d_k)) and gathers values of the value width; keys of width 32 (the
pages' (h_k, d_k) = (2, 32) variant) take the score pass's 64-byte-swizzle tiles.  Every row is checked
against the oracle with the rules of ``parity_utils`` (scores with d_k terms,
outputs of width d_v), on the candidate path (N <= 2048 and short of the row)
and on the score-row path (N >= L_b: every position).
"""
import pytest
import torch

from test_gpu_parity import check_rows, run_decode
from sparse_asymmetric_gqa_b200 import SagaDecoder, SagaError, workload

pytestmark = pytest.mark.gpu


def make_kv(seed, B, L, lens, h_q, h_k, h_v, d_k, d_v):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, h_q, d_k, generator=g).to(torch.bfloat16)
    k = torch.randn(B, h_k, L, d_k, generator=g).to(torch.bfloat16)
    v = torch.randn(B, h_v, L, d_v, generator=g).to(torch.bfloat16)
    return workload.DecodeInputs(q, k, v, torch.tensor(lens, dtype=torch.int32))


@pytest.mark.parametrize("d_k,d_v", [(64, 128), (128, 64), (32, 64), (32, 128)])
@pytest.mark.parametrize("case", [
    # (B, L, lens, h_q, h_k, h_v, N)
    (3, 20000, [20000, 9000, 777], 8, 2, 4, 512),     # candidate path, ragged rows
    (2, 3000, [3000, 2100], 4, 1, 2, 4096),           # score-row path: N >= L_b
])
def test_keys_and_values_of_different_widths(d_k, d_v, case):
    B, L, lens, h_q, h_k, h_v, N = case
    inp = make_kv(17 + d_k, B, L, lens, h_q, h_k, h_v, d_k, d_v)
    dec = SagaDecoder(B, L, h_q, h_k, h_v, d_k, N, head_dim_v=d_v)
    q, k, v, sl = inp.q.cuda(), inp.k_cache.cuda(), inp.v_cache.cuda(), inp.seq_lens.cuda()
    out, idx, logit, st = run_decode(dec, q, k, v, sl, N)
    assert out.shape == (B, h_q, d_v)
    assert st & 0xFF == 0
    rows = [(b, j) for b in range(B) for j in range(h_q)]
    check_rows(inp, h_q, h_k, h_v, N, out, idx, logit, rows)


def test_mixed_widths_refuse_the_stateful_and_group_calls():
    B, L, h_q, h_k, h_v, N = 1, 4096, 4, 1, 2, 256
    inp = make_kv(3, B, L, [L], h_q, h_k, h_v, 64, 128)
    dec = SagaDecoder(B, L, h_q, h_k, h_v, 64, N, head_dim_v=128)
    q, k, v, sl = inp.q.cuda(), inp.k_cache.cuda(), inp.v_cache.cuda(), inp.seq_lens.cuda()
    with pytest.raises(SagaError):
        dec.atopn_calibrate(q, k, v, sl, N)
    with pytest.raises(SagaError):
        dec.group_attn(q, k, v, sl, N)
    out = dec.attn(q, k, v, sl, N)                   # the exact step still runs on the handle
    assert dec.status() & 0xFF == 0 and torch.isfinite(out.float()).all()
