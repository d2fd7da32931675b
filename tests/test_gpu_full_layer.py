"""Every row of one full-size layer against the plain C++ oracle (float64).

The sampled-row parity tests check a dozen rows of each full-size workload
with the Python oracle; here the threaded C++ oracle (``oracle/decode_ref.cpp``)
decodes every (b, j) row of layer 0 of the Qwen 32K batch and of the ragged
Llama batch, and the GPU's selection and output are compared row by row with
the rules of ``parity_utils``: the sets may differ only at positions whose
float64 score lies within BAND of the oracle's N_b-th score, and the output
matches the oracle's softmax and P.V (on the oracle's set when the sets agree,
else on the GPU's set).
"""
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import cref
from parity_utils import BAND, assert_out_close, to_np
from sparse_asymmetric_gqa_b200 import SagaDecoder, workload

pytestmark = pytest.mark.gpu


def _scores64(q_row, k_rows):
    d = q_row.shape[0]
    return (k_rows.astype(np.float64) @ q_row.astype(np.float64)) / np.sqrt(d)


@pytest.mark.parametrize("spec", [workload.QWEN_32K, workload.LLAMA_RAGGED], ids=lambda s: s.name)
def test_full_layer_every_row_vs_cpp_oracle(spec):
    inp = workload.make_inputs(spec, layer=0, device="cuda")
    B, h_q, N = spec.batch, spec.h_q, spec.N
    dec = SagaDecoder(B, spec.seq_len, h_q, spec.h_k, spec.h_v, spec.head_dim, N)
    idx = torch.empty(B, h_q, N, dtype=torch.int32, device="cuda")
    logit = torch.empty(B, h_q, N, dtype=torch.float32, device="cuda")
    out = dec.attn(inp.q, inp.k_cache, inp.v_cache, inp.seq_lens, N, sel_idx=idx, sel_logit=logit)
    assert dec.status() & 0xFF == 0
    lens = inp.seq_lens.cpu().numpy()
    out_o, idx_o, logit_o = cref.decode(inp.q.cpu(), inp.k_cache.cpu(), inp.v_cache.cpu(), lens,
                                        h_q, spec.h_k, spec.h_v, N, threads=os.cpu_count() or 1)
    q = to_np(inp.q)
    k = inp.k_cache.cpu()
    v = inp.v_cache.cpu()
    g, g_v = spec.g, spec.g_v
    gi, go = idx.cpu().numpy(), to_np(out)
    differing = 0
    for b in range(B):
        L = int(lens[b])
        n_b = min(N, L)
        k_b = [to_np(k[b, kh, :L]) for kh in range(spec.h_k)]
        for j in range(h_q):
            what = f"{spec.name} (b={b}, j={j})"
            sel = gi[b, j, :n_b]
            assert (gi[b, j, n_b:] == -1).all(), f"{what}: padding"
            assert (np.diff(sel) > 0).all() and sel[0] >= 0 and sel[-1] < L, f"{what}: indices"
            ref = np.sort(idx_o[b, j, :n_b])
            t = logit_o[b, j, :n_b].min()                 # the oracle's N_b-th score
            diff = np.setxor1d(sel, ref)
            if diff.size:
                differing += diff.size
                z_diff = _scores64(q[b, j], k_b[j // g][diff])
                assert (np.abs(z_diff - t) <= BAND).all(), f"{what}: sets differ outside the band"
                z_sel = _scores64(q[b, j], k_b[j // g][sel])
                ref_out = oracle.combine(z_sel, to_np(v[b, j // g_v, :L])[sel])
            else:
                ref_out = out_o[b, j]
            assert_out_close(go[b, j], ref_out, what)
    # a handful of positions may sit inside the band; a large count means a wrong rule
    assert differing <= B * h_q, f"{differing} positions differ"
