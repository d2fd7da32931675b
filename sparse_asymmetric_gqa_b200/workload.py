"""Seeded synthetic decode workloads (inputs only; none of the method's arithmetic).

Both the CUDA path and the CPU oracle consume what this module produces; it
imports neither of them.  Every tensor is bf16 drawn from N(0, 1) (an fp32
draw rounded to nearest-even), from a ``torch.Generator`` seeded per workload.

"Planted" keys stand in for the sharp attention peaks of a trained model: a
planted position p of key head kh is assigned (round-robin) to one query head j
of that key head's group and gets the key bf16(s * q[b, j, :]), so its score
for head j is about s * |q_j|^2 / sqrt(d) = s * sqrt(d), far above the N(0, 1)
background.  The shapes are those of the decode workloads the paper measures
(Qwen2.5-1.5B: h_q = 12, h_k = 1 after merging, h_v = 2, d = 128; Llama-3.2-1B:
h_q = 32, h_k = 4, h_v = 8, d = 64).  The real workloads are model decodes on
RULER / GPQA prompts with trained weights, which are not available here.
"""
from __future__ import annotations

from dataclasses import dataclass, field, replace
from typing import Optional, Tuple

import torch


@dataclass(frozen=True)
class DecodeSpec:
    """Shape and planting recipe of one decode-attention workload."""
    name: str
    batch: int
    seq_len: int                  # L_max, the cache's position capacity
    h_q: int
    h_k: int
    h_v: int
    head_dim: int
    N: int
    planted_per_query_head: int = 0          # exact count per query head, or
    planted_frac: float = 0.0                # fraction of L_b per key head
    plant_scale: Tuple[float, float] = (3.0, 3.0)   # s fixed or ~U[lo, hi]
    ragged: Optional[Tuple[int, int]] = None  # seq_lens ~ U{lo..hi} if set
    layers: int = 1
    seed: int = 0
    head_dim_v: Optional[int] = None          # value width when it differs from head_dim

    @property
    def d_v(self) -> int:
        return self.head_dim if self.head_dim_v is None else self.head_dim_v

    @property
    def g(self) -> int:
        return self.h_q // self.h_k

    @property
    def g_v(self) -> int:
        return self.h_q // self.h_v


# The five workloads: a tiny parity case, a dense (N = seq_len) Llama-shaped
# layer, the Qwen-shaped 32K headline, a Llama-shaped ragged batch and the
# Qwen-shaped long-context sweep (one entry per point, built by sweep_specs()).
TINY = DecodeSpec("tiny_b1_l1k", batch=1, seq_len=1024, h_q=16, h_k=1, h_v=8,
                  head_dim=64, N=128, planted_per_query_head=16,
                  plant_scale=(3.0, 3.0), seed=0)
DENSE_LLAMA = DecodeSpec("dense_llama_b8_l8k", batch=8, seq_len=8192, h_q=32, h_k=4,
                         h_v=8, head_dim=64, N=8192, planted_frac=0.01,
                         plant_scale=(2.0, 4.0), seed=2000)
QWEN_32K = DecodeSpec("qwen2.5-1.5b_b16_l32k_n1024", batch=16, seq_len=32768, h_q=12,
                      h_k=1, h_v=2, head_dim=128, N=1024, planted_frac=0.02,
                      plant_scale=(2.0, 4.0), layers=28, seed=3000)
LLAMA_RAGGED = DecodeSpec("llama3.2-1b_b32_l16k_ragged_n512", batch=32, seq_len=16384,
                          h_q=32, h_k=4, h_v=8, head_dim=64, N=512,
                          planted_frac=0.02, plant_scale=(2.0, 4.0),
                          ragged=(8192, 16384), seed=4000)


def sweep_specs():
    """Qwen-shaped long-context sweep: B x L x N grid, 1% planted keys."""
    out = []
    k = 0
    for B in (1, 8, 64):
        for L in (8192, 32768, 131072):
            for N in (512, 1024, 2048):
                out.append(DecodeSpec(f"qwen_sweep_b{B}_l{L // 1024}k_n{N}", batch=B,
                                      seq_len=L, h_q=12, h_k=1, h_v=2, head_dim=128,
                                      N=N, planted_frac=0.01, plant_scale=(2.0, 4.0),
                                      seed=5000 + k))
                k += 1
    return out


# The pages' key-dimension variant of the Qwen shape ("More Value per Key" §5.2):
# (h_k, d_k) = (2, 32) with full-width values, so the key cache is half of the
# merged h_k = 1, d = 128 one.
QWEN_32K_DK32 = DecodeSpec("qwen2.5-1.5b_b16_l32k_n1024_hk2_dk32", batch=16, seq_len=32768, h_q=12,
                           h_k=2, h_v=2, head_dim=32, N=1024, planted_frac=0.02,
                           plant_scale=(2.0, 4.0), seed=3500, head_dim_v=128)

CONFIGS = {s.name: s for s in (TINY, DENSE_LLAMA, QWEN_32K, LLAMA_RAGGED, QWEN_32K_DK32)}


@dataclass
class DecodeInputs:
    q: torch.Tensor          # [B, h_q, d] bf16
    k_cache: torch.Tensor    # [B, h_k, L_max, d] bf16
    v_cache: torch.Tensor    # [B, h_v, L_max, d] bf16
    seq_lens: torch.Tensor   # [B] int32
    planted: list = field(default_factory=list)   # (b, j, position) triples


def make_inputs(spec: DecodeSpec, layer: int = 0, device="cpu",
                seed: Optional[int] = None) -> DecodeInputs:
    """Draw one layer's decode inputs for ``spec`` (seed = spec.seed + layer)."""
    if seed is None:
        seed = spec.seed + layer
    dev = torch.device(device)
    gen = torch.Generator(device=dev)
    gen.manual_seed(seed)
    B, L, d = spec.batch, spec.seq_len, spec.head_dim
    bf16 = torch.bfloat16

    def randn(*shape):
        return torch.randn(*shape, generator=gen, device=dev, dtype=torch.float32).to(bf16)

    q = randn(B, spec.h_q, d)
    k_cache = randn(B, spec.h_k, L, d)
    v_cache = randn(B, spec.h_v, L, spec.d_v)
    if spec.ragged is not None:
        lo, hi = spec.ragged
        seq_lens = torch.randint(lo, hi + 1, (B,), generator=gen, device=dev,
                                 dtype=torch.int64).to(torch.int32)
    else:
        seq_lens = torch.full((B,), L, dtype=torch.int32, device=dev)

    planted = []
    g = spec.g
    lens_host = seq_lens.tolist()
    q_f = q.float()
    for b in range(B):
        L_b = lens_host[b]
        for kh in range(spec.h_k):
            if spec.planted_per_query_head:
                count = spec.planted_per_query_head * g
            else:
                count = int(round(spec.planted_frac * L_b))
            count = min(count, L_b)
            if count == 0:
                continue
            pos = torch.randperm(L_b, generator=gen, device=dev)[:count]
            heads = kh * g + (torch.arange(count, device=dev) % g)
            lo, hi = spec.plant_scale
            if lo == hi:
                s = torch.full((count,), lo, device=dev)
            else:
                s = lo + (hi - lo) * torch.rand(count, generator=gen, device=dev)
            k_cache[b, kh, pos] = (s[:, None] * q_f[b, heads]).to(bf16)
            planted.extend((b, int(j), int(p)) for j, p in zip(heads.tolist(), pos.tolist()))
    return DecodeInputs(q, k_cache, v_cache, seq_lens, planted)


def scaled(spec: DecodeSpec, **changes) -> DecodeSpec:
    """A copy of ``spec`` with some fields changed (smaller parity cases)."""
    return replace(spec, **changes)
