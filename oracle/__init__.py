"""CPU oracle for the SAGA + Atop-N decode step (test infrastructure only).

Only tests, the smoke check and the bench's CPU-baseline / reference legs may
import this package; the CUDA path never does.
"""
from .saga_oracle import (head_maps, scores, top_n, nth_score, softmax_selected,
                          gathered_pv, decode_row, decode_attn, combine)

__all__ = ["head_maps", "scores", "top_n", "nth_score", "softmax_selected",
           "gathered_pv", "decode_row", "decode_attn", "combine"]
