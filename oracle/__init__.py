"""CPU oracle for the SAGA + Atop-N decode step (test infrastructure only).

Only tests, the smoke check and the bench's CPU-baseline / reference legs may
import this package; the CUDA path never does.
"""
from .saga_oracle import (head_maps, scores, top_n, nth_score, softmax_selected,
                          gathered_pv, decode_row, decode_attn, combine)
from .atopn_oracle import (calibrate_tau, tail_max, step_threshold, step_select,
                           step_row, calibrate_row, step_attn)
from .group_oracle import group_statistic, group_select, group_rows, group_attn

__all__ = ["head_maps", "scores", "top_n", "nth_score", "softmax_selected",
           "gathered_pv", "decode_row", "decode_attn", "combine",
           "calibrate_tau", "tail_max", "step_threshold", "step_select",
           "step_row", "calibrate_row", "step_attn",
           "group_statistic", "group_select", "group_rows", "group_attn"]
