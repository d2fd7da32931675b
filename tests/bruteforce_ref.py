"""Pure-Python brute force of top-N sparse attention, for tiny inputs only.

Written independently of ``oracle/`` (plain loops, Python floats, a full sort
with an explicit (score descending, index ascending) key) so that it can pin the
oracle: "More Value per Key: Asymmetric Sparse Attention for Faster LLM
Decoding", §2.1 Eq. (2), §2.5 Eq. (6), §3.1 Eq. (7).
"""
import math


def brute_row(q_j, keys, values, N):
    """q_j: list[d]; keys, values: list[L][d]. Returns (out, idx, z_sel)."""
    d = len(q_j)
    L = len(keys)
    z = []
    for i in range(L):
        acc = 0.0
        for t in range(d):
            acc += float(q_j[t]) * float(keys[i][t])
        z.append(acc / math.sqrt(d))
    ranked = sorted(range(L), key=lambda i: (-z[i], i))
    chosen = sorted(ranked[:min(N, L)])
    zmax = max(z[i] for i in chosen)
    w = [math.exp(z[i] - zmax) for i in chosen]
    tot = sum(w)
    out = [0.0] * len(values[0])
    for wi, i in zip(w, chosen):
        for t in range(len(out)):
            out[t] += (wi / tot) * float(values[i][t])
    return out, chosen, [z[i] for i in chosen]
