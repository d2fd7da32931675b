"""A CPU model of the candidate bound (the sample and bound kernels' rule), checked
statistically: the bound must lie at or below the N_b-th score of a row (else the
selector has to score the row again) and keep the candidate list short.

The rule: 1024 sampled scores, 32 blocks of 32 consecutive positions starting at
32 * floor(blk * floor(L / 32) / 32); r_s = N_b * 1024 / L; the bound is the
ceil(r_s + 6 sqrt(r_s) + 8)-th largest sample, rounded down to the 16 high bits
of its order-preserving key.  Rows of at most 8192 positions take every
position instead.  This is a model of the kernels' design (not an oracle).
"""
import numpy as np
import pytest

CAP = 8192


def _key(x):
    b = np.asarray(x, dtype=np.float32).view(np.uint32)
    return np.where(b & 0x80000000, ~b, b | 0x80000000).astype(np.uint32)


def _unkey(k):
    k = np.asarray(k, dtype=np.uint32)
    b = np.where(k & 0x80000000, k & 0x7FFFFFFF, ~k).astype(np.uint32)
    return b.view(np.float32)


def sampled_positions(L):
    lpb = L // 32
    return np.array([32 * ((blk * lpb) // 32) + i for blk in range(32) for i in range(32)])


def bound(z, N):
    L = z.shape[0]
    if L <= CAP:
        return -np.inf
    n_b = min(N, L)
    rs = n_b * 1024.0 / L
    r = int(np.ceil(rs + 6.0 * np.sqrt(rs) + 8.0))
    if r >= 1024:
        return -np.inf
    s = np.sort(z[sampled_positions(L)].astype(np.float32))[::-1]
    k = (_key(s[r - 1]) >> 16) << 16
    return float(_unkey(k))


def _rows(kind, rng, L, n):
    if kind == "normal":
        return rng.normal(0, 1, (n, L))
    if kind == "planted":                     # 2% of positions far above the rest
        z = rng.normal(0, 1, (n, L))
        for r in range(n):
            z[r, rng.choice(L, L // 50, replace=False)] += rng.uniform(20, 45, L // 50)
        return z
    if kind == "heavy":                       # heavy-tailed scores
        return rng.standard_t(2, (n, L))
    if kind == "sorted":                      # scores rising along the row (recency bias)
        return np.sort(rng.normal(0, 1, (n, L)), axis=1) + rng.normal(0, 0.1, (n, L))
    raise ValueError(kind)


@pytest.mark.parametrize("kind", ["normal", "planted", "heavy", "sorted"])
@pytest.mark.parametrize("L,N", [(32768, 1024), (16384, 512), (131072, 2048), (9000, 64)])
def test_bound_is_below_the_nth_score_and_keeps_the_list_short(kind, L, N):
    rng = np.random.default_rng(L + N + len(kind))
    z = _rows(kind, rng, L, 40).astype(np.float32)
    for row in z:
        t = bound(row, N)
        c = int((row >= t).sum())
        n_b = min(N, L)
        assert c >= n_b, f"bound missed: {c} candidates for N_b = {n_b}"
        if kind != "sorted" and L <= 256 * 8 * 32:
            # expected count ~ (r_s + 6 sqrt(r_s) + 8) * L / 1024: within the shared-memory
            # list's cap wherever that list is used (rows of at most 8 chunks of 32
            # positions per thread; longer rows are selected from global memory)
            assert c <= CAP, f"{c} candidates exceed the list cap"


def test_a_planted_sample_makes_the_bound_miss():
    # the adversarial case the GPU test plants: the sampled positions hold the
    # top scores, everything else is low, and N is larger than the sample's
    # share -- the bound lands among the planted scores and misses
    L, N = 16384, 2048
    z = np.full(L, -1.0, dtype=np.float32)
    z[sampled_positions(L)] = 5.0
    t = bound(z, N)
    assert (z >= t).sum() < N
