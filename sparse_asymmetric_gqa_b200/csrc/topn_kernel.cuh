// topn_kernel.cuh -- S2, the exact top-N of each (batch row b, query head j)
// from the candidate list that the score pass built for it.
//
// Atop-N ("More Value per Key", §3.1 and App. C.1) keeps the scores at or
// above a threshold, found by a plain compare while the scores are produced;
// top-N itself is §2.5 Eq. (6).  The score pass (score_kernel in candidate
// mode) appended every (key, position) with score >= t_lo, t_lo a lower bound
// for the N-th score from a sample (threshold_kernel).  This kernel, one CTA
// per row, finishes the selection exactly:
//   1  the list (at most kTopnCap entries) is loaded into shared memory;
//   2  the N_b-th largest key T and the number of ties at T that belong to the
//      top N_b come from an MSB-first radix select, three passes of 11/11/10
//      bits over the keys in shared memory;
//   3  two bitmaps of the row mark the positions with key > T and key == T; a
//      block scan of the tie bitmap's word popcounts ranks the ties by
//      position, and the lowest-position ties that are needed join the kept
//      bitmap;
//   4  a block scan of the kept bitmap's word popcounts gives every kept
//      candidate its output slot (the number of kept positions before it), so
//      the list comes out in ascending position order without a sort.
// The list is complete whenever N_b <= C <= kTopnCap: every score >= T is >=
// t_lo, and none was dropped.  Otherwise (the bound was too high or too low,
// or the row is longer than the bitmaps) the row is scored again here on CUDA
// cores into the z scratch row, and the same radix select runs over it,
// followed by one ordered compare pass (INFO_ROBUST_PATH in the status word).
// Keys are order-preserving uint32 images of the fp32 scores, -0 folded onto
// +0; ties at the N-th score go to the lowest position.  NaN scores are not
// supported.
#pragma once

#include <cuda_bf16.h>
#include "ptx.cuh"

namespace saga {

constexpr int kTopnThreads = 512;
constexpr int kTopnWarps = kTopnThreads / 32;
constexpr int kTopnCap = 8192;                    // candidates per row held on chip
constexpr int kTopnMaxL = 131072;                 // longest row of the bitmap emission
constexpr int kTopnWords = kTopnMaxL / 32;        // words per bitmap
constexpr int kTopnBins = 2048;                   // 11-bit radix digits
constexpr int kTopnChunk = 4 * kTopnThreads;      // positions per step of the ordered pass

// Dynamic shared memory, in 32-bit words; every region starts on a 16-byte boundary.
constexpr int kTopnOffKey = 0;                                  // [kTopnCap] keys
constexpr int kTopnOffPos = kTopnOffKey + kTopnCap;             // [kTopnCap] positions
constexpr int kTopnOffGt = kTopnOffPos + kTopnCap;              // [kTopnWords] key > T, then kept
constexpr int kTopnOffEq = kTopnOffGt + kTopnWords;             // [kTopnWords] key == T, then slot base
constexpr int kTopnOffHist = kTopnOffEq + kTopnWords;           // [kTopnBins]
constexpr int kTopnOffScan = kTopnOffHist + kTopnBins;          // [kTopnWarps]
constexpr int kTopnOffMisc = kTopnOffScan + kTopnWarps;         // [4]
constexpr int kTopnSmemWords = kTopnOffMisc + 4;
constexpr size_t kTopnSmemBytes = sizeof(uint32_t) * kTopnSmemWords;
static_assert(kTopnOffPos % 4 == 0 && kTopnOffGt % 4 == 0 && kTopnOffEq % 4 == 0 &&
              kTopnOffHist % 4 == 0 && kTopnOffScan % 4 == 0 && kTopnOffMisc % 4 == 0,
              "shared regions on 16-byte boundaries");

struct TopnParams {
  const uint32_t* cand_key;     // [B*h_q][cand_cap] ordered keys
  const int32_t* cand_pos;      // [B*h_q][cand_cap] positions
  uint32_t* cand_count;         // [B*h_q] entries appended (may exceed cand_cap); reset here
  int cand_cap;
  uint32_t* gather_count;       // per-row counters of the gather kernel, reset here
  const int32_t* seq_lens;      // [B]
  int h_q, h_k, g, L_max, N;
  int32_t* sel_idx;             // [B*h_q][N]
  float* sel_logit;             // [B*h_q][N]
  // scoring a row again (fallback)
  const __nv_bfloat16* q;       // [B][h_q][D]
  const __nv_bfloat16* k_cache; // [B][h_k][L_max][D]
  float scale;
  float* z;                     // [B*h_q][z_stride] scratch
  long long z_stride;
  int* status;
};

// Canonical key of a score (-0 folded onto +0).
__device__ __forceinline__ uint32_t topn_key(float z) { return ordered_key(__fadd_rn(z, 0.0f)); }

// Exclusive scan of one value per thread across the CTA; total = the CTA sum.
__device__ __forceinline__ uint32_t topn_excl_scan(uint32_t v, uint32_t* s_scan, uint32_t& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) s_scan[warp] = x;
  __syncthreads();
  uint32_t before = 0, tot = 0;
#pragma unroll
  for (int w = 0; w < kTopnWarps; ++w) {
    const uint32_t s = s_scan[w];
    before += (w < warp) ? s : 0u;
    tot += s;
  }
  total = tot;
  __syncthreads();                               // s_scan is free again
  return before + x - v;
}

// The n_b-th largest of n keys (keys in shared memory when s_key is set,
// else the canonical keys of zrow[0, n)); *need = how many keys equal to the
// result belong to the top n_b.  Requires 1 <= n_b <= n.  Every thread returns
// the same values.
__device__ uint32_t topn_radix(const uint32_t* s_key, const float* zrow, int n, uint32_t n_b,
                               uint32_t* s_hist, uint32_t* s_scan, uint32_t* s_misc,
                               uint32_t* need) {
  const int tid = threadIdx.x;
  uint32_t prefix = 0u, pmask = 0u, k = n_b;
  for (int pass = 0; pass < 3; ++pass) {
    const int shift = (pass == 0) ? 21 : (pass == 1) ? 10 : 0;
    const uint32_t dmask = (pass == 2) ? 0x3FFu : 0x7FFu;
    for (int i = tid; i < kTopnBins; i += kTopnThreads) s_hist[i] = 0u;
    __syncthreads();
    for (int i = tid; i < n; i += kTopnThreads) {
      const uint32_t key = s_key ? s_key[i] : topn_key(zrow[i]);
      if ((key & pmask) == prefix) atomicAdd(&s_hist[(key >> shift) & dmask], 1u);
    }
    __syncthreads();
    // thread t owns digits [4 (511 - t), +4): thread order runs over the digits top-down
    const int d0 = 4 * (kTopnThreads - 1 - tid);
    const uint32_t h0 = s_hist[d0], h1 = s_hist[d0 + 1], h2 = s_hist[d0 + 2], h3 = s_hist[d0 + 3];
    uint32_t total;
    uint32_t above = topn_excl_scan(h0 + h1 + h2 + h3, s_scan, total);
    const uint32_t hs[4] = {h3, h2, h1, h0};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      if (above < k && above + hs[e] >= k) {     // exactly one digit of the CTA satisfies this
        s_misc[0] = static_cast<uint32_t>(d0 + 3 - e);
        s_misc[1] = above;
      }
      above += hs[e];
    }
    __syncthreads();
    const uint32_t digit = s_misc[0];
    k -= s_misc[1];
    prefix |= digit << shift;
    pmask |= dmask << shift;
    __syncthreads();                             // s_misc and s_hist are reused
  }
  *need = k;
  return prefix;
}

// The lowest m set bits of x (m <= 32).
__device__ __forceinline__ uint32_t topn_low_bits(uint32_t x, uint32_t m) {
  uint32_t r = 0u;
  for (uint32_t c = 0; c < m && x; ++c) {
    const uint32_t b = x & (0u - x);
    r |= b;
    x ^= b;
  }
  return r;
}

// Scores of one row on CUDA cores: z[i] = fl(fl(q . k_i) * scale), -0 -> +0.
template <int D>
__device__ void topn_rescore(const __nv_bfloat16* q, const __nv_bfloat16* keys, int L, float scale,
                             float* row) {
  const uint4* qv = reinterpret_cast<const uint4*>(q);
  for (int i = threadIdx.x; i < L; i += kTopnThreads) {
    const uint4* kv = reinterpret_cast<const uint4*>(keys + static_cast<long long>(i) * D);
    float acc = 0.0f;
#pragma unroll 4
    for (int c = 0; c < D / 8; ++c) {
      const uint4 a = __ldg(kv + c), b = __ldg(qv + c);
      const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&a);
      const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&b);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 x = __bfloat1622float2(a2[e]), y = __bfloat1622float2(b2[e]);
        acc = fmaf(x.x, y.x, acc);
        acc = fmaf(x.y, y.y, acc);
      }
    }
    row[i] = __fadd_rn(__fmul_rn(acc, scale), 0.0f);
  }
}

template <int D>
__global__ void __launch_bounds__(kTopnThreads, 2)
topn_kernel(const TopnParams p) {
  extern __shared__ __align__(16) uint32_t topn_smem[];
  uint32_t* s_key = topn_smem + kTopnOffKey;
  int32_t* s_pos = reinterpret_cast<int32_t*>(topn_smem + kTopnOffPos);
  uint32_t* s_gt = topn_smem + kTopnOffGt;
  uint32_t* s_eq = topn_smem + kTopnOffEq;
  uint32_t* s_hist = topn_smem + kTopnOffHist;
  uint32_t* s_scan = topn_smem + kTopnOffScan;
  uint32_t* s_misc = topn_smem + kTopnOffMisc;

  pdl_wait();                                    // the candidate lists are complete
  pdl_launch_dependents();                       // the gather kernel may be scheduled
  const int tid = threadIdx.x;
  const int bj = blockIdx.x;
  const int b = bj / p.h_q, j = bj % p.h_q;
  const int L = p.seq_lens[b];
  const int N = p.N;
  int32_t* idx_out = p.sel_idx + static_cast<long long>(bj) * N;
  float* logit_out = p.sel_logit + static_cast<long long>(bj) * N;
  const uint32_t C = p.cand_count[bj];
  __syncthreads();                               // every thread holds C before it is reset
  if (tid == 0) {
    p.cand_count[bj] = 0u;                       // ready for the next call
    p.gather_count[bj] = 0u;
  }
  if (L < 1 || L > p.L_max) {
    if (tid == 0) atomicOr(p.status, 0x1 /* SAGA_STATUS_BAD_SEQ_LEN */);
    for (int r = tid; r < N; r += kTopnThreads) { idx_out[r] = -1; logit_out[r] = -INFINITY; }
    return;
  }
  const int n_b = N < L ? N : L;
  const bool from_list = C >= static_cast<uint32_t>(n_b) && C <= static_cast<uint32_t>(p.cand_cap) &&
                         C <= static_cast<uint32_t>(kTopnCap) && L <= kTopnMaxL;
  if (from_list) {
    const int n = static_cast<int>(C);
    const long long o = static_cast<long long>(bj) * p.cand_cap;
    for (int i = tid; i < n; i += kTopnThreads) {
      s_key[i] = p.cand_key[o + i];
      s_pos[i] = p.cand_pos[o + i];
    }
    const int W = (L + 31) / 32;
    for (int w = tid; w < W; w += kTopnThreads) { s_gt[w] = 0u; s_eq[w] = 0u; }
    __syncthreads();
    uint32_t need;
    const uint32_t T = topn_radix(s_key, nullptr, n, static_cast<uint32_t>(n_b), s_hist, s_scan,
                                  s_misc, &need);
    bool bad = false;
    for (int i = tid; i < n; i += kTopnThreads) {
      const uint32_t key = s_key[i];
      const int pos = s_pos[i];
      if (pos < 0 || pos >= L) { bad = true; continue; }
      const uint32_t bit = 1u << (pos & 31);
      if (key > T) atomicOr(&s_gt[pos >> 5], bit);
      else if (key == T) atomicOr(&s_eq[pos >> 5], bit);
    }
    if (bad) atomicOr(p.status, 0x4 /* SAGA_STATUS_BAD_INDEX */);
    __syncthreads();
    // thread t owns the run of words [w0, w1)
    const int wpt = (W + kTopnThreads - 1) / kTopnThreads;
    const int w0 = min(W, tid * wpt), w1 = min(W, w0 + wpt);
    uint32_t ties = 0u;
    for (int w = w0; w < w1; ++w) ties += __popc(s_eq[w]);
    uint32_t total;
    uint32_t rank = topn_excl_scan(ties, s_scan, total);     // ties before this run
    uint32_t kept = 0u;
    for (int w = w0; w < w1; ++w) {
      const uint32_t e = s_eq[w];
      const uint32_t want = rank < need ? need - rank : 0u;
      const uint32_t km = s_gt[w] | topn_low_bits(e, want < 32u ? want : 32u);
      s_gt[w] = km;
      kept += __popc(km);
      rank += __popc(e);
    }
    uint32_t slot0 = topn_excl_scan(kept, s_scan, total);     // kept positions before this run
    for (int w = w0; w < w1; ++w) {
      s_eq[w] = slot0;
      slot0 += __popc(s_gt[w]);
    }
    __syncthreads();
    for (int i = tid; i < n; i += kTopnThreads) {
      const int pos = s_pos[i];
      if (pos < 0 || pos >= L) continue;
      const uint32_t word = s_gt[pos >> 5];
      const uint32_t bit = 1u << (pos & 31);
      if (word & bit) {
        const uint32_t slot = s_eq[pos >> 5] + __popc(word & (bit - 1u));
        if (slot < static_cast<uint32_t>(n_b)) {
          idx_out[slot] = pos;
          logit_out[slot] = key_to_float(s_key[i]);
        }
      }
    }
  } else {
    if (tid == 0) atomicOr(p.status, 0x200 /* SAGA_STATUS_INFO_ROBUST_PATH */);
    float* row = p.z + static_cast<long long>(bj) * p.z_stride;
    const __nv_bfloat16* keys =
        p.k_cache + (static_cast<long long>(b) * p.h_k + j / p.g) * p.L_max * D;
    topn_rescore<D>(p.q + static_cast<long long>(bj) * D, keys, L, p.scale, row);
    __syncthreads();                             // the row is visible to the whole CTA
    uint32_t need;
    const uint32_t T = topn_radix(nullptr, row, L, static_cast<uint32_t>(n_b), s_hist, s_scan,
                                  s_misc, &need);
    // ordered compare pass: thread t takes positions [base + 4t, base + 4t + 4)
    uint32_t ties_before = 0u, kept_before = 0u;
    for (int base = 0; base < L; base += kTopnChunk) {
      const int p0 = base + 4 * tid;
      uint32_t key[4];
      uint32_t n_eq = 0u;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        key[e] = (p0 + e < L) ? topn_key(row[p0 + e]) : 0u;
        n_eq += (p0 + e < L && key[e] == T) ? 1u : 0u;
      }
      uint32_t total_eq;
      uint32_t r = ties_before + topn_excl_scan(n_eq, s_scan, total_eq);
      bool keep[4];
      uint32_t n_keep = 0u;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const bool in = p0 + e < L;
        const bool tie = in && key[e] == T;
        keep[e] = in && (key[e] > T || (tie && r < need));
        r += tie ? 1u : 0u;
        n_keep += keep[e] ? 1u : 0u;
      }
      uint32_t total_keep;
      uint32_t slot = kept_before + topn_excl_scan(n_keep, s_scan, total_keep);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        if (keep[e]) {
          if (slot < static_cast<uint32_t>(n_b)) {
            idx_out[slot] = p0 + e;
            logit_out[slot] = key_to_float(key[e]);
          }
          ++slot;
        }
      }
      ties_before += total_eq;
      kept_before += total_keep;
    }
  }
  for (int r = n_b + tid; r < N; r += kTopnThreads) { idx_out[r] = -1; logit_out[r] = -INFINITY; }
}

}  // namespace saga
