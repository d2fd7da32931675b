// select_kernel.cuh -- S2, exact top-N selection of each (batch row b, query
// head j) score row, one CTA per row.
//
// Atop-N ("More Value per Key", §3.1 and App. C.1) keeps every score at or
// above a threshold by a plain per-element compare into a fixed-capacity
// buffer, the threshold being the N-th largest score; top-N itself is §2.5
// Eq. (6).  Here the threshold is exact and found on every call:
//   1  the row is streamed into shared memory by 1-D TMA bulk copies (a ring of
//      kRing x 16 KB, started at kernel entry);
//   2  meanwhile a lower bound t_lo for the N-th score comes from an evenly
//      spread sample of the row (up to 128 blocks of 32 scores): an
//      equal-width histogram of the sample and the lower edge of the bin below
//      the one holding its (r_s + 6 sqrt(r_s) + 8)-th largest value,
//      r_s = N * sample / L;
//   3  one compare pass (z >= t_lo) appends (key, position) of every passing
//      score to a candidate buffer of kCandCap entries;
//   4  the exact N-th key T among the candidates (equal-width histogram between
//      their min and max, the keys of the bin that holds the N-th, a one-warp
//      rank count or a radix select inside it);
//   5  the kept positions (key > T, and the lowest-position ties = T) are
//      marked in a bitmap of the row; a scan of the bitmap's word popcounts
//      gives each kept candidate its output slot, so positions come out
//      ascending without a sort.
// The result is exact whatever the sample says: if fewer than N_b scores pass
// t_lo, more than kCandCap do, or the row is longer than the bitmap, the
// robust path runs instead (histogram of the whole row over 2048 equal-width
// bins between its min and max, the keys of the boundary bin, a radix select
// inside it, one ordered compare pass).  The binning is monotone in z (a
// rounded subtract, a rounded multiply by a non-negative scale, clamp,
// truncate), so a higher bin always means a strictly larger score, for any
// min/max.  Very flat rows whose boundary bin overflows fall back to a radix
// select over the whole row.
// Keys are order-preserving uint32 images of the fp32 scores, -0 folded onto
// +0; ties at the N-th score go to the lowest position.  NaN scores are not
// supported.
#pragma once

#include <cuda_bf16.h>
#include "ptx.cuh"

namespace saga {

constexpr int kSelThreads = 512;
constexpr int kSelWarps = kSelThreads / 32;
constexpr int kBins = 2048;
constexpr int kCandCap = 4096;                  // candidate buffer (key, position)
constexpr int kBinKeys = 1024;                  // boundary-bin / tie scratch
constexpr int kSampleBlocks = 128;              // sample: up to 128 blocks of 32 scores
constexpr int kItems = 8;                       // scores per thread per chunk
constexpr int kChunk = kSelThreads * kItems;    // 4096 scores = one 16 KB ring buffer
constexpr int kRing = 3;                        // bulk-copy ring depth
constexpr int kMaxBitmapL = 131072;             // longest row of the bitmap emission

struct SelectParams {
  const float* z;               // [B*h_q][z_stride]
  long long z_stride;
  uint32_t* stat_min;           // ordered-key min/max per row, or nullptr
  uint32_t* stat_max;
  uint32_t* gather_count;       // per-row counters of the gather kernel (reset here), or nullptr
  const int32_t* seq_lens;
  int B, h_q, L_max, N;
  int z_vec4;                   // rows are 16-byte aligned (bulk copies allowed)
  int32_t* sel_idx;             // [B*h_q][N]
  float* sel_logit;
  int* status;
};

struct SelectSmem {
  union {
    float ring[kRing][kChunk];                  // compare-pass staging
    struct {
      uint32_t bits[kMaxBitmapL / 32];          // kept positions
      uint32_t wpre[kMaxBitmapL / 32];          // exclusive popcount prefix per word
    } bm;
  } a;
  union {
    uint32_t sample[kSampleBlocks * 32];
    struct {
      uint32_t key[kCandCap];
      int32_t pos[kCandCap];
    } c;
  } b;
  uint32_t hist[kBins];
  uint32_t bin_keys[kBinKeys];
  uint64_t full[kRing];
  uint32_t red[2 * kSelWarps];
  uint32_t scan[kSelWarps];
  uint32_t bcast[4];
  uint32_t cand_n;
  uint32_t tie_n;
};

// Canonical key of a score: -0 is folded onto +0 first.
__device__ __forceinline__ uint32_t score_key(float z) { return ordered_key(__fadd_rn(z, 0.0f)); }

__device__ __forceinline__ int lin_bin(float z, float lo, float scale) {
  float x = __fmul_rn(__fsub_rn(z, lo), scale);
  x = fminf(fmaxf(x, 0.0f), static_cast<float>(kBins - 1));
  return __float2int_rz(x);
}

// Exclusive scan across the block; *total receives the block sum.
__device__ __forceinline__ uint32_t block_excl_scan(uint32_t v, uint32_t* scan, uint32_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) scan[warp] = x;
  __syncthreads();
  if (warp == 0) {
    uint32_t w = lane < kSelWarps ? scan[lane] : 0u;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    if (lane < kSelWarps) scan[lane] = w;
  }
  __syncthreads();
  const uint32_t before = warp ? scan[warp - 1] : 0u;
  *total = scan[kSelWarps - 1];
  __syncthreads();
  return before + x - v;
}

// Block-wide min and max in one barrier round.
__device__ __forceinline__ void block_minmax(uint32_t& lo, uint32_t& hi, SelectSmem& sm) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  lo = __reduce_min_sync(0xffffffffu, lo);
  hi = __reduce_max_sync(0xffffffffu, hi);
  if (lane == 0) { sm.red[warp] = lo; sm.red[kSelWarps + warp] = hi; }
  __syncthreads();
  lo = sm.red[0];
  hi = sm.red[kSelWarps];
#pragma unroll
  for (int w = 1; w < kSelWarps; ++w) { lo = min(lo, sm.red[w]); hi = max(hi, sm.red[kSelWarps + w]); }
  __syncthreads();
}

// MSB-first radix select over a key set: visit(f) makes every thread call
// f(key) for its own share of the set.  Returns the k-th largest key T and,
// in *need, how many keys equal to T belong to the top k (k - #(key > T)).
template <class Visit>
__device__ uint32_t radix_select(Visit visit, uint32_t k, SelectSmem& sm, uint32_t* need) {
  uint32_t prefix = 0, mask = 0;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = threadIdx.x; i < 256; i += kSelThreads) sm.hist[i] = 0;
    __syncthreads();
    visit([&](uint32_t key) {
      if ((key & mask) == prefix) atomicAdd(&sm.hist[(key >> shift) & 255u], 1u);
    });
    __syncthreads();
    if (threadIdx.x < 32) {
      const int lane = threadIdx.x;
      // lane l owns digits [8*(31-l), 8*(31-l)+8): lane 0 holds the top digits
      const int d0 = 8 * (31 - lane);
      uint32_t c = 0;
#pragma unroll
      for (int e = 0; e < 8; ++e) c += sm.hist[d0 + e];
      uint32_t incl = c;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      uint32_t above = incl - c;             // keys in higher digits
      for (int e = 7; e >= 0; --e) {
        const uint32_t h = sm.hist[d0 + e];
        if (above < k && above + h >= k) { sm.bcast[0] = d0 + e; sm.bcast[1] = above; }
        above += h;
      }
    }
    __syncthreads();
    const uint32_t digit = sm.bcast[0];
    k -= sm.bcast[1];
    prefix |= digit << shift;
    mask |= 0xFFu << shift;
    __syncthreads();
  }
  *need = k;
  return prefix;
}

// k-th largest of a set of at most 32 keys held one per lane of warp 0:
// writes T to sm.bcast[0] and the ties needed to sm.bcast[1].
__device__ __forceinline__ void warp_kth(uint32_t key, bool has, uint32_t k, SelectSmem& sm) {
  uint32_t gt = 0, ge = 0;
  for (int m = 0; m < 32; ++m) {
    const uint32_t km = __shfl_sync(0xffffffffu, key, m);
    const bool hm = __shfl_sync(0xffffffffu, has, m);
    if (hm) { gt += km > key; ge += km >= key; }
  }
  if (has && gt < k && k <= ge) { sm.bcast[0] = key; sm.bcast[1] = k - gt; }
}

// k-th largest key of a shared-memory key set (visit as in radix_select):
// equal-width histogram between the set's min and max (rarely colliding
// atomics), the keys of the bin holding the k-th, then an exact finish there.
template <class Visit>
__device__ uint32_t kth_largest(Visit visit, uint32_t k, SelectSmem& sm, uint32_t* need) {
  const int tid = threadIdx.x;
  uint32_t lo_k = 0xFFFFFFFFu, hi_k = 0u;
  visit([&](uint32_t key) { lo_k = min(lo_k, key); hi_k = max(hi_k, key); });
  block_minmax(lo_k, hi_k, sm);
  if (lo_k == hi_k) { *need = k; return lo_k; }
  const float lo = key_to_float(lo_k), hi = key_to_float(hi_k);
  const float scale = static_cast<float>(kBins) / (hi - lo);
  if (!(scale < INFINITY) || !(scale > 0.0f)) return radix_select(visit, k, sm, need);

  for (int i = tid; i < kBins; i += kSelThreads) sm.hist[i] = 0;
  if (tid == 0) sm.cand_n = 0;
  __syncthreads();
  visit([&](uint32_t key) { atomicAdd(&sm.hist[lin_bin(key_to_float(key), lo, scale)], 1u); });
  __syncthreads();
  {
    const int b0 = 4 * (kSelThreads - 1 - tid);   // thread order runs over the bins top-down
    uint32_t c = 0;
#pragma unroll
    for (int e = 0; e < 4; ++e) c += sm.hist[b0 + e];
    uint32_t total;
    uint32_t above = block_excl_scan(c, sm.scan, &total);
    for (int e = 3; e >= 0; --e) {
      const uint32_t h = sm.hist[b0 + e];
      if (above < k && above + h >= k) { sm.bcast[0] = b0 + e; sm.bcast[1] = above; sm.bcast[2] = h; }
      above += h;
    }
  }
  __syncthreads();
  const int bstar = static_cast<int>(sm.bcast[0]);
  const uint32_t above = sm.bcast[1];
  const uint32_t in_bin = sm.bcast[2];
  const uint32_t k2 = k - above;
  __syncthreads();
  if (in_bin > static_cast<uint32_t>(kBinKeys)) return radix_select(visit, k, sm, need);
  visit([&](uint32_t key) {
    if (lin_bin(key_to_float(key), lo, scale) == bstar) sm.bin_keys[atomicAdd(&sm.cand_n, 1u)] = key;
  });
  __syncthreads();
  if (in_bin <= 32) {
    if (tid < 32) warp_kth(tid < static_cast<int>(in_bin) ? sm.bin_keys[tid] : 0u,
                           tid < static_cast<int>(in_bin), k2, sm);
    __syncthreads();
    const uint32_t T = sm.bcast[0];
    *need = sm.bcast[1];
    __syncthreads();
    return T;
  }
  return radix_select(
      [&](auto f) {
        for (int i = tid; i < static_cast<int>(in_bin); i += kSelThreads) f(sm.bin_keys[i]);
      },
      k2, sm, need);
}

// Eight consecutive scores starting at base; entries at or beyond `end` are
// returned as -inf and masked by the caller.
__device__ __forceinline__ void load8(const float* row, int base, int end, bool vec4, float (&v)[8]) {
  if (vec4 && base + 7 < end) {
    const float4 f0 = *reinterpret_cast<const float4*>(row + base);
    const float4 f1 = *reinterpret_cast<const float4*>(row + base + 4);
    v[0] = f0.x; v[1] = f0.y; v[2] = f0.z; v[3] = f0.w;
    v[4] = f1.x; v[5] = f1.y; v[6] = f1.z; v[7] = f1.w;
  } else {
#pragma unroll
    for (int e = 0; e < 8; ++e) v[e] = (base + e < end) ? row[base + e] : -INFINITY;
  }
}

// Lower bound (a score value) for the n_b-th largest score of a row of
// L > kChunk scores, from an evenly spread sample of blocks of 32 consecutive
// scores.  Any value is safe: the caller counts what passes it.
__device__ float sample_bound(const float* row, int L, int n_b, SelectSmem& sm) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nblk = min(kSampleBlocks, L / 32);
  const int S = nblk * 32;
  const int lpb = L / 32;                              // whole 32-score blocks in the row
  float v[kSampleBlocks / kSelWarps];
#pragma unroll
  for (int u = 0; u < kSampleBlocks / kSelWarps; ++u) {   // all loads in flight together
    const int blk = warp + u * kSelWarps;
    v[u] = blk < nblk ? row[32 * ((blk * lpb) / nblk) + lane] : 0.0f;   // blk*lpb < 2^26
  }
  uint32_t lo_k = 0xFFFFFFFFu, hi_k = 0u;
#pragma unroll
  for (int u = 0; u < kSampleBlocks / kSelWarps; ++u) {
    if (warp + u * kSelWarps < nblk) {
      const uint32_t k = score_key(v[u]);
      lo_k = min(lo_k, k);
      hi_k = max(hi_k, k);
    }
  }
  block_minmax(lo_k, hi_k, sm);
  const float lo = key_to_float(lo_k), hi = key_to_float(hi_k);
  if (!(hi > lo)) return lo;
  const float scale = static_cast<float>(kBins) / (hi - lo);
  if (!(scale < INFINITY)) return -INFINITY;
  for (int i = tid; i < kBins; i += kSelThreads) sm.hist[i] = 0;
  __syncthreads();
#pragma unroll
  for (int u = 0; u < kSampleBlocks / kSelWarps; ++u)
    if (warp + u * kSelWarps < nblk) atomicAdd(&sm.hist[lin_bin(v[u], lo, scale)], 1u);
  __syncthreads();
  const float rs = static_cast<float>(n_b) * static_cast<float>(S) / static_cast<float>(L);
  uint32_t r = static_cast<uint32_t>(ceilf(rs + 6.0f * sqrtf(rs) + 8.0f));
  if (r > static_cast<uint32_t>(S)) r = S;
  {
    const int b0 = 4 * (kSelThreads - 1 - tid);   // thread order runs over the bins top-down
    uint32_t c = 0;
#pragma unroll
    for (int e = 0; e < 4; ++e) c += sm.hist[b0 + e];
    uint32_t total;
    uint32_t above = block_excl_scan(c, sm.scan, &total);
    for (int e = 3; e >= 0; --e) {
      const uint32_t h = sm.hist[b0 + e];
      if (above < r && above + h >= r) sm.bcast[0] = b0 + e;
      above += h;
    }
  }
  __syncthreads();
  const int bstar = static_cast<int>(sm.bcast[0]);
  __syncthreads();
  return bstar >= 1 ? lo + static_cast<float>(bstar - 1) / scale : -INFINITY;
}

// One compare pass over the row: (key, position) of every score >= t_lo goes
// to the candidate buffer (warp-aggregated appends; entries past kCandCap are
// counted, not stored).  With bulk copies the row arrives chunk by chunk in a
// ring of shared-memory buffers.  Returns false if a wait timed out.
__device__ bool gather_candidates(const float* row, int L, bool bulk, float t_lo, SelectSmem& sm,
                                  int* status) {
  const int tid = threadIdx.x, lane = tid & 31;
  const int n_chunks = (L + kChunk - 1) / kChunk;
  volatile int never = 0;
  for (int c = 0; c < n_chunks; ++c) {
    const int s = c % kRing;
    const int c0 = c * kChunk;
    const int n_c = min(kChunk, L - c0);
    const int n_bulk = bulk ? (n_c & ~3) : 0;        // floats that arrived by bulk copy
    if (bulk) {
      const bool ok = mbar_wait(smem_addr(&sm.full[s]), (c / kRing) & 1, &never);
      if (__syncthreads_or(!ok)) {
        if (tid == 0) {
          atomicOr(status, 0x2 /* SAGA_STATUS_TIMEOUT */);
          // let the copies still in flight land (bounded) before the CTA exits
          for (int cc = c; cc < c + kRing && cc < n_chunks; ++cc)
            mbar_wait(smem_addr(&sm.full[cc % kRing]), (cc / kRing) & 1, &never);
        }
        __syncthreads();
        return false;
      }
    }
    const int o = tid * kItems;
    float v[8];
    if (o + 7 < n_bulk) {
      const float4 f0 = *reinterpret_cast<const float4*>(&sm.a.ring[s][o]);
      const float4 f1 = *reinterpret_cast<const float4*>(&sm.a.ring[s][o + 4]);
      v[0] = f0.x; v[1] = f0.y; v[2] = f0.z; v[3] = f0.w;
      v[4] = f1.x; v[5] = f1.y; v[6] = f1.z; v[7] = f1.w;
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const int oe = o + e;
        v[e] = oe < n_bulk ? sm.a.ring[s][oe] : (oe < n_c ? row[c0 + oe] : -INFINITY);
      }
    }
    uint32_t fl = 0;
#pragma unroll
    for (int e = 0; e < 8; ++e)
      if (o + e < n_c && v[e] >= t_lo) fl |= 1u << e;
    const uint32_t cnt = __popc(fl);
    uint32_t incl = cnt;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, incl, d);
      if (lane >= d) incl += y;
    }
    const uint32_t wsum = __shfl_sync(0xffffffffu, incl, 31);
    uint32_t base = 0;
    if (lane == 31 && wsum) base = atomicAdd(&sm.cand_n, wsum);
    base = __shfl_sync(0xffffffffu, base, 31);
    uint32_t w = base + incl - cnt;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      if ((fl >> e) & 1u) {
        if (w < static_cast<uint32_t>(kCandCap)) { sm.b.c.key[w] = score_key(v[e]); sm.b.c.pos[w] = c0 + o + e; }
        ++w;
      }
    }
    __syncthreads();                                   // ring buffer s is free again
    if (bulk && tid == 0 && c + kRing < n_chunks) {
      const int cn = c + kRing;
      const int nb = min(kChunk, L - cn * kChunk) & ~3;
      const uint32_t bar = smem_addr(&sm.full[s]);
      if (nb > 0) {
        mbar_arrive_expect_tx(bar, nb * 4);
        bulk_load(smem_addr(sm.a.ring[s]), row + cn * kChunk, nb * 4, bar);
      } else {
        mbar_arrive(bar);
      }
    }
  }
  __syncthreads();
  return true;
}

// Exact selection from the candidate buffer, which holds every score of the
// row that can be among the top n_b (C entries, in no order): the n_b-th
// largest key T; keys > T and the lowest-position ties are marked in a bitmap
// of the row, and each kept candidate writes itself at slot = number of kept
// positions before it.  Returns false (nothing written) if there were more
// ties at T than the tie scratch holds.
__device__ bool emit_from_candidates(int L, int n_b, int32_t* idx_out, float* logit_out,
                                     SelectSmem& sm) {
  const int tid = threadIdx.x;
  const int C = static_cast<int>(sm.cand_n);
  uint32_t need;
  const uint32_t T = kth_largest(
      [&](auto f) {
        for (int i = tid; i < C; i += kSelThreads) f(sm.b.c.key[i]);
      },
      static_cast<uint32_t>(n_b), sm, &need);
  const int W = (L + 31) / 32;
  for (int i = tid; i < W; i += kSelThreads) sm.a.bm.bits[i] = 0;
  if (tid == 0) sm.tie_n = 0;
  __syncthreads();
  for (int i = tid; i < C; i += kSelThreads) {
    const uint32_t key = sm.b.c.key[i];
    const int pos = sm.b.c.pos[i];
    if (key > T) {
      atomicOr(&sm.a.bm.bits[pos >> 5], 1u << (pos & 31));
    } else if (key == T) {
      const uint32_t t = atomicAdd(&sm.tie_n, 1u);
      if (t < static_cast<uint32_t>(kBinKeys)) sm.bin_keys[t] = static_cast<uint32_t>(pos);
    }
  }
  __syncthreads();
  const uint32_t n_tie = sm.tie_n;
  if (n_tie > static_cast<uint32_t>(kBinKeys)) return false;
  for (uint32_t t = tid; t < n_tie; t += kSelThreads) {
    const uint32_t pos = sm.bin_keys[t];
    bool keep = true;
    if (n_tie != need) {            // keep the `need` lowest positions among the ties
      uint32_t rank = 0;
      for (uint32_t u = 0; u < n_tie; ++u) rank += sm.bin_keys[u] < pos;
      keep = rank < need;
    }
    if (keep) atomicOr(&sm.a.bm.bits[pos >> 5], 1u << (pos & 31));
  }
  __syncthreads();
  // exclusive popcount prefix of the bitmap words (thread t owns a run of words)
  const int wpt = (W + kSelThreads - 1) / kSelThreads;
  const int w0 = tid * wpt, w1 = min(W, w0 + wpt);
  uint32_t cnt = 0;
  for (int w = w0; w < w1; ++w) cnt += __popc(sm.a.bm.bits[w]);
  uint32_t total;
  uint32_t run = block_excl_scan(cnt, sm.scan, &total);
  for (int w = w0; w < w1; ++w) {
    sm.a.bm.wpre[w] = run;
    run += __popc(sm.a.bm.bits[w]);
  }
  __syncthreads();
  for (int i = tid; i < C; i += kSelThreads) {
    const int pos = sm.b.c.pos[i];
    const uint32_t word = sm.a.bm.bits[pos >> 5];
    const uint32_t bit = 1u << (pos & 31);
    if (word & bit) {
      const uint32_t slot = sm.a.bm.wpre[pos >> 5] + __popc(word & (bit - 1u));
      idx_out[slot] = pos;
      logit_out[slot] = key_to_float(sm.b.c.key[i]);
    }
  }
  return true;
}

// Robust threshold: exact (T, ties needed) for the n_b-th largest score of the
// row via an equal-width histogram of the whole row between its min and max.
__device__ uint32_t robust_threshold(const float* row, int L, bool vec4, int n_b, uint32_t st_lo,
                                     uint32_t st_hi, bool have_stats, int* status, SelectSmem& sm,
                                     uint32_t* need_ties) {
  const int tid = threadIdx.x, lane = tid & 31;
  if (!have_stats || st_lo > st_hi) {
    uint32_t lo_k = 0xFFFFFFFFu, hi_k = 0u;
    for (int i = tid; i < L; i += kSelThreads) {
      const uint32_t key = score_key(row[i]);
      lo_k = min(lo_k, key);
      hi_k = max(hi_k, key);
    }
    block_minmax(lo_k, hi_k, sm);
    st_lo = lo_k;
    st_hi = hi_k;
  }
  const float lo = key_to_float(st_lo), hi = key_to_float(st_hi);
  float scale = (hi > lo) ? static_cast<float>(kBins) / (hi - lo) : 0.0f;
  if (!(scale < INFINITY)) scale = 0.0f;       // inf or NaN range: everything in bin 0

  // pass A: histogram over equal-width bins
  for (int i = tid; i < kBins; i += kSelThreads) sm.hist[i] = 0;
  if (tid == 0) sm.cand_n = 0;
  __syncthreads();
  const int n_chunks4 = (L + 4 * kSelThreads - 1) / (4 * kSelThreads);
  for (int c = 0; c < n_chunks4; ++c) {
    const int base = c * 4 * kSelThreads + tid * 4;
    if (vec4 && base + 3 < L) {
      const float4 v = *reinterpret_cast<const float4*>(row + base);
      atomicAdd(&sm.hist[lin_bin(v.x, lo, scale)], 1u);
      atomicAdd(&sm.hist[lin_bin(v.y, lo, scale)], 1u);
      atomicAdd(&sm.hist[lin_bin(v.z, lo, scale)], 1u);
      atomicAdd(&sm.hist[lin_bin(v.w, lo, scale)], 1u);
    } else {
      for (int e = 0; e < 4; ++e)
        if (base + e < L) atomicAdd(&sm.hist[lin_bin(row[base + e], lo, scale)], 1u);
    }
  }
  __syncthreads();

  // boundary bin: thread t owns bins [4*(511-t), +4), so thread order runs top-down
  {
    const int b0 = 4 * (kSelThreads - 1 - tid);
    uint32_t c = 0;
#pragma unroll
    for (int e = 0; e < 4; ++e) c += sm.hist[b0 + e];
    uint32_t total;
    uint32_t above = block_excl_scan(c, sm.scan, &total);
    for (int e = 3; e >= 0; --e) {
      const uint32_t h = sm.hist[b0 + e];
      if (above < static_cast<uint32_t>(n_b) && above + h >= static_cast<uint32_t>(n_b)) {
        sm.bcast[0] = b0 + e; sm.bcast[1] = above; sm.bcast[2] = h;
      }
      above += h;
    }
  }
  __syncthreads();
  const int bstar = static_cast<int>(sm.bcast[0]);
  const uint32_t above = sm.bcast[1];
  const uint32_t in_bin = sm.bcast[2];
  __syncthreads();

  if (in_bin <= static_cast<uint32_t>(kCandCap)) {
    // pass B: keys of the boundary bin
    for (int c = 0; c < n_chunks4; ++c) {
      const int base = c * 4 * kSelThreads + tid * 4;
      float v[4];
      if (vec4 && base + 3 < L) {
        const float4 f = *reinterpret_cast<const float4*>(row + base);
        v[0] = f.x; v[1] = f.y; v[2] = f.z; v[3] = f.w;
      } else {
        for (int e = 0; e < 4; ++e) v[e] = (base + e < L) ? row[base + e] : 0.0f;
      }
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const bool pred = (base + e < L) && lin_bin(v[e], lo, scale) == bstar;
        const uint32_t m = __ballot_sync(0xffffffffu, pred);
        if (m) {
          const int leader = __ffs(m) - 1;
          uint32_t slot = 0;
          if (lane == leader) slot = atomicAdd(&sm.cand_n, static_cast<uint32_t>(__popc(m)));
          slot = __shfl_sync(0xffffffffu, slot, leader);
          if (pred) sm.b.c.key[slot + __popc(m & ((1u << lane) - 1u))] = score_key(v[e]);
        }
      }
    }
    __syncthreads();
    const int n_cand = static_cast<int>(sm.cand_n);
    return radix_select(
        [&](auto f) {
          for (int i = tid; i < n_cand; i += kSelThreads) f(sm.b.c.key[i]);
        },
        static_cast<uint32_t>(n_b) - above, sm, need_ties);
  }
  // flat row: exact radix select over the whole row
  if (tid == 0) atomicOr(status, 0x100 /* SAGA_STATUS_INFO_EXACT_FALLBACK */);
  return radix_select(
      [&](auto f) {
        for (int i = tid; i < L; i += kSelThreads) f(score_key(row[i]));
      },
      static_cast<uint32_t>(n_b), sm, need_ties);
}

// Ordered compare pass: keep key > T and the first `need` ties, positions ascending.
__device__ void emit_by_threshold(const float* row, int L, bool vec4, uint32_t T, uint32_t need,
                                  int32_t* idx_out, float* logit_out, SelectSmem& sm) {
  const int tid = threadIdx.x;
  uint32_t run_gt = 0, run_tie = 0;
  const int n_chunks = (L + kChunk - 1) / kChunk;
  for (int c = 0; c < n_chunks; ++c) {
    const int base = c * kChunk + tid * kItems;
    float v[8];
    load8(row, base, L, vec4, v);
    uint32_t gt = 0, tie = 0;
#pragma unroll
    for (int e = 0; e < kItems; ++e) {
      if (base + e < L) {
        const uint32_t key = score_key(v[e]);
        if (key > T) gt |= 1u << e;
        else if (key == T) tie |= 1u << e;
      }
    }
    uint32_t total;
    const uint32_t excl = block_excl_scan((static_cast<uint32_t>(__popc(tie)) << 16) | __popc(gt),
                                          sm.scan, &total);
    uint32_t tr = run_tie + (excl >> 16);
    uint32_t w = run_gt + (excl & 0xFFFFu) + min(need, tr);
#pragma unroll
    for (int e = 0; e < kItems; ++e) {
      bool sel = (gt >> e) & 1u;
      if ((tie >> e) & 1u) { sel = tr < need; ++tr; }
      if (sel) {
        idx_out[w] = base + e;
        logit_out[w] = v[e];
        ++w;
      }
    }
    run_gt += total & 0xFFFFu;
    run_tie += total >> 16;
  }
}

__global__ void __launch_bounds__(kSelThreads, 2)
select_kernel(const SelectParams p) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  SelectSmem& sm = *reinterpret_cast<SelectSmem*>(smem_raw);
  const int tid = threadIdx.x;
  const int bj = blockIdx.x;
  const int b = bj / p.h_q;
  const int L = p.seq_lens[b];
  const int N = p.N;
  int32_t* idx_out = p.sel_idx + static_cast<long long>(bj) * N;
  float* logit_out = p.sel_logit + static_cast<long long>(bj) * N;
  const float* row = p.z + static_cast<long long>(bj) * p.z_stride;
  const bool vec4 = p.z_vec4 != 0;
  const bool valid = L >= 1 && L <= p.L_max;
  const int n_b = N < L ? N : L;
  // the fast path: candidates through shared memory, bitmap emission
  const bool fast = valid && n_b < L && L <= kMaxBitmapL && n_b <= kCandCap / 2;
  const bool bulk = fast && vec4;

  uint32_t st_lo = 0xFFFFFFFFu, st_hi = 0u;
  if (p.stat_min != nullptr) { st_lo = p.stat_min[bj]; st_hi = p.stat_max[bj]; }
  if (tid == 0) {
    sm.cand_n = 0;
    if (bulk) {                     // start streaming the row before anything else
      for (int s = 0; s < kRing; ++s) mbar_init(smem_addr(&sm.full[s]), 1);
      fence_mbar_init();
      const int n_chunks = (L + kChunk - 1) / kChunk;
      for (int c = 0; c < kRing && c < n_chunks; ++c) {
        const int nb = min(kChunk, L - c * kChunk) & ~3;
        const uint32_t bar = smem_addr(&sm.full[c]);
        if (nb > 0) {
          mbar_arrive_expect_tx(bar, nb * 4);
          bulk_load(smem_addr(sm.a.ring[c]), row + c * kChunk, nb * 4, bar);
        } else {
          mbar_arrive(bar);
        }
      }
    }
  }
  __syncthreads();
  if (tid == 0) {
    if (p.stat_min != nullptr) {   // leave the statistics ready for the next call
      p.stat_min[bj] = 0xFFFFFFFFu;
      p.stat_max[bj] = 0u;
    }
    if (p.gather_count != nullptr) p.gather_count[bj] = 0u;
  }

  if (!valid) {
    if (tid == 0) atomicOr(p.status, 0x1 /* SAGA_STATUS_BAD_SEQ_LEN */);
    for (int r = tid; r < N; r += kSelThreads) { idx_out[r] = -1; logit_out[r] = -INFINITY; }
    return;
  }

  if (n_b == L) {
    // every position is selected (dense softmax attention)
    for (int i = tid; i < L; i += kSelThreads) { idx_out[i] = i; logit_out[i] = row[i]; }
  } else {
    bool done = false;
    if (fast) {
      const float t_lo = (L <= kChunk) ? -INFINITY : sample_bound(row, L, n_b, sm);
      const bool ok = gather_candidates(row, L, bulk, t_lo, sm, p.status);
      if (!ok) return;                                   // timed out: status already set
      const uint32_t C = sm.cand_n;
      if (C >= static_cast<uint32_t>(n_b) && C <= static_cast<uint32_t>(kCandCap))
        done = emit_from_candidates(L, n_b, idx_out, logit_out, sm);
      __syncthreads();
    }
    if (!done) {
      if (tid == 0) atomicOr(p.status, 0x200 /* SAGA_STATUS_INFO_ROBUST_PATH */);
      uint32_t need;
      const uint32_t T = robust_threshold(row, L, vec4, n_b, st_lo, st_hi, p.stat_min != nullptr,
                                          p.status, sm, &need);
      emit_by_threshold(row, L, vec4, T, need, idx_out, logit_out, sm);
    }
  }
  for (int r = n_b + tid; r < N; r += kSelThreads) { idx_out[r] = -1; logit_out[r] = -INFINITY; }
}

}  // namespace saga
