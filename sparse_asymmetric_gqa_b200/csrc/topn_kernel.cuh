// topn_kernel.cuh -- S2 to S4 of one (batch row b, query head j) from the
// candidates that the score pass kept for it: the exact top-N, the softmax
// over the selected logits and the gathered P.V, one CTA per row.
//
// Atop-N ("More Value per Key", §3.1 and App. C.1) keeps the scores at or
// above a threshold, found by a plain compare while the scores are produced;
// top-N itself is §2.5 Eq. (6), and S3/S4 are §3.1 Eq. (7).  The score pass
// kept every score >= t_lo, t_lo a lower bound for the N-th score from a
// sample of the row's scores: per 32-position chunk c of the row a mask of the
// passing positions, and their order-preserving keys in position order at the
// row's slots [32c, 32c + popcount).  This kernel:
//   1  the chunk masks give the candidate count C and each chunk's offset (a
//      block scan of popcounts);
//   2  if N_b <= C <= kTopnCap the list is gathered into shared memory, in
//      ascending position order; the first eight key slots of each chunk (one
//      32-byte sector) are loaded in the same round as the masks, so a row
//      costs one round of dependent loads (chunks with more than eight
//      candidates fetch the rest afterwards);
//   3  the N_b-th largest key T, and how many of the keys equal to T belong to
//      the top N_b, come from an MSB-first radix select over key - min key,
//      its first 11-bit digit aligned to the top of the keys' actual range
//      (candidate keys share their high bits: digits of the raw key would
//      pile them into a few bins); once the bin holding T has at most 32
//      keys, one warp ranks them directly;
//   4  one ordered pass keeps every key > T and the lowest-position keys = T
//      that are needed; one block scan of packed (greater, equal) counts gives
//      every kept entry its output slot, so positions come out ascending with
//      no sort; the selection goes to the caller's lists and to shared memory
//      with its softmax weight exp(z - z_max);
//   5  P.V: each warp gathers 32 selected value rows at a time (all loads in
//      flight before use), fp32 accumulation, a CTA-wide sum, one division by
//      the weight sum and one bf16 rounding.
// The list is complete whenever C >= N_b: every score >= T is >= t_lo.  A
// list longer than kTopnCap is selected the same way straight from the slots
// in global memory; a list shorter than N_b (the sampled bound missed) has the
// row scored again here on CUDA cores and selected from all its positions.
// Both set INFO_ROBUST_PATH in the status word.  Keys are order-preserving
// uint32 images of the fp32 scores, -0 folded onto +0; ties at the N-th score
// go to the lowest position.  NaN scores are not supported.
//
// Stateful Atop-N (App. C.1) adds two modes.  Both need the row's log-sum-exp:
// from the score pass's chunk sums of exp(z - m_ref), read in the same round
// as the masks (rows longer than the candidate cap), else from the complete
// candidate list.  Calibration runs steps 1-5 and writes log tau = z(T) -
// logsumexp.  A step replaces 3 and 4 by t = log tau + logsumexp and one
// ordered pass that keeps every key >= key(t), the first 2N in position order
// (one block scan per pass), then takes the softmax weights over the kept
// logits.  The step's candidates cover t whenever t >= t_lo (the bound is for
// the 2N-th score); otherwise, or when the chunk sums left the fp32 range, the
// row is scored again here and its log-sum-exp taken from those keys.
#pragma once

#include <cuda_bf16.h>
#include "ptx.cuh"

namespace saga {

constexpr int kTopnThreads = 256;
constexpr int kTopnWarps = kTopnThreads / 32;
constexpr int kTopnCap = 8192;                    // candidates held in shared memory
constexpr int kTopnSelMax = 4096;                 // widest selection list (2N of a step)
constexpr int kTopnSelNarrow = 2048;              // selection lists of the exact path (N)
constexpr int kTopnBins = 2048;                   // 11-bit radix digits
constexpr int kTopnBinsPer = kTopnBins / kTopnThreads;   // digits owned by a thread in a scan
constexpr int kTopnPer = 16;                      // entries per thread per step of the ordered pass
constexpr int kTopnStep = kTopnPer * kTopnThreads;
constexpr int kTopnRound = 4;                     // chunks per thread per round of loads
constexpr int kTopnRun = 8;                       // chunks per thread on the shared-memory path (rows <= 65536)
constexpr int kTopnLongRun = 16;                  // the long-row variant (rows <= 131072)
constexpr int kTopnMaxD = 128;

// Dynamic shared memory, in 32-bit words, for candidate lists of up to kCap
// and selection lists of up to kSel entries; every region starts on a 16-byte
// boundary.  (90 KB for kSel = 2048: two CTAs per SM; the wide layout of a step
// with N > 1024 takes 106 KB.)
template <int kSel, int kCap = kTopnCap>
struct TopnLayout {
  static constexpr int kOffKey = 0;                             // [kCap] candidate keys
  static constexpr int kOffPos = kOffKey + kCap;                // [kCap] candidate positions
  static constexpr int kOffSelPos = kOffPos + kCap;             // [kSel] selected positions
  static constexpr int kOffSelW = kOffSelPos + kSel;            // [kSel] softmax weights
  static constexpr int kOffHist = kOffSelW + kSel;              // [kTopnBins]; P.V partials [warps][D]
  static constexpr int kOffScan = kOffHist + kTopnBins;         // [kTopnWarps]
  static constexpr int kOffMisc = kOffScan + kTopnWarps;        // [8]
  static constexpr int kWords = kOffMisc + 8;
  static constexpr size_t kBytes = sizeof(uint32_t) * kWords;
  static_assert(kOffPos % 4 == 0 && kOffSelPos % 4 == 0 && kOffSelW % 4 == 0 &&
                kOffHist % 4 == 0 && kOffScan % 4 == 0 && kOffMisc % 4 == 0,
                "shared regions on 16-byte boundaries");
};
static_assert(kTopnWarps * kTopnMaxD <= kTopnBins, "P.V partials fit the histogram region");

// What a call selects.  kModeExact: the top N.  kModeCalibrate: the top N, and
// log tau = z_(N_b) - logsumexp(z), the log-probability of the N_b-th largest
// score, per row.  kModeStep: every score z >= log tau + logsumexp(z) for the
// row's calibrated log tau, in ascending position order, the first cap = 2N
// kept ("More Value per Key", App. C.1).
enum TopnMode { kModeExact = 0, kModeCalibrate = 1, kModeStep = 2 };

struct TopnParams {
  const uint32_t* cand_mask;    // [B*h_q][mask_stride] passing positions per 32-position chunk
  long long mask_stride;
  uint32_t* zkey;               // [B*h_q][z_stride] candidate keys at their chunk slots
  long long z_stride;
  const int32_t* seq_lens;      // [B]
  int h_q, h_k, g, h_v, g_v, L_max, N;
  int cap;                      // width of a selection list row: N, or 2N in step mode
  int cand_cap;                 // rows with L <= cand_cap: every position is a candidate
  const float* lse_part;        // [B*h_q][mask_stride] chunk sums of exp(z - m_ref) (modes 1, 2)
  const float* m_ref;           // [B*h_q] their reference
  const float* t_lo;            // [B*h_q] the candidates' bound (step mode checks t >= t_lo)
  float* log_tau;               // [B*h_q] written by calibration, read by a step
  int32_t* sel_idx;             // [B*h_q][cap]
  float* sel_logit;             // [B*h_q][cap]
  const __nv_bfloat16* q;       // [B][h_q][DK] (scoring a row again, fallback)
  const __nv_bfloat16* k_cache; // [B][h_k][L_max][DK]
  const __nv_bfloat16* v_cache; // [B][h_v][L_max][D]
  float scale;
  __nv_bfloat16* out;           // [B*h_q][D]
  int* status;
};

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

// Index of the j-th lowest set bit of m (j < popcount(m)).
__device__ __forceinline__ int topn_nth_bit(uint32_t m, int j) {
  for (int c = 0; c < j; ++c) m &= m - 1u;
  return __ffs(m) - 1;
}

// The candidate list in shared memory, ascending positions.
struct TopnListSrc {
  const uint32_t* key;
  const int32_t* pos;
  int n;
  __device__ bool get(int i, uint32_t& k) const {
    if (i >= n) return false;
    k = key[i];
    return true;
  }
  __device__ int position(int i) const { return pos[i]; }
};

// The candidate slots of a row in global memory, s < n (n = 32 * chunks of
// the row; all: every s < n = L holds the key of position s, after the row
// was scored again by this CTA).
struct TopnSlotSrc {
  const uint32_t* mask;
  const uint32_t* zkey;
  int n;
  bool all;
  __device__ bool get(int s, uint32_t& k) const {
    if (s >= n) return false;
    if (!all && (s & 31) >= __popc(__ldcg(mask + (s >> 5)))) return false;
    k = all ? zkey[s] : __ldcg(zkey + s);   // rescored keys come from this CTA
    return true;
  }
  __device__ int position(int s) const { return all ? s : (s & ~31) + topn_nth_bit(__ldcg(mask + (s >> 5)), s & 31); }
};

// The n_b-th largest key of the n entries of src, and in *need how many keys
// equal to it belong to the top n_b (requires 1 <= n_b <= valid entries);
// *kmax is the largest key.  Radix select over d = key - kmin, MSB first, in
// digits of at most 11 bits, the first digit ending at the top bit of
// kmax - kmin.  Every thread returns the same values.
template <class Src>
__device__ uint32_t topn_radix(const Src& src, int n, uint32_t n_b, uint32_t* s_hist,
                               uint32_t* s_scan, uint32_t* s_misc, uint32_t* need, uint32_t* kmax_out) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  uint32_t lo = 0xFFFFFFFFu, hi = 0u;
  for (int i = tid; i < n; i += kTopnThreads) {
    uint32_t key;
    if (src.get(i, key)) { lo = min(lo, key); hi = max(hi, key); }
  }
  lo = __reduce_min_sync(0xffffffffu, lo);
  hi = __reduce_max_sync(0xffffffffu, hi);
  if (lane == 0) { s_hist[warp] = lo; s_hist[kTopnWarps + warp] = hi; }
  __syncthreads();
  uint32_t kmin = s_hist[0], kmax = s_hist[kTopnWarps];
#pragma unroll
  for (int w = 1; w < kTopnWarps; ++w) { kmin = min(kmin, s_hist[w]); kmax = max(kmax, s_hist[kTopnWarps + w]); }
  __syncthreads();                               // s_hist is reused below
  *kmax_out = kmax;
  const uint32_t range = kmax - kmin;
  uint32_t prefix = 0u, pmask = 0u, k = n_b;
  int top = 32 - __clz(range);                   // bits of d still to resolve
  while (top > 0) {                              // uniform: every thread has the same range
    const int nb = top < 11 ? top : 11;
    const int shift = top - nb;
    const uint32_t dmask = (1u << nb) - 1u;
    for (int i = tid; i < kTopnBins; i += kTopnThreads) s_hist[i] = 0u;
    __syncthreads();
    for (int i = tid; i < n; i += kTopnThreads) {
      uint32_t key;
      if (src.get(i, key)) {
        const uint32_t d = key - kmin;
        if ((d & pmask) == prefix) atomicAdd(&s_hist[(d >> shift) & dmask], 1u);
      }
    }
    __syncthreads();
    // thread t owns digits [8 (255 - t), +8): thread order runs over the digits top-down
    const int d0 = kTopnBinsPer * (kTopnThreads - 1 - tid);
    uint32_t h[kTopnBinsPer], c = 0u;
#pragma unroll
    for (int e = 0; e < kTopnBinsPer; ++e) { h[e] = s_hist[d0 + e]; c += h[e]; }
    uint32_t total;
    uint32_t above = topn_excl_scan(c, s_scan, total);
#pragma unroll
    for (int e = kTopnBinsPer - 1; e >= 0; --e) {
      if (above < k && above + h[e] >= k) {      // exactly one digit of the CTA satisfies this
        s_misc[0] = static_cast<uint32_t>(d0 + e);
        s_misc[1] = above;
        s_misc[2] = h[e];
      }
      above += h[e];
    }
    __syncthreads();
    const uint32_t digit = s_misc[0];
    k -= s_misc[1];
    const uint32_t in_bin = s_misc[2];
    prefix |= digit << shift;
    pmask |= dmask << shift;
    top = shift;
    __syncthreads();                             // s_misc and s_hist are reused
    if (top > 0 && in_bin <= 32u) {              // uniform: rank the bin's keys in one warp
      if (tid == 0) s_misc[3] = 0u;
      __syncthreads();
      for (int i = tid; i < n; i += kTopnThreads) {
        uint32_t key;
        if (src.get(i, key) && ((key - kmin) & pmask) == prefix) s_hist[atomicAdd(&s_misc[3], 1u)] = key;
      }
      __syncthreads();
      if (warp == 0) {
        const int has = lane < static_cast<int>(in_bin) ? 1 : 0;
        const uint32_t mine = has ? s_hist[lane] : 0u;
        uint32_t gt = 0u, ge = 0u;
        for (int m = 0; m < static_cast<int>(in_bin); ++m) {
          const uint32_t km = __shfl_sync(0xffffffffu, mine, m);
          gt += km > mine ? 1u : 0u;
          ge += km >= mine ? 1u : 0u;
        }
        if (has && gt < k && k <= ge) { s_misc[4] = mine; s_misc[5] = k - gt; }
      }
      __syncthreads();
      const uint32_t T = s_misc[4];
      *need = s_misc[5];
      __syncthreads();
      return T;
    }
  }
  *need = k;
  return kmin + prefix;
}

// The ordered pass: entries are visited in ascending position order, kTopnPer
// consecutive ones per thread per step; kept = key > T, or key == T among the
// first `need` such entries, so a kept entry's slot is (keys > T before it) +
// min(keys == T before it, need): one block scan of packed counts per step.
// Writes the caller's lists and the shared-memory selection with its softmax
// weight exp(z - zmax); returns this thread's sum of weights.
template <class Src>
__device__ float topn_emit(const Src& src, int n, uint32_t T, uint32_t need, uint32_t n_b,
                           float zmax, int32_t* idx_out, float* logit_out, int32_t* s_selpos,
                           float* s_selw, uint32_t* s_scan) {
  uint32_t gt_done = 0u, eq_done = 0u;           // counts of the earlier steps (uniform)
  float wsum = 0.0f;
  for (int base = 0; base < n && gt_done + min(eq_done, need) < n_b; base += kTopnStep) {
    const int i0 = base + kTopnPer * static_cast<int>(threadIdx.x);
    uint32_t key[kTopnPer];
    bool val[kTopnPer];
    uint32_t ngt = 0u, neq = 0u;
#pragma unroll
    for (int e = 0; e < kTopnPer; ++e) {
      val[e] = src.get(i0 + e, key[e]);
      ngt += (val[e] && key[e] > T) ? 1u : 0u;
      neq += (val[e] && key[e] == T) ? 1u : 0u;
    }
    uint32_t tot;
    const uint32_t pre = topn_excl_scan((ngt << 16) | neq, s_scan, tot);   // step totals < 2^16
    uint32_t gb = gt_done + (pre >> 16), qb = eq_done + (pre & 0xFFFFu);
#pragma unroll
    for (int e = 0; e < kTopnPer; ++e) {
      if (!val[e]) continue;
      const bool gtT = key[e] > T, eqT = key[e] == T;
      if (gtT || (eqT && qb < need)) {
        const uint32_t slot = gb + min(qb, need);
        if (slot < n_b) {
          const int pos = src.position(i0 + e);
          const float z = key_to_float(key[e]);
          const float w = expf(z - zmax);
          idx_out[slot] = pos;
          logit_out[slot] = z;
          s_selpos[slot] = pos;
          s_selw[slot] = w;
          wsum += w;
        }
      }
      gb += gtT ? 1u : 0u;
      qb += eqT ? 1u : 0u;
    }
    gt_done += tot >> 16;
    eq_done += tot & 0xFFFFu;
  }
  return wsum;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Block-wide sum and max, every thread the same result (a fixed order of operations).
__device__ __forceinline__ float topn_block_sum(float v, uint32_t* s_scan) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  float* s = reinterpret_cast<float*>(s_scan);
  v = warp_sum(v);
  if (lane == 0) s[warp] = v;
  __syncthreads();
  float t = 0.0f;
#pragma unroll
  for (int w = 0; w < kTopnWarps; ++w) t += s[w];
  __syncthreads();
  return t;
}
__device__ __forceinline__ uint32_t topn_block_max(uint32_t v, uint32_t* s_scan) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  v = __reduce_max_sync(0xffffffffu, v);
  if (lane == 0) s_scan[warp] = v;
  __syncthreads();
  uint32_t t = 0u;
#pragma unroll
  for (int w = 0; w < kTopnWarps; ++w) t = max(t, s_scan[w]);
  __syncthreads();
  return t;
}

// logsumexp of the n entries of src (a whole row): max, then the sum of exp(z - max).
template <class Src>
__device__ float topn_lse(const Src& src, int n, uint32_t* s_scan) {
  uint32_t hi = 0u;
  for (int i = threadIdx.x; i < n; i += kTopnThreads) {
    uint32_t key;
    if (src.get(i, key)) hi = max(hi, key);
  }
  const float m = key_to_float(topn_block_max(hi, s_scan));
  float sum = 0.0f;
  for (int i = threadIdx.x; i < n; i += kTopnThreads) {
    uint32_t key;
    if (src.get(i, key)) sum += expf(key_to_float(key) - m);
  }
  return m + logf(topn_block_sum(sum, s_scan));
}

// Step selection: every entry with key >= kt, visited in ascending position
// order, the first cap kept; a kept entry's slot is the count of passing
// entries before it (one block scan per step of kTopnStep entries).  Writes the
// caller's lists and, in shared memory, the positions and logits; returns how
// many entries were kept (every thread the same).
template <class Src>
__device__ uint32_t topn_emit_ge(const Src& src, int n, uint32_t kt, uint32_t cap, int32_t* idx_out,
                                 float* logit_out, int32_t* s_selpos, float* s_selz, uint32_t* s_scan) {
  uint32_t done = 0u;
  for (int base = 0; base < n && done < cap; base += kTopnStep) {
    const int i0 = base + kTopnPer * static_cast<int>(threadIdx.x);
    uint32_t key[kTopnPer];
    bool val[kTopnPer];
    uint32_t nge = 0u;
#pragma unroll
    for (int e = 0; e < kTopnPer; ++e) {
      val[e] = src.get(i0 + e, key[e]) && key[e] >= kt;
      nge += val[e] ? 1u : 0u;
    }
    uint32_t tot;
    uint32_t slot = done + topn_excl_scan(nge, s_scan, tot);
#pragma unroll
    for (int e = 0; e < kTopnPer; ++e) {
      if (!val[e]) continue;
      if (slot < cap) {
        const int pos = src.position(i0 + e);
        const float z = key_to_float(key[e]);
        idx_out[slot] = pos;
        logit_out[slot] = z;
        s_selpos[slot] = pos;
        s_selz[slot] = z;
      }
      ++slot;
    }
    done += tot;
  }
  return min(done, cap);
}

// Keys of one row scored on CUDA cores: key(fl(fl(q . k_i) * scale)), -0 -> +0.
template <int D>
__device__ void topn_rescore(const __nv_bfloat16* q, const __nv_bfloat16* keys, int L, float scale,
                             uint32_t* out) {
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
    out[i] = ordered_key(__fadd_rn(__fmul_rn(acc, scale), 0.0f));
  }
}

// kMode: a TopnMode; kSel: the layout's selection capacity (>= the list width p.cap).
// D: the value (and output) width; DK: the query and key width, used when a row
// is scored again ("More Value per Key" §5.2 lets keys be narrower than values).
// kRun: chunks per thread the shared-memory path takes (kTopnRun, or kTopnLongRun
// for caches of more than 65536 positions; the longer variant costs the short
// rows a few microseconds).
template <int D, int kMode, int kSel, int kRun = kTopnRun, int DK = D>
__global__ void __launch_bounds__(kTopnThreads, 2)
topn_kernel(const TopnParams p) {
  using Lay = TopnLayout<kSel>;
  extern __shared__ __align__(16) uint32_t topn_smem[];
  uint32_t* s_key = topn_smem + Lay::kOffKey;
  int32_t* s_pos = reinterpret_cast<int32_t*>(topn_smem + Lay::kOffPos);
  int32_t* s_selpos = reinterpret_cast<int32_t*>(topn_smem + Lay::kOffSelPos);
  float* s_selw = reinterpret_cast<float*>(topn_smem + Lay::kOffSelW);
  uint32_t* s_hist = topn_smem + Lay::kOffHist;
  float* s_part = reinterpret_cast<float*>(topn_smem + Lay::kOffHist);   // after the selection
  uint32_t* s_scan = topn_smem + Lay::kOffScan;
  uint32_t* s_misc = topn_smem + Lay::kOffMisc;

  pdl_wait();                                    // the candidate lists are complete
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int bj = blockIdx.x;
  const int b = bj / p.h_q, j = bj % p.h_q;
  const int L = p.seq_lens[b];
  const int N = p.N;
  constexpr int mode = kMode;
  const int cap = p.cap;
  int32_t* idx_out = p.sel_idx + static_cast<long long>(bj) * cap;
  float* logit_out = p.sel_logit + static_cast<long long>(bj) * cap;
  __nv_bfloat16* orow = p.out + static_cast<long long>(bj) * D;
  if (L < 1 || L > p.L_max) {                    // invalid row: padding and a zero output
    if (tid == 0) {
      atomicOr(p.status, 0x1 /* SAGA_STATUS_BAD_SEQ_LEN */);
      if (mode == kModeCalibrate) p.log_tau[bj] = -INFINITY;
    }
    for (int r = tid; r < cap; r += kTopnThreads) { idx_out[r] = -1; logit_out[r] = -INFINITY; }
    for (int e = tid; e < D; e += kTopnThreads) orow[e] = __float2bfloat16_rn(0.0f);
    return;
  }
  const uint32_t* mrow = p.cand_mask + static_cast<long long>(bj) * p.mask_stride;
  uint32_t* krow = p.zkey + static_cast<long long>(bj) * p.z_stride;
  const int nch = (L + 31) / 32;
  // the row's log-sum-exp comes from the score pass's chunk sums when the row
  // has a sampled reference (L > cand_cap), else from its complete candidate list
  const bool sums = mode != kModeExact && L > p.cand_cap;
  const float* lrow = sums ? p.lse_part + static_cast<long long>(bj) * p.mask_stride : nullptr;

  // ---- candidate count and each chunk run's offset: thread t owns chunks [c0, c1);
  // the first round also loads the first key sector of its first kTopnRound chunks
  // (and the chunk sums)
  const int cpt = (nch + kTopnThreads - 1) / kTopnThreads;
  const int c0 = min(nch, tid * cpt), c1 = min(nch, c0 + cpt);
  const bool fits = cpt <= kRun;
  uint32_t run_mask[kRun];
  float run_sum[kRun];
  uint4 sec[kTopnRound][2];
#pragma unroll
  for (int u = 0; u < kRun; ++u) {
    run_mask[u] = (c0 + u < c1) ? __ldcg(mrow + c0 + u) : 0u;
    run_sum[u] = (sums && c0 + u < c1) ? __ldcg(lrow + c0 + u) : 0.0f;
  }
#pragma unroll
  for (int u = 0; u < kTopnRound; ++u) {
    const uint4* kp = reinterpret_cast<const uint4*>(krow + (c0 + u) * 32);
    sec[u][0] = (c0 + u < c1) ? __ldcg(kp) : make_uint4(0u, 0u, 0u, 0u);
    sec[u][1] = (c0 + u < c1) ? __ldcg(kp + 1) : make_uint4(0u, 0u, 0u, 0u);
  }
  uint32_t cnt = 0u;
  float lsum = 0.0f;
#pragma unroll
  for (int u = 0; u < kRun; ++u) { cnt += __popc(run_mask[u]); lsum += run_sum[u]; }
  if (!fits)
    for (int c = c0 + kRun; c < c1; ++c) {
      cnt += __popc(__ldcg(mrow + c));
      if (sums) lsum += __ldcg(lrow + c);
    }
  uint32_t C;
  const uint32_t off = topn_excl_scan(cnt, s_scan, C);
  float lse = 0.0f;
  bool lse_ok = false;
  if (sums) {
    const float S = topn_block_sum(lsum, s_scan);
    const float mref = __ldcg(p.m_ref + bj);
    lse_ok = S > 0.0f && S <= 3.402823466e38f && mref > -INFINITY && mref < INFINITY;
    lse = mref + logf(S);
  }

  // Each chunk's keys are contiguous at its slots, in position order: write
  // them to shared memory with the positions of the mask bits.
  auto gather_list = [&]() {
    uint32_t o = off;
#pragma unroll
    for (int u0 = 0; u0 < kRun; u0 += kTopnRound) {
      if (u0 >= cpt) break;                      // uniform
      if (u0 > 0) {                              // rows longer than kTopnRound chunks per thread
#pragma unroll
        for (int u = 0; u < kTopnRound; ++u) {
          const uint4* kp = reinterpret_cast<const uint4*>(krow + (c0 + u0 + u) * 32);
          const bool live = c0 + u0 + u < c1;
          sec[u][0] = live ? __ldcg(kp) : make_uint4(0u, 0u, 0u, 0u);
          sec[u][1] = live ? __ldcg(kp + 1) : make_uint4(0u, 0u, 0u, 0u);
        }
      }
#pragma unroll
      for (int u = 0; u < kTopnRound; ++u) {
        uint32_t m = run_mask[u0 + u];
        const int n_c = __popc(m);
        const int cb = (c0 + u0 + u) * 32;
        const uint32_t kk[8] = {sec[u][0].x, sec[u][0].y, sec[u][0].z, sec[u][0].w,
                                sec[u][1].x, sec[u][1].y, sec[u][1].z, sec[u][1].w};
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          if (e < n_c) {
            s_key[o + e] = kk[e];
            s_pos[o + e] = cb + (__ffs(m) - 1);
            m &= m - 1u;
          }
        }
        for (int e = 8; e < n_c; ++e) {          // rare: more than eight candidates in a chunk
          s_key[o + e] = __ldcg(krow + cb + e);
          s_pos[o + e] = cb + (__ffs(m) - 1);
          m &= m - 1u;
        }
        o += n_c;
      }
    }
    __syncthreads();
  };
  // The row scored again on CUDA cores (the candidates do not cover what is selected).
  auto rescore = [&]() {
    if (tid == 0) atomicOr(p.status, 0x200 /* SAGA_STATUS_INFO_ROBUST_PATH */);
    const __nv_bfloat16* keys =
        p.k_cache + (static_cast<long long>(b) * p.h_k + j / p.g) * p.L_max * DK;
    topn_rescore<DK>(p.q + static_cast<long long>(bj) * DK, keys, L, p.scale, krow);
    __syncthreads();                             // the row's keys are visible to the whole CTA
  };

  uint32_t n_out;                                // entries of the selection
  float wsum = 0.0f;
  if (mode != kModeStep) {
    const uint32_t n_b = static_cast<uint32_t>(N < L ? N : L);
    uint32_t need, kmax, T;
    const bool all = C < n_b || (sums && !lse_ok);
    if (!all && C <= static_cast<uint32_t>(kTopnCap) && fits) {
      gather_list();
      const TopnListSrc src{s_key, s_pos, static_cast<int>(C)};
      T = topn_radix(src, src.n, n_b, s_hist, s_scan, s_misc, &need, &kmax);
      wsum = topn_emit(src, src.n, T, need, n_b, key_to_float(kmax), idx_out, logit_out, s_selpos,
                       s_selw, s_scan);
      if (mode == kModeCalibrate && !sums) lse = topn_lse(src, src.n, s_scan);
    } else {
      // a list longer than kTopnCap is selected from the slots in global memory;
      // a list shorter than N_b (the sampled bound missed) has the row scored again
      if (all) rescore();
      else if (tid == 0) atomicOr(p.status, 0x200 /* SAGA_STATUS_INFO_ROBUST_PATH */);
      const TopnSlotSrc src{mrow, krow, all ? L : nch * 32, all};
      T = topn_radix(src, src.n, n_b, s_hist, s_scan, s_misc, &need, &kmax);
      wsum = topn_emit(src, src.n, T, need, n_b, key_to_float(kmax), idx_out, logit_out, s_selpos,
                       s_selw, s_scan);
      if (mode == kModeCalibrate && !(sums && lse_ok)) lse = topn_lse(src, src.n, s_scan);
    }
    if (mode == kModeCalibrate && tid == 0) p.log_tau[bj] = key_to_float(T) - lse;
    n_out = n_b;
  } else {
    float lt = __ldcg(p.log_tau + bj);
    if (lt != lt) lt = -INFINITY;                // NaN: no threshold
    float t = lt + lse;
    const bool miss = sums && (!lse_ok || !(t >= __ldcg(p.t_lo + bj)));
    auto threshold_key = [&]() { return ordered_key(__fadd_rn(t, 0.0f)); };
    if (!miss && C <= static_cast<uint32_t>(kTopnCap) && fits) {
      gather_list();
      const TopnListSrc src{s_key, s_pos, static_cast<int>(C)};
      if (!sums) t = lt + topn_lse(src, src.n, s_scan);
      n_out = topn_emit_ge(src, src.n, threshold_key(), static_cast<uint32_t>(cap), idx_out,
                           logit_out, s_selpos, s_selw, s_scan);
    } else {
      if (miss) rescore();
      else if (tid == 0) atomicOr(p.status, 0x200 /* SAGA_STATUS_INFO_ROBUST_PATH */);
      const TopnSlotSrc src{mrow, krow, miss ? L : nch * 32, miss};
      if (!sums || !lse_ok) t = lt + topn_lse(src, src.n, s_scan);
      n_out = topn_emit_ge(src, src.n, threshold_key(), static_cast<uint32_t>(cap), idx_out,
                           logit_out, s_selpos, s_selw, s_scan);
    }
    // softmax weights exp(z - max) over the kept logits, in place of them
    __syncthreads();
    uint32_t hi = 0u;
    for (uint32_t i = tid; i < n_out; i += kTopnThreads) hi = max(hi, ordered_key(s_selw[i]));
    const float zmax = key_to_float(topn_block_max(hi, s_scan));
    for (uint32_t i = tid; i < n_out; i += kTopnThreads) {
      const float w = expf(s_selw[i] - zmax);
      s_selw[i] = w;
      wsum += w;
    }
  }
  for (int r = static_cast<int>(n_out) + tid; r < cap; r += kTopnThreads) {
    idx_out[r] = -1;
    logit_out[r] = -INFINITY;
  }

  // ---- softmax denominator
  wsum = warp_sum(wsum);
  if (lane == 0) reinterpret_cast<float*>(s_scan)[warp] = wsum;
  __syncthreads();                               // also: the selection in shared memory is complete
  float wtot = 0.0f;
#pragma unroll
  for (int w = 0; w < kTopnWarps; ++w) wtot += reinterpret_cast<const float*>(s_scan)[w];

  // ---- P.V: warp w gathers slots [32 (w + 8k), +32), all 32 row loads in flight before use
  constexpr int EPL = D / 32;                    // elements per lane: 2 or 4
  const __nv_bfloat16* vbase = p.v_cache +
      (static_cast<long long>(b) * p.h_v + j / p.g_v) * p.L_max * D + lane * EPL;
  float acc[EPL];
#pragma unroll
  for (int e = 0; e < EPL; ++e) acc[e] = 0.0f;
  for (int g0 = warp * 32; g0 < static_cast<int>(n_out); g0 += kTopnWarps * 32) {
    if constexpr (EPL == 4) {
      uint2 raw[32];
#pragma unroll
      for (int u = 0; u < 32; ++u) {
        const int sl = g0 + u;
        raw[u] = sl < static_cast<int>(n_out)
                     ? __ldg(reinterpret_cast<const uint2*>(vbase + static_cast<long long>(s_selpos[sl]) * D))
                     : make_uint2(0u, 0u);
      }
#pragma unroll
      for (int u = 0; u < 32; ++u) {
        const int sl = g0 + u;
        const float wu = sl < static_cast<int>(n_out) ? s_selw[sl] : 0.0f;
        const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw[u].x));
        const float2 c = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw[u].y));
        acc[0] = fmaf(wu, a.x, acc[0]);
        acc[1] = fmaf(wu, a.y, acc[1]);
        acc[2] = fmaf(wu, c.x, acc[2]);
        acc[3] = fmaf(wu, c.y, acc[3]);
      }
    } else {
      uint32_t raw[32];
#pragma unroll
      for (int u = 0; u < 32; ++u) {
        const int sl = g0 + u;
        raw[u] = sl < static_cast<int>(n_out)
                     ? __ldg(reinterpret_cast<const uint32_t*>(vbase + static_cast<long long>(s_selpos[sl]) * D))
                     : 0u;
      }
#pragma unroll
      for (int u = 0; u < 32; ++u) {
        const int sl = g0 + u;
        const float wu = sl < static_cast<int>(n_out) ? s_selw[sl] : 0.0f;
        const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw[u]));
        acc[0] = fmaf(wu, a.x, acc[0]);
        acc[1] = fmaf(wu, a.y, acc[1]);
      }
    }
  }
#pragma unroll
  for (int e = 0; e < EPL; ++e) s_part[warp * D + lane * EPL + e] = acc[e];
  __syncthreads();
  if (tid < D) {
    float a = 0.0f;
#pragma unroll
    for (int w = 0; w < kTopnWarps; ++w) a += s_part[w * D + tid];
    orow[tid] = __float2bfloat16_rn(wtot > 0.0f ? a / wtot : 0.0f);
  }
}

}  // namespace saga
