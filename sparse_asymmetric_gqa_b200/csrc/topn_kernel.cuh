// topn_kernel.cuh -- S2, the exact top-N of each (batch row b, query head j)
// from the candidates that the score pass kept for it.
//
// Atop-N ("More Value per Key", §3.1 and App. C.1) keeps the scores at or
// above a threshold, found by a plain compare while the scores are produced;
// top-N itself is §2.5 Eq. (6).  The score pass (score_kernel in candidate
// mode) kept every score >= t_lo, t_lo a lower bound for the N-th score from
// a sample of the row's scores: per 32-position chunk c of the row a mask of
// the passing positions, and their order-preserving keys in position order at
// the row's slots [32c, 32c + popcount).  This kernel, one CTA per row,
// finishes the selection exactly:
//   1  the chunk masks give the candidate count C and each chunk's offset (a
//      block scan of popcounts);
//   2  if N_b <= C <= kTopnCap the list is gathered into shared memory, in
//      ascending position order (each thread copies the chunks of its run,
//      eight predicated loads per chunk in flight at once);
//   3  the N_b-th largest key T, and how many of the keys equal to T belong to
//      the top N_b, come from an MSB-first radix select over key - min key,
//      its first 11-bit digit aligned to the top of the keys' actual range
//      (candidate keys share their high bits: digits of the raw key would
//      pile them into a few bins);
//   4  one ordered pass keeps every key > T and the lowest-position keys = T
//      that are needed (block scans of tie and keep counts give each kept
//      entry its output slot), so positions come out ascending with no sort.
// The list is complete whenever C >= N_b: every score >= T is >= t_lo.  A
// list longer than kTopnCap is selected the same way straight from the slots
// in global memory; a list shorter than N_b (the sampled bound missed) has the
// row scored again here on CUDA cores and selected from all its positions.
// Both set INFO_ROBUST_PATH in the status word.  Keys are order-preserving
// uint32 images of the fp32 scores, -0 folded onto +0; ties at the N-th score
// go to the lowest position.  NaN scores are not supported.
#pragma once

#include <cuda_bf16.h>
#include "ptx.cuh"

namespace saga {

constexpr int kTopnThreads = 512;
constexpr int kTopnWarps = kTopnThreads / 32;
constexpr int kTopnCap = 8192;                    // candidates held in shared memory
constexpr int kTopnBins = 2048;                   // 11-bit radix digits
constexpr int kTopnPer = 8;                       // entries per thread per step of the ordered pass
constexpr int kTopnStep = kTopnPer * kTopnThreads;
constexpr int kTopnMaxRun = 8;                    // chunks per thread on the shared-memory path

// Dynamic shared memory, in 32-bit words; every region starts on a 16-byte boundary.
constexpr int kTopnOffKey = 0;                                  // [kTopnCap] keys
constexpr int kTopnOffPos = kTopnOffKey + kTopnCap;             // [kTopnCap] positions
constexpr int kTopnOffHist = kTopnOffPos + kTopnCap;            // [kTopnBins]
constexpr int kTopnOffScan = kTopnOffHist + kTopnBins;          // [kTopnWarps]
constexpr int kTopnOffMisc = kTopnOffScan + kTopnWarps;         // [4]
constexpr int kTopnSmemWords = kTopnOffMisc + 4;
constexpr size_t kTopnSmemBytes = sizeof(uint32_t) * kTopnSmemWords;
static_assert(kTopnOffPos % 4 == 0 && kTopnOffHist % 4 == 0 && kTopnOffScan % 4 == 0 &&
              kTopnOffMisc % 4 == 0, "shared regions on 16-byte boundaries");

struct TopnParams {
  const uint32_t* cand_mask;    // [B*h_q][mask_stride] passing positions per 32-position chunk
  long long mask_stride;
  uint32_t* zkey;               // [B*h_q][z_stride] candidate keys at their chunk slots
  long long z_stride;
  uint32_t* gather_count;       // per-row counters of the gather kernel, reset here
  const int32_t* seq_lens;      // [B]
  int h_q, h_k, g, L_max, N;
  int32_t* sel_idx;             // [B*h_q][N]
  float* sel_logit;             // [B*h_q][N]
  // scoring a row again (fallback)
  const __nv_bfloat16* q;       // [B][h_q][D]
  const __nv_bfloat16* k_cache; // [B][h_k][L_max][D]
  float scale;
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
// was scored again).
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
// equal to it belong to the top n_b (requires 1 <= n_b <= valid entries).
// Radix select over d = key - kmin, MSB first, in digits of at most 11 bits,
// the first digit ending at the top bit of kmax - kmin.  Every thread returns
// the same values.
template <class Src>
__device__ uint32_t topn_radix(const Src& src, int n, uint32_t n_b, uint32_t* s_hist,
                               uint32_t* s_scan, uint32_t* s_misc, uint32_t* need) {
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
    top = shift;
    __syncthreads();                             // s_misc and s_hist are reused
  }
  *need = k;
  return kmin + prefix;
}

// The ordered pass: entries are visited in ascending position order, eight
// consecutive ones per thread per step; kept = key > T, or key == T among the
// first `need` such entries.  The k-th kept entry goes to output slot k.
template <class Src>
__device__ void topn_emit(const Src& src, int n, uint32_t T, uint32_t need, uint32_t n_b,
                          int32_t* idx_out, float* logit_out, uint32_t* s_scan) {
  uint32_t ties_before = 0u, kept_before = 0u;
  for (int base = 0; base < n && kept_before < n_b; base += kTopnStep) {   // uniform
    const int i0 = base + kTopnPer * threadIdx.x;
    uint32_t key[kTopnPer];
    bool val[kTopnPer];
    uint32_t n_eq = 0u;
#pragma unroll
    for (int e = 0; e < kTopnPer; ++e) {
      val[e] = src.get(i0 + e, key[e]);
      n_eq += (val[e] && key[e] == T) ? 1u : 0u;
    }
    uint32_t total_eq;
    uint32_t r = ties_before + topn_excl_scan(n_eq, s_scan, total_eq);
    bool keep[kTopnPer];
    uint32_t n_keep = 0u;
#pragma unroll
    for (int e = 0; e < kTopnPer; ++e) {
      const bool tie = val[e] && key[e] == T;
      keep[e] = val[e] && (key[e] > T || (tie && r < need));
      r += tie ? 1u : 0u;
      n_keep += keep[e] ? 1u : 0u;
    }
    uint32_t total_keep;
    uint32_t slot = kept_before + topn_excl_scan(n_keep, s_scan, total_keep);
#pragma unroll
    for (int e = 0; e < kTopnPer; ++e) {
      if (keep[e]) {
        if (slot < n_b) {
          idx_out[slot] = src.position(i0 + e);
          logit_out[slot] = key_to_float(key[e]);
        }
        ++slot;
      }
    }
    ties_before += total_eq;
    kept_before += total_keep;
  }
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

template <int D>
__global__ void __launch_bounds__(kTopnThreads, 2)
topn_kernel(const TopnParams p) {
  extern __shared__ __align__(16) uint32_t topn_smem[];
  uint32_t* s_key = topn_smem + kTopnOffKey;
  int32_t* s_pos = reinterpret_cast<int32_t*>(topn_smem + kTopnOffPos);
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
  if (tid == 0) p.gather_count[bj] = 0u;
  if (L < 1 || L > p.L_max) {
    if (tid == 0) atomicOr(p.status, 0x1 /* SAGA_STATUS_BAD_SEQ_LEN */);
    for (int r = tid; r < N; r += kTopnThreads) { idx_out[r] = -1; logit_out[r] = -INFINITY; }
    return;
  }
  const uint32_t n_b = static_cast<uint32_t>(N < L ? N : L);
  const uint32_t* mrow = p.cand_mask + static_cast<long long>(bj) * p.mask_stride;
  uint32_t* krow = p.zkey + static_cast<long long>(bj) * p.z_stride;
  const int nch = (L + 31) / 32;

  // ---- candidate count and each chunk run's offset: thread t owns chunks [c0, c1)
  const int cpt = (nch + kTopnThreads - 1) / kTopnThreads;
  const int c0 = min(nch, tid * cpt), c1 = min(nch, c0 + cpt);
  const bool fits = cpt <= kTopnMaxRun;
  uint32_t run_mask[kTopnMaxRun];
  uint32_t cnt = 0u;
#pragma unroll
  for (int u = 0; u < kTopnMaxRun; ++u) {
    run_mask[u] = (u < cpt && c0 + u < c1) ? __ldcg(mrow + c0 + u) : 0u;
    cnt += __popc(run_mask[u]);
  }
  if (!fits)
    for (int c = c0 + kTopnMaxRun; c < c1; ++c) cnt += __popc(__ldcg(mrow + c));
  uint32_t C;
  const uint32_t off = topn_excl_scan(cnt, s_scan, C);

  uint32_t need;
  if (C >= n_b && C <= static_cast<uint32_t>(kTopnCap) && fits) {
    // each chunk's keys are contiguous at its slots; copy them with the
    // positions of the mask bits (up to 8 loads in flight, the rest after)
    uint32_t o = off;
#pragma unroll
    for (int u = 0; u < kTopnMaxRun; ++u) {
      uint32_t m = run_mask[u];
      const int n_c = __popc(m);
      const uint32_t* ks = krow + (c0 + u) * 32;
      uint32_t kv[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) kv[e] = (e < n_c) ? __ldcg(ks + e) : 0u;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        if (e < n_c) {
          s_key[o + e] = kv[e];
          s_pos[o + e] = (c0 + u) * 32 + (__ffs(m) - 1);
          m &= m - 1u;
        }
      }
      for (int e = 8; e < n_c; ++e) {
        s_key[o + e] = __ldcg(ks + e);
        s_pos[o + e] = (c0 + u) * 32 + (__ffs(m) - 1);
        m &= m - 1u;
      }
      o += n_c;
    }
    __syncthreads();
    const TopnListSrc src{s_key, s_pos, static_cast<int>(C)};
    const uint32_t T = topn_radix(src, src.n, n_b, s_hist, s_scan, s_misc, &need);
    topn_emit(src, src.n, T, need, n_b, idx_out, logit_out, s_scan);
  } else {
    if (tid == 0) atomicOr(p.status, 0x200 /* SAGA_STATUS_INFO_ROBUST_PATH */);
    const bool all = C < n_b;                    // the bound missed: score the row again
    if (all) {
      __syncthreads();                           // every chunk mask was read
      const __nv_bfloat16* keys =
          p.k_cache + (static_cast<long long>(b) * p.h_k + j / p.g) * p.L_max * D;
      topn_rescore<D>(p.q + static_cast<long long>(bj) * D, keys, L, p.scale, krow);
      __syncthreads();                           // the row's keys are visible to the whole CTA
    }
    const TopnSlotSrc src{mrow, krow, all ? L : nch * 32, all};
    const uint32_t T = topn_radix(src, src.n, n_b, s_hist, s_scan, s_misc, &need);
    topn_emit(src, src.n, T, need, n_b, idx_out, logit_out, s_scan);
  }
  for (int r = static_cast<int>(n_b) + tid; r < N; r += kTopnThreads) { idx_out[r] = -1; logit_out[r] = -INFINITY; }
}

}  // namespace saga
