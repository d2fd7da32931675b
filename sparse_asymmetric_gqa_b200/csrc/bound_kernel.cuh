// bound_kernel.cuh -- a per-row lower bound t_lo for the N-th largest score,
// from a sample of the row, so that the score pass can keep only the scores
// >= t_lo as selection candidates (Atop-N's threshold compare, "More Value per
// Key", §3.1 and App. C.1, with a bound from a sample in place of the paper's
// threshold calibrated on earlier steps).
//
// Two small kernels ahead of the score pass, chained by programmatic dependent
// launch so that the score pass streams K meanwhile:
//   sample_kernel  the sample of a row of length L is 32 blocks of 32
//                  consecutive positions spread evenly over [0, L): 1024
//                  scores, computed on CUDA cores in fp32 (the bound needs no
//                  match with the tensor-core scores: the selector checks that
//                  its candidates are complete).  The query heads of one key
//                  head share the sampled keys: grid (b, kh) x kSampleParts,
//                  each CTA scoring 64 sampled key rows (four threads per row)
//                  for all g heads.  Shared memory holds only q (g x d fp32),
//                  so the CTAs fit beside the score pass.
//   bound_kernel   one warp per row: with r_s = N_b * 1024 / L, t_lo is the
//                  (r_s + 6 sqrt(r_s) + 8)-th largest sample rounded down to
//                  the 16 high bits of its order-preserving key (a relative
//                  step of 2^-7), built one bit at a time from warp-wide counts
//                  of the samples at or above the trial key.
// The number of samples above the true N_b-th score has mean r_s, so the bound
// lies below it unless that count exceeds its mean by about six standard
// deviations.  Rows that the selector takes whole get t_lo = -inf.
//
// The bound kernel also writes m_ref, the largest sampled score of the row
// (+inf for rows without a sample): the reference that the score pass
// subtracts before it sums exp(z) over the row for the log-sum-exp of the
// calibrated threshold (App. C.1 takes the largest score of a tail of the row;
// the reference cancels from the threshold, it only keeps the sum in range).
#pragma once

#include <cuda_bf16.h>
#include "ptx.cuh"

namespace saga {

constexpr int kSampleThreads = 256;
constexpr int kSampleSize = 1024;                 // 32 blocks of 32 positions per row
constexpr int kSampleParts = 16;                  // CTAs per (b, kh)
constexpr int kSamplePartPos = kSampleSize / kSampleParts;     // 64 sampled positions per CTA
constexpr int kSampleSplit = kSampleThreads / kSamplePartPos;  // threads per sampled position

struct BoundParams {
  const __nv_bfloat16* q;        // [B][h_q][D]
  const __nv_bfloat16* k_cache;  // [B][h_k][L_max][D]
  const int32_t* seq_lens;
  int h_q, h_k, g, L_max, N, cand_cap;
  float scale;
  float* samp;                   // [B*h_q][kSampleSize] scratch
  float* t_lo;                   // [B*h_q]
  float* m_ref;                  // [B*h_q] largest sampled score, or nullptr
};

// Rows whose candidates are every position (t_lo = -inf), or invalid rows.
__device__ __forceinline__ bool bound_takes_all(int L, const BoundParams& p) {
  return L < 1 || L > p.L_max || L <= p.cand_cap;
}

// Dynamic shared memory: g * D floats (q of the group), interleaved so that
// the kSampleSplit slices of one float4 step sit side by side (the four threads
// of a position read different banks): float4 ((jj * DS / 4 + c) * kSampleSplit
// + sl) holds q[jj][sl * DS + 4c, +4).
template <int D>
__global__ void __launch_bounds__(kSampleThreads)
sample_kernel(const BoundParams p) {
  constexpr int DS = D / kSampleSplit;            // elements of a key row per thread
  extern __shared__ __align__(16) float qs[];
  pdl_launch_dependents();                        // the bound kernel may be scheduled
  const int tid = threadIdx.x;
  const int bk = blockIdx.x;                      // b * h_k + kh
  const int part = blockIdx.y;
  const int b = bk / p.h_k, kh = bk % p.h_k;
  const int g = p.g;
  const int row0 = b * p.h_q + kh * g;            // first query-head row of this key head
  const int L = p.seq_lens[b];
  if (bound_takes_all(L, p)) return;
  for (int t = tid; t < g * D; t += kSampleThreads) {
    const int jj = t / D, d = t % D, sl = d / DS, w = d % DS;
    qs[((jj * (DS / 4) + w / 4) * kSampleSplit + sl) * 4 + (w & 3)] =
        __bfloat162float(p.q[static_cast<long long>(row0) * D + t]);
  }
  // thread t takes slice t % 4 of sampled position t / 4
  const int pi = tid / kSampleSplit, sl = tid % kSampleSplit;
  const int blk = part * (kSamplePartPos / 32) + (pi >> 5);   // block of 32 in [0, 32)
  const int lpb = L / 32;                                      // whole blocks in the row
  const int pos = 32 * ((blk * lpb) / 32) + (pi & 31);        // blk * lpb < 2^24
  const uint4* kr = reinterpret_cast<const uint4*>(
      p.k_cache + ((static_cast<long long>(b) * p.h_k + kh) * p.L_max + pos) * D + sl * DS);
  float kf[DS];
#pragma unroll
  for (int c = 0; c < DS / 8; ++c) {
    const uint4 raw = __ldg(kr + c);
    const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = __bfloat1622float2(h2[e]);
      kf[8 * c + 2 * e] = f.x;
      kf[8 * c + 2 * e + 1] = f.y;
    }
  }
  __syncthreads();                                // qs complete
#pragma unroll 2
  for (int jj = 0; jj < g; ++jj) {
    const float4* qv = reinterpret_cast<const float4*>(qs) + jj * (D / 4) + sl;
    float a0 = 0.0f, a1 = 0.0f, a2 = 0.0f, a3 = 0.0f;
#pragma unroll
    for (int c = 0; c < DS / 4; ++c) {
      const float4 x = qv[c * kSampleSplit];
      a0 = fmaf(kf[4 * c], x.x, a0);
      a1 = fmaf(kf[4 * c + 1], x.y, a1);
      a2 = fmaf(kf[4 * c + 2], x.z, a2);
      a3 = fmaf(kf[4 * c + 3], x.w, a3);
    }
    float acc = (a0 + a1) + (a2 + a3);
    acc += __shfl_xor_sync(0xffffffffu, acc, 1);
    acc += __shfl_xor_sync(0xffffffffu, acc, 2);
    if (sl == 0)
      p.samp[static_cast<long long>(row0 + jj) * kSampleSize + blk * 32 + (pi & 31)] = acc * p.scale;
  }
}

// One warp per row (b, j).
__global__ void __launch_bounds__(32)
bound_kernel(const BoundParams p) {
  pdl_launch_dependents();                        // the score pass may start streaming K now
  pdl_wait();                                     // the samples are complete
  const int lane = threadIdx.x;
  const int bj = blockIdx.x;
  const int L = p.seq_lens[bj / p.h_q];
  if (bound_takes_all(L, p)) {
    if (lane == 0) {
      p.t_lo[bj] = -INFINITY;
      if (p.m_ref) p.m_ref[bj] = INFINITY;
    }
    return;
  }
  const float* srow = p.samp + static_cast<long long>(bj) * kSampleSize;
  constexpr int kPer = kSampleSize / 32;
  uint32_t key[kPer];
  uint32_t kmax = 0u;
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    key[i] = ordered_key(__fadd_rn(__ldcg(srow + i * 32 + lane), 0.0f));
    kmax = max(kmax, key[i]);
    key[i] >>= 16;
  }
  if (p.m_ref) {
    kmax = __reduce_max_sync(0xffffffffu, kmax);
    if (lane == 0) p.m_ref[bj] = key_to_float(kmax);
  }
  const int n_b = p.N < L ? p.N : L;
  const float rs = static_cast<float>(n_b) * kSampleSize / static_cast<float>(L);
  const float rf = ceilf(rs + 6.0f * sqrtf(rs) + 8.0f);
  if (!(rf < static_cast<float>(kSampleSize))) {
    if (lane == 0) p.t_lo[bj] = -INFINITY;
    return;
  }
  const uint32_t r = static_cast<uint32_t>(rf);
  uint32_t T = 0u;                                // the largest 16-bit key with >= r samples at or above it
  for (int bit = 15; bit >= 0; --bit) {
    const uint32_t trial = T | (1u << bit);
    uint32_t n0 = 0u, n1 = 0u, n2 = 0u, n3 = 0u;
#pragma unroll
    for (int i = 0; i < kPer; i += 4) {
      n0 += key[i] >= trial ? 1u : 0u;
      n1 += key[i + 1] >= trial ? 1u : 0u;
      n2 += key[i + 2] >= trial ? 1u : 0u;
      n3 += key[i + 3] >= trial ? 1u : 0u;
    }
    if (__reduce_add_sync(0xffffffffu, (n0 + n1) + (n2 + n3)) >= r) T = trial;
  }
  if (lane == 0) p.t_lo[bj] = key_to_float(T << 16);
}

}  // namespace saga
