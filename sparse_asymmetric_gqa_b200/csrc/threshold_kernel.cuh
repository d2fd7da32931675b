// threshold_kernel.cuh -- a per-row lower bound t_lo for the N-th largest
// score, from a sample of the row, so that the score pass can keep only the
// scores >= t_lo as selection candidates (Atop-N's threshold compare, "More
// Value per Key", §3.1 and App. C.1, with a bound in place of the paper's
// threshold calibrated on earlier steps).
//
// One CTA per (batch row b, query head j).  The sample is 32 blocks of 32
// consecutive positions spread evenly over [0, L_b): 1024 scores computed
// here on CUDA cores in fp32 (the bound needs no tensor-core accuracy match:
// the selector checks what passes it).  With r_s = N * 1024 / L_b the bound is
// the lower edge of the bin below the one that holds the sample's
// (r_s + 6 sqrt(r_s) + 8)-th largest score in an equal-width histogram of the
// sample, so the expected number of candidates is a little above
// (r_s + 6 sqrt(r_s) + 8) * L_b / 1024.  Rows short enough for the candidate
// buffer get t_lo = -inf (every position is a candidate).
#pragma once

#include <cuda_bf16.h>
#include "ptx.cuh"

namespace saga {

constexpr int kThrThreads = 256;
constexpr int kThrWarps = kThrThreads / 32;
constexpr int kThrBlocks = 32;                    // sampled blocks of 32 positions
constexpr int kThrSample = kThrBlocks * 32;       // 1024 sampled scores
constexpr int kThrBins = 1024;

struct ThresholdParams {
  const __nv_bfloat16* q;        // [B][h_q][D]
  const __nv_bfloat16* k_cache;  // [B][h_k][L_max][D]
  const int32_t* seq_lens;
  int h_q, h_k, g, L_max, N, cand_cap;
  float scale;
  float* t_lo;                   // [B*h_q]
};

template <int D>
__global__ void __launch_bounds__(kThrThreads)
threshold_kernel(const ThresholdParams p) {
  __shared__ float qs[D];
  __shared__ float samp[kThrSample];
  __shared__ uint32_t hist[kThrBins];
  __shared__ uint32_t red[2 * kThrWarps];
  __shared__ uint32_t wsum[kThrWarps];
  __shared__ int bstar;
  pdl_launch_dependents();                        // the score pass may start streaming now
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int bj = blockIdx.x;
  const int b = bj / p.h_q, j = bj % p.h_q;
  const int L = p.seq_lens[b];
  const int n_b = p.N < L ? p.N : L;
  if (L < 1 || L > p.L_max || L <= p.cand_cap) {  // short (or invalid) row: take everything
    if (tid == 0) p.t_lo[bj] = -INFINITY;
    return;
  }
  for (int t = tid; t < D; t += kThrThreads)
    qs[t] = __bfloat162float(p.q[static_cast<long long>(bj) * D + t]);
  __syncthreads();

  // ---- 1024 sampled scores: warp w scores blocks w, w + 8, w + 16, w + 24, a lane per position
  const __nv_bfloat16* krow0 =
      p.k_cache + (static_cast<long long>(b) * p.h_k + j / p.g) * p.L_max * D;
  const int lpb = L / 32;                         // whole 32-position blocks in the row
  for (int r = 0; r < kThrBlocks / kThrWarps; ++r) {
    const int blk = warp + r * kThrWarps;
    const int pos = 32 * ((blk * lpb) / kThrBlocks) + lane;   // blk * lpb < 2^24
    const uint4* kr = reinterpret_cast<const uint4*>(krow0 + static_cast<long long>(pos) * D);
    uint4 raw[D / 8];
#pragma unroll
    for (int c = 0; c < D / 8; ++c) raw[c] = __ldg(kr + c);
    float acc = 0.0f;
#pragma unroll
    for (int c = 0; c < D / 8; ++c) {
      const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&raw[c]);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __bfloat1622float2(h2[e]);
        acc = fmaf(f.x, qs[c * 8 + 2 * e], acc);
        acc = fmaf(f.y, qs[c * 8 + 2 * e + 1], acc);
      }
    }
    samp[blk * 32 + lane] = acc * p.scale;
  }
  __syncthreads();

  // ---- range of the sample
  float lo = INFINITY, hi = -INFINITY;
  for (int i = tid; i < kThrSample; i += kThrThreads) { lo = fminf(lo, samp[i]); hi = fmaxf(hi, samp[i]); }
  for (int o = 16; o; o >>= 1) {
    lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
    hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
  }
  if (lane == 0) { red[warp] = __float_as_uint(lo); red[kThrWarps + warp] = __float_as_uint(hi); }
  for (int i = tid; i < kThrBins; i += kThrThreads) hist[i] = 0;
  __syncthreads();
  lo = __uint_as_float(red[0]);
  hi = __uint_as_float(red[kThrWarps]);
  for (int w = 1; w < kThrWarps; ++w) {
    lo = fminf(lo, __uint_as_float(red[w]));
    hi = fmaxf(hi, __uint_as_float(red[kThrWarps + w]));
  }
  const float scale = static_cast<float>(kThrBins) / (hi - lo);
  if (!(hi > lo) || !(scale < INFINITY)) {        // flat or extreme sample: no useful bound
    if (tid == 0) p.t_lo[bj] = -INFINITY;
    return;
  }
  for (int i = tid; i < kThrSample; i += kThrThreads) {
    const float x = fminf(fmaxf((samp[i] - lo) * scale, 0.0f), static_cast<float>(kThrBins - 1));
    atomicAdd(&hist[static_cast<int>(x)], 1u);
  }
  __syncthreads();

  // ---- bin holding the r-th largest sample: thread t owns bins [4*(255-t), +4), top-down
  const float rs = static_cast<float>(n_b) * kThrSample / static_cast<float>(L);
  uint32_t r = static_cast<uint32_t>(ceilf(rs + 6.0f * sqrtf(rs) + 8.0f));
  if (r > static_cast<uint32_t>(kThrSample)) r = kThrSample;
  const int b0 = 4 * (kThrThreads - 1 - tid);
  uint32_t c = hist[b0] + hist[b0 + 1] + hist[b0 + 2] + hist[b0 + 3];
  uint32_t incl = c;
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) wsum[warp] = incl;
  if (tid == 0) bstar = -1;
  __syncthreads();
  uint32_t above = incl - c;
  for (int w = 0; w < warp; ++w) above += wsum[w];
  for (int e = 3; e >= 0; --e) {
    const uint32_t h = hist[b0 + e];
    if (above < r && above + h >= r) bstar = b0 + e;
    above += h;
  }
  __syncthreads();
  if (tid == 0) p.t_lo[bj] = (bstar >= 1) ? lo + static_cast<float>(bstar - 1) / scale : -INFINITY;
}

}  // namespace saga
