// gather_kernel.cuh -- S3 (softmax over the selected logits) and S4 (the
// gathered P.V) of "More Value per Key", §3.1 Eq. (7): for each (b, j),
// out = sum_i exp(z_i - m) V[b, j/g_v, i, :] / sum_i exp(z_i - m) over the
// selected positions i, with fp32 accumulation and one bf16 rounding.
//
// The selected value rows are scattered across the cache, so this is a gather
// bound by memory latency and bandwidth.  Each (b, j) selection is cut into
// chunks of kGatherRows slots, one CTA per chunk, so that many CTAs (and 32
// row loads per warp) are in flight at once.  A chunk produces the partial
// (m_c, s_c, acc_c) of a softmax restricted to its rows; the CTA that
// finishes a row last (a per-row atomic counter, no waiting) merges the
// chunks in chunk order -- m = max m_c, s = sum s_c e^(m_c - m), acc = sum
// acc_c e^(m_c - m) -- so the result does not depend on scheduling.
#pragma once

#include <cuda_bf16.h>
#include "ptx.cuh"

namespace saga {

constexpr int kGatherThreads = 256;
constexpr int kGatherWarps = kGatherThreads / 32;
constexpr int kGatherRows = 256;                     // selection slots per CTA (one per thread)

struct GatherParams {
  const int32_t* sel_idx;       // [B*h_q][N]; -1 = padding
  const float* sel_logit;       // [B*h_q][N]
  const int32_t* seq_lens;
  const __nv_bfloat16* v_cache; // [B][h_v][L_max][D]
  int h_q, h_v, g_v, L_max, N;
  float* partial;               // [B*h_q][max_chunks][D + 2]: m_c, s_c, acc_c
  int max_chunks;
  uint32_t* counter;            // [B*h_q], zero on entry, left zero on exit
  __nv_bfloat16* out;           // [B*h_q][D]
  int* status;
};

template <int D>
struct GatherSmem {
  int32_t idx[kGatherRows];
  float w[kGatherRows];
  float red[kGatherWarps][D];
  float fred[kGatherWarps];
  float m_c, s_c;
  int last;
};

template <int D>
__global__ void __launch_bounds__(kGatherThreads)
gather_kernel(const GatherParams p) {
  __shared__ GatherSmem<D> sm;
  pdl_wait();                        // the selection lists are complete (no-op without PDL)
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int bj = blockIdx.x;
  const int chunk = blockIdx.y;
  const int b = bj / p.h_q, j = bj % p.h_q;
  const int L = p.seq_lens[b];
  if (L < 1 || L > p.L_max) {        // invalid row: zero output (flagged by the status word)
    if (chunk == 0) {
      if (tid == 0) atomicOr(p.status, 0x1 /* SAGA_STATUS_BAD_SEQ_LEN */);
      for (int e = tid; e < D; e += kGatherThreads)
        p.out[static_cast<long long>(bj) * D + e] = __float2bfloat16_rn(0.0f);
    }
    return;
  }
  const int n_slots = min(p.N, L);
  const int n_chunks = (n_slots + kGatherRows - 1) / kGatherRows;
  if (chunk >= n_chunks) return;

  // ---- this chunk's slots: positions and logits, one per thread
  const int r = chunk * kGatherRows + tid;
  int id = -1;
  float z = -INFINITY;
  if (r < n_slots) {
    const long long o = static_cast<long long>(bj) * p.N + r;
    id = __ldcg(p.sel_idx + o);
    if (id >= L) { atomicOr(p.status, 0x4 /* SAGA_STATUS_BAD_INDEX */); id = -1; }
    if (id >= 0) z = __ldcg(p.sel_logit + o);
  }
  float m = z;
  for (int s = 16; s; s >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, s));
  if (lane == 0) sm.fred[warp] = m;
  __syncthreads();
  float m_c = sm.fred[0];
#pragma unroll
  for (int w = 1; w < kGatherWarps; ++w) m_c = fmaxf(m_c, sm.fred[w]);
  const float w_t = (id >= 0) ? expf(z - m_c) : 0.0f;
  sm.idx[tid] = id;
  sm.w[tid] = w_t;
  __syncthreads();

  // ---- each warp gathers its 32 rows: all 32 loads issued before any use
  constexpr int EPL = D / 32;                   // elements per lane: 2 or 4
  const __nv_bfloat16* vbase = p.v_cache +
      (static_cast<long long>(b) * p.h_v + j / p.g_v) * p.L_max * D + lane * EPL;
  float acc[EPL];
#pragma unroll
  for (int e = 0; e < EPL; ++e) acc[e] = 0.0f;
  const int r0 = warp * 32;
  if constexpr (EPL == 4) {
    uint2 raw[32];
#pragma unroll
    for (int u = 0; u < 32; ++u) {
      const int rid = sm.idx[r0 + u];
      raw[u] = rid >= 0 ? __ldg(reinterpret_cast<const uint2*>(vbase + static_cast<long long>(rid) * D))
                        : make_uint2(0u, 0u);
    }
#pragma unroll
    for (int u = 0; u < 32; ++u) {
      const float wu = sm.w[r0 + u];
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
      const int rid = sm.idx[r0 + u];
      raw[u] = rid >= 0 ? __ldg(reinterpret_cast<const uint32_t*>(vbase + static_cast<long long>(rid) * D))
                        : 0u;
    }
#pragma unroll
    for (int u = 0; u < 32; ++u) {
      const float wu = sm.w[r0 + u];
      const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw[u]));
      acc[0] = fmaf(wu, a.x, acc[0]);
      acc[1] = fmaf(wu, a.y, acc[1]);
    }
  }
#pragma unroll
  for (int e = 0; e < EPL; ++e) sm.red[warp][lane * EPL + e] = acc[e];
  float s = w_t;
  for (int o = 16; o; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if (lane == 0) sm.fred[warp] = s;   // fred's maxima were consumed before the last barrier
  __syncthreads();

  float* part = p.partial + (static_cast<long long>(bj) * p.max_chunks + chunk) * (D + 2);
  float a_t = 0.0f;
  float s_c = 0.0f;
#pragma unroll
  for (int w = 0; w < kGatherWarps; ++w) s_c += sm.fred[w];
  if (tid < D) {
#pragma unroll
    for (int w = 0; w < kGatherWarps; ++w) a_t += sm.red[w][tid];
  }
  if (n_chunks == 1) {              // the only chunk: no merge needed
    if (tid < D)
      p.out[static_cast<long long>(bj) * D + tid] = __float2bfloat16_rn(s_c > 0.0f ? a_t / s_c : 0.0f);
    return;
  }
  if (tid < D) part[2 + tid] = a_t;
  if (tid == 0) { part[0] = m_c; part[1] = s_c; }
  __threadfence();
  __syncthreads();
  if (tid == 0) sm.last = (atomicAdd(p.counter + bj, 1u) == static_cast<uint32_t>(n_chunks - 1));
  __syncthreads();
  if (!sm.last) return;

  // ---- last chunk of this row: merge every chunk's partial in chunk order
  __threadfence();
  const float* row_part = p.partial + static_cast<long long>(bj) * p.max_chunks * (D + 2);
  float m_all = -INFINITY;
  for (int c = 0; c < n_chunks; ++c) m_all = fmaxf(m_all, __ldcg(row_part + c * (D + 2)));
  if (tid < D) {
    float s_all = 0.0f, a_all = 0.0f;
    for (int c = 0; c < n_chunks; ++c) {
      const float mc = __ldcg(row_part + c * (D + 2));
      const float f = (mc == -INFINITY) ? 0.0f : expf(mc - m_all);
      s_all += __ldcg(row_part + c * (D + 2) + 1) * f;
      a_all += __ldcg(row_part + c * (D + 2) + 2 + tid) * f;
    }
    p.out[static_cast<long long>(bj) * D + tid] = __float2bfloat16_rn(s_all > 0.0f ? a_all / s_all : 0.0f);
  }
  if (tid == 0) p.counter[bj] = 0u;
}

}  // namespace saga
