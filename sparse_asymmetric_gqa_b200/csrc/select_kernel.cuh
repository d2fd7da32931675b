// select_kernel.cuh -- S2 (exact top-N selection), S3 (softmax over the
// selection) and S4 (gathered P.V) for one (batch row b, query head j) per CTA.
//
// Selection ("More Value per Key", §2.5 Eq. (6); Atop-N, §3.1 and App. C.1):
// Atop-N finds the N-th largest score and keeps every score above it by a
// plain per-element compare.  Here the threshold is found exactly on every
// call, in three passes over the fp32 score row (which the score pass left in
// L2):
//   A  histogram of the row over 2048 equal-width bins between the row's min
//      and max (the score pass supplies both), which spreads N(0,1)-like rows
//      evenly over the bins, so shared-memory atomics rarely collide;
//   B  gather the keys of the one bin that holds the N-th score (typically a
//      few dozen) and radix-select inside it (4 x 8-bit digits on
//      order-preserving uint32 keys) -> exact threshold key T and the number of
//      ties at T still needed;
//   C  compare pass in position order with a block-wide scan: keep z > T and
//      the lowest-index ties = T, writing positions ascending.
// Binning is monotone in z (a rounded subtract, a rounded multiply by a
// non-negative scale, clamp, truncate), so a higher bin always means a
// strictly larger score; any min/max (even a stale or missing one) gives a
// correct result.  If the boundary bin overflows the candidate buffer (very
// flat rows) the radix select runs over the whole row instead.
//
// Softmax and P.V ("More Value per Key", §3.1 Eq. (7)): weights exp(z - m)
// with m the largest selected score, fp32 accumulation of the gathered value
// rows (one warp per row, a lane per 2-4 elements), one bf16 rounding at the
// end.
#pragma once

#include <cuda_bf16.h>
#include "ptx.cuh"

namespace saga {

constexpr int kSelThreads = 512;
constexpr int kSelWarps = kSelThreads / 32;
constexpr int kBins = 2048;
constexpr int kCandCap = 4096;
constexpr int kItems = 8;                       // positions per thread per compaction chunk
constexpr int kChunk = kSelThreads * kItems;    // 4096

struct SelectParams {
  const float* z;               // [B*h_q][z_stride]
  long long z_stride;
  uint32_t* stat_min;           // ordered-key min/max per row, or nullptr
  uint32_t* stat_max;
  const int32_t* seq_lens;
  int B, h_q, L_max, N;
  int z_vec4;                   // rows are 16-byte aligned
  int32_t* sel_idx;             // [B*h_q][N]
  float* sel_logit;
  // S3 + S4 (skipped when out == nullptr)
  const __nv_bfloat16* v_cache; // [B][h_v][L_max][D]
  int h_v, g_v;
  __nv_bfloat16* out;           // [B*h_q][D]
  int* status;
};

struct SelectSmem {
  uint32_t hist[kBins];
  union {
    uint32_t cand[kCandCap];
    float red[kSelWarps][128];
  } u;
  uint32_t scan[kSelWarps];
  uint32_t bcast[4];
  float fred[kSelWarps];
  uint32_t cand_n;
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

__device__ __forceinline__ float block_max(float v, float* fred) {
  for (int o = 16; o; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  if ((threadIdx.x & 31) == 0) fred[threadIdx.x >> 5] = v;
  __syncthreads();
  float r = fred[0];
  for (int w = 1; w < kSelWarps; ++w) r = fmaxf(r, fred[w]);
  __syncthreads();
  return r;
}

__device__ __forceinline__ uint32_t block_min_u32(uint32_t v, uint32_t* scan) {
  v = __reduce_min_sync(0xffffffffu, v);
  if ((threadIdx.x & 31) == 0) scan[threadIdx.x >> 5] = v;
  __syncthreads();
  uint32_t r = scan[0];
  for (int w = 1; w < kSelWarps; ++w) r = min(r, scan[w]);
  __syncthreads();
  return r;
}

__device__ __forceinline__ uint32_t block_max_u32(uint32_t v, uint32_t* scan) {
  v = __reduce_max_sync(0xffffffffu, v);
  if ((threadIdx.x & 31) == 0) scan[threadIdx.x >> 5] = v;
  __syncthreads();
  uint32_t r = scan[0];
  for (int w = 1; w < kSelWarps; ++w) r = max(r, scan[w]);
  __syncthreads();
  return r;
}

// MSB-first radix select: the k-th largest key among key(i), i < count (keys
// outside the running prefix are skipped).  Returns the key T and, in *need,
// how many elements equal to T belong to the top k (k - #(key > T)).
template <class KeyAt>
__device__ uint32_t radix_select(KeyAt key_at, int count, uint32_t k, SelectSmem& sm,
                                 uint32_t* need) {
  uint32_t prefix = 0, mask = 0;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = threadIdx.x; i < 256; i += kSelThreads) sm.hist[i] = 0;
    __syncthreads();
    for (int i = threadIdx.x; i < count; i += kSelThreads) {
      const uint32_t key = key_at(i);
      if ((key & mask) == prefix) atomicAdd(&sm.hist[(key >> shift) & 255u], 1u);
    }
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
      uint32_t above = incl - c;             // elements in higher digits
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

// S3 + S4 for one (b, j): weights exp(z - m) over the count selection slots
// (slots with an index outside [0, L) carry no weight), fp32 accumulation of
// the gathered value rows, one bf16 rounding.  Returns the number of slots
// whose index was out of range.
template <int D>
__device__ int combine_rows(const SelectParams& p, int bj, const int32_t* idx_in,
                            const float* logit_in, int count, int L, float m, SelectSmem& sm) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int b = bj / p.h_q, j = bj % p.h_q;
  constexpr int EPL = D / 32;                     // elements per lane: 2 or 4
  const __nv_bfloat16* vrow0 = p.v_cache +
      (static_cast<long long>(b) * p.h_v + j / p.g_v) * p.L_max * D + lane * EPL;
  float acc[EPL];
#pragma unroll
  for (int e = 0; e < EPL; ++e) acc[e] = 0.0f;
  float s_local = 0.0f;
  int bad = 0;
  for (int r0 = warp * 32; r0 < count; r0 += kSelThreads) {
    const int r = r0 + lane;
    int my_idx = -1;
    float my_w = 0.0f;
    if (r < count) {
      my_idx = idx_in[r];
      if (my_idx >= L) { ++bad; my_idx = -1; }
      if (my_idx >= 0) my_w = expf(logit_in[r] - m);
    }
    s_local += my_w;
    const int cnt = min(32, count - r0);
    for (int t0 = 0; t0 < cnt; t0 += 8) {
      float wv[8];
      uint2 raw4[8];
      uint32_t raw2[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int id = __shfl_sync(0xffffffffu, my_idx, (t0 + u) & 31);
        wv[u] = __shfl_sync(0xffffffffu, my_w, (t0 + u) & 31);
        if (t0 + u < cnt && id >= 0) {
          const __nv_bfloat16* src = vrow0 + static_cast<long long>(id) * D;
          if constexpr (EPL == 4) raw4[u] = __ldg(reinterpret_cast<const uint2*>(src));
          else raw2[u] = __ldg(reinterpret_cast<const uint32_t*>(src));
        } else {
          wv[u] = 0.0f;
          if constexpr (EPL == 4) raw4[u] = make_uint2(0u, 0u);
          else raw2[u] = 0u;
        }
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        if constexpr (EPL == 4) {
          const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw4[u].x));
          const float2 c2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw4[u].y));
          acc[0] = fmaf(wv[u], a.x, acc[0]);
          acc[1] = fmaf(wv[u], a.y, acc[1]);
          acc[2] = fmaf(wv[u], c2.x, acc[2]);
          acc[3] = fmaf(wv[u], c2.y, acc[3]);
        } else {
          const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw2[u]));
          acc[0] = fmaf(wv[u], a.x, acc[0]);
          acc[1] = fmaf(wv[u], a.y, acc[1]);
        }
      }
    }
  }
  for (int o = 16; o; o >>= 1) s_local += __shfl_xor_sync(0xffffffffu, s_local, o);
#pragma unroll
  for (int e = 0; e < EPL; ++e) sm.u.red[warp][lane * EPL + e] = acc[e];
  if (lane == 0) sm.fred[warp] = s_local;
  __syncthreads();
  if (tid < D) {
    float o = 0.0f, s = 0.0f;
    for (int w2 = 0; w2 < kSelWarps; ++w2) { o += sm.u.red[w2][tid]; s += sm.fred[w2]; }
    p.out[static_cast<long long>(bj) * D + tid] = __float2bfloat16_rn(s > 0.0f ? o / s : 0.0f);
  }
  return bad;
}

// Stages S3 + S4 alone, from a caller-supplied selection (padding: index -1).
template <int D>
__global__ void __launch_bounds__(kSelThreads)
combine_kernel(const SelectParams p) {
  extern __shared__ uint8_t smem_raw[];
  SelectSmem& sm = *reinterpret_cast<SelectSmem*>(smem_raw);
  const int bj = blockIdx.x;
  const int b = bj / p.h_q;
  const int L = p.seq_lens[b];
  const int32_t* idx_in = p.sel_idx + static_cast<long long>(bj) * p.N;
  const float* logit_in = p.sel_logit + static_cast<long long>(bj) * p.N;
  if (L < 1 || L > p.L_max) {
    if (threadIdx.x == 0) atomicOr(p.status, 0x1 /* SAGA_STATUS_BAD_SEQ_LEN */);
    for (int e = threadIdx.x; e < D; e += kSelThreads)
      p.out[static_cast<long long>(bj) * D + e] = __float2bfloat16_rn(0.0f);
    return;
  }
  float m_local = -INFINITY;
  for (int r = threadIdx.x; r < p.N; r += kSelThreads) {
    const int id = idx_in[r];
    if (id >= 0 && id < L) m_local = fmaxf(m_local, logit_in[r]);
  }
  const float m = block_max(m_local, sm.fred);
  const int bad = combine_rows<D>(p, bj, idx_in, logit_in, p.N, L, m, sm);
  if (bad) atomicOr(p.status, 0x4 /* SAGA_STATUS_BAD_INDEX */);
}

template <int D>
__global__ void __launch_bounds__(kSelThreads)
select_combine_kernel(const SelectParams p) {
  extern __shared__ uint8_t smem_raw[];
  SelectSmem& sm = *reinterpret_cast<SelectSmem*>(smem_raw);
  const int tid = threadIdx.x, lane = tid & 31;
  const int bj = blockIdx.x;
  const int b = bj / p.h_q;
  const int L = p.seq_lens[b];
  const int N = p.N;
  int32_t* idx_out = p.sel_idx + static_cast<long long>(bj) * N;
  float* logit_out = p.sel_logit + static_cast<long long>(bj) * N;
  const float* row = p.z + static_cast<long long>(bj) * p.z_stride;

  uint32_t st_lo = 0xFFFFFFFFu, st_hi = 0u;
  if (p.stat_min != nullptr) { st_lo = p.stat_min[bj]; st_hi = p.stat_max[bj]; }
  __syncthreads();
  if (tid == 0 && p.stat_min != nullptr) {    // leave the statistics ready for the next call
    p.stat_min[bj] = 0xFFFFFFFFu;
    p.stat_max[bj] = 0u;
  }

  if (L < 1 || L > p.L_max) {
    if (tid == 0) atomicOr(p.status, 0x1 /* SAGA_STATUS_BAD_SEQ_LEN */);
    for (int r = tid; r < N; r += kSelThreads) { idx_out[r] = -1; logit_out[r] = -INFINITY; }
    if (p.out != nullptr)
      for (int e = tid; e < D; e += kSelThreads) p.out[static_cast<long long>(bj) * D + e] = __float2bfloat16_rn(0.0f);
    return;
  }
  const int n_b = N < L ? N : L;
  const bool dense = (n_b == L);

  auto load_z = [&](int i) -> float { return row[i]; };

  uint32_t T = 0, need_ties = 0;
  if (!dense) {
    // ---- range of the row: from the score pass, else one min/max pass
    if (p.stat_min == nullptr || st_lo > st_hi) {
      uint32_t lo_k = 0xFFFFFFFFu, hi_k = 0u;
      for (int i = tid; i < L; i += kSelThreads) {
        const uint32_t key = score_key(load_z(i));
        lo_k = min(lo_k, key);
        hi_k = max(hi_k, key);
      }
      st_lo = block_min_u32(lo_k, sm.scan);
      st_hi = block_max_u32(hi_k, sm.scan);
    }
    const float lo = key_to_float(st_lo), hi = key_to_float(st_hi);
    float scale = (hi > lo) ? static_cast<float>(kBins) / (hi - lo) : 0.0f;
    if (!(scale < INFINITY)) scale = 0.0f;       // inf or NaN range: everything in bin 0

    // ---- pass A: histogram over equal-width bins
    for (int i = tid; i < kBins; i += kSelThreads) sm.hist[i] = 0;
    if (tid == 0) sm.cand_n = 0;
    __syncthreads();
    const int n_chunks4 = (L + 4 * kSelThreads - 1) / (4 * kSelThreads);
    for (int c = 0; c < n_chunks4; ++c) {
      const int base = c * 4 * kSelThreads + tid * 4;
      if (p.z_vec4 && base + 3 < L) {
        const float4 v = *reinterpret_cast<const float4*>(row + base);
        atomicAdd(&sm.hist[lin_bin(v.x, lo, scale)], 1u);
        atomicAdd(&sm.hist[lin_bin(v.y, lo, scale)], 1u);
        atomicAdd(&sm.hist[lin_bin(v.z, lo, scale)], 1u);
        atomicAdd(&sm.hist[lin_bin(v.w, lo, scale)], 1u);
      } else {
        for (int e = 0; e < 4; ++e)
          if (base + e < L) atomicAdd(&sm.hist[lin_bin(load_z(base + e), lo, scale)], 1u);
      }
    }
    __syncthreads();

    // ---- boundary bin: thread t owns bins [4*(511-t), +4), so thread order runs top-down
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
      // ---- pass B: keys of the boundary bin
      for (int c = 0; c < n_chunks4; ++c) {
        const int base = c * 4 * kSelThreads + tid * 4;
        float v[4];
        if (p.z_vec4 && base + 3 < L) {
          const float4 f = *reinterpret_cast<const float4*>(row + base);
          v[0] = f.x; v[1] = f.y; v[2] = f.z; v[3] = f.w;
        } else {
          for (int e = 0; e < 4; ++e) v[e] = (base + e < L) ? load_z(base + e) : 0.0f;
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
            if (pred) sm.u.cand[slot + __popc(m & ((1u << lane) - 1u))] = score_key(v[e]);
          }
        }
      }
      __syncthreads();
      const int n_cand = static_cast<int>(sm.cand_n);
      T = radix_select([&](int i) { return sm.u.cand[i]; }, n_cand,
                       static_cast<uint32_t>(n_b) - above, sm, &need_ties);
    } else {
      // ---- flat row: exact radix select over the whole row
      if (tid == 0) atomicOr(p.status, 0x100 /* SAGA_STATUS_INFO_EXACT_FALLBACK */);
      T = radix_select([&](int i) { return score_key(load_z(i)); }, L,
                       static_cast<uint32_t>(n_b), sm, &need_ties);
    }
  }

  // ---- pass C: compare and compact in position order
  uint32_t run_gt = 0, run_tie = 0;
  float m_local = -INFINITY;
  const int n_chunks = (L + kChunk - 1) / kChunk;
  for (int c = 0; c < n_chunks; ++c) {
    const int base = c * kChunk + tid * kItems;
    float v[kItems];
    if (p.z_vec4 && base + kItems - 1 < L) {
      const float4 f0 = *reinterpret_cast<const float4*>(row + base);
      const float4 f1 = *reinterpret_cast<const float4*>(row + base + 4);
      v[0] = f0.x; v[1] = f0.y; v[2] = f0.z; v[3] = f0.w;
      v[4] = f1.x; v[5] = f1.y; v[6] = f1.z; v[7] = f1.w;
    } else {
#pragma unroll
      for (int e = 0; e < kItems; ++e) v[e] = (base + e < L) ? load_z(base + e) : 0.0f;
    }
    uint32_t gt_mask = 0, tie_mask = 0;
#pragma unroll
    for (int e = 0; e < kItems; ++e) {
      if (base + e < L) {
        const uint32_t key = score_key(v[e]);
        if (dense || key > T) gt_mask |= 1u << e;
        else if (key == T) tie_mask |= 1u << e;
      }
    }
    const uint32_t packed = (static_cast<uint32_t>(__popc(tie_mask)) << 16) | __popc(gt_mask);
    uint32_t total;
    const uint32_t excl = block_excl_scan(packed, sm.scan, &total);
    uint32_t tr = run_tie + (excl >> 16);
    uint32_t w = run_gt + (excl & 0xFFFFu) + min(need_ties, tr);
#pragma unroll
    for (int e = 0; e < kItems; ++e) {
      bool sel = (gt_mask >> e) & 1u;
      if ((tie_mask >> e) & 1u) { sel = tr < need_ties; ++tr; }
      if (sel) {
        idx_out[w] = base + e;
        logit_out[w] = v[e];
        m_local = fmaxf(m_local, v[e]);
        ++w;
      }
    }
    run_gt += total & 0xFFFFu;
    run_tie += total >> 16;
  }
  for (int r = n_b + tid; r < N; r += kSelThreads) { idx_out[r] = -1; logit_out[r] = -INFINITY; }
  if (p.out == nullptr) return;
  const float m = block_max(m_local, sm.fred);   // also orders the list writes above

  combine_rows<D>(p, bj, idx_out, logit_out, n_b, L, m, sm);
}

}  // namespace saga
