// group_kernel.cuh -- S2 to S4 of group-shared selection for one (batch row b,
// value head v): the g_v query heads that read value head v share one set of N
// positions, so the value gather reads N rows per value head.
//
// The statistic of a position is s_i = sum over the group's heads j of
// softmax(z_j)_i, the sum of their attention probabilities (the GQA form of
// SparQ's position step as the pages describe it, applied to SAGA's decode
// step, "More Value per Key" §3.1 Eq. (7), §3.2); the set is the N_b positions
// with the largest s (ties to the lowest position); each head then takes the
// softmax of its own logits over the set and the gathered P.V.
//
// The score pass (group variant) kept, per 32-position chunk of the group row,
// every position where some head of the group scored at or above its own
// sampled bound t_lo_j, with all g_v keys of the position, and summed
// exp(z - m_ref) per head.  This kernel:
//   1  masks and per-head chunk sums in one round of loads; log-sum-exp per head;
//   2  s for every kept position, to the group's statistic slots (and to shared
//      memory when the list fits);
//   3  the N_b-th largest s and the selection (the top-N kernel's radix select
//      and ordered pass, on keys of s);
//   4  exactness: a position that was not kept has z_j < t_lo_j for every head,
//      so s < S_lo = sum_j exp(t_lo_j - lse_j); the kept set is complete when
//      the N_b-th kept s is above S_lo (with a relative margin).  Otherwise, and
//      when the sums left the fp32 range, the group's rows are scored again on
//      CUDA cores and the selection is made from every position;
//   5  each head's logits at the set (from the kept keys), its softmax weights,
//      and one pass over the N value rows that accumulates all g_v heads.
#pragma once

#include <cuda_bf16.h>
#include "ptx.cuh"
#include "topn_kernel.cuh"

namespace saga {

constexpr int kGroupMaxGv = 8;            // query heads per value head
constexpr int kGroupMaxN = 1024;          // N * g_v weights live in the key list's region
constexpr float kGroupMargin = 1e-4f;     // relative margin of the completeness check
constexpr int kGroupBatch = 16;           // value rows per warp per round of loads
constexpr int kGroupBlock = 8;            // kept positions whose keys are loaded together
// Candidates of a group held in shared memory: the union of g_v heads' lists
// (one CTA per group, so one CTA per SM costs nothing here).
constexpr int kGroupCap = 16384;
using GroupLayout = TopnLayout<kTopnSelNarrow, kGroupCap>;

struct GroupParams {
  const uint32_t* cand_mask;    // [B*h_v][mask_stride] positions kept for the group
  long long mask_stride;
  uint32_t* zkey;               // group row r's keys at r * g_v * z_stride (see score_kernel)
  long long z_stride;
  uint32_t* gstat;              // [B*h_v][z_stride] keys of s at the candidate slots (scratch)
  const int32_t* seq_lens;      // [B]
  int h_q, h_k, g, h_v, g_v, L_max, N, cand_cap;
  const float* lse_part;        // [B*h_q][mask_stride] chunk sums of exp(z - m_ref)
  const float* m_ref;           // [B*h_q]
  const float* t_lo;            // [B*h_q]
  int32_t* sel_idx;             // [B*h_v][N] the shared positions, ascending; -1 padding
  float* sel_stat;              // [B*h_v][N] s at them; -inf padding
  float* sel_logit;             // [B*h_q][N] each head's logits at them; -inf padding
  const __nv_bfloat16* q;       // [B][h_q][D]
  const __nv_bfloat16* k_cache; // [B][h_k][L_max][D]
  const __nv_bfloat16* v_cache; // [B][h_v][L_max][D]
  float scale;
  __nv_bfloat16* out;           // [B*h_q][D]
  int* status;
};

// Keys of the group's g_v heads for every position, scored on CUDA cores, to
// area[p * g_v + e] (the layout of a group row where every position is kept).
template <int D>
__device__ void group_rescore(const GroupParams& p, int b, int j0, int kh, int L, uint32_t* area) {
  const __nv_bfloat16* keys = p.k_cache + (static_cast<long long>(b) * p.h_k + kh) * p.L_max * D;
  for (int i = threadIdx.x; i < L; i += kTopnThreads) {
    const uint4* kv = reinterpret_cast<const uint4*>(keys + static_cast<long long>(i) * D);
    float acc[kGroupMaxGv];
#pragma unroll
    for (int e = 0; e < kGroupMaxGv; ++e) acc[e] = 0.0f;
    for (int c = 0; c < D / 8; ++c) {
      const uint4 a = __ldg(kv + c);
      const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&a);
#pragma unroll
      for (int e = 0; e < kGroupMaxGv; ++e) {
        if (e < p.g_v) {
          const uint4 qq = __ldg(reinterpret_cast<const uint4*>(
              p.q + (static_cast<long long>(b) * p.h_q + j0 + e) * D) + c);
          const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&qq);
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            const float2 x = __bfloat1622float2(a2[t]), y = __bfloat1622float2(b2[t]);
            acc[e] = fmaf(x.x, y.x, acc[e]);
            acc[e] = fmaf(x.y, y.y, acc[e]);
          }
        }
      }
    }
#pragma unroll
    for (int e = 0; e < kGroupMaxGv; ++e)
      if (e < p.g_v) area[static_cast<long long>(i) * p.g_v + e] = ordered_key(__fadd_rn(__fmul_rn(acc[e], p.scale), 0.0f));
  }
}

// Word offset, in the group's key area, of head e's key at kept position pos.
__device__ __forceinline__ long long group_key_at(const uint32_t* mrow, int pos, int g_v, int e, bool all) {
  if (all) return static_cast<long long>(pos) * g_v + e;
  const int c = pos >> 5, bit = pos & 31;
  const int k = __popc(__ldcg(mrow + c) & ((1u << bit) - 1u));
  return (static_cast<long long>(c) * 32 + k) * g_v + e;
}

template <int D>
__global__ void __launch_bounds__(kTopnThreads, 2)
group_kernel(const GroupParams p) {
  using Lay = GroupLayout;
  extern __shared__ __align__(16) uint32_t group_smem[];
  uint32_t* s_key = group_smem + Lay::kOffKey;       // candidate keys of s; then the weights
  int32_t* s_pos = reinterpret_cast<int32_t*>(group_smem + Lay::kOffPos);   // positions; then P.V partials
  int32_t* s_selpos = reinterpret_cast<int32_t*>(group_smem + Lay::kOffSelPos);
  float* s_selw = reinterpret_cast<float*>(group_smem + Lay::kOffSelW);     // emission scratch
  uint32_t* s_hist = group_smem + Lay::kOffHist;
  uint32_t* s_scan = group_smem + Lay::kOffScan;
  uint32_t* s_misc = group_smem + Lay::kOffMisc;
  float* s_w = reinterpret_cast<float*>(s_key);                              // [n_b][g_v] weights
  float* s_part = reinterpret_cast<float*>(s_pos);                           // [warps][g_v][D]

  pdl_wait();                                    // the candidates and sums are complete
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int r = blockIdx.x;                      // group row: b * h_v + v
  const int b = r / p.h_v, v = r % p.h_v;
  const int g_v = p.g_v, j0 = v * g_v, kh = j0 / p.g;
  const int N = p.N;
  const int L = p.seq_lens[b];
  int32_t* idx_out = p.sel_idx + static_cast<long long>(r) * N;
  float* stat_out = p.sel_stat + static_cast<long long>(r) * N;
  if (L < 1 || L > p.L_max) {                    // invalid row: padding and zero outputs
    if (tid == 0) atomicOr(p.status, 0x1 /* SAGA_STATUS_BAD_SEQ_LEN */);
    for (int i = tid; i < N; i += kTopnThreads) { idx_out[i] = -1; stat_out[i] = -INFINITY; }
    for (int e = 0; e < g_v; ++e) {
      float* lo = p.sel_logit + (static_cast<long long>(b) * p.h_q + j0 + e) * N;
      for (int i = tid; i < N; i += kTopnThreads) lo[i] = -INFINITY;
      for (int t = tid; t < D; t += kTopnThreads)
        p.out[(static_cast<long long>(b) * p.h_q + j0 + e) * D + t] = __float2bfloat16_rn(0.0f);
    }
    return;
  }
  const uint32_t n_b = static_cast<uint32_t>(N < L ? N : L);
  const uint32_t* mrow = p.cand_mask + static_cast<long long>(r) * p.mask_stride;
  uint32_t* area = p.zkey + static_cast<long long>(r) * g_v * p.z_stride;
  uint32_t* srow = p.gstat + static_cast<long long>(r) * p.z_stride;
  const int nch = (L + 31) / 32;
  const bool sums = L > p.cand_cap;

  // ---- 1: masks and per-head chunk sums; thread t owns chunks [c0, c1)
  const int cpt = (nch + kTopnThreads - 1) / kTopnThreads;
  const int c0 = min(nch, tid * cpt), c1 = min(nch, c0 + cpt);
  const bool fits = cpt <= kTopnRun;
  uint32_t cnt = 0u;
  float lsum[kGroupMaxGv];
#pragma unroll
  for (int e = 0; e < kGroupMaxGv; ++e) lsum[e] = 0.0f;
  for (int c = c0; c < c1; ++c) {
    cnt += __popc(__ldcg(mrow + c));
    if (sums) {
#pragma unroll
      for (int e = 0; e < kGroupMaxGv; ++e)
        if (e < g_v)
          lsum[e] += __ldcg(p.lse_part + (static_cast<long long>(b) * p.h_q + j0 + e) * p.mask_stride + c);
    }
  }
  uint32_t C;
  const uint32_t off = topn_excl_scan(cnt, s_scan, C);
  float lse[kGroupMaxGv];
  bool all = false;                              // every position, rescored
#pragma unroll
  for (int e = 0; e < kGroupMaxGv; ++e) lse[e] = 0.0f;
  if (sums) {
#pragma unroll
    for (int e = 0; e < kGroupMaxGv; ++e) {
      if (e < g_v) {
        const float S = topn_block_sum(lsum[e], s_scan);
        const float mref = __ldcg(p.m_ref + static_cast<long long>(b) * p.h_q + j0 + e);
        if (!(S > 0.0f && S <= 3.402823466e38f && mref > -INFINITY && mref < INFINITY)) all = true;
        lse[e] = mref + logf(S);
      }
    }
  } else {
    // rows of at most cand_cap positions: every position was kept with all its keys,
    // at area[p * g_v + e]; the log-sum-exp of each head from them
#pragma unroll
    for (int e = 0; e < kGroupMaxGv; ++e) {
      if (e < g_v) {
        uint32_t hi = 0u;
        for (int i = tid; i < L; i += kTopnThreads) hi = max(hi, __ldcg(area + static_cast<long long>(i) * g_v + e));
        const float m = key_to_float(topn_block_max(hi, s_scan));
        float sum = 0.0f;
        for (int i = tid; i < L; i += kTopnThreads)
          sum += expf(key_to_float(__ldcg(area + static_cast<long long>(i) * g_v + e)) - m);
        lse[e] = m + logf(topn_block_sum(sum, s_scan));
      }
    }
  }

  // ---- 2-4: s of every kept position, the selection and its completeness check.
  // Attempt 0 uses the kept positions; attempt 1 (the check failed, too few were
  // kept, or the sums left the fp32 range) scores the group's rows again and uses
  // every position.  Every decision below is uniform across the CTA.
  uint32_t T = 0u, need = 0u, kmax = 0u;
  bool listp = false;
  for (int attempt = 0; attempt < 2; ++attempt) {
    if (!all && attempt == 0 && C < n_b) all = true;
    if (all) {
      if (tid == 0) atomicOr(p.status, 0x200 /* SAGA_STATUS_INFO_ROBUST_PATH */);
      group_rescore<D>(p, b, j0, kh, L, area);
      __syncthreads();
#pragma unroll
      for (int e = 0; e < kGroupMaxGv; ++e) {
        if (e < g_v) {
          uint32_t hi = 0u;
          for (int i = tid; i < L; i += kTopnThreads) hi = max(hi, area[static_cast<long long>(i) * g_v + e]);
          const float m = key_to_float(topn_block_max(hi, s_scan));
          float sum = 0.0f;
          for (int i = tid; i < L; i += kTopnThreads)
            sum += expf(key_to_float(area[static_cast<long long>(i) * g_v + e]) - m);
          lse[e] = m + logf(topn_block_sum(sum, s_scan));
        }
      }
      for (int i = tid; i < L; i += kTopnThreads) {
        float s = 0.0f;
#pragma unroll
        for (int e = 0; e < kGroupMaxGv; ++e)
          if (e < g_v) s += expf(key_to_float(area[static_cast<long long>(i) * g_v + e]) - lse[e]);
        srow[i] = ordered_key(s);
      }
      __syncthreads();                           // srow is complete for the whole CTA
      listp = false;
    } else {
      listp = C <= static_cast<uint32_t>(kGroupCap) && fits;
      if (listp) {
        // the list in position order: each thread expands its chunks' masks into
        // positions and key slots (slot = 32 c + rank in the chunk; s_key holds the
        // slot until s replaces it), then s of entry i is formed by thread i mod 256,
        // so a warp reads the keys of 32 consecutive entries, mostly consecutive slots
        uint32_t o = off;
        for (int c = c0; c < c1; ++c) {
          uint32_t m = __ldcg(mrow + c);
          const int n_c = __popc(m);
          for (int k = 0; k < n_c; ++k) {
            s_pos[o] = c * 32 + (__ffs(m) - 1);
            s_key[o] = static_cast<uint32_t>(c * 32 + k);
            m &= m - 1u;
            ++o;
          }
        }
        __syncthreads();
        for (int i0 = 0; i0 < static_cast<int>(C); i0 += kTopnThreads * kGroupBlock) {
          uint32_t slot[kGroupBlock], kv[kGroupBlock][kGroupMaxGv];
#pragma unroll
          for (int u = 0; u < kGroupBlock; ++u) {
            const int i = i0 + u * kTopnThreads + tid;
            slot[u] = i < static_cast<int>(C) ? s_key[i] : 0u;
#pragma unroll
            for (int e = 0; e < kGroupMaxGv; ++e)
              kv[u][e] = (i < static_cast<int>(C) && e < g_v)
                             ? __ldcg(area + static_cast<long long>(slot[u]) * g_v + e) : 0u;
          }
#pragma unroll
          for (int u = 0; u < kGroupBlock; ++u) {
            const int i = i0 + u * kTopnThreads + tid;
            if (i < static_cast<int>(C)) {
              float sv = 0.0f;
#pragma unroll
              for (int e = 0; e < kGroupMaxGv; ++e)
                if (e < g_v) sv += expf(key_to_float(kv[u][e]) - lse[e]);
              const uint32_t key = ordered_key(sv);
              srow[slot[u]] = key;
              s_key[i] = key;
            }
          }
        }
      } else {                                   // the slots in global memory: s per chunk
        // a chunk's kept positions hold their keys at consecutive slots: the keys of
        // kGroupBlock positions (all heads) are loaded before any of them is used
        for (int c = c0; c < c1; ++c) {
          uint32_t m = __ldcg(mrow + c);
          const int n_c = __popc(m);
          const uint32_t* ac = area + static_cast<long long>(c) * 32 * g_v;
          for (int k0 = 0; k0 < n_c; k0 += kGroupBlock) {
            uint32_t kv[kGroupBlock][kGroupMaxGv];
#pragma unroll
            for (int u = 0; u < kGroupBlock; ++u)
#pragma unroll
              for (int e = 0; e < kGroupMaxGv; ++e)
                kv[u][e] = (k0 + u < n_c && e < g_v) ? __ldcg(ac + (k0 + u) * g_v + e) : 0u;
#pragma unroll
            for (int u = 0; u < kGroupBlock; ++u) {
              if (k0 + u < n_c) {
                float s = 0.0f;
#pragma unroll
                for (int e = 0; e < kGroupMaxGv; ++e)
                  if (e < g_v) s += expf(key_to_float(kv[u][e]) - lse[e]);
                const uint32_t key = ordered_key(s);
                srow[c * 32 + k0 + u] = key;
              }
            }
          }
        }
      }
      __syncthreads();
    }
    if (listp) {
      const TopnListSrc src{s_key, s_pos, static_cast<int>(C)};
      T = topn_radix(src, src.n, n_b, s_hist, s_scan, s_misc, &need, &kmax);
    } else {
      const TopnSlotSrc src{mrow, srow, all ? L : nch * 32, all};
      T = topn_radix(src, src.n, n_b, s_hist, s_scan, s_misc, &need, &kmax);
    }
    if (all || !sums) break;                     // every position took part
    // positions not kept have s < S_lo: the kept set is complete when s_(N_b) > S_lo
    float S_lo = 0.0f;
#pragma unroll
    for (int e = 0; e < kGroupMaxGv; ++e) {
      if (e < g_v) {
        const float tl = __ldcg(p.t_lo + static_cast<long long>(b) * p.h_q + j0 + e);
        if (tl > -INFINITY) S_lo += expf(tl - lse[e]);
      }
    }
    if (key_to_float(T) > S_lo * (1.0f + kGroupMargin)) break;
    all = true;                                  // not provably complete: every position
  }

  // the selection: positions ascending, s at them
  if (listp) {
    const TopnListSrc src{s_key, s_pos, static_cast<int>(C)};
    topn_emit(src, src.n, T, need, n_b, 0.0f, idx_out, stat_out, s_selpos, s_selw, s_scan);
  } else {
    const TopnSlotSrc src{mrow, srow, all ? L : nch * 32, all};
    topn_emit(src, src.n, T, need, n_b, 0.0f, idx_out, stat_out, s_selpos, s_selw, s_scan);
  }
  for (int i = static_cast<int>(n_b) + tid; i < N; i += kTopnThreads) { idx_out[i] = -1; stat_out[i] = -INFINITY; }
  __syncthreads();                               // s_selpos complete; s_key / s_pos free

  // ---- 5: each head's logits at the set, softmax weights, and one P.V pass
  // one lookup of a position's key slot serves all g_v heads (head e's key at +e)
  float zmax[kGroupMaxGv], wtot[kGroupMaxGv];
  uint32_t khi[kGroupMaxGv];
#pragma unroll
  for (int e = 0; e < kGroupMaxGv; ++e) { zmax[e] = 0.0f; wtot[e] = 0.0f; khi[e] = 0u; }
  float* lo0 = p.sel_logit + (static_cast<long long>(b) * p.h_q + j0) * N;
#pragma unroll 4
  for (int i = tid; i < static_cast<int>(n_b); i += kTopnThreads) {
    const long long at = group_key_at(mrow, s_selpos[i], g_v, 0, all);
    uint32_t kk[kGroupMaxGv];
#pragma unroll
    for (int e = 0; e < kGroupMaxGv; ++e) kk[e] = e < g_v ? __ldcg(area + at + e) : 0u;
#pragma unroll
    for (int e = 0; e < kGroupMaxGv; ++e) {
      if (e < g_v) {
        const float z = key_to_float(kk[e]);
        lo0[static_cast<long long>(e) * N + i] = z;
        s_w[i * g_v + e] = z;
        khi[e] = max(khi[e], kk[e]);
      }
    }
  }
#pragma unroll
  for (int e = 0; e < kGroupMaxGv; ++e) {
    if (e < g_v) {
      for (int i = static_cast<int>(n_b) + tid; i < N; i += kTopnThreads) lo0[static_cast<long long>(e) * N + i] = -INFINITY;
      zmax[e] = key_to_float(topn_block_max(khi[e], s_scan));
    }
  }
#pragma unroll
  for (int e = 0; e < kGroupMaxGv; ++e) {
    if (e < g_v) {
      float ws = 0.0f;
      for (int i = tid; i < static_cast<int>(n_b); i += kTopnThreads) {
        const float w = expf(s_w[i * g_v + e] - zmax[e]);
        s_w[i * g_v + e] = w;
        ws += w;
      }
      wtot[e] = topn_block_sum(ws, s_scan);      // also: the weights are visible to the CTA
    }
  }

  constexpr int EPL = D / 32;                    // elements per lane: 2 or 4
  const __nv_bfloat16* vbase = p.v_cache + (static_cast<long long>(b) * p.h_v + v) * p.L_max * D + lane * EPL;
  float acc[kGroupMaxGv][EPL];
#pragma unroll
  for (int e = 0; e < kGroupMaxGv; ++e)
#pragma unroll
    for (int t = 0; t < EPL; ++t) acc[e][t] = 0.0f;
  for (int g0 = warp * kGroupBatch; g0 < static_cast<int>(n_b); g0 += kTopnWarps * kGroupBatch) {
    float vals[kGroupBatch][EPL];
#pragma unroll
    for (int u = 0; u < kGroupBatch; ++u) {
      const int sl = g0 + u;
      if constexpr (EPL == 4) {
        const uint2 raw = sl < static_cast<int>(n_b)
            ? __ldg(reinterpret_cast<const uint2*>(vbase + static_cast<long long>(s_selpos[sl]) * D))
            : make_uint2(0u, 0u);
        const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw.x));
        const float2 c = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw.y));
        vals[u][0] = a.x; vals[u][1] = a.y; vals[u][2] = c.x; vals[u][3] = c.y;
      } else {
        const uint32_t raw = sl < static_cast<int>(n_b)
            ? __ldg(reinterpret_cast<const uint32_t*>(vbase + static_cast<long long>(s_selpos[sl]) * D))
            : 0u;
        const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw));
        vals[u][0] = a.x; vals[u][1] = a.y;
      }
    }
#pragma unroll
    for (int u = 0; u < kGroupBatch; ++u) {
      const int sl = g0 + u;
      if (sl < static_cast<int>(n_b)) {
#pragma unroll
        for (int e = 0; e < kGroupMaxGv; ++e) {
          if (e < g_v) {
            const float w = s_w[sl * g_v + e];
#pragma unroll
            for (int t = 0; t < EPL; ++t) acc[e][t] = fmaf(w, vals[u][t], acc[e][t]);
          }
        }
      }
    }
  }
#pragma unroll
  for (int e = 0; e < kGroupMaxGv; ++e)
    if (e < g_v)
#pragma unroll
      for (int t = 0; t < EPL; ++t) s_part[(warp * g_v + e) * D + lane * EPL + t] = acc[e][t];
  __syncthreads();
#pragma unroll
  for (int e = 0; e < kGroupMaxGv; ++e) {
    if (e < g_v && tid < D) {
      float a = 0.0f;
#pragma unroll
      for (int w = 0; w < kTopnWarps; ++w) a += s_part[(w * g_v + e) * D + tid];
      p.out[(static_cast<long long>(b) * p.h_q + j0 + e) * D + tid] =
          __float2bfloat16_rn(wtot[e] > 0.0f ? a / wtot[e] : 0.0f);
    }
  }
}

}  // namespace saga
