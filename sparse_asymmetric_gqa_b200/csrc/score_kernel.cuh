// score_kernel.cuh -- S1, the score pass: z[b, j, i] = q[b, j] . K[b, j/g, i] / sqrt(d)
// ("More Value per Key", §2.1 Eq. (2) and §2.2 Eq. (5)), for every cached
// position i < L_b of every query head j.
//
// Shape of the work: for one (batch row b, key head kh) the g query heads that
// share the key head form a [g x d] matrix Q and the cache a [L_b x d] matrix
// K, so the scores are the skinny product K . Q^T.  The K stream is the whole
// cost (g flop per byte), so the kernel is built to move K at HBM speed and to
// read every K row exactly once for all g heads:
//
//   * persistent CTAs, one per SM, each owning a contiguous range of 128-row
//     tiles of the flattened (b, kh, tile) space (ragged seq_lens balanced);
//   * warp 0 streams K tiles (and the group's q rows) into a ring of shared
//     memory stages with TMA (128-byte swizzle, L2 evict-first for K);
//   * warp 1 issues tcgen05.mma (M = 128 positions, N = g padded to 16k,
//     K = 16 per instruction) into a ring of TMEM accumulators that fills all
//     512 columns (32 tiles for g <= 16), so the K stream runs on while the
//     epilogue waits for the sampled bounds;
//   * warps 2-9 read the accumulators back with tcgen05.ld (thread = position,
//     registers = heads), two warps per TMEM lane quarter: for groups of up to
//     32 heads the two warp sets take alternate tiles (so two tiles are read
//     back at once), for larger groups each takes half of the heads.  They
//     scale, and either store z row-wise (coalesced per head) with per-(b, j)
//     min/max statistics, or append the candidates of the selector.
//
// With kLse (candidate mode), the epilogue also writes, per query head and
// 32-position chunk slot, sums of exp(z - m_ref[row]) that add up over a row to
// the row's total: the pieces of its log-sum-exp, from which a calibrated
// probability threshold becomes a logit threshold ("More Value per Key",
// App. C.1).  A term whose exponent exceeds kLseMaxExp makes the row's sum
// +inf, which sends the row to the selector's exact fallback.
#pragma once

#include <cuda.h>
#include "ptx.cuh"

namespace saga {

constexpr int kTileM = 128;          // positions per tile (MMA M)
constexpr int kEpiWarps = 8;         // two per TMEM lane quarter
constexpr int kScoreThreads = 64 + 32 * kEpiWarps;   // TMA, MMA, epilogue warps
constexpr int kMaxBatch = 1024;
// Largest exponent z - m_ref summed: a row of up to 2^24 terms stays below 2^24 e^64 < FLT_MAX.
constexpr float kLseMaxExp = 64.0f;

struct ScoreParams {
  const int32_t* seq_lens;   // [B]
  float* z;                  // [B*h_q][z_stride]: scores, or candidate keys in candidate mode
  // candidate mode: the scores >= t_lo[row] of each 32-position chunk of a row
  uint32_t* cand_mask;       // [B*h_q][mask_stride]: bit i of word c = position 32c + i passed
  long long mask_stride;
  const float* t_lo;         // [B*h_q] candidate bounds, written by the preceding kernel
  const float* m_ref;        // [B*h_q] exp-sum references (+inf: no sums), with lse_part
  float* lse_part;           // [B*h_q][mask_stride] chunk slots of the sums of exp(z - m_ref) (kLse)
  uint32_t* stat_min;        // [B*h_q] ordered keys, or nullptr
  uint32_t* stat_max;
  int* status;
  int B, h_q, h_k, g, L_max;
  long long z_stride;
  float scale;               // 1/sqrt(d), rounded to fp32
};

template <int D, int NPAD>
struct ScoreShape {
  static_assert(D == 32 || D == 64 || D == 128, "head_dim");
  static_assert(NPAD % 16 == 0 && NPAD >= 16 && NPAD <= 64, "padded group");
  // swizzle atoms along d: rows of 64 elements (128-byte swizzle), or of 32
  // elements for d = 32 (64-byte swizzle)
  static constexpr int kAtomElems = D < 64 ? D : 64;
  static constexpr int kAtomBytes = kAtomElems * 2;
  static constexpr int kParts = D / kAtomElems;
  static constexpr int kAPart = kTileM * kAtomBytes;    // K rows per atom (16 KB, or 8 KB for d = 32)
  static constexpr int kBPart = NPAD * kAtomBytes;      // q rows per atom
  static constexpr int kStageBytes = kParts * (kAPart + kBPart);
  // 128 KB of K in flight per SM (four stages for d = 128) measured faster than
  // 160 or 192 KB: more bytes in flight only lengthened the memory queues.
  static constexpr int kStagesRaw = (200 * 1024) / kStageBytes;
  static constexpr int kStagesK = (128 * 1024) / (kParts * kAPart);
  static constexpr int kStages = kStagesRaw < kStagesK ? kStagesRaw : kStagesK;
  static constexpr int kAccStride = NPAD <= 16 ? 16 : NPAD <= 32 ? 32 : 64;   // columns per accumulator
  static constexpr int kTmemCols = 512;                                        // all of TMEM
  static constexpr int kAccBufs = kTmemCols / kAccStride;                      // 32, 16 or 8
  // full, empty, accf[kAccBufs], acce[kAccBufs], drain
  static constexpr int kNumBars = 2 * kStages + 2 * kAccBufs + 1;
  // Epilogue split of the kEpiWarps / 4 warps of a lane quarter: kTileGroups
  // groups taking every kTileGroups-th tile, each group's warps splitting the
  // heads (two tile groups for up to 32 heads, else head halves).
  static constexpr int kTileGroups = NPAD <= 32 ? 2 : 1;
  static constexpr int kEpiHeads = NPAD * kTileGroups / (kEpiWarps / 4);   // heads per warp
  // bars, TMEM slot + abort flag, lens, unit_off
  static constexpr int kCtrlBytes = kNumBars * 8 + 16 + 2 * (kMaxBatch + 1) * 4;
  static constexpr int kSmemBytes = 1024 + kStages * kStageBytes + kCtrlBytes;
  static_assert(kStages >= 2, "stages");
  static_assert(kStageBytes % 1024 == 0, "stage alignment");
};

// Walks the flattened (b, kh, tile) space of one CTA in order.
struct TileCursor {
  int b, kh, t, tiles, Lb;
  __device__ void seek(long long u, const int* unit_off, const int* lens, int B, int h_k) {
    int lo = 0, hi = B;                       // largest b with unit_off[b] <= u
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (unit_off[mid] <= u) lo = mid; else hi = mid;
    }
    b = lo;
    while (b < B && unit_off[b + 1] <= u) ++b;  // skip rows without tiles
    Lb = (b < B) ? lens[b] : 0;
    tiles = (Lb + kTileM - 1) / kTileM;
    const long long r = u - unit_off[b];
    kh = tiles ? static_cast<int>(r / tiles) : 0;
    t = tiles ? static_cast<int>(r % tiles) : 0;
  }
  __device__ void next(const int* unit_off, const int* lens, int B, int h_k) {
    if (++t < tiles) return;
    t = 0;
    if (++kh < h_k) return;
    kh = 0;
    do { ++b; } while (b < B && unit_off[b + 1] == unit_off[b]);
    Lb = (b < B) ? lens[b] : 0;
    tiles = (Lb + kTileM - 1) / kTileM;
  }
};

__device__ __forceinline__ void st_global_hint(float* p, float v, uint64_t pol) {
  asm volatile("st.global.L2::cache_hint.f32 [%0], %1, %2;" :: "l"(p), "f"(v), "l"(pol) : "memory");
}
__device__ __forceinline__ void st_global_hint(uint32_t* p, uint32_t v, uint64_t pol) {
  asm volatile("st.global.L2::cache_hint.u32 [%0], %1, %2;" :: "l"(p), "r"(v), "l"(pol) : "memory");
}

// Sums across the warp of each of the H values of every lane (a butterfly that
// halves the values held per lane at each step: 16 or 31 shuffles for all H).
// Returns, in lane l, the sum for value l / (32 / HP), HP = H rounded up to 16
// or 32; a fixed order of additions, so the result is reproducible.
template <int H>
__device__ __forceinline__ float warp_transpose_sum(const float (&v)[H], int lane) {
  constexpr int HP = H <= 16 ? 16 : 32;
  static_assert(H <= 32, "at most 32 values per lane");
  float w[HP];
#pragma unroll
  for (int i = 0; i < HP; ++i) w[i] = i < H ? v[i] : 0.0f;
#pragma unroll
  for (int c = HP; c > 1; c >>= 1) {
    const int o = HP == 32 ? c / 2 : c;        // the lane bit that picks the half kept
    const bool up = (lane & o) != 0;
#pragma unroll
    for (int i = 0; i < c / 2; ++i) {
      const float send = up ? w[i] : w[i + c / 2];
      const float keep = up ? w[i + c / 2] : w[i];
      w[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
    }
  }
  float r = w[0];
  if (HP == 16) r += __shfl_xor_sync(0xffffffffu, r, 1);
  return r;
}

__device__ __forceinline__ void raise_abort(volatile int* abort_flag, int* status) {
  *abort_flag = 1;
  atomicOr(status, 0x2 /* SAGA_STATUS_TIMEOUT */);
}

// kCand = false: every score is stored to z (row stride z_stride) and per-row
// min/max keys are kept.
// kCand = true (launched as a programmatic dependent of the bound kernel): only
// the candidates of the selector are stored.  The producer and MMA warps start
// streaming at once; the epilogue first waits for the bounds t_lo.  Then, for
// each 32-position chunk c of a row, the mask of positions with score >= t_lo
// goes to cand_mask[row][c] and their order-preserving keys, in position
// order, to the row's z slots [32c, 32c + popcount).  No atomics on the data
// path: every chunk has its own slots.
// kLse (candidate mode only): the chunk sums of exp(z - m_ref) go to lse_part.
// kGroup (with kCand and kLse; g <= 32): candidates are kept per value-head group
// of g_v query heads (group-shared selection): a position passes for its group
// when any head of the group passes its own bound, and then all g_v of its keys
// are stored.  Group row r = b * h_v + (kh * g) / g_v + v' takes the z rows
// [r * g_v, (r + 1) * g_v) as one area: chunk c's passing positions, in position
// order, at [32 c g_v, ...), g_v keys each; its masks go to cand_mask row r.
template <int D, int NPAD, bool kCand, bool kLse = false, bool kGroup = false>
__global__ void __launch_bounds__(kScoreThreads, 1)
score_kernel(const __grid_constant__ CUtensorMap tmap_k,
             const __grid_constant__ CUtensorMap tmap_q, const ScoreParams p, const int g_v) {
  using S = ScoreShape<D, NPAD>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* stages = smem;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::kStages * S::kStageBytes);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + S::kNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* lens = reinterpret_cast<int*>(tmem_slot + 4);
  int* unit_off = lens + kMaxBatch;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t bar0 = smem_addr(bars);
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (S::kStages + s); };
  auto accf_bar = [&](int i) { return bar0 + 8u * (2 * S::kStages + i); };
  auto acce_bar = [&](int i) { return bar0 + 8u * (2 * S::kStages + S::kAccBufs + i); };
  const uint32_t drain_bar = bar0 + 8u * (2 * S::kStages + 2 * S::kAccBufs);

  if (warp == 0) {
    if (lane == 0) {
      if (kCand) pdl_launch_dependents();
      for (int s = 0; s < S::kStages; ++s) { mbar_init(full_bar(s), 1); mbar_init(empty_bar(s), 1); }
      for (int i = 0; i < S::kAccBufs; ++i) {
        mbar_init(accf_bar(i), 1);
        mbar_init(acce_bar(i), kEpiWarps / S::kTileGroups);   // warps that read each tile
      }
      mbar_init(drain_bar, 1);
      *abort_flag = 0;
      fence_mbar_init();
      tma_prefetch_desc(&tmap_k);
      tma_prefetch_desc(&tmap_q);
    }
    // Tile counts per batch row: h_k * ceil(L_b / 128) for a valid L_b, else 0.
    int carry = 0;
    for (int b0 = 0; b0 < p.B; b0 += 32) {
      const int b = b0 + lane;
      int L = 0, units = 0;
      if (b < p.B) {
        L = p.seq_lens[b];
        if (L < 1 || L > p.L_max) L = 0;
        units = p.h_k * ((L + kTileM - 1) / kTileM);
        lens[b] = L;
      }
      int incl = units;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      if (b == 0) unit_off[0] = 0;
      if (b < p.B) unit_off[b + 1] = carry + incl;
      carry += __shfl_sync(0xffffffffu, incl, 31);
    }
  } else if (warp == 1) {
    tmem_alloc(smem_addr(tmem_slot), S::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const long long total = unit_off[p.B];
  const long long u0 = total * blockIdx.x / gridDim.x;
  const long long u1 = total * (blockIdx.x + 1) / gridDim.x;
  const int n_tiles = static_cast<int>(u1 - u0);
  const int n_items = n_tiles;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0 && n_items > 0) {
      const uint64_t pol_k = policy_evict_first();
      const uint64_t pol_q = policy_evict_last();
      TileCursor c;
      c.seek(u0, unit_off, lens, p.B, p.h_k);
      int i = 0;
      for (; i < n_items; ++i) {
        const int s = i % S::kStages;
        const uint32_t ph = (i / S::kStages) & 1;
        if (!mbar_wait(empty_bar(s), ph ^ 1, abort_flag)) { raise_abort(abort_flag, p.status); break; }
        const int b = c.b, kh = c.kh, t = c.t;
        c.next(unit_off, lens, p.B, p.h_k);
        mbar_arrive_expect_tx(full_bar(s), S::kStageBytes);
        const int row = (b * p.h_k + kh) * p.L_max + t * kTileM;
        const int qrow = b * p.h_q + kh * p.g;
        const uint32_t a = smem_addr(stages + s * S::kStageBytes);
        const uint32_t bq = a + S::kParts * S::kAPart;
#pragma unroll
        for (int part = 0; part < S::kParts; ++part)
          tma_load_2d(a + part * S::kAPart, &tmap_k, part * S::kAtomElems, row, full_bar(s), pol_k);
#pragma unroll
        for (int part = 0; part < S::kParts; ++part)
          tma_load_2d(bq + part * S::kBPart, &tmap_q, part * S::kAtomElems, qrow, full_bar(s), pol_q);
      }
      // Let every load this thread issued land before the CTA can exit.
      const int first = i > S::kStages ? i - S::kStages : 0;
      for (int k = first; k < i; ++k) {
        volatile int never = 0;
        mbar_wait(full_bar(k % S::kStages), (k / S::kStages) & 1, &never);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && n_items > 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(kTileM, NPAD);
      int i = 0;
      for (; i < n_items; ++i) {
        const int s = i % S::kStages;
        const uint32_t ph = (i / S::kStages) & 1;
        const int buf = i % S::kAccBufs;
        const uint32_t aph = (i / S::kAccBufs) & 1;
        if (!mbar_wait(acce_bar(buf), aph ^ 1, abort_flag)) { raise_abort(abort_flag, p.status); break; }
        if (!mbar_wait(full_bar(s), ph, abort_flag)) { raise_abort(abort_flag, p.status); break; }
        tc_fence_after();
        const uint32_t a = smem_addr(stages + s * S::kStageBytes);
        const uint32_t bq = a + S::kParts * S::kAPart;
        const uint32_t d_tmem = tmem_base + buf * S::kAccStride;
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          constexpr int kSteps = S::kAtomElems / 16;   // MMAs per atom row
          const int part = k / kSteps;
          const uint32_t off = (k % kSteps) * 32;     // 16 bf16 = 32 bytes along the swizzled row
          const uint32_t da = a + part * S::kAPart + off, db = bq + part * S::kBPart + off;
          if constexpr (S::kAtomBytes == 128)
            tc_mma_bf16(d_tmem, smem_desc_sw128(da), smem_desc_sw128(db), idesc, k > 0 ? 1u : 0u);
          else
            tc_mma_bf16(d_tmem, smem_desc_sw64(da), smem_desc_sw64(db), idesc, k > 0 ? 1u : 0u);
        }
        tc_commit(empty_bar(s));
        tc_commit(accf_bar(buf));
      }
      if (i > 0) {   // all issued MMAs complete before TMEM is released
        volatile int never = 0;
        tc_commit(drain_bar);
        mbar_wait(drain_bar, 0, &never);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    // Warp w reads TMEM lane quarter w % 4 (the hardware rule); its set
    // (w - 2) / 4 gives its tile group (set % TG: the tiles i with i % TG equal
    // to it) and its heads [h0, h0 + H), h0 = (set / TG) * H.
    constexpr int H = S::kEpiHeads;
    constexpr int TG = S::kTileGroups;
    const int quad = warp & 3;
    const int set = (warp - 2) >> 2;
    const int tg = set % TG;
    const int h0 = (set / TG) * H;
    const uint64_t pol_z = policy_evict_last();
    bool alive = true;
    // Item i's accumulator, heads h0 .. h0 + H - 1 of this lane's position.
    auto read_acc = [&](int i, float* acc) -> bool {
      const int buf = i % S::kAccBufs;
      const uint32_t aph = (i / S::kAccBufs) & 1;
      // every lane waits; the decision to go on is taken warp-uniformly
      const bool ok = __all_sync(0xffffffffu, mbar_wait(accf_bar(buf), aph, abort_flag));
      if (!ok) { if (lane == 0) raise_abort(abort_flag, p.status); return false; }
      tc_fence_after();
#pragma unroll
      for (int cc = 0; cc < H / 8; ++cc) {
        float v[8];
        tmem_ld_8(tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + buf * S::kAccStride +
                      h0 + cc * 8, v);
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[cc * 8 + e] = v[e];
      }
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acce_bar(buf));
      return true;
    };
    if (kCand) pdl_wait();                        // t_lo comes from the preceding kernel

    uint32_t rmin[H], rmax[H];
#pragma unroll
    for (int e = 0; e < H; ++e) { rmin[e] = 0xFFFFFFFFu; rmax[e] = 0u; }
    int seg_b = -1, seg_kh = -1;
    auto flush = [&]() {
#pragma unroll
      for (int e = 0; e < H; ++e) {
        const int h = h0 + e;
        if (h < p.g) {
          const uint32_t kmin = __reduce_min_sync(0xffffffffu, rmin[e]);
          const uint32_t kmax = __reduce_max_sync(0xffffffffu, rmax[e]);
          if (lane == 0 && seg_b >= 0 && p.stat_min != nullptr && kmin <= kmax) {
            const int bj = seg_b * p.h_q + seg_kh * p.g + h;
            atomicMin(p.stat_min + bj, kmin);
            atomicMax(p.stat_max + bj, kmax);
          }
        }
        rmin[e] = 0xFFFFFFFFu;
        rmax[e] = 0u;
      }
    };
    float tl[H], mr[H];
#pragma unroll
    for (int e = 0; e < H; ++e) { tl[e] = INFINITY; mr[e] = INFINITY; }
    static_assert(kCand || !kLse, "chunk sums come with the candidate mode");
    constexpr bool lse = kLse;
    // kLse: this lane's running sums of exp(z - m_ref) over the warp's tiles of
    // the current row segment (its "piece"); when the piece ends, one butterfly
    // gives the per-head totals, which go to the slot of the piece's first
    // chunk; every other chunk of the piece gets 0 (so a row's slots still add
    // up to its sum, in a fixed order).
    float ls[H];
    int ls_chunk = -1, ls_row0 = 0;
#pragma unroll
    for (int e = 0; e < H; ++e) ls[e] = 0.0f;
    auto flush_lse = [&]() {
      if (!lse || ls_chunk < 0) return;          // uniform
      constexpr int kSpread = H <= 16 ? 2 : 1;   // lanes per head in the result
      const float sum = warp_transpose_sum<H>(ls, lane);
      const int e = lane / kSpread;
      if (lane % kSpread == 0 && e < H && h0 + e < p.g)
        st_global_hint(p.lse_part + static_cast<long long>(ls_row0 + e) * p.mask_stride + ls_chunk,
                       sum, pol_z);
#pragma unroll
      for (int e2 = 0; e2 < H; ++e2) ls[e2] = 0.0f;
      ls_chunk = -1;
    };
    if (n_tiles > 0) {
      TileCursor c;
      c.seek(u0, unit_off, lens, p.B, p.h_k);
      for (int jt = 0; jt < n_tiles; ++jt, c.next(unit_off, lens, p.B, p.h_k)) {
        const int i = jt;                         // index in the pipeline
        if (!alive || i % TG != tg) continue;
        if (c.b != seg_b || c.kh != seg_kh) {     // a new row segment
          if (!kCand) flush();
          flush_lse();
          seg_b = c.b;
          seg_kh = c.kh;
          if (kCand) {
            const int rowg = c.b * p.h_q + c.kh * p.g + h0;
#pragma unroll
            for (int e = 0; e < H; ++e) tl[e] = (h0 + e < p.g) ? __ldcg(p.t_lo + rowg + e) : INFINITY;
            if (lse) {
#pragma unroll
              for (int e = 0; e < H; ++e) mr[e] = (h0 + e < p.g) ? __ldcg(p.m_ref + rowg + e) : INFINITY;
            }
          }
        }
        float acc[H];
        if (!read_acc(i, acc)) { alive = false; continue; }
        const int row0 = c.b * p.h_q + c.kh * p.g + h0;     // z row of head h0
        const int pos = c.t * kTileM + quad * 32 + lane;
        const bool valid = pos < c.Lb;
        if (kCand) {
          const uint32_t lt = (1u << lane) - 1u;
          const int chunk = c.t * (kTileM / 32) + quad;
          uint32_t* kslot = reinterpret_cast<uint32_t*>(p.z) + static_cast<long long>(row0) * p.z_stride + chunk * 32;
          uint32_t my_m = 0u;
          if constexpr (kGroup) {
            static_assert(!kGroup || (kCand && kLse), "groups come with candidates and sums");
            // h0 = 0 and H >= g here: this lane holds every head of the key group
            float zk[H];
            uint32_t pm = 0u;                  // bit e: head e passes its bound
#pragma unroll
            for (int e = 0; e < H; ++e) {
              const float zz = __fadd_rn(__fmul_rn(acc[e], p.scale), 0.0f);
              zk[e] = zz;
              const float a = zz - mr[e];
              ls[e] += (valid && e < p.g) ? (a > kLseMaxExp ? INFINITY : __expf(a)) : 0.0f;
              pm |= (valid && e < p.g && zz >= tl[e]) ? (1u << e) : 0u;
            }
            const int grow0 = c.b * (p.h_q / g_v) + (c.kh * p.g) / g_v;   // first group row
#pragma unroll
            for (int e = 0; e < H; ++e) {
              if (e < p.g) {
                const int ge = e / g_v, eo = e - ge * g_v;
                const uint32_t gm = static_cast<uint32_t>(((1ull << g_v) - 1ull) << (ge * g_v));
                const bool take = (pm & gm) != 0u;
                const uint32_t m = __ballot_sync(0xffffffffu, take);
                if (eo == 0 && lane == ge) my_m = m;
                if (take) {
                  uint32_t* gslot = reinterpret_cast<uint32_t*>(p.z) +
                      static_cast<long long>(grow0 + ge) * g_v * p.z_stride +
                      static_cast<long long>(chunk) * 32 * g_v;
                  st_global_hint(gslot + __popc(m & lt) * g_v + eo, ordered_key(zk[e]), pol_z);
                }
              }
            }
            const int ng = p.g / g_v;
            if (lane < ng && chunk * 32 < c.Lb)                   // lane v': group v''s mask
              st_global_hint(p.cand_mask + static_cast<long long>(grow0 + lane) * p.mask_stride + chunk,
                             my_m, pol_z);
          } else {
#pragma unroll
          for (int e = 0; e < H; ++e) {
            // fp32 dot product, then one fp32 scale; -0 canonicalised to +0.
            const float zz = __fadd_rn(__fmul_rn(acc[e], p.scale), 0.0f);
            if (lse) {   // exp(-inf) = 0 for rows without a reference
              const float a = zz - mr[e];
              ls[e] += (valid && h0 + e < p.g) ? (a > kLseMaxExp ? INFINITY : __expf(a)) : 0.0f;
            }
            const bool take = valid && h0 + e < p.g && zz >= tl[e];
            const uint32_t m = __ballot_sync(0xffffffffu, take);
            if (lane == e) my_m = m;
            // candidates are written L2-evict-last (the K stream is evict-first), so
            // that the selector finds them in L2
            if (take) st_global_hint(kslot + e * p.z_stride + __popc(m & lt), ordered_key(zz), pol_z);
          }
          if (lane < H && h0 + lane < p.g && chunk * 32 < c.Lb)   // lane e: head e's mask
            st_global_hint(p.cand_mask + static_cast<long long>(row0 + lane) * p.mask_stride + chunk, my_m, pol_z);
          }
          if (lse && chunk * 32 < c.Lb) {
            if (ls_chunk < 0) {                  // the piece's first chunk takes its total
              ls_chunk = chunk;
              ls_row0 = row0;
            } else if (lane < H && h0 + lane < p.g) {
              st_global_hint(p.lse_part + static_cast<long long>(row0 + lane) * p.mask_stride + chunk,
                             0.0f, pol_z);
            }
          }
        } else if (valid) {
          float* zrow = p.z + static_cast<long long>(row0) * p.z_stride + pos;
#pragma unroll
          for (int e = 0; e < H; ++e) {
            if (h0 + e < p.g) {
              // fp32 dot product, then one fp32 scale; -0 canonicalised to +0.
              const float zz = __fadd_rn(__fmul_rn(acc[e], p.scale), 0.0f);
              st_global_hint(zrow + e * p.z_stride, zz, pol_z);
              const uint32_t key = ordered_key(zz);
              rmin[e] = min(rmin[e], key);
              rmax[e] = max(rmax[e], key);
            }
          }
        }
      }
      if (!kCand) flush();
      flush_lse();
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, S::kTmemCols);
  }
}

}  // namespace saga
