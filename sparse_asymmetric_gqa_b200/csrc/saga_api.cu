// saga_api.cu -- the C ABI declared in include/saga.h: argument validation,
// the handle and its workspace, TMA descriptor encoding and the launch plan.
//
// A decode call enqueues four kernels on the handle's stream (the candidate path):
//   sample_kernel  1024 sampled scores per (batch row, query head), CUDA cores
//   bound_kernel   a lower bound t_lo for the selection threshold of each row
//   score_kernel   S1, persistent, one CTA per SM (tcgen05 + TMA), keeping the
//                  scores >= t_lo as candidates
//   topn_kernel    S2 + S3 + S4 from the candidates, one CTA per (b, j)
// The calibration call and a step of stateful Atop-N run the same four, the
// score pass also summing exp(z - m_ref) per chunk for the row's log-sum-exp.
// Selections wider than the candidate path takes (N > 2048) run three:
//   score_kernel   S1, every score to the workspace
//   select_kernel  S2, one CTA per (batch row, query head)
//   gather_kernel  S3 + S4, one CTA per 256 selected rows of a (b, j)
// Nothing is allocated, synchronised or copied to the host on either path.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <new>
#include <utility>
#include <vector>

#include "saga.h"
#include "ptx.cuh"
#include "score_kernel.cuh"
#include "select_kernel.cuh"
#include "gather_kernel.cuh"
#include "topn_kernel.cuh"
#include "bound_kernel.cuh"
#include "group_kernel.cuh"

using namespace saga;

namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, []() {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 2-D bf16 tensor [rows][cols] (cols contiguous), box {64, box_rows}, 128-byte swizzle.
bool encode_bf16_2d(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                    uint32_t box_rows) {
  EncodeTiledFn fn = get_encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  // rows of 64 or more elements: 64-element boxes, 128-byte swizzle; 32-element
  // rows (keys of width 32): one 64-byte box row, 64-byte swizzle
  cuuint32_t box[2] = {static_cast<cuuint32_t>(cols < 64 ? cols : 64), box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  cols < 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

int round_up(int x, int m) { return (x + m - 1) / m * m; }

}  // namespace

struct saga_ctx {
  int device = 0;
  int num_sms = 0;
  int max_batch = 0, batch = 0, max_seq_len = 0, h_q = 0, h_k = 0, h_v = 0, d = 0, max_N = 0;
  int dv = 0;                     // value and output width (d: the query and key width)
  int g = 0, g_v = 0, npad = 0;
  long long z_stride = 0;
  cudaStream_t stream = nullptr;
  // workspace (one allocation)
  void* ws = nullptr;
  float* z = nullptr;
  uint32_t* stat_min = nullptr;
  uint32_t* stat_max = nullptr;
  int32_t* sel_idx = nullptr;
  float* sel_logit = nullptr;
  int* status = nullptr;
  __nv_bfloat16* q_stage = nullptr;
  __nv_bfloat16* out_stage = nullptr;
  int32_t* lens_stage = nullptr;
  float scale = 0.0f;             // 1/sqrt(d) rounded to fp32 (d the key width)
  uint32_t* cand_mask = nullptr;  // candidate chunk masks [rows][mask_stride]
  long long mask_stride = 0;      // z_stride / 32
  float* samp = nullptr;          // sampled scores [rows][kSampleSize]
  float* t_lo = nullptr;          // candidate bounds [rows]
  float* m_ref = nullptr;         // exp-sum references [rows] (calibration and steps)
  float* lse_part = nullptr;      // chunk sums of exp(z - m_ref) [rows][mask_stride]
  uint32_t* gstat = nullptr;      // group statistic keys [max_batch * h_v][z_stride]
  float* gsel_stat = nullptr;     // group statistic at the selection [max_batch * h_v][max_N]
  float* partial = nullptr;       // gather partials [rows][max_chunks][d + 2]
  uint32_t* counter = nullptr;    // gather merge counters [rows]
  int max_chunks = 0;
  long long launches = 0;
  // profiling
  bool prof = false;
  int prof_max = 0, prof_n = 0;
  std::vector<cudaEvent_t> ev;   // 4 per recorded call: start, score start, score end, end
};

namespace {

int set_smem_attrs_once() {
  static int rc = -1;
  static std::once_flag once;
  std::call_once(once, []() {
    cudaError_t e = cudaSuccess;
#define SAGA_ATTR(D, NP)                                                                          \
  if (e == cudaSuccess)                                                                           \
    e = cudaFuncSetAttribute(score_kernel<D, NP, false>,                                          \
                             cudaFuncAttributeMaxDynamicSharedMemorySize, ScoreShape<D, NP>::kSmemBytes); \
  if (e == cudaSuccess)                                                                           \
    e = cudaFuncSetAttribute(score_kernel<D, NP, true>,                                           \
                             cudaFuncAttributeMaxDynamicSharedMemorySize, ScoreShape<D, NP>::kSmemBytes); \
  if (e == cudaSuccess)                                                                           \
    e = cudaFuncSetAttribute(score_kernel<D, NP, true, true>,                                     \
                             cudaFuncAttributeMaxDynamicSharedMemorySize, ScoreShape<D, NP>::kSmemBytes);
    SAGA_ATTR(32, 16) SAGA_ATTR(32, 32) SAGA_ATTR(32, 48) SAGA_ATTR(32, 64)
    SAGA_ATTR(64, 16) SAGA_ATTR(64, 32) SAGA_ATTR(64, 48) SAGA_ATTR(64, 64)
    SAGA_ATTR(128, 16) SAGA_ATTR(128, 32) SAGA_ATTR(128, 48) SAGA_ATTR(128, 64)
#undef SAGA_ATTR
#define SAGA_GATTR(D, NP)                                                                         \
  if (e == cudaSuccess)                                                                           \
    e = cudaFuncSetAttribute(score_kernel<D, NP, true, true, true>,                               \
                             cudaFuncAttributeMaxDynamicSharedMemorySize, ScoreShape<D, NP>::kSmemBytes);
    SAGA_GATTR(64, 16) SAGA_GATTR(64, 32) SAGA_GATTR(128, 16) SAGA_GATTR(128, 32)
#undef SAGA_GATTR
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(sizeof(SelectSmem)));
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(group_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(GroupLayout::kBytes));
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(group_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(GroupLayout::kBytes));
#define SAGA_TOPN_ATTR(D, M, S)                                                                   \
  if (e == cudaSuccess)                                                                           \
    e = cudaFuncSetAttribute(topn_kernel<D, M, S>, cudaFuncAttributeMaxDynamicSharedMemorySize,   \
                             static_cast<int>(TopnLayout<S>::kBytes));
    SAGA_TOPN_ATTR(64, kModeExact, kTopnSelNarrow) SAGA_TOPN_ATTR(128, kModeExact, kTopnSelNarrow)
    SAGA_TOPN_ATTR(64, kModeCalibrate, kTopnSelNarrow) SAGA_TOPN_ATTR(128, kModeCalibrate, kTopnSelNarrow)
    SAGA_TOPN_ATTR(64, kModeStep, kTopnSelNarrow) SAGA_TOPN_ATTR(128, kModeStep, kTopnSelNarrow)
    SAGA_TOPN_ATTR(64, kModeStep, kTopnSelMax) SAGA_TOPN_ATTR(128, kModeStep, kTopnSelMax)
#undef SAGA_TOPN_ATTR
    // the exact kernel's other variants: long rows, and key widths other than the value width
    for (const void* f : {reinterpret_cast<const void*>(topn_kernel<64, kModeExact, kTopnSelNarrow, kTopnLongRun>),
                          reinterpret_cast<const void*>(topn_kernel<128, kModeExact, kTopnSelNarrow, kTopnLongRun>),
                          reinterpret_cast<const void*>(topn_kernel<64, kModeExact, kTopnSelNarrow, kTopnRun, 128>),
                          reinterpret_cast<const void*>(topn_kernel<64, kModeExact, kTopnSelNarrow, kTopnLongRun, 128>),
                          reinterpret_cast<const void*>(topn_kernel<128, kModeExact, kTopnSelNarrow, kTopnRun, 64>),
                          reinterpret_cast<const void*>(topn_kernel<128, kModeExact, kTopnSelNarrow, kTopnLongRun, 64>),
                          reinterpret_cast<const void*>(topn_kernel<64, kModeExact, kTopnSelNarrow, kTopnRun, 32>),
                          reinterpret_cast<const void*>(topn_kernel<64, kModeExact, kTopnSelNarrow, kTopnLongRun, 32>),
                          reinterpret_cast<const void*>(topn_kernel<128, kModeExact, kTopnSelNarrow, kTopnRun, 32>),
                          reinterpret_cast<const void*>(topn_kernel<128, kModeExact, kTopnSelNarrow, kTopnLongRun, 32>)})
      if (e == cudaSuccess)
        e = cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(TopnLayout<kTopnSelNarrow>::kBytes));
    rc = (e == cudaSuccess) ? 0 : 1;
  });
  return rc;
}

// Launch on the handle's stream.  kPdl: the kernel may start before the
// previous kernel in the stream has finished (it waits in-kernel before it
// reads that kernel's results: programmatic dependent launch).  kCoop: all
// CTAs are resident at once (cooperative launch; the kernel synchronises
// across the grid).
enum LaunchMode { kPlain = 0, kPdl = 1, kCoop = 2 };
template <typename... KArgs, typename... Args>
cudaError_t launch(saga_ctx* h, void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                   int mode, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = h->stream;
  cudaLaunchAttribute attr[1];
  if (mode == kPdl) {
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
  } else {
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
  }
  cfg.attrs = attr;
  cfg.numAttrs = (mode == kPlain) ? 0 : 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
  if (e == cudaSuccess) ++h->launches;
  return e;
}

// Score pass.  cand: candidate mode (bounds from h->t_lo, chunk masks and
// candidate keys in the workspace; a programmatic dependent of the bound
// kernel); otherwise every score goes to z.
int launch_score(saga_ctx* h, const void* q, const void* k_cache, const int32_t* seq_lens,
                 float* z, long long z_stride, bool stats, bool cand = false, bool lse = false,
                 bool group = false) {
  CUtensorMap mk, mq;
  const uint64_t k_rows = static_cast<uint64_t>(h->batch) * h->h_k * h->max_seq_len;
  const uint64_t q_rows = static_cast<uint64_t>(h->batch) * h->h_q;
  if (!encode_bf16_2d(&mk, k_cache, k_rows, h->d, kTileM)) return SAGA_ERR_CUDA;
  if (!encode_bf16_2d(&mq, q, q_rows, h->d, h->npad)) return SAGA_ERR_CUDA;
  ScoreParams p;
  std::memset(&p, 0, sizeof(p));
  p.seq_lens = seq_lens;
  p.z = z;
  p.cand_mask = h->cand_mask;
  p.mask_stride = h->mask_stride;
  p.t_lo = h->t_lo;
  p.m_ref = h->m_ref;
  p.lse_part = (cand && lse) ? h->lse_part : nullptr;
  p.stat_min = (stats && !cand) ? h->stat_min : nullptr;
  p.stat_max = (stats && !cand) ? h->stat_max : nullptr;
  p.status = h->status;
  p.B = h->batch;
  p.h_q = h->h_q;
  p.h_k = h->h_k;
  p.g = h->g;
  p.L_max = h->max_seq_len;
  p.z_stride = z_stride;
  p.scale = h->scale;
  const long long max_units =
      static_cast<long long>(h->batch) * h->h_k * ((h->max_seq_len + kTileM - 1) / kTileM);
  const int grid = static_cast<int>(max_units < h->num_sms ? max_units : h->num_sms);
  cudaError_t e = cudaErrorInvalidValue;
  if (group) {   // group candidates (g <= 32)
#define SAGA_GCASE(D, NP)                                                                      \
    if (h->d == D && h->npad == NP)                                                            \
      e = launch(h, score_kernel<D, NP, true, true, true>, dim3(grid), dim3(kScoreThreads),    \
                 ScoreShape<D, NP>::kSmemBytes, kPdl, mk, mq, p, h->g_v);
    SAGA_GCASE(64, 16) SAGA_GCASE(64, 32) SAGA_GCASE(128, 16) SAGA_GCASE(128, 32)
#undef SAGA_GCASE
    return e == cudaSuccess ? SAGA_OK : SAGA_ERR_CUDA;
  }
#define SAGA_CASE(D, NP)                                                                       \
  if (h->d == D && h->npad == NP)                                                              \
    e = (cand && lse) ? launch(h, score_kernel<D, NP, true, true>, dim3(grid), dim3(kScoreThreads), \
                               ScoreShape<D, NP>::kSmemBytes, kPdl, mk, mq, p, h->g_v)                  \
      : cand ? launch(h, score_kernel<D, NP, true>, dim3(grid), dim3(kScoreThreads),           \
                      ScoreShape<D, NP>::kSmemBytes, kPdl, mk, mq, p, h->g_v)                          \
             : launch(h, score_kernel<D, NP, false>, dim3(grid), dim3(kScoreThreads),          \
                      ScoreShape<D, NP>::kSmemBytes, kPlain, mk, mq, p, h->g_v);
  SAGA_CASE(32, 16) SAGA_CASE(32, 32) SAGA_CASE(32, 48) SAGA_CASE(32, 64)
  SAGA_CASE(64, 16) SAGA_CASE(64, 32) SAGA_CASE(64, 48) SAGA_CASE(64, 64)
  SAGA_CASE(128, 16) SAGA_CASE(128, 32) SAGA_CASE(128, 48) SAGA_CASE(128, 64)
#undef SAGA_CASE
  return e == cudaSuccess ? SAGA_OK : SAGA_ERR_CUDA;
}

// The exact top-N kernel for value width DV and key width DK, with the 16-chunk
// candidate path for caches of more than 65536 positions.
template <int DV, int DK>
cudaError_t launch_topn_exact(saga_ctx* h, dim3 grid, dim3 block, size_t smem, const TopnParams& p,
                              bool long_rows) {
  return long_rows
      ? launch(h, topn_kernel<DV, kModeExact, kTopnSelNarrow, kTopnLongRun, DK>, grid, block, smem, kPdl, p)
      : launch(h, topn_kernel<DV, kModeExact, kTopnSelNarrow, kTopnRun, DK>, grid, block, smem, kPdl, p);
}

// Candidate bounds for the n_target largest scores of each row: the sample
// kernel (after the previous kernel in the stream) and the bound kernel (a
// programmatic dependent of it); with ref, also the exp-sum references.
int launch_bounds(saga_ctx* h, const void* q, const void* k_cache, const int32_t* seq_lens,
                  int n_target, bool ref) {
  BoundParams p;
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.k_cache = static_cast<const __nv_bfloat16*>(k_cache);
  p.seq_lens = seq_lens;
  p.h_q = h->h_q;
  p.h_k = h->h_k;
  p.g = h->g;
  p.L_max = h->max_seq_len;
  p.N = n_target;
  p.cand_cap = kTopnCap;
  p.scale = h->scale;
  p.samp = h->samp;
  p.t_lo = h->t_lo;
  p.m_ref = ref ? h->m_ref : nullptr;
  const dim3 sgrid(h->batch * h->h_k, kSampleParts);
  const size_t smem = static_cast<size_t>(h->g) * h->d * sizeof(float);
  cudaError_t e = (h->d == 32)
      ? launch(h, sample_kernel<32>, sgrid, dim3(kSampleThreads), smem, kPlain, p)
      : (h->d == 64)
      ? launch(h, sample_kernel<64>, sgrid, dim3(kSampleThreads), smem, kPlain, p)
      : launch(h, sample_kernel<128>, sgrid, dim3(kSampleThreads), smem, kPlain, p);
  if (e == cudaSuccess) e = launch(h, bound_kernel, dim3(h->batch * h->h_q), dim3(32), 0, kPdl, p);
  return e == cudaSuccess ? SAGA_OK : SAGA_ERR_CUDA;
}

// S2-S4 from the candidate lists (a programmatic dependent of the score pass).
int launch_topn(saga_ctx* h, const void* q, const void* k_cache, const void* v_cache,
                const int32_t* seq_lens, int N, int32_t* sel_idx, float* sel_logit, void* out,
                int mode, float* log_tau) {
  TopnParams p;
  p.cand_mask = h->cand_mask;
  p.mask_stride = h->mask_stride;
  p.zkey = reinterpret_cast<uint32_t*>(h->z);
  p.z_stride = h->z_stride;
  p.seq_lens = seq_lens;
  p.h_q = h->h_q;
  p.h_k = h->h_k;
  p.g = h->g;
  p.h_v = h->h_v;
  p.g_v = h->g_v;
  p.L_max = h->max_seq_len;
  p.N = N;
  p.cap = mode == kModeStep ? 2 * N : N;
  p.cand_cap = kTopnCap;
  p.lse_part = h->lse_part;
  p.m_ref = h->m_ref;
  p.t_lo = h->t_lo;
  p.log_tau = log_tau;
  p.sel_idx = sel_idx;
  p.sel_logit = sel_logit;
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.k_cache = static_cast<const __nv_bfloat16*>(k_cache);
  p.v_cache = static_cast<const __nv_bfloat16*>(v_cache);
  p.scale = h->scale;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.status = h->status;
  const dim3 grid(h->batch * h->h_q);
  const dim3 block(kTopnThreads);
  constexpr size_t narrow = TopnLayout<kTopnSelNarrow>::kBytes, wide = TopnLayout<kTopnSelMax>::kBytes;
  cudaError_t e;
  if (mode == kModeExact) {
    const bool long_rows = h->max_seq_len > kTopnThreads * 32 * kTopnRun;
    if (h->dv == 64 && h->d == 64) e = launch_topn_exact<64, 64>(h, grid, block, narrow, p, long_rows);
    else if (h->dv == 128 && h->d == 128) e = launch_topn_exact<128, 128>(h, grid, block, narrow, p, long_rows);
    else if (h->dv == 128 && h->d == 64) e = launch_topn_exact<128, 64>(h, grid, block, narrow, p, long_rows);
    else if (h->dv == 64 && h->d == 128) e = launch_topn_exact<64, 128>(h, grid, block, narrow, p, long_rows);
    else if (h->dv == 128) e = launch_topn_exact<128, 32>(h, grid, block, narrow, p, long_rows);
    else e = launch_topn_exact<64, 32>(h, grid, block, narrow, p, long_rows);
  } else if (mode == kModeCalibrate)
    e = (h->d == 64) ? launch(h, topn_kernel<64, kModeCalibrate, kTopnSelNarrow>, grid, block, narrow, kPdl, p)
                     : launch(h, topn_kernel<128, kModeCalibrate, kTopnSelNarrow>, grid, block, narrow, kPdl, p);
  else if (p.cap <= kTopnSelNarrow)
    e = (h->d == 64) ? launch(h, topn_kernel<64, kModeStep, kTopnSelNarrow>, grid, block, narrow, kPdl, p)
                     : launch(h, topn_kernel<128, kModeStep, kTopnSelNarrow>, grid, block, narrow, kPdl, p);
  else
    e = (h->d == 64) ? launch(h, topn_kernel<64, kModeStep, kTopnSelMax>, grid, block, wide, kPdl, p)
                     : launch(h, topn_kernel<128, kModeStep, kTopnSelMax>, grid, block, wide, kPdl, p);
  return e == cudaSuccess ? SAGA_OK : SAGA_ERR_CUDA;
}

int launch_select(saga_ctx* h, const float* z, long long z_stride, bool stats,
                  const int32_t* seq_lens, int N, int32_t* sel_idx, float* sel_logit) {
  SelectParams p;
  p.z = z;
  p.z_stride = z_stride;
  p.stat_min = stats ? h->stat_min : nullptr;
  p.stat_max = stats ? h->stat_max : nullptr;
  p.gather_count = h->counter;
  p.seq_lens = seq_lens;
  p.B = h->batch;
  p.h_q = h->h_q;
  p.L_max = h->max_seq_len;
  p.N = N;
  p.z_vec4 = ((z_stride % 4) == 0 && (reinterpret_cast<uintptr_t>(z) % 16) == 0) ? 1 : 0;
  p.sel_idx = sel_idx;
  p.sel_logit = sel_logit;
  p.status = h->status;
  const cudaError_t e = launch(h, select_kernel, dim3(h->batch * h->h_q), dim3(kSelThreads),
                               sizeof(SelectSmem), kPlain, p);
  return e == cudaSuccess ? SAGA_OK : SAGA_ERR_CUDA;
}

int launch_gather(saga_ctx* h, const int32_t* sel_idx, const float* sel_logit,
                  const int32_t* seq_lens, const void* v_cache, int N, void* out, bool pdl) {
  GatherParams p;
  p.sel_idx = sel_idx;
  p.sel_logit = sel_logit;
  p.seq_lens = seq_lens;
  p.v_cache = static_cast<const __nv_bfloat16*>(v_cache);
  p.h_q = h->h_q;
  p.h_v = h->h_v;
  p.g_v = h->g_v;
  p.L_max = h->max_seq_len;
  p.N = N;
  p.partial = h->partial;
  p.max_chunks = h->max_chunks;
  p.counter = h->counter;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.status = h->status;
  const int slots = N < h->max_seq_len ? N : h->max_seq_len;
  const dim3 grid(h->batch * h->h_q, (slots + kGatherRows - 1) / kGatherRows);
  const cudaError_t e = (h->dv == 64)
      ? launch(h, gather_kernel<64>, grid, dim3(kGatherThreads), 0, pdl ? kPdl : kPlain, p)
      : launch(h, gather_kernel<128>, grid, dim3(kGatherThreads), 0, pdl ? kPdl : kPlain, p);
  return e == cudaSuccess ? SAGA_OK : SAGA_ERR_CUDA;
}

// Failure-detection self-test: one thread waits, with the pipeline's bounded
// wait, on an mbarrier that nothing arrives at; when the wait gives up it sets
// SAGA_STATUS_TIMEOUT, as a stalled pipeline stage would.
__global__ void selftest_wait_kernel(int* status) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    const uint32_t b = smem_addr(&bar);
    mbar_init(b, 1);
    fence_mbar_init();
    volatile int never = 0;
    if (!mbar_wait(b, 0, &never)) atomicOr(status, 0x2 /* SAGA_STATUS_TIMEOUT */);
  }
}

// Group-shared selection: S2-S4 per value-head group (a programmatic dependent
// of the group variant of the score pass).
int launch_group(saga_ctx* h, const void* q, const void* k_cache, const void* v_cache,
                 const int32_t* seq_lens, int N, int32_t* sel_idx, float* sel_stat,
                 float* sel_logit, void* out) {
  GroupParams p;
  p.cand_mask = h->cand_mask;
  p.mask_stride = h->mask_stride;
  p.zkey = reinterpret_cast<uint32_t*>(h->z);
  p.z_stride = h->z_stride;
  p.gstat = h->gstat;
  p.seq_lens = seq_lens;
  p.h_q = h->h_q;
  p.h_k = h->h_k;
  p.g = h->g;
  p.h_v = h->h_v;
  p.g_v = h->g_v;
  p.L_max = h->max_seq_len;
  p.N = N;
  p.cand_cap = kTopnCap;
  p.lse_part = h->lse_part;
  p.m_ref = h->m_ref;
  p.t_lo = h->t_lo;
  p.sel_idx = sel_idx;
  p.sel_stat = sel_stat;
  p.sel_logit = sel_logit;
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.k_cache = static_cast<const __nv_bfloat16*>(k_cache);
  p.v_cache = static_cast<const __nv_bfloat16*>(v_cache);
  p.scale = h->scale;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.status = h->status;
  const dim3 grid(h->batch * h->h_v);
  constexpr size_t smem = GroupLayout::kBytes;
  const cudaError_t e = (h->d == 64)
      ? launch(h, group_kernel<64>, grid, dim3(kTopnThreads), smem, kPdl, p)
      : launch(h, group_kernel<128>, grid, dim3(kTopnThreads), smem, kPdl, p);
  return e == cudaSuccess ? SAGA_OK : SAGA_ERR_CUDA;
}

int check_heads(saga_ctx* h, int h_q, int h_k, int h_v, int d) {
  if (h_q != h->h_q || h_k != h->h_k || h_v != h->h_v || d != h->d) return SAGA_ERR_INVALID_ARG;
  return SAGA_OK;
}

// Inside stream capture an event record becomes a graph node only with the
// external flag; then each replay re-records it and elapsed times stay valid.
cudaError_t record_event(cudaEvent_t e, cudaStream_t s) {
  cudaStreamCaptureStatus st = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(s, &st) == cudaSuccess && st == cudaStreamCaptureStatusActive)
    return cudaEventRecordWithFlags(e, s, cudaEventRecordExternal);
  return cudaEventRecord(e, s);
}

struct DeviceGuard {   // run a call on the handle's device, restore the caller's
  int prev = -1;
  bool ok = true;
  explicit DeviceGuard(int dev) {
    if (cudaGetDevice(&prev) != cudaSuccess) { ok = false; return; }
    if (prev != dev && cudaSetDevice(dev) != cudaSuccess) ok = false;
  }
  ~DeviceGuard() {
    int cur = -1;
    if (prev >= 0 && cudaGetDevice(&cur) == cudaSuccess && cur != prev) cudaSetDevice(prev);
  }
};

// q, the caches and the score rows are read with 16-byte vector loads, TMA and
// asynchronous copies: their base addresses must be 16-byte aligned.
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// The candidate path (sampled bounds -> score pass with fused compare ->
// selection from candidates -> gather) needs the candidate lists and a selection small
// enough for them; otherwise every score goes through the score workspace.
bool use_candidates(const saga_ctx* h, int N) {
  return h->cand_mask != nullptr && N <= kTopnSelNarrow && N <= kTopnCap / 4 && h->dv <= kTopnMaxD &&
         (N < h->max_seq_len || h->max_seq_len <= kTopnCap);
}

// mode: kModeExact (the decode step), kModeCalibrate (also writes log_tau) or
// kModeStep (selects with log_tau; selection rows of width 2N).
int decode_impl(saga_ctx* h, const void* q, const void* k_cache, const void* v_cache,
                const int32_t* seq_lens, int N, void* out, int32_t* sel_idx, float* sel_logit,
                int mode = kModeExact, float* log_tau = nullptr) {
  if (!q || !k_cache || !v_cache || !seq_lens || !out) return SAGA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache)) return SAGA_ERR_INVALID_ARG;
  if (N < 1 || N > h->max_N) return SAGA_ERR_INVALID_ARG;
  if (mode != kModeExact) {
    if (!log_tau) return SAGA_ERR_INVALID_ARG;
    if (!use_candidates(h, N) || 2 * N > kTopnSelMax) return SAGA_ERR_UNSUPPORTED;
  }
  DeviceGuard dg(h->device);
  if (!dg.ok) return SAGA_ERR_CUDA;
  const bool prof = h->prof && h->prof_n < h->prof_max;
  cudaEvent_t* ev = prof ? &h->ev[4 * h->prof_n] : nullptr;
  // The selection goes to the caller's arrays when given, else to the workspace
  // (row stride N either way).
  int32_t* si = sel_idx ? sel_idx : h->sel_idx;
  float* sl = sel_logit ? sel_logit : h->sel_logit;
  if (prof && record_event(ev[0], h->stream) != cudaSuccess) return SAGA_ERR_CUDA;
  int rc;
  if (use_candidates(h, N)) {
    // a step keeps up to 2N entries: its candidates cover the 2N largest scores
    const int n_target = mode == kModeStep ? 2 * N : N;
    const bool lse = mode != kModeExact;
    if ((rc = launch_bounds(h, q, k_cache, seq_lens, n_target, lse))) return rc;
    if (prof && record_event(ev[1], h->stream) != cudaSuccess) return SAGA_ERR_CUDA;
    if ((rc = launch_score(h, q, k_cache, seq_lens, h->z, h->z_stride, false, true, lse))) return rc;
    if (prof && record_event(ev[2], h->stream) != cudaSuccess) return SAGA_ERR_CUDA;
    if ((rc = launch_topn(h, q, k_cache, v_cache, seq_lens, N, si, sl, out, mode, log_tau))) return rc;
  } else {
    if (prof && record_event(ev[1], h->stream) != cudaSuccess) return SAGA_ERR_CUDA;
    if ((rc = launch_score(h, q, k_cache, seq_lens, h->z, h->z_stride, true))) return rc;
    if (prof && record_event(ev[2], h->stream) != cudaSuccess) return SAGA_ERR_CUDA;
    if ((rc = launch_select(h, h->z, h->z_stride, true, seq_lens, N, si, sl))) return rc;
    if ((rc = launch_gather(h, si, sl, seq_lens, v_cache, N, out, true))) return rc;
  }
  if (prof) {
    if (record_event(ev[3], h->stream) != cudaSuccess) return SAGA_ERR_CUDA;
    ++h->prof_n;
  }
  return SAGA_OK;
}

}  // namespace

extern "C" {

const char* saga_decode_error_string(int code) {
  switch (code) {
    case SAGA_OK: return "ok";
    case SAGA_ERR_INVALID_ARG: return "invalid argument";
    case SAGA_ERR_UNSUPPORTED: return "unsupported configuration or device";
    case SAGA_ERR_CUDA: return "CUDA call failed";
    case SAGA_ERR_DEVICE: return "device reported an error (see saga_decode_status)";
    case SAGA_ERR_SCRATCH_TOO_SMALL:
      return "problem too large for the fixed scratch of saga_combine_noalloc (4 MiB)";
    default: return "unknown error code";
  }
}

int saga_decode_init(saga_handle* handle, int max_batch, int max_seq_len, int h_q, int h_k,
                     int h_v, int head_dim, int max_N, void* cuda_stream) {
  return saga_decode_init_kv(handle, max_batch, max_seq_len, h_q, h_k, h_v, head_dim, head_dim, max_N,
                             cuda_stream);
}

int saga_decode_init_kv(saga_handle* handle, int max_batch, int max_seq_len, int h_q, int h_k,
                        int h_v, int head_dim, int head_dim_v, int max_N, void* cuda_stream) {
  if (!handle) return SAGA_ERR_INVALID_ARG;
  *handle = nullptr;
  if (max_batch < 1 || max_batch > kMaxBatch) return SAGA_ERR_INVALID_ARG;
  if (max_seq_len < 1 || max_seq_len > (1 << 24)) return SAGA_ERR_INVALID_ARG;
  if (h_q < 1 || h_k < 1 || h_v < 1 || max_N < 1) return SAGA_ERR_INVALID_ARG;
  if (h_q % h_k != 0 || h_q % h_v != 0) return SAGA_ERR_INVALID_ARG;
  if (static_cast<long long>(max_batch) * h_k * max_seq_len >= (1ll << 31)) return SAGA_ERR_INVALID_ARG;
  if (static_cast<long long>(max_batch) * h_q > (1ll << 30)) return SAGA_ERR_INVALID_ARG;
  if (head_dim != 32 && head_dim != 64 && head_dim != 128) return SAGA_ERR_UNSUPPORTED;
  if (head_dim_v != 64 && head_dim_v != 128) return SAGA_ERR_UNSUPPORTED;
  const int g = h_q / h_k;
  if (g > 64) return SAGA_ERR_UNSUPPORTED;

  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SAGA_ERR_CUDA;
  cudaDeviceProp prop;
  if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) return SAGA_ERR_CUDA;
  if (prop.major != 10) return SAGA_ERR_UNSUPPORTED;
  if (set_smem_attrs_once() != 0) return SAGA_ERR_CUDA;
  if (!get_encode_fn()) return SAGA_ERR_CUDA;

  saga_ctx* h = new (std::nothrow) saga_ctx();
  if (!h) return SAGA_ERR_CUDA;
  h->device = dev;
  h->num_sms = prop.multiProcessorCount;
  h->max_batch = h->batch = max_batch;
  h->max_seq_len = max_seq_len;
  h->h_q = h_q; h->h_k = h_k; h->h_v = h_v; h->d = head_dim; h->max_N = max_N;
  h->dv = head_dim_v;
  h->g = g; h->g_v = h_q / h_v;
  h->npad = round_up(g, 16);
  h->z_stride = round_up(max_seq_len, 32);
  h->stream = static_cast<cudaStream_t>(cuda_stream);

  const size_t rows = static_cast<size_t>(max_batch) * h_q;
  const size_t z_bytes = rows * h->z_stride * sizeof(float);
  const size_t stat_bytes = rows * sizeof(uint32_t);
  const size_t sel_bytes = rows * static_cast<size_t>(max_N) * 2 * 4;   // a step keeps up to 2N
  const size_t qo_bytes = rows * (head_dim > head_dim_v ? head_dim : head_dim_v) * 2;
  const int slots = max_N < max_seq_len ? max_N : max_seq_len;
  h->max_chunks = (slots + kGatherRows - 1) / kGatherRows;
  const size_t part_bytes = rows * h->max_chunks * (head_dim_v + 2) * sizeof(float);
  auto al = [](size_t x) { return (x + 255) & ~static_cast<size_t>(255); };
  // candidate path: chunk masks (the keys reuse z), sampled scores, bounds
  h->mask_stride = h->z_stride / 32;
  const size_t mask_bytes = rows * static_cast<size_t>(h->mask_stride) * 4;
  const size_t samp_bytes = rows * static_cast<size_t>(kSampleSize) * 4;
  // group-shared selection: statistic keys per value-head row, and s at the selection
  const size_t rows_v = static_cast<size_t>(max_batch) * h_v;
  const size_t gstat_bytes = rows_v * static_cast<size_t>(h->z_stride) * 4;
  const size_t gsel_bytes = rows_v * static_cast<size_t>(max_N) * 4;
  const size_t total = al(z_bytes) + 2 * al(stat_bytes) + 2 * al(sel_bytes) + al(256) +
                       2 * al(qo_bytes) + al(static_cast<size_t>(max_batch) * 4) +
                       al(part_bytes) + 2 * al(stat_bytes) + al(mask_bytes) + al(samp_bytes) +
                       al(stat_bytes) + al(mask_bytes) + al(gstat_bytes) + al(gsel_bytes);
  if (cudaMalloc(&h->ws, total) != cudaSuccess) { delete h; return SAGA_ERR_CUDA; }
  uint8_t* w = static_cast<uint8_t*>(h->ws);
  h->z = reinterpret_cast<float*>(w); w += al(z_bytes);
  h->stat_min = reinterpret_cast<uint32_t*>(w); w += al(stat_bytes);
  h->stat_max = reinterpret_cast<uint32_t*>(w); w += al(stat_bytes);
  h->sel_idx = reinterpret_cast<int32_t*>(w); w += al(sel_bytes);
  h->sel_logit = reinterpret_cast<float*>(w); w += al(sel_bytes);
  h->status = reinterpret_cast<int*>(w); w += al(256);
  h->q_stage = reinterpret_cast<__nv_bfloat16*>(w); w += al(qo_bytes);
  h->out_stage = reinterpret_cast<__nv_bfloat16*>(w); w += al(qo_bytes);
  h->lens_stage = reinterpret_cast<int32_t*>(w); w += al(static_cast<size_t>(max_batch) * 4);
  h->partial = reinterpret_cast<float*>(w); w += al(part_bytes);
  h->counter = reinterpret_cast<uint32_t*>(w); w += al(stat_bytes);
  h->cand_mask = reinterpret_cast<uint32_t*>(w); w += al(mask_bytes);
  h->samp = reinterpret_cast<float*>(w); w += al(samp_bytes);
  h->t_lo = reinterpret_cast<float*>(w); w += al(stat_bytes);
  h->m_ref = reinterpret_cast<float*>(w); w += al(stat_bytes);
  h->lse_part = reinterpret_cast<float*>(w); w += al(mask_bytes);
  h->gstat = reinterpret_cast<uint32_t*>(w); w += al(gstat_bytes);
  h->gsel_stat = reinterpret_cast<float*>(w);
  h->scale = static_cast<float>(1.0 / std::sqrt(static_cast<double>(head_dim)));
  if (cudaMemset(h->stat_min, 0xFF, stat_bytes) != cudaSuccess ||
      cudaMemset(h->counter, 0x00, stat_bytes) != cudaSuccess ||
      cudaMemset(h->stat_max, 0x00, stat_bytes) != cudaSuccess ||
      cudaMemset(h->status, 0, 256) != cudaSuccess || cudaDeviceSynchronize() != cudaSuccess) {
    cudaFree(h->ws);
    delete h;
    return SAGA_ERR_CUDA;
  }
  *handle = h;
  return SAGA_OK;
}

int saga_decode_set_batch(saga_handle h, int batch) {
  if (!h || batch < 1 || batch > h->max_batch) return SAGA_ERR_INVALID_ARG;
  h->batch = batch;
  return SAGA_OK;
}

int saga_decode_set_stream(saga_handle h, void* cuda_stream) {
  if (!h) return SAGA_ERR_INVALID_ARG;
  h->stream = static_cast<cudaStream_t>(cuda_stream);
  return SAGA_OK;
}

int saga_decode_attn(saga_handle h, const void* q, const void* k_cache, const void* v_cache,
                     const int32_t* seq_lens, int h_q, int h_k, int h_v, int head_dim, int N,
                     void* out) {
  if (!h) return SAGA_ERR_INVALID_ARG;
  if (int rc = check_heads(h, h_q, h_k, h_v, head_dim)) return rc;
  return decode_impl(h, q, k_cache, v_cache, seq_lens, N, out, nullptr, nullptr);
}

int saga_decode_attn_ex(saga_handle h, const void* q, const void* k_cache, const void* v_cache,
                        const int32_t* seq_lens, int h_q, int h_k, int h_v, int head_dim, int N,
                        void* out, int32_t* sel_idx, float* sel_logit) {
  if (!h) return SAGA_ERR_INVALID_ARG;
  if (int rc = check_heads(h, h_q, h_k, h_v, head_dim)) return rc;
  return decode_impl(h, q, k_cache, v_cache, seq_lens, N, out, sel_idx, sel_logit);
}

int saga_atopn_calibrate(saga_handle h, const void* q, const void* k_cache, const void* v_cache,
                         const int32_t* seq_lens, int h_q, int h_k, int h_v, int head_dim, int N,
                         void* out, int32_t* sel_idx, float* sel_logit, float* log_tau) {
  if (!h) return SAGA_ERR_INVALID_ARG;
  if (int rc = check_heads(h, h_q, h_k, h_v, head_dim)) return rc;
  if (h->dv != h->d) return SAGA_ERR_UNSUPPORTED;   // stateful Atop-N: one width
  return decode_impl(h, q, k_cache, v_cache, seq_lens, N, out, sel_idx, sel_logit, kModeCalibrate,
                     log_tau);
}

int saga_atopn_step(saga_handle h, const void* q, const void* k_cache, const void* v_cache,
                    const int32_t* seq_lens, int h_q, int h_k, int h_v, int head_dim, int N,
                    const float* log_tau, void* out, int32_t* sel_idx, float* sel_logit) {
  if (!h) return SAGA_ERR_INVALID_ARG;
  if (int rc = check_heads(h, h_q, h_k, h_v, head_dim)) return rc;
  if (h->dv != h->d) return SAGA_ERR_UNSUPPORTED;   // stateful Atop-N: one width
  return decode_impl(h, q, k_cache, v_cache, seq_lens, N, out, sel_idx, sel_logit, kModeStep,
                     const_cast<float*>(log_tau));
}

int saga_group_attn(saga_handle h, const void* q, const void* k_cache, const void* v_cache,
                    const int32_t* seq_lens, int h_q, int h_k, int h_v, int head_dim, int N,
                    void* out, int32_t* sel_idx, float* sel_stat, float* sel_logit) {
  if (!h) return SAGA_ERR_INVALID_ARG;
  if (int rc = check_heads(h, h_q, h_k, h_v, head_dim)) return rc;
  if (!q || !k_cache || !v_cache || !seq_lens || !out) return SAGA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache)) return SAGA_ERR_INVALID_ARG;
  if (N < 1 || N > h->max_N) return SAGA_ERR_INVALID_ARG;
  // value groups inside key groups, every head of a key group in one epilogue warp,
  // the weights of N x g_v in the key list's shared memory
  if (h->dv != h->d || h->h_v % h->h_k != 0 || h->npad > 32 || h->g_v > kGroupMaxGv || N > kGroupMaxN ||
      N * h->g_v > kTopnCap || !use_candidates(h, N))
    return SAGA_ERR_UNSUPPORTED;
  DeviceGuard dg(h->device);
  if (!dg.ok) return SAGA_ERR_CUDA;
  int32_t* si = sel_idx ? sel_idx : h->sel_idx;
  float* ss = sel_stat ? sel_stat : h->gsel_stat;
  float* sl = sel_logit ? sel_logit : h->sel_logit;
  int rc;
  if ((rc = launch_bounds(h, q, k_cache, seq_lens, N, true))) return rc;
  if ((rc = launch_score(h, q, k_cache, seq_lens, h->z, h->z_stride, false, true, true, true)))
    return rc;
  return launch_group(h, q, k_cache, v_cache, seq_lens, N, si, ss, sl, out);
}

int saga_decode_selftest_timeout(saga_handle h) {
  if (!h) return SAGA_ERR_INVALID_ARG;
  DeviceGuard dg(h->device);
  if (!dg.ok) return SAGA_ERR_CUDA;
  return launch(h, selftest_wait_kernel, dim3(1), dim3(32), 0, kPlain, h->status) == cudaSuccess
             ? SAGA_OK : SAGA_ERR_CUDA;
}

int saga_decode_attn_host(saga_handle h, const void* q_host, const void* k_cache,
                          const void* v_cache, const int32_t* seq_lens_host, int h_q, int h_k,
                          int h_v, int head_dim, int N, void* out_host) {
  if (!h) return SAGA_ERR_INVALID_ARG;
  if (int rc = check_heads(h, h_q, h_k, h_v, head_dim)) return rc;
  if (!q_host || !seq_lens_host || !out_host || !k_cache || !v_cache) return SAGA_ERR_INVALID_ARG;
  if (!aligned16(k_cache) || !aligned16(v_cache)) return SAGA_ERR_INVALID_ARG;
  if (N < 1 || N > h->max_N) return SAGA_ERR_INVALID_ARG;
  DeviceGuard dg(h->device);
  if (!dg.ok) return SAGA_ERR_CUDA;
  const size_t q_bytes = static_cast<size_t>(h->batch) * h->h_q * h->d * 2;
  const size_t o_bytes = static_cast<size_t>(h->batch) * h->h_q * h->dv * 2;
  if (cudaMemcpyAsync(h->q_stage, q_host, q_bytes, cudaMemcpyHostToDevice, h->stream) != cudaSuccess)
    return SAGA_ERR_CUDA;
  if (cudaMemcpyAsync(h->lens_stage, seq_lens_host, static_cast<size_t>(h->batch) * 4,
                      cudaMemcpyHostToDevice, h->stream) != cudaSuccess)
    return SAGA_ERR_CUDA;
  int rc = decode_impl(h, h->q_stage, k_cache, v_cache, h->lens_stage, N, h->out_stage,
                       nullptr, nullptr);
  if (rc) return rc;
  if (cudaMemcpyAsync(out_host, h->out_stage, o_bytes, cudaMemcpyDeviceToHost, h->stream) != cudaSuccess)
    return SAGA_ERR_CUDA;
  return SAGA_OK;
}

int saga_score(saga_handle h, const void* q, const void* k_cache, const int32_t* seq_lens,
               int h_q, int h_k, int head_dim, float* scores, int scores_stride) {
  if (!h || !q || !k_cache || !seq_lens || !scores) return SAGA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_cache)) return SAGA_ERR_INVALID_ARG;
  if (h_q != h->h_q || h_k != h->h_k || head_dim != h->d) return SAGA_ERR_INVALID_ARG;
  if (scores_stride < h->max_seq_len) return SAGA_ERR_INVALID_ARG;
  DeviceGuard dg(h->device);
  if (!dg.ok) return SAGA_ERR_CUDA;
  return launch_score(h, q, k_cache, seq_lens, scores, scores_stride, false);
}

int saga_select(saga_handle h, const float* scores, int scores_stride, const int32_t* seq_lens,
                int h_q, int N, int32_t* sel_idx, float* sel_logit) {
  if (!h || !scores || !seq_lens || !sel_idx || !sel_logit) return SAGA_ERR_INVALID_ARG;
  if (h_q != h->h_q || scores_stride < h->max_seq_len) return SAGA_ERR_INVALID_ARG;
  if (N < 1 || N > h->max_N) return SAGA_ERR_INVALID_ARG;
  DeviceGuard dg(h->device);
  if (!dg.ok) return SAGA_ERR_CUDA;
  return launch_select(h, scores, scores_stride, false, seq_lens, N, sel_idx, sel_logit);
}

int saga_combine(saga_handle h, const int32_t* sel_idx, const float* sel_logit,
                 const void* v_cache, const int32_t* seq_lens, int h_q, int h_v, int head_dim,
                 int N, void* out) {
  if (!h || !sel_idx || !sel_logit || !v_cache || !seq_lens || !out) return SAGA_ERR_INVALID_ARG;
  if (!aligned16(v_cache)) return SAGA_ERR_INVALID_ARG;
  if (h_q != h->h_q || h_v != h->h_v || head_dim != h->dv) return SAGA_ERR_INVALID_ARG;
  if (N < 1 || N > h->max_N) return SAGA_ERR_INVALID_ARG;
  DeviceGuard dg(h->device);
  if (!dg.ok) return SAGA_ERR_CUDA;
  // no select kernel ran before: clear the merge counters here
  if (cudaMemsetAsync(h->counter, 0, static_cast<size_t>(h->batch) * h->h_q * sizeof(uint32_t),
                      h->stream) != cudaSuccess)
    return SAGA_ERR_CUDA;
  return launch_gather(h, sel_idx, sel_logit, seq_lens, v_cache, N, out, false);
}

int saga_decode_status(saga_handle h, int* device_status) {
  if (!h || !device_status) return SAGA_ERR_INVALID_ARG;
  DeviceGuard dg(h->device);
  if (!dg.ok) return SAGA_ERR_CUDA;
  int v = 0;
  if (cudaStreamSynchronize(h->stream) != cudaSuccess) return SAGA_ERR_CUDA;
  if (cudaMemcpy(&v, h->status, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
    return SAGA_ERR_CUDA;
  if (cudaMemset(h->status, 0, sizeof(int)) != cudaSuccess) return SAGA_ERR_CUDA;
  if (cudaDeviceSynchronize() != cudaSuccess) return SAGA_ERR_CUDA;
  *device_status = v;
  return (v & (SAGA_STATUS_BAD_SEQ_LEN | SAGA_STATUS_TIMEOUT | SAGA_STATUS_BAD_INDEX))
             ? SAGA_ERR_DEVICE : SAGA_OK;
}

int saga_decode_launch_count(saga_handle h, long long* count) {
  if (!h || !count) return SAGA_ERR_INVALID_ARG;
  *count = h->launches;
  return SAGA_OK;
}

int saga_decode_profile(saga_handle h, int enable, int max_calls) {
  if (!h || (enable && max_calls < 1)) return SAGA_ERR_INVALID_ARG;
  DeviceGuard dg(h->device);
  if (!dg.ok) return SAGA_ERR_CUDA;
  if (!enable) {                 // stop recording; keep the events (a captured graph may use them)
    h->prof = false;
    return SAGA_OK;
  }
  if (h->ev.size() < 4 * static_cast<size_t>(max_calls)) {
    if (cudaStreamSynchronize(h->stream) != cudaSuccess) return SAGA_ERR_CUDA;
    for (cudaEvent_t e : h->ev) cudaEventDestroy(e);
    h->ev.assign(4 * static_cast<size_t>(max_calls), nullptr);
    for (auto& e : h->ev)
      if (cudaEventCreate(&e) != cudaSuccess) return SAGA_ERR_CUDA;
  }
  h->prof_max = max_calls;
  h->prof_n = 0;
  h->prof = true;
  return SAGA_OK;
}

int saga_decode_profile_read(saga_handle h, double* score_ms, double* call_ms, int* n_calls) {
  if (!h || !score_ms || !call_ms || !n_calls) return SAGA_ERR_INVALID_ARG;
  DeviceGuard dg(h->device);
  if (!dg.ok) return SAGA_ERR_CUDA;
  if (cudaStreamSynchronize(h->stream) != cudaSuccess) return SAGA_ERR_CUDA;
  double s = 0.0, c = 0.0;
  for (int i = 0; i < h->prof_n; ++i) {
    float a = 0.0f, b = 0.0f;
    if (cudaEventElapsedTime(&a, h->ev[4 * i + 1], h->ev[4 * i + 2]) != cudaSuccess) return SAGA_ERR_CUDA;
    if (cudaEventElapsedTime(&b, h->ev[4 * i], h->ev[4 * i + 3]) != cudaSuccess) return SAGA_ERR_CUDA;
    s += a;
    c += b;
  }
  *score_ms = s;
  *call_ms = c;
  *n_calls = h->prof_n;
  return SAGA_OK;
}

int saga_decode_free(saga_handle h) {
  if (!h) return SAGA_ERR_INVALID_ARG;
  int rc = SAGA_OK;
  {
    DeviceGuard dg(h->device);
    if (h->stream && cudaStreamSynchronize(h->stream) != cudaSuccess) rc = SAGA_ERR_CUDA;
    for (cudaEvent_t e : h->ev) cudaEventDestroy(e);
    if (h->ws && cudaFree(h->ws) != cudaSuccess) rc = SAGA_ERR_CUDA;
  }
  delete h;
  return rc;
}

}  // extern "C"

// ---------------------------------------------------------------------------------------------
// saga_combine_noalloc -- softmax over a selection and the gathered P.V (stages S3 + S4) for
// callers that cannot allocate device memory.
//
// Who needs it: code that must not call cudaMalloc -- for example a serving engine whose memory
// manager reserves all device memory up front and hands out only its own pool, a process sharing
// the GPU under a hard memory cap, or a caller inside CUDA-graph capture or an allocator callback
// where an allocation would fail or deadlock.  Such callers cannot create a saga_decode handle,
// because the handle allocates its workspace.  This entry point needs no handle: the only scratch
// the gather kernel uses (per-chunk softmax partials, per-row merge counters and a status word)
// lives in the fixed array below, which is part of the library image and is reserved on every GPU
// that loads the library until the process exits.
// ---------------------------------------------------------------------------------------------
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(4) << 20;   // 4 MiB per device
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kNoAllocMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_addr[kNoAllocMaxDevices] = {};

// The device address of g_noalloc_scratch on device `dev` (the current device).  Host code may
// not pass the symbol itself to a kernel: on the host it names a host-side stand-in.
int noalloc_scratch(int dev, unsigned char** out) {
  if (dev < 0 || dev >= kNoAllocMaxDevices) return SAGA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
      return SAGA_ERR_CUDA;
    g_noalloc_addr[dev] = p;
  }
  *out = static_cast<unsigned char*>(g_noalloc_addr[dev]);
  return SAGA_OK;
}

size_t al256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

}  // namespace

extern "C" {

int saga_combine_noalloc(const int32_t* sel_idx, const float* sel_logit, const void* v_cache,
                         const int32_t* seq_lens, int batch, int max_seq_len, int h_q, int h_v,
                         int head_dim, int N, void* out, void* cuda_stream) {
  if (!sel_idx || !sel_logit || !v_cache || !seq_lens || !out) return SAGA_ERR_INVALID_ARG;
  if (!aligned16(v_cache)) return SAGA_ERR_INVALID_ARG;
  if (batch < 1 || max_seq_len < 1 || h_q < 1 || h_v < 1 || N < 1) return SAGA_ERR_INVALID_ARG;
  if (h_q % h_v != 0) return SAGA_ERR_INVALID_ARG;
  if (head_dim != 64 && head_dim != 128) return SAGA_ERR_UNSUPPORTED;
  const long long rows = static_cast<long long>(batch) * h_q;
  if (rows > (1ll << 30)) return SAGA_ERR_INVALID_ARG;
  const int slots = N < max_seq_len ? N : max_seq_len;
  const int chunks = (slots + kGatherRows - 1) / kGatherRows;
  if (chunks > 65535) return SAGA_ERR_SCRATCH_TOO_SMALL;
  // scratch layout: status word | merge counters [rows] | partials [rows][chunks][head_dim + 2]
  const size_t status_bytes = 256;
  const size_t counter_bytes = al256(static_cast<size_t>(rows) * sizeof(uint32_t));
  const size_t part_bytes = al256(static_cast<size_t>(rows) * chunks * (head_dim + 2) * sizeof(float));
  if (status_bytes + counter_bytes + part_bytes > kNoAllocScratchBytes) return SAGA_ERR_SCRATCH_TOO_SMALL;

  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SAGA_ERR_CUDA;
  unsigned char* scratch = nullptr;
  if (int rc = noalloc_scratch(dev, &scratch)) return rc;
  cudaStream_t stream = static_cast<cudaStream_t>(cuda_stream);
  // the status word and the counters must start at zero; the array keeps the last call's contents
  if (cudaMemsetAsync(scratch, 0, status_bytes + counter_bytes, stream) != cudaSuccess)
    return SAGA_ERR_CUDA;

  GatherParams p;
  p.sel_idx = sel_idx;
  p.sel_logit = sel_logit;
  p.seq_lens = seq_lens;
  p.v_cache = static_cast<const __nv_bfloat16*>(v_cache);
  p.h_q = h_q;
  p.h_v = h_v;
  p.g_v = h_q / h_v;
  p.L_max = max_seq_len;
  p.N = N;
  p.status = reinterpret_cast<int*>(scratch);
  p.counter = reinterpret_cast<uint32_t*>(scratch + status_bytes);
  p.partial = reinterpret_cast<float*>(scratch + status_bytes + counter_bytes);
  p.max_chunks = chunks;
  p.out = static_cast<__nv_bfloat16*>(out);
  const dim3 grid(static_cast<unsigned>(rows), static_cast<unsigned>(chunks));
  if (head_dim == 64)
    gather_kernel<64><<<grid, kGatherThreads, 0, stream>>>(p);
  else
    gather_kernel<128><<<grid, kGatherThreads, 0, stream>>>(p);
  return cudaGetLastError() == cudaSuccess ? SAGA_OK : SAGA_ERR_CUDA;
}

}  // extern "C"
