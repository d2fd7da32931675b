/*
 * saga.h -- C ABI of the SAGA + Atop-N single-token decode-attention library.
 *
 * Source of the operation: "More Value per Key: Asymmetric Sparse Attention for
 * Faster LLM Decoding" (Elata et al.), cited as [MVK]:
 *   scores     z_i = q . k_i / sqrt(d) over all cached positions, the current
 *              token included                       [MVK] §2.1 Eq. (2), §2.2 Eq. (5)
 *   selection  the N highest-scoring positions of each query head's score row
 *              (Atop-N: compare each score against the N-th largest score; the
 *              threshold is exact and recomputed on every call)
 *                                                   [MVK] §2.5 Eq. (6), §3.1, App. C.1
 *   softmax    over the selected logits only        [MVK] §3.1 Eq. (7), App. C.1
 *   output     O = softmax(A[i]) V[i]               [MVK] §3.1 Eq. (7)
 *   heads      SAGA decouples key heads h_k from value heads h_v; query head j
 *              reads key head j / (h_q/h_k) and value head j / (h_q/h_v)
 *              (contiguous blocks)                  [MVK] §3.2, §2.3, App. B Eq. (29)
 * Ties at the N-th score go to the lowest position.  A row with L_b <= N
 * selects all L_b positions (dense softmax attention).
 *
 * Layouts (all row-major, bf16 = IEEE bfloat16, device memory unless stated):
 *   q         [B][h_q][d]            one query per head (decode, l_q = 1)
 *   k_cache   [B][h_k][L_max][d]     positions 0..L_b-1 valid; the current token's
 *   v_cache   [B][h_v][L_max][d]     key/value are already stored at L_b-1
 *   seq_lens  int32 [B]              L_b, 1 <= L_b <= L_max
 *   out       bf16 [B][h_q][d]       fp32 accumulation, one final round-to-nearest-even
 *   sel_idx   int32 [B][h_q][N]      selected positions, ascending; -1 padding when L_b < N
 *   sel_logit fp32  [B][h_q][N]      their scores z; -inf padding
 *   scores    fp32  [B][h_q][stride] z for positions < L_b (stride >= L_max)
 * B is the handle's current batch (saga_decode_set_batch; initially max_batch);
 * L_max is the handle's max_seq_len, which is also the caches' position stride.
 * q, k_cache and v_cache start on 16-byte boundaries (any cudaMalloc'd buffer
 * does); a base that does not is rejected with SAGA_ERR_INVALID_ARG.
 *
 * Ownership: every tensor argument is caller-owned; the library never frees or
 * retains it past the call.  The handle owns only its workspace (score rows,
 * selection lists, statistics, staging), allocated once by saga_decode_init and
 * released by saga_decode_free.  No call allocates memory, synchronises the
 * stream or copies to the host, except saga_decode_status and the explicit
 * host-buffer entry point saga_decode_attn_host (which copies but does not
 * synchronise).  Calls run asynchronously, in order, on the handle's stream.
 *
 * Errors: every function returns an int code (SAGA_OK = 0).  Arguments are
 * validated on the host before anything is enqueued; on error nothing runs.
 * Data errors only the device can see (a seq_len outside [1, L_max]) zero that
 * row's output, pad its selection and set a bit in the device status word,
 * read and cleared by saga_decode_status.  Kernels never trap; every internal
 * wait is bounded and reports SAGA_STATUS_TIMEOUT instead of hanging.
 * A handle must not be used from two host threads at once.
 *
 * Limits: d in {64, 128}; h_k | h_q and h_v | h_q; g = h_q/h_k <= 64;
 * 1 <= B <= max_batch <= 1024; 1 <= max_seq_len <= 2^24; 1 <= N <= max_N;
 * max_batch * h_k * max_seq_len < 2^31.  Needs a compute capability 10.0 GPU
 * (B200, sm_100a).
 */
#ifndef SAGA_H
#define SAGA_H

#include <stdint.h>

#if defined(__GNUC__)
#define SAGA_API __attribute__((visibility("default")))
#else
#define SAGA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Return codes. */
#define SAGA_OK               0
#define SAGA_ERR_INVALID_ARG  1  /* null pointer, bad size, mismatched heads, N > max_N, a q /
                                     k_cache / v_cache base not 16-byte aligned ... */
#define SAGA_ERR_UNSUPPORTED  2  /* valid but not built: d not in {64,128}, g > 64, wrong GPU */
#define SAGA_ERR_CUDA         3  /* a CUDA runtime/driver call failed */
#define SAGA_ERR_DEVICE       4  /* saga_decode_status found an error bit set */
#define SAGA_ERR_SCRATCH_TOO_SMALL 5  /* saga_combine_noalloc: sizes exceed its fixed scratch */

/* Device status bits (saga_decode_status). */
#define SAGA_STATUS_BAD_SEQ_LEN   0x1   /* some seq_lens[b] outside [1, L_max]: row zeroed */
#define SAGA_STATUS_TIMEOUT       0x2   /* an internal pipeline wait ran out: results invalid */
#define SAGA_STATUS_BAD_INDEX     0x4   /* saga_combine got an index >= L_b (that slot ignored), or
                                           a candidate position was outside [0, L_b) */
#define SAGA_STATUS_INFO_EXACT_FALLBACK 0x100  /* informational: a row needed the full radix
                                                   select (very flat score rows); not an error */
#define SAGA_STATUS_INFO_ROBUST_PATH 0x200     /* informational: a row's sampled threshold bound
                                                   missed (or the row was too long or too flat for
                                                   the candidate list) and the exact whole-row
                                                   path ran; not an error */

typedef struct saga_ctx* saga_handle;

/* Create a handle and its workspace for caches of up to max_batch rows of
 * max_seq_len positions, with h_q query, h_k key and h_v value heads of size
 * head_dim, and selections of up to max_N positions.  cuda_stream is a
 * cudaStream_t (NULL = legacy default stream).  The current CUDA device at
 * this call is the handle's device.  Workspace: about
 * 4*max_batch*h_q*(round_up(max_seq_len,32)*17/16 + 4*max_N + 1029 + head_dim +
 * ceil(min(max_N,max_seq_len)/256)*(head_dim+2)) bytes.
 * Returns SAGA_ERR_INVALID_ARG / SAGA_ERR_UNSUPPORTED / SAGA_ERR_CUDA. */
SAGA_API int saga_decode_init(saga_handle* handle, int max_batch, int max_seq_len,
                     int h_q, int h_k, int h_v, int head_dim, int max_N,
                     void* cuda_stream);

/* As saga_decode_init, with keys (and queries) of width head_dim (32, 64 or 128)
 * and values (and outputs) of width head_dim_v (64 or 128) ("More Value per Key" §5.2: keys
 * narrower than values; the scale stays 1/sqrt(head_dim)).  On such a handle the
 * head_dim argument of every call is the key width; q is [B][h_q][head_dim],
 * k_cache [B][h_k][L_max][head_dim], v_cache [B][h_v][L_max][head_dim_v], out
 * [B][h_q][head_dim_v], and saga_combine takes head_dim_v.  With head_dim_v !=
 * head_dim only the exact decode step (saga_decode_attn*, candidate and score-row
 * paths) and the stage-wise calls are supported: the stateful Atop-N calls and
 * saga_group_attn return SAGA_ERR_UNSUPPORTED.  The workspace takes
 * max(head_dim, head_dim_v) where the formula above has head_dim. */
SAGA_API int saga_decode_init_kv(saga_handle* handle, int max_batch, int max_seq_len,
                        int h_q, int h_k, int h_v, int head_dim, int head_dim_v, int max_N,
                        void* cuda_stream);

/* Set the batch B (1 <= B <= max_batch) used by later calls. */
SAGA_API int saga_decode_set_batch(saga_handle h, int batch);

/* Set the stream later calls are enqueued on (a cudaStream_t). */
SAGA_API int saga_decode_set_stream(saga_handle h, void* cuda_stream);

/* The decode step ([MVK] Eqs. (2), (5)-(7)): scores, exact top-N selection per
 * query head, softmax over the selection and the gathered P.V, for every
 * (b, j).  q, k_cache, v_cache, seq_lens, out: device pointers (layouts above).
 * h_q, h_k, h_v, head_dim must equal the handle's; 1 <= N <= max_N. */
SAGA_API int saga_decode_attn(saga_handle h, const void* q, const void* k_cache,
                     const void* v_cache, const int32_t* seq_lens,
                     int h_q, int h_k, int h_v, int head_dim, int N, void* out);

/* As saga_decode_attn, and also writes the selection: sel_idx / sel_logit are
 * device arrays [B][h_q][N] (either may be NULL). */
SAGA_API int saga_decode_attn_ex(saga_handle h, const void* q, const void* k_cache,
                        const void* v_cache, const int32_t* seq_lens,
                        int h_q, int h_k, int h_v, int head_dim, int N, void* out,
                        int32_t* sel_idx, float* sel_logit);

/* Stateful Atop-N ([MVK] §3.1, App. C.1): a per-row probability threshold tau,
 * calibrated on one decode step and reused by the following ones (the paper
 * recalibrates every n = 32 steps; when is the caller's choice).  The state is
 * the caller's device array log_tau, fp32 [B][h_q], natural log of tau.
 *
 * saga_atopn_calibrate: the decode step of saga_decode_attn_ex (exact top-N,
 * out, optional sel_idx / sel_logit [B][h_q][N]), and for every row
 * log_tau[b][j] = z_(N_b) - log(sum_i exp(z_i)): the log of the softmax
 * probability of the N_b-th largest score (N_b = min(N, L_b)).  A row with an
 * invalid seq_len gets log_tau = -inf.
 *
 * saga_atopn_step: with t = log_tau[b][j] + log(sum_i exp(z_i)) (the paper's
 * m_hat + log(tau * s_hat), in which the reference m_hat cancels), selects every
 * position with z_i >= t in ascending position order, keeps the first 2N (the
 * paper drops the excess in arbitrary order; the lowest positions are kept
 * here, so results are reproducible), and computes the softmax over the kept
 * logits and the gathered P.V into out.  sel_idx / sel_logit, if given, are
 * [B][h_q][2N], padded with -1 / -inf.  A row where nothing reaches t gets a
 * zero output; a NaN log_tau counts as -inf (every position passes).
 *
 * Both: same layouts, ownership and errors as saga_decode_attn_ex; log_tau
 * non-NULL device pointer; 1 <= N <= min(max_N, 2048), else
 * SAGA_ERR_INVALID_ARG / SAGA_ERR_UNSUPPORTED.  The log-sum-exp runs over all
 * L_b scores in fp32; a row whose scores leave the fp32 range of its sums, or
 * whose sampled candidate bound lies above t, is scored again on CUDA cores
 * (SAGA_STATUS_INFO_ROBUST_PATH). */
SAGA_API int saga_atopn_calibrate(saga_handle h, const void* q, const void* k_cache,
                                  const void* v_cache, const int32_t* seq_lens, int h_q, int h_k,
                                  int h_v, int head_dim, int N, void* out, int32_t* sel_idx,
                                  float* sel_logit, float* log_tau);
SAGA_API int saga_atopn_step(saga_handle h, const void* q, const void* k_cache,
                             const void* v_cache, const int32_t* seq_lens, int h_q, int h_k,
                             int h_v, int head_dim, int N, const float* log_tau, void* out,
                             int32_t* sel_idx, float* sel_logit);

/* The decode step with the per-step inputs and result in HOST memory:
 * q_host (bf16 [B][h_q][d]) and seq_lens_host (int32 [B]) are copied to the
 * handle's device staging, the step runs, and the result is copied back to
 * out_host (bf16 [B][h_q][d]).  The caches stay in device memory (they are the
 * resident KV cache).  All three copies are enqueued asynchronously on the
 * handle's stream: host buffers should be pinned, and out_host is valid only
 * after the stream is synchronised (e.g. by saga_decode_status). */
SAGA_API int saga_decode_attn_host(saga_handle h, const void* q_host, const void* k_cache,
                          const void* v_cache, const int32_t* seq_lens_host,
                          int h_q, int h_k, int h_v, int head_dim, int N,
                          void* out_host);

/* Stage S1 alone ([MVK] Eq. (2), (5)): scores[b][j][i] = q[b][j] . k[b][j/g][i]
 * / sqrt(d) for i < L_b, fp32, into the caller's array with row stride
 * scores_stride >= L_max (entries i >= L_b are not written). */
SAGA_API int saga_score(saga_handle h, const void* q, const void* k_cache,
               const int32_t* seq_lens, int h_q, int h_k, int head_dim,
               float* scores, int scores_stride);

/* Stage S2 alone ([MVK] Eq. (6), App. C.1): exact top-N selection of each
 * caller-given fp32 score row (layout of saga_score), ties to the lowest
 * position; writes sel_idx and sel_logit ([B][h_q][N], non-NULL). */
SAGA_API int saga_select(saga_handle h, const float* scores, int scores_stride,
                const int32_t* seq_lens, int h_q, int N,
                int32_t* sel_idx, float* sel_logit);

/* Stages S3+S4 alone ([MVK] Eq. (7)): softmax over the valid entries among
 * the first min(N, L_b) slots of each selection row ([B][h_q][N]; entries
 * with sel_idx < 0 are padding, entries >= L_b are ignored and flagged
 * SAGA_STATUS_BAD_INDEX) and the gathered P.V over v_cache, bf16 out.  A row
 * with no valid entry gets zeros.  1 <= N <= max_N. */
SAGA_API int saga_combine(saga_handle h, const int32_t* sel_idx, const float* sel_logit,
                 const void* v_cache, const int32_t* seq_lens, int h_q, int h_v,
                 int head_dim, int N, void* out);

/* saga_combine_noalloc -- stages S3+S4 (as saga_combine) without a handle and without
 * allocating anything.  The paper has no counterpart: it exists for callers that cannot
 * allocate device memory (a serving engine whose memory manager owns the whole device, a
 * process under a hard memory cap, code running inside graph capture or an allocator
 * callback), which therefore cannot create a handle.  Inputs and outputs are the caller's
 * device arrays, with the layouts above: sel_idx / sel_logit [batch][h_q][N], v_cache
 * [batch][h_v][max_seq_len][head_dim], seq_lens [batch], out bf16 [batch][h_q][head_dim];
 * cuda_stream is a cudaStream_t (NULL = legacy default stream).  The kernel's scratch (a
 * status word, per-row merge counters and per-chunk softmax partials) is a fixed 4 MiB array
 * inside the library, reserved on every GPU that loads the library until the process exits.
 * Limit: 256 + round_up(4*batch*h_q, 256) + round_up(4*batch*h_q*ceil(min(N,max_seq_len)/256)
 * *(head_dim+2), 256) <= 4 MiB (e.g. batch*h_q = 192 rows with N = 1024 and head_dim = 128
 * uses 0.4 MiB), else SAGA_ERR_SCRATCH_TOO_SMALL and nothing runs.  The first call on each
 * device looks up the array's device address; make that first call before any stream
 * capture.  Every call clears the part of the array that must start at zero and reuses the
 * rest, so calls that can overlap on the GPU (different streams) race and must not be issued
 * concurrently.  Device-side data errors are handled as in saga_combine but not reported:
 * with no handle there is no status word to read, so a row with seq_lens[b] outside
 * [1, max_seq_len] gets zeros and an entry with an index >= seq_lens[b] is skipped, silently
 * (a caller that needs the report uses saga_combine).  Asynchronous. */
SAGA_API int saga_combine_noalloc(const int32_t* sel_idx, const float* sel_logit,
                                  const void* v_cache, const int32_t* seq_lens, int batch,
                                  int max_seq_len, int h_q, int h_v, int head_dim, int N,
                                  void* out, void* cuda_stream);

/* Synchronise the handle's stream, then return (in *device_status) and clear
 * the device status word.  Returns SAGA_ERR_DEVICE if an error bit
 * (SAGA_STATUS_BAD_SEQ_LEN, SAGA_STATUS_TIMEOUT or SAGA_STATUS_BAD_INDEX) was
 * set, else SAGA_OK. */
SAGA_API int saga_decode_status(saga_handle h, int* device_status);

/* Group-shared selection (a different method from the decode step: results
 * differ): the g_v = h_q/h_v query heads that read one value head share one set
 * of N positions -- the N_b largest s_i = sum over the group's heads j of
 * softmax(z_j)_i (the GQA form of SparQ's position step as the pages describe
 * it, applied to [MVK] §3.1 Eq. (7), §3.2), ties to the lowest position -- and
 * each head takes the softmax of its own logits over the set and the gathered
 * P.V, so the value gather reads N rows per value head.
 *   sel_idx   int32 [B][h_v][N]   the shared positions, ascending, -1 padding
 *   sel_stat  fp32  [B][h_v][N]   s at them, -inf padding
 *   sel_logit fp32  [B][h_q][N]   each head's logits at them, -inf padding
 * (each may be NULL).  Needs h_k | h_v, g = h_q/h_k <= 32, g_v <= 8,
 * N <= min(max_N, 1024) and N * g_v <= 8192, else SAGA_ERR_UNSUPPORTED.  Rows
 * whose kept positions cannot be shown to contain the top N of s are scored
 * again on CUDA cores (SAGA_STATUS_INFO_ROBUST_PATH).  Layouts, ownership and
 * errors as saga_decode_attn_ex. */
SAGA_API int saga_group_attn(saga_handle h, const void* q, const void* k_cache,
                             const void* v_cache, const int32_t* seq_lens, int h_q, int h_k,
                             int h_v, int head_dim, int N, void* out, int32_t* sel_idx,
                             float* sel_stat, float* sel_logit);

/* Failure-detection self-test: enqueues one kernel whose bounded pipeline wait
 * has nothing to wait for.  After the wait's limit (2 s) the kernel sets
 * SAGA_STATUS_TIMEOUT in the device status word and exits, as a stalled
 * pipeline stage would; saga_decode_status then returns SAGA_ERR_DEVICE with
 * that bit, and the handle and the CUDA context stay usable.  Asynchronous. */
SAGA_API int saga_decode_selftest_timeout(saga_handle h);

/* Total number of kernels this handle has launched. */
SAGA_API int saga_decode_launch_count(saga_handle h, long long* count);

/* Profiling: when enabled, each decode call records CUDA events around its
 * score kernel and around the whole call on the handle's stream (the record
 * before the score kernel keeps it from starting early under programmatic
 * dependent launch, so the interval is the kernel's own duration; up to
 * max_calls calls; inside CUDA-graph capture the
 * records become graph nodes, so every replay re-records them; the events
 * live until the handle is freed).  Disabling stops recording and keeps the
 * events.  saga_decode_profile_read synchronises and returns the summed
 * milliseconds of the calls recorded since profiling was last enabled, and
 * their number; it may be called after every replay of a graph that holds the
 * records (each read gives that replay's times).  Enabling again starts
 * counting calls from zero. */
SAGA_API int saga_decode_profile(saga_handle h, int enable, int max_calls);
SAGA_API int saga_decode_profile_read(saga_handle h, double* score_ms, double* call_ms,
                             int* n_calls);

/* A static description of a return code. */
SAGA_API const char* saga_decode_error_string(int code);

/* Release the handle and its workspace (synchronises its stream first). */
SAGA_API int saga_decode_free(saga_handle h);

#ifdef __cplusplus
}
#endif

#endif /* SAGA_H */
