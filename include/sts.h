/*
 * sts.h -- C ABI of the B200 (sm_100a) sampling-transform scoring core.
 *
 * The operation (defined in "Consolidate sampling-transform scoring on one
 * shared chunked core; implement top-k/top-p/min-p replay for generic
 * ce_modes", xorl pull request 74, section "What this PR does", items 1, 2
 * and 4):
 *
 *   for every row t (a scored token) with hidden state H[t,:]:
 *     z_i   = sum_j H[t,j] * W[i,j]            bf16 operands, fp32 accumulate
 *     s_i   = z_i / tau_t                      per-row temperature, applied
 *                                              after the projection, IEEE fp32
 *                                              division
 *     S_t   = top-k  (k_t)  then top-p (p_t, measured on the top-k-renormalised
 *             mass, inclusive crossing)  then min-p (mu_t, against the
 *             unfiltered row max); ties ordered by token id
 *     logprob_t = min(s_y - log sum_{i in S_t} exp(s_i), 0)   if y_t in S_t
 *               = -inf                                         otherwise
 *
 *   and the closed-form backward (recompute, only per-row scalars kept):
 *     dz_i = g_t * (1[i == y_t] - exp(s_i - LSE_S) * 1[i in S_t]) / tau_t
 *            (a zero row when y_t is outside S_t)
 *     dH = dZ . W,   dW = dZ^T . H
 *
 * Conventions shared by every entry point
 *   - All tensor pointers are DEVICE pointers on the current CUDA device,
 *     owned by the caller. The library allocates no device memory: scratch
 *     comes from the caller's workspace (size from sts_workspace_bytes).
 *   - Calls are asynchronous on the given stream. Errors a host can see
 *     (NULL pointers, bad shapes, small workspace, wrong device) return
 *     immediately and launch nothing. Errors that depend on row values
 *     (temperature, top_p, min_p, target) are written to a status word in
 *     the workspace; sts_get_status() reads it.
 *   - Rows whose values are invalid produce logprob = NaN and a zero
 *     gradient; other rows are unaffected.
 *   - A target outside its row's support is not an error: logprob = -inf
 *     and the row's gradient is zero (item 4 of the page).
 *   - Only bf16 H and W are accepted (an fp8 head is rejected one level up,
 *     in the Python binding, with STS_ERR_DTYPE).
 *   - Layouts: H [T, d] and W [V, d] row-major bf16 (nn.Linear weight
 *     layout); dH [T, d] and dW [V, d] row-major fp32; per-row arrays [T].
 *   - Alignment: d must be a multiple of 8 (16-byte TMA strides); H, W, dH,
 *     dW and the scaled-logits buffer must be 16-byte aligned; the workspace
 *     must be 256-byte aligned (STS_ERR_WORKSPACE otherwise).
 *   - Device: compute capability 10.0 (B200, sm_100a) only.
 */
#ifndef STS_H_
#define STS_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define STS_ABI_VERSION 3

/* cudaStream_t without pulling in the CUDA headers (same opaque type). */
typedef struct CUstream_st* sts_stream_t;

typedef enum {
  STS_OK = 0,
  STS_ERR_NULL = 1,             /* a required pointer is NULL */
  STS_ERR_SHAPE = 2,            /* T, d, V, chunk sizes, alignment, or a
                                   metadata length != T (validated, never
                                   truncated: "Self-review pass") */
  STS_ERR_DTYPE = 3,            /* operand dtype other than bf16 (binding) */
  STS_ERR_TEMPERATURE = 4,      /* some row has tau not finite or <= 0 */
  STS_ERR_TOP_K = 5,            /* reserved: every int32 top_k is valid */
  STS_ERR_TOP_P = 6,            /* some row has top_p not in (0, 1] */
  STS_ERR_MIN_P = 7,            /* some row has min_p not in [0, 1] */
  STS_ERR_TARGET = 8,           /* some row has target not in [0, V) */
  STS_ERR_WORKSPACE = 9,        /* workspace NULL, too small or misaligned */
  STS_ERR_OVERFLOW = 10,        /* an internal bound was exceeded */
  STS_ERR_TIMEOUT = 11,         /* a bounded device wait gave up */
  STS_ERR_CUDA = 12,            /* a CUDA runtime/driver call failed */
  STS_ERR_UNSUPPORTED_ARCH = 13 /* current device is not sm_100 */
} sts_status;

/* Problem shape. */
typedef struct {
  int64_t T;           /* rows (scored tokens), >= 1 */
  int64_t d;           /* hidden size, >= 8, multiple of 8 */
  int64_t V;           /* vocabulary size, >= 1, < 2^31 */
  int64_t vocab_chunk; /* backward vocab chunk (multiple of 256); 0: 28416 */
  int64_t row_chunk;   /* forward row chunk (multiple of 128); 0: default */
} sts_shape;

/* Per-row transform metadata ("What this PR does", items 1-3). */
typedef struct {
  int64_t len;              /* must equal T */
  const int64_t* target;    /* [T] replayed token y, 0 <= y < V */
  const float* temperature; /* [T] finite, > 0 */
  const int32_t* top_k;     /* [T] <= 0 or >= V: off */
  const float* top_p;       /* [T] in (0, 1]; 1.0: exact identity */
  const float* min_p;       /* [T] in [0, 1]; 0: off */
} sts_rows;

/* Per-row scalars written by the forward and read by the backward (the only
 * state kept between them: item 2, "saving only per-row scalars"). */
typedef struct {
  float* row_max;        /* [T] max_i s_i over the unfiltered row */
  float* lse_support;    /* [T] log sum_{i in S} exp(s_i) */
  float* cut_logit;      /* [T] s of the last kept token in (s desc, id asc) */
  int32_t* cut_id;       /* [T] id  of the last kept token */
  int32_t* support_size; /* [T] |S| */
  int32_t* flags;        /* [T] STS_ROW_* bits */
} sts_saved;

#define STS_ROW_TARGET_IN_SUPPORT 1 /* y in S */
#define STS_ROW_INVALID 2           /* row failed validation */
#define STS_ROW_IDENTITY 4          /* no active filter */

/* Bytes of workspace needed. pass: 0 forward (also sts_sample), 1 backward,
 * 2 sts_filter_logits. Returns 0 for an invalid shape. */
size_t sts_workspace_bytes(const sts_shape* shape, int pass);

/* The vocabulary chunk the backward uses for this shape: shape->vocab_chunk,
 * or 28416 when it is 0, clamped to V rounded up to 256. A pure function of
 * the shape (workspace sizes do not depend on the device). Returns -1 for an
 * invalid shape. Not from the pages: they chunk the vocabulary but fix no
 * chunk size. */
int64_t sts_vocab_chunk(const sts_shape* shape);

/* Forward: logprob[T] (fp32) and the saved per-row scalars; optionally the
 * entropy of each row's filtered distribution, entropy[T] (fp32, nats:
 * H_t = -sum_{i in S_t} p_i ln p_i, p_i = exp(s_i - LSE_S); "align
 * architecture v2: proposal", section 5.4 A, entropy from the same sweep),
 * formed from the same per-logit float64 masses as LSE_S (one more float64
 * sum per logit); entropy may be NULL (then nothing extra is computed).
 * Invalid rows get NaN. ws must hold sts_workspace_bytes(shape, 0) bytes. */
sts_status sts_forward(const sts_shape* shape, const void* H_bf16, const void* W_bf16,
                       const sts_rows* rows, float* logprob, float* entropy,
                       const sts_saved* saved, void* ws, size_t ws_bytes, sts_stream_t stream);

/* Backward: dH[T,d] and dW[V,d] (fp32) from grad_logprob[T] and the scalars
 * saved by sts_forward on the same H, W and rows. dH is overwritten; dW is
 * overwritten unless accumulate_dW is non-zero (then dW += result).
 * ws must hold sts_workspace_bytes(shape, 1) bytes. */
sts_status sts_backward(const sts_shape* shape, const void* H_bf16, const void* W_bf16,
                        const sts_rows* rows, const sts_saved* saved,
                        const float* grad_logprob, float* dH, float* dW, int accumulate_dW,
                        void* ws, size_t ws_bytes, sts_stream_t stream);

/* Receives one finished slice of the weight gradient: rows [v0, v0 + rows) of
 * dW, which start at dW_slice (device memory, row-major [rows, d] fp32). */
typedef void (*sts_slice_fn)(void* user, int64_t v0, int64_t rows, float* dW_slice,
                             sts_stream_t stream);

/* sts_backward for data-parallel training: the weight gradient is written once
 * per vocabulary slice ("Self-review pass" of the xorl PR) and its partial sums
 * must be added across the ranks that scored other rows ("What this PR does",
 * item 2). Right after the GEMM that writes slice [v0, v0 + rows) has been
 * enqueued on `stream`, and before anything else is enqueued, on_dw_slice is
 * called on the calling host thread, once per slice in increasing v0. The
 * callee typically records an event on `stream`, makes a communication stream
 * wait for it and enqueues the slice's all-reduce (or reduce-scatter) there,
 * so that the exchange of slice i overlaps the dH GEMM of slice i and the
 * GEMMs of slice i + 1; it must make `stream` wait for its exchanges before
 * dW is read. The library writes no element of a slice after handing it out.
 * The GEMMs are persistent (one CTA per SM) and would hold every SM for
 * their whole run, so comm_sms SMs (0 <= comm_sms < SM count, else
 * STS_ERR_SHAPE) are left free for the exchange kernels. on_dw_slice == NULL
 * with comm_sms == 0 is sts_backward. The callback must not call back into
 * the library on the same workspace. */
sts_status sts_backward_sliced(const sts_shape* shape, const void* H_bf16, const void* W_bf16,
                               const sts_rows* rows, const sts_saved* saved,
                               const float* grad_logprob, float* dH, float* dW, int accumulate_dW,
                               void* ws, size_t ws_bytes, sts_stream_t stream,
                               sts_slice_fn on_dw_slice, void* user, int comm_sms);

/* Vocabulary-parallel tensor parallelism ("What this PR does", item 2 of the
 * xorl PR: chunk-local logits gathered in rank order, hidden gradients summed
 * across vocabulary ranks, weight-shard gradients kept local). Rank k holds
 * the vocabulary rows [k Vl, (k + 1) Vl) of W. Each rank forms its shard's
 * scaled logits (sts_scaled_logits), the ranks all-gather them, and
 * sts_gather_vocab_shards interleaves the gathered blocks into full rows;
 * every rank then runs the support program on the full rows
 * (sts_resolve_logits) and the backward on its own shard
 * (sts_backward_shard), whose partial dH the ranks sum. */

/* dst[r * ld + k * vocab_per_rank + j] = src[(k * T + r) * vocab_per_rank + j]
 * for k < world, r < T, j < vocab_per_rank: the world blocks [T, vocab_per_rank]
 * of an all-gather, in rank order, into rows of stride ld >= world *
 * vocab_per_rank. Device pointers (dst holds T * ld floats); asynchronous;
 * allocates nothing. STS_ERR_SHAPE for non-positive sizes or a short ld. */
sts_status sts_gather_vocab_shards(const float* src, int64_t world, int64_t T,
                                   int64_t vocab_per_rank, float* dst, int64_t ld,
                                   sts_stream_t stream);

/* The forward's support program, logprob and saved scalars (and optionally
 * the entropy) on caller-given fp32 scaled logits S [T, ld] (row stride ld >=
 * shape->V; the first V columns of each row are the row), for example full
 * rows gathered from vocabulary shards. The row max is taken from S. Rows are
 * validated as in sts_forward (temperature included: the backward divides by
 * it). ws: sts_workspace_bytes(shape, 2). saved->flags doubles as the row
 * flags. */
sts_status sts_resolve_logits(const sts_shape* shape, const float* S, int64_t ld,
                              const sts_rows* rows, float* logprob, float* entropy,
                              const sts_saved* saved, void* ws, size_t ws_bytes,
                              sts_stream_t stream);

/* The backward of one rank's vocabulary shard: W_shard holds the vocabulary
 * rows [vocab_offset, vocab_offset + shape->V) of the full W, rows->target and
 * the saved scalars (cut ids) use full-vocabulary ids. Writes dW_shard
 * [shape->V, d] (overwritten unless accumulate_dW) and dH_partial [T, d] =
 * this shard's part of dH, which the ranks sum. ws: sts_workspace_bytes(shape,
 * 1). STS_ERR_SHAPE for a negative offset. */
sts_status sts_backward_shard(const sts_shape* shape, const void* H_bf16, const void* W_shard_bf16,
                              const sts_rows* rows, const sts_saved* saved,
                              const float* grad_logprob, float* dH_partial, float* dW_shard,
                              int accumulate_dW, int64_t vocab_offset, void* ws, size_t ws_bytes,
                              sts_stream_t stream);

/* The statistics merge: the same support program with per-row statistics
 * crossing the ranks instead of logits. Every rank runs the four stages on
 * its own shard S [T, ld] (fp32 scaled logits of vocabulary rows
 * [vocab_offset, vocab_offset + Vl) of V), and the caller combines each
 * stage's outputs over the ranks before the next stage:
 *   1. sts_tp_row_max -> row_max [T]; combine by max: m.
 *   2. sts_tp_count(m) -> counts [T][buckets] int32 of floor((m - s) 128)
 *      clamped to buckets - 1; combine by sum.
 *   3. sts_tp_exact(m, merged counts) -> plan [T][plan_fields] (identical on
 *      every rank), sums [T][sum_fields] float64 (combine by sum), keys
 *      [T][key_fields] int64 (combine by min), ylogit [T][2] (combine by sum),
 *      cand [T][cap] uint64 composite keys and ncand [T] (all-gather both, in
 *      rank order: [world][T][cap] and [world][T]).
 *   4. sts_tp_finish -> logprob and the saved scalars of sts_forward, for
 *      every row where need_gather[r] == 0; need_gather[r] == 1 (the same on
 *      every rank) marks a row whose gathered buckets did not hold its top-p
 *      crossing, or held more keys than one sort (sort_cap) or than a rank's
 *      cap: resolve it from gathered full rows instead
 *      (sts_gather_vocab_shards + sts_resolve_logits). Rows are
 *      validated here (invalid rows: NaN, flag STS_ROW_INVALID, status in
 *      ws, which holds at least the 256-byte status header).
 * Masses are float64 (no fp32-mass shortcut); entropy is not formed.
 * sts_tp_constants reports buckets, plan_fields, sum_fields, key_fields and
 * sort_cap. All pointers are device memory except the constants' outputs;
 * calls are asynchronous on `stream` and allocate nothing. STS_ERR_SHAPE for
 * inconsistent sizes (ld < Vl, vocab_offset + Vl > V, cap < 1). */
sts_status sts_tp_constants(int64_t* buckets, int64_t* plan_fields, int64_t* sum_fields,
                            int64_t* key_fields, int64_t* sort_cap);
sts_status sts_tp_row_max(const float* S, int64_t T, int64_t Vl, int64_t ld, float* row_max,
                          sts_stream_t stream);
sts_status sts_tp_count(const float* S, int64_t T, int64_t Vl, int64_t ld, const float* m,
                        int32_t* counts, sts_stream_t stream);
sts_status sts_tp_exact(const float* S, int64_t T, int64_t Vl, int64_t ld, int64_t vocab_offset,
                        int64_t V, const sts_rows* rows, const float* m, const int32_t* counts,
                        int32_t* plan, double* sums, int64_t* keys, float* ylogit, uint64_t* cand,
                        int32_t* ncand, int64_t cap, sts_stream_t stream);
sts_status sts_tp_finish(int64_t T, int64_t V, int64_t world, const sts_rows* rows, const float* m,
                         const int32_t* plan, const double* sums, const int64_t* keys,
                         const float* ylogit, const uint64_t* cand, const int32_t* ncand,
                         int64_t cap, float* logprob, const sts_saved* saved,
                         int32_t* need_gather, void* ws, size_t ws_bytes, sts_stream_t stream);

/* Draw one token per row from the filtered distribution: the inverse CDF of
 * the support walked in (s desc, id asc) order, taking the first kept token
 * whose inclusive running mass exceeds u[t] * sum_{i in S} exp(s_i - m).
 * rows->target is ignored (may be NULL). u: [T] doubles in [0, 1).
 * ws: sts_workspace_bytes(shape, 0). Used to replay rollouts for tests and
 * benchmarks; the pages fix no sampler, only the support it draws from. */
sts_status sts_sample(const sts_shape* shape, const void* H_bf16, const void* W_bf16,
                      const sts_rows* rows, const double* u, int64_t* sampled,
                      void* ws, size_t ws_bytes, sts_stream_t stream);

/* Test hook: run only the support program on caller-given fp32 scaled logits
 * [T, V] (row stride V). Writes support_size, cut_logit, cut_id per row and,
 * when mask is not NULL, mask[T, V] (1 = kept); when entropy is not NULL, the
 * entropy of each row's filtered distribution as sts_forward forms it.
 * rows->target is ignored. ws: sts_workspace_bytes(shape, 2). */
sts_status sts_filter_logits(const sts_shape* shape, const float* scaled_logits,
                             const sts_rows* rows, int32_t* support_size, float* cut_logit,
                             int32_t* cut_id, uint8_t* mask, float* entropy, void* ws,
                             size_t ws_bytes, sts_stream_t stream);

/* sts_filter_logits for callers that cannot allocate device memory: code
 * running under a fixed device-memory reservation (where cudaMalloc may fail,
 * or implicitly synchronise the device in the middle of a step), or code
 * called from inside an allocator or framework callback that must not
 * re-enter the allocator. The pages have no counterpart: this entry point
 * exists for such callers, not for the method.
 * Same inputs, outputs and results as sts_filter_logits, minus the workspace:
 * the scratch (a 256-byte status header plus one int32 per row) is a
 * file-scope device array of 262,400 bytes that every GPU loading the library
 * holds until process exit. T must be <= 65,536 (else STS_ERR_SHAPE).
 * The first call on each device looks up the array's device address
 * (cudaGetSymbolAddress); make that first call before any stream capture.
 * All calls share the array, which keeps the last call's contents (the header
 * is cleared at the start of each call): calls that overlap on the GPU -- on
 * different streams, or from different host threads -- race. Row-value
 * errors, and a row whose exact search exceeds an internal bound, show per
 * row (support_size 0, cut_id -1, cut_logit NaN, mask row all 0); there is
 * no status word to read back. Allocates nothing. */
sts_status sts_filter_logits_noalloc(const sts_shape* shape, const float* scaled_logits,
                                     const sts_rows* rows, int32_t* support_size,
                                     float* cut_logit, int32_t* cut_id, uint8_t* mask,
                                     sts_stream_t stream);

/* Test hook: the forward's first pass alone, S[t, v] = (H . W^T)[t, v] /
 * temperature[t] for t in [t0, t0 + rows), v in [v0, v0 + cols), written to
 * S_out[(t - t0) * ld + (v - v0)] (fp32). t0 must be a multiple of 128 and v0
 * of 256 (the tile grid of the forward); ld a multiple of 4, >= cols.
 * Allocates nothing; a device-side wait timeout in this hook is not reported. */
sts_status sts_scaled_logits(const sts_shape* shape, const void* H_bf16, const void* W_bf16,
                             const float* temperature, int64_t t0, int64_t rows, int64_t v0,
                             int64_t cols, float* S_out, int64_t ld, sts_stream_t stream);

/* Test hook: the resolver's token-mass function exp(s[i] - m) (float64,
 * table-driven) and the CUDA library exp(s[i] - m) on the same inputs, for
 * i < n. s is a device array of fp32 logits <= m; mass and lib_exp are device
 * arrays of n doubles. Allocates nothing. */
sts_status sts_probe_mass_exp(const float* s, float m, double* mass, double* lib_exp, int64_t n,
                              sts_stream_t stream);

/* Synchronise the stream and read the status word a previous call left in
 * ws. first_bad_row (may be NULL) receives the lowest failing row or -1. */
sts_status sts_get_status(const void* ws, sts_stream_t stream, int64_t* first_bad_row);

/* Diagnostic: how many rows the support resolver decided by each of its
 * paths since the workspace's last reset (every sts_forward, sts_sample and
 * sts_filter_logits call resets it): counts[0] the planned pass (a sampled
 * plan confirmed by one exact pass), counts[1] the fast path (full count
 * histogram, then an exact pass), counts[2] the exact search, counts[3]
 * identity rows (one pass). Synchronises the stream. counts: 4 int64 on the
 * host. Not from the pages: a measure of where the resolver's time goes. */
sts_status sts_path_counts(const void* ws, sts_stream_t stream, int64_t* counts);

/* Policy-gradient objectives for sts_policy_grad. */
typedef enum { STS_PG_CISPO = 0, STS_PG_CLIPPED = 1 } sts_pg_objective;

/* The upstream gradient grad_logprob[t] = dL/dlogprob_t of a policy-gradient
 * token loss L = -J, formed from the forward's fresh logprobs and passed to
 * sts_backward ("align architecture v2: proposal", section 5.4 A, "Why the
 * in-chunk form works for this loss": the logit gradient is a per-token
 * coefficient times (softmax - onehot)). With r_t = exp(logprob_t -
 * old_logprob_t), in float64:
 *   STS_PG_CISPO    -scale * A_t * min(r_t, 1 + eps_high)   (weight held constant)
 *   STS_PG_CLIPPED  -scale * A_t * r_t, 0 where the clip binds: r_t > 1 + eps_high
 *                   with A_t >= 0, r_t < 1 - eps_low with A_t < 0
 * Rows whose logprob is not finite (-inf out of support, NaN invalid) get 0.
 * All arrays [T] fp32 on the device; scale carries the loss normalisation.
 * Returns STS_ERR_SHAPE for T < 0, an unknown objective, negative or
 * non-finite eps or a non-finite scale; STS_ERR_NULL for a NULL array (T > 0).
 * Asynchronous on stream; allocates nothing. */
sts_status sts_policy_grad(int64_t T, const float* logprob, const float* old_logprob,
                           const float* advantage, int objective, float eps_low, float eps_high,
                           float scale, float* grad_logprob, sts_stream_t stream);

const char* sts_status_string(sts_status status);

/* Kernel kinds for the launch counters and the timing facility below. */
typedef enum {
  STS_KERNEL_VALIDATE = 0,    /* per-row metadata validation */
  STS_KERNEL_LOGITS_GEMM = 1, /* forward projection, s = z / tau epilogue */
  STS_KERNEL_RESOLVE = 2,     /* per-row support resolver */
  STS_KERNEL_DZ_GEMM = 3,     /* backward recompute, dz epilogue */
  STS_KERNEL_DW_GEMM = 4,     /* dW slice = dZ^T . H */
  STS_KERNEL_DH_GEMM = 5,     /* dH (+)= dZ . W slice */
  STS_KERNEL_KINDS = 6
} sts_kernel_kind;

/* Number of kernels of a kind this process has launched through the library
 * (always counted; -1 for an unknown kind). */
int64_t sts_launch_count(int kind);

/* Host-side timing of every kernel launch (off by default, process-wide).
 * While on, each launch is bracketed by two CUDA events recorded on the
 * launch stream; turning it on discards earlier records. Events are host
 * objects: no device memory is allocated. */
sts_status sts_timing_enable(int on);

/* Total device time (ms) and launch count of one kind over the records taken
 * since timing was last turned on. Waits for the recorded events. */
sts_status sts_timing_read(int kind, double* total_ms, int64_t* launches);

int sts_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* STS_H_ */
