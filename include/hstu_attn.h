/*
 * hstu_attn.h -- C ABI of the jagged HSTU attention library for NVIDIA B200 (sm_100a).
 *
 * The operation.  For every jagged sequence b (rows seq_offsets[b] .. seq_offsets[b+1]-1
 * of the packed tensors, local positions 0..L-1), every head h and query row i:
 *
 *   s_ij = alpha * <q_i, k_j> + rel_bias[clamp(p(i) - p(j), 0, R-1)]
 *                             + time_bias[min(floor(log(|ts[p(i)] - ts[p(j)]| + 1) / div), NB-1)]
 *   A_ij = valid(i,j) ? SiLU(s_ij) / N : 0,            SiLU(x) = x * sigmoid(x)
 *   Y_i  = sum_j A_ij V_j            (per head; heads concatenated into D = H * d_v features)
 *   O_i  = U_i (.) LayerNorm(Y_i)    (over the D features, biased variance, eps, no affine)
 *
 * Sources (page title, section):
 *  - "HSTU tensor by tensor: SiLU aggregation, temporal bias and gating", "Similar shape,
 *    different aggregation": the pointwise SiLU aggregation A_ij = 1[j<=i] SiLU(q.k+b)/N
 *    followed by U (.) Norm(sum_j A_ij V_j) (the W_o projection and residual that follow on
 *    that page are not part of this library);
 *  - same page, "SiLU aggregation coefficients are not probabilities" (SiLU = x*sigmoid(x)),
 *    "Do not copy softmax masking mechanically" (illegal coefficients are zeroed after the
 *    SiLU, never -inf before it), "Relative time adds information content similarity lacks"
 *    and "Temporal bias is not simply fixed forgetting" (relative position and bucketed
 *    elapsed-time bias), "Trace four projections" (d_qk may differ from d_v);
 *  - "HSTU-MUSA: HSTU for Moore Threads (MUSA)", "Mathematical Equivalence": the mask family
 *    (contextual bidirectional attention, candidate position clamping, target group
 *    masking, max attention length); "Accuracy Alignment": N is the batch max_seqlen;
 *  - "Scaling HSTU: ragged execution, candidate amortization and content features",
 *    "Variable length is a central systems issue": jagged storage = values + offsets.
 *
 * The mask (c = num_contextuals[b], t = num_targets[b], E = L - t, W = max_attn_len):
 *    p(x) = x for x < E, else E - 1 (candidates take the last history position; p(x) = x if E = 0)
 *    valid(i,j) =  j >= E : i == j                      (candidate keys: seen by themselves only)
 *                  i < c  : j < c                       (contextual rows: bidirectional prefix)
 *                  j < c  : true                        (contextual keys: seen by every row)
 *                  else   : j <= p(i) && (W <= 0 || p(i) - j <= W)
 * Two variants, selected by params->flags: HSTU_FLAG_CTX_SEES_HISTORY makes a contextual row
 * see every key before the candidates (i < c : j < E); HSTU_FLAG_REL_ABS indexes the rel
 * table by min(|p(i) - p(j)|, R-1) instead of clamp(p(i) - p(j), 0, R-1), so bidirectional
 * pairs with p(i) < p(j) use their distance.
 *
 * Layouts (all row-major, packed over the T = seq_offsets[B] tokens of the batch):
 *    q, k        [T, H, d_qk]        dtype            dq, dk   [T, H, d_qk]  dtype
 *    v           [T, H, d_v]         dtype            dv       [T, H, d_v]   dtype
 *    u, out      [T, H * d_v]        dtype            du, dout [T, H * d_v]  dtype
 *    saved_y     [T, H * d_v]        fp32 (Y, already scaled by 1/N)
 *    saved_mean, saved_rstd [T]      fp32
 *    seq_offsets [B + 1] int64 (seq_offsets[0] = 0, non-decreasing, seq_offsets[B] = T)
 *    num_contextuals, num_targets [B] int32 (NULL = all zero)
 *    timestamps  [T] int64, in the caller's integer time unit (NULL allowed when NB = 0);
 *                |ts_i - ts_j| within a sequence must be below 2^63
 *    rel_bias [R], time_bias [NB], d_rel_bias [R], d_time_bias [NB]  fp32
 *
 * Ownership and synchronisation.  The caller allocates every buffer, including the
 * workspace.  fwd/bwd allocate nothing, never synchronise, and only enqueue work on
 * `stream` (a cudaStream_t; NULL = the legacy default stream).  All array pointers are
 * device pointers; `params` is a host pointer read before the call returns.  Device
 * pointers must be 16-byte aligned.  A workspace serves one call at a time: each call resets
 * the status word and the work-unit counter at its head, so calls that share a workspace
 * must run in order (one stream, or streams ordered by events).
 *
 * Errors.  Host-checkable problems (NULL required pointer, sizes out of range, misaligned
 * pointer, workspace too small) return a status before anything is enqueued.  Problems in
 * device-resident data (offsets not monotone, not starting at 0 or not ending at T, c + t > L,
 * L > max_seqlen) are not fatal: the offending sequence is skipped and a bit is set in the
 * status word at the start of the workspace; hstu_attn_read_device_status() reads it.  The
 * rows of a skipped sequence, and rows before seq_offsets[0] or from seq_offsets[B] on, get
 * zeros in out, saved_y, dk and dv (and the matching mean 0, rstd 1/sqrt(eps), dq 0, du 0),
 * so every output row is defined while the offsets are non-decreasing; where sequences
 * overlap, their rows are unspecified.  No kernel traps, and every wait inside a kernel is
 * bounded.
 */
#ifndef HSTU_ATTN_H
#define HSTU_ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    HSTU_OK = 0,
    HSTU_ERR_INVALID_ARGUMENT = 1,   /* bad pointer, size, alignment or parameter */
    HSTU_ERR_UNSUPPORTED = 2,        /* valid request outside the compiled kernel set */
    HSTU_ERR_WORKSPACE_TOO_SMALL = 3,
    HSTU_ERR_CUDA = 4,               /* a CUDA runtime call or launch failed */
    HSTU_ERR_DEVICE_DATA = 5         /* returned by hstu_attn_read_device_status only */
} hstu_status_t;

typedef enum { HSTU_F32 = 0, HSTU_BF16 = 1 } hstu_dtype_t;

/* Mask variants (params->flags). */
#define HSTU_FLAG_CTX_SEES_HISTORY 0x1   /* contextual rows attend to every non-candidate key */
#define HSTU_FLAG_REL_ABS          0x2   /* rel index min(|p(i) - p(j)|, R - 1) */
/* Forward (inference) only: compute the query tiles that hold candidate rows (rows >= E) and
 * skip the others, whose rows of out are then unspecified.  With target-group masking a
 * candidate's output depends only on the history and itself, so candidates can be scored in
 * micro-batches appended to a cached history ("Scaling HSTU: ragged execution, candidate
 * amortization and content features", "Many candidates make reuse valuable": M-FALCON). */
#define HSTU_FLAG_CANDIDATES_ONLY  0x4

/* Bits of the device status word. */
#define HSTU_DEV_BAD_OFFSETS   0x1   /* seq_offsets not non-decreasing / not ending at T */
#define HSTU_DEV_BAD_COUNTS    0x2   /* num_contextuals/num_targets negative or c + t > L */
#define HSTU_DEV_SEQ_TOO_LONG  0x4   /* a sequence longer than max_seqlen */
#define HSTU_DEV_WAIT_TIMEOUT  0x8   /* a bounded in-kernel wait gave up */

typedef struct {
    int32_t batch;            /* B >= 0 */
    int32_t num_heads;        /* H >= 1 */
    int32_t d_qk;             /* 1..256 (f32); multiple of 16 in 16..128 (bf16) */
    int32_t d_v;              /* as d_qk; H * d_v <= 2048 */
    int32_t max_seqlen;       /* N >= 1: the batch max of L; the 1/N scale. Host never reads offsets */
    int32_t max_attn_len;     /* W; <= 0 means unlimited */
    int64_t total_tokens;     /* T = seq_offsets[B] */
    float alpha;              /* score scale on q.k (not on the bias) */
    float ln_eps;             /* LayerNorm epsilon, e.g. 1e-5 */
    int32_t rel_bias_len;     /* R >= 0; 0 = no relative-position bias */
    int32_t time_bias_len;    /* NB in 0..256; 0 = no time bias (timestamps may be NULL) */
    double time_bucket_div;   /* > 0, e.g. 0.301 (natural log) */
    int32_t dtype;            /* hstu_dtype_t of q,k,v,u,out,dout,dq,dk,dv,du */
    int32_t flags;            /* HSTU_FLAG_* mask variants (0: the default mask); other bits 0 */
} hstu_attn_params_t;

/* Workspace bytes hstu_attn_fwd needs for these params (saved_y NULL or not). */
hstu_status_t hstu_attn_fwd_workspace_size(const hstu_attn_params_t *params, size_t *bytes);

/*
 * Forward.  Writes out; when saved_y is non-NULL also writes saved_y, saved_mean and
 * saved_rstd (all three or none), which hstu_attn_bwd consumes.
 */
hstu_status_t hstu_attn_fwd(const hstu_attn_params_t *params, const void *q, const void *k,
                            const void *v, const void *u, const int64_t *seq_offsets,
                            const int32_t *num_contextuals, const int32_t *num_targets,
                            const int64_t *timestamps, const float *rel_bias,
                            const float *time_bias, void *out, float *saved_y,
                            float *saved_mean, float *saved_rstd, void *workspace,
                            size_t workspace_bytes, void *stream);

/* Workspace bytes hstu_attn_bwd needs for these params. */
hstu_status_t hstu_attn_bwd_workspace_size(const hstu_attn_params_t *params, size_t *bytes);

/*
 * Backward of loss = sum(dout (.) out).  Inputs as for the forward plus dout and the
 * saved_y/mean/rstd written by the forward on the same inputs.  Overwrites dq, dk, dv, du
 * and (when the table is present) d_rel_bias / d_time_bias.
 */
hstu_status_t hstu_attn_bwd(const hstu_attn_params_t *params, const void *dout, const void *q,
                            const void *k, const void *v, const void *u,
                            const int64_t *seq_offsets, const int32_t *num_contextuals,
                            const int32_t *num_targets, const int64_t *timestamps,
                            const float *rel_bias, const float *time_bias, const float *saved_y,
                            const float *saved_mean, const float *saved_rstd, void *dq, void *dk,
                            void *dv, void *du, float *d_rel_bias, float *d_time_bias,
                            void *workspace, size_t workspace_bytes, void *stream);

/*
 * Reads the device status word at the start of `workspace` after the work queued on
 * `stream` finishes (synchronises `stream`).  *code receives the HSTU_DEV_* bits (0 = ok).
 * Returns HSTU_ERR_DEVICE_DATA when *code != 0.
 */
hstu_status_t hstu_attn_read_device_status(const void *workspace, void *stream, int32_t *code);

/*
 * Test hook: writes the mask of sequence `seq` as evaluated by the device predicate the
 * kernels use, row-major bits (bit j of row i at word (i*L + j) / 32, bit (i*L + j) % 32),
 * into `bits` (device, ceil(L*L/32) words, L = seq_offsets[seq+1]-seq_offsets[seq] which the
 * caller passes as seq_len).  Enqueued on `stream`.
 */
hstu_status_t hstu_attn_debug_mask(const hstu_attn_params_t *params, const int64_t *seq_offsets,
                                   const int32_t *num_contextuals, const int32_t *num_targets,
                                   int32_t seq, int32_t seq_len, uint32_t *bits, void *stream);

/*
 * Test hook: the mask of sequence `seq` as the tensor-core kernels decide it (bf16 inputs;
 * the forward for any admitted head dims, the backward for d_qk and d_v in {64, 128}): a
 * pair is valid when the kernel visits its 128 x 128 tile and
 * the 32-wide block the pair lies in marks it.  kernel = 0 selects the forward's decisions
 * (per query row and 32-key block), kernel = 1 the backward's (per key and 32-query block).
 * Writes rows [row_begin, row_begin + row_count) x keys [0, key_count) of the mask, row-major,
 * bit j of row r at word r * key_count / 32 + j / 32, bit j % 32, into `bits` (device,
 * row_count * key_count / 32 words).  Rows and keys past the sequence's end are included (up
 * to the tile padding, 128 * ceil(L / 128)): a kernel must never mark them valid for a row
 * (forward) or key (backward) it stores.  key_count must be a multiple of 32; row_begin and
 * row_count are >= 0.  Enqueued on `stream`; the same mask as "HSTU-MUSA: HSTU for Moore
 * Threads (MUSA)", section "Mathematical Equivalence", when the kernels are correct.
 */
hstu_status_t hstu_attn_debug_kernel_mask(const hstu_attn_params_t *params,
                                          const int64_t *seq_offsets,
                                          const int32_t *num_contextuals,
                                          const int32_t *num_targets, int32_t seq,
                                          int32_t kernel, int32_t row_begin, int32_t row_count,
                                          int32_t key_count, uint32_t *bits, void *stream);

/*
 * Host helper: the time-bucket thresholds the device compares against.  out[k-1] is the
 * smallest |dt| whose bucket is >= k, for k = 1..nb-1, with the bucket decided in fp64
 * exactly as floor(log((double)|dt| + 1.0) / div) (UINT64_MAX when never reached).
 */
hstu_status_t hstu_attn_time_thresholds(double div, int32_t nb, uint64_t *out);

/*
 * Forward for callers that cannot allocate device memory (no counterpart in the paper; it
 * is a deployment convenience).  Some callers cannot provide the workspace hstu_attn_fwd
 * asks for: a plugin inside a framework that owns all device memory and offers no
 * allocation hook, or a latency-critical serving loop in which cudaMalloc, which can
 * synchronise the device, is not allowed.  This entry point computes the same inference
 * forward as hstu_attn_fwd (out only; no saved activations) with its scratch in a fixed
 * 32 MiB array that the library declares in device memory; each GPU that loads the library
 * keeps that array until the process exits.  It allocates and frees nothing.
 *   - Arguments: as hstu_attn_fwd, without saved_y/mean/rstd and without a workspace.
 *   - Limit: the scratch need is 256 + 4 * total_tokens * num_heads * d_v bytes; a request
 *     above 32 MiB returns HSTU_ERR_WORKSPACE_TOO_SMALL before anything is enqueued.
 *   - Set-up: the first call on each device looks up the array's device address (with that
 *     device current), and so does the first call after that device's context was reset
 *     (cudaDeviceReset); make those calls before any stream capture.
 *   - Sharing: all calls on a device share the one array, which keeps the last call's
 *     contents (the status word is cleared by every call).  Calls that overlap on the GPU
 *     (other streams, other threads) race on it: serialise them.
 *   - Device-data errors skip the offending sequences as in hstu_attn_fwd, but their status
 *     bits stay inside the shared scratch; callers that need them use hstu_attn_fwd.
 */
hstu_status_t hstu_attn_fwd_noalloc(const hstu_attn_params_t *params, const void *q,
                                    const void *k, const void *v, const void *u,
                                    const int64_t *seq_offsets, const int32_t *num_contextuals,
                                    const int32_t *num_targets, const int64_t *timestamps,
                                    const float *rel_bias, const float *time_bias, void *out,
                                    void *stream);

/* Kernel stages of fwd/bwd, for hstu_attn_set_stage_events. */
#define HSTU_STAGE_FWD_ATTN 0   /* forward attention (scores, bias, SiLU, mask, A V) */
#define HSTU_STAGE_FWD_NORM 1   /* forward LayerNorm + U gating */
#define HSTU_STAGE_BWD_NORM 2   /* backward of LayerNorm + U gating (dU, dY) */
#define HSTU_STAGE_BWD_ATTN 3   /* backward attention (dQ, dK, dV, table gradients) */
#define HSTU_NUM_STAGES 4

/*
 * Measurement hook.  While set, every fwd/bwd call records `start_event` on its stream just
 * before launching the kernel(s) of `stage` and `stop_event` just after (both cudaEvent_t).
 * NULL events clear the hook.  Process-wide and not thread-safe: for benchmarks only.  A
 * call made while its stream is being captured into a CUDA graph records the events as
 * graph nodes of their own, so every replay of the graph stamps them.
 */
hstu_status_t hstu_attn_set_stage_events(int32_t stage, void *start_event, void *stop_event);

/*
 * Test hook for the bounded waits.  limit_cycles (> 0) replaces, for every later fwd/bwd
 * launch, the number of SM clock cycles a pipeline wait inside the tensor-core kernels may
 * take before the kernel gives up (0 restores the default, about 2 s); the waits that let
 * copies and MMAs in flight finish before a block exits keep the default.  stall = 1 makes
 * the MMA issuer of those kernels first wait on a barrier that nothing completes, so that
 * wait runs out, HSTU_DEV_WAIT_TIMEOUT is set in the status word and every role of the
 * kernel unwinds as after any timeout (outputs then unspecified); stall = 0 turns it off.
 * Process-wide and not thread-safe: for tests only.
 */
hstu_status_t hstu_attn_set_wait_test(int64_t limit_cycles, int32_t stall);

/*
 * The layer around the attention ("HSTU tensor by tensor: SiLU aggregation, temporal bias and
 * gating": "Similar shape, different aggregation", o_i = W_o[U_i (.) Norm(sum_j A_ij V_j)] + x_i;
 * "Trace four projections": normalised inputs produce U/V/Q/K through one larger projection
 * split to match the weight layout).  bf16 tensors, fp32 biases, row-major, 16-byte aligned
 * device pointers; each call enqueues kernels on `stream` and allocates nothing.  status
 * (device int32, may be NULL) receives HSTU_DEV_WAIT_TIMEOUT if a bounded wait gave up.
 *
 * hstu_layer_norm_rows: y = LayerNorm(x) per row of `width` (multiple of 32, <= 1024) values,
 * no affine (biased variance, eps inside the square root): the input normalisation.
 *
 * hstu_uvqk_proj: [T, N] = x [T, d_model] w [d_model, N] (+ bias [N]) (SiLU of every value when
 * silu = 1), N = 2 H (d_v + d_qk), columns ordered U | V | Q | K, each head-major; written as
 * u [T, H*d_v], v [T, H, d_v], q [T, H, d_qk], k [T, H, d_qk] -- the layouts hstu_attn_fwd
 * takes.  d_model, H*d_v and H*d_qk must be multiples of 64.
 *
 * hstu_out_proj: out [T, d_model] = z [T, d_in] w_o [d_in, d_model] (+ bias [d_model]) (+ x
 * [T, d_model], the residual; NULL for none).  d_in and d_model multiples of 64.
 */
hstu_status_t hstu_layer_norm_rows(const void *x, void *y, int64_t rows, int32_t width,
                                   float eps, void *stream);
hstu_status_t hstu_uvqk_proj(const void *x, const void *w, const float *bias, int64_t tokens,
                             int32_t d_model, int32_t num_heads, int32_t d_qk, int32_t d_v,
                             int32_t silu, void *u, void *v, void *q, void *k, int32_t *status,
                             void *stream);
hstu_status_t hstu_out_proj(const void *z, const void *w_o, const float *bias, const void *x,
                            int64_t tokens, int32_t d_in, int32_t d_model, void *out,
                            int32_t *status, void *stream);

/*
 * Stochastic Length ("Scaling HSTU: ragged execution, candidate amortization and content
 * features", "Variable length is a central systems issue": it samples sequence lengths in
 * training).  Reading (the page gives no formula): sequence b keeps its contextual prefix
 * (num_contextuals[b] tokens) and candidates (the last num_targets[b]), and of its h history
 * tokens the min(h, budget) whose keys are smallest, the earlier position first on equal
 * keys, all in their original order.  keys [total_tokens] fp32 (device, no NaN) are the
 * caller's random numbers, one per token (history tokens' keys are read).  Writes
 * out_offsets [batch + 1] (device, int64; the new jagged offsets) and out_rows (device,
 * int64, room for total_tokens): the kept rows as indices into the input rows, sequence by
 * sequence; hstu_gather_rows then gathers any per-token tensor.  A sequence with invalid
 * offsets or counts keeps nothing and sets a HSTU_DEV_* bit in *status (device int32,
 * NULL = not reported).  Enqueued on `stream`; allocates nothing.
 */
hstu_status_t hstu_stochastic_length(const int64_t *seq_offsets, const int32_t *num_contextuals,
                                     const int32_t *num_targets, int32_t batch,
                                     int64_t total_tokens, const float *keys, int32_t budget,
                                     int64_t *out_rows, int64_t *out_offsets, int32_t *status,
                                     void *stream);

/*
 * dst row r = src row rows[r] for r < min(*n_rows, max_rows); rows of row_bytes bytes.  rows
 * and n_rows (a count, e.g. the last entry of jagged offsets) are device memory, read on the
 * device; max_rows bounds the work from the host.  Indices must lie inside src.
 */
hstu_status_t hstu_gather_rows(const void *src, int64_t row_bytes, const int64_t *rows,
                               const int64_t *n_rows, int64_t max_rows, void *dst, void *stream);

/*
 * Jagged concatenation ("HSTU-MUSA: HSTU for Moore Threads (MUSA)", "Project Structure":
 * jagged tensor concatenation): n_parts (1..16) jagged tensors of the same row width
 * row_bytes, part q given by values[q] and offsets[q] ([batch + 1], device), become one whose
 * sequence b holds the rows of part 0's sequence b, then part 1's, ...  values and offsets
 * are host arrays of device pointers; out_offsets [batch + 1] (device) receives the sums of
 * the parts' offsets, out_values room for all rows.  E.g. contextual, history and candidate
 * tokens into one sequence per user.
 */
hstu_status_t hstu_jagged_concat(int32_t n_parts, const void *const *values,
                                 const int64_t *const *offsets, int32_t batch, int64_t row_bytes,
                                 void *out_values, int64_t *out_offsets, void *stream);

/* Static description of a status code. */
const char *hstu_status_string(hstu_status_t status);

/* Library version, e.g. 100 for 0.1.0. */
int32_t hstu_attn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* HSTU_ATTN_H */
