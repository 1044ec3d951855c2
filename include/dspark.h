/*
 * dspark.h -- C ABI of the DSpark drafter-head hot path on one B200 (sm_100a).
 *
 * The method is described on three web pages about DSpark:
 *   [G] gdymind.com, "DSpark: DeepSeek's new speculative decoding work (Video + Blog)"
 *   [W] wispaper.ai, "DSpark: Overcoming the Efficiency Wall in LLM Speculative Decoding"
 *   [S] seventnews.com, "DeepSeek's DSpark just fixed the two things that held back
 *       faster AI inference"
 *
 * Conventions shared by every call:
 *   - Every array argument is caller-owned DEVICE memory, contiguous and row-major.
 *     The library never allocates or frees device memory and keeps no pointer
 *     after a call returns.
 *   - bf16 arrays are passed as `const void*` (2-byte bf16 storage).
 *   - `stream` is the caller's cudaStream_t.  All work is enqueued on it and is
 *     asynchronous; no call synchronises except dspark_get_error.
 *   - The return value is a dspark_status.  Host-side argument checks run before
 *     anything is enqueued; on a non-zero return nothing was enqueued.
 *   - Problems seen on the device (an out-of-range token id, scores that are not
 *     non-increasing, a wait that ran out) are recorded in a per-device error
 *     word that dspark_get_error reads and clears.
 *   - Not thread-safe across concurrent calls that share a workspace.
 */
#ifndef DSPARK_H
#define DSPARK_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *dspark_stream_t; /* same type as cudaStream_t */

typedef enum {
    DSPARK_OK = 0,
    DSPARK_INVALID_ARG = 1,       /* null pointer, bad size, misaligned pointer   */
    DSPARK_UNSUPPORTED_SHAPE = 2, /* a size outside what the kernels support     */
    DSPARK_WORKSPACE_TOO_SMALL = 3,
    DSPARK_NOT_MONOTONE = 4,      /* device: scores increase along a request      */
    DSPARK_CUDA_ERROR = 5,        /* a CUDA runtime/driver call failed            */
    DSPARK_TIMEOUT = 6,           /* device: a bounded wait ran out               */
    DSPARK_INVALID_TOKEN = 7,     /* device: a token id or length out of range    */
    DSPARK_BAD_LAUNCH = 8         /* device: a kernel found itself launched in a
                                     shape it cannot run in (e.g. a tool re-issued
                                     the launch without its thread-block cluster);
                                     it returned before touching memory          */
} dspark_status;

/* Text for a status code (static storage). */
const char *dspark_status_string(int status);

/* Number of bytes of device workspace dspark_draft_step and dspark_schedule_prefix
 * need for these sizes (the larger of the two).  The workspace must be 256-byte
 * aligned; its contents need no initialisation and are overwritten by each call. */
size_t dspark_workspace_bytes(int B, int gamma, int V, int r);

/*
 * Markov-head drafting, all gamma positions of one draft block.
 * [G] section 4 "Semi-Autoregressive Generation" (sequential stage, Markov head:
 * first-order transition B = W1 W2 with W1 [V, r] an embedding table and W2 [r, V]
 * a logits projection, r = 256) and section 4 "Parallel stage" (the anchor is the
 * first prediction position, so gamma inputs give gamma logits).
 *
 * For k = 1..gamma, with x_0 = anchor[b]:
 *   l_k(v) = U[b, k-1, v] + sum_j W1[x_{k-1}, j] W2[j, v]         (fp32 accumulate)
 *   mode 0 (greedy):     x_k = argmax_v l_k(v), smallest v among equal maxima
 *   mode 1 (Gumbel-max): x_k = argmax_v l_k(v) / temperature + g(b + b_offset, k, v)
 *     with g = -ln(-ln u), u = ((w >> 9) + 0.5) 2^-23 and w word (v mod 4) of
 *     Philox4x32-10(counter = (v / 4, k - 1, b + b_offset, 0),
 *                   key = (low 32 bits of seed, high 32 bits of seed)).
 *   x_out[b, k-1] = x_k;  logit_x_out[b, k-1] = l_k(x_k) (the unperturbed logit).
 * The [B, V] logits are never written to memory.
 *
 *   U        [B, gamma, V] bf16   backbone base logits U_k
 *   anchor   [B] int32            x_0; must lie in [0, V)
 *   W1       [V, r] bf16          Markov embedding table
 *   W2       [r, V] bf16          logits projection
 *   x_out    [B, gamma] int32     drafted tokens
 *   logit_x_out [B, gamma] fp32
 *   workspace, workspace_bytes    >= dspark_workspace_bytes(B, gamma, V, r)
 * Supported sizes: 1 <= B <= 1024, 1 <= gamma <= 64, r == 256, 64 <= V <= 2^24,
 * V % 8 == 0; U, W1, W2 16-byte aligned.  temperature > 0 in mode 1.
 * An anchor outside [0, V) records DSPARK_INVALID_TOKEN and is read as token 0.
 * The kernel is a cooperative launch of one CTA per SM whose steps are joined
 * by a grid barrier; every device-side wait is bounded (dspark_set_wait_timeout_ns)
 * and records DSPARK_TIMEOUT instead of hanging.
 */
int dspark_draft_step(const void *U, const int32_t *anchor, const void *W1, const void *W2,
                      int B, int gamma, int V, int r, int mode, float temperature,
                      uint64_t seed, int b_offset, int32_t *x_out, float *logit_x_out,
                      void *workspace, size_t workspace_bytes, dspark_stream_t stream);

/*
 * RNN-head drafting: the second sequential block of [G] section 4 ("Two
 * instantiations of the sequential block": a recurrent state that accumulates the
 * block's prefix).  The pages give no equations; this is the Elman reading over the
 * Markov head's factors:
 *   s_0 = 0,  s_k = tanh(W1[x_{k-1}] + s_{k-1} Whh)     (fp32 state, r = 256)
 *   l_k(v) = U[b, k-1, v] + sum_j bf16(s_k)[j] W2[j, v]
 * and x_k, logit_x_out as in dspark_draft_step (greedy or Gumbel-max).
 *   Whh [r, r] bf16 (row i, column j: s_{k-1}[i] contributes Whh[i][j] to element j),
 *   16-byte aligned.  Every other argument as for dspark_draft_step; the workspace
 *   from dspark_workspace_bytes also holds the [B, r] state.
 * Cost over the Markov head: one more grid barrier per position and B r^2 MACs.
 */
int dspark_draft_step_rnn(const void *U, const int32_t *anchor, const void *W1, const void *W2,
                          const void *Whh, int B, int gamma, int V, int r, int mode,
                          float temperature, uint64_t seed, int b_offset, int32_t *x_out,
                          float *logit_x_out, void *workspace, size_t workspace_bytes,
                          dspark_stream_t stream);

/*
 * Confidence head with Sequential Temperature Scaling and prefix survival.
 * [G] section 5 "Confidence-Scheduled Verification" (linear projection then
 * sigmoid over the backbone hidden state at position k and the Markov embedding
 * of the previous draft token; temperature scaling per position) and [S]
 * (the survival probability of every prefix of the block, a cumulative product).
 *
 *   z_{b,k} = sum_i w[i] h[b, k-1, i] + sum_j w[d + j] W1[x_{k-1}, j] + b_conf
 *   c_{b,k} = 1 / (1 + exp(-z_{b,k} / T[k-1]))
 *   P_{b,k} = P_{b,k-1} * c_{b,k} in fp32, P_{b,0} = 1
 * with x_0 = anchor[b], x_{k-1} = x[b, k-2] for k >= 2.
 *
 *   h [B, gamma, d] bf16;  anchor [B] int32;  x [B, gamma] int32 (last column unused)
 *   W1 [V, r] bf16;  w [d + r] bf16;  T [gamma] fp32 (> 0)
 *   c_out, P_out [B, gamma] fp32
 * Supported sizes: 1 <= B <= 65535, 1 <= gamma <= 64, d % 8 == 0, r % 8 == 0,
 * (d + r) 2 <= 200 KB; h, W1, w 16-byte aligned.  A token id outside [0, V) records
 * DSPARK_INVALID_TOKEN and is read as 0.  Launched as one thread-block cluster of up to
 * 8 CTAs per request.
 */
int dspark_confidence_sts(const void *h, const int32_t *anchor, const int32_t *x,
                          const void *W1, const void *w, float b_conf, const float *T,
                          int B, int gamma, int d, int r, int V, float *c_out, float *P_out,
                          dspark_stream_t stream);

/*
 * Drafting and the confidence head in one call: the results of dspark_draft_step
 * followed by dspark_confidence_sts on the drafted tokens.
 * [G] section 4 (Markov head) and section 5 (the confidence head reads the backbone
 * hidden state at k and the Markov embedding of x_{k-1}, the row the draft gathers).
 *
 * Arguments as for those two calls (U, anchor, W1, W2, mode, temperature, seed, b_offset,
 * x_out, logit_x_out, workspace as for dspark_draft_step; h, w, b_conf, T, d, c_out,
 * P_out as for dspark_confidence_sts), with the same sizes, alignment and errors.  Both
 * run in one launch: one warp of every CTA of the draft kernel computes the hidden-state
 * part of every logit at the start and the rest of each position's scores as soon as the
 * grid barrier of the previous position has fixed x_{k-1}, beside the drafting; the
 * workspace from dspark_workspace_bytes covers it.  The exception is Gumbel-max drafting
 * (mode 1) with B > 128, whose selection arithmetic is the bound: there the confidence
 * kernel follows as a second launch on the same stream.  c and P agree with
 * dspark_confidence_sts up to the order of the fp32 additions of z.
 */
int dspark_draft_confidence_step(const void *U, const int32_t *anchor, const void *W1,
                                 const void *W2, const void *h, const void *w, float b_conf,
                                 const float *T, int B, int gamma, int V, int r, int d, int mode,
                                 float temperature, uint64_t seed, int b_offset, int32_t *x_out,
                                 float *logit_x_out, float *c_out, float *P_out, void *workspace,
                                 size_t workspace_bytes, dspark_stream_t stream);

/*
 * The whole per-step path in one call: dspark_draft_confidence_step, then
 * dspark_schedule_prefix on the survival scores it wrote, then dspark_verify_prefix on
 * the drafts and the lengths.  [G] sections 4-6 and [W] "The Hardware-Aware Prefix
 * Scheduler"; [S] (strict prefix-match verification with a bonus token).
 *
 * Arguments as for those calls (Tstep_us, L_out, N_out, objective_out as for
 * dspark_schedule_prefix; target, accepted_out, bonus_out as for dspark_verify_prefix),
 * with their sizes, alignment and errors, and one workspace of dspark_workspace_bytes
 * bytes for all of it.  With B <= 128 and B gamma <= 1024 it is one launch: after the
 * last position the draft kernel's CTAs rank every score (one warp per score) and the
 * last CTA to finish scans, picks N*, writes the lengths and verifies every request,
 * with the same device code as the two kernels, so the outputs equal those of the
 * separate calls bit for bit.  Otherwise the calls run as separate launches on the same
 * stream (there the scheduler kernel's many CTAs are faster than the launch saved).
 * Outputs are written in stream order; nothing is read back to the host.
 */
int dspark_step(const void *U, const int32_t *anchor, const void *W1, const void *W2,
                const void *h, const void *w, float b_conf, const float *T,
                const double *Tstep_us, const int32_t *target, int B, int gamma, int V, int r,
                int d, int mode, float temperature, uint64_t seed, int b_offset, int32_t *x_out,
                float *logit_x_out, float *c_out, float *P_out, int32_t *L_out, int32_t *N_out,
                double *objective_out, int32_t *accepted_out, int32_t *bonus_out,
                void *workspace, size_t workspace_bytes, dspark_stream_t stream);

/*
 * Hardware-aware prefix scheduler: per-request verify lengths that maximise
 * expected accepted tokens per unit time.
 * [W] "The Hardware-Aware Prefix Scheduler" (throughput maximisation against a
 * steps-per-second curve) and [G] section 6 (the choice is posed as maximising the
 * throughput of the whole batch).
 *
 * Scores P[b, k-1] (non-increasing in k, within [0, 1]) are ordered by
 * (P desc, b asc, k asc); q = floor(P 2^46); S_N = sum of the first N q's;
 *   F(N) = double(B 2^46 + S_N) / Tstep_us[B + N],   N = 0 .. B gamma
 * (int64 sum, which stays below (B + B gamma) 2^46 < 2^63 at every supported size;
 * round-to-nearest conversion and division).  N* = smallest N with
 * the largest F; L_out[b] = number of request b's entries among the first N*.
 *
 *   P [B, gamma] fp32;  Tstep_us [B (gamma + 1) + 1] fp64, Tstep_us[n] > 0 is the
 *   time of one target step that verifies n tokens (each request feeds its
 *   anchor/bonus position plus L_b drafts, so n = B + sum L).
 *   L_out [B] int32;  N_out [1] int32 (N*);  objective_out [1] fp64 = F(N*) 2^-46,
 *   expected accepted tokens (bonus included) per unit of Tstep's time.
 * Supported sizes: 1 <= B <= 32768, 1 <= gamma <= 64, B gamma <= 65536.
 * A score outside [0, 1] or an increase along a request records
 * DSPARK_NOT_MONOTONE (results are then unspecified but all writes stay in bounds).
 */
int dspark_schedule_prefix(const float *P, int B, int gamma, const double *Tstep_us,
                           int32_t *L_out, int32_t *N_out, double *objective_out,
                           void *workspace, size_t workspace_bytes, dspark_stream_t stream);

/*
 * Strict prefix-match verification.
 * [S]: a block is verified in one target pass; the accepted tokens stick and the
 * first rejected token and everything after it are dropped.
 *   accepted_out[b] = smallest k-1 (1 <= k <= L[b]) with x[b, k-1] != target[b, k-1],
 *                     or L[b] when the first L[b] drafts all agree
 *   bonus_out[b]    = target[b, accepted_out[b]]
 *   x [B, gamma] int32;  L [B] int32 in [0, gamma];  target [B, gamma + 1] int32
 *   (the target model's tokens at positions 1..gamma+1).
 * An L[b] outside [0, gamma] records DSPARK_INVALID_TOKEN and is clamped.
 */
int dspark_verify_prefix(const int32_t *x, const int32_t *L, const int32_t *target, int B,
                         int gamma, int32_t *accepted_out, int32_t *bonus_out,
                         dspark_stream_t stream);

/*
 * Sequential Temperature Scaling: fitting the per-position temperatures T [gamma]
 * that dspark_confidence_sts divides the confidence logits by.
 * [G] section 5 "Sequential Temperature Scaling": the joint (survival) probability is
 * calibrated position by position from left to right; at each position a 1-D grid
 * search picks the temperature minimising the expected calibration error (ECE) of the
 * cumulative product, with the temperatures of earlier positions kept fixed.
 *
 * Calibration set: N held-out draft blocks with raw confidence logits z[n, k-1] (the
 * logit before temperature scaling) and accepted lengths accepted[n] in 0..gamma.
 * For k = 1..gamma, label y = (accepted[n] >= k) and for each candidate
 * T_i = t_min + i t_step, i = 0..n_t-1:
 *   p_i[n] = P_{k-1}[n] / (1 + exp(-z[n, k-1] / T_i))      (fp64; P_0 = 1)
 *   ECE_i  = sum over bins m of |sum_{n in m} y - sum_{n in m} p_i| / N,
 *            bin(p) = min(floor(p n_bins), n_bins - 1)       (equal-width bins on [0, 1])
 * index_out[k-1] = the smallest i with the smallest ECE_i; T_out[k-1] = T_i (fp32);
 * ece_out[k-1] = ECE_i; then P_k = P_{k-1} / (1 + exp(-z[., k-1] / T_i)).
 * p is formed as P / (1 + exp(-z (1/T))) with a Newton-refined reciprocal (a
 * few ulp from the fp64 quotient).  Each CTA's fp64 bin sums are rounded to 2^-40 fixed
 * point before they are added across CTAs, so the result does not depend on the order
 * in which CTAs finish (an ECE moves by at most (CTAs x bins) 2^-41 / N); ties are
 * decided on those exact integer sums.
 *
 *   z          [N, gamma] fp32
 *   accepted   [N] int32
 *   index_out  [gamma] int32   (device memory; also read by the later positions)
 *   T_out      [gamma] fp32,  ece_out [gamma] fp64
 *   workspace, workspace_bytes >= dspark_sts_fit_workspace_bytes(N, gamma, n_t, n_bins)
 * Supported sizes: 1 <= N < 2^23, 1 <= gamma <= 64, 1 <= n_t <= 2^20,
 * 1 <= n_bins <= 256; t_min > 0, t_step >= 0.  Errors: DSPARK_INVALID_ARG (null or
 * misaligned pointer, bad grid), DSPARK_UNSUPPORTED_SHAPE, DSPARK_WORKSPACE_TOO_SMALL.
 */
size_t dspark_sts_fit_workspace_bytes(int N, int gamma, int n_t, int n_bins);
int dspark_sts_fit(const float *z, const int32_t *accepted, int N, int gamma, double t_min,
                   double t_step, int n_t, int n_bins, int32_t *index_out, float *T_out,
                   double *ece_out, void *workspace, size_t workspace_bytes,
                   dspark_stream_t stream);

/*
 * The prefix scheduler for callers that cannot allocate device memory.
 * (No counterpart on the DSpark pages: this is an interface convenience.)
 *
 * Same arguments, results and error behaviour as dspark_schedule_prefix, minus the
 * workspace.  It is meant for callers that have no way to hand the library a workspace:
 * processes whose device memory is fixed when they start (a serving engine that divides
 * all of HBM into its own pools, an embedded runtime with a set memory budget), or code
 * that must not call cudaMalloc at this point because the call can synchronise the device
 * and stall other streams.  The library calls no allocating routine here either.
 *
 * Scratch lives in one statically sized array inside this library's device image
 * (288 KB, held by every GPU that loads the library until the process exits), so:
 *   - B * gamma must not exceed 24576; larger sizes return DSPARK_UNSUPPORTED_SHAPE;
 *   - every call on a device shares that array, and the array keeps the last call's
 *     contents: calls that can overlap on the GPU (different streams, or different host
 *     threads without ordering between their streams) race and give wrong results;
 *     order them on one stream;
 *   - every call looks the array's device address up (cudaGetSymbolAddress) with the
 *     calling device current.  The first call on a device may make the CUDA runtime
 *     load this library's device code there (lazy module loading), which allocates
 *     device memory for the image and can synchronise the device: make that first call
 *     during start-up, before any stream capture.  From the second call on, the call
 *     neither allocates nor synchronises.
 */
int dspark_schedule_prefix_noalloc(const float *P, int B, int gamma, const double *Tstep_us,
                                   int32_t *L_out, int32_t *N_out, double *objective_out,
                                   dspark_stream_t stream);

/* Synchronises `stream`, then reads and clears the device error word of the
 * current device into *status (DSPARK_OK when nothing was recorded). */
int dspark_get_error(dspark_stream_t stream, int *status);

/* Limit in nanoseconds for every device-side wait of dspark_draft_step
 * (default 2e9).  Applies to launches made after the call. */
int dspark_set_wait_timeout_ns(uint64_t ns);

/* Test hook: the draft kernel's grid barrier waits for `extra` more arrivals than
 * there are CTAs, so that its bounded wait runs out (0 restores normal use). */
int dspark_debug_barrier_extra(int extra);

#ifdef __cplusplus
}
#endif

#endif /* DSPARK_H */
