/*
 * specdec.h -- C-ABI of libspecdec.so: the batched speculative-sampling verify
 * step on an NVIDIA B200 (sm_100a).
 *
 * The operation (Leviathan et al., as restated on the speculative decoding blog
 * page "Speculative Decoding ... Llama 70B x2.4", section "The mathematical
 * definition from Leviathan et al. (Google DeepMind, 2023)"):
 *
 *   For each sequence b, with p_i = softmax(target_logits[b,i,:] / T_b) and
 *   q_i = softmax(draft_logits[b,i,:] / T_b):
 *     for i = 0..K-1: accept draft token x_i = draft_tokens[b,i] iff
 *                     u_accept[b,i] * q_i(x_i) < p_i(x_i)
 *                     (i.e. u < alpha(x) = min(1, p/q)); stop at the first
 *                     rejection, at position n;
 *     if n < K : draw y from the corrected distribution
 *                p'(v) = max(0, p_n(v) - q_n(v)) / Z   ("resample");
 *     if n == K: draw y from p_K, the target's extra row ("bonus" token, as
 *                in the SMC-SD page "Faster LLM Inference via Sequential
 *                Monte Carlo", section 2, scoring step);
 *     the draw is the inverse CDF with the supplied uniform:
 *                y = min{ j : sum_{v<=j} r(v) > u_resample[b] * sum_v r(v) },
 *                sums in ascending token order.
 *   Outputs: out_tokens[b,0..n-1] = x_0..x_{n-1}, out_tokens[b,n] = y,
 *            out_tokens[b,n+1..K] = -1, out_num_accepted[b] = n.
 *   Temperature applies to both models (the blog's vLLM example sets
 *   temperature=0.7; its trade-off 4 discusses T=0.3..1.0).
 *
 * Layouts (all row-major, the vocabulary dimension contiguous):
 *   target_logits    [B, K+1, V]  bf16 or fp32 (see specdec_dtype)
 *   draft_logits     [B, K,   V]  same dtype as the target
 *   draft_tokens     [B, K]       int32
 *   u_accept         [B, K]       fp32 in [0, 1)
 *   u_resample       [B]          fp32 in [0, 1)
 *   temperature      [B]          fp32, finite and > 0 (one per sequence)
 *   out_tokens       [B, K+1]     int32
 *   out_num_accepted [B]          int32
 *
 * Ownership: every pointer is owned by the caller.  Unless a function says
 * otherwise, pointers are DEVICE memory of the current CUDA device and the call
 * is asynchronous on `stream` (a cudaStream_t; NULL is the legacy default
 * stream): nothing is synchronised, results are valid once the stream reaches
 * the end of the call.  The kernels are launched with programmatic dependent
 * launch: a call's first kernel may be placed on the GPU while the kernel
 * before it on the stream is still running, but it reads no input and writes
 * nothing until that kernel has completed, so stream order holds for the
 * caller's producers of the inputs.  (Before that wait the statistics sweep
 * may ask for its first input tiles to be brought into L2: a cache hint that
 * reads nothing, and L2 stays coherent with whatever that kernel writes.)  The call's last kernel lets a following
 * kernel launched with programmatic serialisation start early; such a kernel
 * must call cudaGridDependencySynchronize() before it reads the outputs (as
 * the programming model requires of it anyway).  The logit pointers must be
 * aligned to their element size; 16-byte alignment of every row (V * element
 * size a multiple of 16) gives the fast vector path, other layouts take a
 * slower scalar path.
 *
 * Errors:
 *   SPECDEC_EINVAL  an argument is invalid (checked on the host before any
 *                   launch; nothing is written): a null pointer with B > 0,
 *                   B < 0, K outside [1, 32], V < 1, sizes that overflow,
 *                   misaligned logits, an unknown dtype.  B == 0 is a no-op.
 *   SPECDEC_ECUDA   a CUDA runtime call failed (launch, allocation, copy).
 *   SPECDEC_ESTATE  the library-owned workspace would have to grow while
 *                   `stream` is being captured into a CUDA graph (call once
 *                   with the same or larger sizes before capturing).
 *   Per-sequence input errors are found on the device and never fault:
 *   a draft token outside [0, V), a temperature that is not finite and > 0,
 *   or a logit row holding NaN or +Inf or only -Inf make that sequence's
 *   out_num_accepted -1 and all its out_tokens -1, and set a bit in a
 *   per-device error word (see specdec_device_errors).
 * Determinism: results are bit-identical for identical inputs and sizes.
 */
#ifndef SPECDEC_H
#define SPECDEC_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum specdec_status {
  SPECDEC_OK = 0,
  SPECDEC_EINVAL = 1,
  SPECDEC_ECUDA = 2,
  SPECDEC_EDEVICE = 3,
  SPECDEC_ESTATE = 4,
  SPECDEC_ESIZE = 5
} specdec_status;

typedef enum specdec_dtype { SPECDEC_F32 = 0, SPECDEC_BF16 = 1 } specdec_dtype;

/* bits of the per-device error word */
#define SPECDEC_ERR_TOKEN 1u       /* a draft token outside [0, V)            */
#define SPECDEC_ERR_TEMPERATURE 2u /* a temperature not finite and > 0        */
#define SPECDEC_ERR_LOGITS 4u      /* a row with NaN / +Inf / only -Inf       */
#define SPECDEC_ERR_TIMEOUT 8u     /* a bounded on-chip wait ran out: every
                                      sequence whose row statistics it left
                                      incomplete gets outputs -1            */

/* Optional diagnostics (device pointers, each nullable).  Row order per
 * sequence: target rows 0..K, then draft rows 0..K-1.
 *   row_max [B, 2K+1] float : max_v z_v
 *   row_sum [B, 2K+1] double: sum_v exp((z_v - max) / T)
 *   p_x, q_x [B, K]  double: p_i(x_i), q_i(x_i) for positions i <= n only
 *                            (other entries are left untouched)
 *   Z [B]            double: mass of the distribution drawn from,
 *                            sum_v max(0, p_n - q_n) or sum_v p_K (~1)      */
typedef struct specdec_debug {
  float *row_max;
  double *row_sum;
  double *p_x;
  double *q_x;
  double *Z;
} specdec_debug;

/* The verify step (see the top of this file).  Uses a workspace owned by the
 * library, one per (device, stream): calls on different streams may overlap on
 * the GPU and never share one.  A workspace is grown on demand with cudaMalloc,
 * which synchronises the device the first time a stream sees a larger size. */
specdec_status specdec_verify(const void *target_logits, const void *draft_logits,
                              const int32_t *draft_tokens, const float *u_accept,
                              const float *u_resample, const float *temperature, int B, int K,
                              int V, specdec_dtype dtype, int32_t *out_tokens,
                              int32_t *out_num_accepted, void *stream);

/* Same as specdec_verify with the dtype fixed. */
specdec_status specdec_verify_bf16(const void *target_logits, const void *draft_logits,
                                   const int32_t *draft_tokens, const float *u_accept,
                                   const float *u_resample, const float *temperature, int B,
                                   int K, int V, int32_t *out_tokens, int32_t *out_num_accepted,
                                   void *stream);
specdec_status specdec_verify_f32(const void *target_logits, const void *draft_logits,
                                  const int32_t *draft_tokens, const float *u_accept,
                                  const float *u_resample, const float *temperature, int B,
                                  int K, int V, int32_t *out_tokens, int32_t *out_num_accepted,
                                  void *stream);

/* Bytes of device workspace specdec_verify_ex needs for these sizes
 * (0 for invalid sizes). */
size_t specdec_workspace_bytes(int B, int K, int V, specdec_dtype dtype);

/* specdec_verify with a caller-owned workspace (device memory of at least
 * specdec_workspace_bytes bytes, 256-byte aligned; its contents need no
 * initialisation) and optional diagnostics (dbg may be NULL).  Allocates
 * nothing.  Calls that share a workspace must not overlap on the device. */
specdec_status specdec_verify_ex(const void *target_logits, const void *draft_logits,
                                 const int32_t *draft_tokens, const float *u_accept,
                                 const float *u_resample, const float *temperature, int B,
                                 int K, int V, specdec_dtype dtype, void *workspace,
                                 size_t workspace_bytes, const specdec_debug *dbg,
                                 int32_t *out_tokens, int32_t *out_num_accepted, void *stream);

/* Early-exit verify: the same operation, the same outputs, fewer bytes read.
 *
 * The pages stop the verification at the first rejected draft token (the
 * speculative decoding blog, "The mathematical definition from Leviathan et
 * al.": tokens are checked in order and the first disagreement ends the step;
 * the SMC-SD page, section 1 and "Key differences from standard SD": in
 * standard SD the first rejection truncates the draft block and the tokens
 * after it are discarded).  The rows of positions after the first
 * rejection (and the target's bonus row unless every draft token is accepted)
 * never influence the result, so they need not be read.  This call reads the
 * rows of positions 0 and 1 of every sequence first, decides the sequences
 * rejected there, and then reads positions 2..K-1 and the bonus row only of the
 * sequences that accepted both: two statistics sweeps and two finish passes
 * instead of one of each.  Worth it when acceptance is low (at mean acceptance
 * a it reads about (4 + a^2 (2K-3)) / (2K+1) of the logits); at high acceptance
 * the second pass costs more launch latency than it saves.
 * Arguments, layouts, errors and results are those of specdec_verify /
 * specdec_verify_ex (diagnostics: row statistics only of the rows read, p_x
 * and q_x of the positions tested).  The row statistics are reduced over a
 * different split of the rows than in specdec_verify, so probabilities agree
 * with it to rounding (a few 1e-7) rather than bit for bit. */
specdec_status specdec_verify_early_exit(const void *target_logits, const void *draft_logits,
                                         const int32_t *draft_tokens, const float *u_accept,
                                         const float *u_resample, const float *temperature,
                                         int B, int K, int V, specdec_dtype dtype,
                                         int32_t *out_tokens, int32_t *out_num_accepted,
                                         void *stream);
specdec_status specdec_verify_early_exit_ex(const void *target_logits, const void *draft_logits,
                                            const int32_t *draft_tokens, const float *u_accept,
                                            const float *u_resample, const float *temperature,
                                            int B, int K, int V, specdec_dtype dtype,
                                            void *workspace, size_t workspace_bytes,
                                            const specdec_debug *dbg, int32_t *out_tokens,
                                            int32_t *out_num_accepted, void *stream);

/* SMC-SD weight step (the SMC-SD page "Faster LLM Inference via Sequential
 * Monte Carlo", section 2, "Methodology" and "Key differences from standard
 * SD"): N draft particles per group extend their sequences by K draft tokens;
 * the target scores all N x (K+1) positions; no token is rejected.  For each
 * particle b (B = G*N particles, G groups of N consecutive particles):
 *   out_tokens[b, 0..K-1] = draft_tokens[b, :] and out_tokens[b, K] = the
 *     bonus token drawn from p_K = softmax(target_logits[b, K, :] / T_b) with
 *     u_bonus[b] by the inverse-CDF rule of specdec_verify;
 *   log_weight_increment[b] = sum_i [log p_i(x_i) - log q_i(x_i)] (fp64;
 *     p_i, q_i the temperature softmaxes of target and draft row i);
 *   log w = log_weights_in[b] (0 when log_weights_in is NULL) + increment.
 * Per group g: normalised weights wbar = exp(log w - max) / sum, ess[g] =
 * 1 / sum wbar^2 (fp64).  If ess[g] < ess_threshold * N the group is
 * resampled systematically with the single uniform u_resample[g]:
 * ancestors[g*N + k] = min{j : C_j > (k + u)/N} (C the running sum of wbar in
 * particle order; an index within the group) and log_weights_out = 0;
 * otherwise ancestors[g*N + k] = k and log_weights_out = log w.  The caller
 * applies the ancestors to its particle state (e.g. KV-cache pages).
 * Layouts: logits, tokens, temperature as in specdec_verify; u_bonus [B],
 * log_weights_in / log_weights_out / log_weight_increment [B] fp64 (in and
 * increment nullable; out may alias in), u_resample [G], ess [G] fp64,
 * ancestors [B] int32.  Device memory, asynchronous on `stream`, library-owned
 * workspace (as specdec_verify).
 * Errors: SPECDEC_EINVAL for B not a multiple of N, N outside [1, 4096],
 * ess_threshold negative or not finite, and the argument errors of
 * specdec_verify.  A particle with an invalid input gets tokens -1 and log
 * weight -inf (weight 0) and sets the device error word; a group whose
 * particles are all invalid gets ess 0 and ancestors -1. */
specdec_status specdec_smc_step(const void *target_logits, const void *draft_logits,
                                const int32_t *draft_tokens, const float *u_bonus,
                                const float *temperature, const double *log_weights_in,
                                const float *u_resample, double ess_threshold, int B, int N,
                                int K, int V, specdec_dtype dtype, int32_t *out_tokens,
                                double *log_weights_out, double *ess, int32_t *ancestors,
                                double *log_weight_increment, void *stream);

/* Top-k candidates excluding one token (the LogitSpec page "LogitSpec:
 * Accelerating Retrieval-based Speculative Decoding via Next Next Token
 * Speculation", section 2, workflow step 2: once the next token x_{i+1} is
 * known, the top k entries of the last logit row other than x_{i+1} are the
 * candidates for the next-next token; the page uses k around 60).
 * For output row r (0 <= r < rows), the input row is
 *   logits + row_index[r] * row_stride   (row_index NULL: r * row_stride),
 * V elements of dtype, any element alignment.  exclude[r] is the token to
 * leave out (-1, or NULL for all rows, leaves none out).  Writes
 * out_idx[r, 0..k-1] (int32) the token ids of the k largest logits, larger
 * first and equal logits by ascending id, and, when out_val is not NULL,
 * out_val[r, 0..k-1] (fp32) their logits (exactly).  Fewer than k tokens: the
 * remaining entries are -1 / -inf.  A row holding a NaN is invalid: every
 * entry -1 / NaN and SPECDEC_ERR_LOGITS in the device error word.
 * Errors: SPECDEC_EINVAL for k outside [1, 256], row_stride < V, V < 1,
 * rows < 0, null or misaligned pointers.  rows == 0 is a no-op.  Device
 * memory, asynchronous on `stream`; no workspace. */
specdec_status specdec_topk_exclude(const void *logits, long long row_stride,
                                    const long long *row_index, int rows, int V,
                                    specdec_dtype dtype, const int32_t *exclude, int k,
                                    int32_t *out_idx, float *out_val, void *stream);

/* Chained two-stage verify (the HiSpec page "HiSpec: Hierarchical Speculative
 * Decoding for LLMs", section 2: a draft exit L_d, an intermediate verifier
 * exit L_i and the final layer L_f; the intermediate rejects early without
 * relaxing the final criterion; lossless by applying the speculative-decoding
 * argument at both stages, L_d -> L_i -> L_f).
 *   Stage 1 = specdec_verify with target intermediate_logits [B, K+1, V],
 *     draft_logits [B, K, V], draft_tokens, u_accept1 [B, K], u_resample1 [B]:
 *     n1 accepted tokens and one drawn token, m = n1 + 1 tokens s.
 *   Stage 2 verifies s against final_logits [B, K+1, V] (row j scores s_j)
 *     with the intermediate as proposal: s_j accepted iff
 *     u_accept2[b, j] * q_i,j(s_j) < p_f,j(s_j), u_accept2 [B, K+1]; at the
 *     first rejection n2 one token is drawn from max(0, p_f,n2 - q_i,n2)/Z
 *     with u_resample2[b] (the inverse-CDF rule of specdec_verify); when all m
 *     are accepted they are emitted and nothing is drawn (the final layer's row
 *     after them is not an input).
 * out_tokens [B, K+1]: the emitted tokens, then -1; out_num_emitted [B]: how
 * many (n2 + 1, or m), -1 for an invalid sequence (any row of the three
 * tensors, a draft token or the temperature, as in specdec_verify).
 * stage1_tokens [B, K+1] / stage1_num_accepted [B] (nullable) receive stage 1's
 * outputs.  K <= 31.  Device memory, asynchronous on `stream`, library-owned
 * workspace.  Two statistics sweeps: the intermediate and draft tensors for
 * stage 1, then the final layer's rows only for stage 2 (the intermediate
 * rows' statistics are kept from stage 1); the second sweep starts streaming
 * while stage 1's finish pass draws. */
specdec_status specdec_verify_chained(
    const void *final_logits, const void *intermediate_logits, const void *draft_logits,
    const int32_t *draft_tokens, const float *u_accept1, const float *u_resample1,
    const float *u_accept2, const float *u_resample2, const float *temperature, int B, int K,
    int V, specdec_dtype dtype, int32_t *out_tokens, int32_t *out_num_emitted,
    int32_t *stage1_tokens, int32_t *stage1_num_accepted, void *stream);

/* specdec_verify_chained with diagnostics of its second stage (dbg2 may be
 * NULL; every field nullable, device memory):
 *   row_max, row_sum [B, 2K+1]: entries 0..K are the final layer's rows
 *     (max_v z_v and sum_v exp((z_v - max)/T)); entries K+1..2K are untouched;
 *   p_x, q_x [B, K+1]: p_f,j(s_j) and q_i,j(s_j) for the positions j the
 *     second stage tests (others untouched);
 *   Z [B]: the mass sum_v max(0, p_f - q_i) of the second stage's draw
 *     (untouched when all tested tokens are accepted). */
specdec_status specdec_verify_chained_ex(
    const void *final_logits, const void *intermediate_logits, const void *draft_logits,
    const int32_t *draft_tokens, const float *u_accept1, const float *u_resample1,
    const float *u_accept2, const float *u_resample2, const float *temperature, int B, int K,
    int V, specdec_dtype dtype, int32_t *out_tokens, int32_t *out_num_emitted,
    int32_t *stage1_tokens, int32_t *stage1_num_accepted, const specdec_debug *dbg2,
    void *stream);

/* End-to-end variant: every pointer is HOST memory (pinned memory makes the
 * copies asynchronous).  Copies the inputs to library-owned device buffers,
 * runs the verify step on `stream`, copies the outputs back and synchronises
 * `stream` before returning. */
specdec_status specdec_verify_host(const void *target_logits, const void *draft_logits,
                                   const int32_t *draft_tokens, const float *u_accept,
                                   const float *u_resample, const float *temperature, int B,
                                   int K, int V, specdec_dtype dtype, int32_t *out_tokens,
                                   int32_t *out_num_accepted, void *stream);

/* Synchronise `stream`, then read and clear the current device's error word
 * (SPECDEC_ERR_* bits) into *flags.  Returns SPECDEC_EDEVICE when a bit was set. */
specdec_status specdec_device_errors(void *stream, uint32_t *flags);

/* The device error word as a status: synchronises the current device (all
 * streams), reads and clears its error word, and returns SPECDEC_EDEVICE when
 * any SPECDEC_ERR_* bit was set (specdec_device_errors gives the bits),
 * SPECDEC_OK otherwise, SPECDEC_ECUDA when the synchronisation failed. */
specdec_status specdec_get_error(void);

/* A short English description of a status (a static string; never NULL).
 * The same text as specdec_status_string. */
const char *specdec_error_string(specdec_status s);

/* Allocation-free verify (no counterpart on the pages: an interface addition).
 *
 * For callers that cannot allocate device memory -- for example a serving
 * engine that has handed nearly all of HBM to its own pools (KV cache) and
 * forbids allocations behind its back, or a latency-critical loop that cannot
 * afford cudaMalloc's device-wide synchronisation.  Same arguments and results
 * as specdec_verify, but the workspace is a fixed device array inside the
 * library (SPECDEC_STATIC_SCRATCH_BYTES, 4 MiB, held by every device that
 * loads the library until the process exits); the call itself never calls
 * cudaMalloc, cudaFree or any allocating routine.  The caller still provides
 * every input and output buffer.
 *   - Returns SPECDEC_ESIZE, launching nothing, when these sizes need more
 *     workspace than the array holds (compare specdec_workspace_bytes with
 *     SPECDEC_STATIC_SCRATCH_BYTES; B=64,K=5,V=128256 bf16 needs about
 *     0.4 MiB and fits up to B=837; K=8,V=151936 fp32 needs 2.3 MiB at B=256
 *     and fits up to B=449).
 *   - The first call on a device looks up the array's device address (once
 *     per device, with that device current).
 *   - All calls share the one array, which keeps the last call's contents:
 *     calls whose executions overlap on the GPU (on different streams, or
 *     from different host threads) race on it and must be serialised by the
 *     caller.  The kernels rewrite everything they read, so no clearing is
 *     needed between calls. */
#define SPECDEC_STATIC_SCRATCH_BYTES (4u << 20)
specdec_status specdec_verify_static(const void *target_logits, const void *draft_logits,
                                     const int32_t *draft_tokens, const float *u_accept,
                                     const float *u_resample, const float *temperature, int B,
                                     int K, int V, specdec_dtype dtype, int32_t *out_tokens,
                                     int32_t *out_num_accepted, void *stream);

/* Free the library-owned workspaces and staging buffers of every device. */
void specdec_release(void);

const char *specdec_status_string(specdec_status s);

/* Testing hook of the failure path (no counterpart on the pages).  Every
 * on-chip wait of the statistics sweep is bounded; when one runs out the
 * kernel sets SPECDEC_ERR_TIMEOUT, marks the statistics it could not finish as
 * incomplete and winds down, and the sequences depending on them get outputs
 * -1, so the device stays usable.  This hook makes that path testable without
 * a fault: wait_ns sets the bound of every wait in later launches (default
 * 2e9 ns), and skip_tile >= 0 makes the sweep's producer never issue the copy
 * of that tile (its index within one sweep launch), so the waits for it run
 * out.  specdec_test_set_wait_fault(-1, 2000000000) restores the defaults.
 * SPECDEC_EINVAL for skip_tile < -1 or wait_ns == 0.  Not thread-safe with
 * respect to calls in flight on other host threads. */
specdec_status specdec_test_set_wait_fault(long long skip_tile, unsigned long long wait_ns);

/* Testing hook of the statistics sweep's FMA-pipe exponential (no
 * counterpart on the pages): y[i] = 2^a[i] for n device floats, computed by
 * the same device function the sweep uses for part of its exponentials
 * (argument reduction to [-1/2, 1/2] and a degree-5 minimax polynomial; valid
 * for a <= 64, arguments below -125 give about 2^-125).  Asynchronous on
 * `stream`.  SPECDEC_EINVAL for n < 0 or null pointers with n > 0. */
specdec_status specdec_test_exp2(const float *a, float *y, int n, void *stream);

/* Kernel accounting, for benchmarks.  The library has specdec_kernel_count()
 * kernels; specdec_kernel_name(i) names kernel i.  specdec_launch_count(i)
 * counts its launches since the library was loaded.  Between
 * specdec_profile_begin(max) and specdec_profile_end, up to `max` launches per
 * kernel are bracketed with CUDA events on their stream; profile_end
 * synchronises those events and writes, per kernel, the summed device time in
 * milliseconds and the number of timed launches. */
int specdec_kernel_count(void);
const char *specdec_kernel_name(int i);
uint64_t specdec_launch_count(int i);
specdec_status specdec_profile_begin(int max_launches_per_kernel);
specdec_status specdec_profile_end(double *ms_per_kernel, int *launches_per_kernel, int n);

#ifdef __cplusplus
}
#endif
#endif /* SPECDEC_H */
