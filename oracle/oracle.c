/*
 * fp64 CPU oracle for the batched speculative-sampling verify step.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the plain, slow, obviously-correct
 * statement of what the verify step computes.  Only the test-suite, the smoke
 * check and the benchmark's CPU-baseline leg load it; the product path
 * (libspecdec.so and its Python binding) never does, and the two share no code.
 *
 * Method (Leviathan et al., as restated on the speculative decoding blog page
 * "Speculative Decoding ... Llama 70B x2.4", section "The mathematical
 * definition from Leviathan et al. (Google DeepMind, 2023)"):
 *   - the draft proposes K tokens x_0..x_{K-1}; the target scores them in one
 *     pass and yields K+1 rows of logits (the extra row is the "bonus" row, see
 *     the SMC-SD page "Faster LLM Inference via Sequential Monte Carlo",
 *     section 2 "Core mechanism", scoring step, and "Key differences", the
 *     N x (K+1) vectorised verify);
 *   - each draft token x is accepted with probability
 *     alpha(x) = min(1, p_target(x) / p_draft(x));
 *   - the first rejected position stops the walk and a token is drawn from the
 *     corrected distribution p'(x) = max(0, p_target(x) - p_draft(x)) / Z;
 *   - if all K are accepted a bonus token is drawn from the target's row K.
 * Temperature (the blog's vLLM example, temperature=0.7, and trade-off 4
 * "high temperature ruins the gain") enters as softmax(z / T) on BOTH models.
 *
 * Readings taken where the pages are silent:
 *   - accept iff  u * q(x) < p(x)  with u in [0,1)   (same as u < p/q; q = 0 and
 *     p > 0 accepts; p = q = 0 rejects);
 *   - row i of the target pairs with row i of the draft and token x_i; target
 *     row K is the bonus row;
 *   - inverse CDF: y = smallest j with  sum_{v<=j} r(v) > u * Z, sums taken in
 *     ascending token order; if no j qualifies (rounding), y = largest j with
 *     r(j) > 0;
 *   - Z = 0 after a rejection (possible only through rounding): draw from p_n
 *     instead, and report a zero sampling margin;
 *   - outputs: n accepted tokens, then the drawn token at position n, then -1;
 *   - a sequence with an invalid input (draft token outside [0,V), temperature
 *     not finite and > 0, a logit row containing NaN or +Inf, or a row that is
 *     entirely -Inf) yields n = -1 and all tokens -1.
 *
 * All arithmetic is IEEE fp64, round to nearest, sums in index order.  Inputs
 * are bf16 bit patterns or fp32 values and are widened exactly.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_F32 0
#define ORACLE_BF16 1

typedef struct {
  double *row_max;       /* [B, 2K+1]: target rows 0..K then draft rows 0..K-1 */
  double *row_sum;       /* [B, 2K+1]: sum_v exp((z_v - max) / T)              */
  double *p_x;           /* [B, K]   : p_i(x_i) (positions reached only; else NaN) */
  double *q_x;           /* [B, K]   : q_i(x_i)                                */
  double *accept_prob;   /* [B, K]   : sum_v min(p_i(v), q_i(v)) for every i   */
  double *Z;             /* [B]      : mass of the distribution drawn from     */
  double *margin_accept; /* [B]      : min |u_i - p_i/q_i| over tested i with p<q */
  double *margin_sample; /* [B]      : min(t - C_{y-1}, C_y - t) / Z           */
} oracle_diag;

typedef struct {
  const void *target, *draft;
  int dtype;
  const int32_t *tokens;
  const float *u_accept, *u_resample, *temperature;
  int64_t B, V;
  int K;
  int32_t *out_tokens, *out_n;
  const oracle_diag *diag;
  int64_t b0, b1;
} job_t;

/* exact widening of one logit */
static double logit_at(const void *base, int dtype, int64_t idx) {
  if (dtype == ORACLE_BF16) {
    uint32_t bits = (uint32_t)((const uint16_t *)base)[idx] << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
  }
  return (double)((const float *)base)[idx];
}

/* Row maximum.  Returns 0 for an invalid row (NaN, +Inf, or all -Inf). */
static int row_max(const void *base, int dtype, int64_t off, int64_t V, double *M) {
  double m = -INFINITY;
  for (int64_t v = 0; v < V; ++v) {
    double z = logit_at(base, dtype, off + v);
    if (isnan(z) || z == INFINITY) return 0;
    if (z > m) m = z;
  }
  *M = m;
  return m != -INFINITY;
}

/* Softmax normaliser S = sum_v exp((z_v - M) / T), summed in index order. */
static double row_sum(const void *base, int dtype, int64_t off, int64_t V, double M, double T) {
  double s = 0.0;
  for (int64_t v = 0; v < V; ++v) s += exp((logit_at(base, dtype, off + v) - M) / T);
  return s;
}

static double prob(const void *base, int dtype, int64_t off, int64_t v, double M, double S,
                   double T) {
  return exp((logit_at(base, dtype, off + v) - M) / T) / S;
}

static void set_nan(double *a, int64_t i) {
  if (a) a[i] = NAN;
}

static void verify_one(const job_t *j, int64_t b) {
  const int K = j->K;
  const int64_t V = j->V;
  const int R = 2 * K + 1;
  const oracle_diag *d = j->diag;
  int32_t *out = j->out_tokens + b * (K + 1);
  const double T = (double)j->temperature[b];
  int ok = isfinite(T) && T > 0.0;

  /* row offsets in elements: target (b,i) and draft (b,i) */
  double M[2 * 64 + 1], S[2 * 64 + 1];
  int64_t toff[65], doff[64];
  for (int i = 0; i <= K; ++i) toff[i] = (b * (K + 1) + i) * V;
  for (int i = 0; i < K; ++i) doff[i] = (b * K + i) * V;

  for (int r = 0; r < R; ++r) {
    int valid = (r <= K) ? row_max(j->target, j->dtype, toff[r], V, &M[r])
                         : row_max(j->draft, j->dtype, doff[r - K - 1], V, &M[r]);
    if (!valid) ok = 0;
    S[r] = NAN;
  }
  for (int i = 0; i < K; ++i) {
    int32_t x = j->tokens[b * K + i];
    if (x < 0 || (int64_t)x >= V) ok = 0;
  }
  if (d) {
    for (int r = 0; r < R; ++r) {
      set_nan(d->row_max, b * R + r);
      set_nan(d->row_sum, b * R + r);
    }
    for (int i = 0; i < K; ++i) {
      set_nan(d->p_x, b * K + i);
      set_nan(d->q_x, b * K + i);
      set_nan(d->accept_prob, b * K + i);
    }
    set_nan(d->Z, b);
    set_nan(d->margin_accept, b);
    set_nan(d->margin_sample, b);
  }
  if (!ok) {
    for (int i = 0; i <= K; ++i) out[i] = -1;
    j->out_n[b] = -1;
    return;
  }

  /* Softmax normaliser of every row (target rows 0..K, draft rows 0..K-1). */
  for (int r = 0; r < R; ++r)
    S[r] = (r <= K) ? row_sum(j->target, j->dtype, toff[r], V, M[r], T)
                    : row_sum(j->draft, j->dtype, doff[r - K - 1], V, M[r], T);

  /* Diagnostic only: per-position acceptance probability sum_v min(p, q). */
  if (d && d->accept_prob) {
    for (int i = 0; i < K; ++i) {
      double a = 0.0;
      for (int64_t v = 0; v < V; ++v) {
        double p = prob(j->target, j->dtype, toff[i], v, M[i], S[i], T);
        double q = prob(j->draft, j->dtype, doff[i], v, M[K + 1 + i], S[K + 1 + i], T);
        a += (p < q) ? p : q;
      }
      d->accept_prob[b * K + i] = a;
    }
  }

  /* Walk the K positions in order; stop at the first rejection. */
  int n = K;
  double margin_acc = INFINITY;
  for (int i = 0; i < K; ++i) {
    const int32_t x = j->tokens[b * K + i];
    const double p = prob(j->target, j->dtype, toff[i], x, M[i], S[i], T);
    const double q = prob(j->draft, j->dtype, doff[i], x, M[K + 1 + i], S[K + 1 + i], T);
    const double u = (double)j->u_accept[b * K + i];
    if (d && d->p_x) d->p_x[b * K + i] = p;
    if (d && d->q_x) d->q_x[b * K + i] = q;
    if (p < q) { /* alpha = p/q < 1: the test is not a certainty */
      double m = fabs(u - p / q);
      if (m < margin_acc) margin_acc = m;
    }
    if (!(u * q < p)) { /* rejected: u >= min(1, p/q) */
      n = i;
      break;
    }
    out[i] = x;
  }

  /* The distribution to draw from: residual max(0, p_n - q_n) after a
   * rejection, the target's row K (bonus) otherwise. */
  double *r = (double *)malloc((size_t)V * sizeof(double));
  double Z = 0.0;
  int zero_residual = 0;
  if (n == K) {
    for (int64_t v = 0; v < V; ++v) r[v] = prob(j->target, j->dtype, toff[K], v, M[K], S[K], T);
  } else {
    for (int64_t v = 0; v < V; ++v) {
      double p = prob(j->target, j->dtype, toff[n], v, M[n], S[n], T);
      double q = prob(j->draft, j->dtype, doff[n], v, M[K + 1 + n], S[K + 1 + n], T);
      r[v] = (p - q > 0.0) ? p - q : 0.0;
    }
  }
  for (int64_t v = 0; v < V; ++v) Z += r[v];
  if (Z == 0.0) { /* only reachable through rounding: draw from p_n */
    zero_residual = 1;
    for (int64_t v = 0; v < V; ++v) r[v] = prob(j->target, j->dtype, toff[n], v, M[n], S[n], T);
    Z = 0.0;
    for (int64_t v = 0; v < V; ++v) Z += r[v];
  }

  /* Inverse CDF with one uniform. */
  const double t = (double)j->u_resample[b] * Z;
  double C = 0.0, Cprev = 0.0;
  int64_t y = -1;
  for (int64_t v = 0; v < V; ++v) {
    Cprev = C;
    C += r[v];
    if (C > t) {
      y = v;
      break;
    }
  }
  double margin_smp;
  if (y < 0) { /* rounding left t at or above the last partial sum */
    for (int64_t v = V - 1; v >= 0; --v)
      if (r[v] > 0.0) {
        y = v;
        break;
      }
    margin_smp = 0.0;
  } else {
    double lo = t - Cprev, hi = C - t;
    margin_smp = ((lo < hi) ? lo : hi) / Z;
  }
  if (zero_residual) margin_smp = 0.0;
  free(r);

  out[n] = (int32_t)y;
  for (int i = n + 1; i <= K; ++i) out[i] = -1;
  j->out_n[b] = n;
  if (d) {
    for (int r2 = 0; r2 < R; ++r2) {
      if (d->row_max) d->row_max[b * R + r2] = M[r2];
      if (d->row_sum) d->row_sum[b * R + r2] = S[r2];
    }
    if (d->Z) d->Z[b] = Z;
    if (d->margin_accept) d->margin_accept[b] = margin_acc;
    if (d->margin_sample) d->margin_sample[b] = margin_smp;
  }
}

static void *run_job(void *arg) {
  const job_t *j = (const job_t *)arg;
  for (int64_t b = j->b0; b < j->b1; ++b) verify_one(j, b);
  return NULL;
}

/*
 * Verify B sequences.  All pointers are host memory owned by the caller.
 * target [B,K+1,V] and draft [B,K,V] are bf16 bits (dtype 1) or fp32 (dtype 0).
 * Returns 0, or -1 for a bad argument (nothing written).
 * nthreads <= 1 runs on the calling thread; otherwise sequences are split into
 * contiguous blocks over nthreads POSIX threads (results do not depend on it).
 */
int oracle_verify(const void *target, const void *draft, int dtype, const int32_t *tokens,
                  const float *u_accept, const float *u_resample, const float *temperature,
                  int64_t B, int K, int64_t V, int32_t *out_tokens, int32_t *out_n,
                  const oracle_diag *diag, int nthreads) {
  if (!target || !draft || !tokens || !u_accept || !u_resample || !temperature || !out_tokens ||
      !out_n)
    return -1;
  if (B < 0 || K < 1 || K > 32 || V < 1 || (dtype != ORACLE_F32 && dtype != ORACLE_BF16))
    return -1;
  job_t base = {target, draft, dtype, tokens, u_accept, u_resample, temperature,
                B, V, K, out_tokens, out_n, diag, 0, B};
  if (nthreads <= 1 || B < 2) {
    run_job(&base);
    return 0;
  }
  if (nthreads > B) nthreads = (int)B;
  pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)nthreads);
  job_t *jobs = (job_t *)malloc(sizeof(job_t) * (size_t)nthreads);
  for (int t = 0; t < nthreads; ++t) {
    jobs[t] = base;
    jobs[t].b0 = B * t / nthreads;
    jobs[t].b1 = B * (t + 1) / nthreads;
    pthread_create(&th[t], NULL, run_job, &jobs[t]);
  }
  for (int t = 0; t < nthreads; ++t) pthread_join(th[t], NULL);
  free(th);
  free(jobs);
  return 0;
}
