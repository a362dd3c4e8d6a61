// libspecdec: the batched speculative-sampling verify step for B200 (sm_100a).
//
// What it computes is stated in include/specdec.h (accept with
// alpha(x) = min(1, p_target(x)/p_draft(x)), stop at the first rejection, draw
// from max(0, p - q)/Z or from the bonus row; speculative decoding blog
// "Speculative Decoding ... Llama 70B x2.4", section "The mathematical definition
// from Leviathan et al.").  This file is the B200 implementation:
//
//   k_row_stats     one pass over every logit row (B*(2K+1) rows of V): a
//                   producer thread streams 16 KB tiles (4 KB for batches of
//                   a few sequences) with TMA bulk copies into a 3-stage
//                   shared-memory ring (full/empty mbarriers, every wait
//                   bounded); 8 consumer warps fold them into split-V softmax
//                   statistics (row max m, sum of 2^((z-m)*c)) and write, per
//                   row segment, one partial per warp (or one per CTA where
//                   many CTAs share a row).  It streams the whole input once
//                   and is the HBM-bound kernel.
//   k_finish        per sequence, on several CTAs: combines the partials of the
//                   2K+1 rows in fp64, gathers p_i(x_i), q_i(x_i), tests
//                   u*q < p on K lanes (__ballot_sync/__ffs), writes the
//                   accepted prefix; sums r(v) = max(0, p - q) (or the bonus
//                   row) over its chunks of the drawn row pair; the last CTA of
//                   the sequence (atomic ticket, no waiting) finds the chunk
//                   holding u*Z from the fp64 chunk prefix and rescans it.
//   k_smc_resample  SMC-SD: log-weights, effective sample size and systematic
//                   resampling per group of particles.
//   k_topk_exclude  top-k token ids of a row leaving one token out.
// Kernels are launched with programmatic dependent launch: each signals its
// dependents early and waits for its predecessor
// (cudaGridDependencySynchronize) only where it first needs its results; the
// call's first kernel waits before it reads anything (the statistics sweep
// only requests its first tiles into L2 before that; the chained verify's
// second sweep, which reads only inputs no kernel of the call writes, streams
// at once and waits at its end).
//
// Arithmetic: logits are widened exactly to fp32.  Exponentials are
// 2^((z - m) * c) with c = log2(e)/T carried as an fp32 pair (hi + lo, with
// hi = c rounded toward zero) so the rounding of c does not bias the
// temperature, and 2^x from the ex2.approx.ftz.f32 PTX instruction.  Per-thread
// sums are fp32; every combine across threads, CTAs and V-splits, the
// acceptance test and the inverse-CDF prefix are fp64.  No float atomics, fixed
// reduction orders: the result is bit-reproducible.
//
// No tensor cores: nothing here is a dense contraction.

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include <cfloat>
#include <climits>
#include <atomic>
#include <cstring>
#include <map>
#include <mutex>
#include <string>
#include <unordered_map>
#include <vector>

#include "specdec.h"

namespace {

constexpr int NT = 256;               // threads per CTA of the streaming kernels
constexpr int NWARP = NT / 32;
constexpr double kLog2e = 1.4426950408889634073599246810019;  // log2(e)
constexpr unsigned FULL = 0xffffffffu;

// ---------------------------------------------------------------------------
// workspace records
// ---------------------------------------------------------------------------
struct __align__(16) Partial {  // one (row, V-split): max and sum of 2^((z-m)c)
  double s;
  float m;
  uint32_t pad;
};
struct __align__(16) SeqInfo {  // a sequence decided by an earlier pass (early exit)
  double St, Sd;                // row sums (at the row max) of the drawn pair
  float Mt, Md;                 // row maxima of the drawn pair
};
struct __align__(16) ResPartial {  // one (sequence, V-chunk) of the drawn row(s)
  double R;                        // sum of St * max(0, p - q)  (or of 2^((z-m)c), bonus)
  double pad;
};

__device__ unsigned int g_error_flags;  // per device; read/cleared by the host

// ---------------------------------------------------------------------------
// scalar helpers
// ---------------------------------------------------------------------------
struct Scale {
  float hi, lo;  // log2(e)/T = hi + lo, hi rounded toward zero, lo > 0
};

__device__ __forceinline__ Scale make_scale(double c64) {
  Scale c;
  c.hi = __double2float_rz(c64);
  float lo = (float)(c64 - (double)c.hi);
  // lo > 0 keeps (-inf)*lo == -inf, so masked / -inf logits give exactly 0
  c.lo = (lo > 1e-30f) ? lo : 1e-30f;
  return c;
}

// (d * c) for d = z - m <= 0 with c split in two fp32 parts
__device__ __forceinline__ float scaled(float d, Scale c) {
  return __fmaf_rn(d, c.hi, __fmul_rn(d, c.lo));
}

__device__ __forceinline__ float ex2(float a) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(a));
  return y;
}

__device__ __forceinline__ float fmax_nan(float a, float b) {
  float y;
  asm("max.NaN.f32 %0, %1, %2;" : "=f"(y) : "f"(a), "f"(b));
  return y;
}

template <typename T>
struct Dt;
template <>
struct Dt<__nv_bfloat16> {
  static constexpr int VEC = 8;  // elements per 16-byte vector
  static __device__ __forceinline__ float load(const __nv_bfloat16 *p) {
    return __uint_as_float((uint32_t)__ldg(reinterpret_cast<const unsigned short *>(p)) << 16);
  }
  static __device__ __forceinline__ uint4 neg_inf() {
    return make_uint4(0xFF80FF80u, 0xFF80FF80u, 0xFF80FF80u, 0xFF80FF80u);
  }
  // unpack a 16-byte vector into 8 fp32 values (exact)
  static __device__ __forceinline__ void unpack(const uint4 &v, float (&x)[8]) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      x[2 * k] = __uint_as_float(w[k] << 16);
      x[2 * k + 1] = __uint_as_float(w[k] & 0xFFFF0000u);
    }
  }
};
template <>
struct Dt<float> {
  static constexpr int VEC = 4;
  static __device__ __forceinline__ float load(const float *p) { return __ldg(p); }
  static __device__ __forceinline__ uint4 neg_inf() {
    return make_uint4(0xFF800000u, 0xFF800000u, 0xFF800000u, 0xFF800000u);
  }
  static __device__ __forceinline__ void unpack(const uint4 &v, float (&x)[4]) {
    x[0] = __uint_as_float(v.x);
    x[1] = __uint_as_float(v.y);
    x[2] = __uint_as_float(v.z);
    x[3] = __uint_as_float(v.w);
  }
};

// elements before the first 16-byte boundary of a row (row start is
// element-aligned); capped at V
template <typename T>
__device__ __forceinline__ int row_head(const T *p, long long V) {
  const unsigned mis = (unsigned)(reinterpret_cast<uintptr_t>(p) & 15u);
  long long h = (long long)(((16u - mis) & 15u) / sizeof(T));
  return (int)(h < V ? h : V);
}

__device__ __forceinline__ double warp_sum(double v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(FULL, v, o);
  return v;
}
__device__ __forceinline__ float warp_max_nan(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v = fmax_nan(v, __shfl_xor_sync(FULL, v, o));
  return v;
}
// reductions within each 16-lane half of a warp (all 32 lanes call them)
__device__ __forceinline__ double half_sum(double v) {
#pragma unroll
  for (int o = 8; o; o >>= 1) v += __shfl_xor_sync(FULL, v, o);
  return v;
}
__device__ __forceinline__ float half_max_nan(float v) {
#pragma unroll
  for (int o = 8; o; o >>= 1) v = fmax_nan(v, __shfl_xor_sync(FULL, v, o));
  return v;
}

// ---------------------------------------------------------------------------
// kernel 1: softmax statistics of every row
// ---------------------------------------------------------------------------
// A sweep reads the rows of its window (every row of the batch, or some
// positions of it), in sequence order, cut into tiles of CW*32*U 16-byte
// vectors (16 KB for U = 4, 4 KB for U = 1);
// CTA g of a grid of G owns the contiguous tile range [g*T/G, (g+1)*T/G)
// (with 4 KB tiles G is, where rows have 3 tiles or more, a multiple of the
// rows, so each range lies in one row: see sweep_partition).
//
// Warp specialisation: one producer warp streams tiles with cp.async.bulk
// (the TMA bulk-copy engine; each CTA copies only into its own shared memory)
// into an NSTAGE-deep ring in shared memory, tracked by "full" / "empty"
// mbarriers; CW consumer warps take a tile out of the ring (one 16-byte shared
// load per vector), release the slot, and fold it into a per-thread (max, sum)
// in registers.  At the end of each row segment (the CTA's tiles of one row)
// the warps' statistics are combined into one partial per CTA.  Per element
// the consumers spend one exact bf16->fp32 unpack, one FMNMX for the tile max,
// three packed fp32x2 operations at half an issue slot each, one exponential
// (MUFU ex2, or for SPECDEC_EXP_FMA_PAIRS pairs per vector the FMA-pipe
// polynomial) and half a packed add.  Every wait is bounded: a wait that runs
// out sets SPECDEC_ERR_TIMEOUT in the device error word, the CTA's partials
// from then on are marked incomplete, and the kernel winds down (the producer
// first waits, again bounded, for the copies it has in flight).

#ifndef SPECDEC_SWEEP_WARPS
#define SPECDEC_SWEEP_WARPS 8
#endif
#ifndef SPECDEC_SWEEP_CTAS_PER_SM
#define SPECDEC_SWEEP_CTAS_PER_SM 3
#endif
// Registers per thread of the sweep (0: the compiler's choice under the
// launch bound of kStatsCtasPerSm CTAs per SM).
#ifndef SPECDEC_SWEEP_MAXNREG
#define SPECDEC_SWEEP_MAXNREG 0
#endif
constexpr int CW = SPECDEC_SWEEP_WARPS;  // consumer warps of a sweep CTA
constexpr int NTC = CW * 32;        // consumer threads
constexpr int NTS = NTC + 32;       // + one producer warp
constexpr int NSTAGE = 3;           // depth of the shared-memory ring
constexpr unsigned long long kWaitNs = 2000000000ull;  // a wait gives up after 2 s by default
constexpr unsigned kSuspendNs = 20000;  // longest sleep of one try_wait round
constexpr int kStatsCtasPerSm = SPECDEC_SWEEP_CTAS_PER_SM;  // sweep CTAs per SM the grid is sized for
// tiles at the start of each sweep CTA's range prefetched into L2 before the
// CTA waits for the previous kernel on the stream
#ifndef SPECDEC_SWEEP_PREFETCH_TILES
#define SPECDEC_SWEEP_PREFETCH_TILES 1
#endif
constexpr int kFinishUW = 4;        // vectors per lane in a k_finish chunk
constexpr int kFinishThreads = 256;   // threads of a k_finish CTA
constexpr int kFinishCtasPerSm = 4;   // k_finish grids fit one wave of this many CTAs per SM
constexpr int kFinishMaxNreg = 64;    // k_finish registers per thread (launch bound below)
// A sweep combines its warps' partials per CTA when a row can meet more than
// this many of its CTAs.
#ifndef SPECDEC_CTA_COMBINE_SLOTS
#define SPECDEC_CTA_COMBINE_SLOTS 4
#endif
constexpr int kCtaCombineSlots = SPECDEC_CTA_COMBINE_SLOTS;

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ void mbar_init(uint64_t *bar, unsigned count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}
__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void mbar_arrive_tx(uint64_t *bar, unsigned bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}
// One round of waiting for the phase of the given parity.  The suspend-time
// hint lets the hardware park the warp until the phase completes (or the hint
// runs out) instead of having it spin, so waiting warps take no issue slots
// from the warps that are folding.
__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, unsigned parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(kSuspendNs)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
// bounded wait for the phase of the given parity; false when it ran out after
// limit_ns (the bound is wall-clock time, so it does not depend on how long a
// round sleeps)
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, unsigned parity,
                                          unsigned long long limit_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = global_ns();
  do {
    if (mbar_try_wait(bar, parity)) return true;
  } while (global_ns() - t0 < limit_ns);
  atomicOr(&g_error_flags, SPECDEC_ERR_TIMEOUT);
  return false;
}
// barrier of the consumer warps of a sweep CTA only (the producer warp is not
// part of it)
__device__ __forceinline__ void consumer_sync() {
  asm volatile("bar.sync 1, %0;" ::"r"(NTC) : "memory");
}
// hint: bring a global range into L2 (16-byte aligned address, size a
// multiple of 16); reads nothing into the SM and completes on its own
__device__ __forceinline__ void bulk_prefetch_l2(const void *src, unsigned bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}
// global -> shared bulk copy completing on an mbarrier (16-byte aligned
// addresses, size a multiple of 16)
__device__ __forceinline__ void bulk_load(void *dst, const void *src, unsigned bytes,
                                          uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
      ::"r"(smem_u32(dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}
// pairs (x0, x1) of the 8 (bf16) or 4 (fp32) values of a 16-byte vector
template <typename T>
struct Pairs;
template <>
struct Pairs<__nv_bfloat16> {
  static constexpr int N = 4;
  static __device__ __forceinline__ float2 get(const uint4 &v, int q) {
    const uint32_t w = q == 0 ? v.x : q == 1 ? v.y : q == 2 ? v.z : v.w;
    return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
  }
};
template <>
struct Pairs<float> {
  static constexpr int N = 2;
  static __device__ __forceinline__ float2 get(const uint4 &v, int q) {
    return q == 0 ? make_float2(__uint_as_float(v.x), __uint_as_float(v.y))
                  : make_float2(__uint_as_float(v.z), __uint_as_float(v.w));
  }
};

// 2^a for a pair of arguments on the FMA pipe instead of the MUFU unit: the
// sweep evaluates part of its exponentials this way so that the two pipes
// share the work.  Method (the standard software exponential): split
// a = n + f with n = round(a) (adding 1.5 * 2^23 rounds to an integer in the
// low mantissa bits; n and f = a - n are exact) and f in [-1/2, 1/2]; 2^f by a
// degree-5 polynomial whose coefficients minimise the maximum relative error
// on [-1/2, 1/2] (Remez exchange, fitted in fp64 and rounded to fp32: 7.5e-8
// relative error in exact arithmetic, 2.2e-7 = 3.6 ulp including the fp32
// Horner steps, against 2 ulp for ex2.approx); then 2^n is applied by adding
// n to the exponent field.  Arguments below -125 are clamped there (so every
// result is a normal number): such a term, about 2^-125 instead of less, is far
// below the resolution of the sums it enters, which are at least 1.  Valid for
// a <= 64.
constexpr float kExp2C0 = 1.0000001192092896f, kExp2C1 = 0.6931469440460205f,
                kExp2C2 = 0.24022120237350464f, kExp2C3 = 0.05550713092088699f,
                kExp2C4 = 0.009675540961325169f, kExp2C5 = 0.0013276472454890609f;
__device__ __forceinline__ float2 exp2_fma2(float2 a) {
  constexpr float kRound = 12582912.0f;  // 1.5 * 2^23
  a.x = fmaxf(a.x, -125.0f);
  a.y = fmaxf(a.y, -125.0f);
  const float2 t = __fadd2_rn(a, make_float2(kRound, kRound));
  const float2 n = __fadd2_rn(t, make_float2(-kRound, -kRound));
  const float2 f = __ffma2_rn(n, make_float2(-1.0f, -1.0f), a);
  float2 p = __ffma2_rn(make_float2(kExp2C5, kExp2C5), f, make_float2(kExp2C4, kExp2C4));
  p = __ffma2_rn(p, f, make_float2(kExp2C3, kExp2C3));
  p = __ffma2_rn(p, f, make_float2(kExp2C2, kExp2C2));
  p = __ffma2_rn(p, f, make_float2(kExp2C1, kExp2C1));
  p = __ffma2_rn(p, f, make_float2(kExp2C0, kExp2C0));
  // (bits of t) << 23 is n << 23: the rounding constant's own bits shift out
  return make_float2(__int_as_float(__float_as_int(p.x) + (__float_as_int(t.x) << 23)),
                     __int_as_float(__float_as_int(p.y) + (__float_as_int(t.y) << 23)));
}
// pairs of each 16-byte vector whose exponentials the sweep takes on the FMA
// pipe (the rest on MUFU)
#ifndef SPECDEC_EXP_FMA_PAIRS
#define SPECDEC_EXP_FMA_PAIRS 0
#endif

__device__ __forceinline__ float fmax3_nan(float a, float b, float c) {
  float y;
  asm("max.NaN.f32 %0, %1, %2, %3;" : "=f"(y) : "f"(a), "f"(b), "f"(c));
  return y;
}

// Per-thread statistics of a row segment, kept against a lazy reference:
//   r    the exponent reference: acc.x + acc.y = sum 2^((z - r) c) so far;
//   mt   the true running max.
// r moves only when the running max passes it by more than thr = 64/c (a
// term would pass 2^64); with logits this happens once at the start of a row
// and almost never again, so warps do not diverge on running-max updates.
// Terms stay below 2^64 (far inside fp32), and fp32 precision is scale free,
// so nothing is lost.  At the end of the segment the sum is moved to the true
// max once.  The sum is kept as a packed fp32 pair (one FADD2 per vector).
// r: the reference the sum is kept against; mt: the running max; nr = -r
// (with r = -inf clamped to -FLT_MAX, so -inf values give exactly 0 instead of
// NaN while nothing finite has been seen); rt = r + thr, the max beyond which
// the reference moves.  nr and rt only change when r does.
struct RunStat {
  float r, mt, nr, rt;
  float2 acc;
};
__device__ __forceinline__ void runstat_init(RunStat &q) {
  q.r = -INFINITY;
  q.mt = -INFINITY;
  q.nr = FLT_MAX;
  q.rt = -INFINITY;
  q.acc = make_float2(0.0f, 0.0f);
}
// rare path: the running max passed the reference (also the first finite value)
__device__ __forceinline__ void runstat_rebase(RunStat &q, Scale c, float thr) {
  if (q.r != -INFINITY) {
    const float f = ex2(scaled(q.r - q.mt, c));
    q.acc = __fmul2_rn(q.acc, make_float2(f, f));
  }
  q.r = q.mt;
  q.nr = -fmaxf(q.mt, -FLT_MAX);
  q.rt = q.mt + thr;
}
// sum expressed against the true max (call once, at the end of a segment)
__device__ __forceinline__ float runstat_sum_at_max(const RunStat &q, Scale c) {
  const float s = q.acc.x + q.acc.y;
  if (q.r == q.mt || !(q.r > -INFINITY) || !isfinite(q.mt)) return s;
  return s * ex2(scaled(q.r - q.mt, c));
}

// Fold one 16-byte vector: the running max with three-input NaN-propagating
// FMNMX, then packed fp32x2 exponent arguments against r, MUFU ex2 and a
// pairwise packed sum.  Only the vector's 8 (bf16) or 4 (fp32) values are live.
template <typename T>
__device__ __forceinline__ void vec_fold(const uint4 &v, RunStat &q, Scale c, float thr) {
  constexpr int N = Pairs<T>::N;
  float2 x[N];
#pragma unroll
  for (int k = 0; k < N; ++k) x[k] = Pairs<T>::get(v, k);
  if (N == 4) {
    const float a = fmax3_nan(x[0].x, x[0].y, x[1].x);
    const float b = fmax3_nan(x[1].y, x[2].x, x[2].y);
    const float d = fmax3_nan(x[N - 1].x, x[N - 1].y, q.mt);
    q.mt = fmax3_nan(a, b, d);
  } else {
    q.mt = fmax3_nan(fmax3_nan(x[0].x, x[0].y, x[N - 1].x), x[N - 1].y, q.mt);
  }
  if (q.mt > q.rt) runstat_rebase(q, c, thr);
  const float2 nr = make_float2(q.nr, q.nr), hi = make_float2(c.hi, c.hi),
               lo = make_float2(c.lo, c.lo);
  float2 e[N];
#pragma unroll
  for (int k = 0; k < N; ++k) {
    const float2 d = __fadd2_rn(x[k], nr);
    const float2 a = __ffma2_rn(d, hi, __fmul2_rn(d, lo));
    if (k < SPECDEC_EXP_FMA_PAIRS)
      e[k] = exp2_fma2(a);
    else
      e[k] = make_float2(ex2(a.x), ex2(a.y));
  }
#pragma unroll
  for (int w = 1; w < N; w *= 2)
#pragma unroll
    for (int k = 0; k + w < N; k += 2 * w) e[k] = __fadd2_rn(e[k], e[k + w]);
  q.acc = __fadd2_rn(q.acc, e[0]);
}

// the same for one scalar logit (row heads and tails)
__device__ __forceinline__ void elem_fold(float x, RunStat &q, Scale c, float thr) {
  q.mt = fmax_nan(q.mt, x);
  if (q.mt > q.rt) runstat_rebase(q, c, thr);
  q.acc.x += ex2(scaled(x + q.nr, c));
}

// A sweep covers a window of draft positions [p0, p0 + np) (both the target
// and the draft row of each) and, when `bonus` is set, the target's row K.
// Within a sequence the window's rows are walked as target p0, draft p0,
// target p0+1, ..., then the bonus row: rps rows per sequence.  With `state`
// set, only the sequences still undecided (state[b] == kSeqActive) are read.
constexpr int kSeqActive = -2;
struct StatsGeom {
  int K;
  long long V;
  int tpr;          // tiles per row
  long long tiles;  // rows * tpr
  int slots;        // CTA slots per row (>= CTAs that can share one row)
  int p0, np, rps;  // the window: first position, positions, rows per sequence
  const int *state; // per-sequence decision state, or null (every sequence)
  int d_rows;       // rows per sequence of the draft tensor (K, or K+1 when it is an
                    // intermediate verifier's logits)
  int tonly;        // the window holds target rows p0 .. p0+np-1 only (rps = np)
  unsigned long long wait_ns;  // bound of every on-chip wait
  long long skip_tile;         // test hook: the producer never issues this tile's copy
                               // (-1: none), so a consumer wait runs out
  int nb;           // sequences of this sweep
  int pcw;          // partials per (row, CTA): CW (one per consumer warp, no CTA
                    // barrier) or 1 (the warps' partials combined per CTA, for rows
                    // shared by many CTAs, so that the finish pass reads fewer)
  int late_sync;    // (instantiations with LATE only) see k_row_stats
};
__device__ __forceinline__ bool seq_active(const StatsGeom &g, long long b) {
  return g.state == nullptr || __ldcg(g.state + b) == kSeqActive;
}

// CTA g of G owns tiles [g*T/G, (g+1)*T/G); the owner of tile t is then
// floor(((t+1)*G - 1) / T).  Both the statistics kernel and the combine in
// k_finish use these to name a row's partials: CTA slot = owner - first owner,
// and each of the CW consumer warps of a CTA writes its own partial.
__host__ __device__ __forceinline__ long long tile_begin(long long g, long long G, long long T) {
  return g * T / G;
}
__host__ __device__ __forceinline__ long long tile_owner(long long t, long long G, long long T) {
  const long long num = (t + 1) * G - 1;
  // (a 32-bit division where the operands fit: far cheaper than a 64-bit one)
  if (num < 4294967296LL && T < 4294967296LL) return (long long)((unsigned)num / (unsigned)T);
  return num / T;
}

// The current row of a CTA's tile walk.  Rows are numbered b*rps + w, w the
// row of the window (see StatsGeom); the cursor steps row by row without
// divisions.
template <typename T>
struct RowCursor {
  const T *p;
  const uint4 *pv;
  long long row, b, nvec;
  int w, ti, head;
  __device__ __forceinline__ void point(const T *target, const T *draft, const StatsGeom &g) {
    constexpr int VEC = Dt<T>::VEC;
    const int pos = g.tonly ? g.p0 + w : (w < 2 * g.np ? g.p0 + (w >> 1) : g.K);
    const bool is_draft = !g.tonly && w < 2 * g.np && (w & 1);
    p = is_draft ? draft + (b * g.d_rows + pos) * g.V : target + (b * (g.K + 1) + pos) * g.V;
    head = row_head(p, g.V);
    nvec = (g.V - head) / VEC;
    pv = reinterpret_cast<const uint4 *>(p + head);
  }
  __device__ __forceinline__ void start(const T *target, const T *draft, const StatsGeom &g,
                                        long long t) {
    row = t / g.tpr;
    ti = (int)(t - row * g.tpr);
    b = row / g.rps;
    w = (int)(row - b * g.rps);
    point(target, draft, g);
  }
  __device__ __forceinline__ void next_row(const T *target, const T *draft, const StatsGeom &g) {
    ++row;
    ti = 0;
    if (++w == g.rps) {
      w = 0;
      ++b;
    }
    point(target, draft, g);
  }
};

#if SPECDEC_SWEEP_MAXNREG > 0
#define SPECDEC_SWEEP_BOUNDS __maxnreg__(SPECDEC_SWEEP_MAXNREG)
#else
#define SPECDEC_SWEEP_BOUNDS __launch_bounds__(NTS, kStatsCtasPerSm)
#endif

// The partials of one row segment: one per consumer warp (pcw = CW), or the
// CW warps' (max, sum) pairs combined in warp order with fp64 rescales (pcw =
// 1); pad = 1 marks a partial left incomplete because a wait of this CTA ran
// out.
// Programmatic dependent launch: the grid may be placed while the kernel
// before it on the stream drains; every thread waits for that kernel
// (cudaGridDependencySynchronize) after the shared-memory setup, before it
// reads an input or touches the workspace, and only then lets the dependent
// finish pass launch.
// With LATE and g.late_sync set: the previous kernel on the stream writes
// nothing this sweep reads or writes but the finish pass's tickets (a later
// stage of the same call): stream at once, and let one thread wait for that
// kernel (then zero the tickets) at the end, so that this grid still
// completes after it.  (Both sweeps of a call that has such a stage use the
// LATE instantiation: the second stage's CTAs were measured to overlap the
// first stage's finish only when they run the same kernel as its sweep.)
// PLAIN: the sweep of the plain verify (every sequence, target and draft rows
// of every position, a draft tensor of K rows per sequence), compiled with
// those choices fixed: less code, and measured 0.2 us faster per call.
template <typename T, int U, bool LATE = false, bool PLAIN = false>
__global__ void SPECDEC_SWEEP_BOUNDS k_row_stats(const T *__restrict__ target,
                                                 const T *__restrict__ draft,
                                                 const float *__restrict__ temperature,
                                                 StatsGeom g, Partial *__restrict__ part,
                                                 unsigned *__restrict__ tickets, int B) {
  if (PLAIN) {  // (the launch picks PLAIN only for these values)
    g.state = nullptr;
    g.tonly = 0;
    g.d_rows = g.K;
  }
  constexpr int VEC = Dt<T>::VEC;
  constexpr long long TV = (long long)NTC * U;  // vectors per tile
  constexpr unsigned TILE_BYTES = (unsigned)TV * 16u;
  extern __shared__ __align__(128) unsigned char ring[];  // NSTAGE * TILE_BYTES
  __shared__ __align__(8) uint64_t full[NSTAGE], empty[NSTAGE];
  __shared__ int s_abort;
  __shared__ float s_wm[2][CW];   // per-warp partials of the last two row segments
  __shared__ double s_ws[2][CW];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long G = gridDim.x;
  const long long t0 = tile_begin(blockIdx.x, G, g.tiles);
  const long long t1 = tile_begin(blockIdx.x + 1, G, g.tiles);

  if (threadIdx.x == 0) {
    for (int i = 0; i < NSTAGE; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], CW);
    }
    s_abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  // Before waiting for the previous kernel: the first tiles of this CTA's
  // range are requested into L2.  A prefetch reads nothing into the CTA, and
  // L2 is coherent, so whatever that kernel still writes is what the copies
  // below see; when it is the previous call's finish pass, these bytes stream
  // while its draw runs.  (A sweep over the open sequences only reads a state
  // written by the previous kernel and prefetches nothing.)
  if (SPECDEC_SWEEP_PREFETCH_TILES > 0 && warp == CW && lane == 0 && g.state == nullptr &&
      t0 < t1) {
    RowCursor<T> pc;
    pc.start(target, draft, g, t0);
    long long t = t0;
    const long long tend = t0 + SPECDEC_SWEEP_PREFETCH_TILES < t1 ? t0 + SPECDEC_SWEEP_PREFETCH_TILES : t1;
    while (t < tend) {
      const long long row = t / g.tpr;
      if (row != pc.row) pc.next_row(target, draft, g);
      const long long v0 = (t - row * g.tpr) * TV;
      const long long v1 = (v0 + TV < pc.nvec) ? v0 + TV : pc.nvec;
      if (v1 > v0) bulk_prefetch_l2(pc.pv + v0, (unsigned)(v1 - v0) * 16u);
      ++t;
    }
  }
  __syncthreads();
  const bool late = LATE && g.late_sync;
  if (!late) cudaGridDependencySynchronize();
  // the dependent finish pass may be placed now; it reads this kernel's
  // results only after its own cudaGridDependencySynchronize
  cudaTriggerProgrammaticLaunchCompletion();
  // the arrival tickets of the finish pass start at 0
  if (blockIdx.x == 0 && !late)
    for (int i = threadIdx.x; i < g.nb; i += blockDim.x) tickets[i] = 0u;
  auto late_end = [&]() {
    if (late && blockIdx.x == 0 && threadIdx.x == 0) {
      cudaGridDependencySynchronize();
      for (int i = 0; i < g.nb; ++i) tickets[i] = 0u;
    }
  };
  if (t0 >= t1) {
    late_end();
    return;
  }

  // The CTA's tiles [t0, t1) are walked as row segments: the tiles of one row
  // that fall in the range.  Inside a segment the full tiles come first (no
  // per-element predicates), then at most one partial tile.
  const long long row_first = t0 / g.tpr, row_last = (t1 - 1) / g.tpr;

  if (warp == CW) {  // ---------------- producer warp ----------------
    if (lane != 0) return;
    unsigned ph = 0;  // phase parity of the current ring pass
    int st = 0;       // ring slot of the next copy
    // per slot: whether a copy was issued into it and the parity of its phase
    unsigned pend = 0, pend_ph = 0;
    RowCursor<T> rc;
    rc.start(target, draft, g, t0);
    for (long long row = row_first; row <= row_last; ++row) {
      if (row != row_first) rc.next_row(target, draft, g);
      if (!seq_active(g, rc.b)) continue;
      const int tb = (row == row_first) ? (int)(t0 - row * g.tpr) : 0;
      const int te = (row == row_last) ? (int)(t1 - row * g.tpr) : g.tpr;
      for (int ti = tb; ti < te; ++ti) {
        const long long v0 = (long long)ti * TV;
        const long long v1 = (v0 + TV < rc.nvec) ? v0 + TV : rc.nvec;
        if (v0 >= v1) break;  // the rest of the row is its scalar tail
        if (*(volatile int *)&s_abort || !mbar_wait(&empty[st], ph ^ 1u, g.wait_ns)) {
          atomicExch(&s_abort, 1);
          goto drain;
        }
        if (row * g.tpr + ti != g.skip_tile) {
          const unsigned bytes = (unsigned)(v1 - v0) * 16u;
          mbar_arrive_tx(&full[st], bytes);
          bulk_load(ring + (size_t)st * TILE_BYTES, rc.pv + v0, bytes, &full[st]);
          pend |= 1u << st;
          pend_ph = (pend_ph & ~(1u << st)) | (ph << st);
        }
        if (++st == NSTAGE) {
          st = 0;
          ph ^= 1u;
        }
      }
    }
  drain:
    // The CTA must not retire with copies in flight: wait (bounded) until the
    // last copy issued into each slot has landed.
    for (int k = 0; k < NSTAGE; ++k)
      if (pend & (1u << k)) mbar_wait(&full[k], (pend_ph >> k) & 1u, g.wait_ns);
    return;
  }

  // ---------------- consumer warps ----------------
  // Each warp folds its share of every tile.  At the end of a row segment the
  // warps' partials are combined through shared memory (consumer-only barrier)
  // and warp 0 writes one partial for the CTA.  After an abort the waits and
  // the arithmetic are skipped (every warp still walks the same tiles) and the
  // CTA's partials are marked incomplete.
  unsigned ph = 0;  // phase parity of the current ring pass
  int st = 0;       // ring slot of the next tile
  int seg = 0;      // row segments finished (selects the s_wm / s_ws buffer)
  RowCursor<T> rc;
  rc.start(target, draft, g, t0);
  float Tcur = __ldg(temperature + rc.b);
  Scale c = make_scale(kLog2e / (double)Tcur);
  float thr = 64.0f / c.hi;
  // temperature of the sequence after this one, fetched a row ahead
  float T_next = (rc.b + 1 < B) ? __ldg(temperature + rc.b + 1) : 1.0f;
  for (long long row = row_first; row <= row_last; ++row) {
    if (row != row_first) {
      const bool new_seq = (rc.w == g.rps - 1);
      rc.next_row(target, draft, g);
      if (new_seq) {
        Tcur = T_next;
        c = make_scale(kLog2e / (double)Tcur);
        thr = 64.0f / c.hi;
        T_next = (rc.b + 1 < B) ? __ldg(temperature + rc.b + 1) : 1.0f;
      }
    }
    if (!seq_active(g, rc.b)) continue;
    const int tb = (row == row_first) ? (int)(t0 - row * g.tpr) : 0;
    const int te = (row == row_last) ? (int)(t1 - row * g.tpr) : g.tpr;
    const long long full_tiles = rc.nvec / TV;  // tiles with all TV vectors
    const int tf = (int)((long long)te < full_tiles ? te : full_tiles);
    RunStat q;
    runstat_init(q);
    // full tiles
    for (int ti = tb; ti < tf; ++ti) {
      bool have = false;
      if (!*(volatile int *)&s_abort) {
        have = __all_sync(FULL, mbar_wait(&full[st], ph, g.wait_ns));
        if (!have && lane == 0) atomicExch(&s_abort, 1);
      }
      const uint4 *tile = reinterpret_cast<const uint4 *>(ring + (size_t)st * TILE_BYTES);
      if (++st == NSTAGE) {
        st = 0;
        ph ^= 1u;
      }
      if (!have) continue;
      uint4 v[U];
#pragma unroll
      for (int k = 0; k < U; ++k) v[k] = tile[k * NTC + threadIdx.x];
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[st == 0 ? NSTAGE - 1 : st - 1]);
#pragma unroll
      for (int k = 0; k < U; ++k) vec_fold<T>(v[k], q, c, thr);
    }
    // at most one partial tile (the row's last vectors)
    const int tpb = tb > tf ? tb : tf;
    if (tpb < te && (long long)tpb * TV < rc.nvec) {
      const long long nv = rc.nvec - (long long)tpb * TV;
      bool have = false;
      if (!*(volatile int *)&s_abort) {
        have = __all_sync(FULL, mbar_wait(&full[st], ph, g.wait_ns));
        if (!have && lane == 0) atomicExch(&s_abort, 1);
      }
      const uint4 *tile = reinterpret_cast<const uint4 *>(ring + (size_t)st * TILE_BYTES);
      const int cur = st;
      if (++st == NSTAGE) {
        st = 0;
        ph ^= 1u;
      }
      if (have) {
        uint4 v[U];
#pragma unroll
        for (int k = 0; k < U; ++k) {
          const int vi = k * NTC + threadIdx.x;
          v[k] = (vi < nv) ? tile[vi] : Dt<T>::neg_inf();
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[cur]);
#pragma unroll
        for (int k = 0; k < U; ++k) vec_fold<T>(v[k], q, c, thr);
      }
    }
    // scalar head / tail of the row when this CTA holds its first / last tile
    if (tb == 0 && (int)threadIdx.x < rc.head)
      elem_fold(Dt<T>::load(rc.p + threadIdx.x), q, c, thr);
    if (te == g.tpr) {
      const long long tt = rc.head + rc.nvec * VEC + threadIdx.x;
      if (tt < g.V) elem_fold(Dt<T>::load(rc.p + tt), q, c, thr);
    }
    // this warp's partial: lanes combined in fp64 with shuffles
    const float m = q.mt;
    const float sl = runstat_sum_at_max(q, c);
    const float mw = warp_max_nan(m);
    double sw = (m == -INFINITY) ? 0.0 : (double)sl * (double)ex2(scaled(m - mw, c));
    sw = warp_sum(sw);
    if (g.pcw != 1) {
      // one partial per warp: no CTA barrier (a warp that skipped a tile has
      // seen the abort flag by now)
      if (lane == 0) {
        const int aborted = *(volatile int *)&s_abort;
        const long long slot = (long long)blockIdx.x - tile_owner(row * g.tpr, G, g.tiles);
        Partial out;
        out.s = aborted ? 0.0 : sw;
        out.m = aborted ? __int_as_float(0x7fc00000) : mw;
        out.pad = aborted ? 1u : 0u;
        part[(row * g.slots + slot) * CW + warp] = out;
      }
      continue;
    }
    const int pb = seg & 1;
    if (lane == 0) {
      s_wm[pb][warp] = mw;
      s_ws[pb][warp] = sw;
    }
    // (two buffers: a warp writing the next segment's values has passed this
    // barrier again only after warp 0 has read these)
    consumer_sync();
    ++seg;
    if (warp == 0) {
      // the CTA's partial: the warps' sums rescaled to their common max in
      // fp64, added in warp order
      const float mi = lane < CW ? s_wm[pb][lane] : -INFINITY;
      const double si = lane < CW ? s_ws[pb][lane] : 0.0;
      const float M = warp_max_nan(mi);
      const double c64 = kLog2e / (double)Tcur;
      double t = (mi == -INFINITY) ? si : si * exp2(((double)mi - (double)M) * c64);
      t = warp_sum(t);
      const int aborted = *(volatile int *)&s_abort;
      if (lane == 0) {
        const long long slot = (long long)blockIdx.x - tile_owner(row * g.tpr, G, g.tiles);
        Partial out;
        out.s = aborted ? 0.0 : t;
        out.m = aborted ? __int_as_float(0x7fc00000) : M;
        out.pad = aborted ? 1u : 0u;
        part[(row * g.slots + slot) * CW] = out;
      }
    }
  }
  late_end();
}

// ---------------------------------------------------------------------------
// kernel 2: accept test + residual / bonus draw ("finish")
// ---------------------------------------------------------------------------
// Grid: B sequences x nsr V-chunks.  Every CTA of sequence b first repeats the
// (small) acceptance step for b: it combines the V-split partials of the 2K+1
// rows in fp64, gathers p_i(x_i) and q_i(x_i) (fp64 exp2 of exact logits),
// tests u*q < p on K lanes and finds the first rejection n with __ballot_sync /
// __ffs.  Chunk 0 writes the accepted prefix.  Then each CTA streams its chunk
// of the drawn row pair (target/draft row n, or the target's row K for the
// bonus), forming r(v) = St * max(0, p - q) = max(0, e_t - (St/Sd) e_d) on the
// fly (or e_t for the bonus), and adds it up in fp64.  The last CTA of the
// sequence to finish (atomic arrival ticket; nothing waits) draws: block scan
// of the chunk sums in fp64, the chunk holding u*Z, then a block scan over
// that chunk with the weights kept in registers, first crossing wins.  When
// the residual mass is below 2^-64 the fp32 weights have run out of range and
// the draw is redone in fp64 over the whole row pair.

struct DrawRow {
  float Mt, Md, lhi, llo;
  Scale c;
  bool bonus;
};

// r = St * max(0, p - q) = max(0, e_t - (St/Sd) e_d) with e = 2^((z - m)c)
// (or e_t for the bonus row).  The same inlined arithmetic serves the chunk
// sums and the rescan, so both see bit-identical per-element weights.
__device__ __forceinline__ float res_weight(float zt, float zd, const DrawRow &d) {
  const float et = ex2(scaled(zt - d.Mt, d.c));
  if (d.bonus) return et;
  const float ed = ex2(scaled(zd - d.Md, d.c));
  const float t1 = __fmaf_rn(-d.lhi, ed, et);
  const float t2 = __fmaf_rn(-d.llo, ed, t1);
  return t2 > 0.0f ? t2 : 0.0f;
}
// The same weights for two adjacent entries with packed fp32x2 operations:
// each lane of every packed operation rounds exactly as the scalar one above
// (a - b is a + (-b) exactly), so the weights are bit-identical.
__device__ __forceinline__ float2 res_weight2(float2 zt, float2 zd, const DrawRow &d) {
  const float2 hi = make_float2(d.c.hi, d.c.hi), lo = make_float2(d.c.lo, d.c.lo);
  const float2 dt = __fadd2_rn(zt, make_float2(-d.Mt, -d.Mt));
  const float2 at = __ffma2_rn(dt, hi, __fmul2_rn(dt, lo));
  const float2 et = make_float2(ex2(at.x), ex2(at.y));
  if (d.bonus) return et;
  const float2 dd = __fadd2_rn(zd, make_float2(-d.Md, -d.Md));
  const float2 ad = __ffma2_rn(dd, hi, __fmul2_rn(dd, lo));
  const float2 ed = make_float2(ex2(ad.x), ex2(ad.y));
  const float2 t1 = __ffma2_rn(make_float2(-d.lhi, -d.lhi), ed, et);
  const float2 t2 = __ffma2_rn(make_float2(-d.llo, -d.llo), ed, t1);
  return make_float2(t2.x > 0.0f ? t2.x : 0.0f, t2.y > 0.0f ? t2.y : 0.0f);
}

// Block-wide exclusive prefix sum of one double per thread, in thread order
// (fixed association); `total` receives the block sum.  All NTH threads call it.
template <int NTH>
__device__ __forceinline__ double block_excl_scan(double v, double &total) {
  constexpr int NW = NTH / 32;
  __shared__ double sm[NW];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  double incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const double y = __shfl_up_sync(FULL, incl, o);
    if (lane >= o) incl += y;
  }
  double excl = __shfl_up_sync(FULL, incl, 1);
  if (lane == 0) excl = 0.0;
  __syncthreads();  // a previous call may still be reading sm
  if (lane == 31) sm[warp] = incl;
  __syncthreads();
  double base = 0.0, tot = 0.0;
  for (int w = 0; w < NW; ++w) {
    if (w < warp) base += sm[w];
    tot += sm[w];
  }
  total = tot;
  return base + excl;
}

// fp64 probability of one logit: 2^((z - M) c) / S
template <typename T>
__device__ __forceinline__ double prob64(const T *row, long long v, float M, double S, double c64) {
  return exp2(((double)Dt<T>::load(row + v) - (double)M) * c64) / S;
}

// Inverse-CDF draw from max(0, p - q) entirely in fp64 by the whole CTA
// (contiguous segments per thread, block scan, first crossing).  If the fp64
// residual is zero as well, draws from p (as the oracle does).  Used only when
// the fp32 residual weights have run out of range.
template <typename T, int NTH>
__device__ __noinline__ int draw_exact64(const T *pt, const T *pd, long long V, float Mt,
                                         double St, float Md, double Sd, double c64, double u,
                                         int *s_y, int *s_lastpos, double *dbg_Z) {
  const long long E = (V + NTH - 1) / NTH;
  const long long e0 = (long long)threadIdx.x * E < V ? (long long)threadIdx.x * E : V;
  const long long e1 = (e0 + E < V) ? e0 + E : V;
  double sr = 0.0, sp = 0.0;
  for (long long v = e0; v < e1; ++v) {
    const double p = prob64(pt, v, Mt, St, c64);
    const double q = prob64(pd, v, Md, Sd, c64);
    sr += (p - q > 0.0) ? p - q : 0.0;
    sp += p;
  }
  double Zr, Zp;
  const double xr = block_excl_scan<NTH>(sr, Zr);
  const double xp = block_excl_scan<NTH>(sp, Zp);
  const bool use_p = !(Zr > 0.0);
  const double Z = use_p ? Zp : Zr;
  const double t = u * Z;
  double C = use_p ? xp : xr;
  int last = -1;
  bool found = false;
  for (long long v = e0; v < e1; ++v) {
    const double p = prob64(pt, v, Mt, St, c64);
    const double q = prob64(pd, v, Md, Sd, c64);
    const double x = use_p ? p : ((p - q > 0.0) ? p - q : 0.0);
    if (x > 0.0) last = (int)v;
    C += x;
    if (!found && C > t) {
      atomicMin(s_y, (int)v);
      found = true;
    }
  }
  if (last >= 0) atomicMax(s_lastpos, last);
  __syncthreads();
  const int y = (*s_y != INT_MAX) ? *s_y : (*s_lastpos >= 0 ? *s_lastpos : 0);
  if (threadIdx.x == 0 && dbg_Z) *dbg_Z = Z;
  return y;
}

// The window and decision state of a finish pass (the rows of StatsGeom's
// window).  With `state` null the pass decides every sequence over its window
// and draws.  Otherwise (early exit):
//   decide-only pass: a sequence rejected inside the window gets its outputs
//     (but the drawn token), state[b] = n and info[b]; one accepting the whole
//     window gets the window's tokens and stays kSeqActive; an invalid one gets
//     -1 outputs and state[b] = -1;
//   final pass: a sequence decided earlier goes straight to its draw (from
//     info[b]); an active one is tested on this window, then drawn.
//
// SMC-SD mode (`dlogw` set; the SMC-SD page, section 2): no token is rejected;
// every particle keeps its K draft tokens, draws its bonus token from p_K, and
// gets the log importance ratio of its K tokens,
// dlogw[b] = sum_i [log p_i(x_i) - log q_i(x_i)] in fp64 (-inf when invalid).
//
// Chained second stage (`len` set; the HiSpec page, section 2): sequence b
// tests only its first m = len[b] + 1 tokens (the output of the first stage;
// len[b] < 0: invalid there); when all m are accepted they are emitted with no
// draw.  With `emit_count`, out_n holds the number of tokens emitted rather
// than the number accepted.
struct FinishWindow {
  int p0, np, bonus, rps;
  int decide_only;
  int *state;
  SeqInfo *info;
  double *dlogw;
  const int32_t *len;
  int emit_count;
  int dbg_pstride;  // positions per sequence of the p_x / q_x diagnostics (K, or K+1
                    // for a chained second stage)
  // Row statistics kept across passes (the chained verify): with `save_t` set,
  // the combined (max, sum) of every target row of the window is stored at
  // save_t[b*(K+1) + position]; with `dstat` set, the sweep covered only the
  // window's target rows (srows = np per sequence) and the draft rows' (max,
  // sum) are read from dstat[b*(K+1) + position].
  int srows;  // rows per sequence of the sweep's partials
  Partial *save_t;
  const Partial *dstat;
};
constexpr int kChainAll = -3;  // chained stage: every tested token accepted

// PLAIN: the finish of the plain verify (no early-exit state, no SMC-SD
// weights, no chained stage), compiled with those paths removed: less code and
// fewer spilled registers, measured 0.8-1.1 us faster per call.
template <typename T, int UW, int NTH, bool PLAIN = false>
__global__ void __launch_bounds__(NTH, 65536 / (NTH * kFinishMaxNreg)) k_finish(
    const T *__restrict__ target, const T *__restrict__ draft,
    const int32_t *__restrict__ tokens, const float *__restrict__ u_accept,
    const float *__restrict__ u_resample, const float *__restrict__ temperature, int K,
    long long V, int tpr, long long tiles, long long G1, int slots, int pcw, int nsr, int cpb,
    int d_rows, int tok_stride, FinishWindow fw, const Partial *__restrict__ part,
    ResPartial *__restrict__ rpart, unsigned *__restrict__ counters,
    int32_t *__restrict__ out_tokens, int32_t *__restrict__ out_n,
    float *__restrict__ dbg_row_max, double *__restrict__ dbg_row_sum,
    double *__restrict__ dbg_px, double *__restrict__ dbg_qx, double *__restrict__ dbg_Z) {
  constexpr int VEC = Dt<T>::VEC;
  constexpr long long CHV = 32LL * UW;                 // vectors per (warp-)chunk
  constexpr long long CH = CHV * VEC;                  // elements per chunk
  constexpr int NW = NTH / 32;
  constexpr int EMAX = (int)((CH + 2 * VEC + NTH - 1) / NTH);  // rescan elements per thread
  __shared__ float sM[66];
  __shared__ double sS[66];
  __shared__ int s_n, s_last, s_mode, s_chunk, s_y, s_lastpos;
  __shared__ unsigned s_tmo[2 * NW];  // per half-warp: a partial it read was marked incomplete
  __shared__ double s_base, s_t;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int ncb = (nsr + cpb - 1) / cpb;  // CTAs per sequence
  const long long b = (long long)blockIdx.x / ncb;
  const int cb = (int)((long long)blockIdx.x - b * ncb);  // this CTA: chunks cb*cpb ...
  const int R = 2 * K + 1;
  if (PLAIN) {  // (the launch picks PLAIN only for these values)
    fw.state = nullptr;
    fw.info = nullptr;
    fw.decide_only = 0;
    fw.dlogw = nullptr;
    fw.len = nullptr;
    fw.emit_count = 0;
    fw.save_t = nullptr;
    fw.dstat = nullptr;
  }
  const int RW = fw.rps;  // rows of the window per sequence
  // The kernel after this one on the stream (the next call's statistics sweep,
  // or the SMC-SD resampling) may be placed as this grid's CTAs finish; it
  // waits for this grid to complete before it touches anything this grid uses.
  cudaTriggerProgrammaticLaunchCompletion();
  // A chained second stage tests the first stage's tokens (written by the
  // finish pass two kernels back): those are read only after the wait for the
  // statistics sweep, whose completion implies that pass's.
  if (fw.len) cudaGridDependencySynchronize();

  // ---- inputs of this call (independent of the statistics kernel) ----
  const float Tf = __ldg(temperature + b);
  const bool t_ok = isfinite(Tf) && Tf > 0.0f;
  const double c64 = kLog2e / (double)Tf;
  int x = 0;
  bool x_ok = true;
  float zt_x = 0.f, zd_x = 0.f, u = 0.f;
  const int pos = fw.p0 + lane;  // the position lane `lane` of warp 0 tests
  // positions of the window this sequence tests (chained stage: its first m)
  const int len_b = fw.len ? __ldg(fw.len + b) : 0;
  const int m_b = fw.len ? (len_b >= 0 ? len_b + 1 : 0) : fw.np;
  if (warp == 0 && lane < m_b) {
    x = __ldg(tokens + b * tok_stride + pos);
    x_ok = (x >= 0) && ((long long)x < V);
    u = fw.dlogw ? 0.f : __ldg(u_accept + b * tok_stride + pos);  // (SMC-SD accepts no test)
    if (x_ok) {
      zt_x = Dt<T>::load(target + (b * (K + 1) + pos) * V + x);
      zd_x = Dt<T>::load(draft + (b * d_rows + pos) * V + x);
    }
  }
  const float ures = __ldg(u_resample + b);
  cudaGridDependencySynchronize();  // the row statistics are complete from here on

  // (the decide-only pass is the first: every sequence is open there)
  const int st_b = (fw.state && !fw.decide_only) ? __ldcg(fw.state + b) : kSeqActive;
  if (st_b == -1) return;  // found invalid by an earlier pass: its outputs are written
  int n;
  float Mt, Md;
  double St, Sd;
  if (st_b >= 0) {
    // decided by an earlier pass: straight to the draw
    const SeqInfo *si = fw.info + b;
    n = st_b;
    Mt = __ldcg(&si->Mt);
    Md = __ldcg(&si->Md);
    St = __ldcg(&si->St);
    Sd = __ldcg(&si->Sd);
  } else {
    // ---- combine the V-split partials of every row of the window (fp64) ----
    // Half-warp h (16 lanes) takes rows h, h + 2*NW, ..., so a window of up to
    // 2*NW rows is reduced in one step.  The partials of a row are those of the
    // CTAs of the statistics sweep that hold its tiles, in order, pcw per CTA
    // (stored CW apart when pcw = 1); a lane loads up to four of them in one
    // round (longer lists, as at B = 1, are read in a loop), so the L2 round
    // trips overlap.  A partial marked incomplete (a wait of its sweep CTA ran
    // out) makes the sequence invalid.
    const int RS = fw.srows;  // the sweep's rows per sequence (RW unless only targets)
    auto row_slots = [&](int r) -> int {
      const long long row = b * RS + r;
      return (int)(tile_owner(row * tpr + tpr - 1, G1, tiles) - tile_owner(row * tpr, G1, tiles) +
                   1) * pcw;
    };
    const int pst = pcw == 1 ? CW : 1;  // stride between a row's partials
    const int hw = threadIdx.x >> 4, hl = lane & 15;
    const unsigned hmask = 0xFFFFu << (lane & 16);
    unsigned tmo = 0u;
    for (int r0 = 0; r0 < RS; r0 += 2 * NW) {
      const int r = r0 + hw;
      const bool has = r < RS;
      const Partial *P = part + (b * RS + (has ? r : 0)) * slots * CW;
      const int nslot = has ? row_slots(r) : 0;
      Partial px[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        px[k].m = -INFINITY;
        px[k].s = 0.0;
        px[k].pad = 0;
        const int sk = hl + 16 * k;
        if (sk < nslot) px[k] = P[sk * pst];
      }
      float m = fmax_nan(fmax3_nan(px[0].m, px[1].m, px[2].m), px[3].m);
      unsigned ab = px[0].pad | px[1].pad | px[2].pad | px[3].pad;
#pragma unroll 4
      for (int s = hl + 64; s < nslot; s += 16) {
        m = fmax_nan(m, P[s * pst].m);
        ab |= P[s * pst].pad;
      }
      m = half_max_nan(m);
      tmo |= (__ballot_sync(FULL, ab != 0u) & hmask) ? 1u : 0u;
      auto rescale = [&](const Partial &ps) -> double {
        return (ps.m == -INFINITY) ? ps.s : ps.s * exp2(((double)ps.m - (double)m) * c64);
      };
      double acc = 0.0;
#pragma unroll
      for (int k = 0; k < 4; ++k)
        if (hl + 16 * k < nslot) acc += rescale(px[k]);
#pragma unroll 4
      for (int s = hl + 64; s < nslot; s += 16) acc += rescale(P[s * pst]);
      acc = half_sum(acc);
      if (has && hl == 0) {
        // the row's position and role, and its place in the window's order
        const bool is_t = fw.dstat || !(r < 2 * fw.np && (r & 1));
        const int rp = fw.dstat ? fw.p0 + r : (r < 2 * fw.np ? fw.p0 + (r >> 1) : K);
        const int w = fw.dstat ? 2 * r : r;
        sM[w] = m;
        sS[w] = acc;
        // natural row index: target rows 0..K, then draft rows 0..K-1
        const int j = is_t ? rp : K + 1 + rp;
        if (cb == 0 && dbg_row_max) dbg_row_max[b * R + j] = m;
        if (cb == 0 && dbg_row_sum) dbg_row_sum[b * R + j] = acc;
        if (cb == 0 && fw.save_t && is_t) {
          Partial o;
          o.s = acc;
          o.m = m;
          o.pad = 0;
          fw.save_t[b * (K + 1) + rp] = o;
        }
      }
    }
    if (hl == 0) s_tmo[hw] = tmo;
    if (fw.dstat) {  // the draft rows' statistics, kept by an earlier pass
      for (int i = threadIdx.x; i < fw.np; i += blockDim.x) {
        const Partial *q = fw.dstat + b * (K + 1) + fw.p0 + i;
        sM[2 * i + 1] = __ldcg(&q->m);
        sS[2 * i + 1] = __ldcg(&q->s);
      }
    }
    __syncthreads();

    // ---- acceptance test and first rejection (warp 0) ----
    if (warp == 0) {
      // a statistics partial left incomplete by a wait that ran out makes the
      // sequence invalid rather than silently wrong (every CTA of the sequence
      // reads the same partials, so they all decide alike)
      unsigned tmo_any = 0u;
      for (int w = 0; w < 2 * NW; ++w) tmo_any |= s_tmo[w];
      const bool timed_out = tmo_any != 0u;
      bool rows_ok = true;
      for (int r = lane; r < RW; r += 32)
        rows_ok = rows_ok && isfinite(sM[r]) && isfinite(sS[r]) && sS[r] > 0.0;
      rows_ok = __all_sync(FULL, rows_ok) && !timed_out;
      bool acc_i = false;
      double p = 0.0, q = 0.0;
      if (lane < m_b && x_ok && rows_ok && t_ok) {
        p = exp2(((double)zt_x - (double)sM[2 * lane]) * c64) / sS[2 * lane];
        q = exp2(((double)zd_x - (double)sM[2 * lane + 1]) * c64) / sS[2 * lane + 1];
        acc_i = (double)u * q < p;
      }
      const unsigned bad_x = __ballot_sync(FULL, lane < m_b && !x_ok);
      const unsigned accm = __ballot_sync(FULL, lane < m_b && acc_i);
      const bool seq_ok = t_ok && rows_ok && bad_x == 0 && !(fw.len && len_b < 0);
      const unsigned kmask = (m_b >= 32) ? FULL : ((1u << m_b) - 1u);
      unsigned rej = ~accm & kmask;
      if (fw.dlogw) {
        // SMC-SD: keep every draft token; weight by the log ratio of the window
        double lr = 0.0;
        if (lane < fw.np && seq_ok) {
          const double iT = 1.0 / (double)Tf;
          lr = (((double)zt_x - (double)sM[2 * lane]) * iT - log(sS[2 * lane])) -
               (((double)zd_x - (double)sM[2 * lane + 1]) * iT - log(sS[2 * lane + 1]));
        }
        lr = warp_sum(lr);
        if (cb == 0 && lane == 0) fw.dlogw[b] = seq_ok ? lr : -INFINITY;
        rej = 0u;
      }
      // the decision: rejected at n, all of K accepted (bonus), still open,
      // or (chained stage) all tested tokens accepted
      int nn = rej ? fw.p0 + __ffs(rej) - 1 : (fw.bonus ? K : (fw.len ? kChainAll : kSeqActive));
      if (!seq_ok) nn = -1;
      if (lane == 0) s_n = nn;
      if (cb == 0) {
        int32_t *ot = out_tokens + b * (K + 1);
        if (nn == -1) {
          for (int i = lane; i <= K; i += 32) ot[i] = -1;
        } else {
          // tokens accepted in the window, then -1 after the decided position
          const int last = nn >= 0 ? nn : (nn == kChainAll ? m_b : fw.p0 + fw.np);
          if (lane < m_b && pos < last) ot[pos] = x;
          const int tail = nn >= 0 ? nn + 1 : (nn == kChainAll ? m_b : K + 1);
          for (int i = tail + lane; i <= K; i += 32) ot[i] = -1;
          if (lane < m_b && pos <= (nn >= 0 ? nn : K)) {
            if (dbg_px) dbg_px[b * fw.dbg_pstride + pos] = p;
            if (dbg_qx) dbg_qx[b * fw.dbg_pstride + pos] = q;
          }
        }
        if (lane == 0) {
          if (nn == kChainAll) out_n[b] = m_b;
          else if (nn != kSeqActive) out_n[b] = (fw.emit_count && nn >= 0) ? nn + 1 : nn;
          if (fw.state) fw.state[b] = nn;
          if (nn == -1) {
            unsigned f = 0;
            if (!t_ok) f |= SPECDEC_ERR_TEMPERATURE;
            if (bad_x) f |= SPECDEC_ERR_TOKEN;
            if (!rows_ok && !timed_out) f |= SPECDEC_ERR_LOGITS;
            atomicOr(&g_error_flags, f);
          }
          if (fw.decide_only && nn >= 0) {  // the drawn pair for the final pass
            const bool nb = nn == K && fw.bonus;  // drawn from the bonus row
            const int wt = nb ? 2 * fw.np : 2 * (nn - fw.p0);
            SeqInfo si;
            si.Mt = sM[wt];
            si.St = sS[wt];
            si.Md = nb ? 0.f : sM[wt + 1];
            si.Sd = nb ? 1.0 : sS[wt + 1];
            fw.info[b] = si;
          }
        }
      }
    }
    __syncthreads();
    n = s_n;
    if (n < 0 || fw.decide_only) return;  // invalid, still open, or not drawn in this pass
    // the bonus row only when the window holds it (a chained second stage
    // rejecting its position K draws from that row's residual instead)
    const bool nb = n == K && fw.bonus;
    const int wt = nb ? 2 * fw.np : 2 * (n - fw.p0);
    Mt = sM[wt];
    St = sS[wt];
    Md = nb ? 0.f : sM[wt + 1];
    Sd = nb ? 1.0 : sS[wt + 1];
  }

  // ---- this CTA's chunk of the drawn row pair ----
  DrawRow d;
  // (a sequence decided by an earlier pass at n == K was decided on the bonus)
  d.bonus = (n == K) && (fw.bonus || st_b >= 0);
  d.Mt = Mt;
  d.Md = d.bonus ? 0.f : Md;
  if (d.bonus) Sd = 1.0;
  d.c = make_scale(c64);
  const double lam = d.bonus ? 0.0 : St / Sd;
  d.lhi = (float)lam;
  d.llo = (float)(lam - (double)d.lhi);
  const T *pt = target + (b * (K + 1) + n) * V;
  const T *pd = d.bonus ? pt : draft + (b * d_rows + n) * V;

  const int head = row_head(pt, V);
  const bool vec_ok = row_head(pd, V) == head;
  const long long nvec = vec_ok ? (V - head) / VEC : 0;
  // chunk c covers elements [lo_c, hi_c): chunk 0 also takes the head, and the
  // chunk whose range holds the < VEC tail elements takes those
  auto chunk_lo = [&](int cidx) -> long long {
    if (cidx == 0) return 0;
    const long long v = head + (long long)cidx * CH;
    return v < V ? v : V;
  };
  auto chunk_hi = [&](int cidx) -> long long {
    if (cidx == nsr - 1) return V;
    const long long v = head + (long long)(cidx + 1) * CH;
    return v < V ? v : V;
  };

  // Chunk sums: the warps of this CTA take its chunks round robin; a chunk is
  // 32 lanes x UW vectors of the row pair, summed per lane in fp32 and across
  // the warp in fp64 with shuffles (no CTA barrier).  Then one arrival ticket.
  const uint4 *vt = reinterpret_cast<const uint4 *>(pt + head);
  const uint4 *vd = reinterpret_cast<const uint4 *>(pd + head);
  const long long tail_chunk = nvec / CHV < nsr - 1 ? nvec / CHV : (long long)(nsr - 1);
  const int c_beg = cb * cpb;
  const int c_end = (cb + 1) * cpb < nsr ? (cb + 1) * cpb : nsr;
  bool wrote = false;
  for (int chunk = c_beg + warp; chunk < c_end; chunk += NW) {
    float rs = 0.f;
    float2 rs2 = make_float2(0.f, 0.f);  // packed partial sums of the vector body
    if (vec_ok) {
      uint4 at[UW], ad[UW];
#pragma unroll
      for (int k = 0; k < UW; ++k) {
        const long long vi = (long long)chunk * CHV + (long long)k * 32 + lane;
        at[k] = vi < nvec ? __ldg(vt + vi) : make_uint4(0, 0, 0, 0);
        ad[k] = (vi < nvec && !d.bonus) ? __ldg(vd + vi) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int k = 0; k < UW; ++k) {
        const long long vi = (long long)chunk * CHV + (long long)k * 32 + lane;
        if (vi < nvec) {
          float xt[VEC], xd[VEC];
          Dt<T>::unpack(at[k], xt);
          Dt<T>::unpack(ad[k], xd);
#pragma unroll
          for (int q = 0; q < VEC; q += 2)
            rs2 = __fadd2_rn(rs2, res_weight2(make_float2(xt[q], xt[q + 1]),
                                              make_float2(xd[q], xd[q + 1]), d));
        }
      }
      // head elements (chunk 0) and the < VEC tail elements (their chunk)
      const long long tail = head + nvec * VEC + lane;
      const long long extra[2] = {(chunk == 0 && lane < head) ? (long long)lane : -1,
                                  (chunk == tail_chunk && tail < V && lane < VEC) ? tail : -1};
#pragma unroll
      for (int e = 0; e < 2; ++e)
        if (extra[e] >= 0)
          rs += res_weight(Dt<T>::load(pt + extra[e]), d.bonus ? 0.f : Dt<T>::load(pd + extra[e]),
                           d);
    } else {  // rows of different alignment: scalar loads over the chunk
      const long long lo = chunk_lo(chunk), hi = chunk_hi(chunk);
      for (long long v = lo + lane; v < hi; v += 32)
        rs += res_weight(Dt<T>::load(pt + v), d.bonus ? 0.f : Dt<T>::load(pd + v), d);
    }
    const double tot = warp_sum((double)rs + ((double)rs2.x + (double)rs2.y));
    if (lane == 0) {
      ResPartial o;
      o.R = tot;
      o.pad = 0.0;
      rpart[b * nsr + chunk] = o;
      wrote = true;
    }
  }
  if (wrote) __threadfence();  // chunk sums visible before this CTA's ticket
  __syncthreads();
  if (threadIdx.x == 0) {
    const unsigned t = atomicAdd(&counters[b], 1u);
    s_last = (t == (unsigned)(ncb - 1));
    s_chunk = INT_MAX;
    s_y = INT_MAX;
    s_lastpos = -1;
    s_base = -1.0;  // < 0 selects the "last positive element" rule
  }
  __syncthreads();
  if (!s_last) return;

  // ---- the last CTA of sequence b draws ----
  __threadfence();
  const ResPartial *rp = rpart + b * nsr;
  const int cper = (nsr + NTH - 1) / NTH;  // chunks per thread, contiguous
  const int c0 = threadIdx.x * cper < nsr ? threadIdx.x * cper : nsr;
  const int c1 = c0 + cper < nsr ? c0 + cper : nsr;
  // the thread's chunk sums are read once: the first kDrawRegChunks kept in
  // registers (every chunk when nsr <= kDrawRegChunks * NTH), later ones re-read
  constexpr int kDrawRegChunks = 4;
  double rv[kDrawRegChunks];
  double my = 0.0;
#pragma unroll
  for (int k = 0; k < kDrawRegChunks; ++k) {
    rv[k] = (c0 + k < c1) ? __ldcg(&rp[c0 + k].R) : 0.0;
    my += rv[k];
  }
  for (int c2 = c0 + kDrawRegChunks; c2 < c1; ++c2) my += __ldcg(&rp[c2].R);
  double Z;
  const double cexcl = block_excl_scan<NTH>(my, Z);
  if (threadIdx.x == 0) s_mode = (!d.bonus && !(Z >= ldexp(St, -64))) ? 1 : 0;
  __syncthreads();
  if (s_mode == 1) {
    const int y = draw_exact64<T, NTH>(pt, pd, V, d.Mt, St, d.Md, Sd, c64, (double)ures, &s_y, &s_lastpos,
                               dbg_Z ? dbg_Z + b : nullptr);
    if (threadIdx.x == 0) out_tokens[b * (K + 1) + n] = y;
    return;
  }
  const double t = (double)ures * Z;
  // the chunk holding t: its thread claims it and keeps its exclusive prefix
  int my_chunk = INT_MAX;
  double my_base = -1.0;
  {
    double C = cexcl;
#pragma unroll
    for (int k = 0; k < kDrawRegChunks; ++k) {
      if (my_chunk == INT_MAX && c0 + k < c1) {
        if (C <= t && t < C + rv[k]) {
          my_chunk = c0 + k;
          my_base = C;
        }
        C += rv[k];
      }
    }
    for (int c2 = c0 + kDrawRegChunks; my_chunk == INT_MAX && c2 < c1; ++c2) {
      const double v = __ldcg(&rp[c2].R);
      if (C <= t && t < C + v) {
        my_chunk = c2;
        my_base = C;
      }
      C += v;
    }
    if (my_chunk != INT_MAX) atomicMin(&s_chunk, my_chunk);
  }
  __syncthreads();
  // (rounding may let two neighbours claim: the first chunk wins, and only its
  // claimant writes the base)
  if (my_chunk == s_chunk) s_base = my_base;
  if (threadIdx.x == 0) {
    s_t = t;
    if (s_chunk == INT_MAX) {  // rounding left t at or past the total
      int cs = 0;
      for (int c2 = nsr - 1; c2 >= 0; --c2)
        if (__ldcg(&rp[c2].R) > 0.0) {
          cs = c2;
          break;
        }
      s_chunk = cs;
    }
    if (dbg_Z) dbg_Z[b] = Z / St;
  }
  __syncthreads();

  // rescan of the chosen chunk: contiguous elements per thread, in registers
  const long long lo = chunk_lo(s_chunk), hi = chunk_hi(s_chunk);
  const long long L = hi - lo;
  const long long E = (L + NTH - 1) / NTH;
  const long long e0 = lo + (long long)threadIdx.x * E < hi ? lo + (long long)threadIdx.x * E : hi;
  const long long e1 = (e0 + E < hi) ? e0 + E : hi;
  float w[EMAX];
#pragma unroll
  for (int k = 0; k < EMAX; ++k) {
    const long long v = e0 + k;
    w[k] = (v < e1) ? res_weight(Dt<T>::load(pt + v), d.bonus ? 0.f : Dt<T>::load(pd + v), d)
                    : 0.0f;
  }
  double mysum = 0.0;
  int lastpos = -1;
#pragma unroll
  for (int k = 0; k < EMAX; ++k) {
    mysum += (double)w[k];
    if (w[k] > 0.0f) lastpos = (int)(e0 + k);
  }
  double ctot;
  const double excl = block_excl_scan<NTH>(mysum, ctot);
  if (lastpos >= 0) atomicMax(&s_lastpos, lastpos);
  if (s_base >= 0.0) {
    double C = s_base + excl;
#pragma unroll
    for (int k = 0; k < EMAX; ++k) {
      if (e0 + k < e1) {
        C += (double)w[k];
        if (C > t) {
          atomicMin(&s_y, (int)(e0 + k));
          break;
        }
      }
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int y = s_y;
    if (y == INT_MAX) y = (s_lastpos >= 0) ? s_lastpos : (int)lo;
    out_tokens[b * (K + 1) + n] = y;
  }
}

// ---------------------------------------------------------------------------
// kernel 3 (SMC-SD): weights, effective sample size, systematic resampling
// ---------------------------------------------------------------------------
// One CTA per group of N particles (the SMC-SD page, section 2: "if the
// effective sample size falls below a threshold, low-weight particles are
// dropped and high-weight ones copied").  log w_n = log w_n(before) +
// dlogw_n; normalised weights wbar = exp(log w - max) / sum, ESS =
// 1 / sum wbar^2, all in fp64.  When ESS < threshold * N: systematic
// resampling with the group's uniform u, ancestor a_k = min{j : C_j > (k+u)/N}
// with C the inclusive running sum of wbar in particle order (a block scan,
// contiguous particles per thread), found by binary search; every log-weight
// of the group becomes 0.  Otherwise a_k = k and the log-weights carry over.
// A group whose particles are all invalid (log-weight -inf) gets ESS 0,
// ancestors -1 and log-weights -inf.
constexpr int kSmcMaxN = 4096;  // particles per group (shared-memory running sums)

__global__ void __launch_bounds__(NT) k_smc_resample(const double *__restrict__ dlogw,
                                                     const double *__restrict__ logw_in,
                                                     const float *__restrict__ u_resample,
                                                     double ess_threshold, int N,
                                                     double *__restrict__ logw_out,
                                                     double *__restrict__ ess_out,
                                                     int32_t *__restrict__ ancestors) {
  extern __shared__ double sC[];  // N running sums
  __shared__ double s_red[NWARP];
  __shared__ int s_res;
  const int g = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  cudaGridDependencySynchronize();  // the increments of this call are written
  const long long base = (long long)g * N;
  const int per = (N + NT - 1) / NT;  // contiguous particles per thread
  const int k0 = tid * per < N ? tid * per : N;
  const int k1 = k0 + per < N ? k0 + per : N;
  auto lw = [&](int k) -> double {
    const double a = __ldcg(dlogw + base + k);
    return logw_in ? __ldcg(logw_in + base + k) + a : a;
  };
  // max
  double m = -INFINITY;
  for (int k = k0; k < k1; ++k) m = fmax(m, lw(k));
#pragma unroll
  for (int o = 16; o; o >>= 1) m = fmax(m, __shfl_xor_sync(FULL, m, o));
  if (lane == 0) s_red[warp] = m;
  __syncthreads();
  m = s_red[0];
  for (int w = 1; w < NWARP; ++w) m = fmax(m, s_red[w]);
  __syncthreads();
  if (!(m > -INFINITY) || !isfinite(m)) {  // every particle invalid (or NaN)
    for (int k = tid; k < N; k += NT) {
      logw_out[base + k] = -INFINITY;
      ancestors[base + k] = -1;
    }
    if (tid == 0) ess_out[g] = 0.0;
    return;
  }
  // weights relative to the max, their exclusive prefix (contiguous per thread)
  double sw = 0.0;
  for (int k = k0; k < k1; ++k) {
    const double w = exp(lw(k) - m);
    sC[k] = w;
    sw += w;
  }
  double incl = sw;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const double y = __shfl_up_sync(FULL, incl, o);
    if (lane >= o) incl += y;
  }
  double excl = __shfl_up_sync(FULL, incl, 1);
  if (lane == 0) excl = 0.0;
  if (lane == 31) s_red[warp] = incl;
  __syncthreads();
  double before = 0.0, S = 0.0;
  for (int w = 0; w < NWARP; ++w) {
    if (w < warp) before += s_red[w];
    S += s_red[w];
  }
  excl += before;
  __syncthreads();
  // normalised running sums and the sum of squares
  double sq = 0.0, C = excl;
  for (int k = k0; k < k1; ++k) {
    const double wb = sC[k] / S;
    sq += wb * wb;
    C += sC[k];
    sC[k] = C / S;
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) sq += __shfl_xor_sync(FULL, sq, o);
  if (lane == 0) s_red[warp] = sq;
  __syncthreads();
  double q2 = 0.0;
  for (int w = 0; w < NWARP; ++w) q2 += s_red[w];
  const double ess = 1.0 / q2;
  if (tid == 0) {
    ess_out[g] = ess;
    s_res = ess < ess_threshold * (double)N;
  }
  __syncthreads();
  if (!s_res) {
    for (int k = tid; k < N; k += NT) {
      logw_out[base + k] = lw(k);
      ancestors[base + k] = k;
    }
    return;
  }
  // last particle with positive weight (for targets rounding leaves past C)
  int lastpos = -1;
  for (int k = k0; k < k1; ++k)
    if (sC[k] > (k > 0 ? sC[k - 1] : 0.0)) lastpos = k;
#pragma unroll
  for (int o = 16; o; o >>= 1) lastpos = max(lastpos, __shfl_xor_sync(FULL, lastpos, o));
  __shared__ int s_last[NWARP];
  if (lane == 0) s_last[warp] = lastpos;
  __syncthreads();
  for (int w = 0; w < NWARP; ++w) lastpos = max(lastpos, s_last[w]);
  const double u = (double)__ldg(u_resample + g);
  for (int k = tid; k < N; k += NT) {
    const double t = ((double)k + u) / (double)N;
    int lo = 0, hi = N;  // first j with C_j > t, in [0, N]
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (sC[mid] > t) hi = mid;
      else lo = mid + 1;
    }
    ancestors[base + k] = lo < N ? lo : lastpos;
    logw_out[base + k] = 0.0;
  }
}

// ---------------------------------------------------------------------------
// kernel 4 (LogitSpec): top-k of a logit row, excluding one token
// ---------------------------------------------------------------------------
// The LogitSpec page ("LogitSpec: Accelerating Retrieval-based Speculative
// Decoding via Next Next Token Speculation", section 2, workflow step 2):
// after the next token x_{i+1} is known, the top k entries of the last logit
// row other than x_{i+1} are the candidates for the next-next token.  Order:
// larger logit first, equal logits by ascending token id; a row with a NaN is
// invalid.  One CTA per row:
//   1. one pass over the row (HBM) keeps each thread's maximum, the maximum
//      of each of its groups of vectors (top 16 key bits, in shared memory)
//      and whether it met a NaN; the thread maxima give a lower bound tau of
//      the row's k-th largest key (the largest 16-bit key bucket holding at
//      least k of them, by bisection with block-wide counts);
//   2. only the groups whose maximum reaches tau (about k of them for real
//      logits) are read again (from L2), spread over all threads, and every
//      non-excluded element with key >= tau goes to a shared buffer; when
//      too many groups qualify (heavy ties) the whole row is read again;
//   3. each candidate's rank (the number of candidates above it) places it;
//      up to the buffer's size a bitonic sort of (key, ~index) does it
//      instead, and when ties at the top overflow the buffer (e.g. a constant
//      row) an exact radix select of the k-th key (8 bits per pass) and an
//      index-ordered pick among the keys equal to it take over.
// 512 threads per row, three CTAs per SM (all 320 rows of a B=64, K=5 batch
// resident at once).
constexpr int kTopkThreads = 512;
constexpr int kTopkCtasPerSm = 3;
constexpr int kTopkMaxK = 256;
constexpr int kTopkCap = 2048;   // candidate buffer (power of two)
constexpr int kTopkGroups = 16;  // vector groups per thread whose maxima pass 1 keeps
constexpr int kTopkWork = 1024;  // qualifying groups pass 2 reads selectively, at most

// order-preserving key: a larger logit has a larger key, -0 and +0 the same
// key (equal logits); never 0 for a non-NaN value
__device__ __forceinline__ uint32_t logit_key(float f) {
  uint32_t u = __float_as_uint(f);
  if (u == 0x80000000u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// the logit of a key (logit_key is one-to-one but for -0 and +0, which share
// a key: those are read back from the row)
template <typename T>
__device__ __forceinline__ float key_logit(uint32_t key, const T *p) {
  if (key == 0x80000000u) return Dt<T>::load(p);
  return __uint_as_float((key & 0x80000000u) ? (key & 0x7FFFFFFFu) : ~key);
}

// f(index, logit) for every element of a row: scalar head, 16-byte vectors
// (four independent loads in flight per thread), scalar tail
template <typename T, typename F>
__device__ __forceinline__ void row_foreach(const T *row, int V, F f) {
  constexpr int VEC = Dt<T>::VEC;
  constexpr int UNR = 4;
  const int head = row_head(row, (long long)V);
  const int nvec = (V - head) / VEC;
  if ((int)threadIdx.x < head) f((int)threadIdx.x, Dt<T>::load(row + threadIdx.x));
  const uint4 *pv = reinterpret_cast<const uint4 *>(row + head);
  const int step = (int)blockDim.x;
  for (int i0 = threadIdx.x; i0 < nvec; i0 += step * UNR) {
    uint4 v[UNR];
#pragma unroll
    for (int u = 0; u < UNR; ++u) {
      const int i = i0 + u * step;
      v[u] = i < nvec ? __ldg(pv + i) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < UNR; ++u) {
      const int i = i0 + u * step;
      if (i < nvec) {
        float x[VEC];
        Dt<T>::unpack(v[u], x);
#pragma unroll
        for (int e = 0; e < VEC; ++e) f(head + i * VEC + e, x[e]);
      }
    }
  }
  const int t0 = head + nvec * VEC;
  if (t0 + (int)threadIdx.x < V) f(t0 + (int)threadIdx.x, Dt<T>::load(row + t0 + threadIdx.x));
}

// NaN-propagating max of the 8 (bf16) or 4 (fp32) logits of a 16-byte vector
__device__ __forceinline__ uint32_t bf16x2_max_nan(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.NaN.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
template <typename T>
__device__ __forceinline__ float vec_max_nan(const uint4 &v);
template <>
__device__ __forceinline__ float vec_max_nan<__nv_bfloat16>(const uint4 &v) {
  const uint32_t m = bf16x2_max_nan(bf16x2_max_nan(v.x, v.y), bf16x2_max_nan(v.z, v.w));
  return fmax_nan(__uint_as_float(m << 16), __uint_as_float(m & 0xFFFF0000u));
}
template <>
__device__ __forceinline__ float vec_max_nan<float>(const uint4 &v) {
  return fmax3_nan(fmax3_nan(__uint_as_float(v.x), __uint_as_float(v.y), __uint_as_float(v.z)),
                   __uint_as_float(v.w), -INFINITY);
}

// bitonic sort, descending, of n (a power of two, <= the block's reach) keys
template <typename K>
__device__ __forceinline__ void bitonic_desc(K *a, int n) {
  for (int size = 2; size <= n; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      __syncthreads();
      for (int i = threadIdx.x; i < n / 2; i += blockDim.x) {
        const int lo = 2 * i - (i & (stride - 1));  // first of the pair
        const int hi = lo + stride;
        const bool desc = ((lo & size) == 0);
        const K x = a[lo], y = a[hi];
        if ((x < y) == desc) {
          a[lo] = y;
          a[hi] = x;
        }
      }
    }
  }
  __syncthreads();
}

template <typename T>
__global__ void __launch_bounds__(kTopkThreads, kTopkCtasPerSm) k_topk_exclude(
    const T *__restrict__ logits, long long row_stride, const long long *__restrict__ row_index,
    int V, const int32_t *__restrict__ exclude, int k, int32_t *__restrict__ out_idx,
    float *__restrict__ out_val) {
  __shared__ unsigned long long cand[kTopkCap];  // (key << 32) | ~index
  __shared__ unsigned hist[256];
  __shared__ unsigned short s_gkey[kTopkGroups][kTopkThreads];  // group maxima (key >> 16)
  __shared__ uint32_t s_work[kTopkWork];  // qualifying groups: thread | group << 16
  __shared__ int s_n, s_bad, s_rem, s_nw, s_cnt[kTopkThreads / 32];
  __shared__ uint32_t s_prefix;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const long long r = blockIdx.x;
  // Programmatic dependent launch: this CTA may be placed while the previous
  // kernel on the stream drains; it reads every input after waiting for it,
  // and lets the next kernel be placed as this grid drains.
  cudaGridDependencySynchronize();
  cudaTriggerProgrammaticLaunchCompletion();
  const long long src = row_index ? row_index[r] : r;
  const T *row = logits + src * row_stride;
  const int ex0 = exclude ? exclude[r] : -1;
  const int ex = (ex0 >= 0 && ex0 < V) ? ex0 : -1;
  int32_t *oi = out_idx + r * k;
  float *ov = out_val ? out_val + r * k : nullptr;
  if (tid == 0) {
    s_n = 0;
    s_bad = 0;
  }
  // 1. One pass over the row.  Thread t reads vectors t + 512*m in rounds of
  // four (round j: m = 4j .. 4j+3); rounds are grouped ipg at a time into at
  // most kTopkGroups groups whose maxima (top 16 bits of the key, 0 = no
  // value) go to shared memory.  The thread maxima are distinct elements, so
  // their k-th largest is at most the row's: tau is the smallest key of the
  // largest 16-bit bucket holding at least k thread maxima (exact for bf16
  // keys).  NaNs are left out of the maxima and mark the row invalid.
  constexpr int VEC = Dt<T>::VEC;
  const int head = row_head(row, (long long)V);
  const int nvec = (V - head) / VEC;
  const int P = nvec;
  const uint4 *pv = reinterpret_cast<const uint4 *>(row + head);
  const int niter = (P + 4 * kTopkThreads - 1) / (4 * kTopkThreads);  // rounds
  const int ipg = (niter + kTopkGroups - 1) / kTopkGroups;           // rounds per group
  const int ngrp = ipg > 0 ? (niter + ipg - 1) / ipg : 0;
  const int tail0 = head + nvec * VEC;
  float mx = -INFINITY, gmx = -INFINITY;
  bool seen = false, gseen = false, bad = false;
  auto take1 = [&](int v, float x) {
    bad |= isnan(x);
    if (v != ex && !isnan(x)) {
      mx = fmaxf(mx, x);
      seen = true;
    }
  };
  if (tid < head) take1(tid, Dt<T>::load(row + tid));
  if (tail0 + tid < V) take1(tail0 + tid, Dt<T>::load(row + tail0 + tid));
  for (int j = 0; j < niter; ++j) {
    const int i0 = tid + j * 4 * kTopkThreads;
    uint4 w[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int i = i0 + u * kTopkThreads;
      w[u] = i < P ? __ldg(pv + i) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int i = i0 + u * kTopkThreads;
      if (i >= P) continue;
      const int v0 = head + i * VEC;
      const float m = vec_max_nan<T>(w[u]);
      if (ex >= v0 && ex < v0 + VEC || isnan(m)) {
        float x[VEC];
        Dt<T>::unpack(w[u], x);
#pragma unroll
        for (int e2 = 0; e2 < VEC; ++e2) {
          bad |= isnan(x[e2]);
          if (v0 + e2 != ex && !isnan(x[e2])) {
            gmx = fmaxf(gmx, x[e2]);
            gseen = true;
          }
        }
      } else {
        gmx = fmaxf(gmx, m);
        gseen = true;
      }
    }
    if ((j + 1) % ipg == 0 || j + 1 == niter) {  // the group ends
      s_gkey[j / ipg][tid] = gseen ? (unsigned short)(logit_key(gmx) >> 16) : (unsigned short)0;
      if (gseen) {
        mx = fmaxf(mx, gmx);
        seen = true;
      }
      gmx = -INFINITY;
      gseen = false;
    }
  }
  const uint32_t tkey = seen ? logit_key(mx) : 0u;  // 0: no value (below every key)
  // bisection over the 16-bit buckets with block-wide counts
  uint32_t blo = 0, bhi = 65535;
  while (blo < bhi) {
    const uint32_t mid = (blo + bhi + 1) >> 1;
    if (__syncthreads_count(tkey >= (mid << 16)) >= k) blo = mid;
    else bhi = mid - 1;
  }
  const uint32_t tau = blo << 16;  // the bucket's smallest key (low 16 bits 0)
  // 2. The qualifying groups (maximum >= tau) go to a work list; every thread
  // then takes vectors of the listed groups in turn (one L2 round trip for
  // about k groups), and every non-excluded key >= tau goes to the candidate
  // buffer (a vector is unpacked only when its max reaches tau).
  if (tid == 0) s_nw = 0;
  __syncthreads();
  for (int gi = 0; gi < ngrp; ++gi)
    if ((uint32_t)s_gkey[gi][tid] << 16 >= tau && s_gkey[gi][tid] != 0) {
      const int pos = atomicAdd(&s_nw, 1);
      if (pos < kTopkWork) s_work[pos] = (uint32_t)tid | ((uint32_t)gi << 16);
    }
  auto scalar2 = [&](int v, float x) {
    const uint32_t key = logit_key(x);
    if (v != ex && key >= tau && !isnan(x)) {
      const int pos = atomicAdd(&s_n, 1);
      if (pos < kTopkCap)
        cand[pos] = ((unsigned long long)key << 32) | (unsigned)(0xFFFFFFFFu - (unsigned)v);
    }
  };
  auto vec2 = [&](int i, const uint4 &w) {
    const float m = vec_max_nan<T>(w);
    if (!isnan(m) && logit_key(m) >= tau) {
      float x[VEC];
      Dt<T>::unpack(w, x);
      const int v0 = head + i * VEC;
#pragma unroll
      for (int e2 = 0; e2 < VEC; ++e2) scalar2(v0 + e2, x[e2]);
    }
  };
  __syncthreads();
  const int nw = s_nw;
  if (tid < head) scalar2(tid, Dt<T>::load(row + tid));
  if (tail0 + tid < V) scalar2(tail0 + tid, Dt<T>::load(row + tail0 + tid));
  if (nw <= kTopkWork) {
    const int per = 4 * ipg;  // vectors of one group
    for (int f0 = tid; f0 < nw * per; f0 += 4 * kTopkThreads) {
      uint4 w[4];
      int iv[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int f = f0 + u * kTopkThreads;
        iv[u] = -1;
        if (f < nw * per) {
          const uint32_t e = s_work[f / per];
          const int r2 = f % per;
          const int j = (int)(e >> 16) * ipg + r2 / 4;
          const int i = (int)(e & 0xFFFFu) + (4 * j + (r2 & 3)) * kTopkThreads;
          if (j < niter && i < P) iv[u] = i;
        }
        w[u] = iv[u] >= 0 ? __ldg(pv + iv[u]) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u)
        if (iv[u] >= 0) vec2(iv[u], w[u]);
    }
  } else {  // many groups reach tau (heavy ties): the whole row again
    for (int i0 = tid; i0 < P; i0 += 4 * kTopkThreads) {
      uint4 w[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int i = i0 + u * kTopkThreads;
        w[u] = i < P ? __ldg(pv + i) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int i = i0 + u * kTopkThreads;
        if (i < P) vec2(i, w[u]);
      }
    }
  }
  if (__any_sync(FULL, bad) && lane == 0) s_bad = 1;
  __syncthreads();
  if (s_bad) {  // invalid row
    for (int i = tid; i < k; i += blockDim.x) {
      oi[i] = -1;
      if (ov) ov[i] = __int_as_float(0x7fc00000);
    }
    if (tid == 0) atomicOr(&g_error_flags, SPECDEC_ERR_LOGITS);
    return;
  }
  int n = s_n;
  if (n <= 2 * kTopkThreads) {
    // 3. few candidates (about k for real logits): each one's place in the
    // order is the number of candidates above it ((key, ~index) pairs are
    // unique); no sort
    for (int i = tid; i < n; i += kTopkThreads) {
      const unsigned long long c = cand[i];
      int rank = 0;
      for (int j = 0; j < n; ++j) rank += cand[j] > c ? 1 : 0;
      if (rank < k) {
        const int v = (int)(0xFFFFFFFFu - (unsigned)(c & 0xFFFFFFFFull));
        oi[rank] = v;
        if (ov) ov[rank] = key_logit((uint32_t)(c >> 32), row + v);
      }
    }
    for (int i = n + tid; i < k; i += blockDim.x) {
      oi[i] = -1;
      if (ov) ov[i] = -INFINITY;
    }
    return;
  }
  if (n > kTopkCap) {
    // 3. ties overflowed the buffer: exact k-th key by radix select
    const int KB = sizeof(T) == 2 ? 16 : 32;  // bf16 keys live in the top 16 bits
    uint32_t prefix = 0;
    int rem = k;
    for (int shift = 24; shift >= 32 - KB; shift -= 8) {
      for (int i = tid; i < 256; i += blockDim.x) hist[i] = 0;
      __syncthreads();
      const uint32_t hi_mask = (shift == 24) ? 0u : (0xFFFFFFFFu << (shift + 8));
      row_foreach(row, V, [&](int v, float x) {
        const uint32_t key = logit_key(x);
        if (v != ex && (key & hi_mask) == (prefix & hi_mask)) atomicAdd(&hist[(key >> shift) & 255u], 1u);
      });
      __syncthreads();
      if (tid == 0) {
        int cum = 0, d = 255;
        for (; d > 0; --d) {
          if (cum + (int)hist[d] >= rem) break;
          cum += (int)hist[d];
        }
        s_rem = rem - cum;
        s_prefix = prefix | ((uint32_t)d << shift);
      }
      __syncthreads();
      prefix = s_prefix;
      rem = s_rem;
      __syncthreads();
    }
    // tau = prefix (in the top KB bits); keys above it are k - rem elements,
    // and the first `rem` (by index) of the keys equal to it complete the k
    const uint32_t kmask = (KB == 32) ? 0xFFFFFFFFu : 0xFFFF0000u;
    if (tid == 0) s_n = 0;
    __syncthreads();
    row_foreach(row, V, [&](int v, float x) {
      const uint32_t key = logit_key(x) & kmask;
      if (v != ex && key > prefix) {
        const int pos = atomicAdd(&s_n, 1);
        cand[pos] = ((unsigned long long)logit_key(x) << 32) |
                    (unsigned)(0xFFFFFFFFu - (unsigned)v);
      }
    });
    // equal keys in index order: contiguous elements per thread, block scan
    const int E = (V + blockDim.x - 1) / blockDim.x;
    const int e0 = min(tid * E, V), e1 = min(e0 + E, V);
    int ce = 0;
    for (int v = e0; v < e1; ++v)
      if (v != ex && (logit_key(Dt<T>::load(row + v)) & kmask) == prefix) ++ce;
    int incl = ce;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(FULL, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane == 31) s_cnt[warp] = incl;
    __syncthreads();
    int base = incl - ce;
    for (int w = 0; w < warp; ++w) base += s_cnt[w];
    const int ngt = k - rem;
    for (int v = e0; v < e1 && base < rem; ++v) {
      const float x = Dt<T>::load(row + v);
      if (v != ex && (logit_key(x) & kmask) == prefix) {
        cand[ngt + base] = ((unsigned long long)logit_key(x) << 32) |
                           (unsigned)(0xFFFFFFFFu - (unsigned)v);
        ++base;
      }
    }
    __syncthreads();
    n = k;
  }
  // sort the candidates (padded with 0 to a power of two) and write the first k
  int np2 = 1;
  while (np2 < n || np2 < k) np2 <<= 1;
  for (int i = n + tid; i < np2; i += blockDim.x) cand[i] = 0ull;
  bitonic_desc(cand, np2);
  for (int i = tid; i < k; i += blockDim.x) {
    const unsigned long long c = cand[i];
    if (i < n && c != 0ull) {
      const int v = (int)(0xFFFFFFFFu - (unsigned)(c & 0xFFFFFFFFull));
      oi[i] = v;
      if (ov) ov[i] = Dt<T>::load(row + v);
    } else {
      oi[i] = -1;
      if (ov) ov[i] = -INFINITY;
    }
  }
}

// the FMA-pipe exponential on its own, for its accuracy test
__global__ void k_test_exp2(const float *__restrict__ a, float *__restrict__ y, int n) {
  const int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
  if (i + 1 < n) {
    const float2 r = exp2_fma2(make_float2(a[i], a[i + 1]));
    y[i] = r.x;
    y[i + 1] = r.y;
  } else if (i < n) {
    y[i] = exp2_fma2(make_float2(a[i], 0.0f)).x;
  }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
enum KernelId { KID_STATS = 0, KID_FINISH = 1, KID_SMC = 2, KID_TOPK = 3, KID_COUNT = 4 };
const char *kKernelNames[KID_COUNT] = {"k_row_stats", "k_finish", "k_smc_resample",
                                       "k_topk_exclude"};

std::mutex g_mu;
uint64_t g_launches[KID_COUNT];
struct Profiler {
  bool on = false;
  int max = 0;
  std::vector<std::pair<cudaEvent_t, cudaEvent_t>> ev[KID_COUNT];
} g_prof;

struct DeviceBuf {
  void *ptr = nullptr;
  size_t bytes = 0;
};
// Library-owned buffers, one per (device, stream): calls on different streams
// may overlap on the GPU, so they must not share partials, chunk sums or
// arrival tickets.
using BufKey = std::pair<int, uintptr_t>;
std::map<BufKey, DeviceBuf> g_ws;       // workspace
std::map<BufKey, DeviceBuf> g_staging;  // end-to-end staging

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// One statistics sweep: the window of positions it reads and its static
// partition of tiles over CTAs.
struct Sweep {
  int p0, np, bonus, rps;
  int tonly;                  // target rows only (see StatsGeom)
  int nb;                     // sequences
  long long rows, tiles, G1;  // G1: CTAs of the statistics sweep
  int slots;                  // partial slots per row
};

struct Plan {
  int esize, vec, U, tpr, nsr;
  Sweep full;            // the whole batch, every row
  Sweep first, second;   // early exit: positions [0, P), then [P, K] with the bonus row
  Sweep chain;           // chained second stage: the final layer's K+1 rows (the
                         // intermediate's statistics are kept from the first stage)
  int slots_max;         // partial slots per row in the workspace (the stride of every sweep)
  size_t off_part, off_part2, off_rpart, off_cnt, off_state, off_info, off_dlogw, off_s1tok,
      off_s1n, off_rstat, total, total_chained;
};

int num_sms() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

// partition of a sweep's tiles over its CTAs and the partial slots per row:
// the most CTAs whose tile ranges meet one row.  With small (4 KB) tiles the
// grid is m CTAs per row, so that every CTA's range lies inside one row (one
// partial, no row changes), with at least 3 tiles per CTA and at most `cap`
// CTAs.  Measured against the full 444-CTA grid: B = 1 15.9 -> 13.9 us per
// call, B = 4 17.9 -> 16.3 us.
void sweep_partition(Sweep &w, int tpr, long long cap, bool small_tiles) {
  w.rows = (long long)w.nb * w.rps;
  w.tiles = w.rows * tpr;
  if (small_tiles && w.rows > 0) {
    long long m = cap / w.rows;
    if (m > tpr / 3) m = tpr / 3;
    if (m >= 1) cap = w.rows * m;
  }
  w.G1 = w.tiles < cap ? w.tiles : cap;
  if (w.G1 < 1) w.G1 = 1;
  const long long minr = w.tiles / w.G1;  // shortest range
  w.slots = minr > 0 ? (int)((tpr - 1 + minr - 1) / minr + 1) : 1;
}

// A sweep over nb sequences: the target and draft rows of positions
// p0 .. p0+np-1 and, with `bonus`, the target's row K.
Sweep make_sweep(int nb, int p0, int np, int bonus, int tpr, long long cap, bool small_tiles) {
  Sweep w;
  w.p0 = p0;
  w.np = np;
  w.bonus = bonus;
  w.rps = 2 * np + bonus;
  w.tonly = 0;
  w.nb = nb;
  sweep_partition(w, tpr, cap, small_tiles);
  return w;
}

// A sweep over the target tensor's rows p0 .. p0+np-1 only.
Sweep make_target_sweep(int nb, int p0, int np, int tpr, long long cap, bool small_tiles) {
  Sweep w = make_sweep(nb, p0, np, 0, tpr, cap, small_tiles);
  w.tonly = 1;
  w.rps = np;
  sweep_partition(w, tpr, cap, small_tiles);
  return w;
}

// Positions the first early-exit sweep reads: two (a sequence whose first two
// draft tokens are both accepted goes on to the second sweep).
inline int early_split(int K) { return K < 2 ? K : 2; }

// Work decomposition for these sizes; a pure function of the sizes and the SM
// count, so repeated calls reduce in the same order (bit-reproducible).
bool make_plan(int B, int K, int V, specdec_dtype dtype, int sms, Plan &pl) {
  if (B < 0 || K < 1 || K > 32 || V < 1) return false;
  if (dtype != SPECDEC_F32 && dtype != SPECDEC_BF16) return false;
  pl.esize = dtype == SPECDEC_BF16 ? 2 : 4;
  pl.vec = 16 / pl.esize;
  const long long rows = (long long)B * (2 * K + 1);
  const long long nvec_max = ((long long)V + pl.vec - 1) / pl.vec;
  // tiles of 4 vectors per consumer thread (16 KB); 1 vector per thread when
  // 16 KB tiles would leave SMs idle (batches of a few sequences)
  const long long cap = (long long)kStatsCtasPerSm * sms;
  long long tpr = (nvec_max + NTC * 4 - 1) / (NTC * 4);
  pl.U = 4;
  if (rows * tpr < 2 * cap) {
    pl.U = 1;
    tpr = (nvec_max + NTC - 1) / NTC;
  }
  if (tpr < 1) tpr = 1;
  pl.tpr = (int)tpr;
  const bool small = pl.U == 1;
  pl.full = make_sweep(B, 0, K, 1, pl.tpr, cap, small);
  const int P = early_split(K);
  pl.first = make_sweep(B, 0, P, 0, pl.tpr, cap, small);
  pl.second = make_sweep(B, P, K - P, 1, pl.tpr, cap, small);
  pl.chain = make_target_sweep(B, 0, K + 1, pl.tpr, cap, small);
  pl.slots_max = pl.full.slots;
  for (const Sweep *w : {&pl.first, &pl.second, &pl.chain})
    if (w->slots > pl.slots_max) pl.slots_max = w->slots;
  // k_finish chunks: 32 lanes x kFinishUW vectors of the drawn row pair
  const long long nr = (nvec_max + 32LL * kFinishUW - 1) / (32LL * kFinishUW);
  pl.nsr = (int)(nr > 0 ? nr : 1);
  if ((long long)B * pl.nsr > INT_MAX) return false;
  if ((long long)B * (K + 1) * (long long)V > (1LL << 56)) return false;
  size_t off = 0;
  pl.off_part = off;
  long long rows_max = pl.full.rows;
  for (const Sweep *w : {&pl.first, &pl.second, &pl.chain})
    if (w->rows > rows_max) rows_max = w->rows;
  off = align256(off + sizeof(Partial) * (size_t)rows_max * pl.slots_max * CW);
  pl.off_rpart = off;
  off = align256(off + sizeof(ResPartial) * (size_t)B * pl.nsr);
  pl.off_cnt = off;
  off = align256(off + sizeof(unsigned) * (size_t)B);
  pl.off_state = off;
  off = align256(off + sizeof(int) * (size_t)B);
  pl.off_info = off;
  off = align256(off + sizeof(SeqInfo) * (size_t)B);
  pl.off_dlogw = off;
  off = align256(off + sizeof(double) * (size_t)B);
  pl.off_s1tok = off;
  off = align256(off + sizeof(int32_t) * (size_t)B * (K + 1));
  pl.off_s1n = off;
  off = align256(off + sizeof(int32_t) * (size_t)B);
  pl.off_rstat = off;
  off = align256(off + sizeof(Partial) * (size_t)B * (K + 1));
  pl.total = off > 0 ? off : 256;
  // the chained verify's second sweep writes its partials apart (the first
  // stage's finish pass may still read its own): a region after the others,
  // in the chained verify's workspace only
  pl.off_part2 = pl.total;
  pl.total_chained = align256(pl.total + sizeof(Partial) * (size_t)pl.chain.rows * pl.slots_max * CW);
  return true;
}

// resident CTAs per SM of a kernel with the given block and dynamic shared
// memory (queried once per device and kernel; also raises the kernel's
// dynamic shared-memory limit to what it asks for)
template <typename KernelT>
int resident_ctas(KernelT kernel, int threads, size_t smem) {
  static std::mutex mu;
  static std::unordered_map<std::string, int> cache;  // (device, kernel) -> CTAs per SM
  int dev = 0;
  cudaGetDevice(&dev);
  const std::string key = std::to_string(dev) + ":" +
                          std::to_string(reinterpret_cast<uintptr_t>((const void *)kernel));
  std::lock_guard<std::mutex> lk(mu);
  auto it = cache.find(key);
  if (it != cache.end()) return it->second;
  cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, threads, smem) != cudaSuccess ||
      n < 1)
    n = 1;
  cache[key] = n;
  return n;
}

// launch with programmatic stream serialisation: the kernel may be scheduled
// while the previous one drains and waits for it with cudaGridDependencySynchronize
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), unsigned grid, unsigned block, size_t smem,
                       cudaStream_t st, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(block);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

struct LaunchTimer {
  cudaEvent_t a = nullptr, b = nullptr;
  int kid;
  cudaStream_t st;
  LaunchTimer(int k, cudaStream_t s) : kid(k), st(s) {
    std::lock_guard<std::mutex> lk(g_mu);
    ++g_launches[k];
    if (g_prof.on && (int)g_prof.ev[k].size() < g_prof.max) {
      cudaEventCreate(&a);
      cudaEventCreate(&b);
      cudaEventRecord(a, st);
    }
  }
  ~LaunchTimer() {
    if (a) {
      cudaEventRecord(b, st);
      std::lock_guard<std::mutex> lk(g_mu);
      g_prof.ev[kid].push_back({a, b});
    }
  }
};

// Test hooks (specdec_test_set_wait_fault): the bound of every on-chip wait,
// and one tile (local index of a sweep) whose copy the sweep's producer never
// issues, so that the waits for it run out.
std::atomic<unsigned long long> g_hook_wait_ns{kWaitNs};
std::atomic<long long> g_hook_skip_tile{-1};

// Options of one pass (see StatsGeom and FinishWindow).
struct PassOpts {
  int *state = nullptr;          // early exit: per-sequence decision state
  SeqInfo *info = nullptr;       // early exit: drawn pairs decided by the first pass
  bool decide_only = false;      // early exit, first pass
  double *dlogw = nullptr;       // SMC-SD mode
  const int32_t *len = nullptr;  // chained second stage: first-stage accepted counts
  int d_rows = -1;               // rows per sequence of the draft tensor (default K)
  int tok_stride = -1;           // row stride of tokens and u_accept (default K)
  int emit_count = 0;            // out_n = tokens emitted instead of accepted
  int dbg_pstride = -1;          // positions per sequence of p_x / q_x (default K)
  Partial *save_t = nullptr;      // keep the target rows' statistics here (see FinishWindow)
  const Partial *dstat = nullptr; // the draft rows' statistics from an earlier pass
  Partial *part = nullptr;        // the sweep's partials (default: the workspace's first region)
  bool late_capable = false;      // run the sweep's LATE instantiation (see k_row_stats)
  bool late_sync = false;         // ... and let it stream before its wait
};

template <typename T, int NTH>
cudaError_t launch_finish(const T *t, const T *d, const int32_t *tok, const float *ua,
                          const float *ur, const float *temp, int K, int V, const Plan &pl,
                          const Sweep &sw, int pcw, int ctas_per_sm, bool decide_only, int d_rows,
                          int tok_stride, const FinishWindow &fw, const Partial *part,
                          ResPartial *rp, unsigned *cnt, const specdec_debug *dbg,
                          int32_t *out_tokens, int32_t *out_n, cudaStream_t st) {
  // CTAs per sequence: as many as keep the grid inside one wave of
  // ctas_per_sm CTAs per SM (each CTA repeats the small acceptance step); a
  // decide-only pass draws nothing: one CTA per sequence
  long long ncb = (long long)ctas_per_sm * num_sms() / (sw.nb > 0 ? sw.nb : 1);
  if (ncb < 1) ncb = 1;
  if (ncb > pl.nsr) ncb = pl.nsr;
  // long rows: at least two chunks per CTA (fewer CTAs repeating the combine
  // and taking tickets; measured at 128256 entries: B = 1 13.8 -> 13.1 us,
  // B = 4 16.7 -> 16.3 us; at 32000 entries it cost 0.3 us, so not there)
  if (pl.nsr >= 64 && ncb > (pl.nsr + 1) / 2) ncb = (pl.nsr + 1) / 2;
  const int cpb = decide_only ? pl.nsr : (int)((pl.nsr + ncb - 1) / ncb);
  const unsigned g2 = (unsigned)((long long)sw.nb * ((pl.nsr + cpb - 1) / cpb));
  const bool plain = fw.state == nullptr && fw.dlogw == nullptr && fw.len == nullptr &&
                     fw.dstat == nullptr && fw.save_t == nullptr && !decide_only && !fw.emit_count;
  auto kern = plain ? k_finish<T, kFinishUW, NTH, true> : k_finish<T, kFinishUW, NTH>;
  return launch_pdl(kern, g2, NTH, 0, st, t, d, tok, ua, ur, temp, K, (long long)V, pl.tpr, sw.tiles, sw.G1, pl.slots_max, pcw, pl.nsr, cpb, d_rows, tok_stride, fw,
                    part, rp, cnt, out_tokens, out_n, dbg ? dbg->row_max : nullptr,
                    dbg ? dbg->row_sum : nullptr, dbg ? dbg->p_x : nullptr,
                    dbg ? dbg->q_x : nullptr, dbg ? dbg->Z : nullptr);
}

// One pass: a statistics sweep over `sw` (of the open sequences when `state`
// is set and the pass is not the first), then k_finish over the same window
// and sequences (programmatic dependent launch: its launch and gathers overlap
// the sweep).
template <typename T>
specdec_status launch_pass(const void *tg, const void *dr, const int32_t *tok, const float *ua,
                           const float *ur, const float *temp, int B, int K, int V,
                           const Plan &pl, const Sweep &sw, const PassOpts &o, char *ws,
                           const specdec_debug *dbg, int32_t *out_tokens, int32_t *out_n,
                           cudaStream_t st) {
  const T *t = static_cast<const T *>(tg);
  const T *d = static_cast<const T *>(dr);
  Partial *part = o.part ? o.part : reinterpret_cast<Partial *>(ws + pl.off_part);
  ResPartial *rp = reinterpret_cast<ResPartial *>(ws + pl.off_rpart);
  unsigned *cnt = reinterpret_cast<unsigned *>(ws + pl.off_cnt);
  const int d_rows = o.d_rows > 0 ? o.d_rows : K;
  const int tok_stride = o.tok_stride > 0 ? o.tok_stride : K;
  StatsGeom g;
  g.K = K;
  g.V = V;
  g.tpr = pl.tpr;
  g.tiles = sw.tiles;
  g.slots = pl.slots_max;
  g.p0 = sw.p0;
  g.np = sw.np;
  g.rps = sw.rps;
  g.state = o.decide_only ? nullptr : o.state;  // the first pass reads every sequence
  g.d_rows = d_rows;
  g.tonly = sw.tonly;
  g.wait_ns = g_hook_wait_ns.load();
  g.skip_tile = g_hook_skip_tile.load();
  g.nb = sw.nb;
  // per-CTA partials where many CTAs share a row (small batches): the finish
  // pass then reads fewer; otherwise one per warp and no CTA barrier
  g.pcw = sw.slots > kCtaCombineSlots ? 1 : CW;
  g.late_sync = o.late_sync ? 1 : 0;
  cudaError_t e = cudaSuccess;
  {
    LaunchTimer lt(KID_STATS, st);
    const bool plain = !o.late_capable && g.state == nullptr && !g.tonly && g.d_rows == K;
    auto kern = o.late_capable
                    ? (pl.U == 4 ? k_row_stats<T, 4, true> : k_row_stats<T, 1, true>)
                    : plain ? (pl.U == 4 ? k_row_stats<T, 4, false, true>
                                         : k_row_stats<T, 1, false, true>)
                            : (pl.U == 4 ? k_row_stats<T, 4> : k_row_stats<T, 1>);
    const size_t smem = (size_t)NSTAGE * NTC * pl.U * 16;
    // the sweep assumes its CTAs are co-resident only for speed, not for
    // progress: nothing waits on another CTA
    resident_ctas(kern, NTS, smem);
    e = launch_pdl(kern, (unsigned)sw.G1, NTS, smem, st, t, d, temp, g, part, cnt, B);
  }
  if (e != cudaSuccess) return SPECDEC_ECUDA;
  {
    LaunchTimer lt(KID_FINISH, st);
    FinishWindow fw;
    fw.p0 = sw.p0;
    fw.np = sw.np;
    fw.bonus = sw.bonus;
    fw.rps = sw.tonly ? 2 * sw.np : sw.rps;  // the window: target and draft row per position
    fw.srows = sw.rps;
    fw.save_t = o.save_t;
    fw.dstat = o.dstat;
    fw.decide_only = o.decide_only ? 1 : 0;
    fw.state = o.state;
    fw.info = o.info;
    fw.dlogw = o.dlogw;
    fw.len = o.len;
    fw.emit_count = o.emit_count;
    fw.dbg_pstride = o.dbg_pstride > 0 ? o.dbg_pstride : K;
    e = launch_finish<T, kFinishThreads>(t, d, tok, ua, ur, temp, K, V, pl, sw, g.pcw,
                                         kFinishCtasPerSm, o.decide_only, d_rows, tok_stride, fw,
                                         part, rp, cnt, dbg, out_tokens, out_n, st);
  }
  return e == cudaSuccess ? SPECDEC_OK : SPECDEC_ECUDA;
}

template <typename T>
specdec_status launch_all(const void *tg, const void *dr, const int32_t *tok, const float *ua,
                          const float *ur, const float *temp, int B, int K, int V,
                          const Plan &pl, bool early_exit, char *ws, const specdec_debug *dbg,
                          int32_t *out_tokens, int32_t *out_n, cudaStream_t st) {
  if (!early_exit)
    return launch_pass<T>(tg, dr, tok, ua, ur, temp, B, K, V, pl, pl.full, PassOpts(), ws, dbg,
                          out_tokens, out_n, st);
  PassOpts o;
  o.state = reinterpret_cast<int *>(ws + pl.off_state);
  o.info = reinterpret_cast<SeqInfo *>(ws + pl.off_info);
  o.decide_only = true;
  specdec_status s = launch_pass<T>(tg, dr, tok, ua, ur, temp, B, K, V, pl, pl.first, o, ws, dbg,
                                    out_tokens, out_n, st);
  if (s != SPECDEC_OK) return s;
  o.decide_only = false;
  return launch_pass<T>(tg, dr, tok, ua, ur, temp, B, K, V, pl, pl.second, o, ws, dbg,
                        out_tokens, out_n, st);
}

// The chained two-stage verify: stage 1 is the verify with the intermediate
// logits as target; stage 2 verifies its tokens against the final logits with
// the intermediate as proposal (draft tensor of K+1 rows, tokens and uniforms
// of K+1 per sequence, m = n1 + 1 tested positions, no bonus).
template <typename T>
specdec_status launch_chained(const void *fin, const void *inter, const void *dr,
                              const int32_t *tok, const float *ua1, const float *ur1,
                              const float *ua2, const float *ur2, const float *temp, int B,
                              int K, int V, const Plan &pl, char *ws, int32_t *s1_tok,
                              int32_t *s1_n, int32_t *out_tokens, int32_t *out_emitted,
                              const specdec_debug *dbg2, cudaStream_t st) {
  Partial *rstat = reinterpret_cast<Partial *>(ws + pl.off_rstat);
  PassOpts o1;
  o1.save_t = rstat;  // the intermediate rows' statistics, for the second stage
  o1.late_capable = true;
  specdec_status s = launch_pass<T>(inter, dr, tok, ua1, ur1, temp, B, K, V, pl, pl.full, o1, ws,
                                    nullptr, s1_tok, s1_n, st);
  if (s != SPECDEC_OK) return s;
  PassOpts o;
  o.len = s1_n;
  o.d_rows = K + 1;
  o.tok_stride = K + 1;
  o.emit_count = 1;
  o.dstat = rstat;  // the second stage sweeps the final layer's rows only
  o.dbg_pstride = K + 1;
  // The final layer's logits are written by no kernel of this call: the
  // second sweep streams them at once, while the first stage's finish pass
  // still draws, into partials of its own.
  o.part = reinterpret_cast<Partial *>(ws + pl.off_part2);
  o.late_capable = true;
  o.late_sync = true;
  return launch_pass<T>(fin, inter, s1_tok, ua2, ur2, temp, B, K, V, pl, pl.chain, o, ws,
                        dbg2, out_tokens, out_emitted, st);
}

specdec_status check_args(const void *tg, const void *dr, const int32_t *tok, const float *ua,
                          const float *ur, const float *temp, int B, int K, int V,
                          specdec_dtype dtype, const int32_t *ot, const int32_t *on) {
  if (B < 0 || K < 1 || K > 32 || V < 1) return SPECDEC_EINVAL;
  if (dtype != SPECDEC_F32 && dtype != SPECDEC_BF16) return SPECDEC_EINVAL;
  if (B == 0) return SPECDEC_OK;
  if (!tg || !dr || !tok || !ua || !ur || !temp || !ot || !on) return SPECDEC_EINVAL;
  const uintptr_t es = dtype == SPECDEC_BF16 ? 2 : 4;
  if ((reinterpret_cast<uintptr_t>(tg) % es) || (reinterpret_cast<uintptr_t>(dr) % es))
    return SPECDEC_EINVAL;
  if ((reinterpret_cast<uintptr_t>(tok) | reinterpret_cast<uintptr_t>(ua) |
       reinterpret_cast<uintptr_t>(ur) | reinterpret_cast<uintptr_t>(temp) |
       reinterpret_cast<uintptr_t>(ot) | reinterpret_cast<uintptr_t>(on)) % 4)
    return SPECDEC_EINVAL;
  return SPECDEC_OK;
}

specdec_status run(const void *tg, const void *dr, const int32_t *tok, const float *ua,
                   const float *ur, const float *temp, int B, int K, int V, specdec_dtype dtype,
                   void *ws, size_t ws_bytes, const specdec_debug *dbg, int32_t *ot, int32_t *on,
                   cudaStream_t st, bool early_exit = false) {
  specdec_status s = check_args(tg, dr, tok, ua, ur, temp, B, K, V, dtype, ot, on);
  if (s != SPECDEC_OK || B == 0) return s;
  Plan pl;
  if (!make_plan(B, K, V, dtype, num_sms(), pl)) return SPECDEC_EINVAL;
  if (!ws || ws_bytes < pl.total || (reinterpret_cast<uintptr_t>(ws) & 255)) return SPECDEC_EINVAL;
  if (dtype == SPECDEC_BF16)
    return launch_all<__nv_bfloat16>(tg, dr, tok, ua, ur, temp, B, K, V, pl, early_exit,
                                     static_cast<char *>(ws), dbg, ot, on, st);
  return launch_all<float>(tg, dr, tok, ua, ur, temp, B, K, V, pl, early_exit,
                           static_cast<char *>(ws), dbg, ot, on, st);
}

// One SMC-SD round: the statistics sweep over every row, k_finish in SMC-SD
// mode (log ratios, bonus draws), then k_smc_resample per group.
specdec_status run_smc(const void *tg, const void *dr, const int32_t *tok, const float *ub,
                       const float *temp, const double *lw_in, const float *ur, double thr,
                       int B, int N, int K, int V, specdec_dtype dtype, void *ws,
                       int32_t *ot, double *lw_out, double *ess, int32_t *anc, double *dlw,
                       cudaStream_t st) {
  if (B < 0 || N < 1 || N > kSmcMaxN || K < 1 || K > 32 || V < 1) return SPECDEC_EINVAL;
  if (dtype != SPECDEC_F32 && dtype != SPECDEC_BF16) return SPECDEC_EINVAL;
  if (B % N != 0 || !(thr >= 0.0) || !isfinite(thr)) return SPECDEC_EINVAL;
  if (B == 0) return SPECDEC_OK;
  if (!tg || !dr || !tok || !ub || !temp || !ur || !ot || !lw_out || !ess || !anc || !ws)
    return SPECDEC_EINVAL;
  const uintptr_t es = dtype == SPECDEC_BF16 ? 2 : 4;
  if ((reinterpret_cast<uintptr_t>(tg) % es) || (reinterpret_cast<uintptr_t>(dr) % es))
    return SPECDEC_EINVAL;
  if ((reinterpret_cast<uintptr_t>(tok) | reinterpret_cast<uintptr_t>(ub) |
       reinterpret_cast<uintptr_t>(ur) | reinterpret_cast<uintptr_t>(temp) |
       reinterpret_cast<uintptr_t>(ot) | reinterpret_cast<uintptr_t>(anc)) % 4)
    return SPECDEC_EINVAL;
  if ((reinterpret_cast<uintptr_t>(lw_in) | reinterpret_cast<uintptr_t>(lw_out) |
       reinterpret_cast<uintptr_t>(ess) | reinterpret_cast<uintptr_t>(dlw)) % 8)
    return SPECDEC_EINVAL;
  Plan pl;
  if (!make_plan(B, K, V, dtype, num_sms(), pl)) return SPECDEC_EINVAL;
  char *w = static_cast<char *>(ws);
  int32_t *n_scratch = reinterpret_cast<int32_t *>(w + pl.off_state);
  double *inc = dlw ? dlw : reinterpret_cast<double *>(w + pl.off_dlogw);
  PassOpts o;
  o.dlogw = inc;
  specdec_status s = (dtype == SPECDEC_BF16)
      ? launch_pass<__nv_bfloat16>(tg, dr, tok, nullptr, ub, temp, B, K, V, pl, pl.full, o, w,
                                   nullptr, ot, n_scratch, st)
      : launch_pass<float>(tg, dr, tok, nullptr, ub, temp, B, K, V, pl, pl.full, o, w, nullptr,
                           ot, n_scratch, st);
  if (s != SPECDEC_OK) return s;
  LaunchTimer lt(KID_SMC, st);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(B / N));
  cfg.blockDim = dim3(NT);
  cfg.dynamicSmemBytes = sizeof(double) * (size_t)N;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, k_smc_resample, (const double *)inc, lw_in, ur,
                                           thr, N, lw_out, ess, anc);
  return e == cudaSuccess ? SPECDEC_OK : SPECDEC_ECUDA;
}

// grow-only device buffer of the current device and this stream (zero-filled
// when (re)allocated)
specdec_status ensure_buf(std::map<BufKey, DeviceBuf> &map, size_t bytes, cudaStream_t st,
                          void **out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SPECDEC_ECUDA;
  std::lock_guard<std::mutex> lk(g_mu);
  DeviceBuf &db = map[BufKey(dev, reinterpret_cast<uintptr_t>(st))];
  if (db.bytes < bytes) {
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(st, &cs) != cudaSuccess) return SPECDEC_ECUDA;
    if (cs != cudaStreamCaptureStatusNone) return SPECDEC_ESTATE;
    if (db.ptr) {
      if (cudaDeviceSynchronize() != cudaSuccess) return SPECDEC_ECUDA;
      cudaFree(db.ptr);
      db.ptr = nullptr;
      db.bytes = 0;
    }
    void *p = nullptr;
    if (cudaMalloc(&p, bytes) != cudaSuccess) return SPECDEC_ECUDA;
    if (cudaMemset(p, 0, bytes) != cudaSuccess) {
      cudaFree(p);
      return SPECDEC_ECUDA;
    }
    db.ptr = p;
    db.bytes = bytes;
  }
  *out = db.ptr;
  return SPECDEC_OK;
}

}  // namespace

// ---------------------------------------------------------------------------
// Fixed scratch for specdec_verify_static.  Some callers cannot allocate device
// memory at all: a serving engine that has reserved nearly all of HBM for its
// own pools (KV cache) and forbids allocations behind its back, or a caller
// that cannot afford cudaMalloc's device-wide synchronisation on its path.
// For them the workspace lives in this module-level device array instead: it
// is created when the module is loaded on a device and stays until the process
// exits, on every device that loads the library.
// ---------------------------------------------------------------------------
static __device__ __align__(256) unsigned char g_static_scratch[SPECDEC_STATIC_SCRATCH_BYTES];

namespace {
std::mutex g_static_mu;
std::unordered_map<int, void *> g_static_addr;  // device -> address of g_static_scratch

// Device address of the fixed scratch on the current device.  In host code the
// array's name only stands for the symbol; its device address is looked up
// once per device (with that device current) and cached.
specdec_status static_scratch_address(void **out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SPECDEC_ECUDA;
  std::lock_guard<std::mutex> lk(g_static_mu);
  auto it = g_static_addr.find(dev);
  if (it == g_static_addr.end()) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || p == nullptr)
      return SPECDEC_ECUDA;
    it = g_static_addr.emplace(dev, p).first;
  }
  *out = it->second;
  return SPECDEC_OK;
}
}  // namespace

// ---------------------------------------------------------------------------
// C-ABI
// ---------------------------------------------------------------------------
extern "C" {

size_t specdec_workspace_bytes(int B, int K, int V, specdec_dtype dtype) {
  Plan pl;
  if (!make_plan(B, K, V, dtype, num_sms(), pl)) return 0;
  return pl.total;
}

specdec_status specdec_verify_ex(const void *target_logits, const void *draft_logits,
                                 const int32_t *draft_tokens, const float *u_accept,
                                 const float *u_resample, const float *temperature, int B,
                                 int K, int V, specdec_dtype dtype, void *workspace,
                                 size_t workspace_bytes, const specdec_debug *dbg,
                                 int32_t *out_tokens, int32_t *out_num_accepted, void *stream) {
  return run(target_logits, draft_logits, draft_tokens, u_accept, u_resample, temperature, B, K,
             V, dtype, workspace, workspace_bytes, dbg, out_tokens, out_num_accepted,
             static_cast<cudaStream_t>(stream));
}

specdec_status specdec_verify(const void *target_logits, const void *draft_logits,
                              const int32_t *draft_tokens, const float *u_accept,
                              const float *u_resample, const float *temperature, int B, int K,
                              int V, specdec_dtype dtype, int32_t *out_tokens,
                              int32_t *out_num_accepted, void *stream) {
  specdec_status s = check_args(target_logits, draft_logits, draft_tokens, u_accept, u_resample,
                                temperature, B, K, V, dtype, out_tokens, out_num_accepted);
  if (s != SPECDEC_OK || B == 0) return s;
  const size_t need = specdec_workspace_bytes(B, K, V, dtype);
  if (need == 0) return SPECDEC_EINVAL;
  void *ws = nullptr;
  s = ensure_buf(g_ws, need, static_cast<cudaStream_t>(stream), &ws);
  if (s != SPECDEC_OK) return s;
  return run(target_logits, draft_logits, draft_tokens, u_accept, u_resample, temperature, B, K,
             V, dtype, ws, need, nullptr, out_tokens, out_num_accepted,
             static_cast<cudaStream_t>(stream));
}

specdec_status specdec_verify_early_exit_ex(const void *target_logits, const void *draft_logits,
                                            const int32_t *draft_tokens, const float *u_accept,
                                            const float *u_resample, const float *temperature,
                                            int B, int K, int V, specdec_dtype dtype,
                                            void *workspace, size_t workspace_bytes,
                                            const specdec_debug *dbg, int32_t *out_tokens,
                                            int32_t *out_num_accepted, void *stream) {
  return run(target_logits, draft_logits, draft_tokens, u_accept, u_resample, temperature, B, K,
             V, dtype, workspace, workspace_bytes, dbg, out_tokens, out_num_accepted,
             static_cast<cudaStream_t>(stream), true);
}

specdec_status specdec_verify_early_exit(const void *target_logits, const void *draft_logits,
                                         const int32_t *draft_tokens, const float *u_accept,
                                         const float *u_resample, const float *temperature,
                                         int B, int K, int V, specdec_dtype dtype,
                                         int32_t *out_tokens, int32_t *out_num_accepted,
                                         void *stream) {
  specdec_status s = check_args(target_logits, draft_logits, draft_tokens, u_accept, u_resample,
                                temperature, B, K, V, dtype, out_tokens, out_num_accepted);
  if (s != SPECDEC_OK || B == 0) return s;
  const size_t need = specdec_workspace_bytes(B, K, V, dtype);
  if (need == 0) return SPECDEC_EINVAL;
  void *ws = nullptr;
  s = ensure_buf(g_ws, need, static_cast<cudaStream_t>(stream), &ws);
  if (s != SPECDEC_OK) return s;
  return run(target_logits, draft_logits, draft_tokens, u_accept, u_resample, temperature, B, K,
             V, dtype, ws, need, nullptr, out_tokens, out_num_accepted,
             static_cast<cudaStream_t>(stream), true);
}

specdec_status specdec_smc_step(const void *target_logits, const void *draft_logits,
                                const int32_t *draft_tokens, const float *u_bonus,
                                const float *temperature, const double *log_weights_in,
                                const float *u_resample, double ess_threshold, int B, int N,
                                int K, int V, specdec_dtype dtype, int32_t *out_tokens,
                                double *log_weights_out, double *ess, int32_t *ancestors,
                                double *log_weight_increment, void *stream) {
  if (B < 0 || N < 1 || K < 1 || K > 32 || V < 1) return SPECDEC_EINVAL;
  if (B == 0) return SPECDEC_OK;
  const size_t need = specdec_workspace_bytes(B, K, V, dtype);
  if (need == 0) return SPECDEC_EINVAL;
  void *ws = nullptr;
  specdec_status s = ensure_buf(g_ws, need, static_cast<cudaStream_t>(stream), &ws);
  if (s != SPECDEC_OK) return s;
  return run_smc(target_logits, draft_logits, draft_tokens, u_bonus, temperature,
                 log_weights_in, u_resample, ess_threshold, B, N, K, V, dtype, ws, out_tokens,
                 log_weights_out, ess, ancestors, log_weight_increment,
                 static_cast<cudaStream_t>(stream));
}

specdec_status specdec_topk_exclude(const void *logits, long long row_stride,
                                    const long long *row_index, int rows, int V,
                                    specdec_dtype dtype, const int32_t *exclude, int k,
                                    int32_t *out_idx, float *out_val, void *stream) {
  if (rows < 0 || V < 1 || k < 1 || k > kTopkMaxK || row_stride < V) return SPECDEC_EINVAL;
  if (dtype != SPECDEC_F32 && dtype != SPECDEC_BF16) return SPECDEC_EINVAL;
  if (rows == 0) return SPECDEC_OK;
  if (!logits || !out_idx) return SPECDEC_EINVAL;
  const uintptr_t es = dtype == SPECDEC_BF16 ? 2 : 4;
  if (reinterpret_cast<uintptr_t>(logits) % es) return SPECDEC_EINVAL;
  if ((reinterpret_cast<uintptr_t>(exclude) | reinterpret_cast<uintptr_t>(out_idx) |
       reinterpret_cast<uintptr_t>(out_val)) % 4 ||
      reinterpret_cast<uintptr_t>(row_index) % 8)
    return SPECDEC_EINVAL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  LaunchTimer lt(KID_TOPK, st);
  cudaError_t e;
  if (dtype == SPECDEC_BF16)
    e = launch_pdl(k_topk_exclude<__nv_bfloat16>, (unsigned)rows, kTopkThreads, 0, st,
                   static_cast<const __nv_bfloat16 *>(logits), row_stride, row_index, V, exclude,
                   k, out_idx, out_val);
  else
    e = launch_pdl(k_topk_exclude<float>, (unsigned)rows, kTopkThreads, 0, st,
                   static_cast<const float *>(logits), row_stride, row_index, V, exclude, k,
                   out_idx, out_val);
  return e == cudaSuccess ? SPECDEC_OK : SPECDEC_ECUDA;
}

specdec_status specdec_verify_chained_ex(
    const void *final_logits, const void *intermediate_logits, const void *draft_logits,
    const int32_t *draft_tokens, const float *u_accept1, const float *u_resample1,
    const float *u_accept2, const float *u_resample2, const float *temperature, int B, int K,
    int V, specdec_dtype dtype, int32_t *out_tokens, int32_t *out_num_emitted,
    int32_t *stage1_tokens, int32_t *stage1_num_accepted, const specdec_debug *dbg2,
    void *stream) {
  if (K > 31) return SPECDEC_EINVAL;  // the second stage tests K+1 positions on one warp
  specdec_status s = check_args(intermediate_logits, draft_logits, draft_tokens, u_accept1,
                                u_resample1, temperature, B, K, V, dtype, out_tokens,
                                out_num_emitted);
  if (s != SPECDEC_OK || B == 0) return s;
  const uintptr_t es = dtype == SPECDEC_BF16 ? 2 : 4;
  if (!final_logits || !u_accept2 || !u_resample2 ||
      reinterpret_cast<uintptr_t>(final_logits) % es ||
      (reinterpret_cast<uintptr_t>(u_accept2) | reinterpret_cast<uintptr_t>(u_resample2) |
       reinterpret_cast<uintptr_t>(stage1_tokens) |
       reinterpret_cast<uintptr_t>(stage1_num_accepted)) % 4)
    return SPECDEC_EINVAL;
  Plan pl;
  if (!make_plan(B, K, V, dtype, num_sms(), pl)) return SPECDEC_EINVAL;
  void *ws = nullptr;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  s = ensure_buf(g_ws, pl.total_chained, st, &ws);
  if (s != SPECDEC_OK) return s;
  char *w = static_cast<char *>(ws);
  int32_t *s1t = stage1_tokens ? stage1_tokens : reinterpret_cast<int32_t *>(w + pl.off_s1tok);
  int32_t *s1n =
      stage1_num_accepted ? stage1_num_accepted : reinterpret_cast<int32_t *>(w + pl.off_s1n);
  if (dtype == SPECDEC_BF16)
    return launch_chained<__nv_bfloat16>(final_logits, intermediate_logits, draft_logits,
                                         draft_tokens, u_accept1, u_resample1, u_accept2,
                                         u_resample2, temperature, B, K, V, pl, w, s1t, s1n,
                                         out_tokens, out_num_emitted, dbg2, st);
  return launch_chained<float>(final_logits, intermediate_logits, draft_logits, draft_tokens,
                               u_accept1, u_resample1, u_accept2, u_resample2, temperature, B,
                               K, V, pl, w, s1t, s1n, out_tokens, out_num_emitted, dbg2, st);
}

specdec_status specdec_verify_chained(
    const void *final_logits, const void *intermediate_logits, const void *draft_logits,
    const int32_t *draft_tokens, const float *u_accept1, const float *u_resample1,
    const float *u_accept2, const float *u_resample2, const float *temperature, int B, int K,
    int V, specdec_dtype dtype, int32_t *out_tokens, int32_t *out_num_emitted,
    int32_t *stage1_tokens, int32_t *stage1_num_accepted, void *stream) {
  return specdec_verify_chained_ex(final_logits, intermediate_logits, draft_logits, draft_tokens,
                                   u_accept1, u_resample1, u_accept2, u_resample2, temperature,
                                   B, K, V, dtype, out_tokens, out_num_emitted, stage1_tokens,
                                   stage1_num_accepted, nullptr, stream);
}

specdec_status specdec_verify_bf16(const void *target_logits, const void *draft_logits,
                                   const int32_t *draft_tokens, const float *u_accept,
                                   const float *u_resample, const float *temperature, int B,
                                   int K, int V, int32_t *out_tokens, int32_t *out_num_accepted,
                                   void *stream) {
  return specdec_verify(target_logits, draft_logits, draft_tokens, u_accept, u_resample,
                        temperature, B, K, V, SPECDEC_BF16, out_tokens, out_num_accepted, stream);
}

specdec_status specdec_verify_f32(const void *target_logits, const void *draft_logits,
                                  const int32_t *draft_tokens, const float *u_accept,
                                  const float *u_resample, const float *temperature, int B,
                                  int K, int V, int32_t *out_tokens, int32_t *out_num_accepted,
                                  void *stream) {
  return specdec_verify(target_logits, draft_logits, draft_tokens, u_accept, u_resample,
                        temperature, B, K, V, SPECDEC_F32, out_tokens, out_num_accepted, stream);
}

specdec_status specdec_verify_host(const void *target_logits, const void *draft_logits,
                                   const int32_t *draft_tokens, const float *u_accept,
                                   const float *u_resample, const float *temperature, int B,
                                   int K, int V, specdec_dtype dtype, int32_t *out_tokens,
                                   int32_t *out_num_accepted, void *stream) {
  specdec_status s = check_args(target_logits, draft_logits, draft_tokens, u_accept, u_resample,
                                temperature, B, K, V, dtype, out_tokens, out_num_accepted);
  if (s != SPECDEC_OK || B == 0) return s;
  Plan pl;
  if (!make_plan(B, K, V, dtype, num_sms(), pl)) return SPECDEC_EINVAL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t es = (size_t)pl.esize;
  const size_t n_t = (size_t)B * (K + 1) * (size_t)V * es, n_d = (size_t)B * K * (size_t)V * es;
  const size_t n_tok = sizeof(int32_t) * (size_t)B * K, n_ua = sizeof(float) * (size_t)B * K;
  const size_t n_b = sizeof(float) * (size_t)B, n_ot = sizeof(int32_t) * (size_t)B * (K + 1);
  size_t off[9], tot = 0;
  const size_t sizes[8] = {n_t, n_d, n_tok, n_ua, n_b, n_b, n_ot, n_b};
  for (int i = 0; i < 8; ++i) {
    off[i] = tot;
    tot = align256(tot + sizes[i]);
  }
  off[8] = tot;
  tot += pl.total;
  void *base = nullptr;
  s = ensure_buf(g_staging, tot, st, &base);
  if (s != SPECDEC_OK) return s;
  char *c = static_cast<char *>(base);
  const void *src[6] = {target_logits, draft_logits, draft_tokens, u_accept, u_resample,
                        temperature};
  for (int i = 0; i < 6; ++i)
    if (cudaMemcpyAsync(c + off[i], src[i], sizes[i], cudaMemcpyHostToDevice, st) != cudaSuccess)
      return SPECDEC_ECUDA;
  s = run(c + off[0], c + off[1], reinterpret_cast<const int32_t *>(c + off[2]),
          reinterpret_cast<const float *>(c + off[3]), reinterpret_cast<const float *>(c + off[4]),
          reinterpret_cast<const float *>(c + off[5]), B, K, V, dtype, c + off[8], pl.total,
          nullptr, reinterpret_cast<int32_t *>(c + off[6]), reinterpret_cast<int32_t *>(c + off[7]),
          st);
  if (s != SPECDEC_OK) return s;
  if (cudaMemcpyAsync(out_tokens, c + off[6], n_ot, cudaMemcpyDeviceToHost, st) != cudaSuccess ||
      cudaMemcpyAsync(out_num_accepted, c + off[7], n_b, cudaMemcpyDeviceToHost, st) !=
          cudaSuccess)
    return SPECDEC_ECUDA;
  return cudaStreamSynchronize(st) == cudaSuccess ? SPECDEC_OK : SPECDEC_ECUDA;
}

specdec_status specdec_device_errors(void *stream, uint32_t *flags) {
  if (!flags) return SPECDEC_EINVAL;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return SPECDEC_ECUDA;
  unsigned v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, g_error_flags, sizeof v) != cudaSuccess) return SPECDEC_ECUDA;
  if (cudaMemcpyToSymbol(g_error_flags, &zero, sizeof zero) != cudaSuccess) return SPECDEC_ECUDA;
  *flags = v;
  return v ? SPECDEC_EDEVICE : SPECDEC_OK;
}

specdec_status specdec_verify_static(const void *target_logits, const void *draft_logits,
                                     const int32_t *draft_tokens, const float *u_accept,
                                     const float *u_resample, const float *temperature, int B,
                                     int K, int V, specdec_dtype dtype, int32_t *out_tokens,
                                     int32_t *out_num_accepted, void *stream) {
  specdec_status s = check_args(target_logits, draft_logits, draft_tokens, u_accept, u_resample,
                                temperature, B, K, V, dtype, out_tokens, out_num_accepted);
  if (s != SPECDEC_OK || B == 0) return s;
  const size_t need = specdec_workspace_bytes(B, K, V, dtype);
  if (need == 0) return SPECDEC_EINVAL;
  if (need > (size_t)SPECDEC_STATIC_SCRATCH_BYTES) return SPECDEC_ESIZE;
  void *scratch = nullptr;
  s = static_scratch_address(&scratch);
  if (s != SPECDEC_OK) return s;
  // Nothing in the scratch has to start at zero: every record the kernels read
  // (V-split partials, decisions, chunk sums, the arrival tickets that
  // k_row_stats zeroes) is written earlier in the same call.
  return run(target_logits, draft_logits, draft_tokens, u_accept, u_resample, temperature, B, K,
             V, dtype, scratch, (size_t)SPECDEC_STATIC_SCRATCH_BYTES, nullptr, out_tokens,
             out_num_accepted, static_cast<cudaStream_t>(stream));
}

void specdec_release(void) {
  std::lock_guard<std::mutex> lk(g_mu);
  int cur = 0;
  cudaGetDevice(&cur);
  for (auto *m : {&g_ws, &g_staging}) {
    for (auto &kv : *m) {
      if (kv.second.ptr) {
        cudaSetDevice(kv.first.first);
        cudaDeviceSynchronize();
        cudaFree(kv.second.ptr);
      }
    }
    m->clear();
  }
  cudaSetDevice(cur);
}

specdec_status specdec_get_error(void) {
  if (cudaDeviceSynchronize() != cudaSuccess) return SPECDEC_ECUDA;
  unsigned v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, g_error_flags, sizeof v) != cudaSuccess) return SPECDEC_ECUDA;
  if (cudaMemcpyToSymbol(g_error_flags, &zero, sizeof zero) != cudaSuccess) return SPECDEC_ECUDA;
  return v ? SPECDEC_EDEVICE : SPECDEC_OK;
}

const char *specdec_error_string(specdec_status s) { return specdec_status_string(s); }

specdec_status specdec_test_exp2(const float *a, float *y, int n, void *stream) {
  if (n < 0 || (n > 0 && (!a || !y))) return SPECDEC_EINVAL;
  if (n == 0) return SPECDEC_OK;
  const int threads = 256;
  const int blocks = (int)(((long long)(n + 1) / 2 + threads - 1) / threads);
  k_test_exp2<<<blocks, threads, 0, static_cast<cudaStream_t>(stream)>>>(a, y, n);
  return cudaGetLastError() == cudaSuccess ? SPECDEC_OK : SPECDEC_ECUDA;
}

specdec_status specdec_test_set_wait_fault(long long skip_tile, unsigned long long wait_ns) {
  if (skip_tile < -1 || wait_ns == 0) return SPECDEC_EINVAL;
  g_hook_skip_tile.store(skip_tile);
  g_hook_wait_ns.store(wait_ns);
  return SPECDEC_OK;
}

const char *specdec_status_string(specdec_status s) {
  switch (s) {
    case SPECDEC_OK: return "ok";
    case SPECDEC_EINVAL: return "invalid argument";
    case SPECDEC_ECUDA: return "CUDA runtime error";
    case SPECDEC_EDEVICE: return "invalid inputs flagged on the device";
    case SPECDEC_ESTATE: return "workspace would grow during stream capture";
    case SPECDEC_ESIZE: return "sizes need more than the fixed scratch of specdec_verify_static";
  }
  return "unknown status";
}

int specdec_kernel_count(void) { return KID_COUNT; }

const char *specdec_kernel_name(int i) {
  return (i >= 0 && i < KID_COUNT) ? kKernelNames[i] : nullptr;
}

uint64_t specdec_launch_count(int i) {
  std::lock_guard<std::mutex> lk(g_mu);
  return (i >= 0 && i < KID_COUNT) ? g_launches[i] : 0;
}

specdec_status specdec_profile_begin(int max_launches_per_kernel) {
  if (max_launches_per_kernel < 1) return SPECDEC_EINVAL;
  std::lock_guard<std::mutex> lk(g_mu);
  for (auto &v : g_prof.ev) {
    for (auto &e : v) {
      cudaEventDestroy(e.first);
      cudaEventDestroy(e.second);
    }
    v.clear();
    v.reserve(max_launches_per_kernel);
  }
  g_prof.max = max_launches_per_kernel;
  g_prof.on = true;
  return SPECDEC_OK;
}

specdec_status specdec_profile_end(double *ms_per_kernel, int *launches_per_kernel, int n) {
  std::lock_guard<std::mutex> lk(g_mu);
  g_prof.on = false;
  specdec_status st = SPECDEC_OK;
  for (int k = 0; k < KID_COUNT; ++k) {
    double tot = 0.0;
    int cnt = 0;
    for (auto &e : g_prof.ev[k]) {
      float ms = 0.f;
      if (cudaEventSynchronize(e.second) != cudaSuccess ||
          cudaEventElapsedTime(&ms, e.first, e.second) != cudaSuccess) {
        st = SPECDEC_ECUDA;
      } else {
        tot += ms;
        ++cnt;
      }
      cudaEventDestroy(e.first);
      cudaEventDestroy(e.second);
    }
    g_prof.ev[k].clear();
    if (k < n) {
      if (ms_per_kernel) ms_per_kernel[k] = tot;
      if (launches_per_kernel) launches_per_kernel[k] = cnt;
    }
  }
  return st;
}

}  // extern "C"
