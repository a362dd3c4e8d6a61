// libspecdec: the batched speculative-sampling verify step for B200 (sm_100a).
//
// What it computes is stated in include/specdec.h (accept with
// alpha(x) = min(1, p_target(x)/p_draft(x)), stop at the first rejection, draw
// from max(0, p - q)/Z or from the bonus row; speculative decoding blog
// "Speculative Decoding ... Llama 70B x2.4", section "The mathematical definition
// from Leviathan et al.").  This file is the B200 implementation: one
// persistent kernel, k_verify, runs the whole step.
//
//   Work units, claimed one at a time from a global counter in a fixed order:
//     statistics units  a few consecutive 16 KB tiles of one logit row; each
//                       consumer warp leaves the (max, sum of 2^((z-max)c)) of
//                       its share of the unit (split-V online softmax);
//     residual units    one chunk of the drawn row pair of a sequence (target /
//                       draft row n, or the target's bonus row K); each warp
//                       leaves the sum of r(v) = St * max(0, p - q) over its
//                       contiguous segment of the chunk.
//   The residual units of sequence b follow the statistics units of sequence
//   b + D, with the lag D sized so that b is normally decided (and its rows
//   still in L2) by the time they are claimed.
//   Tasks, run by the CTA that retires the last unit of a kind of a sequence
//   (per-sequence arrival counters):
//     ACCEPT  combine the row partials of the 2K+1 rows in fp64, gather
//             p_i(x_i) and q_i(x_i), test u*q < p on K lanes, first rejection
//             with __ballot_sync/__ffs, write the accepted prefix, publish the
//             drawn row pair (a release flag the residual units wait on);
//     DRAW    fp64 exclusive prefix over the segment sums, the segment holding
//             u*Z, a block-wide rescan of that one segment, the drawn token.
//
// Inside a CTA: one producer thread streams the tiles of its units with
// cp.async.bulk (the TMA bulk-copy engine; CTA-local copies, no multicast) into
// an NSTAGE-deep shared-memory ring and schedules everything else (claims,
// unit retirement, tasks) through the same ring; CW consumer warps fold tiles
// in registers and run units and tasks in ring order.  Every wait (ring
// barriers, the wait for a sequence to be decided, barriers among the consumer
// warps) is bounded in wall-clock time: a wait that runs out sets
// SPECDEC_ERR_TIMEOUT and the kernel winds down.  The grid is launched
// cooperatively, so every CTA that another one may wait for is resident.
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
#include <cstring>
#include <mutex>
#include <string>
#include <unordered_map>
#include <vector>

#include "specdec.h"

namespace {

constexpr double kLog2e = 1.4426950408889634073599246810019;  // log2(e)
constexpr unsigned FULL = 0xffffffffu;

// ---------------------------------------------------------------------------
// workspace records
// ---------------------------------------------------------------------------
struct __align__(16) Partial {  // one warp's share of a statistics unit
  double s;                     // sum of 2^((z - m) c)
  float m;                      // max
  uint32_t pad;
};
struct __align__(16) SeqInfo {  // written by a sequence's ACCEPT task
  double St, Sd;                // row sums (at the row max) of the drawn pair
  float Mt, Md;                 // row maxima of the drawn pair
  int n;                        // accepted length; -1 for an invalid sequence
  int pad;
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


// ---------------------------------------------------------------------------
// kernel geometry and synchronisation primitives
// ---------------------------------------------------------------------------
constexpr int CW = 8;               // consumer warps
constexpr int NTC = CW * 32;        // consumer threads
constexpr int NTS = NTC + 32;       // + one producer warp
constexpr int NSTAGE = 3;           // depth of the shared-memory ring
constexpr int NDONE = 8;            // units in flight per CTA (unit-done barriers)
constexpr int NTASKQ = NDONE + 1;   // queued tasks per CTA
constexpr int kCtasPerSm = 4;       // resident CTAs per SM the kernel is built for
constexpr int UR = 4;               // vectors per lane and row in a residual segment
constexpr int SV = 32 * UR;         // vectors per residual segment (one warp)
constexpr int RV = CW * SV;         // vectors per residual unit and row
constexpr int RMAX = 65;            // rows per sequence at K = 32
constexpr unsigned long long kWaitNs = 2000000000ull;  // a wait gives up after 2 s
constexpr unsigned kSuspendNs = 20000;  // longest sleep of one try_wait round

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
// non-blocking test of the phase of the given parity
__device__ __forceinline__ bool mbar_test(uint64_t *bar, unsigned parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
// bounded wait for the phase of the given parity; false when it ran out (the
// bound is wall-clock time, so it does not depend on how long a round sleeps)
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, unsigned parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = global_ns();
  do {
    if (mbar_try_wait(bar, parity)) return true;
  } while (global_ns() - t0 < kWaitNs);
  atomicOr(&g_error_flags, SPECDEC_ERR_TIMEOUT);
  return false;
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
// GPU-scope flag and counter operations between CTAs
__device__ __forceinline__ unsigned ld_acquire(const unsigned *p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_release(unsigned *p, unsigned v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ unsigned atom_add_acq_rel(unsigned *p, unsigned v) {
  unsigned old;
  asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;"
               : "=r"(old)
               : "l"(p), "r"(v)
               : "memory");
  return old;
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

// ---------------------------------------------------------------------------
// k_verify: the whole verify step in one persistent kernel
// ---------------------------------------------------------------------------
enum : int { E_STATS = 0, E_RES = 1, E_ACCEPT = 2, E_DRAW = 3, E_STOP = 4 };
enum : int { F_FIRST = 1, F_LAST = 2, F_HEAD = 4, F_TAIL = 8 };

// One ring entry, written by the producer before it arrives on the entry's
// "full" barrier (which orders these stores before the consumers' reads).
struct __align__(16) Entry {
  int kind, b, j, flags;     // j: row of the sequence (statistics) or chunk (residual)
  int nv, done, n, pad;      // nv: vectors in the tile; done: unit-done barrier; n: accepted length
  long long unit, pad2;      // statistics unit: its partials are part[unit * CW + warp]
  float chi, clo, thr, Mt;   // log2(e)/T of the sequence; residual: target row max
  float Md, lhi, llo, pad3;  // residual: draft row max, St/Sd = lhi + llo
};

struct Params {
  const void *target, *draft;
  const int32_t *tokens;
  const float *u_accept, *u_resample, *temperature;
  int B, K;
  long long V;
  int tpr, tps, spr, nru, lag;  // tiles per row, tiles per unit, units per row, residual units
  unsigned n_units;             // per sequence, lag in sequences; all units of the call
  Partial *part;                // [B, 2K+1, spr, CW]
  double *rpart;                // [B, nru, CW]   residual sums per segment
  SeqInfo *seq;                 // [B]
  unsigned *ctr;                // counters, see counter_words
  int32_t *out_tokens, *out_n;
  float *dbg_row_max;
  double *dbg_row_sum, *dbg_px, *dbg_qx, *dbg_Z;
};

// The counters are 32-bit words, all zero when a call starts and left zero
// when it ends (the last CTA to exit clears them): [0] the unit claim counter,
// [1] the CTA exit ticket, then per sequence b: [4+3b] statistics units
// retired, [5+3b] residual units retired, [6+3b] the "decided" flag.
constexpr int kCtrHead = 4;
__host__ __device__ __forceinline__ long long counter_words(long long B) {
  return kCtrHead + 3 * B;
}

// The work list: S statistics units per sequence (2K+1 rows x spr units),
// NR residual units per sequence; the residual units of sequence b come right
// after the statistics units of sequence b + D (or at the end of the list).
struct UnitRef {
  int kind;
  long long b, k;  // sequence; statistics unit within it, or residual chunk
};
__host__ __device__ __forceinline__ UnitRef decode_unit(long long u, long long B, long long S,
                                                      long long NR, long long D) {
  UnitRef r;
  const long long E1 = D * S, E2 = E1 + (B - D) * (S + NR);
  if (u < E1) {
    r.kind = E_STATS;
    r.b = u / S;
    r.k = u - r.b * S;
  } else if (u < E2) {
    const long long m = (u - E1) / (S + NR), k = (u - E1) - m * (S + NR);
    if (k < S) {
      r.kind = E_STATS;
      r.b = D + m;
      r.k = k;
    } else {
      r.kind = E_RES;
      r.b = m;
      r.k = k - S;
    }
  } else {
    const long long v = u - E2, m = v / NR;
    r.kind = E_RES;
    r.b = B - D + m;
    r.k = v - m * NR;
  }
  return r;
}

struct Smem {
  uint64_t full[NSTAGE], empty[NSTAGE], done[NDONE], cbar;
  Entry ent[NSTAGE];
  float sM[RMAX];
  double sS[RMAX];
  double scan[CW];
  double s_base;
  int abort, last_cta;
  int s_seg, s_y, s_lastpos;
};

// Barrier of the CW consumer warps on an mbarrier, bounded like every other
// wait; false when it ran out or the CTA is winding down (the caller stops).
__device__ __forceinline__ bool csync(Smem &sm, unsigned &cph) {
  if (*(volatile int *)&sm.abort) return false;
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(&sm.cbar);
  const bool ok = __all_sync(FULL, mbar_wait(&sm.cbar, cph));
  cph ^= 1u;
  if (!ok && (threadIdx.x & 31) == 0) atomicExch(&sm.abort, 1);
  return ok;
}

// Exclusive prefix sum of one double per consumer thread, in thread order
// (fixed association); `total` receives the sum over all of them.
__device__ __forceinline__ bool cta_excl_scan(double v, double &excl, double &total, Smem &sm,
                                              unsigned &cph) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  double incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const double y = __shfl_up_sync(FULL, incl, o);
    if (lane >= o) incl += y;
  }
  double ex = __shfl_up_sync(FULL, incl, 1);
  if (lane == 0) ex = 0.0;
  if (!csync(sm, cph)) return false;  // earlier readers of sm.scan are done
  if (lane == 31) sm.scan[warp] = incl;
  if (!csync(sm, cph)) return false;
  double base = 0.0, tot = 0.0;
#pragma unroll
  for (int w = 0; w < CW; ++w) {
    if (w < warp) base += sm.scan[w];
    tot += sm.scan[w];
  }
  excl = base + ex;
  total = tot;
  return true;
}

// The drawn row pair of a sequence: r = St * max(0, p - q) = max(0, e_t -
// (St/Sd) e_d) with e = 2^((z - m)c), or e_t for the bonus row.  The same
// inlined arithmetic serves the segment sums and the rescan, so both see
// bit-identical per-element weights.
struct DrawRow {
  float Mt, Md, lhi, llo;
  Scale c;
  bool bonus;
};
__device__ __forceinline__ float res_weight(float zt, float zd, const DrawRow &d) {
  const float et = ex2(scaled(zt - d.Mt, d.c));
  if (d.bonus) return et;
  const float ed = ex2(scaled(zd - d.Md, d.c));
  const float t1 = __fmaf_rn(-d.lhi, ed, et);
  const float t2 = __fmaf_rn(-d.llo, ed, t1);
  return t2 > 0.0f ? t2 : 0.0f;
}

// Element range [lo, hi) of residual segment s (of NS) of a row whose first
// 16-byte boundary is `head` elements in and which holds nvec whole vectors:
// segment s takes vectors [s*SV, (s+1)*SV); segment 0 also the head, the last
// segment also the scalar tail.
template <int VEC>
__device__ __forceinline__ void segment_range(int s, int NS, int head, long long nvec, long long V,
                                              long long &lo, long long &hi) {
  const long long a = (long long)s * SV, e = (long long)(s + 1) * SV;
  lo = (s == 0) ? 0 : head + (a < nvec ? a : nvec) * VEC;
  hi = (s == NS - 1) ? V : head + (e < nvec ? e : nvec) * VEC;
}

// fp64 probability of one logit: 2^((z - M) c) / S
template <typename T>
__device__ __forceinline__ double prob64(const T *row, long long v, float M, double S, double c64) {
  return exp2(((double)Dt<T>::load(row + v) - (double)M) * c64) / S;
}

// Inverse-CDF draw from max(0, p - q) entirely in fp64 by the consumer warps
// (contiguous ranges per thread, block scan, first crossing).  If the fp64
// residual is zero as well, draws from p (as the oracle does).  Used only when
// the fp32 residual weights have run out of range.  sm.s_y / sm.s_lastpos
// must hold INT_MAX / -1 on entry.
template <typename T>
__device__ __noinline__ bool draw_exact64(const T *pt, const T *pd, long long V, float Mt,
                                          double St, float Md, double Sd, double c64, double u,
                                          Smem &sm, unsigned &cph, int &y, double &Z) {
  const long long E = (V + NTC - 1) / NTC;
  const long long e0 = (long long)threadIdx.x * E < V ? (long long)threadIdx.x * E : V;
  const long long e1 = (e0 + E < V) ? e0 + E : V;
  double sr = 0.0, sp = 0.0;
  for (long long v = e0; v < e1; ++v) {
    const double p = prob64(pt, v, Mt, St, c64);
    const double q = prob64(pd, v, Md, Sd, c64);
    sr += (p - q > 0.0) ? p - q : 0.0;
    sp += p;
  }
  double xr, Zr, xp, Zp;
  if (!cta_excl_scan(sr, xr, Zr, sm, cph) || !cta_excl_scan(sp, xp, Zp, sm, cph)) return false;
  const bool use_p = !(Zr > 0.0);
  Z = use_p ? Zp : Zr;
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
      atomicMin(&sm.s_y, (int)v);
      found = true;
    }
  }
  if (last >= 0) atomicMax(&sm.s_lastpos, last);
  if (!csync(sm, cph)) return false;
  y = (sm.s_y != INT_MAX) ? sm.s_y : (sm.s_lastpos >= 0 ? sm.s_lastpos : 0);
  return true;
}

// ---- ACCEPT: decide sequence b (all consumer warps) ----
template <typename T>
__device__ __noinline__ void accept_task(const Params &p, int b, Smem &sm, unsigned &cph) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int K = p.K, R = 2 * K + 1;
  const long long V = p.V;
  const T *target = static_cast<const T *>(p.target);
  const T *draft = static_cast<const T *>(p.draft);
  const float Tf = __ldg(p.temperature + b);
  const bool t_ok = isfinite(Tf) && Tf > 0.0f;
  const double c64 = kLog2e / (double)Tf;
  // the gathers first, so their latency overlaps the combine
  int x = 0;
  bool x_ok = true;
  float zt_x = 0.f, zd_x = 0.f, u = 0.f;
  if (warp == 0 && lane < K) {
    x = __ldg(p.tokens + (long long)b * K + lane);
    x_ok = (x >= 0) && ((long long)x < V);
    u = __ldg(p.u_accept + (long long)b * K + lane);
    if (x_ok) {
      zt_x = Dt<T>::load(target + ((long long)b * (K + 1) + lane) * V + x);
      zd_x = Dt<T>::load(draft + ((long long)b * K + lane) * V + x);
    }
  }
  // combine the partials of each row in fp64 (written by other CTAs in this
  // call: read through L2)
  const int np = p.spr * CW;
  for (int r = warp; r < R; r += CW) {
    const Partial *P = p.part + ((long long)b * R + r) * np;
    constexpr int PL = 4;  // partials per lane kept in registers
    double ps[PL];
    float pm[PL];
    float m = -INFINITY;
#pragma unroll
    for (int k = 0; k < PL; ++k) {
      const int s = lane + 32 * k;
      ps[k] = 0.0;
      pm[k] = -INFINITY;
      if (s < np) {
        ps[k] = __ldcg(&P[s].s);
        pm[k] = __ldcg(&P[s].m);
      }
      m = fmax_nan(m, pm[k]);
    }
    for (int s = lane + 32 * PL; s < np; s += 32) m = fmax_nan(m, __ldcg(&P[s].m));
    m = warp_max_nan(m);
    double acc = 0.0;
#pragma unroll
    for (int k = 0; k < PL; ++k)
      acc += (pm[k] == -INFINITY) ? ps[k] : ps[k] * exp2(((double)pm[k] - (double)m) * c64);
    for (int s = lane + 32 * PL; s < np; s += 32) {
      const float ms = __ldcg(&P[s].m);
      const double ss = __ldcg(&P[s].s);
      acc += (ms == -INFINITY) ? ss : ss * exp2(((double)ms - (double)m) * c64);
    }
    acc = warp_sum(acc);
    if (lane == 0) {
      sm.sM[r] = m;
      sm.sS[r] = acc;
      if (p.dbg_row_max) p.dbg_row_max[(long long)b * R + r] = m;
      if (p.dbg_row_sum) p.dbg_row_sum[(long long)b * R + r] = acc;
    }
  }
  if (!csync(sm, cph)) return;

  if (warp == 0) {
    // a timed-out wait in this call (or an earlier, unacknowledged one) makes
    // every sequence invalid rather than silently wrong
    const bool timed_out = (*(volatile unsigned *)&g_error_flags & SPECDEC_ERR_TIMEOUT) != 0;
    bool rows_ok = true;
    for (int r = lane; r < R; r += 32)
      rows_ok = rows_ok && isfinite(sm.sM[r]) && isfinite(sm.sS[r]) && sm.sS[r] > 0.0;
    rows_ok = __all_sync(FULL, rows_ok) && !timed_out;
    bool acc_i = false;
    double pp = 0.0, qq = 0.0;
    if (lane < K && x_ok && rows_ok && t_ok) {
      pp = exp2(((double)zt_x - (double)sm.sM[lane]) * c64) / sm.sS[lane];
      qq = exp2(((double)zd_x - (double)sm.sM[K + 1 + lane]) * c64) / sm.sS[K + 1 + lane];
      acc_i = (double)u * qq < pp;
    }
    const unsigned bad_x = __ballot_sync(FULL, lane < K && !x_ok);
    const unsigned accm = __ballot_sync(FULL, lane < K && acc_i);
    const bool seq_ok = t_ok && rows_ok && bad_x == 0;
    const unsigned kmask = (K >= 32) ? FULL : ((1u << K) - 1u);
    const unsigned rej = ~accm & kmask;
    const int n = seq_ok ? (rej ? __ffs(rej) - 1 : K) : -1;
    int32_t *ot = p.out_tokens + (long long)b * (K + 1);
    if (!seq_ok) {
      for (int i = lane; i <= K; i += 32) ot[i] = -1;
    } else {
      if (lane < n) ot[lane] = x;
      for (int i = n + 1 + lane; i <= K; i += 32) ot[i] = -1;
      if (lane < K && lane <= n) {
        if (p.dbg_px) p.dbg_px[(long long)b * K + lane] = pp;
        if (p.dbg_qx) p.dbg_qx[(long long)b * K + lane] = qq;
      }
    }
    if (lane == 0) {
      p.out_n[b] = n;
      if (!seq_ok) {
        unsigned f = 0;
        if (!t_ok) f |= SPECDEC_ERR_TEMPERATURE;
        if (bad_x) f |= SPECDEC_ERR_TOKEN;
        if (!rows_ok && !timed_out) f |= SPECDEC_ERR_LOGITS;
        if (f) atomicOr(&g_error_flags, f);
      }
      SeqInfo si;
      si.n = n;
      si.pad = 0;
      si.Mt = n >= 0 ? sm.sM[n] : 0.f;
      si.St = n >= 0 ? sm.sS[n] : 1.0;
      si.Md = (n >= 0 && n < K) ? sm.sM[K + 1 + n] : 0.f;
      si.Sd = (n >= 0 && n < K) ? sm.sS[K + 1 + n] : 1.0;
      p.seq[b] = si;
      // publish: the residual units of b wait for this flag
      st_release(p.ctr + kCtrHead + 3LL * b + 2, 1u);
    }
  }
  csync(sm, cph);  // sM / sS are free again
}

// ---- residual unit: one warp's segment sum of the drawn row pair ----
template <typename T>
__device__ __forceinline__ double residual_sum(const Params &p, int b, int chunk, int n,
                                               const DrawRow &d) {
  constexpr int VEC = Dt<T>::VEC;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (n < 0) return 0.0;
  const int K = p.K;
  const long long V = p.V;
  const T *pt = static_cast<const T *>(p.target) + ((long long)b * (K + 1) + n) * V;
  const T *pd = d.bonus ? pt : static_cast<const T *>(p.draft) + ((long long)b * K + n) * V;
  const int head = row_head(pt, V);
  const long long nvec = (V - head) / VEC;
  const int NS = p.nru * CW;
  const int s = chunk * CW + warp;
  float rs = 0.f;
  if (d.bonus || row_head(pd, V) == head) {
    const uint4 *vt = reinterpret_cast<const uint4 *>(pt + head);
    const uint4 *vd = reinterpret_cast<const uint4 *>(pd + head);
    const long long v0 = (long long)s * SV;
    uint4 at[UR], ad[UR];
#pragma unroll
    for (int k = 0; k < UR; ++k) {
      const long long vi = v0 + k * 32 + lane;
      at[k] = vi < nvec ? __ldg(vt + vi) : make_uint4(0, 0, 0, 0);
      ad[k] = (vi < nvec && !d.bonus) ? __ldg(vd + vi) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int k = 0; k < UR; ++k) {
      if (v0 + k * 32 + lane < nvec) {
        float xt[VEC], xd[VEC];
        Dt<T>::unpack(at[k], xt);
        Dt<T>::unpack(ad[k], xd);
#pragma unroll
        for (int e = 0; e < VEC; ++e) rs += res_weight(xt[e], xd[e], d);
      }
    }
    if (s == 0 && lane < head)
      rs += res_weight(Dt<T>::load(pt + lane), d.bonus ? 0.f : Dt<T>::load(pd + lane), d);
    if (s == NS - 1) {
      const long long tt = head + nvec * VEC + lane;
      if (lane < VEC && tt < V)
        rs += res_weight(Dt<T>::load(pt + tt), d.bonus ? 0.f : Dt<T>::load(pd + tt), d);
    }
  } else {  // rows of different alignment: scalar loads over the segment
    long long lo, hi;
    segment_range<VEC>(s, NS, head, nvec, V, lo, hi);
    for (long long v = lo + lane; v < hi; v += 32)
      rs += res_weight(Dt<T>::load(pt + v), Dt<T>::load(pd + v), d);
  }
  return warp_sum((double)rs);
}

// ---- DRAW: the drawn token of sequence b (all consumer warps) ----
template <typename T>
__device__ __noinline__ void draw_task(const Params &p, int b, Smem &sm, unsigned &cph) {
  constexpr int VEC = Dt<T>::VEC;
  constexpr int EMAX = (SV * VEC + 2 * VEC + NTC - 1) / NTC;  // rescan elements per thread
  const int tid = threadIdx.x;
  const int K = p.K;
  const long long V = p.V;
  const SeqInfo *si = p.seq + b;
  const int n = __ldcg(&si->n);
  if (n < 0) return;  // invalid sequence: its outputs are written (the same n for all warps)
  const bool bonus = (n == K);
  const double St = __ldcg(&si->St), Sd = bonus ? 1.0 : __ldcg(&si->Sd);
  const float Mt = __ldcg(&si->Mt), Md = bonus ? 0.f : __ldcg(&si->Md);
  const double c64 = kLog2e / (double)__ldg(p.temperature + b);
  DrawRow d;
  d.bonus = bonus;
  d.Mt = Mt;
  d.Md = Md;
  d.c = make_scale(c64);
  const double lam = bonus ? 0.0 : St / Sd;
  d.lhi = (float)lam;
  d.llo = (float)(lam - (double)d.lhi);
  const T *pt = static_cast<const T *>(p.target) + ((long long)b * (K + 1) + n) * V;
  const T *pd = bonus ? pt : static_cast<const T *>(p.draft) + ((long long)b * K + n) * V;
  const int head = row_head(pt, V);
  const long long nvec = (V - head) / VEC;
  const int NS = p.nru * CW;
  const double *rp = p.rpart + (long long)b * NS;
  const double ures = (double)__ldg(p.u_resample + b);
  int32_t *oty = p.out_tokens + (long long)b * (K + 1) + n;

  // fp64 prefix over the segment sums (contiguous segments per thread)
  const int cper = (NS + NTC - 1) / NTC;
  const int c0 = tid * cper < NS ? tid * cper : NS;
  const int c1 = c0 + cper < NS ? c0 + cper : NS;
  double my = 0.0;
  for (int c2 = c0; c2 < c1; ++c2) my += __ldcg(rp + c2);
  if (tid == 0) {
    sm.s_seg = INT_MAX;
    sm.s_y = INT_MAX;
    sm.s_lastpos = -1;
    sm.s_base = -1.0;  // < 0 selects the "last positive element" rule
  }
  double cexcl, Z;
  if (!cta_excl_scan(my, cexcl, Z, sm, cph)) return;
  if (!bonus && !(Z >= ldexp(St, -64))) {
    // the fp32 weights ran out of range: redo the draw in fp64
    int y;
    double Zx;
    if (!draw_exact64<T>(pt, pd, V, Mt, St, Md, Sd, c64, ures, sm, cph, y, Zx)) return;
    if (tid == 0) {
      *oty = y;
      if (p.dbg_Z) p.dbg_Z[b] = Zx;
    }
    csync(sm, cph);
    return;
  }
  const double t = ures * Z;
  {
    double C = cexcl;
    for (int c2 = c0; c2 < c1; ++c2) {
      const double v = __ldcg(rp + c2);
      if (C <= t && t < C + v) {
        atomicMin(&sm.s_seg, c2);
        break;
      }
      C += v;
    }
  }
  if (!csync(sm, cph)) return;
  if (tid == 0) {
    if (sm.s_seg == INT_MAX) {  // rounding left t at or past the total
      int cs = 0;
      for (int c2 = NS - 1; c2 >= 0; --c2)
        if (__ldcg(rp + c2) > 0.0) {
          cs = c2;
          break;
        }
      sm.s_seg = cs;
    }
    if (p.dbg_Z) p.dbg_Z[b] = Z / St;
  }
  if (!csync(sm, cph)) return;
  const int s = sm.s_seg;
  // the owner of the chosen segment publishes its exclusive prefix
  if (s >= c0 && s < c1) {
    double C = cexcl;
    for (int c2 = c0; c2 < s; ++c2) C += __ldcg(rp + c2);
    const double v = __ldcg(rp + s);
    if (C <= t && t < C + v) sm.s_base = C;
  }
  if (!csync(sm, cph)) return;

  // rescan of the chosen segment: contiguous elements per thread, in registers
  long long lo, hi;
  segment_range<VEC>(s, NS, head, nvec, V, lo, hi);
  const long long L = hi - lo;
  const long long E = (L + NTC - 1) / NTC;
  const long long e0 = lo + (long long)tid * E < hi ? lo + (long long)tid * E : hi;
  const long long e1 = (e0 + E < hi) ? e0 + E : hi;
  float w[EMAX];
#pragma unroll
  for (int k = 0; k < EMAX; ++k) {
    const long long v = e0 + k;
    w[k] = (v < e1) ? res_weight(Dt<T>::load(pt + v), bonus ? 0.f : Dt<T>::load(pd + v), d)
                    : 0.0f;
  }
  double mysum = 0.0;
  int lastpos = -1;
#pragma unroll
  for (int k = 0; k < EMAX; ++k) {
    mysum += (double)w[k];
    if (w[k] > 0.0f) lastpos = (int)(e0 + k);
  }
  double excl, ctot;
  if (!cta_excl_scan(mysum, excl, ctot, sm, cph)) return;
  if (lastpos >= 0) atomicMax(&sm.s_lastpos, lastpos);
  const double base = sm.s_base;
  if (base >= 0.0) {
    double C = base + excl;
#pragma unroll
    for (int k = 0; k < EMAX; ++k) {
      if (e0 + k < e1) {
        C += (double)w[k];
        if (C > t) {
          atomicMin(&sm.s_y, (int)(e0 + k));
          break;
        }
      }
    }
  }
  if (!csync(sm, cph)) return;
  if (tid == 0) *oty = (sm.s_y != INT_MAX) ? sm.s_y : (sm.s_lastpos >= 0 ? sm.s_lastpos : (int)lo);
  csync(sm, cph);  // the shared draw state is free again
}

// ---- the producer thread: claims units, streams tiles, schedules tasks ----
template <typename T, int U>
__device__ __noinline__ void producer(const Params &p, Smem &sm, unsigned char *ring) {
  constexpr int VEC = Dt<T>::VEC;
  constexpr long long TV = (long long)NTC * U;  // vectors per tile
  constexpr unsigned TILE_BYTES = (unsigned)TV * 16u;
  const T *target = static_cast<const T *>(p.target);
  const T *draft = static_cast<const T *>(p.draft);
  const int K = p.K, R = 2 * K + 1;
  const long long V = p.V, B = p.B;
  const long long S = (long long)R * p.spr, NR = p.nru;
  unsigned *cnt = p.ctr + kCtrHead;

  int st = 0;       // ring slot of the next entry
  unsigned ph = 0;  // its phase parity
  bool copy_last[NSTAGE];     // the last entry pushed into a slot was a copy ...
  unsigned copy_par[NSTAGE];  // ... of this phase parity
  for (int i = 0; i < NSTAGE; ++i) copy_last[i] = false, copy_par[i] = 0;
  // units pushed and not yet retired (FIFO), with their unit-done barriers
  int pk[NDONE], pb[NDONE], pslot[NDONE];
  unsigned ppar[NDONE], duse[NDONE];
  for (int i = 0; i < NDONE; ++i) duse[i] = 0;
  int phead = 0, npend = 0, dnext = 0;
  // tasks waiting for a ring slot (FIFO)
  int tk[NTASKQ], tb[NTASKQ];
  int thead = 0, ntask = 0;
  bool abort = false;

  auto advance = [&]() {
    if (++st == NSTAGE) {
      st = 0;
      ph ^= 1u;
    }
  };
  auto acquire = [&]() -> bool {  // the next ring slot is free (bounded wait)
    if (abort || *(volatile int *)&sm.abort) {
      abort = true;
      return false;
    }
    if (!mbar_wait(&sm.empty[st], ph ^ 1u)) {
      abort = true;
      return false;
    }
    return true;
  };
  auto push_tasks = [&]() -> bool {
    while (ntask > 0) {
      if (!acquire()) return false;
      Entry &e = sm.ent[st];
      e.kind = tk[thead];
      e.b = tb[thead];
      mbar_arrive(&sm.full[st]);
      copy_last[st] = false;
      advance();
      thead = (thead + 1) % NTASKQ;
      --ntask;
    }
    return true;
  };
  // Retire the units the consumers have finished, oldest first (blocking for
  // the oldest if asked): one arrival on the sequence's counter each; the unit
  // that completes a sequence's statistics (residual sums) queues its ACCEPT
  // (DRAW) task.
  auto retire = [&](bool block) {
    while (npend > 0 && !abort) {
      const int i = phead;
      bool ok;
      if (block) {
        ok = mbar_wait(&sm.done[pslot[i]], ppar[i]);
        block = false;
        if (!ok) {
          abort = true;
          return;
        }
      } else {
        ok = mbar_test(&sm.done[pslot[i]], ppar[i]);
      }
      if (!ok) return;
      phead = (phead + 1) % NDONE;
      --npend;
      const long long b = pb[i];
      const bool stats = pk[i] == E_STATS;
      const unsigned need = stats ? (unsigned)S : (unsigned)NR;
      if (atom_add_acq_rel(cnt + 3 * b + (stats ? 0 : 1), 1u) + 1u == need) {
        const int q = (thead + ntask) % NTASKQ;
        tk[q] = stats ? E_ACCEPT : E_DRAW;
        tb[q] = (int)b;
        ++ntask;
      }
    }
  };
  // wait until sequence b is decided, retiring units and pushing tasks meanwhile
  auto wait_ready = [&](long long b) -> bool {
    const unsigned *flag = cnt + 3 * b + 2;
    if (ld_acquire(flag)) return true;
    const unsigned long long t0 = global_ns();
    for (;;) {
      retire(false);
      if (!push_tasks()) return false;
      if (ld_acquire(flag)) return true;
      if (abort || (*(volatile unsigned *)&g_error_flags & SPECDEC_ERR_TIMEOUT)) {
        abort = true;
        return false;
      }
      if (global_ns() - t0 > kWaitNs) {
        atomicOr(&g_error_flags, SPECDEC_ERR_TIMEOUT);
        abort = true;
        return false;
      }
      __nanosleep(128);
    }
  };

  for (;;) {
    retire(false);
    if (!push_tasks() || abort) break;
    const unsigned u = atomicAdd(p.ctr, 1u);
    if (u >= p.n_units) break;
    const UnitRef un = decode_unit(u, B, S, NR, p.lag);
    while (npend == NDONE && !abort) {  // a unit-done barrier for this unit
      retire(true);
      push_tasks();
    }
    if (abort) break;
    const int ds = dnext;
    dnext = (dnext + 1) % NDONE;
    const unsigned dpar = duse[ds] & 1u;
    ++duse[ds];
    const long long b = un.b;
    const Scale c = make_scale(kLog2e / (double)__ldg(p.temperature + b));
    if (un.kind == E_STATS) {
      const int j = (int)(un.k / p.spr), seg = (int)(un.k - (long long)j * p.spr);
      const T *row = j <= K ? target + (b * (K + 1) + j) * V : draft + (b * K + (j - K - 1)) * V;
      const int head = row_head(row, V);
      const long long nvec = (V - head) / VEC;
      const uint4 *pv = reinterpret_cast<const uint4 *>(row + head);
      const int t0 = seg * p.tps, t1 = (t0 + p.tps < p.tpr) ? t0 + p.tps : p.tpr;
      for (int t = t0; t < t1; ++t) {
        if (!acquire()) break;
        const long long v0 = (long long)t * TV;
        long long nv = nvec - v0;
        nv = nv < 0 ? 0 : (nv > TV ? TV : nv);
        Entry &e = sm.ent[st];
        e.kind = E_STATS;
        e.b = (int)b;
        e.j = j;
        e.flags = (t == t0 ? F_FIRST : 0) | (t == t1 - 1 ? F_LAST : 0) |
                  ((t == t0 && seg == 0) ? F_HEAD : 0) | ((t == t1 - 1 && t1 == p.tpr) ? F_TAIL : 0);
        e.nv = (int)nv;
        e.done = ds;
        e.unit = (b * R + j) * p.spr + seg;
        e.chi = c.hi;
        e.clo = c.lo;
        e.thr = 64.0f / c.hi;
        if (nv > 0) {
          const unsigned bytes = (unsigned)nv * 16u;
          mbar_arrive_tx(&sm.full[st], bytes);
          bulk_load(ring + (size_t)st * TILE_BYTES, pv + v0, bytes, &sm.full[st]);
          copy_last[st] = true;
          copy_par[st] = ph;
        } else {
          mbar_arrive(&sm.full[st]);
          copy_last[st] = false;
        }
        advance();
      }
      if (abort) break;
    } else {
      if (!wait_ready(b)) break;
      const SeqInfo *si = p.seq + b;
      const int n = __ldcg(&si->n);
      if (!acquire()) break;
      Entry &e = sm.ent[st];
      e.kind = E_RES;
      e.b = (int)b;
      e.j = (int)un.k;
      e.done = ds;
      e.n = n;
      e.chi = c.hi;
      e.clo = c.lo;
      e.Mt = e.Md = e.lhi = e.llo = 0.f;
      if (n >= 0) {
        const bool bonus = (n == K);
        e.Mt = __ldcg(&si->Mt);
        e.Md = bonus ? 0.f : __ldcg(&si->Md);
        const double lam = bonus ? 0.0 : __ldcg(&si->St) / __ldcg(&si->Sd);
        e.lhi = (float)lam;
        e.llo = (float)(lam - (double)e.lhi);
      }
      mbar_arrive(&sm.full[st]);
      copy_last[st] = false;
      advance();
    }
    const int q = (phead + npend) % NDONE;
    pk[q] = un.kind;
    pb[q] = (int)b;
    pslot[q] = ds;
    ppar[q] = dpar;
    ++npend;
  }
  // no more units: retire what is in flight, push the tasks that frees, stop
  while (npend > 0 && !abort) {
    retire(true);
    if (!push_tasks()) break;
  }
  if (!abort && push_tasks() && acquire()) {
    sm.ent[st].kind = E_STOP;
    mbar_arrive(&sm.full[st]);
    copy_last[st] = false;
    advance();
  }
  if (abort) {
    // the CTA must not retire with copies in flight
    atomicExch(&sm.abort, 1);
    for (int i = 0; i < NSTAGE; ++i)
      if (copy_last[i]) mbar_wait(&sm.full[i], copy_par[i]);
  }
}

// ---- the consumer warps: run the ring's entries in order ----
template <typename T, int U>
__device__ __forceinline__ void consumers(const Params &p, Smem &sm, const unsigned char *ring) {
  constexpr int VEC = Dt<T>::VEC;
  constexpr int TV = NTC * U;
  constexpr unsigned TILE_BYTES = (unsigned)TV * 16u;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int K = p.K;
  const long long V = p.V;
  unsigned ph = 0, cph = 0;
  int st = 0;
  RunStat q;
  runstat_init(q);
  Scale c;
  c.hi = 1.0f;
  c.lo = 1e-30f;
  float thr = 64.0f;
  for (;;) {
    if (*(volatile int *)&sm.abort) break;
    if (!__all_sync(FULL, mbar_wait(&sm.full[st], ph))) {
      if (lane == 0) atomicExch(&sm.abort, 1);
      break;
    }
    const Entry &e = sm.ent[st];
    const int kind = e.kind;
    if (kind == E_STATS) {
      const int flags = e.flags, nv = e.nv;
      if (flags & F_FIRST) {
        runstat_init(q);
        c.hi = e.chi;
        c.lo = e.clo;
        thr = e.thr;
      }
      // this warp's contiguous quarter of the tile, lanes on consecutive vectors
      const uint4 *tile = reinterpret_cast<const uint4 *>(ring + (size_t)st * TILE_BYTES);
      const int base = warp * 32 * U + lane;
      uint4 v[U];
      if (nv == TV) {
#pragma unroll
        for (int k = 0; k < U; ++k) v[k] = tile[base + k * 32];
      } else {
#pragma unroll
        for (int k = 0; k < U; ++k) {
          const int vi = base + k * 32;
          v[k] = vi < nv ? tile[vi] : Dt<T>::neg_inf();
        }
      }
      const int b = e.b, j = e.j, ds = e.done;
      const long long unit = e.unit;
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.empty[st]);
#pragma unroll
      for (int k = 0; k < U; ++k) vec_fold<T>(v[k], q, c, thr);
      if ((flags & (F_HEAD | F_TAIL)) && warp == 0) {  // the row's scalar head / tail
        const T *row = j <= K ? static_cast<const T *>(p.target) + ((long long)b * (K + 1) + j) * V
                              : static_cast<const T *>(p.draft) +
                                    ((long long)b * K + (j - K - 1)) * V;
        const int head = row_head(row, V);
        if ((flags & F_HEAD) && lane < head) elem_fold(Dt<T>::load(row + lane), q, c, thr);
        if (flags & F_TAIL) {
          const long long tt = head + ((V - head) / VEC) * VEC + lane;
          if (lane < VEC && tt < V) elem_fold(Dt<T>::load(row + tt), q, c, thr);
        }
      }
      if (flags & F_LAST) {  // this warp's partial of the unit
        const float m = q.mt;
        const float sl = runstat_sum_at_max(q, c);
        const float mw = warp_max_nan(m);
        double sw = (m == -INFINITY) ? 0.0 : (double)sl * (double)ex2(scaled(m - mw, c));
        sw = warp_sum(sw);
        if (lane == 0) {
          Partial o;
          o.s = sw;
          o.m = mw;
          o.pad = 0;
          p.part[unit * CW + warp] = o;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.done[ds]);
      }
    } else {
      const int b = e.b, j = e.j, ds = e.done, n = e.n;
      DrawRow d;
      d.Mt = e.Mt;
      d.Md = e.Md;
      d.lhi = e.lhi;
      d.llo = e.llo;
      d.c.hi = e.chi;
      d.c.lo = e.clo;
      d.bonus = (n == K);
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.empty[st]);
      if (kind == E_STOP) break;
      if (kind == E_RES) {
        const double r = residual_sum<T>(p, b, j, n, d);
        if (lane == 0) p.rpart[((long long)b * p.nru + j) * CW + warp] = r;
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.done[ds]);
      } else if (kind == E_ACCEPT) {
        accept_task<T>(p, b, sm, cph);
      } else {
        draw_task<T>(p, b, sm, cph);
      }
    }
    if (++st == NSTAGE) {
      st = 0;
      ph ^= 1u;
    }
  }
}

template <typename T, int U>
__global__ void __launch_bounds__(NTS, kCtasPerSm) k_verify(const __grid_constant__ Params p) {
  extern __shared__ __align__(128) unsigned char ring[];  // NSTAGE tiles
  __shared__ Smem sm;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < NSTAGE; ++i) {
      mbar_init(&sm.full[i], 1);
      mbar_init(&sm.empty[i], CW);
    }
    for (int i = 0; i < NDONE; ++i) mbar_init(&sm.done[i], CW);
    mbar_init(&sm.cbar, CW);
    sm.abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  if (warp == CW) {
    if (lane == 0) producer<T, U>(p, sm, ring);
    __syncwarp();
  } else {
    consumers<T, U>(p, sm, ring);
  }
  __syncthreads();
  // the last CTA to leave clears the counters for the next call (and, if a
  // wait ran out, invalidates every output of this one)
  if (threadIdx.x == 0) {
    __threadfence();
    sm.last_cta = (atomicAdd(p.ctr + 1, 1u) == gridDim.x - 1) ? 1 : 0;
  }
  __syncthreads();
  if (sm.last_cta) {
    __threadfence();
    if (*(volatile unsigned *)&g_error_flags & SPECDEC_ERR_TIMEOUT) {
      const long long nt = (long long)p.B * (p.K + 1);
      for (long long i = threadIdx.x; i < nt; i += blockDim.x) p.out_tokens[i] = -1;
      for (long long i = threadIdx.x; i < p.B; i += blockDim.x) p.out_n[i] = -1;
    }
    const long long nw = counter_words(p.B);
    for (long long i = threadIdx.x; i < nw; i += blockDim.x) p.ctr[i] = 0u;
  }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
enum KernelId { KID_VERIFY = 0, KID_COUNT = 1 };
const char *kKernelNames[KID_COUNT] = {"k_verify"};

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
std::unordered_map<int, DeviceBuf> g_ws;       // workspace per device
std::unordered_map<int, DeviceBuf> g_staging;  // end-to-end staging per device

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// The counter region of a workspace of W bytes: its first bytes, sized by W
// alone, so that every call on one workspace finds its counters where the
// previous calls left them zero, whatever their sizes.  A call on B sequences
// uses 4 + 3B words of it; every call needs at least 384 B of records per
// sequence, so a workspace that holds a call's records also holds its
// counters.
inline size_t counter_region(size_t W) { return align256(64 + W / 16); }
// bytes of records a workspace of W bytes holds after its counter region
inline size_t record_capacity(size_t W) {
  const size_t c = counter_region(W);
  return W > c ? W - c : 0;
}

#ifndef SPECDEC_TILES_PER_UNIT
#define SPECDEC_TILES_PER_UNIT 0  // 0: chosen from the sizes
#endif
#ifndef SPECDEC_LAG_TILES_PER_CTA
#define SPECDEC_LAG_TILES_PER_CTA 10
#endif

struct Plan {
  int esize, vec, U, tpr, tps, spr, nru;
  long long rows, tiles;
  unsigned n_units;
  size_t off_part, off_rpart, off_seq, records;  // inside the record region
  size_t total;                                  // smallest workspace that holds them
};

int num_sms() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

// Work decomposition for these sizes; a pure function of the sizes and the SM
// count, so repeated calls reduce in the same order (bit-reproducible).
bool make_plan(int B, int K, int V, specdec_dtype dtype, int sms, Plan &pl) {
  if (B < 0 || K < 1 || K > 32 || V < 1) return false;
  if (dtype != SPECDEC_F32 && dtype != SPECDEC_BF16) return false;
  if ((long long)B * (K + 1) * (long long)V > (1LL << 56)) return false;
  pl.esize = dtype == SPECDEC_BF16 ? 2 : 4;
  pl.vec = 16 / pl.esize;
  const int R = 2 * K + 1;
  pl.rows = (long long)B * R;
  const long long nvec_max = ((long long)V + pl.vec - 1) / pl.vec;
  const long long cap = (long long)kCtasPerSm * sms;
  // tiles of 4 vectors per consumer thread (16 KB); 1 vector per thread when
  // 16 KB tiles would leave SMs idle (single-sequence batches)
  long long tpr = (nvec_max + NTC * 4 - 1) / (NTC * 4);
  pl.U = 4;
  if (pl.rows * tpr < 2 * cap) {
    pl.U = 1;
    tpr = (nvec_max + NTC - 1) / NTC;
  }
  if (tpr < 1) tpr = 1;
  if (tpr > INT_MAX / 4) return false;
  pl.tpr = (int)tpr;
  pl.tiles = pl.rows * tpr;
  int tps = SPECDEC_TILES_PER_UNIT;
  if (tps <= 0) tps = (pl.tiles >= 16 * cap) ? 2 : 1;
  if (tps > pl.tpr) tps = pl.tpr;
  pl.tps = tps;
  pl.spr = (pl.tpr + tps - 1) / tps;
  const long long nru = (nvec_max + RV - 1) / RV;
  pl.nru = (int)(nru > 0 ? nru : 1);
  const long long units = (long long)B * ((long long)R * pl.spr + pl.nru);
  if (units >= (1LL << 31)) return false;
  pl.n_units = (unsigned)units;
  size_t off = 0;
  pl.off_part = off;
  off = align256(off + sizeof(Partial) * (size_t)pl.rows * pl.spr * CW);
  pl.off_rpart = off;
  off = align256(off + sizeof(double) * (size_t)B * pl.nru * CW);
  pl.off_seq = off;
  off = align256(off + sizeof(SeqInfo) * (size_t)B);
  pl.records = off;
  size_t W = align256(off + off / 15 + 512);
  while (record_capacity(W) < off) W += 256;
  pl.total = W;
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
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, threads, smem) != cudaSuccess)
    n = 0;
  cache[key] = n;
  return n;
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

// One cooperative launch: every CTA is resident for the whole kernel, which
// the waits between CTAs rely on for progress.
template <typename T, int U>
specdec_status launch_verify(Params prm, const Plan &pl, cudaStream_t st) {
  auto kern = k_verify<T, U>;
  const size_t smem = (size_t)NSTAGE * NTC * U * 16;
  const int per_sm = resident_ctas(kern, NTS, smem);
  if (per_sm < 1) return SPECDEC_ECUDA;
  const long long cap = (long long)per_sm * num_sms();
  const unsigned grid = (unsigned)((long long)pl.n_units < cap ? (long long)pl.n_units : cap);
  // lag of the residual units behind the statistics units, in sequences: about
  // SPECDEC_LAG_TILES_PER_CTA tiles per CTA of the grid
  const long long tiles_per_seq = (long long)(2 * prm.K + 1) * pl.tpr;
  long long lag = ((long long)SPECDEC_LAG_TILES_PER_CTA * grid + tiles_per_seq - 1) / tiles_per_seq;
  if (lag < 1) lag = 1;
  if (lag > prm.B) lag = prm.B;
  prm.lag = (int)lag;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(NTS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  LaunchTimer lt(KID_VERIFY, st);
  return cudaLaunchKernelEx(&cfg, kern, prm) == cudaSuccess ? SPECDEC_OK : SPECDEC_ECUDA;
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

// ws / ws_bytes: a workspace whose counter region (counter_region(ws_bytes)
// first bytes) is zero, as every call leaves it
specdec_status run(const void *tg, const void *dr, const int32_t *tok, const float *ua,
                   const float *ur, const float *temp, int B, int K, int V, specdec_dtype dtype,
                   void *ws, size_t ws_bytes, const specdec_debug *dbg, int32_t *ot, int32_t *on,
                   cudaStream_t st) {
  specdec_status s = check_args(tg, dr, tok, ua, ur, temp, B, K, V, dtype, ot, on);
  if (s != SPECDEC_OK || B == 0) return s;
  Plan pl;
  if (!make_plan(B, K, V, dtype, num_sms(), pl)) return SPECDEC_EINVAL;
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255) || record_capacity(ws_bytes) < pl.records)
    return SPECDEC_EINVAL;
  char *rec = static_cast<char *>(ws) + counter_region(ws_bytes);
  Params prm;
  prm.target = tg;
  prm.draft = dr;
  prm.tokens = tok;
  prm.u_accept = ua;
  prm.u_resample = ur;
  prm.temperature = temp;
  prm.B = B;
  prm.K = K;
  prm.V = V;
  prm.tpr = pl.tpr;
  prm.tps = pl.tps;
  prm.spr = pl.spr;
  prm.nru = pl.nru;
  prm.lag = 1;
  prm.n_units = pl.n_units;
  prm.part = reinterpret_cast<Partial *>(rec + pl.off_part);
  prm.rpart = reinterpret_cast<double *>(rec + pl.off_rpart);
  prm.seq = reinterpret_cast<SeqInfo *>(rec + pl.off_seq);
  prm.ctr = static_cast<unsigned *>(ws);
  prm.out_tokens = ot;
  prm.out_n = on;
  prm.dbg_row_max = dbg ? dbg->row_max : nullptr;
  prm.dbg_row_sum = dbg ? dbg->row_sum : nullptr;
  prm.dbg_px = dbg ? dbg->p_x : nullptr;
  prm.dbg_qx = dbg ? dbg->q_x : nullptr;
  prm.dbg_Z = dbg ? dbg->Z : nullptr;
  if (dtype == SPECDEC_BF16)
    return pl.U == 4 ? launch_verify<__nv_bfloat16, 4>(prm, pl, st)
                     : launch_verify<__nv_bfloat16, 1>(prm, pl, st);
  return pl.U == 4 ? launch_verify<float, 4>(prm, pl, st) : launch_verify<float, 1>(prm, pl, st);
}

// grow-only device buffer of the current device (zero-filled when (re)allocated)
specdec_status ensure_buf(std::unordered_map<int, DeviceBuf> &map, size_t bytes,
                          cudaStream_t st, void **out, size_t *out_bytes) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SPECDEC_ECUDA;
  std::lock_guard<std::mutex> lk(g_mu);
  DeviceBuf &db = map[dev];
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
  if (out_bytes) *out_bytes = db.bytes;
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

specdec_status specdec_workspace_init(void *workspace, size_t workspace_bytes, void *stream) {
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255) || workspace_bytes < 256)
    return SPECDEC_EINVAL;
  size_t n = counter_region(workspace_bytes);
  if (n > workspace_bytes) n = workspace_bytes;
  return cudaMemsetAsync(workspace, 0, n, static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? SPECDEC_OK
             : SPECDEC_ECUDA;
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
  size_t ws_bytes = 0;
  s = ensure_buf(g_ws, need, static_cast<cudaStream_t>(stream), &ws, &ws_bytes);
  if (s != SPECDEC_OK) return s;
  return run(target_logits, draft_logits, draft_tokens, u_accept, u_resample, temperature, B, K,
             V, dtype, ws, ws_bytes, nullptr, out_tokens, out_num_accepted,
             static_cast<cudaStream_t>(stream));
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
  size_t off[8], tot = 0;
  const size_t sizes[8] = {n_t, n_d, n_tok, n_ua, n_b, n_b, n_ot, n_b};
  for (int i = 0; i < 8; ++i) {
    off[i] = tot;
    tot = align256(tot + sizes[i]);
  }
  void *base = nullptr, *ws = nullptr;
  size_t ws_bytes = 0;
  s = ensure_buf(g_staging, tot, st, &base, nullptr);
  if (s != SPECDEC_OK) return s;
  s = ensure_buf(g_ws, pl.total, st, &ws, &ws_bytes);
  if (s != SPECDEC_OK) return s;
  char *c = static_cast<char *>(base);
  const void *src[6] = {target_logits, draft_logits, draft_tokens, u_accept, u_resample,
                        temperature};
  for (int i = 0; i < 6; ++i)
    if (cudaMemcpyAsync(c + off[i], src[i], sizes[i], cudaMemcpyHostToDevice, st) != cudaSuccess)
      return SPECDEC_ECUDA;
  s = run(c + off[0], c + off[1], reinterpret_cast<const int32_t *>(c + off[2]),
          reinterpret_cast<const float *>(c + off[3]), reinterpret_cast<const float *>(c + off[4]),
          reinterpret_cast<const float *>(c + off[5]), B, K, V, dtype, ws, ws_bytes, nullptr, reinterpret_cast<int32_t *>(c + off[6]), reinterpret_cast<int32_t *>(c + off[7]),
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
  Plan pl;
  if (!make_plan(B, K, V, dtype, num_sms(), pl)) return SPECDEC_EINVAL;
  if (record_capacity((size_t)SPECDEC_STATIC_SCRATCH_BYTES) < pl.records) return SPECDEC_ESIZE;
  void *scratch = nullptr;
  s = static_scratch_address(&scratch);
  if (s != SPECDEC_OK) return s;
  // The array starts zeroed (it is a zero-initialised device variable) and
  // every call leaves its counter region zeroed again; the records the kernel
  // reads are written earlier in the same call.
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
        cudaSetDevice(kv.first);
        cudaDeviceSynchronize();
        cudaFree(kv.second.ptr);
      }
    }
    m->clear();
  }
  cudaSetDevice(cur);
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
