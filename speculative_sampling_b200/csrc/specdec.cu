// libspecdec: the batched speculative-sampling verify step for B200 (sm_100a).
//
// What it computes is stated in include/specdec.h (accept with
// alpha(x) = min(1, p_target(x)/p_draft(x)), stop at the first rejection, draw
// from max(0, p - q)/Z or from the bonus row; speculative decoding blog
// "Speculative Decoding ... Llama 70B x2.4", section "The mathematical definition
// from Leviathan et al.").  This file is the B200 implementation:
//
//   k_row_stats  one pass over every logit row (B*(2K+1) rows of V): split-V
//                online softmax statistics (row max m, sum of 2^((z-m)*c)) with
//                16-byte non-temporal-in-L1 vector loads, a per-thread running
//                max, warp-shuffle and shared-memory combines.  It streams the
//                whole input once and is the HBM-bound kernel of the step.
//   k_accept     one warp per sequence: combines the V-split partials of each of
//                the 2K+1 rows in fp64, gathers p_i(x_i), q_i(x_i), tests
//                u*q < p on K lanes and finds the first rejection with
//                __ballot_sync/__ffs; writes the accepted prefix.
//   k_resample   streams only the selected row pair (target/draft row n, or the
//                target's bonus row K), forms r(v) = max(0, p - q) on the fly,
//                reduces it per V-chunk; the last CTA of each sequence (atomic
//                ticket, no waiting) takes the fp64 exclusive prefix over
//                chunks, finds the chunk holding u*Z and rescans that one chunk
//                with a block-wide fp64 scan to emit the drawn token.
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

#include <climits>
#include <cstring>
#include <mutex>
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
struct __align__(16) Sel {  // per sequence: what the draw needs
  double St, Sd;            // normalisers of the drawn target/draft rows
  double c64;               // log2(e) / T
  float Mt, Md;             // maxima of the drawn rows
  int n;                    // draw position (= accepted count), -1 if invalid
  int pad;
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

__device__ __forceinline__ uint4 ld_stream(const uint4 *p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ __nv_bfloat162 as_bf162(uint32_t w) {
  __nv_bfloat162 v;
  memcpy(&v, &w, sizeof v);
  return v;
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
  template <int U>
  static __device__ __forceinline__ float tile_max(const uint4 (&buf)[U]) {
    __nv_bfloat162 mx = as_bf162(buf[0].x);
#pragma unroll
    for (int k = 0; k < U; ++k) {
      const uint32_t w[4] = {buf[k].x, buf[k].y, buf[k].z, buf[k].w};
#pragma unroll
      for (int q = (k == 0 ? 1 : 0); q < 4; ++q)
        mx = __hmax2_nan(mx, as_bf162(w[q]));
    }
    return fmax_nan(__low2float(mx), __high2float(mx));
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
  template <int U>
  static __device__ __forceinline__ float tile_max(const uint4 (&buf)[U]) {
    float m = __uint_as_float(buf[0].x);
#pragma unroll
    for (int k = 0; k < U; ++k) {
      float x[4];
      unpack(buf[k], x);
#pragma unroll
      for (int q = (k == 0 ? 1 : 0); q < 4; ++q) m = fmax_nan(m, x[q]);
    }
    return m;
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

// Online update of (m, s) = (running max, sum 2^((z-m)c)) with one logit.
// NaN propagates into s; +Inf makes m = +Inf (the row is rejected later).
__device__ __forceinline__ void online_add(float &m, float &s, float x, Scale c) {
  if (!(x <= m)) {
    s = s * ex2(scaled(m - x, c)) + 1.0f;
    m = x;
  } else if (m != -INFINITY) {
    s += ex2(scaled(x - m, c));
  }
}

// Fold one register tile (U vectors per thread) into (m, s).
template <typename T, int U>
__device__ __forceinline__ void tile_update(const uint4 (&buf)[U], float &m, float &s, Scale c) {
  constexpr int VEC = Dt<T>::VEC;
  const float tmax = Dt<T>::template tile_max<U>(buf);
  if (!(tmax <= m)) {  // new max (or NaN): rescale what we have
    s = s * ex2(scaled(m - tmax, c));
    m = tmax;
  }
  if (m != -INFINITY) {
    float vs[U];
#pragma unroll
    for (int k = 0; k < U; ++k) {
      float x[VEC];
      Dt<T>::unpack(buf[k], x);
      float e[VEC];
#pragma unroll
      for (int q = 0; q < VEC; ++q) e[q] = ex2(scaled(x[q] - m, c));
#pragma unroll
      for (int w = 1; w < VEC; w *= 2)  // pairwise tree within the vector
#pragma unroll
        for (int q = 0; q < VEC; q += 2 * w) e[q] += e[q + w];
      vs[k] = e[0];
    }
#pragma unroll
    for (int w = 1; w < U; w *= 2)
#pragma unroll
      for (int k = 0; k + w < U; k += 2 * w) vs[k] += vs[k + w];
    s += vs[0];
  }
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

// Combine per-thread (m, s) over the CTA: returns (M, S) in thread 0.
__device__ __forceinline__ void block_combine(float m, float s, Scale c, float &M, double &S) {
  __shared__ float sm_m[NWARP];
  __shared__ double sm_s[NWARP];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const float mw = warp_max_nan(m);
  double sl = (m == -INFINITY) ? 0.0 : (double)s * (double)ex2(scaled(m - mw, c));
  sl = warp_sum(sl);
  if (lane == 0) {
    sm_m[warp] = mw;
    sm_s[warp] = sl;
  }
  __syncthreads();
  if (warp == 0) {
    const float m2 = lane < NWARP ? sm_m[lane] : -INFINITY;
    const double s2 = lane < NWARP ? sm_s[lane] : 0.0;
    const float mb = warp_max_nan(m2);
    double f = (m2 == -INFINITY) ? 0.0 : s2 * (double)ex2(scaled(m2 - mb, c));
    f = warp_sum(f);
    M = mb;
    S = f;
  }
}

// ---------------------------------------------------------------------------
// kernel 1: per-(row, V-split) softmax statistics
// ---------------------------------------------------------------------------
template <typename T, int U>
__global__ void __launch_bounds__(NT) k_row_stats(const T *__restrict__ target,
                                                  const T *__restrict__ draft,
                                                  const float *__restrict__ temperature, int K,
                                                  long long V, int nsplit,
                                                  Partial *__restrict__ part) {
  constexpr int VEC = Dt<T>::VEC;
  const int R = 2 * K + 1;
  const long long row = (long long)blockIdx.x / nsplit;
  const int split = (int)((long long)blockIdx.x - row * nsplit);
  const long long b = row / R;
  const int j = (int)(row - b * R);
  const T *p = (j <= K) ? target + (b * (K + 1) + j) * V : draft + (b * K + (j - K - 1)) * V;
  const Scale c = make_scale(kLog2e / (double)temperature[b]);

  const int head = row_head(p, V);
  const long long nvec = (V - head) / VEC;
  const uint4 *pv = reinterpret_cast<const uint4 *>(p + head);
  const long long v0 = (long long)split * (NT * U) + threadIdx.x;

  uint4 buf[U];
#pragma unroll
  for (int k = 0; k < U; ++k) {
    const long long vi = v0 + (long long)k * NT;
    buf[k] = (vi < nvec) ? ld_stream(pv + vi) : Dt<T>::neg_inf();
  }
  float m = -INFINITY, s = 0.0f;
  tile_update<T, U>(buf, m, s, c);
  if (split == 0 && (int)threadIdx.x < head) online_add(m, s, Dt<T>::load(p + threadIdx.x), c);
  if (split == nsplit - 1) {
    const long long t = head + nvec * VEC + threadIdx.x;
    if (t < V) online_add(m, s, Dt<T>::load(p + t), c);
  }
  float M;
  double S;
  block_combine(m, s, c, M, S);
  if (threadIdx.x == 0) {
    Partial out;
    out.s = S;
    out.m = M;
    out.pad = 0;
    part[row * nsplit + split] = out;
  }
}

// ---------------------------------------------------------------------------
// kernel 2: combine, gather p(x), q(x), accept test, first rejection
// ---------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(128) k_accept(
    const T *__restrict__ target, const T *__restrict__ draft,
    const int32_t *__restrict__ tokens, const float *__restrict__ u_accept,
    const float *__restrict__ temperature, int B, int K, long long V, int nsplit,
    const Partial *__restrict__ part, Sel *__restrict__ sel, unsigned *__restrict__ counters,
    int32_t *__restrict__ out_tokens, int32_t *__restrict__ out_n,
    float *__restrict__ dbg_row_max, double *__restrict__ dbg_row_sum,
    double *__restrict__ dbg_px, double *__restrict__ dbg_qx) {
  const int lane = threadIdx.x & 31;
  const long long b = (long long)blockIdx.x * 4 + (threadIdx.x >> 5);
  if (b >= B) return;
  const int R = 2 * K + 1;
  const float Tf = temperature[b];
  const bool t_ok = isfinite(Tf) && Tf > 0.0f;
  const double c64 = kLog2e / (double)Tf;

  // combine the V-splits of every row in fp64; lane i keeps the statistics of
  // target row i and draft row i, every lane keeps those of target row K
  float my_mt = 0.f, my_md = 0.f, mk = 0.f;
  double my_st = 1.0, my_sd = 1.0, sk = 1.0;
  bool rows_ok = true;
  for (int r = 0; r < R; ++r) {
    const Partial *P = part + (b * R + r) * nsplit;
    float m = -INFINITY;
    for (int s = lane; s < nsplit; s += 32) m = fmaxf(m, P[s].m);
    m = warp_max_nan(m);
    double acc = 0.0;
    for (int s = lane; s < nsplit; s += 32) {
      const Partial ps = P[s];
      acc += (ps.m == -INFINITY) ? ps.s : ps.s * exp2(((double)ps.m - (double)m) * c64);
    }
    acc = warp_sum(acc);
    rows_ok = rows_ok && isfinite(m) && isfinite(acc) && acc > 0.0;
    if (r < K && lane == r) {
      my_mt = m;
      my_st = acc;
    } else if (r == K) {
      mk = m;
      sk = acc;
    } else if (r > K && lane == r - K - 1) {
      my_md = m;
      my_sd = acc;
    }
    if (lane == 0) {
      if (dbg_row_max) dbg_row_max[b * R + r] = m;
      if (dbg_row_sum) dbg_row_sum[b * R + r] = acc;
    }
  }

  // gather and test, one draft position per lane
  int x = 0;
  bool x_ok = true, acc_i = false;
  double p = 0.0, q = 0.0;
  if (lane < K) {
    x = tokens[b * K + lane];
    x_ok = (x >= 0) && ((long long)x < V);
    if (x_ok && rows_ok && t_ok) {
      const float zt = Dt<T>::load(target + (b * (K + 1) + lane) * V + x);
      const float zd = Dt<T>::load(draft + (b * K + lane) * V + x);
      p = exp2(((double)zt - (double)my_mt) * c64) / my_st;
      q = exp2(((double)zd - (double)my_md) * c64) / my_sd;
      acc_i = (double)u_accept[b * K + lane] * q < p;
    }
  }
  const unsigned bad_x = __ballot_sync(FULL, lane < K && !x_ok);
  const unsigned accm = __ballot_sync(FULL, lane < K && acc_i);
  const bool seq_ok = t_ok && rows_ok && bad_x == 0;
  const unsigned kmask = (K >= 32) ? FULL : ((1u << K) - 1u);
  const unsigned rej = ~accm & kmask;
  const int n = seq_ok ? (rej ? __ffs(rej) - 1 : K) : -1;

  int32_t *ot = out_tokens + b * (K + 1);
  if (!seq_ok) {
    for (int i = lane; i <= K; i += 32) ot[i] = -1;
  } else {
    if (lane < n) ot[lane] = x;
    for (int i = n + 1 + lane; i <= K; i += 32) ot[i] = -1;
    if (lane < K && lane <= n) {
      if (dbg_px) dbg_px[b * K + lane] = p;
      if (dbg_qx) dbg_qx[b * K + lane] = q;
    }
  }
  // the lane holding the drawn row's statistics publishes them
  const int owner = (seq_ok && n < K) ? n : 0;
  if (lane == owner) {
    Sel o;
    o.n = n;
    o.pad = 0;
    o.c64 = c64;
    if (seq_ok && n < K) {
      o.Mt = my_mt;
      o.St = my_st;
      o.Md = my_md;
      o.Sd = my_sd;
    } else {
      o.Mt = mk;
      o.St = sk;
      o.Md = 0.f;
      o.Sd = 1.0;
    }
    sel[b] = o;
    counters[b] = 0;  // arrival ticket of k_resample for this sequence
    out_n[b] = n;
    if (!seq_ok) {
      unsigned f = 0;
      if (!t_ok) f |= SPECDEC_ERR_TEMPERATURE;
      if (bad_x) f |= SPECDEC_ERR_TOKEN;
      if (!rows_ok) f |= SPECDEC_ERR_LOGITS;
      atomicOr(&g_error_flags, f);
    }
  }
}

// ---------------------------------------------------------------------------
// kernel 3: residual / bonus draw
// ---------------------------------------------------------------------------
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

// Block-wide exclusive prefix sum of one double per thread, in thread order
// (fixed association); `total` receives the block sum.  All threads call it.
__device__ __forceinline__ double block_excl_scan(double v, double &total) {
  __shared__ double sm[NWARP];
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
  for (int w = 0; w < NWARP; ++w) {
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
template <typename T>
__device__ __noinline__ int draw_exact64(const T *pt, const T *pd, long long V, const Sel &sl, double u,
                            int *s_y, int *s_lastpos, double *dbg_Z) {
  const long long E = (V + NT - 1) / NT;
  const long long e0 = (long long)threadIdx.x * E < V ? (long long)threadIdx.x * E : V;
  const long long e1 = (e0 + E < V) ? e0 + E : V;
  double sr = 0.0, sp = 0.0;
  for (long long v = e0; v < e1; ++v) {
    const double p = prob64(pt, v, sl.Mt, sl.St, sl.c64);
    const double q = prob64(pd, v, sl.Md, sl.Sd, sl.c64);
    sr += (p - q > 0.0) ? p - q : 0.0;
    sp += p;
  }
  double Zr, Zp;
  const double xr = block_excl_scan(sr, Zr);
  const double xp = block_excl_scan(sp, Zp);
  const bool use_p = !(Zr > 0.0);
  const double Z = use_p ? Zp : Zr;
  const double t = u * Z;
  double C = use_p ? xp : xr;
  int last = -1;
  bool found = false;
  for (long long v = e0; v < e1; ++v) {
    const double p = prob64(pt, v, sl.Mt, sl.St, sl.c64);
    const double q = prob64(pd, v, sl.Md, sl.Sd, sl.c64);
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

template <typename T, int UR>
__global__ void __launch_bounds__(NT) k_resample(
    const T *__restrict__ target, const T *__restrict__ draft,
    const float *__restrict__ u_resample, int K, long long V, int nsr,
    const Sel *__restrict__ sel, ResPartial *__restrict__ rpart, unsigned *__restrict__ counters,
    int32_t *__restrict__ out_tokens, double *__restrict__ dbg_Z) {
  constexpr int VEC = Dt<T>::VEC;
  constexpr long long CH = (long long)NT * UR * VEC;  // elements per chunk
  const long long b = (long long)blockIdx.x / nsr;
  const int chunk = (int)((long long)blockIdx.x - b * nsr);
  const Sel sl = sel[b];
  if (sl.n < 0) return;  // invalid sequence: the accept kernel wrote its outputs
  DrawRow d;
  d.bonus = (sl.n == K);
  d.Mt = sl.Mt;
  d.Md = sl.Md;
  d.c = make_scale(sl.c64);
  const double lam = d.bonus ? 0.0 : sl.St / sl.Sd;
  d.lhi = (float)lam;
  d.llo = (float)(lam - (double)d.lhi);
  const T *pt = target + (b * (K + 1) + sl.n) * V;
  const T *pd = d.bonus ? pt : draft + (b * K + sl.n) * V;

  const int head = row_head(pt, V);
  const bool vec_ok = row_head(pd, V) == head;
  const long long nvec = vec_ok ? (V - head) / VEC : 0;
  // chunk c covers elements [lo_c, hi_c): chunk 0 also takes the head, the
  // last chunk also takes the tail
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

  float rs = 0.f;
  if (vec_ok) {
    const uint4 *vt = reinterpret_cast<const uint4 *>(pt + head);
    const uint4 *vd = reinterpret_cast<const uint4 *>(pd + head);
#pragma unroll
    for (int k = 0; k < UR; ++k) {
      const long long vi = (long long)chunk * NT * UR + (long long)k * NT + threadIdx.x;
      if (vi < nvec) {
        float xt[VEC], xd[VEC] = {};
        Dt<T>::unpack(ld_stream(vt + vi), xt);
        if (!d.bonus) Dt<T>::unpack(ld_stream(vd + vi), xd);
#pragma unroll
        for (int q = 0; q < VEC; ++q) rs += res_weight(xt[q], d.bonus ? 0.f : xd[q], d);
      }
    }
    // head elements belong to chunk 0; the < VEC tail elements to the chunk
    // whose element range [lo_c, hi_c) holds them (the rescan uses the same)
    // (a thread may own one head and one tail element of the same chunk)
    const long long tail_chunk = nvec / ((long long)NT * UR) < nsr - 1
                                     ? nvec / ((long long)NT * UR) : (long long)(nsr - 1);
    const long long tail = head + nvec * VEC + threadIdx.x;
    const long long extra[2] = {(chunk == 0 && (int)threadIdx.x < head) ? (long long)threadIdx.x : -1,
                                (chunk == tail_chunk && tail < V && threadIdx.x < VEC) ? tail : -1};
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      if (extra[e] >= 0)
        rs += res_weight(Dt<T>::load(pt + extra[e]), d.bonus ? 0.f : Dt<T>::load(pd + extra[e]), d);
    }
  } else {  // rows of different alignment: scalar loads over the chunk
    const long long lo = chunk_lo(chunk), hi = chunk_hi(chunk);
    for (long long v = lo + threadIdx.x; v < hi; v += NT)
      rs += res_weight(Dt<T>::load(pt + v), d.bonus ? 0.f : Dt<T>::load(pd + v), d);
  }

  // chunk sums (fp64 across threads)
  __shared__ double sm_r[NWARP];
  __shared__ int s_last;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const double r64 = warp_sum((double)rs);
  if (lane == 0) sm_r[warp] = r64;
  __syncthreads();
  if (threadIdx.x == 0) {
    double a = 0.0;
    for (int w = 0; w < NWARP; ++w) a += sm_r[w];
    ResPartial o;
    o.R = a;
    o.pad = 0.0;
    rpart[b * nsr + chunk] = o;
    __threadfence();
    const unsigned t = atomicAdd(&counters[b], 1u);
    s_last = (t == (unsigned)(nsr - 1));
  }
  __syncthreads();
  if (!s_last) return;

  // ---- the last CTA of sequence b draws ----
  __shared__ double s_base, s_t;
  __shared__ int s_chunk, s_mode, s_y, s_lastpos;
  if (threadIdx.x == 0) {
    __threadfence();
    const ResPartial *rp = rpart + b * nsr;
    double Z = 0.0;
    for (int c2 = 0; c2 < nsr; ++c2) Z += __ldcg(&rp[c2].R);
    s_y = INT_MAX;
    s_lastpos = -1;
    // Residual mass below 2^-64 (relative to the target row's largest
    // probability): the fp32 weights have run out of range, so the draw is
    // redone in fp64 over the whole row pair.
    s_mode = (!d.bonus && !(Z >= ldexp(sl.St, -64))) ? 1 : 0;
    if (s_mode == 0) {
      const double t = (double)u_resample[b] * Z;
      double acc = 0.0, base = -1.0;
      int cs = -1;
      for (int c2 = 0; c2 < nsr; ++c2) {
        const double v = __ldcg(&rp[c2].R);
        if (acc + v > t) {
          cs = c2;
          base = acc;
          break;
        }
        acc += v;
      }
      if (cs < 0) {  // defensive: rounding left t at or past the total
        for (int c2 = nsr - 1; c2 >= 0 && cs < 0; --c2)
          if (__ldcg(&rp[c2].R) > 0.0) cs = c2;
        if (cs < 0) cs = 0;
      }
      s_base = base;  // < 0 selects the "last positive element" rule
      s_t = t;
      s_chunk = cs;
      if (dbg_Z) dbg_Z[b] = Z / sl.St;
    }
  }
  __syncthreads();
  if (s_mode == 1) {
    int y = draw_exact64(pt, pd, V, sl, (double)u_resample[b], &s_y, &s_lastpos,
                         dbg_Z ? dbg_Z + b : nullptr);
    if (threadIdx.x == 0) out_tokens[b * (K + 1) + sl.n] = y;
    return;
  }
  const long long lo = chunk_lo(s_chunk), hi = chunk_hi(s_chunk);
  const long long L = hi - lo;
  const long long E = (L + NT - 1) / NT;  // contiguous elements per thread
  const long long e0 = lo + (long long)threadIdx.x * E < hi ? lo + (long long)threadIdx.x * E : hi;
  const long long e1 = (e0 + E < hi) ? e0 + E : hi;
  double mysum = 0.0;
  int lastpos = -1;
  for (long long v = e0; v < e1; ++v) {
    const float x = res_weight(Dt<T>::load(pt + v), d.bonus ? 0.f : Dt<T>::load(pd + v), d);
    mysum += (double)x;
    if (x > 0.0f) lastpos = (int)v;
  }
  double total;
  const double excl = block_excl_scan(mysum, total);
  if (lastpos >= 0) atomicMax(&s_lastpos, lastpos);
  if (s_base >= 0.0) {
    double C = s_base + excl;
    const double t = s_t;
    for (long long v = e0; v < e1; ++v) {
      C += (double)res_weight(Dt<T>::load(pt + v), d.bonus ? 0.f : Dt<T>::load(pd + v), d);
      if (C > t) {
        atomicMin(&s_y, (int)v);
        break;
      }
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int y = s_y;
    if (y == INT_MAX) y = (s_lastpos >= 0) ? s_lastpos : (int)lo;
    out_tokens[b * (K + 1) + sl.n] = y;
  }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
enum KernelId { KID_STATS = 0, KID_ACCEPT = 1, KID_RESAMPLE = 2, KID_COUNT = 3 };
const char *kKernelNames[KID_COUNT] = {"k_row_stats", "k_accept", "k_resample"};

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

struct Plan {
  int esize, vec, U, nsplit, UR, nsr;
  long long rows;
  size_t off_part, off_sel, off_rpart, off_cnt, total;
};

int num_sms() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

bool make_plan(int B, int K, int V, specdec_dtype dtype, int sms, Plan &pl) {
  if (B < 0 || K < 1 || K > 32 || V < 1) return false;
  if (dtype != SPECDEC_F32 && dtype != SPECDEC_BF16) return false;
  pl.esize = dtype == SPECDEC_BF16 ? 2 : 4;
  pl.vec = 16 / pl.esize;
  pl.rows = (long long)B * (2 * K + 1);
  const long long nvec_max = ((long long)V + pl.vec - 1) / pl.vec;
  // 4 vectors per thread when that still gives >= 4 CTAs per SM; otherwise 1,
  // so that small batches (B = 1) still spread over every SM
  const long long ns4 = (nvec_max + NT * 4 - 1) / (NT * 4);
  pl.U = (pl.rows * ns4 >= 4LL * sms) ? 4 : 1;
  const long long ns = (nvec_max + (long long)NT * pl.U - 1) / ((long long)NT * pl.U);
  pl.nsplit = (int)(ns > 0 ? ns : 1);
  const long long nr2 = (nvec_max + NT * 2 - 1) / (NT * 2);
  pl.UR = ((long long)B * nr2 >= 2LL * sms) ? 2 : 1;
  const long long nr = (nvec_max + (long long)NT * pl.UR - 1) / ((long long)NT * pl.UR);
  pl.nsr = (int)(nr > 0 ? nr : 1);
  if (pl.rows * pl.nsplit > INT_MAX || (long long)B * pl.nsr > INT_MAX) return false;
  if ((long long)B * (K + 1) * (long long)V > (1LL << 56)) return false;
  size_t off = 0;
  pl.off_part = off;
  off = align256(off + sizeof(Partial) * (size_t)pl.rows * pl.nsplit);
  pl.off_sel = off;
  off = align256(off + sizeof(Sel) * (size_t)B);
  pl.off_rpart = off;
  off = align256(off + sizeof(ResPartial) * (size_t)B * pl.nsr);
  pl.off_cnt = off;
  off = align256(off + sizeof(unsigned) * (size_t)B);
  pl.total = off > 0 ? off : 256;
  return true;
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

template <typename T>
specdec_status launch_all(const void *tg, const void *dr, const int32_t *tok, const float *ua,
                          const float *ur, const float *temp, int B, int K, int V,
                          const Plan &pl, char *ws, const specdec_debug *dbg, int32_t *out_tokens,
                          int32_t *out_n, cudaStream_t st) {
  const T *t = static_cast<const T *>(tg);
  const T *d = static_cast<const T *>(dr);
  Partial *part = reinterpret_cast<Partial *>(ws + pl.off_part);
  Sel *sel = reinterpret_cast<Sel *>(ws + pl.off_sel);
  ResPartial *rp = reinterpret_cast<ResPartial *>(ws + pl.off_rpart);
  unsigned *cnt = reinterpret_cast<unsigned *>(ws + pl.off_cnt);
  const unsigned g1 = (unsigned)(pl.rows * pl.nsplit);
  {
    LaunchTimer lt(KID_STATS, st);
    if (pl.U == 4)
      k_row_stats<T, 4><<<g1, NT, 0, st>>>(t, d, temp, K, V, pl.nsplit, part);
    else
      k_row_stats<T, 1><<<g1, NT, 0, st>>>(t, d, temp, K, V, pl.nsplit, part);
  }
  {
    LaunchTimer lt(KID_ACCEPT, st);
    k_accept<T><<<(unsigned)((B + 3) / 4), 128, 0, st>>>(
        t, d, tok, ua, temp, B, K, V, pl.nsplit, part, sel, cnt, out_tokens, out_n,
        dbg ? dbg->row_max : nullptr, dbg ? dbg->row_sum : nullptr, dbg ? dbg->p_x : nullptr,
        dbg ? dbg->q_x : nullptr);
  }
  {
    LaunchTimer lt(KID_RESAMPLE, st);
    const unsigned g3 = (unsigned)((long long)B * pl.nsr);
    if (pl.UR == 2)
      k_resample<T, 2><<<g3, NT, 0, st>>>(t, d, ur, K, V, pl.nsr, sel, rp, cnt, out_tokens,
                                          dbg ? dbg->Z : nullptr);
    else
      k_resample<T, 1><<<g3, NT, 0, st>>>(t, d, ur, K, V, pl.nsr, sel, rp, cnt, out_tokens,
                                          dbg ? dbg->Z : nullptr);
  }
  return cudaGetLastError() == cudaSuccess ? SPECDEC_OK : SPECDEC_ECUDA;
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
                   cudaStream_t st) {
  specdec_status s = check_args(tg, dr, tok, ua, ur, temp, B, K, V, dtype, ot, on);
  if (s != SPECDEC_OK || B == 0) return s;
  Plan pl;
  if (!make_plan(B, K, V, dtype, num_sms(), pl)) return SPECDEC_EINVAL;
  if (!ws || ws_bytes < pl.total || (reinterpret_cast<uintptr_t>(ws) & 255)) return SPECDEC_EINVAL;
  if (dtype == SPECDEC_BF16)
    return launch_all<__nv_bfloat16>(tg, dr, tok, ua, ur, temp, B, K, V, pl,
                                     static_cast<char *>(ws), dbg, ot, on, st);
  return launch_all<float>(tg, dr, tok, ua, ur, temp, B, K, V, pl, static_cast<char *>(ws), dbg,
                           ot, on, st);
}

// grow-only device buffer of the current device (zero-filled when (re)allocated)
specdec_status ensure_buf(std::unordered_map<int, DeviceBuf> &map, size_t bytes,
                          cudaStream_t st, void **out) {
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
  // (V-split partials, per-sequence selection, chunk sums, the arrival counters
  // that k_accept resets) is written earlier in the same call.
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
