// common.cuh -- device building blocks of the B200 LapSum soft top-k.
//
// Method: "Fast LapSum: Exact Differentiable Top-k at Million Scale"
// (Technical Summary sections 2.1-2.2; arXiv abstract of the same paper).
#pragma once

#include <cstdint>
#include <cstring>
#include <cuda_runtime.h>
#include <math_constants.h>

namespace lapsum {

// ---------------------------------------------------------------------------
// row status bits.  The low byte mirrors LAPSUM_ROW_* of lapsum_topk.h; the
// rest are internal hand-offs between kernels and never reach the caller.
// ---------------------------------------------------------------------------
constexpr uint32_t ROW_CERTIFIED = 0x01u;
constexpr uint32_t ROW_WIDENED = 0x02u;
constexpr uint32_t ROW_FALLBACK = 0x04u;
constexpr uint32_t ROW_NONFINITE = 0x08u;
constexpr uint32_t ROW_TIMEOUT = 0x10u;
constexpr uint32_t ROW_OVERFLOW = 0x20u;
constexpr uint32_t ROW_TRUNCATED = 0x40u;  // sparse output: more entries than its capacity
constexpr uint32_t ROW_BADARG = 0x80u;     // per-row k or alpha out of range: outputs NaN
constexpr uint32_t ROW_PUBLIC = 0xFFu;
constexpr uint32_t ROW_MISS_LEFT = 0x100u;   // S(a_L) < k: b lies below a_L
constexpr uint32_t ROW_MISS_RIGHT = 0x200u;  // S(a_R) >= k: b lies at or above a_R
constexpr uint32_t ROW_FORCE_FB = 0x400u;    // test knob: take the full sort
constexpr uint32_t ROW_FORCE_TO = 0x800u;    // test knob: the recovery barrier times out
constexpr uint32_t ROW_NEEDS_RECOVERY = ROW_MISS_LEFT | ROW_MISS_RIGHT | ROW_OVERFLOW | ROW_FORCE_FB | ROW_FORCE_TO;
// rows whose outputs are NaN
constexpr uint32_t ROW_NAN_OUT = ROW_NONFINITE | ROW_BADARG | ROW_TIMEOUT;

constexpr float kLog2e = 1.4426950408889634f;

// ---------------------------------------------------------------------------
// splitmix64 (Steele, Lea & Flood, OOPSLA 2014), used counter-style: the i-th
// output (i >= 1) of a generator whose state starts at s is mix(s + i*gamma).
// ---------------------------------------------------------------------------
constexpr uint64_t kGamma = 0x9E3779B97F4A7C15ull;

__host__ __device__ __forceinline__ uint64_t sm64_mix(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}
__host__ __device__ __forceinline__ uint64_t sm64_out(uint64_t s, uint64_t i) {
  return sm64_mix(s + i * kGamma);
}
// stream of one row: the (row+1)-th output of a generator seeded with `seed`
__host__ __device__ __forceinline__ uint64_t row_stream(uint64_t seed, uint64_t row) {
  return sm64_out(seed, row + 1);
}

// Localization sample j of a row (section 2.2: scores with Laplace noise):
// draw 2j+1 picks an index uniformly in [0, n) (high word of draw * n), draw
// 2j+2 gives u in (0,1) and Laplace(0, alpha) noise by the inverse CDF.
// Y = r[I] + eps is formed in fp64 and rounded to fp32.
__device__ __forceinline__ uint64_t sample_index(uint64_t s, uint64_t j, uint64_t n) {
  return __umul64hi(sm64_out(s, 2 * j + 1), n);
}
__device__ __forceinline__ double laplace_noise(uint64_t s, uint64_t j, double alpha) {
  const uint64_t d = sm64_out(s, 2 * j + 2);
  const double u = ((double)(d >> 11) + 0.5) * 0x1p-53;
  const double e = (u < 0.5) ? log(2.0 * u) : -log(2.0 - 2.0 * u);
  return alpha * e;
}

// ---------------------------------------------------------------------------
// per-row budget and scale.  The method is stated for one vector with one k
// and one alpha (technical summary section 2.1); a batch may give every row
// its own.  An out-of-range value marks the row ROW_BADARG and is replaced by
// a harmless one (k = n/2, alpha = 1) so that every pass still runs; the
// row's outputs are NaN.
// ---------------------------------------------------------------------------
struct RowArgs {
  double k;        // budget
  double alpha;    // scale of the threshold solve
  double alpha_p;  // scale of the memberships (differs for the DFTopK form)
  bool bad;
};
__device__ __forceinline__ RowArgs row_args(double k, double alpha, double alpha_p, int dftopk,
                                            const double* k_rows, const double* alpha_rows, int64_t r,
                                            int64_t n) {
  RowArgs a{k, alpha, alpha_p, false};
  if (k_rows) {
    const double kr = __ldg(k_rows + r);
    if (kr > 0.0 && kr < (double)n) a.k = kr;  // NaN fails the test
    else a.bad = true;
  }
  if (alpha_rows) {
    const double ar = __ldg(alpha_rows + r);
    if (ar >= 1e-30 && ar <= 1e30) {
      a.alpha_p = ar;
      if (!dftopk) a.alpha = ar;
    } else {
      a.bad = true;
    }
  }
  if (a.bad) {
    a.k = 0.5 * (double)n;
    a.alpha = 1.0;
    a.alpha_p = 1.0;
  }
  return a;
}
template <class Plan>
__device__ __forceinline__ RowArgs row_args(const Plan& P, int64_t r) {
  return row_args(P.k, P.alpha, P.alpha_p, P.dftopk, P.k_rows, P.alpha_rows, r, P.n);
}
// alpha of row r for the backward (no k there)
__device__ __forceinline__ double row_alpha(double alpha, const double* alpha_rows, int64_t r, bool* bad) {
  if (!alpha_rows) return alpha;
  const double ar = __ldg(alpha_rows + r);
  if (ar >= 1e-30 && ar <= 1e30) return ar;
  *bad = true;
  return 1.0;
}

// Localization ranks (section 2.2): #{Y > b} ~ Binomial(m, q = k/n); the
// bracket edges are the c_lo-th and (c_hi+1)-th largest samples with
// c_lo/hi = mq -/+ z sigma, as ascending indices.  Every operation is rounded
// on its own (no fused multiply-add), the order of the host's computation,
// so a row that gets its k from a vector has the ranks a scalar call gets.
struct RowRanks {
  int rank_lo, rank_hi, valid_lo, valid_hi, widen_delta;
};
__device__ __forceinline__ RowRanks sample_ranks_dev(int64_t n, double k, int m, double z) {
  const double q = __ddiv_rn(k, (double)n);
  const double mq = __dmul_rn((double)m, q);
  const double sigma = __dsqrt_rn(__dmul_rn(mq, __dsub_rn(1.0, q)));
  const long long c_lo = (long long)floor(__dsub_rn(mq, __dmul_rn(z, sigma)));
  const long long c_hi = (long long)ceil(__dadd_rn(mq, __dmul_rn(z, sigma)));
  RowRanks R;
  R.valid_hi = c_lo >= 1;
  R.rank_hi = R.valid_hi ? (int)(m - c_lo) : m - 1;
  R.valid_lo = (c_hi + 1) <= m;
  R.rank_lo = R.valid_lo ? (int)(m - c_hi - 1) : 0;
  R.widen_delta = (int)ceil(__dmul_rn(__dmul_rn(2.0, z), sigma)) + 1;
  return R;
}
template <class Plan>
__device__ __forceinline__ RowRanks row_ranks(const Plan& P, double k) {
  if (!P.k_rows) return RowRanks{P.rank_lo, P.rank_hi, P.valid_lo, P.valid_hi, P.widen_delta};
  return sample_ranks_dev(P.n, k, P.m, P.z);
}

// ---------------------------------------------------------------------------
// order-preserving map between fp32 values and uint32 keys (-0 < +0)
// ---------------------------------------------------------------------------
__host__ __device__ __forceinline__ uint32_t f2key(float f) {
#ifdef __CUDA_ARCH__
  const uint32_t u = __float_as_uint(f);
#else
  uint32_t u;
  memcpy(&u, &f, 4);
#endif
  return u ^ ((uint32_t)((int32_t)u >> 31) | 0x80000000u);
}
__host__ __device__ __forceinline__ float key2f(uint32_t k) {
  const uint32_t u = k ^ ((k & 0x80000000u) ? 0x80000000u : 0xFFFFFFFFu);
#ifdef __CUDA_ARCH__
  return __uint_as_float(u);
#else
  float f;
  memcpy(&f, &u, 4);
  return f;
#endif
}

// ---------------------------------------------------------------------------
// rows that do not start on a 16-byte boundary (odd n, offset views): the
// first `head` (0-3) scores are taken one at a time and the body as float4
// from row + head; arrays walked together (scores with p, g or grad) start at
// the same address mod 16, so one head serves them all
// ---------------------------------------------------------------------------
__device__ __forceinline__ int row_head(const void* p, int64_t n) {
  const int h = (int)(((0u - (uint32_t)(uintptr_t)p) & 15u) >> 2);
  return n < h ? (int)n : h;
}
// index of the j-th score outside the body of n4 float4: [0, head), then
// [head + 4 n4, n)
__device__ __forceinline__ int64_t rest_index(int64_t j, int head, int64_t n4) {
  return j < head ? j : j + 4 * n4;
}

// ---------------------------------------------------------------------------
// per-row control block kept in the workspace (256 bytes per row)
// ---------------------------------------------------------------------------
struct alignas(256) RowCtl {
  // bracket and band plan, written by the selection step
  float aL, aR;        // bracket [aL, aR); -inf / +inf when open
  uint32_t band_cnt;   // band values appended by the filter (may exceed the capacity)
  uint32_t band_kmax;  // largest key appended
  uint32_t band_nkmin; // bitwise complement of the smallest key appended
  int32_t bins;        // key bins the band solve used (diagnostic)
  int32_t rank_lo, rank_hi;  // ascending sample ranks of the two edges
  uint32_t valid_lo, valid_hi;
  uint32_t cand_cnt;   // keys in the row's level-3 candidate list
  int32_t m;
  // aggregates and result
  int64_t nL, nR, M;
  double SL, SR;
  double b;
  double sumf, sump;
  uint32_t status;     // ROW_* bits
  uint32_t flags;      // atomicOr target of the streaming pass
  uint32_t done_sel, done_solve, done_memb, done_bwd;
  uint32_t bar_count, bar_gen;
  uint32_t sel_key[2];
  double lam;
  uint32_t timeout;    // set when a bounded grid-wide wait gives up
  uint32_t done_s1, done_s2;   // last-block counters of the selection levels
  int32_t sel_bin[2][2];       // radix-select bins of levels 1 and 2, per edge
  uint32_t sel_rem[2][2];      // rank left inside those bins
};
static_assert(sizeof(RowCtl) == 256, "RowCtl must stay one 256-byte slot");

// aggregates of one sorted group of band values (a group of the resident band, or a slice of a
// fully sorted row): count, min, max, P = sum exp((y - ymax)/alpha),
// Q = sum exp((ymin - y)/alpha); plus scan results filled in by the solver.
struct alignas(16) GroupAgg {
  int32_t cnt;
  float ymin, ymax;
  int32_t pad;
  double P, Q;
  double Apre;           // prefix anchored at ymax (left tail + groups <= t)
  double Bx, Bs;         // suffix state of everything after the group
  long long after;       // number of values after the group (incl. right tail)
};

// fp64 exp and log called (not inlined) from code that runs once per row:
// one shared copy of each routine keeps that code small, which matters when
// its instructions have to be fetched from HBM
static __device__ __noinline__ double exp_call(double x) { return exp(x); }
static __device__ __noinline__ double log_call(double x) { return log(x); }

// ---------------------------------------------------------------------------
// anchored exponential sums: a state (x, s) means sum_v exp(+-(v - x)/alpha)
// over a run of sorted values.  s == 0 is the empty run.
// Prefix states are anchored at the run's maximum (terms exp((v - x)/alpha)),
// suffix states at its minimum (terms exp((x - v)/alpha)); all terms <= 1.
// ---------------------------------------------------------------------------
struct Anch {
  double x, s;
};
__device__ __forceinline__ Anch anch_empty() { return Anch{-CUDART_INF, 0.0}; }

// earlier run a, later run b -> prefix state of a followed by b
__device__ __forceinline__ Anch comb_pre(Anch a, Anch b, double inva) {
  if (b.s == 0.0) return a;
  if (a.s == 0.0) return b;
  return Anch{b.x, fma(a.s, exp((a.x - b.x) * inva), b.s)};
}
// earlier run a, later run b -> suffix state of a followed by b
__device__ __forceinline__ Anch comb_suf(Anch a, Anch b, double inva) {
  if (a.s == 0.0) return b;
  if (b.s == 0.0) return a;
  return Anch{a.x, fma(b.s, exp((a.x - b.x) * inva), a.s)};
}
// value of a prefix state re-anchored at y >= st.x
__device__ __forceinline__ double pre_at(Anch st, double y, double inva) {
  return st.s == 0.0 ? 0.0 : st.s * exp((st.x - y) * inva);
}
// value of a suffix state re-anchored at y <= st.x
__device__ __forceinline__ double suf_at(Anch st, double y, double inva) {
  return st.s == 0.0 ? 0.0 : st.s * exp((y - st.x) * inva);
}

// ln(m + sqrt(m^2 + e^L)) for m >= 0, without overflow or underflow
__device__ __forceinline__ double lnsum(double m, double L) {
  if (m == 0.0) return 0.5 * L;
  const double lm = log_call(m);
  const double D = L - 2.0 * lm;
  if (D > 0.0) return 0.5 * L + log_call(exp_call(-0.5 * D) + sqrt(exp_call(-D) + 1.0));
  return lm + log_call(1.0 + sqrt(1.0 + exp_call(D)));
}

// Closed-form root on one interval [xj, xj1] of the threshold curve
// (section 2.2: once the interval holding b is known, b has a closed form).
// A  = prefix sum anchored at xj  (values <= xj, the left tail included),
// Bp = suffix sum anchored at xj1 (values >= xj1, the right tail included),
// c  = number of values above xj.  With u = exp_call((b - xj)/alpha) the budget
// equation is B u^2 - 2 mu u - A = 0, mu = c - k, B = Bp exp_call(-(xj1-xj)/alpha).
// The root is taken from the right knot when mu >= 0, from the left otherwise,
// in log form; the result is clamped into the interval.
__device__ __forceinline__ double closed_form_root(double xj, double xj1, double A, double Bp,
                                                   double c, double k, double alpha) {
  const double mu = c - k;
  const double lnA = A > 0.0 ? log_call(A) : -CUDART_INF;
  const double lnB = Bp > 0.0 ? log_call(Bp) : -CUDART_INF;
  double L = -CUDART_INF;
  if (A > 0.0 && Bp > 0.0) L = lnA + lnB - (xj1 - xj) / alpha;
  double b;
  if (mu >= 0.0) {
    b = (Bp > 0.0) ? xj1 + alpha * (lnsum(mu, L) - lnB) : xj1;
  } else {
    b = (A > 0.0) ? xj + alpha * (lnA - lnsum(-mu, L)) : xj;
  }
  if (b < xj) b = xj;
  if (b > xj1) b = xj1;
  return b;
}

// sum_i f_i at the root b in [xj, xj1], f_i = exp_call(-|r_i - b|/alpha)/(2 alpha):
// the values up to xj contribute A exp_call((xj - b)/alpha), those from xj1 on
// contribute Bp exp_call((b - xj1)/alpha) (A, Bp anchored as in closed_form_root).
// Exact in fp64, so it does not underflow with the fp32 per-score terms.
__device__ __forceinline__ double sum_f_at(double xj, double xj1, double A, double Bp, double b, double inva) {
  const double t1 = A > 0.0 ? A * exp_call((xj - b) * inva) : 0.0;
  const double t2 = Bp > 0.0 ? Bp * exp_call((b - xj1) * inva) : 0.0;
  return 0.5 * (t1 + t2) * inva;
}

// ---------------------------------------------------------------------------
// deterministic block reductions (fixed xor trees; scratch >= NT/32 slots)
// ---------------------------------------------------------------------------
template <typename T>
__device__ __forceinline__ T warp_sum(T v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

template <int NT, typename T>
__device__ __forceinline__ T block_sum(T v, T* scratch) {
  constexpr int NW = NT / 32;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  v = warp_sum(v);
  __syncthreads();
  if (lane == 0) scratch[warp] = v;
  __syncthreads();
  T t = (lane < NW) ? scratch[lane] : T(0);
  t = warp_sum(t);
  return t;  // every thread holds the total
}

template <int NT>
__device__ __forceinline__ int block_max_int(int v, int* scratch) {
  constexpr int NW = NT / 32;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = max(v, __shfl_xor_sync(0xffffffffu, v, o));
  __syncthreads();
  if (lane == 0) scratch[warp] = v;
  __syncthreads();
  int t = (lane < NW) ? scratch[lane] : INT32_MIN;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) t = max(t, __shfl_xor_sync(0xffffffffu, t, o));
  return t;
}

template <int NT>
__device__ __forceinline__ uint32_t block_or(uint32_t v, uint32_t* scratch) {
  constexpr int NW = NT / 32;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  v = __reduce_or_sync(0xffffffffu, v);
  __syncthreads();
  if (lane == 0) scratch[warp] = v;
  __syncthreads();
  uint32_t t = (lane < NW) ? scratch[lane] : 0u;
  return __reduce_or_sync(0xffffffffu, t);
}

// Block-wide exclusive scan of anchored states (prefix or suffix direction),
// one state per thread, deterministic.  `scr` needs 2*NT/32 doubles.
// Forward (prefix): thread t receives the combination of threads < t.
// Backward (suffix): thread t receives the combination of threads > t.
template <int NT, bool kPrefix>
__device__ __forceinline__ Anch block_excl_scan_anch(Anch v, double inva, double* scr) {
  constexpr int NW = NT / 32;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  Anch inc = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    Anch oth;
    if (kPrefix) {
      oth.x = __shfl_up_sync(0xffffffffu, inc.x, o);
      oth.s = __shfl_up_sync(0xffffffffu, inc.s, o);
      if (lane >= o) inc = comb_pre(oth, inc, inva);
    } else {
      oth.x = __shfl_down_sync(0xffffffffu, inc.x, o);
      oth.s = __shfl_down_sync(0xffffffffu, inc.s, o);
      if (lane + o < 32) inc = comb_suf(inc, oth, inva);
    }
  }
  Anch exl;
  if (kPrefix) {
    exl.x = __shfl_up_sync(0xffffffffu, inc.x, 1);
    exl.s = __shfl_up_sync(0xffffffffu, inc.s, 1);
    if (lane == 0) exl = anch_empty();
  } else {
    exl.x = __shfl_down_sync(0xffffffffu, inc.x, 1);
    exl.s = __shfl_down_sync(0xffffffffu, inc.s, 1);
    if (lane == 31) exl = anch_empty();
  }
  __syncthreads();
  if ((kPrefix && lane == 31) || (!kPrefix && lane == 0)) {
    scr[2 * warp] = inc.x;
    scr[2 * warp + 1] = inc.s;
  }
  __syncthreads();
  Anch wacc = anch_empty();
  if (kPrefix) {
    for (int w = 0; w < warp; ++w) wacc = comb_pre(wacc, Anch{scr[2 * w], scr[2 * w + 1]}, inva);
    return comb_pre(wacc, exl, inva);
  } else {
    for (int w = NW - 1; w > warp; --w) wacc = comb_suf(Anch{scr[2 * w], scr[2 * w + 1]}, wacc, inva);
    return comb_suf(exl, wacc, inva);
  }
}

// block-wide exclusive scan of int64 counts in the suffix direction
template <int NT>
__device__ __forceinline__ long long block_excl_suffix_sum(long long v, long long* scr) {
  constexpr int NW = NT / 32;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  long long inc = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    long long oth = __shfl_down_sync(0xffffffffu, inc, o);
    if (lane + o < 32) inc += oth;
  }
  long long exl = __shfl_down_sync(0xffffffffu, inc, 1);
  if (lane == 31) exl = 0;
  __syncthreads();
  if (lane == 0) scr[warp] = inc;
  __syncthreads();
  long long wacc = 0;
  for (int w = NW - 1; w > warp; --w) wacc += scr[w];
  return exl + wacc;
}

// block-wide exclusive scan of uint32 values (prefix direction)
template <int NT>
__device__ __forceinline__ uint32_t block_excl_prefix_u32(uint32_t v, uint32_t* scr, uint32_t* total) {
  constexpr int NW = NT / 32;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t inc = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    uint32_t oth = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += oth;
  }
  __syncthreads();
  if (lane == 31) scr[warp] = inc;
  __syncthreads();
  uint32_t wacc = 0, tot = 0;
  for (int w = 0; w < NW; ++w) {
    if (w < warp) wacc += scr[w];
    tot += scr[w];
  }
  if (total) *total = tot;
  return wacc + inc - v;
}

// ---------------------------------------------------------------------------
// backward reduction: lambda = sum g f / sum f with f = 2^{-a} up to a common
// factor.  Terms are kept relative to the smallest a seen so far (the score
// nearest to b), so neither sum underflows even when every f is below the
// fp32 range; the shift cancels in the ratio.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void shift_add(float a, float g, float& m, float& ps, float& psg, double& S,
                                          double& SG) {
  if (a < m) {  // a new nearest score: rescale what was accumulated
    const float sc = exp2f(a - m);
    ps *= sc;
    psg *= sc;
    S *= (double)sc;
    SG *= (double)sc;
    m = a;
  }
  const float e = exp2f(m - a);
  ps += e;
  psg = fmaf(g, e, psg);
}

// The same with two more sums weighted by z = r - b, for dL/dalpha:
// sum f z and sum g f z, rescaled together with the other two.
__device__ __forceinline__ void shift_add_z(float a, float g, float z, float& m, float& ps, float& psg,
                                            float& psz, float& psgz, double& S, double& SG, double& SZ,
                                            double& SGZ) {
  if (a < m) {
    const float sc = exp2f(a - m);
    ps *= sc;
    psg *= sc;
    psz *= sc;
    psgz *= sc;
    S *= (double)sc;
    SG *= (double)sc;
    SZ *= (double)sc;
    SGZ *= (double)sc;
    m = a;
  }
  const float e = exp2f(m - a);
  const float ez = e * z;
  ps += e;
  psg = fmaf(g, e, psg);
  psz += ez;
  psgz = fmaf(g, ez, psgz);
}

template <int NT>
__device__ __forceinline__ double block_min_double(double v, double* scratch) {
  constexpr int NW = NT / 32;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmin(v, __shfl_xor_sync(0xffffffffu, v, o));
  __syncthreads();
  if (lane == 0) scratch[warp] = v;
  __syncthreads();
  double t = (lane < NW) ? scratch[lane] : CUDART_INF;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) t = fmin(t, __shfl_xor_sync(0xffffffffu, t, o));
  return t;
}

// Sum of exp(-|x - b|/alpha) over a set of scores, kept relative to the
// nearest distance seen so far (d_min, S: the sum is exp(-d_min/alpha) S), so
// that it underflows only where the fp64 sum itself does.  b = bh + bl as two
// floats; each distance is formed as an unevaluated float pair (error-free
// two-sum), so the differences to d_min that go through the fp32 exp2 are
// exact to about 2^-48 of the distance even when distance/alpha is large.
__device__ __forceinline__ void near_add(float x, float bh, float bl, float c2, float& mh, float& ml, double& S) {
  const float s = x - bh;  // exact near b
  const float nb = -bl;
  float dh = s + nb;
  const float bv = dh - s;
  float dl = (s - (dh - bv)) + (nb - bv);
  if (dh < 0.0f || (dh == 0.0f && dl < 0.0f)) {
    dh = -dh;
    dl = -dl;
  }
  if (dh < mh) {  // a new nearest score: rescale what was accumulated
    S *= (double)exp2f(((dh - mh) + (dl - ml)) * c2);
    mh = dh;
    ml = dl;
  }
  S += (double)exp2f(((mh - dh) + (ml - dl)) * c2);
}
// the nearest distance of a thread's pair as one fp64 value (+inf if none)
__device__ __forceinline__ double near_dist(float mh, float ml) {
  return mh < CUDART_INF_F ? (double)mh + (double)ml : CUDART_INF;
}
// the same pair over a block: every thread gets the block's (d_min, S)
template <int NT>
__device__ __forceinline__ void block_near_reduce(double& dmin, double& S, double inva, double* red) {
  const double M = block_min_double<NT>(dmin, red);
  const double sc = (dmin < CUDART_INF) ? exp_call((M - dmin) * inva) : 0.0;
  S = block_sum<NT, double>(S * sc, red);
  dmin = M;
}

template <int NT>
__device__ __forceinline__ float block_min_float(float v, float* scratch) {
  constexpr int NW = NT / 32;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fminf(v, __shfl_xor_sync(0xffffffffu, v, o));
  __syncthreads();
  if (lane == 0) scratch[warp] = v;
  __syncthreads();
  float t = (lane < NW) ? scratch[lane] : CUDART_INF_F;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) t = fminf(t, __shfl_xor_sync(0xffffffffu, t, o));
  return t;
}

// Combines every thread's (m, S, SG) into the block's, relative to the block
// minimum of m (returned in m of every thread).
template <int NT>
__device__ __forceinline__ void block_shift_reduce(float& m, double& S, double& SG, double* red) {
  const float M = block_min_float<NT>(m, reinterpret_cast<float*>(red));
  const double sc = (m == CUDART_INF_F) ? 0.0 : exp2((double)M - (double)m);
  S = block_sum<NT, double>(S * sc, red);
  SG = block_sum<NT, double>(SG * sc, red);
  m = M;
}

template <int NT>
__device__ __forceinline__ void block_shift_reduce4(float& m, double& S, double& SG, double& SZ, double& SGZ,
                                                    double* red) {
  const float M = block_min_float<NT>(m, reinterpret_cast<float*>(red));
  const double sc = (m == CUDART_INF_F) ? 0.0 : exp2((double)M - (double)m);
  S = block_sum<NT, double>(S * sc, red);
  SG = block_sum<NT, double>(SG * sc, red);
  SZ = block_sum<NT, double>(SZ * sc, red);
  SGZ = block_sum<NT, double>(SGZ * sc, red);
  m = M;
}

// dL/dalpha from the rescaled sums: with a = |r - b| log2(e)/alpha and the
// terms accumulated as 2^(m - a), sum f w = 2^(-m) / (2 alpha) sum 2^(m-a) w,
// and dL/dalpha = -(1/alpha) sum (r - b) f (g - lambda).
__device__ __forceinline__ double alpha_grad(double m, double SZ, double SGZ, double lam, double inva) {
  if (!(m < 1e300)) return 0.0;  // no finite term
  return -inva * 0.5 * inva * exp2(-m) * (SGZ - lam * SZ);
}

// ---------------------------------------------------------------------------
// Classification of a score against the bracket [aL, aR) on the FMA pipe.
// The streaming filter is bound by instruction issue, and compares, selects
// and min/max run on the half-rate ALU pipe; here the left/right indicators
// come from saturating multiplies instead (a saturated product of NaN is 0):
//   L = sat(-(x - aL) 2^126)      1 if x < aL, else 0
//   R = sat(-(aR - x) 2^126 + 1)  1 if x >= aR, else 0
// Every normal difference is at least 2^-126 in magnitude, so the product
// reaches 1; a difference below that is flushed to zero (--ftz), which places
// a score within a subnormal step of an edge on the band's side of it.  A
// score is in the band iff L + R == 0 (NaN lands there).  The tail term is
//   e = exp2(min(min(x - aL, aR - x) c2, 0)),
// which is exp((x - aL)/alpha) on the left and exp((aR - x)/alpha) on the
// right (where the inner min is not positive); the clamp at 0 makes the
// band's (unused) terms 1, so that 0 * e is never 0 * inf.  Both differences
// are formed as they are used (aR - x, not -(x - aR)) and the clamp replaces
// an absolute value, so no operand needs a sign or magnitude change: the
// min/max and exp2 instructions take none for free.
// ---------------------------------------------------------------------------
__device__ __forceinline__ float mul_sat(float a, float b) {
  float r;
  asm("mul.rn.ftz.sat.f32 %0, %1, %2;" : "=f"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ float fma_sat(float a, float b, float c) {
  float r;
  asm("fma.rn.ftz.sat.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}
// Packed fp32x2 arithmetic (two lanes per instruction on sm_100), with
// denormals flushed like the scalar fp32 instructions under --ftz, so that a
// packed and a scalar evaluation of the same formula agree bit for bit.
__device__ __forceinline__ float2 add2(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "add.rn.ftz.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}
__device__ __forceinline__ float2 mul2(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "mul.rn.ftz.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
      "fma.rn.ftz.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return d;
}

struct Side {
  float L, R, e;
};
struct Side2 {  // two scores (packed fp32x2 arithmetic where it exists)
  float2 L, R, e;
};
__device__ __forceinline__ Side classify(float x, float aL, float aR, float c2) {
  const float dl = x - aL;
  const float ndr = aR - x;
  Side s;
  s.L = mul_sat(dl, -0x1p126f);
  s.R = fma_sat(ndr, -0x1p126f, 1.0f);
  s.e = exp2f(fminf(fminf(dl, ndr) * c2, 0.0f));
  return s;
}
// classify for two scores: naL = (-aL, -aL), aR2 = (aR, aR), c22 = (c2, c2).
// The same rounded values as classify (x - aL as x + (-aL); aR - x as one
// fused x * (-1) + aR), so both give identical sides and terms.
__device__ __forceinline__ Side2 classify2(float2 x, float2 naL, float2 aR2, float2 c22) {
  const float2 dl = add2(x, naL);
  const float2 ndr = fma2(x, make_float2(-1.0f, -1.0f), aR2);
  Side2 s;
  s.L = make_float2(mul_sat(dl.x, -0x1p126f), mul_sat(dl.y, -0x1p126f));
  s.R = make_float2(fma_sat(ndr.x, -0x1p126f, 1.0f), fma_sat(ndr.y, -0x1p126f, 1.0f));
  const float2 t = mul2(make_float2(fminf(dl.x, ndr.x), fminf(dl.y, ndr.y)), c22);
  s.e = make_float2(exp2f(fminf(t.x, 0.0f)), exp2f(fminf(t.y, 0.0f)));
  return s;
}

// ---------------------------------------------------------------------------
// Programmatic dependent launch.  The short kernels of the forward pipeline
// are launched with programmatic stream serialization, so that each can be
// scheduled while the kernel ahead of it drains; it waits here, before it
// reads anything that kernel wrote.  Launched without that attribute, this
// returns at once.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void wait_prior_grid() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// ---------------------------------------------------------------------------
// bounded waits.  Every spin in this library gives up after a fixed number
// of polls, records ROW_TIMEOUT and returns, so a logic error can never hang
// the GPU.
// ---------------------------------------------------------------------------
constexpr uint32_t kSpinLimitDefault = 1u << 22;  // x ~256 ns sleeps: about a second

__host__ __device__ __forceinline__ uint32_t spin_limit_of(uint32_t requested) {
  return requested ? requested : kSpinLimitDefault;
}

// Grid-wide barrier for a cooperatively launched grid (all blocks resident):
// waits until `nblocks` blocks have arrived, polling at most `limit` times.
// Returns false if the wait timed out (or another block's did); the caller
// must then stop.
__device__ __forceinline__ bool grid_barrier(uint32_t* count, uint32_t* gen, uint32_t nblocks,
                                             uint32_t* timeout_flag, uint32_t limit) {
  __shared__ uint32_t s_ok;
  __syncthreads();
  if (threadIdx.x == 0) {
    s_ok = 1u;
    volatile uint32_t* vgen = gen;
    const uint32_t my_gen = *vgen;
    __threadfence();
    const uint32_t arrived = atomicAdd(count, 1u);
    if (arrived == nblocks - 1) {
      *count = 0u;
      __threadfence();
      atomicAdd(gen, 1u);
    } else {
      uint32_t polls = 0;
      while (*vgen == my_gen) {
        if (++polls > limit || *((volatile uint32_t*)timeout_flag) != 0u) {
          atomicOr(timeout_flag, 1u);
          s_ok = 0u;
          break;
        }
        __nanosleep(256);
      }
    }
    __threadfence();
  }
  __syncthreads();
  return s_ok != 0u;
}

// last-block-done: returns true in exactly one block (the last to arrive)
__device__ __forceinline__ bool last_block_done(uint32_t* counter, uint32_t nblocks) {
  __shared__ uint32_t s_last;
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) s_last = (atomicAdd(counter, 1u) == nblocks - 1) ? 1u : 0u;
  __syncthreads();
  if (s_last) __threadfence();
  return s_last != 0u;
}

// ---------------------------------------------------------------------------
// streaming loads/stores with cache hints
// ---------------------------------------------------------------------------
__device__ __forceinline__ float4 ldg_stream(const float4* p) { return __ldcs(p); }
__device__ __forceinline__ float4 ldg_keep(const float4* p) { return __ldg(p); }
__device__ __forceinline__ void stg_stream(float4* p, float4 v) { __stcs(p, v); }

}  // namespace lapsum
