// solve.cuh -- exact threshold on a sorted band, run by one thread block.
//
// Fast LapSum technical summary, section 2.2: the exact solver runs on the
// band only, with the scores outside the bracket [a_L, a_R) folded into two
// stable tail sums; a certification step checks that b lies in the bracket.
// Section 2.1 fixes the equation: sum_i F((r_i - b)/alpha) = k.
//
// Input: the bracket, the tail aggregates (n_L, S_L anchored at a_L; n_R, S_R
// anchored at a_R), and the band as T groups whose values are sorted inside
// each group and ordered across groups (group t <= group t+1).  With a_L = -inf
// and a_R = +inf and no tails this is the full-sort solver of the same section.
//
// Knot values.  For a sorted value x_j,
//   S(x_j) = A_j/2 + c_j - B_j/2,
// A_j the prefix sum of exp((v - x_j)/alpha) over v <= x_j (left tail
// included), B_j the suffix sum of exp((x_j - v)/alpha) over values after j
// (right tail included), c_j the number of values after j.  S is strictly
// decreasing, so b lies in [x_j*, x_j*+1) for the last knot j* with
// S(x_j*) >= k.  The search is two-level: group maxima first, then the values
// of the one group that holds j*+1.  The root on that interval is the closed
// form of common.cuh.
#pragma once

#include <cstring>

#include "common.cuh"

namespace lapsum {

struct SolveIn {
  float aL, aR;
  long long nL, nR;
  double SL, SR;
  double k, alpha, inva;
};

struct SolveOut {
  uint32_t status;  // ROW_CERTIFIED, or ROW_MISS_LEFT / ROW_MISS_RIGHT
  double b;
  double sumf;      // sum_i f_i at b
  long long M;      // band size (sum of group counts)
  double S_aL, S_aR;
};

// Loads of data that other blocks of the same kernel wrote must skip L1
// (ld.global.cg); kG selects that for global arrays, plain loads otherwise
// (shared memory).
template <bool kG, typename T>
__device__ __forceinline__ T ld(const T* p) {
  if constexpr (kG) return __ldcg(p);
  else return *p;
}

template <int NT>
__device__ __forceinline__ int block_min_int(int v, int* scratch) {
  return -block_max_int<NT>(-v, scratch);
}

// ---------------------------------------------------------------------------
// Anchored sums as affine maps.  Along sorted values y_0 <= y_1 <= ..., the
// prefix sum anchored at the latest value obeys A_i = A_{i-1} f_i + w_i with
// the link factor f_i = exp((y_{i-1} - y_i)/alpha) <= 1, which depends only on
// the values.  Each step is the map v -> v F + S; a run of steps composes to
// one such map, and composition is associative, so the scan across threads is
// FMA-only and every exp is independent of every other.  The suffix direction
// is the same with the roles of left and right swapped.
// ---------------------------------------------------------------------------
struct Aff {
  double F, S;  // v -> v * F + S
};
__device__ __forceinline__ Aff aff_id() { return Aff{1.0, 0.0}; }
// apply a first, then b
__device__ __forceinline__ Aff aff_then(Aff a, Aff b) { return Aff{a.F * b.F, fma(a.S, b.F, b.S)}; }

// Block-wide exclusive scan of affine maps.  kForward: thread t receives the
// composition of threads 0..t-1 (applied in that order); otherwise of threads
// NT-1..t+1 (applied from the right).  scr: >= 2*NT/32 doubles.
template <int NT, bool kForward>
__device__ __forceinline__ Aff block_excl_scan_aff(Aff v, double* scr) {
  constexpr int NW = NT / 32;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  Aff inc = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    Aff oth;
    if (kForward) {
      oth.F = __shfl_up_sync(0xffffffffu, inc.F, o);
      oth.S = __shfl_up_sync(0xffffffffu, inc.S, o);
      if (lane >= o) inc = aff_then(oth, inc);
    } else {
      oth.F = __shfl_down_sync(0xffffffffu, inc.F, o);
      oth.S = __shfl_down_sync(0xffffffffu, inc.S, o);
      if (lane + o < 32) inc = aff_then(oth, inc);
    }
  }
  Aff exl;
  if (kForward) {
    exl.F = __shfl_up_sync(0xffffffffu, inc.F, 1);
    exl.S = __shfl_up_sync(0xffffffffu, inc.S, 1);
    if (lane == 0) exl = aff_id();
  } else {
    exl.F = __shfl_down_sync(0xffffffffu, inc.F, 1);
    exl.S = __shfl_down_sync(0xffffffffu, inc.S, 1);
    if (lane == 31) exl = aff_id();
  }
  __syncthreads();
  if ((kForward && lane == 31) || (!kForward && lane == 0)) {
    scr[2 * warp] = inc.F;
    scr[2 * warp + 1] = inc.S;
  }
  __syncthreads();
  Aff wacc = aff_id();
  if (kForward) {
    for (int w = 0; w < warp; ++w) wacc = aff_then(wacc, Aff{scr[2 * w], scr[2 * w + 1]});
  } else {
    for (int w = NW - 1; w > warp; --w) wacc = aff_then(wacc, Aff{scr[2 * w], scr[2 * w + 1]});
  }
  return aff_then(wacc, exl);
}

// block-wide exclusive scans of anchors: forward max (the last anchor before
// a thread's chunk), backward min (the first anchor after it)
template <int NT, bool kForward>
__device__ __forceinline__ double block_excl_scan_anchor(double v, double init, double* scr) {
  constexpr int NW = NT / 32;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  double inc = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const double oth = kForward ? __shfl_up_sync(0xffffffffu, inc, o) : __shfl_down_sync(0xffffffffu, inc, o);
    if (kForward ? (lane >= o) : (lane + o < 32)) inc = kForward ? fmax(inc, oth) : fmin(inc, oth);
  }
  double exl = kForward ? __shfl_up_sync(0xffffffffu, inc, 1) : __shfl_down_sync(0xffffffffu, inc, 1);
  if (kForward ? lane == 0 : lane == 31) exl = init;
  __syncthreads();
  if (kForward ? lane == 31 : lane == 0) scr[warp] = inc;
  __syncthreads();
  double acc = init;
  if (kForward) {
    for (int w = 0; w < warp; ++w) acc = fmax(acc, scr[w]);
    return fmax(acc, exl);
  } else {
    for (int w = NW - 1; w > warp; --w) acc = fmin(acc, scr[w]);
    return fmin(acc, exl);
  }
}

// link factor exp((from - to)/alpha) for from <= to; 0 when from = -inf (or to = +inf)
__device__ __forceinline__ double link(double from, double to, double inva) {
  return isfinite(from) && isfinite(to) ? exp_call((from - to) * inva) : 0.0;
}

// Result of the group-level step, shared by every thread of the block.
struct GroupPick {
  uint32_t status;     // ROW_CERTIFIED (go on) or ROW_MISS_LEFT / ROW_MISS_RIGHT
  int tg;              // group holding knot j*+1, or -1: b lies in [x_in, a_R)
  double inc_x, inc_s; // prefix state at the knot x_in (the last knot with S >= k
                       // among a_L and the group maxima)
  double out_x, out_s; // suffix state of everything after group tg
  long long g_after;   // number of values after group tg (right tail included)
  long long M;         // band size
  double S_aL, S_aR;
};

// Group level: prefix sums at each group maximum, suffix sums at each group
// minimum, knot values S(ymax_t), certification, and the group that holds the
// knot after the root.  agg[0..T): cnt, ymin, ymax, P, Q filled in (Apre, Bx,
// Bs, after are written).  red: >= 4 * NT/32 + 8 doubles of shared scratch.
// The result is in *pk (shared) on return, in every thread.
template <int NT, bool kG>
__device__ void solve_groups(const SolveIn in, GroupAgg* agg, int T, double* red, GroupPick* pk) {
#define AGG(t, f) ld<kG>(&agg[t].f)
  const double inva = in.inva;
  const int tid = threadIdx.x;
  __shared__ double s_dbl[8];
  __shared__ long long s_ll[2];
  int* iscr = reinterpret_cast<int*>(red);
  long long* lscr = reinterpret_cast<long long*>(red);
  const bool finL = isfinite(in.aL), finR = isfinite(in.aR);
  const double xL = finL ? (double)in.aL : -CUDART_INF;
  const double xR = finR ? (double)in.aR : CUDART_INF;
  const double A0 = finL ? in.SL : 0.0;  // prefix state at a_L
  const double B0 = finR ? in.SR : 0.0;  // suffix state at a_R

  const int q = (T + NT - 1) / NT;
  const int t0 = min(T, tid * q), t1 = min(T, t0 + q);

  // anchors: the last group maximum before the chunk, the first group minimum after it
  double lastmax = -CUDART_INF, firstmin = CUDART_INF;
  long long cloc = 0;
  for (int t = t0; t < t1; ++t) {
    const int c = AGG(t, cnt);
    if (c > 0) {
      lastmax = (double)AGG(t, ymax);
      if (firstmin == CUDART_INF) firstmin = (double)AGG(t, ymin);
      cloc += c;
    }
  }
  const double Xin = block_excl_scan_anchor<NT, true>(lastmax, xL, red);
  const double Yin = block_excl_scan_anchor<NT, false>(firstmin, xR, red);
  const long long cexc = block_excl_suffix_sum<NT>(cloc, lscr);

  // forward: chunk map, scan, then A at every group maximum
  Aff m = aff_id();
  {
    double X = Xin;
    for (int t = t0; t < t1; ++t) {
      if (AGG(t, cnt) > 0) {
        const double ym = (double)AGG(t, ymax);
        m = aff_then(m, Aff{link(X, ym, inva), AGG(t, P)});
        X = ym;
      }
    }
  }
  const Aff fe = block_excl_scan_aff<NT, true>(m, red);
  double A = fma(A0, fe.F, fe.S);  // prefix state at Xin
  {
    double X = Xin;
    for (int t = t0; t < t1; ++t) {
      if (AGG(t, cnt) > 0) {
        const double ym = (double)AGG(t, ymax);
        A = fma(A, link(X, ym, inva), AGG(t, P));
        agg[t].Apre = A;
        X = ym;
      }
    }
    if (tid == NT - 1) {  // prefix over everything below a_R, anchored at X
      s_dbl[0] = X;
      s_dbl[1] = A;
    }
  }

  // backward: chunk map, scan, suffix states, knot values
  Aff mb = aff_id();
  {
    double Y = Yin;
    for (int t = t1 - 1; t >= t0; --t) {
      if (AGG(t, cnt) > 0) {
        const double yn = (double)AGG(t, ymin);
        mb = aff_then(mb, Aff{link(yn, Y, inva), AGG(t, Q)});
        Y = yn;
      }
    }
  }
  const Aff be = block_excl_scan_aff<NT, false>(mb, red);
  double B = fma(B0, be.F, be.S);  // suffix state at Yin
  long long after = cexc + in.nR;
  int cand = -1;
  {
    double Y = Yin;
    for (int t = t1 - 1; t >= t0; --t) {
      agg[t].Bx = Y;
      agg[t].Bs = B;
      agg[t].after = after;
      if (AGG(t, cnt) > 0) {
        const double ym = (double)AGG(t, ymax), yn = (double)AGG(t, ymin);
        const double S = 0.5 * AGG(t, Apre) + (double)after - 0.5 * B * link(ym, Y, inva);
        if (cand < 0 && S >= in.k) cand = t;
        B = fma(B, link(yn, Y, inva), AGG(t, Q));
        Y = yn;
        after += AGG(t, cnt);
      }
    }
    if (tid == 0) {  // suffix over everything at or above a_L, anchored at Y
      s_dbl[2] = Y;
      s_dbl[3] = B;
      s_ll[0] = after;  // M + n_R
    }
  }
  const int t_star = block_max_int<NT>(cand, iscr);
  __syncthreads();

  // certification (arXiv abstract: the bracket is proven, not trusted)
  const long long M = s_ll[0] - in.nR;
  const double S_aL = finL ? 0.5 * in.SL + (double)(M + in.nR) - 0.5 * s_dbl[3] * link(xL, s_dbl[2], inva)
                           : CUDART_INF;
  const double S_aR = finR ? 0.5 * s_dbl[1] * link(s_dbl[0], xR, inva) + (double)in.nR - 0.5 * in.SR
                           : -CUDART_INF;
  const bool cert = (S_aL >= in.k) && (S_aR < in.k);

  // the group that holds knot j*+1
  int tg_loc = INT32_MAX;
  for (int t = t0; t < t1; ++t)
    if (t > t_star && AGG(t, cnt) > 0) { tg_loc = t; break; }
  const int tg = block_min_int<NT>(tg_loc, iscr);
  if (tid == 0) {
    pk->status = cert ? ROW_CERTIFIED
                      : ((!(S_aL >= in.k) ? ROW_MISS_LEFT : 0u) | (!(S_aR < in.k) ? ROW_MISS_RIGHT : 0u));
    pk->M = M;
    pk->S_aL = S_aL;
    pk->S_aR = S_aR;
    if (t_star >= 0) {
      pk->inc_x = (double)AGG(t_star, ymax);
      pk->inc_s = AGG(t_star, Apre);
    } else {
      pk->inc_x = xL;
      pk->inc_s = A0;
    }
    if (tg == INT32_MAX) {
      pk->tg = -1;
      pk->out_x = xR;
      pk->out_s = B0;
      pk->g_after = in.nR;
    } else {
      pk->tg = tg;
      pk->out_x = AGG(tg, Bx);
      pk->out_s = AGG(tg, Bs);
      pk->g_after = AGG(tg, after);
    }
  }
  __syncthreads();
#undef AGG
}

// Root when no value lies above the last group knot: b in [x_in, a_R).
__device__ inline void solve_tail_interval(const SolveIn& in, const GroupPick& pk, SolveOut* out) {
  out->b = closed_form_root(pk.inc_x, pk.out_x, pk.inc_s, pk.out_s, (double)pk.g_after, in.k, in.alpha);
  out->sumf = sum_f_at(pk.inc_x, pk.out_x, pk.inc_s, pk.out_s, out->b, in.inva);
  out->status = ROW_CERTIFIED;
  out->M = pk.M;
  out->S_aL = pk.S_aL;
  out->S_aR = pk.S_aR;
}

// Value level inside the picked group: its c values in ascending order are
// el.get(i); A at each value, the knot after which S drops below k, the
// closed-form root.  dscr: >= c doubles.  Every thread must call it.
template <int NT, typename Vals>
__device__ void solve_values(const SolveIn in, const GroupPick& pk, int c, const Vals& el, double* dscr,
                             double* red, SolveOut* out) {
  const double inva = in.inva;
  const int tid = threadIdx.x;
  __shared__ double s_bp;
  int* iscr = reinterpret_cast<int*>(red);
  const long long g_after = pk.g_after;
  const int qe = ((c + NT - 1) / NT) | 1;  // odd: a warp's chunk starts fall in distinct banks
  const int i0 = min(c, tid * qe), i1 = min(c, i0 + qe);
  const double xprev = (i0 > 0) ? (double)el.get(i0 - 1) : pk.inc_x;   // anchor before the chunk
  const double xnext = (i1 < c) ? (double)el.get(i1) : pk.out_x;       // anchor after the chunk

  // forward: A_i = A_{i-1} f_i + 1
  Aff m = aff_id();
  {
    double X = xprev;
    for (int i = i0; i < i1; ++i) {
      const double y = (double)el.get(i);
      m = aff_then(m, Aff{link(X, y, inva), 1.0});
      X = y;
    }
  }
  const Aff fe = block_excl_scan_aff<NT, true>(m, red);
  {
    double A = fma(pk.inc_s, fe.F, fe.S);  // prefix state at xprev
    double X = xprev;
    for (int i = i0; i < i1; ++i) {
      const double y = (double)el.get(i);
      A = fma(A, link(X, y, inva), 1.0);
      dscr[i] = A;  // A_i anchored at y_i
      X = y;
    }
  }
  // backward: B'_i = B'_{i+1} g_i + 1 (values >= y_i, anchored at y_i)
  Aff mb = aff_id();
  {
    double Y = xnext;
    for (int i = i1 - 1; i >= i0; --i) {
      const double y = (double)el.get(i);
      mb = aff_then(mb, Aff{link(y, Y, inva), 1.0});
      Y = y;
    }
  }
  const Aff be = block_excl_scan_aff<NT, false>(mb, red);
  const double Bin = fma(pk.out_s, be.F, be.S);  // suffix state at xnext
  __syncthreads();  // dscr complete
  int icand = -1;
  {
    double B = Bin, Y = xnext;
    for (int i = i1 - 1; i >= i0; --i) {
      const double y = (double)el.get(i);
      const double S = 0.5 * dscr[i] + (double)((long long)(c - 1 - i) + g_after) - 0.5 * B * link(y, Y, inva);
      if (icand < 0 && S >= in.k) icand = i;
      B = fma(B, link(y, Y, inva), 1.0);
      Y = y;
    }
  }
  const int i_star = block_max_int<NT>(icand, iscr);
  const int jn = i_star + 1;  // right knot index inside the group (c = beyond)
  if (jn < c && jn >= i0 && jn < i1) {
    double B = Bin, Y = xnext;
    for (int i = i1 - 1; i >= jn; --i) {
      const double y = (double)el.get(i);
      B = fma(B, link(y, Y, inva), 1.0);
      Y = y;
    }
    s_bp = B;  // B' at y_jn, anchored there
  }
  __syncthreads();
  if (tid == 0) {
    double xj, A, xj1, Bp;
    if (i_star < 0) {
      xj = pk.inc_x;
      A = pk.inc_s;
    } else {
      xj = (double)el.get(i_star);
      A = dscr[i_star];
    }
    if (jn < c) {
      xj1 = (double)el.get(jn);
      Bp = s_bp;
    } else {
      xj1 = pk.out_x;
      Bp = pk.out_s;
    }
    const double cj = (double)((long long)(c - 1 - i_star) + g_after);
    out->b = closed_form_root(xj, xj1, A, Bp, cj, in.k, in.alpha);
    out->sumf = sum_f_at(xj, xj1, A, Bp, out->b, inva);
    out->status = ROW_CERTIFIED;
    out->M = pk.M;
    out->S_aL = pk.S_aL;
    out->S_aR = pk.S_aR;
  }
  __syncthreads();
}

// ---------------------------------------------------------------------------
// The group level over key bins (the streaming band solve).  Bin t holds the
// values in [e_t, e_{t+1}) of a key window (the top bin also its upper edge).
// States are anchored at the bin edges:
//   prefix  Ahat_{t+1} = sum over values below e_{t+1} of exp((y - e_{t+1})/a)
//                      = Ahat_t s_t + P_t g_t
//   suffix  Bhat_t     = sum over values from e_t on of exp((e_t - y)/a)
//                      = Bhat_{t+1} s_t + Q_t r_t
// with s_t = exp((e_t - e_{t+1})/a), g_t = exp((ymax_t - e_{t+1})/a),
// r_t = exp((e_t - ymin_t)/a), and P_t, Q_t the bin's sums anchored at its own
// maximum and minimum.  Every factor is computed beforehand (in parallel, by
// whoever fills the table), so the solve is exps-free: two scans of affine
// maps and the knot values
//   S(ymax_t) = (Ahat_t h_t + P_t) / 2 + after_t - Bhat_{t+1} g_t / 2,
// h_t = exp((e_t - ymax_t)/a).  Edge states are floating point, so a state
// that underflows stands only for contributions that are negligible next to
// the value-anchored sums (each of which is at least 1).
// ---------------------------------------------------------------------------
template <int NB>
struct BinTable {
  uint32_t cnt[NB];
  float ymin[NB];
  float ymax[NB];
  float eup[NB];  // upper edge e_{t+1}
  double s[NB];   // exp((e_t - e_{t+1})/a)
  double g[NB];   // exp((ymax_t - e_{t+1})/a)
  double h[NB];   // exp((e_t - ymax_t)/a)
  double P[NB];   // sum exp((y - ymax_t)/a)
  double Pg[NB];  // P_t g_t
  double Qr[NB];  // Q_t r_t, Q_t = sum exp((ymin_t - y)/a)
};

template <int Q, typename T>
__device__ __forceinline__ void load_chunk(T (&dst)[Q], const T* src) {
  static_assert((Q * sizeof(T)) % 16 == 0, "chunk must be whole 16-byte words");
  constexpr int V = (int)(Q * sizeof(T) / 16);
  uint4 w[V];
  const uint4* s = reinterpret_cast<const uint4*>(src);
#pragma unroll
  for (int v = 0; v < V; ++v) w[v] = s[v];
  memcpy(dst, w, sizeof(dst));
}

// e0, eN: the first lower edge and the last upper edge of the window (every
// band value of the level lies in [e0, eN]).  Same pick as solve_groups, with
// out_x the upper edge of the picked bin.
template <int NT, int NB>
__device__ __noinline__ void solve_bins(const SolveIn in, const BinTable<NB>& tb, double e0, double eN, double* red,
                           GroupPick* pk) {
  constexpr int Q = NB / NT;
  static_assert(Q >= 4 && NB % NT == 0, "at least four bins per thread");
  const double inva = in.inva;
  const int tid = threadIdx.x;
  __shared__ double s_dbl[2];
  __shared__ long long s_ll[1];
  int* iscr = reinterpret_cast<int*>(red);
  long long* lscr = reinterpret_cast<long long*>(red);
  const bool finL = isfinite(in.aL), finR = isfinite(in.aR);
  const double xL = finL ? (double)in.aL : -CUDART_INF;
  const double xR = finR ? (double)in.aR : CUDART_INF;
  const double tL = finL ? exp_call((xL - e0) * inva) : 0.0;  // a_L -> e0
  const double tR = finR ? exp_call((eN - xR) * inva) : 0.0;  // eN -> a_R
  const double Ah0 = finL ? in.SL * tL : 0.0;            // values below a_L, anchored at e0
  const double BhN = finR ? in.SR * tR : 0.0;            // values from a_R on, anchored at eN
  const int t0 = tid * Q;

  uint32_t cn[Q];
  double sv[Q], pg[Q], qr[Q];
  load_chunk(cn, tb.cnt + t0);
  load_chunk(sv, tb.s + t0);
  load_chunk(pg, tb.Pg + t0);
  load_chunk(qr, tb.Qr + t0);
  long long cloc = 0;
#pragma unroll
  for (int j = 0; j < Q; ++j) cloc += cn[j];
  const long long cexc = block_excl_suffix_sum<NT>(cloc, lscr);

  // forward: edge prefix states
  Aff m = aff_id();
#pragma unroll
  for (int j = 0; j < Q; ++j) m = aff_then(m, Aff{sv[j], pg[j]});
  const Aff fe = block_excl_scan_aff<NT, true>(m, red);
  const double Ah_in = fma(Ah0, fe.F, fe.S);  // at this chunk's lower edge
  double Ah[Q];
  {
    double a = Ah_in;
#pragma unroll
    for (int j = 0; j < Q; ++j) {
      Ah[j] = a;
      a = fma(a, sv[j], pg[j]);
    }
    if (tid == NT - 1) s_dbl[0] = a;  // at eN
  }

  // backward: edge suffix states and the knot values S(ymax_t)
  Aff mb = aff_id();
#pragma unroll
  for (int j = Q - 1; j >= 0; --j) mb = aff_then(mb, Aff{sv[j], qr[j]});
  const Aff be = block_excl_scan_aff<NT, false>(mb, red);
  const double Bh_in = fma(BhN, be.F, be.S);  // at this chunk's upper edge
  double gv[Q], hv[Q], pv[Q];
  load_chunk(gv, tb.g + t0);
  load_chunk(hv, tb.h + t0);
  load_chunk(pv, tb.P + t0);
  int cand = -1;
  {
    double bb = Bh_in;
    long long after = cexc + in.nR;
#pragma unroll
    for (int j = Q - 1; j >= 0; --j) {
      if (cn[j]) {
        const double A = fma(Ah[j], hv[j], pv[j]);
        const double S = 0.5 * A + (double)after - 0.5 * bb * gv[j];
        if (cand < 0 && S >= in.k) cand = t0 + j;
      }
      bb = fma(bb, sv[j], qr[j]);
      after += cn[j];
    }
    if (tid == 0) {
      s_dbl[1] = bb;     // at e0
      s_ll[0] = after;   // M + n_R
    }
  }
  const int t_star = block_max_int<NT>(cand, iscr);

  const long long M = s_ll[0] - in.nR;
  const double S_aL = finL ? 0.5 * in.SL + (double)(M + in.nR) - 0.5 * s_dbl[1] * tL : CUDART_INF;
  const double S_aR = finR ? 0.5 * s_dbl[0] * tR + (double)in.nR - 0.5 * in.SR : -CUDART_INF;
  const bool cert = (S_aL >= in.k) && (S_aR < in.k);

  int tg_loc = INT32_MAX;
#pragma unroll
  for (int j = Q - 1; j >= 0; --j)
    if (t0 + j > t_star && cn[j]) tg_loc = t0 + j;
  const int tg = block_min_int<NT>(tg_loc, iscr);

  // the owners of t* and tg rerun their chunk for the states they hand over
  const bool own_st = t_star >= t0 && t_star < t0 + Q;
  const bool own_tg = tg >= t0 && tg < t0 + Q;
  if (own_st || own_tg) {
    double bb = Bh_in;
    long long after = cexc + in.nR;
#pragma unroll
    for (int j = Q - 1; j >= 0; --j) {
      if (t0 + j == t_star) {
        pk->inc_x = (double)tb.ymax[t0 + j];
        pk->inc_s = fma(Ah[j], hv[j], pv[j]);
      }
      if (t0 + j == tg) {
        pk->out_x = (double)tb.eup[t0 + j];
        pk->out_s = bb;
        pk->g_after = after;
      }
      bb = fma(bb, sv[j], qr[j]);
      after += cn[j];
    }
  }
  if (tid == 0) {
    pk->status = cert ? ROW_CERTIFIED
                      : ((!(S_aL >= in.k) ? ROW_MISS_LEFT : 0u) | (!(S_aR < in.k) ? ROW_MISS_RIGHT : 0u));
    pk->M = M;
    pk->S_aL = S_aL;
    pk->S_aR = S_aR;
    pk->tg = (tg == INT32_MAX) ? -1 : tg;
    if (t_star < 0) {
      pk->inc_x = xL;
      pk->inc_s = finL ? in.SL : 0.0;
    }
    if (tg == INT32_MAX) {
      pk->out_x = xR;
      pk->out_s = finR ? in.SR : 0.0;
      pk->g_after = in.nR;
    }
  }
  __syncthreads();
}

// Both levels, for groups whose values are already sorted and readable
// through el.get(g, i).
template <int NT, bool kG, typename Elems>
__device__ void solve_band(const SolveIn in, GroupAgg* agg, int T, const Elems& el, double* dscr, double* red,
                           SolveOut* out) {
  __shared__ GroupPick pk;
  solve_groups<NT, kG>(in, agg, T, red, &pk);
  if (pk.status != ROW_CERTIFIED) {
    if (threadIdx.x == 0) {
      out->status = pk.status;
      out->b = 0.0;
      out->sumf = 0.0;
      out->M = pk.M;
      out->S_aL = pk.S_aL;
      out->S_aR = pk.S_aR;
    }
    __syncthreads();
    return;
  }
  if (pk.tg < 0) {
    if (threadIdx.x == 0) solve_tail_interval(in, pk, out);
    __syncthreads();
    return;
  }
  struct One {
    const Elems& e;
    int g;
    __device__ float get(int i) const { return e.get(g, i); }
  };
  solve_values<NT>(in, pk, ld<kG>(&agg[pk.tg].cnt), One{el, pk.tg}, dscr, red, out);
}

// One sorted run (the one-block path's band, keys[0, M) in shared memory):
// the value level over the whole band at once, with the certification taken
// from the same two scans.  Writing y_{-1} = a_L and y_M = a_R, the link
// factors l_i = exp((y_{i-1} - y_i)/alpha), i = 0..M, are computed once
// (dL[0, M]); A_i = A_{i-1} l_i + 1 starts from S_L at a_L, and the suffix
// B_i = B_{i+1} l_{i+1} + 1 (values >= y_i, anchored at y_i) from S_R at a_R.
// Then S(y_i) = A_i/2 + (M - 1 - i + n_R) - B_{i+1} l_{i+1}/2, and at the
// bracket edges S(a_L) = S_L/2 + M + n_R - B_0 l_0/2, S(a_R) = A_{M-1} l_M/2 +
// n_R - S_R/2 (with B_0 = S_R, A_{M-1} = S_L when M = 0).  dA: >= M doubles,
// dL: >= M + 1 doubles.  Every thread must call it; *out in shared memory.
template <int NT>
__device__ void solve_run(const SolveIn in, const uint32_t* keys, int M, double* dA, double* dL, double* red,
                          SolveOut* out) {
  const double inva = in.inva;
  const int tid = threadIdx.x;
  __shared__ double s_edge[2];  // B_0, A_{M-1}
  __shared__ double s_bp;
  int* iscr = reinterpret_cast<int*>(red);
  const bool finL = isfinite(in.aL), finR = isfinite(in.aR);
  const double xL = finL ? (double)in.aL : -CUDART_INF;
  const double xR = finR ? (double)in.aR : CUDART_INF;
  const double A0 = finL ? in.SL : 0.0;  // prefix state at a_L
  const double B0 = finR ? in.SR : 0.0;  // suffix state at a_R
  auto y = [&](int i) -> double { return i < 0 ? xL : (i >= M ? xR : (double)key2f(keys[i])); };
  for (int i = tid; i <= M; i += NT) dL[i] = link(y(i - 1), y(i), inva);
  if (tid == 0) {
    s_edge[0] = B0;
    s_edge[1] = A0;
  }
  __syncthreads();
  // contiguous chunks of an odd length: the threads of a warp, stepping
  // through their chunks together, touch distinct shared-memory banks
  const int qe = ((M + NT - 1) / NT) | 1;
  const int i0 = min(M, tid * qe), i1 = min(M, i0 + qe);

  // forward: chunk map, scan, A at every value
  Aff m = aff_id();
  for (int i = i0; i < i1; ++i) m = aff_then(m, Aff{dL[i], 1.0});
  const Aff fe = block_excl_scan_aff<NT, true>(m, red);
  {
    double A = fma(A0, fe.F, fe.S);  // prefix state at y_{i0 - 1}
    for (int i = i0; i < i1; ++i) {
      A = fma(A, dL[i], 1.0);
      dA[i] = A;
    }
    if (i1 == M && i1 > i0) s_edge[1] = A;
  }
  // backward: chunk map, scan, knot values
  Aff mb = aff_id();
  for (int i = i1 - 1; i >= i0; --i) mb = aff_then(mb, Aff{dL[i + 1], 1.0});
  const Aff be = block_excl_scan_aff<NT, false>(mb, red);
  const double Bin = fma(B0, be.F, be.S);  // B_{i1}, anchored at y_{i1}
  int icand = -1;
  {
    double B = Bin;
    for (int i = i1 - 1; i >= i0; --i) {
      const double S = 0.5 * dA[i] + (double)((long long)(M - 1 - i) + in.nR) - 0.5 * B * dL[i + 1];
      if (icand < 0 && S >= in.k) icand = i;
      B = fma(B, dL[i + 1], 1.0);
    }
    if (i0 == 0 && i1 > 0) s_edge[0] = B;
  }
  const int i_star = block_max_int<NT>(icand, iscr);  // its barriers publish s_edge
  const int jn = i_star + 1;
  if (jn < M && jn >= i0 && jn < i1) {
    double B = Bin;
    for (int i = i1 - 1; i >= jn; --i) B = fma(B, dL[i + 1], 1.0);
    s_bp = B;  // B_jn
  }
  __syncthreads();
  if (tid == 0) {
    const double S_aL = finL ? 0.5 * in.SL + (double)((long long)M + in.nR) - 0.5 * s_edge[0] * dL[0] : CUDART_INF;
    const double S_aR = finR ? 0.5 * s_edge[1] * dL[M] + (double)in.nR - 0.5 * in.SR : -CUDART_INF;
    out->M = M;
    out->S_aL = S_aL;
    out->S_aR = S_aR;
    if (S_aL >= in.k && S_aR < in.k) {
      const double xj = i_star < 0 ? xL : y(i_star);
      const double A = i_star < 0 ? A0 : dA[i_star];
      const double xj1 = jn < M ? y(jn) : xR;
      const double Bp = jn < M ? s_bp : B0;
      const double cj = (double)((long long)(M - 1 - i_star) + in.nR);
      out->b = closed_form_root(xj, xj1, A, Bp, cj, in.k, in.alpha);
      out->sumf = sum_f_at(xj, xj1, A, Bp, out->b, inva);
      out->status = ROW_CERTIFIED;
    } else {
      out->b = 0.0;
      out->sumf = 0.0;
      out->status = (!(S_aL >= in.k) ? ROW_MISS_LEFT : 0u) | (!(S_aR < in.k) ? ROW_MISS_RIGHT : 0u);
    }
  }
  __syncthreads();
}

// Warp-wide exclusive scan of affine maps (the shuffle part of
// block_excl_scan_aff): lane l receives the composition of lanes 0..l-1
// (kForward) or of lanes 31..l+1.
template <bool kForward>
__device__ __forceinline__ Aff warp_excl_scan_aff(Aff v) {
  const int lane = threadIdx.x & 31;
  Aff inc = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    Aff oth;
    if (kForward) {
      oth.F = __shfl_up_sync(0xffffffffu, inc.F, o);
      oth.S = __shfl_up_sync(0xffffffffu, inc.S, o);
      if (lane >= o) inc = aff_then(oth, inc);
    } else {
      oth.F = __shfl_down_sync(0xffffffffu, inc.F, o);
      oth.S = __shfl_down_sync(0xffffffffu, inc.S, o);
      if (lane + o < 32) inc = aff_then(oth, inc);
    }
  }
  Aff exl;
  if (kForward) {
    exl.F = __shfl_up_sync(0xffffffffu, inc.F, 1);
    exl.S = __shfl_up_sync(0xffffffffu, inc.S, 1);
    if (lane == 0) exl = aff_id();
  } else {
    exl.F = __shfl_down_sync(0xffffffffu, inc.F, 1);
    exl.S = __shfl_down_sync(0xffffffffu, inc.S, 1);
    if (lane == 31) exl = aff_id();
  }
  return exl;
}

// solve_run with its scans taken by one warp: the whole block computes the
// link factors (the exps), then warp 0 walks the run in 32 chunks, with
// shuffles instead of block barriers between its phases.  The same
// recurrences, knot values, certification and closed form as solve_run; only
// the chunking, hence the rounding order of the compositions, differs.  For
// the one-block rows, where other blocks on the SM keep the issue slots busy
// while the other warps wait.  dA: >= M doubles, dL: >= M + 1 doubles.  Every
// thread must call it; *out in shared memory.
template <int NT>
__device__ void solve_run_warp(const SolveIn in, const uint32_t* keys, int M, double* dA, double* dL,
                               SolveOut* out) {
  const double inva = in.inva;
  const bool finL = isfinite(in.aL), finR = isfinite(in.aR);
  const double xL = finL ? (double)in.aL : -CUDART_INF;
  const double xR = finR ? (double)in.aR : CUDART_INF;
  const double A0 = finL ? in.SL : 0.0;  // prefix state at a_L
  const double B0 = finR ? in.SR : 0.0;  // suffix state at a_R
  auto y = [&](int i) -> double { return i < 0 ? xL : (i >= M ? xR : (double)key2f(keys[i])); };
  for (int i = threadIdx.x; i <= M; i += NT) dL[i] = link(y(i - 1), y(i), inva);
  __syncthreads();
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    // odd chunk lengths: the lanes' chunk starts fall in distinct banks
    const int qe = ((M + 31) / 32) | 1;
    const int i0 = min(M, lane * qe), i1 = min(M, i0 + qe);
    // forward: chunk map, scan, A at every value
    Aff m = aff_id();
    for (int i = i0; i < i1; ++i) m = aff_then(m, Aff{dL[i], 1.0});
    const Aff fe = warp_excl_scan_aff<true>(m);
    double A = fma(A0, fe.F, fe.S);  // prefix state at y_{i0 - 1}
    for (int i = i0; i < i1; ++i) {
      A = fma(A, dL[i], 1.0);
      dA[i] = A;
    }
    // A_{M-1} (A0 when M = 0) from the lane whose chunk ends the run
    const double Alast = M > 0 ? __shfl_sync(0xffffffffu, A, (M - 1) / qe) : A0;
    // backward: chunk map, scan, knot values
    Aff mb = aff_id();
    for (int i = i1 - 1; i >= i0; --i) mb = aff_then(mb, Aff{dL[i + 1], 1.0});
    const Aff be = warp_excl_scan_aff<false>(mb);
    const double Bin = fma(B0, be.F, be.S);  // B_{i1}, anchored at y_{i1}
    int icand = -1;
    double B = Bin;
    for (int i = i1 - 1; i >= i0; --i) {
      const double S = 0.5 * dA[i] + (double)((long long)(M - 1 - i) + in.nR) - 0.5 * B * dL[i + 1];
      if (icand < 0 && S >= in.k) icand = i;
      B = fma(B, dL[i + 1], 1.0);
    }
    const double Bfirst = M > 0 ? __shfl_sync(0xffffffffu, B, 0) : B0;  // B_0
    const int i_star = __reduce_max_sync(0xffffffffu, icand);
    const int jn = i_star + 1;
    // B_jn from the lane whose chunk holds jn
    double Bj = Bin;
    if (jn < M && jn >= i0 && jn < i1)
      for (int i = i1 - 1; i >= jn; --i) Bj = fma(Bj, dL[i + 1], 1.0);
    const double Bp_run = __shfl_sync(0xffffffffu, Bj, jn < M ? jn / qe : 0);
    __syncwarp();  // dA of every lane visible to lane 0
    if (lane == 0) {
      const double S_aL = finL ? 0.5 * in.SL + (double)((long long)M + in.nR) - 0.5 * Bfirst * dL[0] : CUDART_INF;
      const double S_aR = finR ? 0.5 * Alast * dL[M] + (double)in.nR - 0.5 * in.SR : -CUDART_INF;
      out->M = M;
      out->S_aL = S_aL;
      out->S_aR = S_aR;
      if (S_aL >= in.k && S_aR < in.k) {
        const double xj = i_star < 0 ? xL : y(i_star);
        const double Ai = i_star < 0 ? A0 : dA[i_star];
        const double xj1 = jn < M ? y(jn) : xR;
        const double Bp = jn < M ? Bp_run : B0;
        const double cj = (double)((long long)(M - 1 - i_star) + in.nR);
        out->b = closed_form_root(xj, xj1, Ai, Bp, cj, in.k, in.alpha);
        out->sumf = sum_f_at(xj, xj1, Ai, Bp, out->b, inva);
        out->status = ROW_CERTIFIED;
      } else {
        out->b = 0.0;
        out->sumf = 0.0;
        out->status = (!(S_aL >= in.k) ? ROW_MISS_LEFT : 0u) | (!(S_aR < in.k) ? ROW_MISS_RIGHT : 0u);
      }
    }
  }
  __syncthreads();
}

template <int NT>
__device__ __forceinline__ uint32_t block_minmax_u32(uint32_t v, bool is_max, uint32_t* scratch) {
  constexpr int NW = NT / 32;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  v = is_max ? __reduce_max_sync(0xffffffffu, v) : __reduce_min_sync(0xffffffffu, v);
  __syncthreads();
  if (lane == 0) scratch[warp] = v;
  __syncthreads();
  uint32_t t = (lane < NW) ? scratch[lane] : (is_max ? 0u : 0xFFFFFFFFu);
  return is_max ? __reduce_max_sync(0xffffffffu, t) : __reduce_min_sync(0xffffffffu, t);
}

// Aggregates of one unsorted group whose values other blocks wrote to global
// memory (so they are read around L1): count, min, max, and the anchored sums
// P = sum exp((y - ymax)/alpha), Q = sum exp((ymin - y)/alpha).  Every term
// lies in (0, 1]; the sums are taken in 2^-40 fixed point, which makes them
// independent of the order in which the values arrived (run-to-run
// determinism) at an absolute error below cnt * 2^-41.
template <int NT>
__device__ void aggregate_unsorted(const float* vals, int cnt, double inva, double* red, GroupAgg* out) {
  uint32_t kmin = 0xFFFFFFFFu, kmax = 0u;
  for (int i = threadIdx.x; i < cnt; i += NT) {
    const uint32_t k = f2key(__ldcg(vals + i));
    kmin = min(kmin, k);
    kmax = max(kmax, k);
  }
  kmin = block_minmax_u32<NT>(kmin, false, reinterpret_cast<uint32_t*>(red));
  kmax = block_minmax_u32<NT>(kmax, true, reinterpret_cast<uint32_t*>(red));
  const double ymin = (double)key2f(kmin), ymax = (double)key2f(kmax);
  long long P = 0, Q = 0;
  for (int i = threadIdx.x; i < cnt; i += NT) {
    const double y = (double)__ldcg(vals + i);
    P += llrint(exp((y - ymax) * inva) * 0x1p40);
    Q += llrint(exp((ymin - y) * inva) * 0x1p40);
  }
  P = block_sum<NT, long long>(P, reinterpret_cast<long long*>(red));
  Q = block_sum<NT, long long>(Q, reinterpret_cast<long long*>(red));
  if (threadIdx.x == 0) {
    out->cnt = cnt;
    out->ymin = cnt > 0 ? (float)ymin : 0.0f;
    out->ymax = cnt > 0 ? (float)ymax : 0.0f;
    out->P = (double)P * 0x1p-40;
    out->Q = (double)Q * 0x1p-40;
  }
  __syncthreads();
}

// Aggregates of an already sorted run held as keys.
template <int NT, bool kG>
__device__ void aggregate_sorted_keys(const uint32_t* keys, int n, double* red, GroupAgg* out,
                                      double inva) {
  __shared__ float s_mm[2];
  if (threadIdx.x == 0 && n > 0) {
    s_mm[0] = key2f(ld<kG>(keys));
    s_mm[1] = key2f(ld<kG>(keys + n - 1));
  }
  __syncthreads();
  const double ymin = n > 0 ? (double)s_mm[0] : 0.0, ymax = n > 0 ? (double)s_mm[1] : 0.0;
  double P = 0.0, Q = 0.0;
  for (int i = threadIdx.x; i < n; i += NT) {
    const double y = (double)key2f(ld<kG>(keys + i));
    P += exp((y - ymax) * inva);
    Q += exp((ymin - y) * inva);
  }
  P = block_sum<NT, double>(P, red);
  Q = block_sum<NT, double>(Q, red);
  if (threadIdx.x == 0) {
    out->cnt = n;
    out->ymin = n > 0 ? s_mm[0] : 0.0f;
    out->ymax = n > 0 ? s_mm[1] : 0.0f;
    out->P = P;
    out->Q = Q;
  }
  __syncthreads();
}

}  // namespace lapsum
