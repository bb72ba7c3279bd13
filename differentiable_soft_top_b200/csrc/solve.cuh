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

// Elems: float get(int g, int i) returns value i of group g.
// agg[0..T): cnt, ymin, ymax, P, Q filled in; Apre/Bx/Bs/after are written.
// dscr: >= (largest group count) doubles of scratch (shared or global).
// red:  >= 4 * NT/32 + 8 doubles of shared scratch.
// The result is valid in every thread on return.
template <int NT, bool kG, typename Elems>
__device__ void solve_band(const SolveIn in, GroupAgg* agg, int T, const Elems& el,
                           double* dscr, double* red, SolveOut* out) {
#define AGG(t, f) ld<kG>(&agg[t].f)
  const double inva = in.inva;
  const int tid = threadIdx.x;
  __shared__ double s_dbl[8];
  __shared__ long long s_ll[4];
  int* iscr = reinterpret_cast<int*>(red);
  long long* lscr = reinterpret_cast<long long*>(red);

  const bool finL = isfinite(in.aL), finR = isfinite(in.aR);
  const Anch left = (finL && in.SL > 0.0) ? Anch{(double)in.aL, in.SL} : anch_empty();
  const Anch right = (finR && in.SR > 0.0) ? Anch{(double)in.aR, in.SR} : anch_empty();

  // ---- group level, prefix direction: A at each group maximum ----------
  const int q = (T + NT - 1) / NT;
  const int t0 = min(T, tid * q), t1 = min(T, t0 + q);
  Anch loc = anch_empty();
  for (int t = t0; t < t1; ++t)
    if (AGG(t, cnt) > 0) loc = comb_pre(loc, Anch{(double)AGG(t, ymax), AGG(t, P)}, inva);
  Anch st = comb_pre(left, block_excl_scan_anch<NT, true>(loc, inva, red), inva);
  for (int t = t0; t < t1; ++t) {
    if (AGG(t, cnt) > 0) {
      st = comb_pre(st, Anch{(double)AGG(t, ymax), AGG(t, P)}, inva);
      agg[t].Apre = st.s;
    }
  }
  if (tid == NT - 1) {  // prefix over everything below a_R
    s_dbl[0] = st.x;
    s_dbl[1] = st.s;
  }

  // ---- group level, suffix direction, and the group knot values ---------
  Anch sloc = anch_empty();
  long long cloc = 0;
  for (int t = t1 - 1; t >= t0; --t) {
    if (AGG(t, cnt) > 0) {
      sloc = comb_suf(Anch{(double)AGG(t, ymin), AGG(t, Q)}, sloc, inva);
      cloc += AGG(t, cnt);
    }
  }
  const Anch sexc = block_excl_scan_anch<NT, false>(sloc, inva, red);
  const long long cexc = block_excl_suffix_sum<NT>(cloc, lscr);
  __syncthreads();  // agg[].Apre of every thread is visible below
  Anch ss = comb_suf(sexc, right, inva);
  long long after = cexc + in.nR;
  int cand = -1;
  for (int t = t1 - 1; t >= t0; --t) {
    agg[t].Bx = ss.x;
    agg[t].Bs = ss.s;
    agg[t].after = after;
    if (AGG(t, cnt) > 0) {
      const double ymax = (double)AGG(t, ymax);
      const double S = 0.5 * AGG(t, Apre) + (double)after - 0.5 * suf_at(ss, ymax, inva);
      if (cand < 0 && S >= in.k) cand = t;
      ss = comb_suf(Anch{(double)AGG(t, ymin), AGG(t, Q)}, ss, inva);
      after += AGG(t, cnt);
    }
  }
  if (tid == 0) {  // suffix over everything at or above a_L
    s_dbl[2] = ss.x;
    s_dbl[3] = ss.s;
    s_ll[0] = after;  // M + n_R
  }
  const int t_star = block_max_int<NT>(cand, iscr);
  __syncthreads();

  // ---- certification (arXiv abstract: the bracket is proven, not trusted) --
  const Anch pre_all = Anch{s_dbl[0], s_dbl[1]};
  const Anch suf_all = Anch{s_dbl[2], s_dbl[3]};
  const long long M = s_ll[0] - in.nR;
  const double S_aL = finL ? 0.5 * in.SL + (double)(M + in.nR) - 0.5 * suf_at(suf_all, (double)in.aL, inva)
                           : CUDART_INF;
  const double S_aR = finR ? 0.5 * pre_at(pre_all, (double)in.aR, inva) + (double)in.nR - 0.5 * in.SR
                           : -CUDART_INF;
  if (!(S_aL >= in.k) || !(S_aR < in.k)) {
    if (tid == 0) {
      out->status = (!(S_aL >= in.k) ? ROW_MISS_LEFT : 0u) | (!(S_aR < in.k) ? ROW_MISS_RIGHT : 0u);
      out->b = 0.0;
      out->sumf = 0.0;
      out->M = M;
      out->S_aL = S_aL;
      out->S_aR = S_aR;
    }
    __syncthreads();
    return;
  }

  // ---- the group that holds knot j*+1 -----------------------------------
  int tg_loc = INT32_MAX;
  for (int t = t0; t < t1; ++t)
    if (t > t_star && AGG(t, cnt) > 0) { tg_loc = t; break; }
  const int tg = block_min_int<NT>(tg_loc, iscr);
  Anch inc;  // prefix state up to and including knot x_in (anchored there)
  if (t_star >= 0) inc = Anch{(double)AGG(t_star, ymax), AGG(t_star, Apre)};
  else inc = finL ? Anch{(double)in.aL, in.SL} : Anch{-CUDART_INF, 0.0};

  if (tg == INT32_MAX) {
    // no values above the last knot: b in [x_in, a_R)
    if (tid == 0) {
      const double xj1 = finR ? (double)in.aR : CUDART_INF;
      const double Bp = finR ? in.SR : 0.0;
      out->b = closed_form_root(inc.x, xj1, inc.s, Bp, (double)in.nR, in.k, in.alpha);
      out->sumf = sum_f_at(inc.x, xj1, inc.s, Bp, out->b, inva);
      out->status = ROW_CERTIFIED;
      out->M = M;
      out->S_aL = S_aL;
      out->S_aR = S_aR;
    }
    __syncthreads();
    return;
  }

  // ---- value level inside group tg -------------------------------------
  const int c = AGG(tg, cnt);
  const Anch outg = Anch{AGG(tg, Bx), AGG(tg, Bs)};
  const long long g_after = AGG(tg, after);
  const int qe = (c + NT - 1) / NT;
  const int i0 = min(c, tid * qe), i1 = min(c, i0 + qe);
  Anch lp = anch_empty();
  for (int i = i0; i < i1; ++i) lp = comb_pre(lp, Anch{(double)el.get(tg, i), 1.0}, inva);
  Anch ps = comb_pre(inc, block_excl_scan_anch<NT, true>(lp, inva, red), inva);
  for (int i = i0; i < i1; ++i) {
    ps = comb_pre(ps, Anch{(double)el.get(tg, i), 1.0}, inva);
    dscr[i] = ps.s;  // A_i anchored at y_i
  }
  Anch ls = anch_empty();
  for (int i = i1 - 1; i >= i0; --i) ls = comb_suf(Anch{(double)el.get(tg, i), 1.0}, ls, inva);
  const Anch chunk_in = comb_suf(block_excl_scan_anch<NT, false>(ls, inva, red), outg, inva);
  __syncthreads();  // dscr complete
  Anch sv = chunk_in;
  int icand = -1;
  for (int i = i1 - 1; i >= i0; --i) {
    const double y = (double)el.get(tg, i);
    const double S = 0.5 * dscr[i] + (double)((long long)(c - 1 - i) + g_after) - 0.5 * suf_at(sv, y, inva);
    if (icand < 0 && S >= in.k) icand = i;
    sv = comb_suf(Anch{y, 1.0}, sv, inva);
  }
  const int i_star = block_max_int<NT>(icand, iscr);
  const int jn = i_star + 1;  // right knot index inside the group (c = beyond)
  if (jn < c && jn >= i0 && jn < i1) {
    Anch w = chunk_in;
    for (int i = i1 - 1; i >= jn; --i) w = comb_suf(Anch{(double)el.get(tg, i), 1.0}, w, inva);
    s_dbl[4] = w.s;  // B' at y_jn, anchored there
  }
  __syncthreads();
  if (tid == 0) {
    double xj, A, xj1, Bp;
    if (i_star < 0) {
      xj = inc.x;
      A = inc.s;
    } else {
      xj = (double)el.get(tg, i_star);
      A = dscr[i_star];
    }
    if (jn < c) {
      xj1 = (double)el.get(tg, jn);
      Bp = s_dbl[4];
    } else {
      xj1 = (outg.s > 0.0) ? outg.x : (finR ? (double)in.aR : CUDART_INF);
      Bp = outg.s;
    }
    const double cj = (double)((long long)(c - 1 - i_star) + g_after);
    out->b = closed_form_root(xj, xj1, A, Bp, cj, in.k, in.alpha);
    out->sumf = sum_f_at(xj, xj1, A, Bp, out->b, inva);
    out->status = ROW_CERTIFIED;
    out->M = M;
    out->S_aL = S_aL;
    out->S_aR = S_aR;
  }
  __syncthreads();
#undef AGG
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
