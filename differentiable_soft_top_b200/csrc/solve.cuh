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
  __shared__ long long s_ll[4];
  int* iscr = reinterpret_cast<int*>(red);
  long long* lscr = reinterpret_cast<long long*>(red);

  const bool finL = isfinite(in.aL), finR = isfinite(in.aR);
  const Anch left = (finL && in.SL > 0.0) ? Anch{(double)in.aL, in.SL} : anch_empty();
  const Anch right = (finR && in.SR > 0.0) ? Anch{(double)in.aR, in.SR} : anch_empty();

  // prefix direction: A at each group maximum
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

  // suffix direction and the group knot values
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
  __syncthreads();
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

  // certification (arXiv abstract: the bracket is proven, not trusted)
  const Anch pre_all = Anch{s_dbl[0], s_dbl[1]};
  const Anch suf_all = Anch{s_dbl[2], s_dbl[3]};
  const long long M = s_ll[0] - in.nR;
  const double S_aL = finL ? 0.5 * in.SL + (double)(M + in.nR) - 0.5 * suf_at(suf_all, (double)in.aL, inva)
                           : CUDART_INF;
  const double S_aR = finR ? 0.5 * pre_at(pre_all, (double)in.aR, inva) + (double)in.nR - 0.5 * in.SR
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
    } else if (finL) {
      pk->inc_x = (double)in.aL;
      pk->inc_s = in.SL;
    } else {
      pk->inc_x = -CUDART_INF;
      pk->inc_s = 0.0;
    }
    if (tg == INT32_MAX) {
      pk->tg = -1;
      pk->out_x = finR ? (double)in.aR : CUDART_INF;
      pk->out_s = finR ? in.SR : 0.0;
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
  const double xj1 = isfinite(in.aR) ? (double)in.aR : CUDART_INF;
  out->b = closed_form_root(pk.inc_x, xj1, pk.inc_s, pk.out_s, (double)pk.g_after, in.k, in.alpha);
  out->sumf = sum_f_at(pk.inc_x, xj1, pk.inc_s, pk.out_s, out->b, in.inva);
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
  const Anch inc = Anch{pk.inc_x, pk.inc_s};
  const Anch outg = Anch{pk.out_x, pk.out_s};
  const long long g_after = pk.g_after;
  const int qe = (c + NT - 1) / NT;
  const int i0 = min(c, tid * qe), i1 = min(c, i0 + qe);
  Anch lp = anch_empty();
  for (int i = i0; i < i1; ++i) lp = comb_pre(lp, Anch{(double)el.get(i), 1.0}, inva);
  Anch ps = comb_pre(inc, block_excl_scan_anch<NT, true>(lp, inva, red), inva);
  for (int i = i0; i < i1; ++i) {
    ps = comb_pre(ps, Anch{(double)el.get(i), 1.0}, inva);
    dscr[i] = ps.s;  // A_i anchored at y_i
  }
  Anch ls = anch_empty();
  for (int i = i1 - 1; i >= i0; --i) ls = comb_suf(Anch{(double)el.get(i), 1.0}, ls, inva);
  const Anch chunk_in = comb_suf(block_excl_scan_anch<NT, false>(ls, inva, red), outg, inva);
  __syncthreads();  // dscr complete
  Anch sv = chunk_in;
  int icand = -1;
  for (int i = i1 - 1; i >= i0; --i) {
    const double y = (double)el.get(i);
    const double S = 0.5 * dscr[i] + (double)((long long)(c - 1 - i) + g_after) - 0.5 * suf_at(sv, y, inva);
    if (icand < 0 && S >= in.k) icand = i;
    sv = comb_suf(Anch{y, 1.0}, sv, inva);
  }
  const int i_star = block_max_int<NT>(icand, iscr);
  const int jn = i_star + 1;  // right knot index inside the group (c = beyond)
  if (jn < c && jn >= i0 && jn < i1) {
    Anch w = chunk_in;
    for (int i = i1 - 1; i >= jn; --i) w = comb_suf(Anch{(double)el.get(i), 1.0}, w, inva);
    s_bp = w.s;  // B' at y_jn, anchored there
  }
  __syncthreads();
  if (tid == 0) {
    double xj, A, xj1, Bp;
    if (i_star < 0) {
      xj = inc.x;
      A = inc.s;
    } else {
      xj = (double)el.get(i_star);
      A = dscr[i_star];
    }
    if (jn < c) {
      xj1 = (double)el.get(jn);
      Bp = s_bp;
    } else {
      xj1 = (outg.s > 0.0) ? outg.x : (isfinite(in.aR) ? (double)in.aR : CUDART_INF);
      Bp = outg.s;
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
