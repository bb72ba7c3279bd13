// warp_solve.cuh -- one warp sorts the key bin that holds the root and solves
// the budget equation on it (Fast LapSum technical summary, section 2.2: the
// exact solver applied to the values near the threshold only).
//
// Everything stays in registers and shuffles: no block barrier is involved,
// which is what makes the last step of the band solve short.
#pragma once

#include "common.cuh"
#include "solve.cuh"

namespace lapsum {

// keys per lane of the warp sort; the warp handles buckets of up to 32*kWarpKeys
constexpr int kWarpKeys = 8;
constexpr int kWarpSortMax = 32 * kWarpKeys;

// Compare-exchange of the register pairs (r, r + RJ) of one lane for stage kk
// of the bitonic network (the partner sits in the same lane).
template <int RJ>
__device__ __forceinline__ void warp_bitonic_regs(uint32_t (&k)[kWarpKeys], int kk, int lane) {
#pragma unroll
  for (int r = 0; r < kWarpKeys; ++r) {
    if ((r & RJ) == 0) {
      const int e = r * 32 + lane;
      const uint32_t a = k[r], b = k[r | RJ];
      const bool asc = (e & kk) == 0;
      k[r] = asc ? min(a, b) : max(a, b);
      k[r | RJ] = asc ? max(a, b) : min(a, b);
    }
  }
}

// Bitonic network over 32*kWarpKeys keys held as k[r] = element r*32 + lane.
// Pads (0xFFFFFFFF) sort to the end.  The stage loops are not unrolled: this
// runs once per row, and compact code is what keeps it fast.
__device__ __forceinline__ void warp_bitonic_sort(uint32_t (&k)[kWarpKeys]) {
  static_assert(kWarpKeys == 8, "the cross-register stages below cover 8 keys per lane");
  const int lane = threadIdx.x & 31;
  constexpr int N = 32 * kWarpKeys;
#pragma unroll 1
  for (int kk = 2; kk <= N; kk <<= 1) {
#pragma unroll 1
    for (int j = kk >> 1; j > 0; j >>= 1) {
      if (j < 32) {
#pragma unroll
        for (int r = 0; r < kWarpKeys; ++r) {
          const int e = r * 32 + lane;
          const uint32_t o = __shfl_xor_sync(0xffffffffu, k[r], j);
          const bool take_min = ((e & j) == 0) == ((e & kk) == 0);
          k[r] = take_min ? min(k[r], o) : max(k[r], o);
        }
      } else if (j == 32) {
        warp_bitonic_regs<1>(k, kk, lane);
      } else if (j == 64) {
        warp_bitonic_regs<2>(k, kk, lane);
      } else {
        warp_bitonic_regs<4>(k, kk, lane);
      }
    }
  }
}

// warp-wide exclusive scan of affine maps (forward: lanes < l; backward: lanes > l)
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

// Sorts the c <= kWarpSortMax keys of one bin (unsorted, in shared memory)
// and solves on their values, given the group-level pick: the same result as
// sorting and calling solve_values.  Must be called by one full warp.  `spill`
// is kWarpSortMax words of shared memory used to hand the sorted keys from
// the network layout to contiguous lane chunks.  Lane 0 writes the result.
__device__ inline void warp_solve_bin(const SolveIn& in, const GroupPick& pk, const uint32_t* keys, int c,
                                      uint32_t* spill, SolveOut* out) {
  const int lane = threadIdx.x & 31;
  const double inva = in.inva;
  uint32_t k[kWarpKeys];
#pragma unroll
  for (int r = 0; r < kWarpKeys; ++r) {
    const int e = r * 32 + lane;
    k[r] = (e < c) ? keys[e] : 0xFFFFFFFFu;
  }
  warp_bitonic_sort(k);
#pragma unroll
  for (int r = 0; r < kWarpKeys; ++r) spill[r * 32 + lane] = k[r];
  __syncwarp();
  // lane l now owns the contiguous sorted values [l*kWarpKeys, (l+1)*kWarpKeys)
  const int i0 = lane * kWarpKeys;
  double y[kWarpKeys];
#pragma unroll
  for (int r = 0; r < kWarpKeys; ++r) y[r] = (double)key2f(spill[i0 + r]);
  const double xprev = (i0 > 0 && i0 - 1 < c) ? (double)key2f(spill[i0 - 1]) : pk.inc_x;
  const double xnext = (i0 + kWarpKeys < c) ? (double)key2f(spill[i0 + kWarpKeys]) : pk.out_x;
  // link factors: f[r] joins value r-1 (or xprev) to value r; fl joins the
  // last owned value to xnext.  All independent.
  double f[kWarpKeys];
#pragma unroll
  for (int r = 0; r < kWarpKeys; ++r) f[r] = (i0 + r < c) ? link(r == 0 ? xprev : y[r - 1], y[r], inva) : 1.0;
  const int last = min(c - i0, kWarpKeys) - 1;  // index of the last owned value, < 0 if none
  double ylast = 0.0;
#pragma unroll
  for (int r = 0; r < kWarpKeys; ++r)
    if (r == last) ylast = y[r];
  const double fl = (last >= 0) ? link(ylast, xnext, inva) : 1.0;

  // forward: A_i = A_{i-1} f_i + 1
  Aff m = aff_id();
#pragma unroll
  for (int r = 0; r < kWarpKeys; ++r)
    if (i0 + r < c) m = aff_then(m, Aff{f[r], 1.0});
  const Aff fe = warp_excl_scan_aff<true>(m);
  double A[kWarpKeys];
  {
    double a = fma(pk.inc_s, fe.F, fe.S);
#pragma unroll
    for (int r = 0; r < kWarpKeys; ++r) {
      if (i0 + r < c) a = fma(a, f[r], 1.0);
      A[r] = a;
    }
  }
  // backward: B'_i = B'_{i+1} g_i + 1, g_i the link from value i to the next one
  Aff mb = aff_id();
#pragma unroll
  for (int r = kWarpKeys - 1; r >= 0; --r) {
    if (i0 + r < c) mb = aff_then(mb, Aff{r == last ? fl : f[r + 1 < kWarpKeys ? r + 1 : r], 1.0});
  }
  const Aff be = warp_excl_scan_aff<false>(mb);
  const double Bin = fma(pk.out_s, be.F, be.S);  // suffix state at xnext
  int icand = -1;
  double Bp[kWarpKeys];  // B' at each owned value
  {
    double bs = Bin;
#pragma unroll
    for (int r = kWarpKeys - 1; r >= 0; --r) {
      if (i0 + r < c) {
        const double g = (r == last) ? fl : f[r + 1 < kWarpKeys ? r + 1 : r];
        const double S = 0.5 * A[r] + (double)((long long)(c - 1 - (i0 + r)) + pk.g_after) - 0.5 * bs * g;
        if (icand < 0 && S >= in.k) icand = i0 + r;
        bs = fma(bs, g, 1.0);
      }
      Bp[r] = bs;
    }
  }
  const int i_star = __reduce_max_sync(0xffffffffu, icand + 1) - 1;
  const int jn = i_star + 1;
  // the owners of i_star and jn hand over A and B'
  double Ast = 0.0, Bjn = 0.0, xst = 0.0, xjn = 0.0;
#pragma unroll
  for (int r = 0; r < kWarpKeys; ++r) {
    if (i0 + r == i_star) {
      Ast = A[r];
      xst = y[r];
    }
    if (i0 + r == jn) {
      Bjn = Bp[r];
      xjn = y[r];
    }
  }
  const int own_st = (i_star >= 0) ? i_star / kWarpKeys : 0;
  const int own_jn = (jn < c) ? jn / kWarpKeys : 0;
  Ast = __shfl_sync(0xffffffffu, Ast, own_st);
  xst = __shfl_sync(0xffffffffu, xst, own_st);
  Bjn = __shfl_sync(0xffffffffu, Bjn, own_jn);
  xjn = __shfl_sync(0xffffffffu, xjn, own_jn);
  if (lane == 0) {
    double xj, Aj, xj1, Bj1;
    if (i_star < 0) {
      xj = pk.inc_x;
      Aj = pk.inc_s;
    } else {
      xj = xst;
      Aj = Ast;
    }
    if (jn < c) {
      xj1 = xjn;
      Bj1 = Bjn;
    } else {
      xj1 = pk.out_x;
      Bj1 = pk.out_s;
    }
    const double cj = (double)((long long)(c - 1 - i_star) + pk.g_after);
    out->b = closed_form_root(xj, xj1, Aj, Bj1, cj, in.k, in.alpha);
    out->sumf = sum_f_at(xj, xj1, Aj, Bj1, out->b, inva);
    out->status = ROW_CERTIFIED;
    out->M = pk.M;
    out->S_aL = pk.S_aL;
    out->S_aR = pk.S_aR;
  }
  __syncwarp();
}

}  // namespace lapsum
