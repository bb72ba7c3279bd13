// resident.cu -- rows of at most 16384 scores, one thread block per row.
//
// One thread block owns a row.  Short rows are brought into shared memory
// once by a bulk (TMA) copy, longer ones are read from global memory (L2
// after the first pass); every step of the Fast LapSum pipeline (technical
// summary section 2.2: localization sample, stream-and-filter, exact solve on
// the band, certification with one widening) then runs on the row, and the
// memberships (section 2.1) are written straight from it.  HBM traffic is one
// read of the row and one write of p.  Rows whose bracket cannot be certified
// go to a full-sort fallback kernel (the worst-case branch of the arXiv
// abstract).  The backward pass (section 2.1's analytic VJP) is one block per
// row: a reduction for lambda and an elementwise pass.
#include <algorithm>
#include <type_traits>

#include "block_sort.cuh"
#include "common.cuh"
#include "launch.h"
#include "solve.cuh"
#include "tma.cuh"

namespace lapsum {
namespace {

constexpr int NT = kResidentThreads;
constexpr int kFbGroup = 1024;  // fallback: sorted values per group

struct ResLayout {
  size_t row, samp, samp_tmp, band, band_tmp, dscr, dlink, sortscr, red, mbar, total;
};

__host__ __device__ inline ResLayout res_layout(int64_t n, int m, int bcap, bool row_in_smem) {
  ResLayout L;
  size_t o = 0;
  L.row = o;      o = (o + (row_in_smem ? 4 * (size_t)n + 12 : 0) + 15) & ~size_t(15);
  L.samp = o;     o = (o + 4 * (size_t)m + 15) & ~size_t(15);
  L.samp_tmp = o; o = (o + 4 * (size_t)m + 15) & ~size_t(15);
  // the band region also holds the selection's scratch before the filter
  L.band = o;     o = (o + 4 * (size_t)(bcap > kSelectWords ? bcap : kSelectWords) + 15) & ~size_t(15);
  L.band_tmp = o; o = (o + 4 * (size_t)bcap + 15) & ~size_t(15);
  L.dscr = o;     o = (o + 8 * (size_t)bcap + 15) & ~size_t(15);
  L.dlink = o;    o = (o + 8 * (size_t)bcap + 8 + 15) & ~size_t(15);
  L.sortscr = o;  o = o + 4 * (size_t)bucket_sort_scr_words(NT);  // the band's bucket sort
  L.red = o;      o = o + 8 * 64;
  L.mbar = o;     o = o + 16;
  L.total = o;
  return L;
}

struct KeyGroups {  // consecutive groups of `g` sorted keys
  const uint32_t* k;
  int g;
  __device__ float get(int grp, int i) const { return key2f(k[grp * g + i]); }
};

struct Filtered {
  long long nL, nR;
  double SL, SR;
  int M;
  uint32_t bad;
  uint32_t kmin, kmax;  // smallest and largest key appended to the band
};

// The filter's four block reductions (n_L, S_L, S_R, the non-finite flag)
// with one pair of barriers; the same xor trees as block_sum and block_or.
__device__ __forceinline__ void block_reduce_filtered(long long& nl, double& sl, double& sr, uint32_t& bad,
                                                      double* red) {
  constexpr int NW = NT / 32;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  long long* rl = reinterpret_cast<long long*>(red + 2 * NW);
  uint32_t* rb = reinterpret_cast<uint32_t*>(red + 3 * NW);
  nl = warp_sum(nl);
  sl = warp_sum(sl);
  sr = warp_sum(sr);
  bad = __reduce_or_sync(0xffffffffu, bad);
  __syncthreads();
  if (lane == 0) {
    red[warp] = sl;
    red[NW + warp] = sr;
    rl[warp] = nl;
    rb[warp] = bad;
  }
  __syncthreads();
  sl = warp_sum(lane < NW ? red[lane] : 0.0);
  sr = warp_sum(lane < NW ? red[NW + lane] : 0.0);
  nl = warp_sum(lane < NW ? rl[lane] : 0ll);
  bad = __reduce_or_sync(0xffffffffu, lane < NW ? rb[lane] : 0u);
}

// One pass over the row, in shared memory or (kGlobal) in global memory
// (section 2.2 stream-and-filter):
// scores below a_L and at/above a_R go into counts and anchored tail sums
// (every term exp(-dist/alpha) <= 1, fp32 exp, fp64 sums); scores inside the
// bracket are appended to the band with one shared atomic each.  A thread
// takes 16 scores a step (four float4, their loads issued together) and
// learns which of them lie in the band from the bits of an exact fp32 sum;
// those few are read again by position (from L1 or shared memory), so the
// common step has no branch per score.
template <bool kGlobal>
__device__ Filtered filter_row(const float* row, int n, float aL, float aR, float c2, uint32_t* band,
                               int bcap, int* s_cnt, uint32_t* s_kr, double* red) {
  if (threadIdx.x == 0) {
    *s_cnt = 0;
    s_kr[0] = 0xFFFFFFFFu;
    s_kr[1] = 0u;
  }
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const uint32_t lt = (1u << lane) - 1u;
  int nl = 0;  // n_R is n - n_L - (band count): no per-score count for it
  double sl = 0.0, sr = 0.0;
  uint32_t bad = 0u;
  // sum of the scores scaled by 2^-64: +-inf or NaN shows here
  float2 fs2 = make_float2(0.0f, 0.0f);
  const float2 naL2 = make_float2(-aL, -aL), aR2 = make_float2(aR, aR), c22 = make_float2(c2, c2);
  const float2 k64 = make_float2(0x1p-64f, 0x1p-64f);
  constexpr int kB = 4;
  const int head = row_head(row, n);
  const int n4 = (n - head) >> 2;
  const float* rowh = row + head;
  const float4* row4 = reinterpret_cast<const float4*>(rowh);
  for (int base0 = 0; base0 < n4; base0 += kB * NT) {
    float4 qs[kB];
#pragma unroll
    for (int u = 0; u < kB; ++u) {
      const int v = base0 + u * NT + threadIdx.x;
      qs[u] = v < n4 ? (kGlobal ? __ldg(row4 + v) : row4[v]) : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    }
    // a step whose lanes all lie inside the row needs no per-score range check
    auto step = [&](auto checked) {
      float2 pl2 = make_float2(0.0f, 0.0f), pr2 = pl2, cl2 = pl2, ob2 = pl2;
#pragma unroll
      for (int u = 0; u < kB; ++u) {
        const bool act = !decltype(checked)::value || base0 + u * NT + (int)threadIdx.x < n4;
        const float4 q = qs[u];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const float2 x2 = h ? make_float2(q.z, q.w) : make_float2(q.x, q.y);
          const Side2 sd = classify2(x2, naL2, aR2, c22);
          float2 L = sd.L, R = sd.R;
          if (!act) L = R = make_float2(0.0f, 0.0f);
          const float bit = (float)(1u << (4 * u + 2 * h));
          pl2 = fma2(L, sd.e, pl2);
          pr2 = fma2(R, sd.e, pr2);
          cl2 = add2(cl2, L);
          // positions outside the band (a padding position counts as outside)
          ob2 = fma2(act ? add2(L, R) : make_float2(1.0f, 1.0f), make_float2(bit, 2.0f * bit), ob2);
          fs2 = fma2(x2, k64, fs2);  // padding lanes hold 0
        }
      }
      sl += (double)(pl2.x + pl2.y);
      sr += (double)(pr2.x + pr2.y);
      nl += (int)(cl2.x + cl2.y);
      uint32_t mask = ~(uint32_t)(ob2.x + ob2.y) & 0xFFFFu;  // in-band positions of this thread's 16
      while (mask) {  // rare: read each again by position and append it
        const int i = __ffs(mask) - 1;
        mask &= mask - 1u;
        const float x = rowh[4 * (base0 + (i >> 2) * NT + (int)threadIdx.x) + (i & 3)];
        if (!(fabsf(x) < CUDART_INF_F)) bad = 1u;  // NaN
        const uint32_t key = f2key(x);
        const int pos = atomicAdd(s_cnt, 1);
        if (pos < bcap) band[pos] = key;
        atomicMin(&s_kr[0], key);
        atomicMax(&s_kr[1], key);
      }
    };
    if (base0 + kB * NT <= n4) step(std::false_type{});
    else step(std::true_type{});
  }
  // the scores outside the body: one per thread and step, the loads of kB
  // steps issued ahead from global memory
  const int nrest = n - (n4 << 2);
  for (int base0 = 0; base0 < nrest; base0 += kB * NT) {
  float xq[kB];
#pragma unroll
  for (int u = 0; u < kB; ++u) {
    const int j = base0 + u * NT + threadIdx.x;
    xq[u] = j < nrest ? row[rest_index(j, head, n4)] : 0.0f;
  }
#pragma unroll
  for (int u = 0; u < kB; ++u) {
    const bool act = base0 + u * NT + (int)threadIdx.x < nrest;
    const float x = xq[u];
    const Side sd = classify(x, aL, aR, c2);
    if (act) {
      if (sd.L != 0.0f) { sl += (double)sd.e; ++nl; }
      if (sd.R != 0.0f) sr += (double)sd.e;
      if (!(fabsf(x) < CUDART_INF_F)) bad = 1u;
    }
    const bool inb = act && sd.L + sd.R == 0.0f;
    const uint32_t msk = __ballot_sync(0xffffffffu, inb);
    if (msk) {
      const int leader = __ffs(msk) - 1;
      int wbase = 0;
      if (lane == leader) wbase = atomicAdd(s_cnt, __popc(msk));
      wbase = __shfl_sync(0xffffffffu, wbase, leader);
      if (inb) {
        const int pos = wbase + __popc(msk & lt);
        const uint32_t key = f2key(x);
        if (pos < bcap) band[pos] = key;
        atomicMin(&s_kr[0], key);
        atomicMax(&s_kr[1], key);
      }
    }
  }
  }
  if (!(fabsf(fs2.x + fs2.y) < CUDART_INF_F)) bad = 1u;
  Filtered f;
  long long nll = nl;
  block_reduce_filtered(nll, sl, sr, bad, red);
  f.nL = nll;
  f.SL = sl;
  f.SR = sr;
  f.bad = bad;
  f.M = *s_cnt;
  f.kmin = s_kr[0];
  f.kmax = s_kr[1];
  f.nR = (long long)n - f.nL - (long long)f.M;  // every score is left, right or in the band
  __syncthreads();
  return f;
}

__device__ void write_stats(lapsum_row_stats* st, float aL, float aR, long long nL, long long nR, long long M,
                            double SL, double SR, double b, double sump, double sumf, int m, int buckets,
                            uint32_t status) {
  st->a_L = aL;
  st->a_R = aR;
  st->n_L = nL;
  st->n_R = nR;
  st->band = M;
  st->S_L = SL;
  st->S_R = SR;
  st->b = b;
  st->sum_p = sump;
  st->sum_f = sumf;
  st->sample_m = m;
  st->buckets = buckets;
  st->status = status;
  st->reserved = 0;
}

// p_i = F((r_i - b)/alpha) as an fp32 value; (r_i - b) is formed from b split
// into two fp32 words (b = bh + bl), which keeps it accurate to fp64 level.
// The side of b is taken as a saturated product on the FMA pipe (s = 1 at or
// above b, 0 below), not a compare and select on the ALU pipe; 1 - h is then
// formed as h + s (1 - 2h), within an ulp of 1 - h.
__device__ __forceinline__ float membership(float x, float bh, float bl, float c2) {
  const float d = (x - bh) - bl;
  const float h = 0.5f * exp2f(-fabsf(d) * c2);
  const float s = fma_sat(d, 0x1p126f, 1.0f);
  return fmaf(s, fmaf(-2.0f, h, 1.0f), h);
}
// membership for two scores with packed arithmetic: the same values bit for
// bit (nbh = (-bh, -bh), nbl = (-bl, -bl), nc2 = -c2).  The exponent is the
// scalar product |d| (-c2), which equals -|d c2| exactly and needs no
// separate sign or magnitude change before the exp2.
__device__ __forceinline__ float2 membership2(float2 x, float2 nbh, float2 nbl, float nc2) {
  const float2 d = add2(add2(x, nbh), nbl);
  const float2 h = mul2(make_float2(exp2f(fabsf(d.x) * nc2), exp2f(fabsf(d.y) * nc2)), make_float2(0.5f, 0.5f));
  const float2 s = make_float2(fma_sat(d.x, 0x1p126f, 1.0f), fma_sat(d.y, 0x1p126f, 1.0f));
  return fma2(s, fma2(make_float2(-2.0f, -2.0f), h, make_float2(1.0f, 1.0f)), h);
}

// Writes p for a row from `src` (shared or global) and finishes the row's
// outputs; sumf is the solver's exact sum of f.  Every thread must call it.
__device__ void finish_row(const ResidentFwd& a, int64_t r, const float* src, double b, double sumf,
                           uint32_t status, float aL, float aR, long long nL, long long nR, long long M,
                           double SL, double SR, int buckets, double* red) {
  const int n = (int)a.n;
  const RowArgs ra = row_args(a, r);
  if (ra.bad) status |= ROW_BADARG;
  const double inva = 1.0 / ra.alpha_p;
  const float c2 = (float)(inva * (double)kLog2e);
  const float bh = __double2float_rn(b);
  const float bl = __double2float_rn(b - (double)bh);
  const float2 nbh2 = make_float2(-bh, -bh), nbl2 = make_float2(-bl, -bl);
  double ps = 0.0;
  const bool nonfinite = (status & ROW_NAN_OUT) != 0u;
  if (a.dftopk) {
    // sum f at the membership scale alpha_p, relative to the score nearest b
    float mh = CUDART_INF_F, ml = 0.0f;
    double S = 0.0;
    for (int i = threadIdx.x; i < n; i += NT) near_add(src[i], bh, bl, c2, mh, ml, S);
    double dmin = near_dist(mh, ml);
    block_near_reduce<NT>(dmin, S, inva, red);
    sumf = (dmin < CUDART_INF) ? 0.5 * inva * exp_call(-dmin * inva) * S : 0.0;
  }
  if (a.sp.idx) {
    // sparse output, in index order: each thread takes 4 consecutive scores
    // of a 4*NT window, a block scan places its hits
    int32_t* oi = a.sp.idx + r * a.sp.cap;
    float* ov = a.sp.val + r * a.sp.cap;
    uint64_t total = 0;
    uint32_t* scr = reinterpret_cast<uint32_t*>(red);
    for (int i0 = 0; i0 < n; i0 += 4 * NT) {
      float pv[4];
      uint32_t hits = 0u;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int i = i0 + 4 * (int)threadIdx.x + j;
        pv[j] = 0.0f;
        if (i < n) {
          pv[j] = nonfinite ? CUDART_NAN_F : membership(src[i], bh, bl, c2);
          ps += (double)pv[j];
          if (pv[j] >= a.sp.eps) hits |= 1u << j;
        }
      }
      uint32_t tot;
      uint64_t pos = total + block_excl_prefix_u32<NT>((uint32_t)__popc(hits), scr, &tot);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        if (hits & (1u << j)) {
          if (pos < (uint64_t)a.sp.cap) {
            oi[pos] = i0 + 4 * (int)threadIdx.x + j;
            ov[pos] = pv[j];
          }
          ++pos;
        }
      }
      total += tot;
    }
    if (total > (uint64_t)a.sp.cap) status |= ROW_TRUNCATED;
    if (threadIdx.x == 0) a.sp.count[r] = total;
    __syncthreads();
  } else if (a.vec) {
    // src and dst start at the same address mod 16 (a shared-memory copy is
    // placed that way): one head, then float4 from both.  sum p is only
    // accumulated when the caller asked for it (sump_out, stats).
    float* dst = a.p_out + r * a.stride;
    const int head = row_head(src, n);
    const float4* s4 = reinterpret_cast<const float4*>(src + head);
    float4* d4 = reinterpret_cast<float4*>(dst + head);
    const int n4 = (n - head) >> 2;
    constexpr int kB = 4;  // loads in flight per thread (the row may be in global memory)
    auto pass = [&](auto want_ps) {
      for (int v0 = threadIdx.x; v0 < n4; v0 += kB * NT) {
        float4 xs[kB];
#pragma unroll
        for (int u = 0; u < kB; ++u) {
          const int v = v0 + u * NT;
          xs[u] = v < n4 ? s4[v] : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
        }
        auto put = [&](auto checked) {
#pragma unroll
          for (int u = 0; u < kB; ++u) {
            const int v = v0 + u * NT;
            if (decltype(checked)::value && v >= n4) break;
            const float4 x = xs[u];
            const float2 p01 = membership2(make_float2(x.x, x.y), nbh2, nbl2, -c2);
            const float2 p23 = membership2(make_float2(x.z, x.w), nbh2, nbl2, -c2);
            if (decltype(want_ps)::value) ps += (double)((p01.x + p01.y) + (p23.x + p23.y));
            stg_stream(d4 + v, make_float4(p01.x, p01.y, p23.x, p23.y));
          }
        };
        if (v0 - (int)threadIdx.x + kB * NT <= n4) put(std::false_type{});
        else put(std::true_type{});
      }
    };
    if (nonfinite) {
      const float4 nan4 = make_float4(CUDART_NAN_F, CUDART_NAN_F, CUDART_NAN_F, CUDART_NAN_F);
      for (int v = threadIdx.x; v < n4; v += NT) stg_stream(d4 + v, nan4);
    } else if (a.sump_out || a.stats) {
      pass(std::true_type{});
    } else {
      pass(std::false_type{});
    }
    for (int j = threadIdx.x; j < n - (n4 << 2); j += NT) {
      const int i = (int)rest_index(j, head, n4);
      const float p = nonfinite ? CUDART_NAN_F : membership(src[i], bh, bl, c2);
      ps += (double)p;
      dst[i] = p;
    }
  } else {
    float* dst = a.p_out + r * a.stride;
    for (int i = threadIdx.x; i < n; i += NT) {
      const float p = nonfinite ? CUDART_NAN_F : membership(src[i], bh, bl, c2);
      ps += (double)p;
      dst[i] = p;
    }
  }
  ps = block_sum<NT, double>(ps, red);
  if (threadIdx.x == 0) {
    const double bo = nonfinite ? CUDART_NAN : b;
    const double so = nonfinite ? CUDART_NAN : sumf;
    a.b_out[r] = bo;
    if (a.sumf_out) a.sumf_out[r] = so;
    if (a.sump_out) a.sump_out[r] = nonfinite ? CUDART_NAN : ps;
    if (a.status_out) a.status_out[r] = status & ROW_PUBLIC;
    if (a.stats) write_stats(a.stats + r, aL, aR, nL, nR, M, SL, SR, bo, ps, so, a.m, buckets, status & ROW_PUBLIC);
  }
}

// Rows up to kRowSmemMaxN scores are copied into shared memory (one bulk copy)
// and read there three times; longer ones are read from global memory (the
// second and third reads hit L2).  Both forms run four rows per SM (64
// registers a thread); a larger shared copy would leave room for fewer
// (measured, 2048 rows of 8192: 148 us from global memory, 160 us from a
// shared copy at three rows per SM).
constexpr int64_t kRowSmemMaxN = 4096;

template <bool kSmemRow>
__global__ void __launch_bounds__(NT, kResidentBlocksPerSm) k_row_fwd(const ResidentFwd a) {
  extern __shared__ __align__(16) unsigned char smem[];
  const ResLayout L = res_layout(a.n, a.m, a.bcap, kSmemRow);
  uint32_t* samp = reinterpret_cast<uint32_t*>(smem + L.samp);
  uint32_t* band = reinterpret_cast<uint32_t*>(smem + L.band);
  double* dscr = reinterpret_cast<double*>(smem + L.dscr);
  double* dlink = reinterpret_cast<double*>(smem + L.dlink);
  uint32_t* band_tmp = reinterpret_cast<uint32_t*>(smem + L.band_tmp);
  uint32_t* sortscr = reinterpret_cast<uint32_t*>(smem + L.sortscr);
  double* red = reinterpret_cast<double*>(smem + L.red);
  uint64_t* mbar = reinterpret_cast<uint64_t*>(smem + L.mbar);
  __shared__ int s_cnt;
  __shared__ uint32_t s_kr[2];
  __shared__ SolveOut s_out;

  const int64_t r = blockIdx.x;
  const int n = (int)a.n;
  const float* src = a.scores + r * a.stride;
  // the shared copy starts at src's address mod 16 when p is written with
  // float4 (the region has 16 spare bytes), so that both walk one body
  const int head = (kSmemRow && a.vec) ? row_head(src, n) : 0;
  float* srow = reinterpret_cast<float*>(smem + L.row) + ((4 - head) & 3);
  const float* row = kSmemRow ? srow : src;
  const RowArgs ra = row_args(a, r);
  const RowRanks rr = row_ranks(a, ra.k);
  const double inva = 1.0 / ra.alpha;
  const float c2 = (float)(inva * (double)kLog2e);

  // ---- start bringing the row in: a bulk copy into shared memory, or (rows
  // read from global memory) an L2 prefetch; either overlaps the sample
  uint32_t status = 0u;
  const int n4c = (n - head) >> 2;
  const uint32_t cbytes = (kSmemRow && a.vec) ? (uint32_t)n4c * 16u : 0u;
  // test knob: odd rows issue no copy, so their bounded wait below runs out
  const bool force_to = kSmemRow && a.vec && a.force_timeout && (r & 1);
  const uint32_t limit = spin_limit_of(a.spin_limit);
  if (threadIdx.x == 0) {
    if constexpr (kSmemRow) {
      if (a.vec) {
        mbar_init(mbar, 1);
        fence_proxy_async_smem();
        if (cbytes > 0 && !force_to) {
          mbar_arrive_expect_tx(mbar, cbytes);
          unsigned char* d = reinterpret_cast<unsigned char*>(srow + head);
          const unsigned char* s = reinterpret_cast<const unsigned char*>(src + head);
          for (uint32_t off = 0; off < cbytes; off += 16384u)
            bulk_load(d + off, s + off, min(16384u, cbytes - off), mbar);
        }
      }
    } else {
      const int h = row_head(src, n);
      const uint32_t pb = (uint32_t)((n - h) >> 2) * 16u;
      const unsigned char* s = reinterpret_cast<const unsigned char*>(src + h);
      for (uint32_t off = 0; off < pb; off += 16384u) bulk_prefetch_l2(s + off, min(16384u, pb - off));
    }
  }

  // ---- localization (section 2.2, step 1), from global memory -------------
  // Only the two order statistics of the bracket are needed: they are
  // selected, not sorted for; the sample is sorted only if a widening needs
  // other ranks.
  const int m = a.m;
  const uint64_t s = row_stream(a.seed, (uint64_t)r);
  for (int j = threadIdx.x; j < m; j += NT) {
    const uint64_t I = sample_index(s, (uint64_t)j, (uint64_t)n);
    const double Y = (double)src[I] + laplace_noise(s, (uint64_t)j, ra.alpha);
    samp[j] = f2key(__double2float_rn(Y));
  }
  __syncthreads();
  int rlo = rr.rank_lo, rhi = rr.rank_hi;
  bool vlo = rr.valid_lo != 0, vhi = rr.valid_hi != 0;
  float aL, aR;
  {
    const int want[2] = {vlo ? rlo : 0, vhi ? rhi : m - 1};
    uint32_t got[2];
    block_select2<NT>(samp, m, want, got, band);  // band is not written before the filter
    aL = vlo ? key2f(got[0]) : -CUDART_INF_F;
    aR = vhi ? key2f(got[1]) : CUDART_INF_F;
  }
  bool samp_sorted = false;

  // ---- finish the shared copy ----------------------------------------------
  if constexpr (kSmemRow) {
    if (a.vec) {
      for (int j = threadIdx.x; j < n - 4 * n4c; j += NT) {
        const int i = (int)rest_index(j, head, n4c);
        srow[i] = src[i];
      }
      const int timed_out = ((cbytes > 0 || force_to) && !mbar_wait_bounded(mbar, 0, limit)) ? 1 : 0;
      if (__syncthreads_or(timed_out)) status |= ROW_TIMEOUT;
    } else {
      for (int i = threadIdx.x; i < n; i += NT) srow[i] = src[i];
    }
    __syncthreads();
    if (status & ROW_TIMEOUT) {
      // the copy did not complete in time: wait once more, bounded, then give
      // up on the row.  Its outputs are written as NaN from the global row
      // (not the shared copy, which the bulk copy may still be filling).  If
      // that copy is still in flight when the block exits, it may land in
      // shared memory that a later block on this SM has been given.
      mbar_wait_bounded(mbar, 0, limit);
      finish_row(a, r, src, CUDART_NAN, CUDART_NAN, ROW_TIMEOUT, aL, aR, 0, 0, 0, 0.0, 0.0, 0, red);
      return;
    }
  }

  // ---- filter, sort the band, solve, certify (steps 2-4) ------------------
  bool solved = false;
  Filtered f{};
  if (!a.force_fallback) {
    for (int attempt = 0;; ++attempt) {
      f = filter_row<!kSmemRow>(row, n, aL, aR, c2, band, a.bcap, &s_cnt, s_kr, red);
      if (f.bad) { status |= ROW_NONFINITE; break; }
      if (f.M > a.bcap) { status |= ROW_OVERFLOW; break; }
      // one bucket pass over the band's key range; a band stretched by
      // outliers into crowded buckets takes the bitonic network instead
      const uint32_t* sorted = block_bucket_sort<NT>(band, band_tmp, f.M, f.kmin, f.kmax, sortscr);
      if (!sorted) {
        block_bitonic_sort<NT>(band, f.M);  // band and band_tmp form one buffer of 2 bcap keys
        sorted = band;
      }
      SolveIn in{aL, aR, f.nL, f.nR, f.SL, f.SR, ra.k, ra.alpha, inva};
      solve_run_warp<NT>(in, sorted, f.M, dscr, dlink, &s_out);
      if (s_out.status & ROW_CERTIFIED) { solved = true; break; }
      if (attempt >= a.max_widen) break;
      // widen once on the side that missed; the other edge moves to the old
      // edge, which is now known to lie on the correct side of b
      status |= ROW_WIDENED;
      if (!samp_sorted) {
        block_bitonic_sort<NT>(samp, m);  // samp and samp_tmp form one buffer of 2m keys
        samp_sorted = true;
      }
      const uint32_t* ss = samp;
      if (s_out.status & ROW_MISS_LEFT) {
        rhi = rlo; vhi = true; aR = aL;
        rlo -= rr.widen_delta;
        vlo = rlo >= 0;
        if (!vlo) rlo = 0;
        aL = vlo ? key2f(ss[rlo]) : -CUDART_INF_F;
      } else {
        rlo = rhi; vlo = true; aL = aR;
        rhi += rr.widen_delta;
        vhi = rhi <= m - 1;
        if (!vhi) rhi = m - 1;
        aR = vhi ? key2f(ss[rhi]) : CUDART_INF_F;
      }
    }
  }

  if (solved) {
    finish_row(a, r, row, s_out.b, s_out.sumf, status | ROW_CERTIFIED, aL, aR, f.nL, f.nR, f.M, f.SL, f.SR, 1,
               red);
  } else if (status & ROW_NONFINITE) {
    finish_row(a, r, row, CUDART_NAN, CUDART_NAN, status, aL, aR, f.nL, f.nR, f.M, f.SL, f.SR, 1, red);
  } else if (threadIdx.x == 0) {
    const uint32_t idx = atomicAdd(a.fb_count, 1u);
    a.fb_list[idx] = (int32_t)r;
    a.ws_status[r] = status;
  }
}

struct FbLayout {
  size_t keys, tmp, hist, dscr, aggs, red, total;
};
__host__ __device__ inline FbLayout fb_layout(int64_t n) {
  FbLayout L;
  size_t o = 0;
  const size_t groups = (size_t)((n + kFbGroup - 1) / kFbGroup);
  L.keys = o; o = (o + 4 * (size_t)n + 15) & ~size_t(15);
  L.tmp = o;  o = (o + 4 * (size_t)n + 15) & ~size_t(15);
  L.hist = o; o = (o + 4 * (size_t)SortScratch<NT>::kWords + 15) & ~size_t(15);
  L.dscr = o; o = (o + 8 * (size_t)kFbGroup + 15) & ~size_t(15);
  L.aggs = o; o = (o + sizeof(GroupAgg) * groups + 15) & ~size_t(15);
  L.red = o;  o = o + 8 * 64;
  L.total = o;
  return L;
}

// Full-sort fallback (arXiv abstract: covers the worst case; section 2.2:
// the full-sort solver).  Rows queued by k_row_fwd are sorted whole in shared
// memory and solved with no bracket.
__global__ void __launch_bounds__(NT) k_row_fallback(const ResidentFwd a) {
  extern __shared__ __align__(16) unsigned char smem[];
  const FbLayout L = fb_layout(a.n);
  uint32_t* keys = reinterpret_cast<uint32_t*>(smem + L.keys);
  uint32_t* tmp = reinterpret_cast<uint32_t*>(smem + L.tmp);
  uint32_t* hist = reinterpret_cast<uint32_t*>(smem + L.hist);
  double* dscr = reinterpret_cast<double*>(smem + L.dscr);
  GroupAgg* aggs = reinterpret_cast<GroupAgg*>(smem + L.aggs);
  double* red = reinterpret_cast<double*>(smem + L.red);
  __shared__ SolveOut s_out;
  wait_prior_grid();
  const int n = (int)a.n;
  const uint32_t cnt = *reinterpret_cast<volatile uint32_t*>(a.fb_count);
  for (uint32_t idx = blockIdx.x; idx < cnt; idx += gridDim.x) {
    const int64_t r = a.fb_list[idx];
    const float* src = a.scores + r * a.stride;
    const RowArgs ra = row_args(a, r);
    const double inva = 1.0 / ra.alpha;
    __syncthreads();
    {
      // eight loads a thread in flight (one block per SM: the loop would
      // otherwise wait on every load)
      constexpr int kLd = 8;
      for (int i0 = 0; i0 < n; i0 += kLd * NT) {
        float xx[kLd];
#pragma unroll
        for (int u = 0; u < kLd; ++u) {
          const int i = i0 + u * NT + (int)threadIdx.x;
          xx[u] = i < n ? src[i] : 0.0f;
        }
#pragma unroll
        for (int u = 0; u < kLd; ++u) {
          const int i = i0 + u * NT + (int)threadIdx.x;
          if (i < n) keys[i] = f2key(xx[u]);
        }
      }
    }
    __syncthreads();
    const uint32_t* sorted = block_radix_sort<NT>(keys, tmp, n, hist);
    __syncthreads();
    const int T = (n + kFbGroup - 1) / kFbGroup;
    for (int g = 0; g < T; ++g)
      aggregate_sorted_keys<NT, false>(sorted + g * kFbGroup, min(kFbGroup, n - g * kFbGroup), red, &aggs[g], inva);
    SolveIn in{-CUDART_INF_F, CUDART_INF_F, 0, 0, 0.0, 0.0, ra.k, ra.alpha, inva};
    solve_band<NT, false>(in, aggs, T, KeyGroups{sorted, kFbGroup}, dscr, red, &s_out);
    const uint32_t status = a.ws_status[r] | ROW_FALLBACK | ROW_CERTIFIED;
    finish_row(a, r, src, s_out.b, s_out.sumf, status, -CUDART_INF_F, CUDART_INF_F, 0, 0, n, 0.0, 0.0, T, red);
  }
}

// Backward for one row per block (section 2.1, analytic VJP):
// lambda = sum g f / sum f by the rescaled reduction of common.cuh, then
// grad = f (g - lambda) with f = 2^(log2(1/(2 alpha)) - |r - b| log2(e)/alpha)
// computed in one exponent, and lambda split into two fp32 words so that
// g - lambda keeps its accuracy when g is close to lambda.
template <bool kAlpha>
__global__ void __launch_bounds__(NT) k_row_bwd(const RowBwd a) {
  __shared__ double red[64];
  const int n = (int)a.n;
  for (int64_t r = blockIdx.x; r < a.rows; r += gridDim.x) {
    bool bad = false;
    const double inva = 1.0 / row_alpha(a.alpha, a.alpha_rows, r, &bad);
    const float c2 = (float)(inva * (double)kLog2e);
    const float lg = (float)log2(0.5 * inva);
    const float* x = a.scores + r * a.stride;
    const float* g = a.grad_p + r * a.stride;
    float* o = a.grad + r * a.stride;
    const double b = a.b[r];
    const float bh = __double2float_rn(b);
    const float bl = __double2float_rn(b - (double)bh);
    float m = CUDART_INF_F;
    double S = 0.0, SG = 0.0, SZ = 0.0, SGZ = 0.0;
    // one score: the two sums of lambda, and with kAlpha the two of dL/dalpha
    auto acc = [&](float xv, float gv, float& ps, float& psg, float& psz, float& psgz) {
      const float z = (xv - bh) - bl;
      if (kAlpha) shift_add_z(fabsf(z) * c2, gv, z, m, ps, psg, psz, psgz, S, SG, SZ, SGZ);
      else shift_add(fabsf(z) * c2, gv, m, ps, psg, S, SG);
    };
    // x, g and grad start at the same address mod 16: one head, then the
    // body as float4, kB float4 of r and of g in flight per thread
    const int head = a.vec ? row_head(x, n) : 0;
    const int n4 = a.vec ? ((n - head) >> 2) : 0;
    const float4* x4 = reinterpret_cast<const float4*>(x + head);
    const float4* g4 = reinterpret_cast<const float4*>(g + head);
    constexpr int kB = 4;
    const float2 nbh2 = make_float2(-bh, -bh), nbl2 = make_float2(-bl, -bl), c22 = make_float2(c2, c2);
    for (int v0 = threadIdx.x; v0 < n4; v0 += kB * NT) {
      float4 xv[kB], gv[kB];
#pragma unroll
      for (int u = 0; u < kB; ++u) {
        const int v = v0 + u * NT;
        xv[u] = v < n4 ? __ldg(x4 + v) : make_float4(0.f, 0.f, 0.f, 0.f);
        gv[u] = v < n4 ? __ldg(g4 + v) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
      // The step's 16 exponents a = |r - b| log2(e)/alpha in packed
      // arithmetic; the terms 2^(m - a) are taken relative to the running
      // minimum m, moved (and the sums rescaled) at most once a step rather
      // than tested for every score.  Padding positions get a = +inf.  With
      // kAlpha the z-weighted sums of dL/dalpha ride along; the two sums of
      // lambda take the same operations either way.
      float ae[4 * kB];
      float2 zz[kAlpha ? 2 * kB : 1];
#pragma unroll
      for (int u = 0; u < kB; ++u) {
        const bool act = v0 + u * NT < n4;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const float2 x2 = h ? make_float2(xv[u].z, xv[u].w) : make_float2(xv[u].x, xv[u].y);
          const float2 z = add2(add2(x2, nbh2), nbl2);
          if (kAlpha) zz[2 * u + h] = z;
          const float2 q = mul2(z, c22);
          ae[4 * u + 2 * h] = act ? fabsf(q.x) : CUDART_INF_F;
          ae[4 * u + 2 * h + 1] = act ? fabsf(q.y) : CUDART_INF_F;
        }
      }
      float mstep = ae[0];
#pragma unroll
      for (int i = 1; i < 4 * kB; ++i) mstep = fminf(mstep, ae[i]);
      if (mstep < m) {  // a new nearest score: rescale what was accumulated
        const double sc = (double)exp2f(mstep - m);
        S *= sc;
        SG *= sc;
        if (kAlpha) {
          SZ *= sc;
          SGZ *= sc;
        }
        m = mstep;
      }
      float2 ps2 = make_float2(0.0f, 0.0f), psg2 = ps2, psz2 = ps2, psgz2 = ps2;
#pragma unroll
      for (int u = 0; u < kB; ++u) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const float2 g2 = h ? make_float2(gv[u].z, gv[u].w) : make_float2(gv[u].x, gv[u].y);
          const float2 e2 = make_float2(exp2f(m - ae[4 * u + 2 * h]), exp2f(m - ae[4 * u + 2 * h + 1]));
          ps2 = add2(ps2, e2);
          psg2 = fma2(g2, e2, psg2);
          if (kAlpha) {
            const float2 ez = mul2(e2, zz[2 * u + h]);
            psz2 = add2(psz2, ez);
            psgz2 = fma2(g2, ez, psgz2);
          }
        }
      }
      if (m < CUDART_INF_F) {  // no finite exponent yet: nothing to add
        S += (double)(ps2.x + ps2.y);
        SG += (double)(psg2.x + psg2.y);
        if (kAlpha) {
          SZ += (double)(psz2.x + psz2.y);
          SGZ += (double)(psgz2.x + psgz2.y);
        }
      }
    }
    const int nrest = n - (n4 << 2);
    for (int j = threadIdx.x; j < nrest; j += NT) {
      const int i = (int)rest_index(j, head, n4);
      float ps = 0.0f, psg = 0.0f, psz = 0.0f, psgz = 0.0f;
      acc(x[i], g[i], ps, psg, psz, psgz);
      S += (double)ps;
      SG += (double)psg;
      SZ += (double)psz;
      SGZ += (double)psgz;
    }
    if (kAlpha) block_shift_reduce4<NT>(m, S, SG, SZ, SGZ, red);
    else block_shift_reduce<NT>(m, S, SG, red);
    const double lam = bad ? CUDART_NAN : SG / S;  // NaN also reaches every grad of the row
    const float lh = __double2float_rn(lam);
    const float ll = __double2float_rn(lam - (double)lh);
    const float2 nlh2 = make_float2(-lh, -lh), nll2 = make_float2(-ll, -ll);
    for (int v0 = threadIdx.x; v0 < n4; v0 += kB * NT) {
      float4 xv[kB], gv[kB];
#pragma unroll
      for (int u = 0; u < kB; ++u) {
        const int v = v0 + u * NT;
        xv[u] = v < n4 ? __ldcs(x4 + v) : make_float4(0.f, 0.f, 0.f, 0.f);
        gv[u] = v < n4 ? __ldcs(g4 + v) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int u = 0; u < kB; ++u) {
        const int v = v0 + u * NT;
        if (v >= n4) break;
        // the same operations as the scalar form below, two scores at a time
        float2 o2[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const float2 x2 = h ? make_float2(xv[u].z, xv[u].w) : make_float2(xv[u].x, xv[u].y);
          const float2 g2 = h ? make_float2(gv[u].z, gv[u].w) : make_float2(gv[u].x, gv[u].y);
          const float2 z = add2(add2(x2, nbh2), nbl2);
          const float2 f = make_float2(exp2f(fmaf(-fabsf(z.x), c2, lg)), exp2f(fmaf(-fabsf(z.y), c2, lg)));
          o2[h] = mul2(f, add2(add2(g2, nlh2), nll2));
        }
        stg_stream(reinterpret_cast<float4*>(o + head) + v, make_float4(o2[0].x, o2[0].y, o2[1].x, o2[1].y));
      }
    }
    for (int j = threadIdx.x; j < nrest; j += NT) {
      const int i = (int)rest_index(j, head, n4);
      o[i] = exp2f(fmaf(-fabsf((x[i] - bh) - bl), c2, lg)) * ((g[i] - lh) - ll);
    }
    if (threadIdx.x == 0 && a.grad_k) a.grad_k[r] = lam;
    if (kAlpha && threadIdx.x == 0) a.grad_alpha[r] = bad ? CUDART_NAN : alpha_grad((double)m, SZ, SGZ, lam, inva);
    __syncthreads();
  }
}

}  // namespace

size_t resident_fwd_smem(const ResidentFwd& a) {
  return res_layout(a.n, a.m, a.bcap, a.n <= kRowSmemMaxN).total;
}
size_t resident_fallback_smem(int64_t n) { return fb_layout(n).total; }

// Lets both kernels use all the shared memory a block may opt in to (less
// their static shared memory); the size each launch actually requests decides
// its occupancy.
cudaError_t resident_init(int optin_bytes) {
  cudaFuncAttributes fa;
  cudaError_t e = cudaFuncGetAttributes(&fa, k_row_fwd<true>);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(k_row_fwd<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           optin_bytes - (int)fa.sharedSizeBytes);
  if (e != cudaSuccess) return e;
  e = cudaFuncGetAttributes(&fa, k_row_fwd<false>);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(k_row_fwd<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           optin_bytes - (int)fa.sharedSizeBytes);
  if (e != cudaSuccess) return e;
  e = cudaFuncGetAttributes(&fa, k_row_fallback);
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(k_row_fallback, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              optin_bytes - (int)fa.sharedSizeBytes);
}

cudaError_t launch_resident_fwd(const ResidentFwd& a, int sm_count, cudaStream_t st) {
  const size_t smem = resident_fwd_smem(a);
  const size_t fsmem = resident_fallback_smem(a.n);
  cudaError_t e = cudaMemsetAsync(a.fb_count, 0, sizeof(uint32_t), st);
  if (e != cudaSuccess) return e;
  {
    Launch l("k_row_fwd", st);
    if (a.n <= kRowSmemMaxN) k_row_fwd<true><<<(unsigned)a.rows, NT, smem, st>>>(a);
    else k_row_fwd<false><<<(unsigned)a.rows, NT, smem, st>>>(a);
  }
  const unsigned fgrid = (unsigned)std::min<int64_t>(a.rows, (int64_t)sm_count);
  {
    Launch l("k_row_fallback", st);
    e = launch_ex(kPdlTail, k_row_fallback, dim3(fgrid), dim3(NT), fsmem, st, a);
    if (e != cudaSuccess) return e;
  }
  return cudaGetLastError();
}

cudaError_t launch_resident_bwd(const RowBwd& a, int sm_count, cudaStream_t st) {
  const unsigned grid = (unsigned)std::min<int64_t>(a.rows, (int64_t)sm_count * 4);
  {
    Launch l("k_row_bwd", st);
    if (a.grad_alpha) k_row_bwd<true><<<grid, NT, 0, st>>>(a);
    else k_row_bwd<false><<<grid, NT, 0, st>>>(a);
  }
  return cudaGetLastError();
}

}  // namespace lapsum
