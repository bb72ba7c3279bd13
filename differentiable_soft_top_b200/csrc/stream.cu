// stream.cu -- rows longer than one block's shared memory (n > 16384).
//
// The Fast LapSum pipeline (technical summary section 2.2; arXiv abstract)
// as a short sequence of grid-wide kernels per forward pass:
//
//   k_sample    localization sample: m Laplace-noised scores, level-1
//               histogram of their fp32 keys
//   k_select2/3 radix select of the two binomial order statistics that bound
//               the bracket [a_L, a_R)
//   k_filter    the HBM-bound stream-and-filter pass: 128-bit loads, tail
//               counts and anchored tail sums (fp32 exp, fp64 partials), and
//               in-band values appended, unsorted, to the row's band
//   k_band      a cluster of CTAs bins the band by key, certifies the bracket
//               and solves on the one bin that holds the root (solve.cuh)
//   k_recover   cooperative, exits at once unless a row failed certification:
//               widens the bracket once, then falls back to a full radix sort
//               of the row (the worst-case branch of the abstract)
//   k_memb      memberships p (section 2.1) plus sum f and sum p
//
// and two for the backward pass (section 2.1, analytic VJP): a reduction for
// lambda = sum g f / sum f, then grad = f (g - lambda).  The HBM passes run in
// alternating directions so that the part of the row the previous pass left in
// L2 is read first.
#include <algorithm>

#include <cooperative_groups.h>

#include "block_sort.cuh"
#include "common.cuh"
#include "launch.h"
#include "solve.cuh"
#include "tma.cuh"

namespace lapsum {
namespace {

namespace cg = cooperative_groups;

constexpr int NT = kStreamThreads;
constexpr int NW = NT / 32;
constexpr int U = 4;              // float4 loads per thread per chunk
constexpr int CHUNK4 = NT * U;    // float4 per chunk (4096 scores)
constexpr int kTile = 2048;       // fallback scatter tile (keys)

struct FPart {
  long long nL;
  double SL, SR;
  uint32_t bad, pad;
};
struct MPart {
  double a, b, c, pad;
};

__device__ __forceinline__ RowCtl* ctl_of(const StreamPlan& P, int64_t r) {
  return reinterpret_cast<RowCtl*>(P.ctl) + r;
}
__device__ __forceinline__ FPart* fpart_of(const StreamPlan& P, int64_t r) {
  return reinterpret_cast<FPart*>(P.fpart) + r * kMaxGridPerRow;
}
__device__ __forceinline__ MPart* mpart_of(const StreamPlan& P, int64_t r) {
  return reinterpret_cast<MPart*>(P.mpart) + r * kMaxGridPerRow;
}
__device__ __forceinline__ float* band_of(const StreamPlan& P, int64_t r) { return P.band + r * P.band_cap; }
__device__ __forceinline__ uint32_t* samp_of(const StreamPlan& P, int64_t r) { return P.samp + r * (int64_t)P.m; }
// the candidate list of a row starts 16-byte aligned (rows m rounded up to 4)
__device__ __forceinline__ uint32_t* cand_of(const StreamPlan& P, int64_t r) {
  return P.cand + r * (int64_t)((P.m + 3) & ~3);
}
__device__ __forceinline__ uint32_t* h1_of(const StreamPlan& P, int64_t r) { return P.hist1 + r * 2048; }
__device__ __forceinline__ uint32_t* h2_of(const StreamPlan& P, int64_t r) { return P.hist2 + r * 4096; }
__device__ __forceinline__ uint32_t* h3_of(const StreamPlan& P, int64_t r) { return P.hist3 + r * 2048; }

// control words written earlier in the same kernel are read around L1
template <typename T>
__device__ __forceinline__ T vld(const T* p) {
  return *reinterpret_cast<const volatile T*>(p);
}

// ===========================================================================
// localization: sample keys and the radix select of two order statistics
// ===========================================================================

// bin holding ascending rank `rank` in a global histogram of NB bins; every
// thread receives (bin, rank inside the bin)
template <int NB>
__device__ void find_bin(const uint32_t* gh, uint32_t rank, uint32_t* scr, int* bin, uint32_t* rem) {
  constexpr int PER = NB / NT;
  __shared__ int s_bin;
  __shared__ uint32_t s_rem;
  uint32_t v[PER];
  uint32_t loc = 0;
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    v[i] = __ldcg(gh + threadIdx.x * PER + i);
    loc += v[i];
  }
  if (threadIdx.x == 0) {
    s_bin = NB - 1;
    s_rem = 0;
  }
  const uint32_t base = block_excl_prefix_u32<NT>(loc, scr, nullptr);
  if (rank >= base && rank < base + loc) {
    uint32_t c = base;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      if (rank < c + v[i]) {
        s_bin = threadIdx.x * PER + i;
        s_rem = rank - c;
        break;
      }
      c += v[i];
    }
  }
  __syncthreads();
  *bin = s_bin;
  *rem = s_rem;
  __syncthreads();
}

// warp-aggregated shared-memory histogram increment
__device__ __forceinline__ void hist_add(uint32_t* h, uint32_t bin, bool act) {
  const uint32_t amask = __ballot_sync(0xffffffffu, act);
  if (act) {
    const uint32_t peers = __match_any_sync(amask, bin);
    if ((threadIdx.x & 31) == __ffs(peers) - 1) atomicAdd(h + bin, __popc(peers));
  }
}

__device__ void flush_hist(const uint32_t* sh, uint32_t* gh, int nb) {
  __syncthreads();
  for (int i = threadIdx.x; i < nb; i += NT)
    if (sh[i]) atomicAdd(gh + i, sh[i]);
  __syncthreads();
}

// Radix select of the two bracket edges over the stored sample keys, 11, 11
// and 10 bits per level.  Each level is a histogram of the keys that share the
// prefix found so far; one block then finds, for both edges, the bin holding
// the wanted rank and the rank left inside it (sel_pick).

__device__ void sel_hist1(const uint32_t* samp, int m, int cta, int ncta, uint32_t* gh1, uint32_t* sh) {
  for (int i = threadIdx.x; i < 2048; i += NT) sh[i] = 0u;
  __syncthreads();
  for (int j0 = cta * NT; j0 < m; j0 += ncta * NT) {
    const int j = j0 + threadIdx.x;
    const bool act = j < m;
    const uint32_t key = act ? __ldcg(samp + j) : 0u;
    hist_add(sh, key >> 21, act);
  }
  flush_hist(sh, gh1, 2048);
}

__device__ void sel_hist2(const uint32_t* samp, int m, int cta, int ncta, const int b1[2], uint32_t* gh2,
                          uint32_t* sh) {
  for (int i = threadIdx.x; i < 4096; i += NT) sh[i] = 0u;
  __syncthreads();
  for (int j0 = cta * NT; j0 < m; j0 += ncta * NT) {
    const int j = j0 + threadIdx.x;
    const bool act = j < m;
    const uint32_t key = act ? __ldcg(samp + j) : 0u;
    const uint32_t top = key >> 21, d = (key >> 10) & 2047u;
    hist_add(sh, d, act && top == (uint32_t)b1[0]);
    hist_add(sh + 2048, d, act && top == (uint32_t)b1[1]);
  }
  flush_hist(sh, gh2, 4096);
}

// sel_hist2, and the keys of the two level-1 bins appended to `cand` (one
// atomic on *cnt per warp step that holds any)
__device__ void sel_hist2_stash(const uint32_t* samp, int m, int cta, int ncta, const int b1[2], uint32_t* gh2,
                                uint32_t* sh, uint32_t* cand, uint32_t* cnt) {
  const int lane = threadIdx.x & 31;
  for (int i = threadIdx.x; i < 4096; i += NT) sh[i] = 0u;
  __syncthreads();
  constexpr int kU = 4;  // keys loaded before any is used
  const int step = ncta * NT;
  for (int j0 = cta * NT; j0 < m; j0 += kU * step) {
    uint32_t keys[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int j = j0 + u * step + (int)threadIdx.x;
      keys[u] = j < m ? __ldcg(samp + j) : 0u;
    }
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const bool act = j0 + u * step + (int)threadIdx.x < m;
      const uint32_t key = keys[u];
      const uint32_t top = key >> 21, d = (key >> 10) & 2047u;
      const bool in0 = act && top == (uint32_t)b1[0], in1 = act && top == (uint32_t)b1[1];
      hist_add(sh, d, in0);
      hist_add(sh + 2048, d, in1);
      const uint32_t cm = __ballot_sync(0xffffffffu, in0 || in1);
      if (cm) {
        uint32_t base = 0u;
        if (lane == 0) base = atomicAdd(cnt, (uint32_t)__popc(cm));
        base = __shfl_sync(0xffffffffu, base, 0);
        if (in0 || in1) cand[base + (uint32_t)__popc(cm & ((1u << lane) - 1u))] = key;
      }
    }
  }
  flush_hist(sh, gh2, 4096);
}

__device__ void sel_hist3(const uint32_t* samp, int m, int cta, int ncta, const uint32_t pre[2], uint32_t* gh3,
                          uint32_t* sh) {
  for (int i = threadIdx.x; i < 2048; i += NT) sh[i] = 0u;
  __syncthreads();
  for (int j0 = cta * NT; j0 < m; j0 += ncta * NT) {
    const int j = j0 + threadIdx.x;
    const bool act = j < m;
    const uint32_t key = act ? __ldcg(samp + j) : 0u;
    const uint32_t p = key >> 10, d = key & 1023u;
    hist_add(sh, d, act && p == pre[0]);
    hist_add(sh + 1024, d, act && p == pre[1]);
  }
  flush_hist(sh, gh3, 2048);
}

// one level's pick for both edges (one block): the bin of histogram gh (the
// edge's own histogram at gh + t*NB when per_edge) that holds rank rk[t], and
// the rank left inside it
template <int NB>
__device__ void sel_pick(const uint32_t* gh, bool per_edge, const uint32_t rk[2], uint32_t* scr, int bin[2],
                         uint32_t rem[2]) {
  for (int t = 0; t < 2; ++t) find_bin<NB>(gh + (per_edge ? t * NB : 0), rk[t], scr, &bin[t], &rem[t]);
}

__device__ void store_pick(RowCtl* c, int level, const int bin[2], const uint32_t rem[2]) {
  if (threadIdx.x == 0) {
    for (int t = 0; t < 2; ++t) {
      c->sel_bin[level][t] = bin[t];
      c->sel_rem[level][t] = rem[t];
    }
    __threadfence();
  }
  __syncthreads();
}

__device__ __forceinline__ uint32_t level3_prefix(const RowCtl* c, int t) {
  return ((uint32_t)vld(&c->sel_bin[0][t]) << 11) | (uint32_t)vld(&c->sel_bin[1][t]);
}

// bracket of a row (one thread)
__device__ void write_plan(RowCtl* c, int m, const uint32_t keys[2], int rlo, int rhi, bool vlo, bool vhi) {
  const float vl = key2f(keys[0]), vh = key2f(keys[1]);
  c->aL = vlo ? vl : -CUDART_INF_F;
  c->aR = vhi ? vh : CUDART_INF_F;
  c->rank_lo = rlo;
  c->rank_hi = rhi;
  c->valid_lo = vlo ? 1u : 0u;
  c->valid_hi = vhi ? 1u : 0u;
  c->m = m;
  c->sel_key[0] = keys[0];
  c->sel_key[1] = keys[1];
}

__global__ void __launch_bounds__(NT) k_sample(const StreamPlan P, const float* __restrict__ scores) {
  __shared__ uint32_t sh[2048];
  __shared__ uint32_t scr[64];
  const int64_t r = blockIdx.y;
  for (int i = threadIdx.x; i < 2048; i += NT) sh[i] = 0u;
  __syncthreads();
  const float* row = scores + r * P.stride;
  const uint64_t s = row_stream(P.seed, (uint64_t)r);
  uint32_t* samp = samp_of(P, r);
  const RowArgs ra = row_args(P, r);
  const int stride = gridDim.x * NT;
  // a sharded row draws the indices of the whole row and gathers those of its
  // shard; the others stay key 0 (no finite score has that key), so the sum
  // of the GPUs' sample arrays is the full sample
  const uint64_t nt = (uint64_t)(P.shard ? P.n_total : P.n);
  const uint64_t lo = P.shard ? (uint64_t)P.shard_lo : 0u;
  for (int j0 = blockIdx.x * NT; j0 < P.m; j0 += 4 * stride) {
    float v[4];
    bool own[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int j = j0 + u * stride + threadIdx.x;
      const uint64_t I = (j < P.m) ? sample_index(s, (uint64_t)j, nt) : 0u;
      own[u] = j < P.m && I >= lo && I - lo < (uint64_t)P.n;
      v[u] = own[u] ? __ldg(row + (I - lo)) : 0.0f;
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int j = j0 + u * stride + threadIdx.x;
      uint32_t key = 0u;
      if (own[u]) {
        const double Y = (double)v[u] + laplace_noise(s, (uint64_t)j, ra.alpha);
        key = f2key(__double2float_rn(Y));
      }
      if (j < P.m) samp[j] = key;
      hist_add(sh, key >> 21, own[u]);
    }
  }
  flush_hist(sh, h1_of(P, r), 2048);
  if (P.shard) return;  // the pick waits for the other GPUs' histograms
  RowCtl* c = ctl_of(P, r);
  if (last_block_done(&c->done_s1, gridDim.x)) {
    const RowRanks rr = row_ranks(P, ra.k);
    const uint32_t rk[2] = {(uint32_t)rr.rank_lo, (uint32_t)rr.rank_hi};
    int bin[2];
    uint32_t rem[2];
    sel_pick<2048>(h1_of(P, r), false, rk, scr, bin, rem);
    store_pick(c, 0, bin, rem);
  }
}

// sharded rows: the level-1 pick, once the histograms of all GPUs are summed
__global__ void __launch_bounds__(NT) k_pick1(const StreamPlan P) {
  __shared__ uint32_t scr[64];
  const int64_t r = blockIdx.y;
  const RowRanks rr = row_ranks(P, row_args(P, r).k);
  const uint32_t rk[2] = {(uint32_t)rr.rank_lo, (uint32_t)rr.rank_hi};
  int bin[2];
  uint32_t rem[2];
  sel_pick<2048>(h1_of(P, r), false, rk, scr, bin, rem);
  store_pick(ctl_of(P, r), 0, bin, rem);
}

__global__ void __launch_bounds__(NT) k_select2(const StreamPlan P) {
  __shared__ uint32_t sh[4096];
  __shared__ uint32_t scr[64];
  wait_prior_grid();
  const int64_t r = blockIdx.y;
  RowCtl* c = ctl_of(P, r);
  const int b1[2] = {c->sel_bin[0][0], c->sel_bin[0][1]};
  sel_hist2(samp_of(P, r), P.m, blockIdx.x, gridDim.x, b1, h2_of(P, r), sh);
  if (last_block_done(&c->done_s2, gridDim.x)) {
    const uint32_t rk[2] = {c->sel_rem[0][0], c->sel_rem[0][1]};
    int bin[2];
    uint32_t rem[2];
    sel_pick<2048>(h2_of(P, r), true, rk, scr, bin, rem);
    store_pick(c, 1, bin, rem);
  }
}

// Levels 2 and 3 of the selection in one launch: every block histograms the
// second level and stashes the keys of the two level-1 bins; the last block
// picks level 2, then runs level 3 over the stash alone.
__global__ void __launch_bounds__(NT) k_select23(const StreamPlan P) {
  __shared__ uint32_t sh[4096];
  __shared__ uint32_t scr[64];
  wait_prior_grid();
  const int64_t r = blockIdx.y;
  RowCtl* c = ctl_of(P, r);
  const int b1[2] = {c->sel_bin[0][0], c->sel_bin[0][1]};
  uint32_t* cand = cand_of(P, r);
  sel_hist2_stash(samp_of(P, r), P.m, blockIdx.x, gridDim.x, b1, h2_of(P, r), sh, cand, &c->cand_cnt);
  if (last_block_done(&c->done_s2, gridDim.x)) {
    uint32_t rk[2] = {c->sel_rem[0][0], c->sel_rem[0][1]};
    int bin[2];
    uint32_t rem[2];
    sel_pick<2048>(h2_of(P, r), true, rk, scr, bin, rem);
    const uint32_t pre[2] = {((uint32_t)b1[0] << 11) | (uint32_t)bin[0], ((uint32_t)b1[1] << 11) | (uint32_t)bin[1]};
    // level 3 over the stashed keys (every key that can share a 22-bit prefix)
    const uint32_t nc = vld(&c->cand_cnt);
    for (int i = threadIdx.x; i < 2048; i += NT) sh[i] = 0u;
    __syncthreads();
    // 16-byte loads, kQ of them in flight per thread (one block walks the
    // whole stash); the list starts 16-byte aligned (m is a multiple of 4)
    constexpr int kQ = 4;
    const uint4* c4 = reinterpret_cast<const uint4*>(cand);
    const uint32_t nq = nc >> 2;
    for (uint32_t q0 = 0; q0 < nq; q0 += kQ * NT) {
      uint4 v[kQ];
#pragma unroll
      for (int u = 0; u < kQ; ++u) {
        const uint32_t q = q0 + u * NT + threadIdx.x;
        v[u] = q < nq ? __ldcg(c4 + q) : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int u = 0; u < kQ; ++u) {
        const bool act = q0 + u * NT + threadIdx.x < nq;
        const uint32_t ks[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          hist_add(sh, ks[w] & 1023u, act && (ks[w] >> 10) == pre[0]);
          hist_add(sh + 1024, ks[w] & 1023u, act && (ks[w] >> 10) == pre[1]);
        }
      }
    }
    for (uint32_t j = 4 * nq + threadIdx.x; j < 4 * nq + NT; j += NT) {  // the last 0-3 keys
      const bool act = j < nc;
      const uint32_t key = act ? __ldcg(cand + j) : 0u;
      hist_add(sh, key & 1023u, act && (key >> 10) == pre[0]);
      hist_add(sh + 1024, key & 1023u, act && (key >> 10) == pre[1]);
    }
    __syncthreads();
    uint32_t* h3 = h3_of(P, r);
    for (int i = threadIdx.x; i < 2048; i += NT) h3[i] = sh[i];
    __syncthreads();
    rk[0] = rem[0];
    rk[1] = rem[1];
    sel_pick<1024>(h3, true, rk, scr, bin, rem);
    const uint32_t keys[2] = {(pre[0] << 10) | (uint32_t)bin[0], (pre[1] << 10) | (uint32_t)bin[1]};
    const RowRanks rr = row_ranks(P, row_args(P, r).k);
    if (threadIdx.x == 0) write_plan(c, P.m, keys, rr.rank_lo, rr.rank_hi, rr.valid_lo, rr.valid_hi);
  }
}

__global__ void __launch_bounds__(NT) k_select3(const StreamPlan P) {
  __shared__ uint32_t sh[2048];
  __shared__ uint32_t scr[64];
  wait_prior_grid();
  const int64_t r = blockIdx.y;
  RowCtl* c = ctl_of(P, r);
  const uint32_t pre[2] = {level3_prefix(c, 0), level3_prefix(c, 1)};
  sel_hist3(samp_of(P, r), P.m, blockIdx.x, gridDim.x, pre, h3_of(P, r), sh);
  if (last_block_done(&c->done_sel, gridDim.x)) {
    const uint32_t rk[2] = {c->sel_rem[1][0], c->sel_rem[1][1]};
    int bin[2];
    uint32_t rem[2];
    sel_pick<1024>(h3_of(P, r), true, rk, scr, bin, rem);
    const uint32_t keys[2] = {(pre[0] << 10) | (uint32_t)bin[0], (pre[1] << 10) | (uint32_t)bin[1]};
    const RowRanks rr = row_ranks(P, row_args(P, r).k);
    if (threadIdx.x == 0) write_plan(c, P.m, keys, rr.rank_lo, rr.rank_hi, rr.valid_lo, rr.valid_hi);
  }
}

// ===========================================================================
// stream and filter (section 2.2, step 2)
// ===========================================================================

// In-band values never leave the streaming loop through global memory: a
// lane holding some writes its chunk to a shared scratch slot and copies the
// flagged values into its own column of a shared stage (no atomics, no global
// reload).  A warp empties its 32 columns into the row's band with one atomic
// for the whole warp, when one of them is about to fill and at the end.  The
// band is one unsorted array per row; the band kernel bins it by key.
constexpr int kLaneStage = 24;  // stage column per lane (floats)

struct FilterCtx {
  float aL, aR, c2;
  uint32_t* cnt;    // values appended to the band so far (may exceed cap)
  uint32_t* kmax;   // largest key appended
  uint32_t* nkmin;  // bitwise complement of the smallest key appended
  float* band;
  uint32_t cap;
};

// Appends the staged values of all 32 lanes (col[j * NT], j < ncol) to the
// band; NaN and inf are flagged instead.  All lanes of the warp call it.
__device__ __noinline__ void flush_warp(const FilterCtx& f, const float* col, int ncol, uint32_t& bad,
                                        uint32_t& ovf) {
  const int lane = threadIdx.x & 31;
  int good = 0;
  uint32_t kmin = 0xFFFFFFFFu, kmax = 0u;
  for (int j = 0; j < ncol; ++j) {
    const float x = col[j * NT];
    if (fabsf(x) < CUDART_INF_F) {
      ++good;
      const uint32_t k = f2key(x);
      kmin = min(kmin, k);
      kmax = max(kmax, k);
    } else {
      bad = 1u;
    }
  }
  int incl = good;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  const int total = __shfl_sync(0xffffffffu, incl, 31);
  if (total == 0) return;
  kmin = __reduce_min_sync(0xffffffffu, kmin);
  kmax = __reduce_max_sync(0xffffffffu, kmax);
  uint32_t base = 0u;
  if (lane == 0) {
    base = atomicAdd(f.cnt, (uint32_t)total);
    atomicMax(f.kmax, kmax);
    atomicMax(f.nkmin, ~kmin);
  }
  base = __shfl_sync(0xffffffffu, base, 0);
  uint32_t pos = base + (uint32_t)(incl - good);
  for (int j = 0; j < ncol; ++j) {
    const float x = col[j * NT];
    if (fabsf(x) < CUDART_INF_F) {
      if (pos < f.cap) f.band[pos] = x;
      else ovf = 1u;
      ++pos;
    }
  }
}

// The running sums of one lane of the filter.
struct FilterAcc {
  long long nl = 0;
  double sl = 0.0, sr = 0.0;
  // sum of the scores scaled by 2^-64: finite for any finite scores (at most
  // 2^40 of them), inf or NaN as soon as one score is
  float2 fs2 = make_float2(0.0f, 0.0f);
  int ncol = 0;  // values staged in this lane's column
};

// One lane's U float4 of a chunk (v): classification and tail terms two
// scores at a time (packed fp32x2 arithmetic; the saturated side indicators
// of classify): tail sums, the left count, and the positions of the scores
// outside the band as bits of an exact fp32 sum.  The rare in-band values are
// copied into the lane's column (stride NT) from at(i), the lane's i-th score
// of the chunk (i = 4u + component).
template <typename At>
__device__ __forceinline__ void filter_chunk(const float4 (&v)[U], float2 naL2, float2 aR2, float2 c22,
                                             const At& at, float* col, FilterAcc& a) {
  const float2 k64 = make_float2(0x1p-64f, 0x1p-64f);
  float2 pl2 = make_float2(0.0f, 0.0f), pr2 = pl2, cl2 = pl2, ob2 = pl2;
#pragma unroll
  for (int u = 0; u < U; ++u) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const float2 x2 = h ? make_float2(v[u].z, v[u].w) : make_float2(v[u].x, v[u].y);
      const Side2 sd = classify2(x2, naL2, aR2, c22);
      const float bit = (float)(1u << (4 * u + 2 * h));
      pl2 = fma2(sd.L, sd.e, pl2);
      pr2 = fma2(sd.R, sd.e, pr2);
      cl2 = add2(cl2, sd.L);
      ob2 = fma2(add2(sd.L, sd.R), make_float2(bit, 2.0f * bit), ob2);
      a.fs2 = fma2(x2, k64, a.fs2);
    }
  }
  a.sl += (double)(pl2.x + pl2.y);
  a.sr += (double)(pr2.x + pr2.y);
  a.nl += (long long)(cl2.x + cl2.y);
  uint32_t mask = ~(uint32_t)(ob2.x + ob2.y) & ((1u << (4 * U)) - 1u);  // in-band positions
  while (mask) {  // rare
    const int i = __ffs(mask) - 1;
    mask &= mask - 1u;
    col[a.ncol * NT] = at(i);
    ++a.ncol;
  }
}

__device__ __forceinline__ FilterCtx filter_ctx(const StreamPlan& P, int64_t r, RowCtl* c) {
  FilterCtx f;
  f.aL = vld(&c->aL);
  f.aR = vld(&c->aR);
  f.c2 = (float)((1.0 / row_args(P, r).alpha) * (double)kLog2e);
  f.cnt = &c->band_cnt;
  f.kmax = &c->band_kmax;
  f.nkmin = &c->band_nkmin;
  f.band = band_of(P, r);
  f.cap = (uint32_t)P.band_cap;
  return f;
}

// The scores outside the float4 body (one per thread per step, the same trip
// count for the whole block), the last flush, and the block's partial sums.
// NTB: the block's threads; the first NT of them take the tail.
template <int NTB>
__device__ void filter_finish(const StreamPlan& P, int64_t r, const float* __restrict__ row, RowCtl* c, int cta,
                              int ncta, double* red, float* col, const FilterCtx& f, FilterAcc& a, int head,
                              int64_t nb4, uint32_t bad, uint32_t ovf) {
  float fsum = a.fs2.x + a.fs2.y;
  const int64_t nrest = threadIdx.x < NT ? P.n - 4 * nb4 : 0;
  for (int64_t j0 = (int64_t)cta * NT; j0 < nrest; j0 += (int64_t)ncta * NT) {
    const int64_t j = j0 + threadIdx.x;
    if (j < nrest) {
      const float x = row[rest_index(j, head, nb4)];
      const Side sd = classify(x, f.aL, f.aR, f.c2);
      if (sd.L != 0.0f) {
        a.sl += (double)sd.e;
        ++a.nl;
      }
      if (sd.R != 0.0f) a.sr += (double)sd.e;
      fsum = fmaf(x, 0x1p-64f, fsum);
      if (sd.L + sd.R == 0.0f) {
        col[a.ncol * NT] = x;
        ++a.ncol;
      }
    }
    if (__any_sync(0xffffffffu, a.ncol >= kLaneStage)) {
      flush_warp(f, col, a.ncol, bad, ovf);
      a.ncol = 0;
    }
  }
  if (threadIdx.x < NT && __any_sync(0xffffffffu, a.ncol > 0)) flush_warp(f, col, a.ncol, bad, ovf);
  if (!(fabsf(fsum) < CUDART_INF_F)) bad = 1u;
  if (ovf) atomicOr(&c->flags, ROW_OVERFLOW);
  const long long nl = block_sum<NTB, long long>(a.nl, reinterpret_cast<long long*>(red));
  const double sl = block_sum<NTB, double>(a.sl, red);
  const double sr = block_sum<NTB, double>(a.sr, red);
  bad = block_or<NTB>(bad, reinterpret_cast<uint32_t*>(red));
  if (threadIdx.x == 0) {
    FPart p;
    p.nL = nl;
    p.SL = sl;
    p.SR = sr;
    p.bad = bad;
    p.pad = 0u;
    fpart_of(P, r)[cta] = p;
  }
  __syncthreads();
}

// The filter pass of the recovery kernel (a re-filter after a widening):
// chunks loaded straight into registers, two in flight per thread (the next
// chunk's loads are issued before the current one is processed).  stage:
// the lane columns, then one scratch chunk per lane.
__device__ void filter_phase(const StreamPlan& P, int64_t r, const float* __restrict__ row, RowCtl* c, int cta,
                             int ncta, double* red, float* stage) {
  const int64_t n = P.n;
  // the 16-byte aligned body in chunks of CHUNK4 float4 (after a head of 0-3
  // scores); the scores outside it go through filter_finish
  const int head = row_head(row, n);
  const float4* x4 = reinterpret_cast<const float4*>(row + head);
  const int64_t nchunks = ((n - head) >> 2) / CHUNK4;
  float4 nx[U];
  if (cta < nchunks) {
#pragma unroll
    for (int u = 0; u < U; ++u) nx[u] = __ldg(x4 + (int64_t)cta * CHUNK4 + threadIdx.x + u * NT);
  }
  const FilterCtx f = filter_ctx(P, r, c);
  float* col = stage + threadIdx.x;  // this lane's column, stride NT
  float4* scratch = reinterpret_cast<float4*>(stage + kLaneStage * NT) + threadIdx.x * U;  // U float4
  const float2 naL2 = make_float2(-f.aL, -f.aL), aR2 = make_float2(f.aR, f.aR), c22 = make_float2(f.c2, f.c2);
  FilterAcc acc;
  uint32_t bad = 0u, ovf = 0u;
  for (int64_t q = cta; q < nchunks; q += ncta) {
    float4 v[U];
#pragma unroll
    for (int u = 0; u < U; ++u) v[u] = nx[u];
    if (q + ncta < nchunks) {
#pragma unroll
      for (int u = 0; u < U; ++u) nx[u] = __ldg(x4 + (q + ncta) * CHUNK4 + threadIdx.x + u * NT);
    }
    // the lane's chunk goes to its scratch slot only when it holds in-band
    // values (read back there by position)
    bool spilled = false;
    filter_chunk(v, naL2, aR2, c22,
                 [&](int i) {
                   if (!spilled) {
#pragma unroll
                     for (int u = 0; u < U; ++u) scratch[u] = v[u];
                     spilled = true;
                   }
                   return reinterpret_cast<const float*>(scratch)[i];
                 },
                 col, acc);
    if (__any_sync(0xffffffffu, acc.ncol > kLaneStage - 4 * U)) {
      flush_warp(f, col, acc.ncol, bad, ovf);
      acc.ncol = 0;
    }
  }
  filter_finish<NT>(P, r, row, c, cta, ncta, red, col, f, acc, head, nchunks * CHUNK4, bad, ovf);
}

// shared memory of the recovery kernel's filter pass: lane columns plus one
// scratch chunk per lane
constexpr size_t kFilterStageBytes = (size_t)(kLaneStage * NT) * 4 + (size_t)NT * U * 16;

// The filter kernel: the chunks of a block reach shared memory through bulk
// copies (the Tensor Memory Accelerator) into a ring of kFilterRing stages.
// One producer warp (one lane of it) issues them, up to kFilterRing chunks
// ahead: the bytes in flight per SM are the ring's, not what registers can
// hold.  Eight consumer warps classify each chunk as it lands (full barrier of
// its stage) and release the stage (empty barrier, one arrival per warp)
// once they have copied out its rare in-band values; no block-wide barrier
// per chunk, so the warps drift apart by up to the ring's depth.
constexpr int kFilterRing = 4;
constexpr int kFilterThreads = NT + 32;  // consumers + the producer warp
constexpr uint32_t kChunkBytes = CHUNK4 * 16u;
struct FilterSmem {
  float4 ring[kFilterRing][CHUNK4];
  float stage[kLaneStage * NT];  // the consumer lanes' columns
  double red[64];
  uint64_t full[kFilterRing];   // a stage has landed (the copy's bytes)
  uint64_t empty[kFilterRing];  // a stage has been read by every consumer warp
  int issued;                   // chunks the producer issued
  int late;                     // a wait ran out
};
constexpr size_t kFilterSmemBytes = sizeof(FilterSmem);

__global__ void __launch_bounds__(kFilterThreads, 2) k_filter(const StreamPlan P, const float* __restrict__ scores) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  FilterSmem& S = *reinterpret_cast<FilterSmem*>(smem_raw);
  const int64_t r = blockIdx.y;
  const int cta = blockIdx.x, ncta = gridDim.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const float* row = scores + r * P.stride;
  RowCtl* c = ctl_of(P, r);
  const int head = row_head(row, P.n);
  const float4* x4 = reinterpret_cast<const float4*>(row + head);
  const int64_t nchunks = ((P.n - head) >> 2) / CHUNK4;
  const int mine = cta < nchunks ? (int)((nchunks - 1 - cta) / ncta) + 1 : 0;  // this block's chunks
  auto chunk = [&](int it) { return x4 + (cta + (int64_t)it * ncta) * CHUNK4; };
  // test knob: rows 1, 5, 9, ... issue no copy for their first chunk, so
  // that the waits for it run out (rows 3, 7, ... time out in the recovery
  // kernel instead)
  const bool force_to = P.force_timeout && !P.shard && (r & 3) == 1;
  // the scores are the caller's: the first stages are requested before
  // waiting for the kernel that wrote the bracket
  if (threadIdx.x == 0) {
    for (int s = 0; s < kFilterRing; ++s) {
      mbar_init(&S.full[s], 1u);
      mbar_init(&S.empty[s], (uint32_t)NW);
    }
    for (int s = force_to ? 1 : 0; s < kFilterRing && s < mine; ++s) {
      mbar_arrive_expect_tx(&S.full[s], kChunkBytes);
      bulk_load(S.ring[s], chunk(s), kChunkBytes, &S.full[s]);
    }
    S.issued = min(kFilterRing, mine);
    S.late = 0;
  }
  __syncthreads();
  wait_prior_grid();
  const uint32_t limit = spin_limit_of(P.spin_limit);
  const FilterCtx f = filter_ctx(P, r, c);
  float* col = S.stage + (threadIdx.x < NT ? threadIdx.x : 0);
  FilterAcc acc;
  uint32_t bad = 0u, ovf = 0u;
  if (warp == NW) {
    // producer: refill a stage once every consumer warp has released it
    if (lane == 0) {
      int it = kFilterRing;
      for (; it < mine; ++it) {
        const int slot = it % kFilterRing;
        if (!mbar_wait_bounded(&S.empty[slot], (uint32_t)(it / kFilterRing - 1) & 1u, limit)) {
          S.late = 1;
          break;
        }
        fence_proxy_async_smem();
        mbar_arrive_expect_tx(&S.full[slot], kChunkBytes);
        bulk_load(S.ring[slot], chunk(it), kChunkBytes, &S.full[slot]);
      }
      const int issued = it < mine ? it : mine;  // chunks [0, issued) were requested
      if (issued > S.issued) S.issued = issued;
    }
  } else {
    const float2 naL2 = make_float2(-f.aL, -f.aL), aR2 = make_float2(f.aR, f.aR);
    const float2 c22 = make_float2(f.c2, f.c2);
    for (int it = 0; it < mine; ++it) {
      const int slot = it % kFilterRing;
      // a warp-uniform decision: every lane polls, the warp gives up together
      const bool ok = mbar_wait_bounded(&S.full[slot], (uint32_t)(it / kFilterRing) & 1u, limit);
      if (!__all_sync(0xffffffffu, ok)) {
        S.late = 1;  // a copy that did not land in time: the row's results are void
        break;
      }
      const float4* st = S.ring[slot] + threadIdx.x;
      float4 v[U];
#pragma unroll
      for (int u = 0; u < U; ++u) v[u] = st[u * NT];
      filter_chunk(v, naL2, aR2, c22,
                   [&](int i) { return reinterpret_cast<const float*>(st + (i >> 2) * NT)[i & 3]; }, col, acc);
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.empty[slot]);
      if (__any_sync(0xffffffffu, acc.ncol > kLaneStage - 4 * U)) {
        flush_warp(f, col, acc.ncol, bad, ovf);
        acc.ncol = 0;
      }
    }
  }
  __syncthreads();
  if (S.late) {
    // the last chunks issued may still be in flight: let them land (again
    // with a limit) before the block leaves; the band kernel reads the flag
    // and solves nothing
    if (threadIdx.x == 0) {
      for (int j = max(0, S.issued - kFilterRing); j < S.issued; ++j)
        (void)mbar_wait_bounded(&S.full[j % kFilterRing], (uint32_t)(j / kFilterRing) & 1u, limit);
      atomicOr(&c->flags, ROW_TIMEOUT);
    }
    __syncthreads();
  }
  filter_finish<kFilterThreads>(P, r, row, c, cta, ncta, S.red, col, f, acc, head, nchunks * CHUNK4, bad, ovf);
}

// ===========================================================================
// band: key bins, certification, and the exact solve on the one bin that
// holds the root (section 2.2, steps 3-4)
// ===========================================================================

struct KeyGroupsG {  // consecutive groups of `g` sorted keys in global memory
  const uint32_t* k;
  int g;
  __device__ float get(int grp, int i) const { return key2f(__ldcg(k + (int64_t)grp * g + i)); }
};

// Shared-memory layout of the recovery kernel's full sort for tiles of up to
// C keys: keys and radix scratch (4C + 4C bytes), per-value prefix sums of
// the solve (8C bytes), the radix histograms and the reduction scratch.
struct BandSmem {
  uint32_t* kbuf;
  uint32_t* tbuf;
  double* dscr;
  uint32_t* hist;
  double* red;
  __device__ BandSmem(unsigned char* smem, int C) {
    kbuf = reinterpret_cast<uint32_t*>(smem);
    tbuf = kbuf + C;
    dscr = reinterpret_cast<double*>(tbuf + C);
    hist = reinterpret_cast<uint32_t*>(dscr + C);
    red = reinterpret_cast<double*>(hist + SortScratch<NT>::kWords);
  }
  static constexpr size_t bytes(int C) { return (size_t)16 * C + (size_t)SortScratch<NT>::kWords * 4 + 64 * 8; }
};

// ---------------------------------------------------------------------------
// The band solve.  A cluster of CTAs (one CTA in the recovery kernel) owns a
// row's unsorted band; with more than one CTA, the leader (rank 0) holds no
// slice of it and is free for the solve.  Each level:
//   A  every worker CTA copies its slice of the band into shared memory and
//      bins it by key (2048 bins over the key window): count and extremes,
//      then the sums P = sum exp((y - ymax)/a), Q = sum exp((ymin - y)/a)
//      anchored at the bin's own extremes, in 2^-31 fixed point with exact
//      64-bit sums (order-independent, hence deterministic);
//   B  the CTAs merge the bins through distributed shared memory, in CTA
//      order, into the leader's bin table;
//   C  the leader runs the certified group solve (solve_bins): the bin that
//      holds the knot after the root.
// A single-key bin is solved at once; a bin of at most kTargetCap values is
// gathered into the leader's shared memory, sorted and solved value by value
// (by one warp when it has at most kWarpSortMax values); a larger one becomes
// the key window of the next level (three levels reach single keys).
// ---------------------------------------------------------------------------
constexpr int kBins = 2048;
constexpr int kTargetCap = kBins;  // a gathered bin becomes a table of its values
constexpr int kMaxLevels = 4;
constexpr int kMaxCluster = 16;
constexpr int kBandThreads = 512;
// P and Q are kept as exact integer sums of 2^-31 fixed-point terms (at most
// 2^31 each), split into 32-bit words that cannot overflow for the slice:
constexpr int kHalfSliceMax = 65535;          // two 16-bit limbs (two adds per term)
constexpr int kLimbBits = 11;                 // or three 11-bit limbs (three adds)
constexpr int kLimbSliceMax = (1 << 21) - 1;  // up to this many terms; beyond, a carried 64-bit sum
enum : uint32_t { kSumHalves = 0, kSumLimbs = 1, kSumWide = 2 };

struct BinPart {  // one CTA's bins
  uint32_t cnt[kBins];
  uint32_t kmin[kBins];  // this CTA's extreme keys per bin
  uint32_t kmax[kBins];
  uint32_t gmin[kBins];  // the whole cluster's: the anchors of the sums, so that
  uint32_t gmax[kBins];  // every CTA's terms are the same integers whatever its slice
  uint32_t P[3][kBins];  // limb words, by `mode`
  uint32_t Q[3][kBins];
  uint32_t mode;         // kSumHalves, kSumLimbs or kSumWide (low word, high word)
};
struct TargetBuf {
  uint32_t keys[kTargetCap];
  uint32_t sorted[kTargetCap];  // the bucket sort's output
  uint32_t scr[bucket_sort_scr_words(kBandThreads)];  // and its scratch
};
enum : int { kBandDone = 0, kBandRefine = 1, kBandExtract = 2 };
struct BandDecision {
  int action, tg, shift, level;
  uint32_t klo, khi;
  uint32_t count;  // gathered values of the target bin
};
constexpr int kStageCap = (int)(sizeof(BinTable<kBins>) / 4);
struct BandShared {
  union {
    BinTable<kBins> tab;     // the leader's merged bins
    float stage[kStageCap];  // a worker's slice of the band
  } tu;
  union {
    BinPart part;
    TargetBuf tgt;
  } u;
  double red[64];
  GroupPick pk;
  GroupPick pk2;  // the pick among the values of the gathered bin
  SolveOut so;
  SolveIn in;
  BandDecision dec;
};
constexpr size_t kBandSmemBytes = sizeof(BandShared);
// A lone band CTA sorts a band of at most kRunCap values whole (keys, the
// sort's output, then the prefix states and link factors of the one run, in
// the stage area) and solves it without key bins.
constexpr int kRunCap = 4096;
static_assert((size_t)kRunCap * (4 + 4 + 8 + 8) + 8 <= sizeof(float) * kStageCap, "run fits the stage");

template <typename T>
__device__ __forceinline__ T* at_rank(T* p, int q, int cs) {
  if (cs == 1) return p;
  return cg::this_cluster().map_shared_rank(p, q);
}
__device__ __forceinline__ void cl_sync(int cs) {
  if (cs > 1) cg::this_cluster().sync();
  else __syncthreads();
}

// smallest shift that maps the key window onto kBins bins
__device__ __forceinline__ int bin_shift(uint32_t klo, uint32_t khi) {
  const uint32_t d = khi - klo;
  int s = 0;
  while ((d >> s) >= (uint32_t)kBins) ++s;
  return s;
}
// key of edge e_t of the window (clamped to its top)
__device__ __forceinline__ uint32_t edge_key(uint32_t klo, uint32_t khi, int shift, int t) {
  const uint64_t e = (uint64_t)klo + ((uint64_t)t << shift);
  return e > (uint64_t)khi ? khi : (uint32_t)e;
}

// one term exp(d/alpha) (d <= 0) in 2^-31 fixed point (at most 2^31)
__device__ __forceinline__ uint32_t fx_term(float d, float c2) {
  return __float2uint_rn(exp2f(d * c2) * 0x1p31f);
}
// a term into two 16-bit limb words (plain reductions)
__device__ __forceinline__ void add_halves(uint32_t (*L)[kBins], int t, uint32_t v) {
  atomicAdd(&L[0][t], v & 0xFFFFu);
  atomicAdd(&L[1][t], v >> 16);
}
// a term into three limb words (no return value needed: plain reductions)
__device__ __forceinline__ void add_limbs(uint32_t (*L)[kBins], int t, uint32_t v) {
  constexpr uint32_t m = (1u << kLimbBits) - 1u;
  atomicAdd(&L[0][t], v & m);
  atomicAdd(&L[1][t], (v >> kLimbBits) & m);
  atomicAdd(&L[2][t], v >> (2 * kLimbBits));
}
// exact 64-bit sum in two words: the add that wraps the low word carries
__device__ __forceinline__ void add_wide(uint32_t (*L)[kBins], int t, uint32_t v) {
  const uint32_t old = atomicAdd(&L[0][t], v);
  if (old > 0xFFFFFFFFu - v) atomicAdd(&L[1][t], 1u);
}

// value j of a worker's slice: from the shared copy, or from L2
__device__ __forceinline__ float slice_val(const float* src, const float* stage, bool staged, int j) {
  return (staged && j < kStageCap) ? stage[j] : __ldcg(src + j);
}

constexpr int kSliceBatch = 8;  // loads in flight per thread

// Pass 1 over the n values at src: count and extreme keys per bin into bp.
// write_stage: copy the first kStageCap of them into `stage` on the way
// (otherwise they come from `stage` when read_stage).  All threads of the
// block call it.
template <int NTX>
__device__ void bin_count(const float* src, int n, bool write_stage, bool read_stage, float* stage, uint32_t klo,
                          uint32_t khi, int shift, BinPart& bp) {
  const uint32_t mode = n <= kHalfSliceMax ? kSumHalves : (n <= kLimbSliceMax ? kSumLimbs : kSumWide);
  for (int t = threadIdx.x; t < kBins; t += NTX) {
    bp.cnt[t] = 0u;
    bp.kmin[t] = 0xFFFFFFFFu;
    bp.kmax[t] = 0u;
#pragma unroll
    for (int l = 0; l < 3; ++l) {
      bp.P[l][t] = 0u;
      bp.Q[l][t] = 0u;
    }
  }
  if (threadIdx.x == 0) bp.mode = mode;
  __syncthreads();
  const bool first_from_stage = read_stage && !write_stage;
  for (int j0 = 0; j0 < n; j0 += NTX * kSliceBatch) {
    float v[kSliceBatch];
#pragma unroll
    for (int u = 0; u < kSliceBatch; ++u) {
      const int j = j0 + u * NTX + (int)threadIdx.x;
      v[u] = 0.0f;
      if (j < n) v[u] = slice_val(src, stage, first_from_stage, j);
    }
#pragma unroll
    for (int u = 0; u < kSliceBatch; ++u) {
      const int j = j0 + u * NTX + (int)threadIdx.x;
      if (j < n) {
        if (write_stage && j < kStageCap) stage[j] = v[u];
        const uint32_t key = f2key(v[u]);
        if (key >= klo && key <= khi) {
          const int t = (int)((key - klo) >> shift);
          atomicAdd(&bp.cnt[t], 1u);
          atomicMin(&bp.kmin[t], key);
          atomicMax(&bp.kmax[t], key);
        }
      }
    }
  }
  __syncthreads();
}

// The cluster's extreme keys per bin, into every CTA's gmin / gmax: this CTA
// merges its kBins / cs bins over all CTAs (L lanes per bin, each taking every
// L-th CTA) and writes them to all CTAs.  A cluster barrier must follow
// before they are read.
template <int NTX>
__device__ void merge_extremes(BandShared& S, int cs, int rank) {
  const int per = kBins / cs;
  int L = NTX / per;
  L = L < 1 ? 1 : (L > cs ? cs : L);
  const int sub = (int)threadIdx.x & (L - 1);
  for (int base = (int)threadIdx.x / L; base < per; base += NTX / L) {
    const int t = rank * per + base;
    uint32_t mn = 0xFFFFFFFFu, mx = 0u;
    for (int q = sub; q < cs; q += L) {
      const BinPart* pq = at_rank(&S.u.part, q, cs);
      mn = min(mn, pq->kmin[t]);
      mx = max(mx, pq->kmax[t]);
    }
    for (int o = 1; o < L; o <<= 1) {
      mn = min(mn, __shfl_xor_sync(0xffffffffu, mn, o));
      mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    }
    for (int q = sub; q < cs; q += L) {
      BinPart* pq = at_rank(&S.u.part, q, cs);
      pq->gmin[t] = mn;
      pq->gmax[t] = mx;
    }
  }
}

// Pass 2: the sums P = sum exp((y - ymax)/a) and Q = sum exp((ymin - y)/a) per
// bin, with ymax, ymin the cluster's extremes (bp.gmin / gmax), as integer
// sums of 2^-31 fixed-point terms: the same integers whichever CTA holds a
// value, so the merged sums do not depend on how the band was split.
template <int NTX>
__device__ void bin_sums(const float* src, int n, bool read_stage, const float* stage, uint32_t klo, uint32_t khi,
                         int shift, float c2, BinPart& bp) {
  const uint32_t mode = bp.mode;
  for (int j0 = 0; j0 < n; j0 += NTX * kSliceBatch) {
    float v[kSliceBatch];
#pragma unroll
    for (int u = 0; u < kSliceBatch; ++u) {
      const int j = j0 + u * NTX + (int)threadIdx.x;
      v[u] = (j < n) ? slice_val(src, stage, read_stage, j) : 0.0f;
    }
#pragma unroll
    for (int u = 0; u < kSliceBatch; ++u) {
      const int j = j0 + u * NTX + (int)threadIdx.x;
      if (j < n) {
        const float y = v[u];
        const uint32_t key = f2key(y);
        if (key >= klo && key <= khi) {
          const int t = (int)((key - klo) >> shift);
          const uint32_t tp = fx_term(y - key2f(bp.gmax[t]), c2);
          const uint32_t tq = fx_term(key2f(bp.gmin[t]) - y, c2);
          if (mode == kSumHalves) {
            add_halves(bp.P, t, tp);
            add_halves(bp.Q, t, tq);
          } else if (mode == kSumLimbs) {
            add_limbs(bp.P, t, tp);
            add_limbs(bp.Q, t, tq);
          } else {
            add_wide(bp.P, t, tp);
            add_wide(bp.Q, t, tq);
          }
        }
      }
    }
  }
}

// a CTA's limb words of one sum as the exact integer they stand for
__device__ __forceinline__ unsigned long long fx_int(uint32_t w0, uint32_t w1, uint32_t w2, uint32_t mode) {
  if (mode == kSumWide) return ((unsigned long long)w1 << 32) | w0;
  if (mode == kSumHalves) return ((unsigned long long)w1 << 16) + w0;
  return ((unsigned long long)w2 << (2 * kLimbBits)) + ((unsigned long long)w1 << kLimbBits) + w0;
}

// This CTA's share of the bins, merged over all CTAs into the leader's table
// together with the edge factors of solve_bins.  The sums are integers anchored
// at the cluster's extremes, so merging is an exact integer addition (the same
// result in any order).  L lanes per bin, each taking every L-th CTA; every
// load of a CTA's bin is issued before any is used.
template <int NTX>
__device__ void merge_bins(BandShared& S, int cs, int rank, uint32_t klo, uint32_t khi, int shift, double inva) {
  const int per = kBins / cs;
  int L = NTX / per;
  L = L < 1 ? 1 : (L > cs ? cs : L);
  // CTAs per lane: L = NTX cs / kBins (at least 1), so a lane takes at most
  // max(cs / L) = kBins / NTX of them
  constexpr int QM = kBins / NTX;
  static_assert(QM >= 1 && QM * NTX == kBins && kMaxCluster <= 16, "lanes per bin must cover the cluster");
  const int sub = (int)threadIdx.x & (L - 1);
  BinTable<kBins>* tab0 = at_rank(&S.tu.tab, 0, cs);
  for (int base = (int)threadIdx.x / L; base < per; base += NTX / L) {
    const int t = rank * per + base;
    uint32_t c[QM], p0[QM], p1[QM], p2[QM], q0[QM], q1[QM], q2[QM], md[QM];
#pragma unroll
    for (int i = 0; i < QM; ++i) {
      const int q = sub + i * L;
      c[i] = 0u;
      if (q < cs) {
        const BinPart* pq = at_rank(&S.u.part, q, cs);
        c[i] = pq->cnt[t];
        p0[i] = pq->P[0][t];
        p1[i] = pq->P[1][t];
        p2[i] = pq->P[2][t];
        q0[i] = pq->Q[0][t];
        q1[i] = pq->Q[1][t];
        q2[i] = pq->Q[2][t];
        md[i] = pq->mode;
      }
    }
    uint32_t cnt = 0u;
    unsigned long long Pi = 0ull, Qi = 0ull;
#pragma unroll
    for (int i = 0; i < QM; ++i) {
      if (c[i]) {
        cnt += c[i];
        Pi += fx_int(p0[i], p1[i], p2[i], md[i]);
        Qi += fx_int(q0[i], q1[i], q2[i], md[i]);
      }
    }
    for (int o = 1; o < L; o <<= 1) {
      cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
      Pi += __shfl_xor_sync(0xffffffffu, Pi, o);
      Qi += __shfl_xor_sync(0xffffffffu, Qi, o);
    }
    if (sub == 0) {
      const BinPart& own = S.u.part;
      const double ymax = (double)key2f(own.gmax[t]), ymin = (double)key2f(own.gmin[t]);
      const double Ps = (double)Pi * 0x1p-31, Qs = (double)Qi * 0x1p-31;
      const double elo = (double)key2f(edge_key(klo, khi, shift, t));
      const float eup = key2f(edge_key(klo, khi, shift, t + 1));
      const double ehi = (double)eup;
      BinTable<kBins>& T = *tab0;
      T.cnt[t] = cnt;
      T.ymin[t] = cnt ? (float)ymin : 0.0f;
      T.ymax[t] = cnt ? (float)ymax : 0.0f;
      T.eup[t] = eup;
      T.s[t] = exp_call((elo - ehi) * inva);
      if (cnt) {
        const double g = exp_call((ymax - ehi) * inva);
        T.g[t] = g;
        T.h[t] = exp_call((elo - ymax) * inva);
        T.P[t] = Ps;
        T.Pg[t] = Ps * g;
        T.Qr[t] = Qs * exp_call((elo - ymin) * inva);
      } else {
        T.g[t] = 0.0;
        T.h[t] = 0.0;
        T.P[t] = 0.0;
        T.Pg[t] = 0.0;
        T.Qr[t] = 0.0;
      }
    }
  }
}

// Solves row r from its filter partials and band.  cs CTAs of one cluster
// (rank = the CTA's rank in it) or, with cs == 1, one block alone; nparts:
// filter partials of the row.  kRun: a lone CTA solves a band of at most
// kRunCap values as one sorted run instead of binning it (a separate
// instantiation, so that the cluster's bin path keeps its registers).  Every
// thread of every CTA calls it.
template <int NTX, bool kRun>
__device__ void band_solve(const StreamPlan& P, int64_t r, RowCtl* c, unsigned char* smem, int nparts, int cs,
                           int rank) {
  BandShared& S = *reinterpret_cast<BandShared*>(smem);
  double* red = S.red;
  const RowArgs ra = row_args(P, r);
  const double inva = 1.0 / ra.alpha;
  const float c2 = (float)(inva * (double)kLog2e);
  const bool leader = rank == 0;

  // row totals from the filter partials (every CTA, same order)
  const FPart* parts = fpart_of(P, r);
  long long nl = 0;
  double sl = 0.0, sr = 0.0;
  uint32_t bad = 0u;
  for (int i = threadIdx.x; i < nparts; i += NTX) {
    nl += __ldcg(&parts[i].nL);
    sl += __ldcg(&parts[i].SL);
    sr += __ldcg(&parts[i].SR);
    bad |= __ldcg(&parts[i].bad);
  }
  nl = block_sum<NTX, long long>(nl, reinterpret_cast<long long*>(red));
  sl = block_sum<NTX, double>(sl, red);
  sr = block_sum<NTX, double>(sr, red);
  bad = block_or<NTX>(bad, reinterpret_cast<uint32_t*>(red));
  const uint32_t flags = vld(&c->flags);
  const uint32_t mt = vld(&c->band_cnt);
  const long long nr = (P.shard ? P.n_total : P.n) - nl - (long long)mt;
  const int64_t M = min((int64_t)mt, P.band_cap);
  uint32_t st = vld(&c->status) & ROW_WIDENED;
  double b = 0.0, sumf = 0.0;
  int levels = 0;

  if (flags & ROW_TIMEOUT) {
    st |= ROW_TIMEOUT;  // a filter block gave up waiting for its copies
  } else if (bad) {
    st |= ROW_NONFINITE;
  } else if ((flags & ROW_OVERFLOW) || (int64_t)mt > P.band_cap) {
    st |= ROW_OVERFLOW;
  } else if (P.force_fallback) {
    st |= ROW_FORCE_FB;
  } else {
    // this CTA's slice [lo, lo + n) of the band
    const int workers = cs > 1 ? cs - 1 : 1;
    const int w = cs > 1 ? rank - 1 : 0;
    const int64_t lo = (w < 0) ? 0 : M * w / workers;
    const int n = (w < 0) ? 0 : (int)(M * (w + 1) / workers - lo);
    const float* src = band_of(P, r) + lo;
    uint32_t klo = ~vld(&c->band_nkmin), khi = vld(&c->band_kmax);
    if (M == 0) klo = khi = 0u;
    int shift = bin_shift(klo, khi);
    if (leader && threadIdx.x == 0) S.in = SolveIn{vld(&c->aL), vld(&c->aR), nl, nr, sl, sr, ra.k, ra.alpha, inva};
    int action = kBandDone;
    bool run = false;
    if constexpr (kRun) {
      if (cs == 1 && M > 0 && M <= kRunCap) {
        // the whole band as one sorted run; a key range too stretched for
        // the bucket pass leaves it to the bins.  [klo, khi] are the exact
        // extremes of the appended keys.
        uint32_t* keys = reinterpret_cast<uint32_t*>(S.tu.stage);
        uint32_t* tmp = keys + kRunCap;
        double* dA = reinterpret_cast<double*>(tmp + kRunCap);
        double* dL = dA + kRunCap;
        for (int i = threadIdx.x; i < n; i += NTX) keys[i] = f2key(__ldcg(src + i));
        __syncthreads();
        const uint32_t* sorted = block_bucket_sort<NTX>(keys, tmp, n, klo, khi, S.u.tgt.scr);
        if (sorted) {
          solve_run<NTX>(S.in, sorted, n, dA, dL, red, &S.so);
          run = true;
        }
      }
    }
    for (int level = 0; level < kMaxLevels && !run; ++level) {
      levels = level + 1;
      // a worker keeps its slice in shared memory; a lone CTA (cs == 1) holds
      // the table in the same place, so it rereads its slice from L2 past level 0
      const bool staged = level == 0 || cs > 1;
      bin_count<NTX>(src, n, level == 0, staged, S.tu.stage, klo, khi, shift, S.u.part);
      cl_sync(cs);
      merge_extremes<NTX>(S, cs, rank);
      cl_sync(cs);
      bin_sums<NTX>(src, n, staged, S.tu.stage, klo, khi, shift, c2, S.u.part);
      cl_sync(cs);
      merge_bins<NTX>(S, cs, rank, klo, khi, shift, inva);
      cl_sync(cs);
      if (leader) {
        solve_bins<NTX, kBins>(S.in, S.tu.tab, (double)key2f(klo), (double)key2f(khi), red, &S.pk);
        if (threadIdx.x == 0) {
          const GroupPick& pk = S.pk;
          BandDecision d{kBandDone, pk.tg, shift, level, klo, khi, 0u};
          S.so.status = pk.status;
          S.so.M = pk.M;
          S.so.S_aL = pk.S_aL;
          S.so.S_aR = pk.S_aR;
          S.so.b = 0.0;
          S.so.sumf = 0.0;
          if (pk.status != ROW_CERTIFIED) {
          } else if (pk.tg < 0) {
            solve_tail_interval(S.in, pk, &S.so);
          } else {
            const uint32_t gcnt = S.tu.tab.cnt[pk.tg];
            const float gmin = S.tu.tab.ymin[pk.tg], gmax = S.tu.tab.ymax[pk.tg];
            const uint32_t gk0 = f2key(gmin), gk1 = f2key(gmax);
            if (gk0 == gk1) {
              // every value of the bin equals y: the root lies in [inc_x, y]
              const double y = (double)gmax;
              const double Bp = (double)gcnt + pk.out_s * link(y, pk.out_x, S.in.inva);
              S.so.b = closed_form_root(pk.inc_x, y, pk.inc_s, Bp, (double)((long long)gcnt + pk.g_after), S.in.k,
                                        S.in.alpha);
              S.so.sumf = sum_f_at(pk.inc_x, y, pk.inc_s, Bp, S.so.b, S.in.inva);
            } else if (gcnt <= (uint32_t)kTargetCap) {
              d.action = kBandExtract;
            } else if (level + 1 < kMaxLevels) {
              d.action = kBandRefine;
              d.klo = gk0;
              d.khi = gk1;
              d.shift = bin_shift(gk0, gk1);
              // everything outside the bin becomes the two tails of the next level
              S.in.aL = (float)pk.inc_x;
              S.in.SL = pk.inc_s;
              S.in.aR = (float)pk.out_x;
              S.in.SR = pk.out_s;
              S.in.nR = pk.g_after;
            } else {
              S.so.status = ROW_FORCE_FB;
            }
          }
          S.dec = d;
        }
      }
      cl_sync(cs);
      const BandDecision d = *at_rank(&S.dec, 0, cs);
      action = d.action;
      if (action != kBandRefine) break;
      klo = d.klo;
      khi = d.khi;
      shift = d.shift;
    }
    if (action == kBandExtract) {
      // gather the target bin into the leader's buffer, one atomic per warp
      const BandDecision d = *at_rank(&S.dec, 0, cs);
      uint32_t* cnt0 = &at_rank(&S.dec, 0, cs)->count;
      uint32_t* keys0 = at_rank(S.u.tgt.keys, 0, cs);
      const int lane = threadIdx.x & 31;
      for (int j0 = 0; j0 < n; j0 += NTX) {
        const int j = j0 + (int)threadIdx.x;
        uint32_t key = 0u;
        bool hit = false;
        if (j < n) {
          key = f2key(slice_val(src, S.tu.stage, cs > 1, j));
          hit = key >= d.klo && key <= d.khi && (int)((key - d.klo) >> d.shift) == d.tg;
        }
        const uint32_t m = __ballot_sync(0xffffffffu, hit);
        if (m) {
          uint32_t pos = 0u;
          if (lane == 0) pos = atomicAdd(cnt0, (uint32_t)__popc(m));
          pos = __shfl_sync(0xffffffffu, pos, 0) + (uint32_t)__popc(m & ((1u << lane) - 1u));
          if (hit && pos < (uint32_t)kTargetCap) keys0[pos] = key;
        }
      }
      cl_sync(cs);
      if (leader) {
        // the bin's values, sorted, each one entry of a bin table: the same
        // group solve then picks the interval between two values that holds
        // the root, and the closed form finishes
        const int cnt = (int)min(S.dec.count, (uint32_t)kTargetCap);
        BinTable<kBins>& T = S.tu.tab;
        // one bucket pass over the bin's key range (its extremes from the
        // merge); a bin stretched by outliers takes the bitonic network
        const uint32_t bk0 = f2key(T.ymin[S.pk.tg]), bk1 = f2key(T.ymax[S.pk.tg]);
        const uint32_t* keys = block_bucket_sort<NTX>(S.u.tgt.keys, S.u.tgt.sorted, cnt, bk0, bk1, S.u.tgt.scr);
        if (!keys) {
          block_bitonic_sort<NTX>(S.u.tgt.keys, cnt);
          keys = S.u.tgt.keys;
        }
        const float ylast = key2f(keys[cnt - 1]);
        for (int i = threadIdx.x; i < kBins; i += NTX) {
          if (i < cnt) {
            const float y = key2f(keys[i]);
            const float yn = (i + 1 < cnt) ? key2f(keys[i + 1]) : y;
            const double sv = exp_call(((double)y - (double)yn) * inva);
            T.cnt[i] = 1u;
            T.ymin[i] = y;
            T.ymax[i] = y;
            T.eup[i] = yn;
            T.s[i] = sv;
            T.g[i] = sv;
            T.h[i] = 1.0;
            T.P[i] = 1.0;
            T.Pg[i] = sv;
            T.Qr[i] = 1.0;
          } else {
            T.cnt[i] = 0u;
            T.ymin[i] = ylast;
            T.ymax[i] = ylast;
            T.eup[i] = ylast;
            T.s[i] = 1.0;
            T.g[i] = 0.0;
            T.h[i] = 0.0;
            T.P[i] = 0.0;
            T.Pg[i] = 0.0;
            T.Qr[i] = 0.0;
          }
        }
        __syncthreads();
        const GroupPick& pk = S.pk;
        const SolveIn vin{(float)pk.inc_x, (float)pk.out_x, 0, pk.g_after, pk.inc_s, pk.out_s,
                          S.in.k, S.in.alpha, S.in.inva};
        solve_bins<NTX, kBins>(vin, T, (double)key2f(keys[0]), (double)ylast, red, &S.pk2);
        if (threadIdx.x == 0) {
          const GroupPick& q = S.pk2;
          if (q.status != ROW_CERTIFIED || q.tg < 0) {
            S.so.status = ROW_FORCE_FB;  // the two levels disagree at rounding level: full sort
          } else {
            const double y = (double)T.ymax[q.tg];
            const double Bp = 1.0 + q.out_s * link(y, q.out_x, inva);
            S.so.b = closed_form_root(q.inc_x, y, q.inc_s, Bp, (double)(1 + q.g_after), S.in.k, S.in.alpha);
            S.so.sumf = sum_f_at(q.inc_x, y, q.inc_s, Bp, S.so.b, inva);
            S.so.status = ROW_CERTIFIED;
          }
        }
      }
    }
    if (leader) {
      __syncthreads();
      st |= S.so.status;
      b = S.so.b;
      sumf = S.so.sumf;
    }
  }
  if (leader && threadIdx.x == 0) {
    c->sumf = sumf;
    c->nL = nl;
    c->nR = nr;
    c->M = (long long)mt;
    c->SL = sl;
    c->SR = sr;
    c->b = b;
    c->bins = kBins * levels;
    // test knob: odd rows go to the recovery kernel, whose barrier runs out
    if (P.force_timeout && !P.shard && (r & 1) && !(st & (ROW_NONFINITE | ROW_TIMEOUT))) st |= ROW_FORCE_TO;
    c->status = st;
    __threadfence();
  }
  cl_sync(cs);  // no CTA leaves while another may still read its shared memory
}

template <bool kRun>
__global__ void __launch_bounds__(kBandThreads, 1) k_band(const StreamPlan P) {
  extern __shared__ __align__(16) unsigned char smem[];
  wait_prior_grid();
  const int64_t r = blockIdx.y;
  const int cs = (int)cg::this_cluster().num_blocks();
  const int rank = (int)cg::this_cluster().block_rank();
  band_solve<kBandThreads, kRun>(P, r, ctl_of(P, r), smem, P.Gf, cs, rank);
}
// a lone band CTA may solve its band as one run; a cluster bins it
using BandKernel = void (*)(const StreamPlan);
BandKernel band_kernel(int cs) { return cs == 1 ? k_band<true> : k_band<false>; }

// ===========================================================================
// recovery: one widening, then the full-sort fallback (cooperative launch)
// ===========================================================================

// filter_phase in the recovery kernel uses the sort buffers kbuf, tbuf and
// dscr (contiguous, 16 C bytes) as its stage
static_assert(kFilterStageBytes <= (size_t)16 * kBucketMax, "the recovery kernel's filter stage does not fit");
struct RecSmem {
  static constexpr size_t kSort = BandSmem::bytes(kBucketMax);
  static constexpr size_t kTotal = kSort > kBandSmemBytes ? kSort : kBandSmemBytes;
};

// exclusive prefix over `cnt` entries of a global array, in place; returns the total
__device__ uint32_t block_scan_global_u32(uint32_t* a, int cnt, uint32_t* scr) {
  const int q = (cnt + NT - 1) / NT;
  const int i0 = min(cnt, (int)threadIdx.x * q), i1 = min(cnt, i0 + q);
  uint32_t loc = 0;
  for (int i = i0; i < i1; ++i) loc += __ldcg(a + i);
  uint32_t tot;
  uint32_t run = block_excl_prefix_u32<NT>(loc, scr, &tot);
  for (int i = i0; i < i1; ++i) {
    const uint32_t v = __ldcg(a + i);
    a[i] = run;
    run += v;
  }
  __syncthreads();
  return tot;
}

__global__ void __launch_bounds__(NT) k_recover(const StreamPlan P, const float* __restrict__ scores,
                                                 float* __restrict__ p_out) {
  extern __shared__ __align__(16) unsigned char smem[];
  const BandSmem sm(smem, kBucketMax);
  uint32_t* kbuf = sm.kbuf;
  uint32_t* tbuf = sm.tbuf;
  uint32_t* hist = sm.hist;
  double* red = sm.red;
  double* dscr = sm.dscr;
  uint32_t* sh = kbuf;  // selection histograms (4096 words)
  uint32_t* scr = reinterpret_cast<uint32_t*>(red);
  __shared__ SolveOut so;
  __shared__ int s_skip;

  const int cta = blockIdx.x, ncta = gridDim.x;
  RowCtl* c0 = ctl_of(P, 0);
  const uint32_t limit = spin_limit_of(P.spin_limit);
  uint32_t bar_n = (uint32_t)ncta;  // arrivals each barrier waits for
  // A barrier that gives up ends the kernel: the row being recovered and every
  // later row that needs recovery are marked as timed out (NaN outputs).
#define REC_BARRIER()                                                          \
  do {                                                                         \
    if (!grid_barrier(&c0->bar_count, &c0->bar_gen, bar_n, &c0->timeout, limit)) { \
      if (threadIdx.x == 0) {                                                  \
        atomicOr(&c->status, ROW_TIMEOUT);                                     \
        for (int64_t rr = r + 1; rr < P.rows; ++rr) {                          \
          RowCtl* cr = ctl_of(P, rr);                                          \
          const uint32_t sr = vld(&cr->status);                                \
          if ((sr & ROW_NEEDS_RECOVERY) && !(sr & ROW_NONFINITE)) atomicOr(&cr->status, ROW_TIMEOUT); \
        }                                                                      \
        __threadfence();                                                       \
      }                                                                        \
      return;                                                                  \
    }                                                                          \
  } while (0)

  for (int64_t r = 0; r < P.rows; ++r) {
    RowCtl* c = ctl_of(P, r);
    const uint32_t st0 = vld(&c->status);
    if (!(st0 & ROW_NEEDS_RECOVERY) || (st0 & ROW_NONFINITE)) continue;
    // test knob: wait for one block more than the grid holds, so that the
    // barrier runs out (every block gives up after `limit` polls)
    bar_n = (uint32_t)ncta + ((st0 & ROW_FORCE_TO) ? 1u : 0u);
    const RowArgs ra = row_args(P, r);
    const double inva = 1.0 / ra.alpha;
    const int widen_delta = row_ranks(P, ra.k).widen_delta;
    bool fallback = (st0 & (ROW_OVERFLOW | ROW_FORCE_FB)) != 0u || P.max_widen <= 0;

    if (!fallback) {
      // ---- widen once: the missed side moves out by widen_delta sample
      // ranks, the other edge moves to the old edge (known to lie on the
      // correct side of b) ----
      const bool left = (st0 & ROW_MISS_LEFT) != 0u;
      int rlo = vld(&c->rank_lo), rhi = vld(&c->rank_hi);
      bool vlo = vld(&c->valid_lo) != 0u, vhi = vld(&c->valid_hi) != 0u;
      if (left) {
        rhi = rlo; vhi = true;
        rlo -= widen_delta; vlo = rlo >= 0;
        if (!vlo) rlo = 0;
      } else {
        rlo = rhi; vlo = true;
        rhi += widen_delta; vhi = rhi <= P.m - 1;
        if (!vhi) rhi = P.m - 1;
      }
      for (int i = cta * NT + threadIdx.x; i < 2048; i += ncta * NT) { h1_of(P, r)[i] = 0u; h3_of(P, r)[i] = 0u; }
      for (int i = cta * NT + threadIdx.x; i < 4096; i += ncta * NT) h2_of(P, r)[i] = 0u;
      REC_BARRIER();
      sel_hist1(samp_of(P, r), P.m, cta, ncta, h1_of(P, r), sh);
      REC_BARRIER();
      if (cta == 0) {
        const uint32_t rk[2] = {(uint32_t)rlo, (uint32_t)rhi};
        int bin[2];
        uint32_t rem[2];
        sel_pick<2048>(h1_of(P, r), false, rk, scr, bin, rem);
        store_pick(c, 0, bin, rem);
      }
      REC_BARRIER();
      {
        const int b1[2] = {vld(&c->sel_bin[0][0]), vld(&c->sel_bin[0][1])};
        sel_hist2(samp_of(P, r), P.m, cta, ncta, b1, h2_of(P, r), sh);
      }
      REC_BARRIER();
      if (cta == 0) {
        const uint32_t rk[2] = {vld(&c->sel_rem[0][0]), vld(&c->sel_rem[0][1])};
        int bin[2];
        uint32_t rem[2];
        sel_pick<2048>(h2_of(P, r), true, rk, scr, bin, rem);
        store_pick(c, 1, bin, rem);
      }
      REC_BARRIER();
      const uint32_t pre[2] = {level3_prefix(c, 0), level3_prefix(c, 1)};
      sel_hist3(samp_of(P, r), P.m, cta, ncta, pre, h3_of(P, r), sh);
      REC_BARRIER();
      if (cta == 0) {
        const uint32_t rk[2] = {vld(&c->sel_rem[1][0]), vld(&c->sel_rem[1][1])};
        int bin[2];
        uint32_t rem[2];
        sel_pick<1024>(h3_of(P, r), true, rk, scr, bin, rem);
        if (threadIdx.x == 0) {
          const uint32_t keys[2] = {(pre[0] << 10) | (uint32_t)bin[0], (pre[1] << 10) | (uint32_t)bin[1]};
          write_plan(c, P.m, keys, rlo, rhi, vlo, vhi);
          c->flags = 0u;
          c->band_cnt = 0u;
          c->band_kmax = 0u;
          c->band_nkmin = 0u;
          c->status = ROW_WIDENED;
          __threadfence();
        }
      }
      REC_BARRIER();
      filter_phase(P, r, scores + r * P.stride, c, cta, ncta, red, reinterpret_cast<float*>(kbuf));
      REC_BARRIER();
      if (cta == 0) {
        band_solve<NT, false>(P, r, c, smem, ncta, 1, 0);
        if (threadIdx.x == 0) {
          c->status |= ROW_WIDENED;
          __threadfence();
        }
      }
      REC_BARRIER();
      const uint32_t st1 = vld(&c->status);
      if (st1 & (ROW_CERTIFIED | ROW_NONFINITE)) continue;
    }

    // ---- full-sort fallback: LSD radix sort of the whole row, then the
    // solver of section 2.2 with no bracket ----
    {
      const int64_t n = P.n;
      const float* src = scores + r * P.stride;
      uint32_t* A = P.fb_keys;
      uint32_t* B = p_out ? reinterpret_cast<uint32_t*>(p_out + r * P.stride) : P.fb_keys2;
      uint32_t* cnts = P.rcount;                          // [256][ncta]
      uint32_t* tots = P.rcount + 256 * (size_t)ncta;     // [256]
      const int64_t L = (n + ncta - 1) / ncta;
      const int64_t lo_i = min(n, (int64_t)cta * L), hi_i = min(n, lo_i + L);
      uint32_t* cur = nullptr;  // pass 0 reads the scores themselves
      uint32_t* sbuf = kbuf;
      uint32_t* stmp = kbuf + kTile;
      uint32_t* off = tbuf;
      uint32_t* dig = tbuf + 256;
      uint32_t* hh = tbuf + 512;
      const uint32_t* dcount = hist + NW * 256 + 64;
      const uint32_t* dstart = dcount + 256;
      for (int pass = 0; pass < 4; ++pass) {
        const int shift = 8 * pass;
        for (int i = threadIdx.x; i < 256; i += NT) hh[i] = 0u;
        __syncthreads();
        // kLd keys a thread, their loads issued before any is used (one
        // block per SM: the loop would otherwise wait on every load)
        constexpr int kLd = 8;
        for (int64_t i0 = lo_i; i0 < hi_i; i0 += kLd * NT) {
          uint32_t kk[kLd];
#pragma unroll
          for (int u = 0; u < kLd; ++u) {
            const int64_t i = i0 + u * NT + threadIdx.x;
            kk[u] = i < hi_i ? (cur ? __ldcg(cur + i) : f2key(__ldg(src + i))) : 0u;
          }
#pragma unroll
          for (int u = 0; u < kLd; ++u) hist_add(hh, (kk[u] >> shift) & 255u, i0 + u * NT + threadIdx.x < hi_i);
        }
        __syncthreads();
        for (int d = threadIdx.x; d < 256; d += NT) cnts[(size_t)d * ncta + cta] = hh[d];
        REC_BARRIER();
        for (int d = cta; d < 256; d += ncta) {
          const uint32_t tot = block_scan_global_u32(cnts + (size_t)d * ncta, ncta, scr);
          if (threadIdx.x == 0) tots[d] = tot;
        }
        REC_BARRIER();
        if (threadIdx.x == 0) s_skip = 0;
        __syncthreads();
        uint32_t tv = 0u;
        if (threadIdx.x < 256) {
          tv = __ldcg(tots + threadIdx.x);
          if ((int64_t)tv == n) s_skip = 1;
        }
        const uint32_t base_d = block_excl_prefix_u32<NT>(tv, scr, nullptr);
        if (pass > 0 && s_skip) continue;  // every key shares this digit
        uint32_t* dst = (cur == A) ? B : A;
        if (threadIdx.x < 256) {
          dig[threadIdx.x] = base_d;
          off[threadIdx.x] = base_d + __ldcg(cnts + (size_t)threadIdx.x * ncta + cta);
        }
        __syncthreads();
        for (int64_t t0 = lo_i; t0 < hi_i; t0 += kTile) {
          const int tn = (int)min((int64_t)kTile, hi_i - t0);
          for (int i0 = 0; i0 < tn; i0 += kLd * NT) {
            uint32_t kk[kLd];
#pragma unroll
            for (int u = 0; u < kLd; ++u) {
              const int i = i0 + u * NT + (int)threadIdx.x;
              kk[u] = i < tn ? (cur ? __ldcg(cur + t0 + i) : f2key(__ldg(src + t0 + i))) : 0u;
            }
#pragma unroll
            for (int u = 0; u < kLd; ++u) {
              const int i = i0 + u * NT + (int)threadIdx.x;
              if (i < tn) sbuf[i] = kk[u];
            }
          }
          __syncthreads();
          radix_pass<NT>(sbuf, stmp, tn, hist, shift, false);
          for (int q = threadIdx.x; q < tn; q += NT) {
            const uint32_t k = stmp[q];
            const uint32_t d = (k >> shift) & 255u;
            dst[off[d] + (q - dstart[d])] = k;
          }
          __syncthreads();
          if (threadIdx.x < 256) off[threadIdx.x] += dcount[threadIdx.x];
          __syncthreads();
        }
        cur = dst;
        REC_BARRIER();
      }
      const int ng = (int)((n + kFallbackGroup - 1) / kFallbackGroup);
      GroupAgg* fa = reinterpret_cast<GroupAgg*>(P.fb_aggs);
      for (int g = cta; g < ng; g += ncta)
        aggregate_sorted_keys<NT, true>(cur + (int64_t)g * kFallbackGroup,
                                        (int)min((int64_t)kFallbackGroup, n - (int64_t)g * kFallbackGroup), red,
                                        fa + g, inva);
      REC_BARRIER();
      if (cta == 0) {
        const SolveIn in{-CUDART_INF_F, CUDART_INF_F, 0, 0, 0.0, 0.0, ra.k, ra.alpha, inva};
        solve_band<NT, true>(in, fa, ng, KeyGroupsG{cur, kFallbackGroup}, dscr, red, &so);
        if (threadIdx.x == 0) {
          const uint32_t keep = (vld(&c->status) | st0) & (ROW_WIDENED | ROW_OVERFLOW);
          c->b = so.b;
          c->sumf = so.sumf;
          c->status = keep | ROW_FALLBACK | ROW_CERTIFIED;
          c->aL = -CUDART_INF_F;
          c->aR = CUDART_INF_F;
          c->nL = 0;
          c->nR = 0;
          c->M = n;
          c->SL = 0.0;
          c->SR = 0.0;
          c->bins = ng;
          __threadfence();
        }
      }
      REC_BARRIER();
    }
  }
#undef REC_BARRIER
}

// ===========================================================================
// memberships (section 2.1) and the backward pass
// ===========================================================================

// p = F((x - b)/alpha), with x - b formed from b = bh + bl (two fp32 words);
// also returns h = exp(-|x - b|/alpha)/2 and |x - b|
__device__ __forceinline__ float memb_h(float x, float bh, float bl, float c2, float& h, float& ad) {
  const float d = (x - bh) - bl;
  ad = fabsf(d);
  h = 0.5f * exp2f(-ad * c2);
  return d < 0.0f ? h : 1.0f - h;
}
// A block whose nearest |x - b| is above this many alpha_p / ln 2 has every
// fp32 term exp(-|x - b|/alpha_p) below 2^-64: it counts its sum f again,
// relative to its nearest score (near_add), instead of from the fp32 terms.
constexpr float kDfDeepLog2 = 64.0f;

// Sparse mode: each warp stages its entries with p >= eps in its own slice of
// shared memory (ballots place them, no atomics) and, once it holds
// kSpFlush of them, reserves room in the row's output with one global atomic
// and copies them out; no block-wide barrier is involved.  The order of the
// entries is unspecified.
constexpr int kSpFlush = 128;
constexpr int kSpWarpStage = kSpFlush + 32 * 4;  // a step adds at most 4 per lane

// kDf: the DFTopK relaxation; sum f is also taken here, at alpha_p, from the
// fp32 terms of the memberships, or (blocks far from b) relative to the
// block's nearest score.  Per block MPart holds (sum p, S, d): the block's
// sum of exp(-|x - b|/alpha_p) is exp(-d/alpha_p) S.
template <bool kSparse, bool kDf>
__global__ void __launch_bounds__(NT) k_memb(const StreamPlan P, const float* __restrict__ scores,
                                              float* __restrict__ p_out, double* b_out, double* sumf_out,
                                              uint32_t* status_out, lapsum_row_stats* stats) {
  __shared__ double red[64];
  __shared__ int32_t s_idx[kSparse ? NW * kSpWarpStage : 1];
  __shared__ float s_val[kSparse ? NW * kSpWarpStage : 1];
  wait_prior_grid();
  const int64_t r = blockIdx.y;
  RowCtl* c = ctl_of(P, r);
  const double b = c->b;
  const RowArgs ra = row_args(P, r);
  uint32_t status = c->status | (ra.bad ? ROW_BADARG : 0u);
  if (status & ROW_TIMEOUT) status &= ~ROW_CERTIFIED;
  const bool nonfinite = (status & ROW_NAN_OUT) != 0u;
  const double inva = 1.0 / ra.alpha_p;
  const float c2 = (float)(inva * (double)kLog2e);
  const float bh = __double2float_rn(b);
  const float bl = __double2float_rn(b - (double)bh);
  const float* row = scores + r * P.stride;
  float* dst = kSparse ? nullptr : p_out + r * P.stride;
  double hs = 0.0;             // kDf: sum of h = exp(-|x - b|/alpha_p)/2
  float amin = CUDART_INF_F;   // kDf: nearest |x - b| of this thread
  const int64_t n = P.n;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const uint32_t lt_mask = (1u << lane) - 1u;
  int32_t* widx = s_idx + (kSparse ? warp * kSpWarpStage : 0);
  float* wval = s_val + (kSparse ? warp * kSpWarpStage : 0);
  uint32_t wn = 0u;  // entries in this warp's stage (the same in every lane)
  double ps = 0.0;
  // sparse: stage this lane's hits (bit j of `hits`: index i0 + j, value pv[j])
  auto append = [&](uint32_t hits, int64_t i0, const float* pv, int cnt) {
    for (int j = 0; j < cnt; ++j) {
      const uint32_t m = __ballot_sync(0xffffffffu, (hits >> j) & 1u);
      if ((hits >> j) & 1u) {
        const uint32_t pos = wn + (uint32_t)__popc(m & lt_mask);
        widx[pos] = (int32_t)(i0 + j);
        wval[pos] = pv[j];
      }
      wn += (uint32_t)__popc(m);
    }
  };
  auto flush = [&](bool force) {
    if (wn >= (uint32_t)kSpFlush || (force && wn > 0u)) {
      __syncwarp();
      unsigned long long gb = 0ull;
      if (lane == 0) gb = atomicAdd(reinterpret_cast<unsigned long long*>(P.sp.count + r), (unsigned long long)wn);
      gb = __shfl_sync(0xffffffffu, gb, 0);
      int32_t* oi = P.sp.idx + r * P.sp.cap;
      float* ov = P.sp.val + r * P.sp.cap;
      for (uint32_t j = lane; j < wn; j += 32) {
        if (gb + j < (unsigned long long)P.sp.cap) {
          oi[gb + j] = widx[j];
          ov[gb + j] = wval[j];
        }
      }
      __syncwarp();
      wn = 0u;
    }
  };
  auto one = [&](int64_t i, bool act) {  // the scalar loops: every thread of the block calls it
    float p = 0.0f;
    if (act) {
      float h, ad;
      p = memb_h(row[i], bh, bl, c2, h, ad);
      if (nonfinite) p = CUDART_NAN_F;
      ps += (double)p;
      if (kDf) {
        hs += (double)h;
        amin = fminf(amin, ad);
      }
      if (!kSparse) dst[i] = p;
    }
    if (kSparse) {
      append((act && p >= P.sp.eps) ? 1u : 0u, i, &p, 1);
      flush(false);
    }
  };
  // the body as float4 after a head of 0-3 scores (p starts at the scores'
  // address mod 16 when vec; the sparse form writes no p)
  const bool vec = kSparse || P.vec;
  const int head = vec ? row_head(row, n) : 0;
  const int64_t nb4 = vec ? ((n - head) >> 2) / CHUNK4 * CHUNK4 : 0;
  {
    const float4* x4 = reinterpret_cast<const float4*>(row + head);
    float4* d4 = reinterpret_cast<float4*>(kSparse ? nullptr : dst + head);
    const int64_t nchunks = nb4 / CHUNK4;
    for (int64_t q = blockIdx.x; q < nchunks; q += gridDim.x) {
      const int64_t qq = nchunks - 1 - q;  // reverse of the filter pass
      const int64_t base = qq * CHUNK4 + threadIdx.x;
      float4 v[U];
#pragma unroll
      for (int u = 0; u < U; ++u) v[u] = __ldg(x4 + base + u * NT);
      float pl = 0.0f, hl = 0.0f;
#pragma unroll
      for (int u = 0; u < U; ++u) {
        float4 p;
        float h0, h1, h2, h3, a0, a1, a2, a3;
        p.x = memb_h(v[u].x, bh, bl, c2, h0, a0);
        p.y = memb_h(v[u].y, bh, bl, c2, h1, a1);
        p.z = memb_h(v[u].z, bh, bl, c2, h2, a2);
        p.w = memb_h(v[u].w, bh, bl, c2, h3, a3);
        if (nonfinite) p = make_float4(CUDART_NAN_F, CUDART_NAN_F, CUDART_NAN_F, CUDART_NAN_F);
        pl += (p.x + p.y) + (p.z + p.w);
        if (kDf) {
          hl += (h0 + h1) + (h2 + h3);
          amin = fminf(amin, fminf(fminf(a0, a1), fminf(a2, a3)));
        }
        if (kSparse) {
          const float pv[4] = {p.x, p.y, p.z, p.w};
          uint32_t hits = 0u;
#pragma unroll
          for (int j = 0; j < 4; ++j) hits |= (pv[j] >= P.sp.eps) ? (1u << j) : 0u;
          append(hits, head + (base + u * NT) * 4, pv, 4);
          flush(false);
        } else {
          stg_stream(d4 + base + u * NT, p);
        }
      }
      ps += (double)pl;
      if (kDf) hs += (double)hl;
    }
  }
  const int64_t nrest = n - 4 * nb4;  // [0, head) and the tail; every score when !vec
  for (int64_t j0 = (int64_t)blockIdx.x * NT; j0 < nrest; j0 += (int64_t)gridDim.x * NT) {
    const int64_t j = j0 + threadIdx.x;
    one(rest_index(j < nrest ? j : 0, head, nb4), j < nrest);
  }
  if (kSparse) flush(true);
  ps = block_sum<NT, double>(ps, red);
  double dmin = 0.0;
  if (kDf) {
    const float M = block_min_float<NT>(amin, reinterpret_cast<float*>(red));
    if (M * c2 > kDfDeepLog2) {
      // every fp32 term of this block is tiny: count again relative to its
      // nearest score (its values are read a second time)
      float mh = CUDART_INF_F, ml = 0.0f;
      double S = 0.0;
      {
        const float4* x4 = reinterpret_cast<const float4*>(row + head);
        const int64_t nchunks = nb4 / CHUNK4;
        for (int64_t q = blockIdx.x; q < nchunks; q += gridDim.x) {
          const int64_t base = (nchunks - 1 - q) * CHUNK4 + threadIdx.x;
#pragma unroll
          for (int u = 0; u < U; ++u) {
            const float4 v = __ldg(x4 + base + u * NT);
            near_add(v.x, bh, bl, c2, mh, ml, S);
            near_add(v.y, bh, bl, c2, mh, ml, S);
            near_add(v.z, bh, bl, c2, mh, ml, S);
            near_add(v.w, bh, bl, c2, mh, ml, S);
          }
        }
      }
      for (int64_t j = (int64_t)blockIdx.x * NT + threadIdx.x; j < nrest; j += (int64_t)gridDim.x * NT)
        near_add(row[rest_index(j, head, nb4)], bh, bl, c2, mh, ml, S);
      dmin = near_dist(mh, ml);
      block_near_reduce<NT>(dmin, S, inva, red);
      hs = S;
    } else {
      hs = 2.0 * block_sum<NT, double>(hs, red);  // anchored at distance 0
    }
  }
  if (threadIdx.x == 0) mpart_of(P, r)[blockIdx.x] = MPart{ps, hs, dmin, 0.0};
  if (last_block_done(&c->done_memb, gridDim.x)) {
    const MPart* mp = mpart_of(P, r);
    double p = 0.0, h = 0.0, hm = CUDART_INF;
    for (int i = threadIdx.x; i < (int)gridDim.x; i += NT) p += __ldcg(&mp[i].a);
    p = block_sum<NT, double>(p, red);
    if (kDf) {
      for (int i = threadIdx.x; i < (int)gridDim.x; i += NT) hm = fmin(hm, __ldcg(&mp[i].c));
      hm = block_min_double<NT>(hm, red);
      for (int i = threadIdx.x; i < (int)gridDim.x; i += NT) {
        const double di = __ldcg(&mp[i].c);
        if (di < CUDART_INF) h += __ldcg(&mp[i].b) * exp_call((hm - di) * inva);
      }
      h = block_sum<NT, double>(h, red);
    }
    if (threadIdx.x == 0) {
      if (kDf) c->sumf = (hm < CUDART_INF) ? 0.5 * inva * exp_call(-hm * inva) * h : 0.0;
      if (kSparse && *reinterpret_cast<volatile unsigned long long*>(P.sp.count + r) > (unsigned long long)P.sp.cap)
        status |= ROW_TRUNCATED;
      const double bo = nonfinite ? CUDART_NAN : b;
      const double so = nonfinite ? CUDART_NAN : c->sumf;
      const uint32_t pub = status & ROW_PUBLIC;
      b_out[r] = bo;
      if (sumf_out) sumf_out[r] = so;
      if (P.sump_out) P.sump_out[r] = nonfinite ? CUDART_NAN : p;
      if (status_out) status_out[r] = pub;
      c->sump = p;
      if (stats) {
        lapsum_row_stats* s = stats + r;
        s->a_L = c->aL;
        s->a_R = c->aR;
        s->n_L = c->nL;
        s->n_R = c->nR;
        s->band = c->M;
        s->S_L = c->SL;
        s->S_R = c->SR;
        s->b = bo;
        s->sum_p = p;
        s->sum_f = so;
        s->sample_m = P.m;
        s->buckets = c->bins;
        s->status = pub;
        s->reserved = 0;
      }
    }
  }
}

struct BPart {
  double m, S, SG, SZ, SGZ, pad;
};

// lambda (and dL/dalpha) of row r from `world` groups of reduction partials
// (group w at parts + w * wstride; per partials in each, or the count a
// sharded GPU left in slot 0 when per < 0), in a fixed order.  All threads of
// one block call it.
template <bool kAlpha>
__device__ void combine_parts(const StreamBwd& a, int64_t r, const BPart* parts, int64_t wstride, int world, int per,
                              bool bad, double inva, double* red) {
  auto count = [&](int w) {
    return per >= 0 ? per : (int)__ldcg(&parts[w * wstride].pad);
  };
  float mloc = CUDART_INF_F;
  for (int w = 0; w < world; ++w) {
    const BPart* pw = parts + w * wstride;
    const int c = count(w);
    for (int i = threadIdx.x; i < c; i += NT) mloc = fminf(mloc, (float)__ldcg(&pw[i].m));
  }
  const double M = (double)block_min_float<NT>(mloc, reinterpret_cast<float*>(red));
  double s = 0.0, sg = 0.0, sz = 0.0, sgz = 0.0;
  for (int w = 0; w < world; ++w) {
    const BPart* pw = parts + w * wstride;
    const int c = count(w);
    for (int i = threadIdx.x; i < c; i += NT) {
      const double pm = __ldcg(&pw[i].m);
      const double sc = (pm == CUDART_INF) ? 0.0 : exp2(M - pm);
      s += __ldcg(&pw[i].S) * sc;
      sg += __ldcg(&pw[i].SG) * sc;
      if (kAlpha) {
        sz += __ldcg(&pw[i].SZ) * sc;
        sgz += __ldcg(&pw[i].SGZ) * sc;
      }
    }
  }
  s = block_sum<NT, double>(s, red);
  sg = block_sum<NT, double>(sg, red);
  if (kAlpha) {
    sz = block_sum<NT, double>(sz, red);
    sgz = block_sum<NT, double>(sgz, red);
  }
  if (threadIdx.x == 0) {
    const double lam = bad ? CUDART_NAN : sg / s;  // NaN also reaches every grad of the row
    a.lam[r] = lam;
    if (a.grad_k) a.grad_k[r] = lam;
    if (kAlpha) a.grad_alpha[r] = bad ? CUDART_NAN : alpha_grad(M, sz, sgz, lam, inva);
  }
}

// lambda = sum g f / sum f by the rescaled reduction of common.cuh; with
// kAlpha also sum f z and sum g f z (z = r - b) for dL/dalpha
template <bool kAlpha>
__global__ void __launch_bounds__(NT) k_bwd_reduce(const StreamBwd a) {
  __shared__ double red[64];
  const int64_t r = blockIdx.y;
  const double b = a.b[r];
  bool bad = false;
  const double inva = 1.0 / row_alpha(a.alpha, a.alpha_rows, r, &bad);
  const float c2 = (float)(inva * (double)kLog2e);
  const float bh = __double2float_rn(b);
  const float bl = __double2float_rn(b - (double)bh);
  const float* x = a.scores + r * a.stride;
  const float* g = a.grad_p + r * a.stride;
  const int64_t n = a.n;
  float m = CUDART_INF_F;
  double S = 0.0, SG = 0.0, SZ = 0.0, SGZ = 0.0;
  auto acc = [&](float xv, float gv, float& ps, float& psg, float& psz, float& psgz) {
    const float z = (xv - bh) - bl;
    if (kAlpha) shift_add_z(fabsf(z) * c2, gv, z, m, ps, psg, psz, psgz, S, SG, SZ, SGZ);
    else shift_add(fabsf(z) * c2, gv, m, ps, psg, S, SG);
  };
  // x and g start at the same address mod 16 when vec: a head of 0-3
  // scores, the body as float4, then the tail
  const int head = a.vec ? row_head(x, n) : 0;
  const int64_t nb4 = a.vec ? ((n - head) >> 2) / CHUNK4 * CHUNK4 : 0;
  {
    const float4* x4 = reinterpret_cast<const float4*>(x + head);
    const float4* g4 = reinterpret_cast<const float4*>(g + head);
    const int64_t nchunks = nb4 / CHUNK4;
    for (int64_t q = blockIdx.x; q < nchunks; q += gridDim.x) {
      const int64_t base = q * CHUNK4 + threadIdx.x;
      float4 xv[U], gv[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        xv[u] = __ldg(x4 + base + u * NT);
        gv[u] = __ldg(g4 + base + u * NT);
      }
      float ps = 0.0f, psg = 0.0f, psz = 0.0f, psgz = 0.0f;
#pragma unroll
      for (int u = 0; u < U; ++u) {
        acc(xv[u].x, gv[u].x, ps, psg, psz, psgz);
        acc(xv[u].y, gv[u].y, ps, psg, psz, psgz);
        acc(xv[u].z, gv[u].z, ps, psg, psz, psgz);
        acc(xv[u].w, gv[u].w, ps, psg, psz, psgz);
      }
      S += (double)ps;
      SG += (double)psg;
      if (kAlpha) {
        SZ += (double)psz;
        SGZ += (double)psgz;
      }
    }
  }
  const int64_t nrest = n - 4 * nb4;
  for (int64_t j = (int64_t)blockIdx.x * NT + threadIdx.x; j < nrest; j += (int64_t)gridDim.x * NT) {
    const int64_t i = rest_index(j, head, nb4);
    float ps = 0.0f, psg = 0.0f, psz = 0.0f, psgz = 0.0f;
    acc(x[i], g[i], ps, psg, psz, psgz);
    S += (double)ps;
    SG += (double)psg;
    if (kAlpha) {
      SZ += (double)psz;
      SGZ += (double)psgz;
    }
  }
  if (kAlpha) block_shift_reduce4<NT>(m, S, SG, SZ, SGZ, red);
  else block_shift_reduce<NT>(m, S, SG, red);
  BPart* part = reinterpret_cast<BPart*>(a.part) + r * kMaxGridPerRow;
  if (threadIdx.x == 0) part[blockIdx.x] = BPart{(double)m, S, SG, SZ, SGZ, 0.0};
  if (a.parts_only) {
    // sharded rows: slot 0 also carries this GPU's number of partials
    if (threadIdx.x == 0 && blockIdx.x == 0) part[0].pad = (double)gridDim.x;
    return;
  }
  if (last_block_done(a.done + r, gridDim.x)) combine_parts<kAlpha>(a, r, part, 0, 1, (int)gridDim.x, bad, inva, red);
}

// sharded rows: lambda from the partials of all GPUs (gathered: GPU w's
// [rows][kMaxGridPerRow] block at w * rows * kMaxGridPerRow)
template <bool kAlpha>
__global__ void __launch_bounds__(NT) k_bwd_combine(const StreamBwd a, const BPart* parts_all, int world) {
  __shared__ double red[64];
  const int64_t r = blockIdx.x;
  bool bad = false;
  const double inva = 1.0 / row_alpha(a.alpha, a.alpha_rows, r, &bad);
  combine_parts<kAlpha>(a, r, parts_all + r * kMaxGridPerRow, a.rows * kMaxGridPerRow, world, -1, bad, inva, red);
}

// grad = f (g - lambda), f = 2^(log2(1/(2 alpha)) - |x - b| log2(e)/alpha) in
// one exponent, lambda split into two fp32 words
__global__ void __launch_bounds__(NT) k_bwd_apply(const StreamBwd a) {
  wait_prior_grid();
  const int64_t r = blockIdx.y;
  const double b = a.b[r];
  bool bad = false;
  const double inva = 1.0 / row_alpha(a.alpha, a.alpha_rows, r, &bad);
  const float c2 = (float)(inva * (double)kLog2e);
  const float lg = (float)log2(0.5 * inva);
  const float bh = __double2float_rn(b);
  const float bl = __double2float_rn(b - (double)bh);
  const double lam = a.lam[r];
  const float lh = __double2float_rn(lam);
  const float ll = __double2float_rn(lam - (double)lh);
  const float* x = a.scores + r * a.stride;
  const float* g = a.grad_p + r * a.stride;
  float* o = a.grad + r * a.stride;
  const int64_t n = a.n;
  // x, g and grad start at the same address mod 16 when vec
  const int head = a.vec ? row_head(x, n) : 0;
  const int64_t nb4 = a.vec ? ((n - head) >> 2) / CHUNK4 * CHUNK4 : 0;
  {
    const float4* x4 = reinterpret_cast<const float4*>(x + head);
    const float4* g4 = reinterpret_cast<const float4*>(g + head);
    float4* o4 = reinterpret_cast<float4*>(o + head);
    const int64_t nchunks = nb4 / CHUNK4;
    for (int64_t q = blockIdx.x; q < nchunks; q += gridDim.x) {
      const int64_t qq = nchunks - 1 - q;  // reverse of the reduction pass
      const int64_t base = qq * CHUNK4 + threadIdx.x;
      float4 xv[U], gv[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        xv[u] = __ldcs(x4 + base + u * NT);
        gv[u] = __ldcs(g4 + base + u * NT);
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        float4 ov;
        ov.x = exp2f(fmaf(-fabsf((xv[u].x - bh) - bl), c2, lg)) * ((gv[u].x - lh) - ll);
        ov.y = exp2f(fmaf(-fabsf((xv[u].y - bh) - bl), c2, lg)) * ((gv[u].y - lh) - ll);
        ov.z = exp2f(fmaf(-fabsf((xv[u].z - bh) - bl), c2, lg)) * ((gv[u].z - lh) - ll);
        ov.w = exp2f(fmaf(-fabsf((xv[u].w - bh) - bl), c2, lg)) * ((gv[u].w - lh) - ll);
        stg_stream(o4 + base + u * NT, ov);
      }
    }
  }
  const int64_t nrest = n - 4 * nb4;
  for (int64_t j = (int64_t)blockIdx.x * NT + threadIdx.x; j < nrest; j += (int64_t)gridDim.x * NT) {
    const int64_t i = rest_index(j, head, nb4);
    o[i] = exp2f(fmaf(-fabsf((x[i] - bh) - bl), c2, lg)) * ((g[i] - lh) - ll);
  }
}


// ===========================================================================
// sharded rows: one long row split over GPUs in contiguous shards.  The
// pipeline above runs per GPU on its shard; three exchanges, made by the
// caller (NCCL), join the GPUs: the sample and level-1 histogram are summed,
// the filter's partials, band and band statistics are gathered, and every GPU
// then solves the same band for the same b.  Nothing here waits on another
// GPU.
// ===========================================================================

// this GPU's band statistics for the gather
__global__ void k_shard_pack(const StreamPlan P, uint32_t* meta) {
  const int64_t r = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (r >= P.rows) return;
  const RowCtl* c = ctl_of(P, r);
  uint32_t* m = meta + r * kShardMeta;
  m[0] = c->band_cnt;
  m[1] = c->band_kmax;
  m[2] = c->band_nkmin;
  m[3] = c->flags;
  m[4] = (uint32_t)P.Gf;
  m[5] = m[6] = m[7] = 0u;
}

// the gathered statistics and filter partials of all GPUs into this GPU's
// row control and one filter partial per row (fixed order over GPUs)
__global__ void __launch_bounds__(NT) k_shard_unpack(const StreamPlan Pb, int world, const FPart* g_fpart,
                                                      const uint32_t* g_meta) {
  __shared__ double red[64];
  const int64_t r = blockIdx.x;
  RowCtl* c = ctl_of(Pb, r);
  long long nl = 0;
  double sl = 0.0, sr = 0.0;
  uint32_t bad = 0u;
  for (int w = 0; w < world; ++w) {
    const uint32_t* m = g_meta + ((int64_t)w * Pb.rows + r) * kShardMeta;
    const int gf = min((int)m[4], kMaxGridPerRow);
    const FPart* fp = g_fpart + ((int64_t)w * Pb.rows + r) * kMaxGridPerRow;
    for (int i = threadIdx.x; i < gf; i += NT) {
      nl += fp[i].nL;
      sl += fp[i].SL;
      sr += fp[i].SR;
      bad |= fp[i].bad;
    }
  }
  nl = block_sum<NT, long long>(nl, reinterpret_cast<long long*>(red));
  sl = block_sum<NT, double>(sl, red);
  sr = block_sum<NT, double>(sr, red);
  bad = block_or<NT>(bad, reinterpret_cast<uint32_t*>(red));
  if (threadIdx.x == 0) {
    unsigned long long cnt = 0ull;
    uint32_t kmax = 0u, nkmin = 0u, flags = 0u;
    for (int w = 0; w < world; ++w) {
      const uint32_t* m = g_meta + ((int64_t)w * Pb.rows + r) * kShardMeta;
      cnt += m[0];
      kmax = max(kmax, m[1]);
      nkmin = max(nkmin, m[2]);
      flags |= m[3];
    }
    if (cnt > (unsigned long long)Pb.band_cap) flags |= ROW_OVERFLOW;
    c->band_cnt = (uint32_t)min(cnt, 0xFFFFFFFFull);
    c->band_kmax = kmax;
    c->band_nkmin = nkmin;
    c->flags = flags;
    FPart* f = fpart_of(Pb, r);
    f[0] = FPart{nl, sl, sr, bad, 0u};
  }
}

// the gathered bands, one after the other, into this GPU's band of each row
__global__ void __launch_bounds__(NT) k_shard_compact(const StreamPlan Pb, int world, const float* g_band,
                                                       const uint32_t* g_meta) {
  const int64_t r = blockIdx.y;
  float* dst = band_of(Pb, r);
  int64_t off = 0;
  for (int w = 0; w < world; ++w) {
    const int64_t cnt = min((int64_t)g_meta[((int64_t)w * Pb.rows + r) * kShardMeta], Pb.band_cap);
    const float* src = g_band + ((int64_t)w * Pb.rows + r) * Pb.band_cap;
    for (int64_t i = (int64_t)blockIdx.x * NT + threadIdx.x; i < cnt && off + i < Pb.band_cap;
         i += (int64_t)gridDim.x * NT)
      dst[off + i] = src[i];
    off += cnt;
  }
}

}  // namespace

cudaError_t stream_occupancy(StreamOcc* out) {
  cudaError_t e = cudaSuccess;
  for (BandKernel kb : {k_band<false>, k_band<true>}) {
    e = cudaFuncSetAttribute(kb, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kBandSmemBytes);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(kb, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
  }
  e = cudaFuncSetAttribute(k_filter, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kFilterSmemBytes);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(k_recover, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)RecSmem::kTotal);
  if (e != cudaSuccess) return e;
  int fb = 0, rb = 0, mb = 0, qb = 0, ab = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&fb, k_filter, kFilterThreads, kFilterSmemBytes);
  if (e != cudaSuccess) return e;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&mb, k_memb<false, false>, NT, 0);
  if (e != cudaSuccess) return e;
  int sb = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&sb, k_memb<true, false>, NT, 0);
  if (e != cudaSuccess) return e;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&qb, k_bwd_reduce<false>, NT, 0);
  if (e != cudaSuccess) return e;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&ab, k_bwd_apply, NT, 0);
  if (e != cudaSuccess) return e;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&rb, k_recover, NT, RecSmem::kTotal);
  if (e != cudaSuccess) return e;
  out->filter_blocks = std::max(fb, 1);
  out->memb_blocks = std::max(mb, 1);
  out->memb_sparse_blocks = std::max(sb, 1);
  out->reduce_blocks = std::max(qb, 1);
  out->apply_blocks = std::max(ab, 1);
  out->recover_blocks = std::max(rb, 1);
  // the largest cluster of band CTAs the device can hold at once
  out->band_max_cluster = 1;
  for (int cs = kMaxCluster; cs >= 2; cs >>= 1) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)cs, 1, 1);
    cfg.blockDim = dim3(kBandThreads, 1, 1);
    cfg.dynamicSmemBytes = kBandSmemBytes;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = (unsigned)cs;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    int nc = 0;
    if (cudaOccupancyMaxActiveClusters(&nc, k_band<false>, &cfg) == cudaSuccess && nc >= 1) {
      out->band_max_cluster = cs;
      break;
    }
    (void)cudaGetLastError();
  }
  return cudaSuccess;
}

// the short kernels of the forward pipeline are launched with programmatic
// stream serialization (each waits for the one ahead: wait_prior_grid)
constexpr bool kUsePdl = true;
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       Args... args) {
  return launch_ex(kUsePdl, kern, grid, block, smem, st, args...);
}

cudaError_t launch_stream_fwd(const StreamPlan& P, const float* scores, float* p_out, double* b_out,
                              double* sumf_out, uint32_t* status_out, lapsum_row_stats* stats, int sm_count,
                              cudaStream_t st) {
  (void)sm_count;
  cudaError_t e = cudaMemsetAsync(P.ctl, 0, P.zero_bytes, st);
  if (e != cudaSuccess) return e;
  const unsigned rows = (unsigned)P.rows;
  {
    Launch l("k_sample", st);
    k_sample<<<dim3(P.Gs, rows), NT, 0, st>>>(P, scores);
  }
  // the kernels below may be scheduled while the one ahead drains (each
  // waits for it at entry: wait_prior_grid)
  {
    Launch l("k_select23", st);
    e = launch_pdl(k_select23, dim3(P.Gs, rows), dim3(NT), 0, st, P);
    if (e != cudaSuccess) return e;
  }
  {
    Launch l("k_filter", st);
    e = launch_pdl(k_filter, dim3(P.Gf, rows), dim3(kFilterThreads), kFilterSmemBytes, st, P, scores);
    if (e != cudaSuccess) return e;
  }
  {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)P.band_cs, rows, 1);
    cfg.blockDim = dim3(kBandThreads, 1, 1);
    cfg.dynamicSmemBytes = kBandSmemBytes;
    cfg.stream = st;
    cudaLaunchAttribute at[2];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = (unsigned)P.band_cs;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    at[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[1].val.programmaticStreamSerializationAllowed = kUsePdl ? 1 : 0;
    cfg.attrs = at;
    cfg.numAttrs = 2;
    Launch l("k_band", st);
    e = cudaLaunchKernelEx(&cfg, band_kernel(P.band_cs), P);
    if (e != cudaSuccess) return e;
  }
  {
    StreamPlan Pc = P;
    const float* sc = scores;
    float* po = p_out;
    void* args[] = {&Pc, &sc, &po};
    Launch l("k_recover", st);
    e = cudaLaunchCooperativeKernel((const void*)k_recover, dim3(P.Gr), dim3(NT), args, RecSmem::kTotal, st);
    if (e != cudaSuccess) return e;
  }
  {
    if (P.sp.idx) {
      e = cudaMemsetAsync(P.sp.count, 0, sizeof(uint64_t) * (size_t)P.rows, st);
      if (e != cudaSuccess) return e;
      Launch l("k_memb_sparse", st);
      k_memb<true, false><<<dim3(P.Gms, rows), NT, 0, st>>>(P, scores, p_out, b_out, sumf_out, status_out, stats);
    } else {
      Launch l(P.dftopk ? "k_memb_dftopk" : "k_memb", st);
      if (P.dftopk)
        e = launch_ex(kPdlTail, k_memb<false, true>, dim3(P.Gm, rows), dim3(NT), 0, st, P, scores, p_out, b_out,
                      sumf_out, status_out, stats);
      else
        e = launch_ex(kPdlTail, k_memb<false, false>, dim3(P.Gm, rows), dim3(NT), 0, st, P, scores, p_out, b_out,
                      sumf_out, status_out, stats);
      if (e != cudaSuccess) return e;
    }
  }
  return cudaGetLastError();
}

cudaError_t launch_stream_bwd(const StreamBwd& a, cudaStream_t st) {
  cudaError_t e = cudaMemsetAsync(a.done, 0, sizeof(uint32_t) * (size_t)a.rows, st);
  if (e != cudaSuccess) return e;
  {
    Launch l("k_bwd_reduce", st);
    if (a.grad_alpha) k_bwd_reduce<true><<<dim3(a.Gb, (unsigned)a.rows), NT, 0, st>>>(a);
    else k_bwd_reduce<false><<<dim3(a.Gb, (unsigned)a.rows), NT, 0, st>>>(a);
  }
  {
    Launch l("k_bwd_apply", st);
    e = launch_ex(kPdlTail, k_bwd_apply, dim3(a.Ga, (unsigned)a.rows), dim3(NT), 0, st, a);
    if (e != cudaSuccess) return e;
  }
  return cudaGetLastError();
}

cudaError_t launch_shard_sample(const StreamPlan& P, const float* scores, cudaStream_t st) {
  cudaError_t e = cudaMemsetAsync(P.ctl, 0, P.zero_bytes, st);
  if (e != cudaSuccess) return e;
  // the level-1 histogram is part of the exchange, outside the zeroed block
  e = cudaMemsetAsync(P.hist1, 0, sizeof(uint32_t) * 2048 * (size_t)P.rows, st);
  if (e != cudaSuccess) return e;
  Launch l("k_sample", st);
  k_sample<<<dim3(P.Gs, (unsigned)P.rows), NT, 0, st>>>(P, scores);
  return cudaGetLastError();
}

cudaError_t launch_shard_filter(const StreamPlan& P, const float* scores, uint32_t* meta, cudaStream_t st) {
  const unsigned rows = (unsigned)P.rows;
  {
    Launch l("k_pick1", st);
    k_pick1<<<dim3(1, rows), NT, 0, st>>>(P);
  }
  {
    Launch l("k_select2", st);
    k_select2<<<dim3(P.Gs, rows), NT, 0, st>>>(P);
  }
  {
    Launch l("k_select3", st);
    k_select3<<<dim3(P.Gs, rows), NT, 0, st>>>(P);
  }
  {
    Launch l("k_filter", st);
    k_filter<<<dim3(P.Gf, rows), kFilterThreads, kFilterSmemBytes, st>>>(P, scores);
  }
  {
    Launch l("k_shard_pack", st);
    k_shard_pack<<<(rows + 127) / 128, 128, 0, st>>>(P, meta);
  }
  return cudaGetLastError();
}

cudaError_t launch_shard_finish(const StreamPlan& P, const StreamPlan& Pb, const float* scores, float* p_out,
                                double* b_out, double* sumf_out, uint32_t* status_out, int world,
                                const void* g_fpart, const uint32_t* g_meta, const float* g_band, cudaStream_t st) {
  const unsigned rows = (unsigned)P.rows;
  cudaError_t e;
  {
    Launch l("k_shard_unpack", st);
    k_shard_unpack<<<rows, NT, 0, st>>>(Pb, world, reinterpret_cast<const FPart*>(g_fpart), g_meta);
  }
  {
    Launch l("k_shard_compact", st);
    k_shard_compact<<<dim3(64, rows), NT, 0, st>>>(Pb, world, g_band, g_meta);
  }
  {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)Pb.band_cs, rows, 1);
    cfg.blockDim = dim3(kBandThreads, 1, 1);
    cfg.dynamicSmemBytes = kBandSmemBytes;
    cfg.stream = st;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = (unsigned)Pb.band_cs;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    Launch l("k_band", st);
    e = cudaLaunchKernelEx(&cfg, band_kernel(Pb.band_cs), Pb);
    if (e != cudaSuccess) return e;
  }
  // no recovery here: a row the band does not certify keeps its miss bits and
  // the caller solves it again from the whole row
  {
    Launch l("k_memb", st);
    k_memb<false, false><<<dim3(P.Gm, rows), NT, 0, st>>>(P, scores, p_out, b_out, sumf_out, status_out, nullptr);
  }
  return cudaGetLastError();
}

cudaError_t launch_shard_bwd_partials(const StreamBwd& a, bool with_alpha, cudaStream_t st) {
  Launch l("k_bwd_reduce", st);
  if (with_alpha) k_bwd_reduce<true><<<dim3(a.Gb, (unsigned)a.rows), NT, 0, st>>>(a);
  else k_bwd_reduce<false><<<dim3(a.Gb, (unsigned)a.rows), NT, 0, st>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_shard_bwd_finish(const StreamBwd& a, const void* parts_all, int world, cudaStream_t st) {
  {
    Launch l("k_bwd_combine", st);
    const BPart* pa = reinterpret_cast<const BPart*>(parts_all);
    if (a.grad_alpha) k_bwd_combine<true><<<(unsigned)a.rows, NT, 0, st>>>(a, pa, world);
    else k_bwd_combine<false><<<(unsigned)a.rows, NT, 0, st>>>(a, pa, world);
  }
  {
    Launch l("k_bwd_apply", st);
    const cudaError_t e = launch_ex(kPdlTail, k_bwd_apply, dim3(a.Ga, (unsigned)a.rows), dim3(NT), 0, st, a);
    if (e != cudaSuccess) return e;
  }
  return cudaGetLastError();
}

}  // namespace lapsum
