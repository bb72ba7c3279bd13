// block_sort.cuh -- sorting and selection of uint32 keys in shared memory,
// by one thread block.
//
// Section 2.2 of the Fast LapSum technical summary sorts only the band around
// the threshold, and the bracket needs two order statistics of the
// localization sample.  Here: a stable LSD radix sort (whole rows in the
// full-sort fallback), an MSD radix selection of two ranks (the one-block
// path's sample), a one-pass bucket sort over a known key range (a band, a
// small streaming band, the streaming band's root bin), and a bitonic network
// (the bucket sort's fallback when outliers crowd a bucket, and the sample
// when a widening needs other ranks).
//
// Radix sort: 8-bit digits, four passes.  Each warp owns one contiguous segment of the
// keys and walks it 32 keys at a time; __match_any_sync groups the lanes that
// share a digit, so ranks inside a warp follow key order and the pass is
// stable.  Offsets are laid out digit-major, warp-minor.  A pass whose digit
// is the same for every key is skipped (band keys usually share their top
// byte).
#pragma once

#include "common.cuh"

namespace lapsum {

// shared scratch for the radix routines: NT/32 * 256 counters, a flag word,
// NT/32 scan words, and 2 * 256 digit words for radix_pass's outputs
template <int NT>
struct SortScratch {
  static constexpr int kWords = (NT / 32) * 256 + 64 + 512;
};

// One stable pass: keys[0, n) -> tmp[0, n) ordered by digit (key >> shift) & 255.
// If the digit is the same for every key, nothing is moved and the function
// returns false (uniformly in all threads); otherwise it returns true.
// On return hist[NW*256 + 64 + d] holds the count of digit d and
// hist[NW*256 + 64 + 256 + d] its first position in tmp.
template <int NT>
__device__ bool radix_pass(const uint32_t* keys, uint32_t* tmp, int n, uint32_t* hist, int shift,
                           bool allow_skip = true) {
  static_assert(NT >= 256 && NT % 32 == 0, "radix_pass needs >= 256 threads");
  constexpr int NW = NT / 32;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const uint32_t lt_mask = (1u << lane) - 1u;
  const int per = (n + NW - 1) / NW;
  const int seg_lo = min(n, warp * per);
  const int seg_hi = min(n, seg_lo + per);
  uint32_t* whist = hist + warp * 256;
  uint32_t* flag = hist + NW * 256;
  uint32_t* scan_scr = flag + 1;  // NW words
  uint32_t* dcount = hist + NW * 256 + 64;
  uint32_t* dstart = dcount + 256;

  __syncthreads();  // previous users of hist are done
  for (int i = threadIdx.x; i < NW * 256; i += NT) hist[i] = 0u;
  if (threadIdx.x == 0) flag[0] = 0u;
  __syncthreads();
  for (int base = seg_lo; base < seg_hi; base += 32) {
    const int i = base + lane;
    const bool act = i < seg_hi;
    const uint32_t d = act ? ((keys[i] >> shift) & 255u) : 0u;
    const uint32_t amask = __ballot_sync(0xffffffffu, act);
    if (act) {
      const uint32_t peers = __match_any_sync(amask, d);
      if (lane == __ffs(peers) - 1) whist[d] += __popc(peers);
    }
    __syncwarp();
  }
  __syncthreads();
  uint32_t tot = 0;
  if (threadIdx.x < 256) {
    const uint32_t d = threadIdx.x;
    for (int w = 0; w < NW; ++w) {
      const uint32_t c = hist[w * 256 + d];
      hist[w * 256 + d] = tot;
      tot += c;
    }
    if (tot == (uint32_t)n) flag[0] = 1u;
  }
  const uint32_t base_d = block_excl_prefix_u32<NT>(threadIdx.x < 256 ? tot : 0u, scan_scr, nullptr);
  if (threadIdx.x < 256) {
    for (int w = 0; w < NW; ++w) hist[w * 256 + threadIdx.x] += base_d;
    dcount[threadIdx.x] = tot;
    dstart[threadIdx.x] = base_d;
  }
  __syncthreads();
  const bool skip = allow_skip && flag[0] != 0u;
  if (skip) return false;
  for (int base = seg_lo; base < seg_hi; base += 32) {
    const int i = base + lane;
    const bool act = i < seg_hi;
    const uint32_t k = act ? keys[i] : 0u;
    const uint32_t d = (k >> shift) & 255u;
    const uint32_t amask = __ballot_sync(0xffffffffu, act);
    uint32_t peers = 0u;
    if (act) {
      peers = __match_any_sync(amask, d);
      tmp[whist[d] + __popc(peers & lt_mask)] = k;
    }
    __syncwarp();
    if (act && lane == __ffs(peers) - 1) whist[d] += __popc(peers);
    __syncwarp();
  }
  __syncthreads();
  return true;
}

// Sorts keys[0, n) ascending.  `tmp` must hold n keys; `hist` must hold
// SortScratch<NT>::kWords words.  Returns the buffer (keys or tmp) that holds
// the result.  All NT threads of the block must call it.
template <int NT>
__device__ uint32_t* block_radix_sort(uint32_t* keys, uint32_t* tmp, int n, uint32_t* hist) {
  for (int shift = 0; shift < 32; shift += 8) {
    if (radix_pass<NT>(keys, tmp, n, hist, shift)) {
      uint32_t* t = keys;
      keys = tmp;
      tmp = t;
    }
  }
  return keys;
}

// The keys of ascending ranks r[0] and r[1] among keys[0, n) (0 <= r < n),
// without sorting: an MSD radix selection, 8 bits a level, one histogram per
// rank over the keys that share its prefix so far.  Lanes of a warp that add
// to the same bin are merged first (__match_any_sync), so equal keys cost one
// atomic per warp.  scr: >= kSelectWords words of shared memory.  All NT
// threads must call it; the result is returned in every thread.
constexpr int kSelectWords = 2 * 256 + 4;
template <int NT>
__device__ void block_select2(const uint32_t* keys, int n, const int (&r)[2], uint32_t (&out)[2], uint32_t* scr) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t* st = scr + 512;  // prefix of rank 0 and 1, then the ranks left inside them
  if (threadIdx.x == 0) {
    st[0] = st[1] = 0u;
    st[2] = (uint32_t)r[0];
    st[3] = (uint32_t)r[1];
  }
  for (int level = 0; level < 4; ++level) {
    const int shift = 24 - 8 * level;
    const uint32_t pmask = level == 0 ? 0u : (0xFFFFFFFFu << (32 - 8 * level));
    for (int i = threadIdx.x; i < 512; i += NT) scr[i] = 0u;
    __syncthreads();
    const uint32_t p0 = st[0], p1 = st[1];
    for (int base = 0; base < n; base += NT) {
      const int i = base + (int)threadIdx.x;
      const bool act = i < n;
      const uint32_t k = act ? keys[i] : 0u;
      const uint32_t d = (k >> shift) & 255u;
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        const bool in = act && (k & pmask) == (t == 0 ? p0 : p1);
        const uint32_t im = __ballot_sync(0xffffffffu, in);
        if (in) {
          const uint32_t peers = __match_any_sync(im, d);
          if (lane == __ffs(peers) - 1) atomicAdd(&scr[256 * t + d], (uint32_t)__popc(peers));
        }
      }
    }
    __syncthreads();
    if (warp < 2) {  // warp t finds the digit of rank t: lane l scans bins 8l .. 8l+7
      const uint32_t* h = scr + 256 * warp;
      const uint32_t rem = st[2 + warp];
      uint32_t c[8], s = 0u;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        c[j] = h[8 * lane + j];
        s += c[j];
      }
      uint32_t incl = s;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      const uint32_t excl = incl - s;
      __syncwarp();
      if (rem >= excl && rem < incl) {
        uint32_t acc = excl;  // keys of this prefix in lower bins
        int d = 0;
        bool found = false;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          if (!found) {
            if (rem < acc + c[j]) {
              d = j;
              found = true;
            } else {
              acc += c[j];
            }
          }
        }
        st[warp] |= (uint32_t)(8 * lane + d) << shift;
        st[2 + warp] = rem - acc;
      }
    }
    __syncthreads();
  }
  out[0] = st[0];
  out[1] = st[1];
  __syncthreads();  // st may be reused by the caller
}

// Sorts keys[0, n) ascending with one bucket pass: NT buckets over the key
// range [kmin, kmax] (the caller's bounds of the keys; NT a power of two >=
// 256), a histogram, a scan, a scatter into tmp, then one thread sorts each
// bucket by insertion (equal keys cost no moves).  About five barriers
// instead of a network's log2(N)^2/2 stages.  If any bucket holds more than
// kMaxBucket keys (a range stretched by outliers), it returns null and nothing
// is sorted: the caller falls back to a network.  tmp must hold n keys, scr
// bucket_sort_scr_words(NT) words.  Returns tmp (sorted) on success.  All NT
// threads must call it.
constexpr int kMaxBucket = 48;
__host__ __device__ constexpr int bucket_sort_scr_words(int nt) { return 2 * nt + 64; }
template <int NT>
__device__ uint32_t* block_bucket_sort(const uint32_t* keys, uint32_t* tmp, int n, uint32_t kmin, uint32_t kmax,
                                       uint32_t* scr) {
  static_assert(NT >= 256 && (NT & (NT - 1)) == 0, "one thread per bucket");
  uint32_t* cnt = scr;          // NT counts, then cursors
  uint32_t* start = scr + NT;   // NT bucket starts
  uint32_t* big = scr + 2 * NT; // flag: a crowded bucket
  int shift = 0;
  while (((kmax - kmin) >> shift) >= (uint32_t)NT) ++shift;
  cnt[threadIdx.x] = 0u;
  if (threadIdx.x == 0) *big = 0u;
  __syncthreads();
  for (int i = threadIdx.x; i < n; i += NT) atomicAdd(&cnt[(keys[i] - kmin) >> shift], 1u);
  __syncthreads();
  const uint32_t c = cnt[threadIdx.x];
  const uint32_t st = block_excl_prefix_u32<NT>(c, scr + 2 * NT + 8, nullptr);
  start[threadIdx.x] = st;
  cnt[threadIdx.x] = st;  // cursor
  if (c > (uint32_t)kMaxBucket) *big = 1u;
  __syncthreads();
  if (*big) return nullptr;  // uniform: read after the barrier
  for (int i = threadIdx.x; i < n; i += NT) {
    const uint32_t k = keys[i];
    tmp[atomicAdd(&cnt[(k - kmin) >> shift], 1u)] = k;
  }
  __syncthreads();
  {
    const int lo = (int)start[threadIdx.x], hi = lo + (int)c;
    for (int i = lo + 1; i < hi; ++i) {
      const uint32_t k = tmp[i];
      int j = i - 1;
      while (j >= lo && tmp[j] > k) {
        tmp[j + 1] = tmp[j];
        --j;
      }
      tmp[j + 1] = k;
    }
  }
  __syncthreads();
  return tmp;
}

// Sorts buf[0, n) ascending in place with a bitonic network over N = the next
// power of two >= n; buf must hold N keys (entries n..N-1 are overwritten with
// the largest key, which no finite value maps to).  Order-independent and
// insensitive to ties; about log2(N)^2 / 2 barrier stages.
template <int NT>
__device__ void block_bitonic_sort(uint32_t* buf, int n) {
  int N = 1;
  while (N < n) N <<= 1;
  for (int i = n + threadIdx.x; i < N; i += NT) buf[i] = 0xFFFFFFFFu;
  __syncthreads();
  for (int k = 2; k <= N; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int i = threadIdx.x; i < (N >> 1); i += NT) {
        const int lo = ((i & ~(j - 1)) << 1) | (i & (j - 1));
        const int hi = lo | j;
        const uint32_t a = buf[lo], b = buf[hi];
        if ((a > b) == ((lo & k) == 0)) {
          buf[lo] = b;
          buf[hi] = a;
        }
      }
      __syncthreads();
    }
  }
}

}  // namespace lapsum
