// abi.cu -- the C ABI of lapsum_topk.h: argument checks, the localization
// plan, workspace layout and dispatch to the resident (one block per row) or
// streaming (many blocks per row) kernels.
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "common.cuh"
#include "launch.h"
#include "lapsum_topk.h"

namespace lapsum {

cudaError_t resident_init(int optin_bytes);

namespace {

constexpr int kMaxDevices = 64;
struct DevInfo {
  bool ready = false;
  int sm_count = 0;
  int smem_optin = 0;  // bytes of shared memory a block may opt in to
  StreamOcc occ{};
};
DevInfo g_dev[kMaxDevices];
std::mutex g_mu;

cudaError_t device_info(DevInfo** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  DevInfo* d = &g_dev[dev];
  if (!d->ready) {
    std::lock_guard<std::mutex> lk(g_mu);
    if (!d->ready) {
      e = cudaDeviceGetAttribute(&d->sm_count, cudaDevAttrMultiProcessorCount, dev);
      if (e != cudaSuccess) return e;
      e = cudaDeviceGetAttribute(&d->smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
      if (e != cudaSuccess) return e;
      e = resident_init(d->smem_optin);
      if (e != cudaSuccess) return e;
      e = stream_occupancy(&d->occ);
      if (e != cudaSuccess) return e;
      d->ready = true;
    }
  }
  *out = d;
  return cudaSuccess;
}

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

constexpr double kDftopkSolveAlpha = 1e-30;  // the smallest scale the solver accepts

// the text of the last failed CUDA call on this host thread
thread_local const char* t_last_error = "no error";
bool cuda_ok(cudaError_t e) {
  if (e == cudaSuccess) return true;
  t_last_error = cudaGetErrorString(e);
  return false;
}

struct Resolved {
  double z;
  uint64_t seed;
  int max_widen;
  uint32_t force;
  uint32_t m_user;
  int64_t bcap_user;
  uint32_t spin_limit;  // 0 = the kernels' default
};

Resolved resolve(const lapsum_params* p) {
  Resolved r;
  // z = 4: a bracket edge misses b with probability ~3e-5 (normal
  // approximation of the binomial); a miss costs one widening pass, so the
  // expected cost is far below what the narrower band saves
  r.z = (p && p->z > 0.0 && std::isfinite(p->z)) ? p->z : 4.0;
  r.seed = p ? p->seed : 0;
  r.max_widen = (p && p->max_widen >= 0) ? std::min(p->max_widen, 1) : 1;
  r.force = p ? p->force_path : 0u;
  r.m_user = p ? p->sample_m : 0u;
  r.bcap_user = p ? p->band_capacity : 0;
  r.spin_limit = (p && p->spin_limit > 0) ? (uint32_t)p->spin_limit : 0u;
  return r;
}

// Localization ranks (section 2.2): #{Y > b} ~ Binomial(m, k/n); the bracket
// edges are the c_lo-th and (c_hi+1)-th largest samples, c_lo/hi = mq -/+ z sigma.
struct Ranks {
  int rank_lo, rank_hi;  // ascending indices into the sorted sample
  int valid_lo, valid_hi;
  int widen_delta;
};
Ranks sample_ranks(int64_t n, double k, int m, double z) {
  const double q = k / (double)n;
  const double mq = (double)m * q;
  const double sigma = std::sqrt(mq * (1.0 - q));
  const int64_t c_lo = (int64_t)std::floor(mq - z * sigma);
  const int64_t c_hi = (int64_t)std::ceil(mq + z * sigma);
  Ranks R;
  R.valid_hi = c_lo >= 1;
  R.rank_hi = R.valid_hi ? (int)(m - c_lo) : m - 1;
  R.valid_lo = (c_hi + 1) <= m;
  R.rank_lo = R.valid_lo ? (int)(m - c_hi - 1) : 0;
  R.widen_delta = (int)std::ceil(2.0 * z * sigma) + 1;
  return R;
}

// Arrays walked together as float4 must start at the same address mod 16:
// every row of them then shares one head of 0-3 scores, which the kernels
// take one at a time before the float4 body.  A null array (not written)
// imposes nothing.
int same_phase(const void* a, const void* b, const void* c = nullptr) {
  const uintptr_t ph = (uintptr_t)a & 15u;
  return (!b || ((uintptr_t)b & 15u) == ph) && (!c || ((uintptr_t)c & 15u) == ph);
}

int round_up(int64_t x, int64_t a) { return (int)(((x + a - 1) / a) * a); }

bool resident_path(int64_t n, const Resolved& R) {
  return n <= kResidentMaxN && !(R.force & LAPSUM_FORCE_STREAMING);
}

// ---- resident plan -------------------------------------------------------
struct ResPlan {
  int m, bcap;
  Ranks rk;
};
// The sample size balances the sample and its selection (cost ~ m) against
// the band (size ~ n / sqrt(m)): m ~ (z n sqrt(q (1 - q)))^(2/3).  A batch
// of the longest rows (more rows than the GPU holds at once, `batch`, of
// more than 8192 scores) is bound by the throughput of its rows rather than
// the latency of one; where the balanced size is already at least 384 (the
// band is large), a sample of 1024 shrinks the band and its sort and solve
// by more than the longer sample costs.  Fwd+bwd of 2048 x 16384 (the tied
// batch): k = 256, 228 -> 224 us; k = 1024, 394 -> 324 us; k = 4096, 560 ->
// 556 us; k = 256 at alpha 0.05, 271 -> 268 us; 600 rows at k = 256, 102 ->
// 98 us.  Where the balanced size is smaller the larger sample lost (k = 64:
// 202 -> 206 us; 2048 x 12001 at k = 200: 195 -> 197 us; rows of 4096 and
// 8192 scores: 108 -> 111 and 142 -> 146 us), and beyond 1024 the sample's
// shared memory costs a resident row per SM.
ResPlan resident_plan(int64_t n, double k, const Resolved& R, bool batch) {
  ResPlan p;
  const double q = k / (double)n;
  if (R.m_user) {
    p.m = (int)std::min<uint32_t>(R.m_user, 4096u);
  } else {
    const double opt = std::pow(R.z * (double)n * std::sqrt(q * (1.0 - q)), 2.0 / 3.0);
    p.m = std::min(2048, std::max(128, round_up((int64_t)std::ceil(opt), 32)));
    if (batch && n > 8192 && opt >= 384.0) p.m = std::max(p.m, 1024);
  }
  p.rk = sample_ranks(n, k, p.m, R.z);
  const double M_est = (double)(p.rk.rank_hi - p.rk.rank_lo + 1) * (double)n / (double)p.m;
  int64_t bcap = R.bcap_user > 0 ? R.bcap_user : (int64_t)(2.0 * M_est) + 256;
  bcap = std::max<int64_t>(1, std::min<int64_t>(bcap, std::min<int64_t>(n, 8192)));
  p.bcap = round_up(bcap, 4);
  return p;
}

// ---- streaming plan and workspace ---------------------------------------
struct StreamSizes {
  int m;
  Ranks rk;
  double M_est;  // expected band size
  int64_t band_cap;
};
StreamSizes stream_sizes(int64_t n, double k, const Resolved& R) {
  StreamSizes s;
  s.m = R.m_user ? (int)std::min<uint32_t>(R.m_user, 1u << 20)
                 : (int)std::min<int64_t>(1 << 17, std::max<int64_t>(2048, round_up(n / 8, 1024)));
  s.rk = sample_ranks(n, k, s.m, R.z);
  s.M_est = (double)(s.rk.rank_hi - s.rk.rank_lo + 1) * (double)n / (double)s.m;
  // default capacity: four times the expected band plus slack (overflow sends
  // the row to the fallback)
  int64_t cap = R.bcap_user > 0 ? R.bcap_user : (int64_t)(4.0 * s.M_est) + 16384;
  cap = std::max<int64_t>(R.bcap_user > 0 ? 4 : 1024, std::min<int64_t>(cap, (int64_t)round_up(n, 1024)));
  s.band_cap = round_up(cap, 4);
  return s;
}

struct StreamLayout {
  size_t ctl, h1, h2, h3, zero_end, samp, cand, fpart, band, mpart, fb_keys, fb_aggs, rcount, total;
};
StreamLayout stream_layout(int64_t rows, int64_t n, const StreamSizes& s) {
  StreamLayout L;
  size_t o = 0;
  L.ctl = o;     o = align256(o + sizeof(RowCtl) * (size_t)rows);
  L.h1 = o;      o = align256(o + 4 * 2048 * (size_t)rows);
  L.h2 = o;      o = align256(o + 4 * 4096 * (size_t)rows);
  L.h3 = o;      o = align256(o + 4 * 2048 * (size_t)rows);
  L.zero_end = o;
  L.samp = o;    o = align256(o + 4 * (size_t)s.m * (size_t)rows);
  L.cand = o;    o = align256(o + 4 * (size_t)((s.m + 3) & ~3) * (size_t)rows);
  L.fpart = o;   o = align256(o + 32 * (size_t)kMaxGridPerRow * (size_t)rows);
  L.band = o;    o = align256(o + 4 * (size_t)s.band_cap * (size_t)rows);
  L.mpart = o;   o = align256(o + 32 * (size_t)kMaxGridPerRow * (size_t)rows);
  L.fb_keys = o; o = align256(o + 4 * (size_t)n);
  L.fb_aggs = o; o = align256(o + sizeof(GroupAgg) * (size_t)(n / kFallbackGroup + 2));
  L.rcount = o;  o = align256(o + 4 * (256 * (size_t)kMaxGridPerRow + 512));
  L.total = o;
  return L;
}

size_t resident_ws_bytes(int64_t rows) { return align256(4 * (size_t)rows) + 256 + align256(4 * (size_t)rows); }

size_t bwd_ws_bytes(int64_t rows, int64_t n) {
  if (n <= kResidentMaxN) return 0;
  return align256(48 * (size_t)kMaxGridPerRow * (size_t)rows) + align256(4 * (size_t)rows) +
         align256(8 * (size_t)rows);
}

size_t fwd_ws_bytes(int64_t rows, int64_t n, double k, const Resolved& R) {
  if (resident_path(n, R)) return resident_ws_bytes(rows);
  return stream_layout(rows, n, stream_sizes(n, k, R)).total;
}

// Blocks per row of a streaming pass: one full wave of the device shared by
// the rows, but no more blocks than 4096-score chunks in a row.
int stream_grid(int sm_count, int blocks_per_sm, int64_t rows, int64_t n) {
  const int64_t per_row = std::max<int64_t>(1, (int64_t)sm_count * blocks_per_sm / rows);
  const int64_t chunks = std::max<int64_t>(1, (n / 4 + 1023) / 1024);
  return (int)std::min<int64_t>({(int64_t)kMaxGridPerRow, per_row, chunks});
}

// The plan of the streaming pipeline for rows of n scores (the band sized by
// s), its pieces at the offsets L of the workspace ws.
StreamPlan stream_plan(int64_t rows, int64_t n, int64_t row_stride, double k, double alpha, const StreamSizes& s,
                       const StreamLayout& L, const Resolved& R, const DevInfo& dev, int vec, unsigned char* ws) {
  const StreamOcc& occ = dev.occ;
  StreamPlan P{};
  P.rows = rows;
  P.n = n;
  P.stride = row_stride;
  P.k = k;
  P.alpha = alpha;
  P.alpha_p = alpha;
  P.m = s.m;
  P.rank_lo = s.rk.rank_lo;
  P.rank_hi = s.rk.rank_hi;
  P.valid_lo = s.rk.valid_lo;
  P.valid_hi = s.rk.valid_hi;
  P.widen_delta = s.rk.widen_delta;
  P.max_widen = R.max_widen;
  P.band_cap = s.band_cap;
  P.seed = R.seed;
  P.force_fallback = (R.force & LAPSUM_FORCE_FALLBACK) != 0;
  P.force_timeout = (R.force & LAPSUM_FORCE_TIMEOUT) != 0;
  P.spin_limit = R.spin_limit;
  P.vec = vec;
  const int sm = dev.sm_count;
  P.Gs = (int)std::min<int64_t>(1024, std::max<int64_t>(1, (s.m + 1023) / 1024));
  P.Gf = stream_grid(sm, occ.filter_blocks, rows, n);
  P.Gm = stream_grid(sm, occ.memb_blocks, rows, n);
  P.Gr = std::min(kMaxGridPerRow, sm * occ.recover_blocks);
  // band cluster: about kBandValuesPerCta expected band values per CTA
  // (with more than one CTA the leader holds no slice)
  int cs = 1;
  while (cs < occ.band_max_cluster && (double)(cs > 1 ? cs - 1 : 1) * kBandValuesPerCta < s.M_est) cs <<= 1;
  P.band_cs = cs;
  P.ctl = ws + L.ctl;
  P.zero_bytes = L.zero_end - L.ctl;
  P.hist1 = reinterpret_cast<uint32_t*>(ws + L.h1);
  P.hist2 = reinterpret_cast<uint32_t*>(ws + L.h2);
  P.hist3 = reinterpret_cast<uint32_t*>(ws + L.h3);
  P.samp = reinterpret_cast<uint32_t*>(ws + L.samp);
  P.cand = reinterpret_cast<uint32_t*>(ws + L.cand);
  P.fpart = ws + L.fpart;
  P.band = reinterpret_cast<float*>(ws + L.band);
  P.mpart = ws + L.mpart;
  P.fb_keys = reinterpret_cast<uint32_t*>(ws + L.fb_keys);
  P.fb_aggs = ws + L.fb_aggs;
  P.rcount = reinterpret_cast<uint32_t*>(ws + L.rcount);
  P.z = R.z;
  return P;
}

bool overlaps(const void* a, size_t an, const void* b, size_t bn) {
  const uintptr_t x = (uintptr_t)a, y = (uintptr_t)b;
  return x < y + bn && y < x + an;
}

// The forward pass behind lapsum_topk_fwd (sp == null: dense p),
// lapsum_topk_fwd_sparse (sp: the entries with p >= eps) and lapsum_dftopk_fwd
// (dftopk: b solved at the tiny scale `alpha`, memberships at alpha_p).
int fwd_impl(const float* scores, int64_t rows, int64_t n, int64_t row_stride, double k, double alpha, float* p_out,
             double* b_out, double* sumf_out, uint32_t* row_status, lapsum_row_stats* stats, void* workspace,
             size_t workspace_bytes, const lapsum_params* params, void* stream, const SparseOut* sp,
             double alpha_p, bool dftopk, double* sump_out, const double* k_rows = nullptr,
             const double* alpha_rows = nullptr) {
  if (!scores || !b_out || (!sp && !p_out)) return LAPSUM_EINVAL;
  if (rows < 1 || n < 1 || n > INT32_MAX || row_stride < n) return LAPSUM_EINVAL;
  if (((uintptr_t)scores & 3u) || ((uintptr_t)p_out & 3u) || ((uintptr_t)b_out & 7u)) return LAPSUM_EINVAL;
  if (sp) {
    if (!sp->idx || !sp->val || !sp->count || sp->cap < 0) return LAPSUM_EINVAL;
    if (((uintptr_t)sp->idx & 3u) || ((uintptr_t)sp->val & 3u) || ((uintptr_t)sp->count & 7u)) return LAPSUM_EINVAL;
    if (!std::isfinite(sp->eps) || !(sp->eps > 0.0f) || !(sp->eps <= 1.0f)) return LAPSUM_EINVAL;
    p_out = nullptr;
  }
  if (sumf_out && ((uintptr_t)sumf_out & 7u)) return LAPSUM_EINVAL;
  if (sump_out && ((uintptr_t)sump_out & 7u)) return LAPSUM_EINVAL;
  if (((uintptr_t)k_rows & 7u) || ((uintptr_t)alpha_rows & 7u)) return LAPSUM_EINVAL;
  // per-row values are checked on the device; the host plans for the widest
  // bracket (k = n/2) and takes the ranks of each row from its own k there
  if (k_rows) k = 0.5 * (double)n;
  if (alpha_rows) alpha = alpha_p = 1.0;
  if (!std::isfinite(k) || !(k > 0.0) || !(k < (double)n)) return LAPSUM_EBADK;
  if (!std::isfinite(alpha) || !(alpha >= 1e-30) || !(alpha <= 1e30)) return LAPSUM_EBADALPHA;
  const size_t span = 4 * (size_t)((rows - 1) * row_stride + n);
  if (p_out && overlaps(scores, span, p_out, span)) return LAPSUM_EINVAL;
  if (sp) {
    const size_t ob = 4 * (size_t)sp->cap * (size_t)rows;
    if (ob && (overlaps(scores, span, sp->idx, ob) || overlaps(scores, span, sp->val, ob) ||
               overlaps(sp->idx, ob, sp->val, ob)))
      return LAPSUM_EINVAL;
  }
  const Resolved R = resolve(params);
  const bool res = resident_path(n, R);
  if (!res && rows > 65535) return LAPSUM_EINVAL;
  const size_t need = fwd_ws_bytes(rows, n, k, R) + ((sp && !res) ? align256(4 * (size_t)n) : 0);
  if (!workspace || workspace_bytes < need || ((uintptr_t)workspace & 255u)) return LAPSUM_EWORKSPACE;

  DevInfo* dev = nullptr;
  if (!cuda_ok(device_info(&dev))) return LAPSUM_ECUDA;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int vec = same_phase(scores, p_out);
  unsigned char* ws = static_cast<unsigned char*>(workspace);

  if (res) {
    const ResPlan rp = resident_plan(n, k, R, rows > (int64_t)dev->sm_count * kResidentBlocksPerSm);
    ResidentFwd a{};
    a.scores = scores;
    a.rows = rows;
    a.n = n;
    a.stride = row_stride;
    a.k = k;
    a.alpha = alpha;
    a.p_out = p_out;
    a.b_out = b_out;
    a.sumf_out = sumf_out;
    a.status_out = row_status;
    a.stats = stats;
    a.m = rp.m;
    a.rank_lo = rp.rk.rank_lo;
    a.rank_hi = rp.rk.rank_hi;
    a.valid_lo = rp.rk.valid_lo;
    a.valid_hi = rp.rk.valid_hi;
    a.widen_delta = rp.rk.widen_delta;
    a.max_widen = R.max_widen;
    a.bcap = rp.bcap;
    a.seed = R.seed;
    a.force_fallback = (R.force & LAPSUM_FORCE_FALLBACK) != 0;
    a.force_timeout = (R.force & LAPSUM_FORCE_TIMEOUT) != 0;
    a.spin_limit = R.spin_limit;
    a.vec = vec;
    a.ws_status = reinterpret_cast<uint32_t*>(ws);
    a.fb_count = reinterpret_cast<uint32_t*>(ws + align256(4 * (size_t)rows));
    a.fb_list = reinterpret_cast<int32_t*>(ws + align256(4 * (size_t)rows) + 256);
    if (sp) a.sp = *sp;
    a.alpha_p = alpha_p;
    a.dftopk = dftopk ? 1 : 0;
    a.sump_out = sump_out;
    a.k_rows = k_rows;
    a.alpha_rows = alpha_rows;
    a.z = R.z;
    if (resident_fwd_smem(a) + 1024 > (size_t)dev->smem_optin) return LAPSUM_EINVAL;
    return cuda_ok(launch_resident_fwd(a, dev->sm_count, st)) ? LAPSUM_OK : LAPSUM_ECUDA;
  }

  const StreamSizes s = stream_sizes(n, k, R);
  const StreamLayout L = stream_layout(rows, n, s);
  const StreamOcc& occ = dev->occ;
  const int sm = dev->sm_count;
  StreamPlan P = stream_plan(rows, n, row_stride, k, alpha, s, L, R, *dev, vec, ws);
  P.alpha_p = alpha_p;
  P.dftopk = dftopk ? 1 : 0;
  P.sump_out = sump_out;
  P.k_rows = k_rows;
  P.alpha_rows = alpha_rows;
  P.z = R.z;
  if (sp) {
    P.sp = *sp;
    P.fb_keys2 = reinterpret_cast<uint32_t*>(ws + L.total);  // past the dense layout
    P.Gms = stream_grid(sm, occ.memb_sparse_blocks, rows, n);
  }
  P.rcount = reinterpret_cast<uint32_t*>(ws + L.rcount);
  return cuda_ok(launch_stream_fwd(P, scores, p_out, b_out, sumf_out, row_status, stats, sm, st)) ? LAPSUM_OK
                                                                                                : LAPSUM_ECUDA;
}

// ---- sharded rows ------------------------------------------------------------
// The band of a sharded row is sized for the widest bracket (as the workspace
// of the one-GPU forward is), so that the gathered exchange buffers have one
// layout whatever k is.
int64_t shard_band_cap(int64_t n_total, const Resolved& R) {
  int64_t cap = 0;
  for (double kk : {1.0, 0.5 * (double)n_total, (double)n_total - 1.0})
    if (kk > 0.0 && kk < (double)n_total) cap = std::max(cap, stream_sizes(n_total, kk, R).band_cap);
  return std::max<int64_t>(cap, 4);
}

void shard_layout(int64_t rows, int64_t n_total, const Resolved& R, lapsum_shard_layout* o) {
  StreamSizes s = stream_sizes(n_total, 0.5 * (double)n_total, R);
  s.band_cap = shard_band_cap(n_total, R);
  const StreamLayout L = stream_layout(rows, 0, s);
  o->sample_m = s.m;
  o->band_cap = s.band_cap;
  o->sample_bytes = 4 * (size_t)s.m * (size_t)rows;
  o->hist_bytes = 4 * 2048 * (size_t)rows;
  o->meta_bytes = 4 * (size_t)kShardMeta * (size_t)rows;
  o->fpart_bytes = 32 * (size_t)kMaxGridPerRow * (size_t)rows;
  o->band_bytes = 4 * (size_t)s.band_cap * (size_t)rows;
  o->parts_bytes = 48 * (size_t)kMaxGridPerRow * (size_t)rows;
  o->workspace_bytes = std::max(L.total, align256(8 * (size_t)rows) + align256(4 * (size_t)rows));
}

bool aligned16(const void* p) { return p && ((uintptr_t)p & 15u) == 0; }

// Checks the arguments every sharded forward call shares and builds the plan
// of this GPU's shard (P) and of the band step (Pb) in the workspace.
int shard_fwd_plan(const float* scores, int64_t rows, int64_t n, int64_t row_stride, int64_t shard_lo,
                   int64_t n_total, double k, double alpha, void* workspace, size_t workspace_bytes,
                   const lapsum_params* params, const float* p_out, StreamPlan* P, StreamPlan* Pb, DevInfo** dev) {
  if (!scores || ((uintptr_t)scores & 3u)) return LAPSUM_EINVAL;
  if (rows < 1 || rows > 65535 || n < 1 || row_stride < n || shard_lo < 0 || n_total > INT32_MAX ||
      shard_lo + n > n_total)
    return LAPSUM_EINVAL;
  if (!std::isfinite(k) || !(k > 0.0) || !(k < (double)n_total)) return LAPSUM_EBADK;
  if (!std::isfinite(alpha) || !(alpha >= 1e-30) || !(alpha <= 1e30)) return LAPSUM_EBADALPHA;
  const Resolved R = resolve(params);
  lapsum_shard_layout lay;
  shard_layout(rows, n_total, R, &lay);
  if (!workspace || workspace_bytes < lay.workspace_bytes || ((uintptr_t)workspace & 255u)) return LAPSUM_EWORKSPACE;
  if (!cuda_ok(device_info(dev))) return LAPSUM_ECUDA;
  StreamSizes s = stream_sizes(n_total, k, R);  // ranks and cluster size from this k
  s.band_cap = lay.band_cap;
  StreamSizes sl = s;
  const StreamLayout L = stream_layout(rows, 0, sl);
  const int vec = same_phase(scores, p_out);
  *P = stream_plan(rows, n, row_stride, k, alpha, s, L, R, **dev, vec, static_cast<unsigned char*>(workspace));
  P->shard = 1;
  P->n_total = n_total;
  P->shard_lo = shard_lo;
  *Pb = *P;
  Pb->Gf = 1;  // the gathered filter partials arrive summed into one per row
  return LAPSUM_OK;
}

// The backward behind lapsum_topk_bwd (one alpha) and lapsum_topk_bwd_rows
// (alpha_rows: one per row, checked on the device).
int bwd_impl(const float* scores, const float* grad_p, const double* b, int64_t rows, int64_t n,
             int64_t row_stride, double alpha, const double* alpha_rows, float* grad_scores, double* grad_k,
             double* grad_alpha, void* workspace, size_t workspace_bytes, void* stream) {
  if (!scores || !grad_p || !b || !grad_scores) return LAPSUM_EINVAL;
  if (rows < 1 || n < 1 || n > INT32_MAX || row_stride < n) return LAPSUM_EINVAL;
  if (((uintptr_t)scores & 3u) || ((uintptr_t)grad_p & 3u) || ((uintptr_t)grad_scores & 3u) ||
      ((uintptr_t)b & 7u))
    return LAPSUM_EINVAL;
  if (grad_k && ((uintptr_t)grad_k & 7u)) return LAPSUM_EINVAL;
  if (grad_alpha && ((uintptr_t)grad_alpha & 7u)) return LAPSUM_EINVAL;
  if (alpha_rows) {
    if ((uintptr_t)alpha_rows & 7u) return LAPSUM_EINVAL;
    alpha = 1.0;
  }
  if (!std::isfinite(alpha) || !(alpha >= 1e-30) || !(alpha <= 1e30)) return LAPSUM_EBADALPHA;
  const size_t span = 4 * (size_t)((rows - 1) * row_stride + n);
  if (overlaps(scores, span, grad_scores, span) || overlaps(grad_p, span, grad_scores, span)) return LAPSUM_EINVAL;
  const size_t need = bwd_ws_bytes(rows, n);
  if (need > 0 && (!workspace || workspace_bytes < need || ((uintptr_t)workspace & 255u))) return LAPSUM_EWORKSPACE;
  if (n > kResidentMaxN && rows > 65535) return LAPSUM_EINVAL;
  DevInfo* dev = nullptr;
  if (!cuda_ok(device_info(&dev))) return LAPSUM_ECUDA;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int vec = same_phase(scores, grad_p, grad_scores);
  if (n <= kResidentMaxN) {
    RowBwd a{scores, grad_p, b, rows, n, row_stride, alpha, grad_scores, grad_k, vec, grad_alpha, alpha_rows};
    return cuda_ok(launch_resident_bwd(a, dev->sm_count, st)) ? LAPSUM_OK : LAPSUM_ECUDA;
  }
  unsigned char* ws = static_cast<unsigned char*>(workspace);
  StreamBwd a{};
  a.scores = scores;
  a.grad_p = grad_p;
  a.b = b;
  a.rows = rows;
  a.n = n;
  a.stride = row_stride;
  a.alpha = alpha;
  a.grad = grad_scores;
  a.grad_k = grad_k;
  a.grad_alpha = grad_alpha;
  a.alpha_rows = alpha_rows;
  a.vec = vec;
  a.Gb = stream_grid(dev->sm_count, dev->occ.reduce_blocks, rows, n);
  a.Ga = stream_grid(dev->sm_count, dev->occ.apply_blocks, rows, n);
  size_t o = 0;
  a.part = ws + o;
  o = align256(o + 48 * (size_t)kMaxGridPerRow * (size_t)rows);
  a.done = reinterpret_cast<uint32_t*>(ws + o);
  o = align256(o + 4 * (size_t)rows);
  a.lam = reinterpret_cast<double*>(ws + o);
  return cuda_ok(launch_stream_bwd(a, st)) ? LAPSUM_OK : LAPSUM_ECUDA;
}

}  // namespace
}  // namespace lapsum

using namespace lapsum;

extern "C" {

void lapsum_default_params(lapsum_params* p) {
  if (!p) return;
  std::memset(p, 0, sizeof(*p));
  p->z = 4.0;
  p->max_widen = -1;
}

const char* lapsum_last_cuda_error(void) { return t_last_error; }

const char* lapsum_status_string(int code) {
  switch (code) {
    case LAPSUM_OK: return "ok";
    case LAPSUM_EINVAL: return "invalid argument (null or misaligned pointer, bad shape, or overlapping buffers)";
    case LAPSUM_EBADK: return "k must be finite with 0 < k < n";
    case LAPSUM_EBADALPHA: return "alpha must be finite and in [1e-30, 1e30]";
    case LAPSUM_EWORKSPACE: return "workspace missing or smaller than lapsum_topk_workspace_size()";
    case LAPSUM_ECUDA: return "a CUDA call or kernel launch failed";
    case LAPSUM_ETOOLARGE: return "rows > LAPSUM_NOALLOC_MAX_ROWS or n > LAPSUM_NOALLOC_MAX_N for the allocation-free forward";
    default: return "unknown status";
  }
}

int lapsum_topk_fwd(const float* scores, int64_t rows, int64_t n, int64_t row_stride, double k, double alpha,
                    float* p_out, double* b_out, double* sumf_out, uint32_t* row_status, lapsum_row_stats* stats,
                    void* workspace, size_t workspace_bytes, const lapsum_params* params, void* stream) {
  return fwd_impl(scores, rows, n, row_stride, k, alpha, p_out, b_out, sumf_out, row_status, stats, workspace,
                  workspace_bytes, params, stream, nullptr, alpha, false, nullptr);
}

int lapsum_topk_fwd_sparse(const float* scores, int64_t rows, int64_t n, int64_t row_stride, double k,
                           double alpha, float eps, int32_t* idx_out, float* val_out, int64_t capacity,
                           uint64_t* count_out, double* b_out, double* sumf_out, uint32_t* row_status,
                           lapsum_row_stats* stats, void* workspace, size_t workspace_bytes,
                           const lapsum_params* params, void* stream) {
  const SparseOut sp{eps, idx_out, val_out, capacity, count_out};
  return fwd_impl(scores, rows, n, row_stride, k, alpha, nullptr, b_out, sumf_out, row_status, stats, workspace,
                  workspace_bytes, params, stream, &sp, alpha, false, nullptr);
}

int lapsum_topk_fwd_rows(const float* scores, int64_t rows, int64_t n, int64_t row_stride, const double* k,
                         const double* alpha, float* p_out, double* b_out, double* sumf_out, uint32_t* row_status,
                         lapsum_row_stats* stats, void* workspace, size_t workspace_bytes,
                         const lapsum_params* params, void* stream) {
  if (!k || !alpha) return LAPSUM_EINVAL;
  return fwd_impl(scores, rows, n, row_stride, 1.0, 1.0, p_out, b_out, sumf_out, row_status, stats, workspace,
                  workspace_bytes, params, stream, nullptr, 1.0, false, nullptr, k, alpha);
}

int lapsum_dftopk_fwd(const float* scores, int64_t rows, int64_t n, int64_t row_stride, int64_t k, double alpha,
                      float* p_out, double* b_out, double* sumf_out, double* mass_out, uint32_t* row_status,
                      lapsum_row_stats* stats, void* workspace, size_t workspace_bytes, const lapsum_params* params,
                      void* stream) {
  if (k < 1 || k >= n) return LAPSUM_EBADK;
  if (!std::isfinite(alpha) || !(alpha >= 1e-30) || !(alpha <= 1e30)) return LAPSUM_EBADALPHA;
  // the budget solve at a vanishing scale lands on the midpoint of the k-th
  // and (k+1)-th largest scores (closed form: mid + (a/2) ln(A/B), a -> 0)
  return fwd_impl(scores, rows, n, row_stride, (double)k, kDftopkSolveAlpha, p_out, b_out, sumf_out, row_status,
                  stats, workspace, workspace_bytes, params, stream, nullptr, alpha, true, mass_out);
}

size_t lapsum_topk_sparse_workspace_size(int64_t rows, int64_t n, const lapsum_params* params) {
  const size_t dense = lapsum_topk_workspace_size(rows, n, params);
  if (dense == 0) return 0;
  const Resolved R = resolve(params);
  return dense + (resident_path(n, R) ? 0 : align256(4 * (size_t)n));
}

size_t lapsum_topk_workspace_size(int64_t rows, int64_t n, const lapsum_params* params) {
  if (rows < 1 || n < 1 || n > INT32_MAX) return 0;
  const Resolved R = resolve(params);
  // k only shapes the band estimate; size for the widest case (k = n/2)
  const size_t fwd = std::max(fwd_ws_bytes(rows, n, 0.5 * (double)n, R),
                              std::max(fwd_ws_bytes(rows, n, 1.0, R), fwd_ws_bytes(rows, n, (double)n - 1.0, R)));
  return std::max(fwd, bwd_ws_bytes(rows, n));
}

int lapsum_topk_bwd(const float* scores, const float* grad_p, const double* b, int64_t rows, int64_t n,
                    int64_t row_stride, double alpha, float* grad_scores, double* grad_k, double* grad_alpha,
                    void* workspace, size_t workspace_bytes, void* stream) {
  return bwd_impl(scores, grad_p, b, rows, n, row_stride, alpha, nullptr, grad_scores, grad_k, grad_alpha, workspace,
                  workspace_bytes, stream);
}

int lapsum_topk_bwd_rows(const float* scores, const float* grad_p, const double* b, int64_t rows, int64_t n,
                         int64_t row_stride, const double* alpha, float* grad_scores, double* grad_k,
                         double* grad_alpha, void* workspace, size_t workspace_bytes, void* stream) {
  if (!alpha) return LAPSUM_EINVAL;
  return bwd_impl(scores, grad_p, b, rows, n, row_stride, 1.0, alpha, grad_scores, grad_k, grad_alpha, workspace,
                  workspace_bytes, stream);
}

void lapsum_shard_layout_get(int64_t rows, int64_t n_total, const lapsum_params* params, lapsum_shard_layout* out) {
  if (!out) return;
  std::memset(out, 0, sizeof(*out));
  if (rows < 1 || n_total < 1 || n_total > INT32_MAX) return;
  shard_layout(rows, n_total, resolve(params), out);
}

int lapsum_shard_fwd_sample(const float* scores, int64_t rows, int64_t n, int64_t row_stride, int64_t shard_lo,
                            int64_t n_total, double k, double alpha, uint32_t* x_sample, uint32_t* x_hist,
                            void* workspace, size_t workspace_bytes, const lapsum_params* params, void* stream) {
  if (!aligned16(x_sample) || !aligned16(x_hist)) return LAPSUM_EINVAL;
  StreamPlan P, Pb;
  DevInfo* dev = nullptr;
  const int rc = shard_fwd_plan(scores, rows, n, row_stride, shard_lo, n_total, k, alpha, workspace,
                                workspace_bytes, params, nullptr, &P, &Pb, &dev);
  if (rc != LAPSUM_OK) return rc;
  P.samp = x_sample;
  P.hist1 = x_hist;
  return cuda_ok(launch_shard_sample(P, scores, reinterpret_cast<cudaStream_t>(stream))) ? LAPSUM_OK : LAPSUM_ECUDA;
}

int lapsum_shard_fwd_filter(const float* scores, int64_t rows, int64_t n, int64_t row_stride, int64_t shard_lo,
                            int64_t n_total, double k, double alpha, const uint32_t* x_sample,
                            const uint32_t* x_hist, uint32_t* x_meta, void* x_fpart, float* x_band,
                            void* workspace, size_t workspace_bytes, const lapsum_params* params, void* stream) {
  if (!aligned16(x_sample) || !aligned16(x_hist) || !aligned16(x_meta) || !aligned16(x_fpart) || !aligned16(x_band))
    return LAPSUM_EINVAL;
  StreamPlan P, Pb;
  DevInfo* dev = nullptr;
  const int rc = shard_fwd_plan(scores, rows, n, row_stride, shard_lo, n_total, k, alpha, workspace,
                                workspace_bytes, params, nullptr, &P, &Pb, &dev);
  if (rc != LAPSUM_OK) return rc;
  P.samp = const_cast<uint32_t*>(x_sample);
  P.hist1 = const_cast<uint32_t*>(x_hist);
  P.fpart = x_fpart;
  P.band = x_band;
  return cuda_ok(launch_shard_filter(P, scores, x_meta, reinterpret_cast<cudaStream_t>(stream))) ? LAPSUM_OK
                                                                                                  : LAPSUM_ECUDA;
}

int lapsum_shard_fwd_finish(const float* scores, int64_t rows, int64_t n, int64_t row_stride, int64_t shard_lo,
                            int64_t n_total, double k, double alpha, int world, const uint32_t* g_meta,
                            const void* g_fpart, const float* g_band, float* p_out, double* b_out, double* sumf_out,
                            uint32_t* row_status, void* workspace, size_t workspace_bytes,
                            const lapsum_params* params, void* stream) {
  if (world < 1 || world > 1024 || !aligned16(g_meta) || !aligned16(g_fpart) || !aligned16(g_band)) return LAPSUM_EINVAL;
  if (!p_out || !b_out || ((uintptr_t)p_out & 3u) || ((uintptr_t)b_out & 7u)) return LAPSUM_EINVAL;
  if (sumf_out && ((uintptr_t)sumf_out & 7u)) return LAPSUM_EINVAL;
  const size_t span = 4 * (size_t)((rows - 1) * row_stride + n);
  if (rows >= 1 && n >= 1 && overlaps(scores, span, p_out, span)) return LAPSUM_EINVAL;
  StreamPlan P, Pb;
  DevInfo* dev = nullptr;
  const int rc = shard_fwd_plan(scores, rows, n, row_stride, shard_lo, n_total, k, alpha, workspace,
                                workspace_bytes, params, p_out, &P, &Pb, &dev);
  if (rc != LAPSUM_OK) return rc;
  return cuda_ok(launch_shard_finish(P, Pb, scores, p_out, b_out, sumf_out, row_status, world, g_fpart, g_meta, g_band,
                                     reinterpret_cast<cudaStream_t>(stream)))
             ? LAPSUM_OK
             : LAPSUM_ECUDA;
}

int lapsum_shard_bwd_partials(const float* scores, const float* grad_p, const double* b, int64_t rows, int64_t n,
                              int64_t row_stride, double alpha, int with_alpha, void* x_parts, void* stream) {
  if (!scores || !grad_p || !b || !aligned16(x_parts)) return LAPSUM_EINVAL;
  if (rows < 1 || rows > 65535 || n < 1 || n > INT32_MAX || row_stride < n) return LAPSUM_EINVAL;
  if (((uintptr_t)scores & 3u) || ((uintptr_t)grad_p & 3u) || ((uintptr_t)b & 7u)) return LAPSUM_EINVAL;
  if (!std::isfinite(alpha) || !(alpha >= 1e-30) || !(alpha <= 1e30)) return LAPSUM_EBADALPHA;
  DevInfo* dev = nullptr;
  if (!cuda_ok(device_info(&dev))) return LAPSUM_ECUDA;
  StreamBwd a{};
  a.scores = scores;
  a.grad_p = grad_p;
  a.b = b;
  a.rows = rows;
  a.n = n;
  a.stride = row_stride;
  a.alpha = alpha;
  a.vec = same_phase(scores, grad_p);
  a.parts_only = 1;
  a.part = x_parts;
  a.Gb = stream_grid(dev->sm_count, dev->occ.reduce_blocks, rows, n);
  return cuda_ok(launch_shard_bwd_partials(a, with_alpha != 0, reinterpret_cast<cudaStream_t>(stream))) ? LAPSUM_OK
                                                                                                    : LAPSUM_ECUDA;
}

int lapsum_shard_bwd_finish(const float* scores, const float* grad_p, const double* b, int64_t rows, int64_t n,
                            int64_t row_stride, double alpha, int world, const void* g_parts, float* grad_scores,
                            double* grad_k, double* grad_alpha, void* workspace, size_t workspace_bytes,
                            void* stream) {
  if (!scores || !grad_p || !b || !grad_scores || !aligned16(g_parts) || world < 1 || world > 1024)
    return LAPSUM_EINVAL;
  if (rows < 1 || rows > 65535 || n < 1 || n > INT32_MAX || row_stride < n) return LAPSUM_EINVAL;
  if (((uintptr_t)scores & 3u) || ((uintptr_t)grad_p & 3u) || ((uintptr_t)grad_scores & 3u) || ((uintptr_t)b & 7u))
    return LAPSUM_EINVAL;
  if ((grad_k && ((uintptr_t)grad_k & 7u)) || (grad_alpha && ((uintptr_t)grad_alpha & 7u))) return LAPSUM_EINVAL;
  if (!std::isfinite(alpha) || !(alpha >= 1e-30) || !(alpha <= 1e30)) return LAPSUM_EBADALPHA;
  const size_t span = 4 * (size_t)((rows - 1) * row_stride + n);
  if (overlaps(scores, span, grad_scores, span) || overlaps(grad_p, span, grad_scores, span)) return LAPSUM_EINVAL;
  const size_t need = align256(8 * (size_t)rows);
  if (!workspace || workspace_bytes < need || ((uintptr_t)workspace & 255u)) return LAPSUM_EWORKSPACE;
  DevInfo* dev = nullptr;
  if (!cuda_ok(device_info(&dev))) return LAPSUM_ECUDA;
  StreamBwd a{};
  a.scores = scores;
  a.grad_p = grad_p;
  a.b = b;
  a.rows = rows;
  a.n = n;
  a.stride = row_stride;
  a.alpha = alpha;
  a.grad = grad_scores;
  a.grad_k = grad_k;
  a.grad_alpha = grad_alpha;
  a.vec = same_phase(scores, grad_p, grad_scores);
  a.lam = static_cast<double*>(workspace);
  a.Ga = stream_grid(dev->sm_count, dev->occ.apply_blocks, rows, n);
  return cuda_ok(launch_shard_bwd_finish(a, g_parts, world, reinterpret_cast<cudaStream_t>(stream))) ? LAPSUM_OK
                                                                                                      : LAPSUM_ECUDA;
}

}  // extern "C"

// ---- allocation-free forward --------------------------------------------
// Some callers cannot allocate device memory at the moment they run the
// operator: an inference engine that hands each plugin a fixed arena, a host
// that has reserved all device memory for its own pool, or a framework that
// must not synchronise (cudaMalloc may) in the middle of a step.  For rows
// that one block holds (n <= 16384), the forward needs only 8 bytes of
// scratch per row and one counter, so that scratch can live in a static
// device array that the library owns.  The paper has no counterpart to this.

// (2 * 256 KiB + 256 bytes: row statuses, the fallback counter, the fallback
// row list for LAPSUM_NOALLOC_MAX_ROWS rows.)  Every GPU that loads the
// library holds it until the process exits.  It is shared by every call on a
// device and keeps the last call's contents; the only word that must start at
// zero (the fallback row counter) is cleared on the caller's stream by each
// call before the kernels that read it.
static __device__ __align__(256) unsigned char g_noalloc_scratch[2 * 4 * LAPSUM_NOALLOC_MAX_ROWS + 256];

namespace lapsum {
namespace {

constexpr int64_t kNoAllocMaxRows = LAPSUM_NOALLOC_MAX_ROWS;
constexpr size_t kNoAllocBytes = sizeof(g_noalloc_scratch);
static_assert(4 * LAPSUM_NOALLOC_MAX_ROWS % 256 == 0, "row arrays must keep 256-byte alignment");
static_assert(LAPSUM_NOALLOC_MAX_N == kResidentMaxN, "the allocation-free forward is the one-block-per-row path");

unsigned char* g_noalloc_ptr[kMaxDevices];  // device address of the array, per device

// The array's device address on the current device, looked up on the first
// call there (in host code the symbol is only a stand-in, not an address).
cudaError_t noalloc_scratch(unsigned char** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_noalloc_ptr[dev] = static_cast<unsigned char*>(p);
  }
  *out = g_noalloc_ptr[dev];
  return cudaSuccess;
}

}  // namespace
}  // namespace lapsum

extern "C" int lapsum_topk_fwd_noalloc(const float* scores, int64_t rows, int64_t n, int64_t row_stride, double k,
                                       double alpha, float* p_out, double* b_out, double* sumf_out,
                                       uint32_t* row_status, lapsum_row_stats* stats, const lapsum_params* params,
                                       void* stream) {
  if (!scores || !p_out || !b_out) return LAPSUM_EINVAL;
  if (rows < 1 || n < 1 || row_stride < n) return LAPSUM_EINVAL;
  if (rows > kNoAllocMaxRows || n > LAPSUM_NOALLOC_MAX_N) return LAPSUM_ETOOLARGE;
  if (((uintptr_t)scores & 3u) || ((uintptr_t)p_out & 3u) || ((uintptr_t)b_out & 7u)) return LAPSUM_EINVAL;
  if (sumf_out && ((uintptr_t)sumf_out & 7u)) return LAPSUM_EINVAL;
  if (!std::isfinite(k) || !(k > 0.0) || !(k < (double)n)) return LAPSUM_EBADK;
  if (!std::isfinite(alpha) || !(alpha >= 1e-30) || !(alpha <= 1e30)) return LAPSUM_EBADALPHA;
  const size_t span = 4 * (size_t)((rows - 1) * row_stride + n);
  if (overlaps(scores, span, p_out, span)) return LAPSUM_EINVAL;
  const Resolved R = resolve(params);
  if (!resident_path(n, R)) return LAPSUM_EINVAL;  // LAPSUM_FORCE_STREAMING is not available here
  DevInfo* dev = nullptr;
  if (!cuda_ok(device_info(&dev))) return LAPSUM_ECUDA;
  unsigned char* ws = nullptr;
  if (!cuda_ok(noalloc_scratch(&ws))) return LAPSUM_ECUDA;

  const ResPlan rp = resident_plan(n, k, R, rows > (int64_t)dev->sm_count * kResidentBlocksPerSm);
  ResidentFwd a{};
  a.scores = scores;
  a.rows = rows;
  a.n = n;
  a.stride = row_stride;
  a.k = k;
  a.alpha = alpha;
  a.p_out = p_out;
  a.b_out = b_out;
  a.sumf_out = sumf_out;
  a.status_out = row_status;
  a.stats = stats;
  a.m = rp.m;
  a.rank_lo = rp.rk.rank_lo;
  a.rank_hi = rp.rk.rank_hi;
  a.valid_lo = rp.rk.valid_lo;
  a.valid_hi = rp.rk.valid_hi;
  a.widen_delta = rp.rk.widen_delta;
  a.max_widen = R.max_widen;
  a.bcap = rp.bcap;
  a.seed = R.seed;
  a.force_fallback = (R.force & LAPSUM_FORCE_FALLBACK) != 0;
  a.force_timeout = (R.force & LAPSUM_FORCE_TIMEOUT) != 0;
  a.spin_limit = R.spin_limit;
  a.vec = same_phase(scores, p_out);
  a.alpha_p = alpha;
  // same layout as the caller-workspace forward: statuses, counter, row list
  const size_t list_off = align256(4 * (size_t)rows);
  if (2 * list_off + 256 > kNoAllocBytes) return LAPSUM_ETOOLARGE;
  a.ws_status = reinterpret_cast<uint32_t*>(ws);
  a.fb_count = reinterpret_cast<uint32_t*>(ws + list_off);
  a.fb_list = reinterpret_cast<int32_t*>(ws + list_off + 256);
  if (resident_fwd_smem(a) + 1024 > (size_t)dev->smem_optin) return LAPSUM_EINVAL;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  return cuda_ok(launch_resident_fwd(a, dev->sm_count, st)) ? LAPSUM_OK : LAPSUM_ECUDA;
}
