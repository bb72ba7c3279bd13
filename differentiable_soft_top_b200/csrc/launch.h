// launch.h -- host-side interface between the C ABI (abi.cu) and the kernel
// translation units.  Not part of the public boundary.
#pragma once

#include <cmath>
#include <cstddef>
#include <cstdint>
#include <cstring>
#include <algorithm>
#include <cuda_runtime.h>

#include "lapsum_topk.h"

namespace lapsum {

void note_launch(int count);

// Scope guard around one kernel launch: counts it and, while tracing is on,
// brackets it with CUDA events on its stream (see trace.cu).
class Launch {
 public:
  Launch(const char* name, cudaStream_t st);
  ~Launch();
  Launch(const Launch&) = delete;
  Launch& operator=(const Launch&) = delete;

 private:
  const char* name_;
  cudaStream_t st_;
  cudaEvent_t a_ = nullptr, b_ = nullptr;
};

// Launches kern on st; with `pdl`, with programmatic stream serialization:
// the kernel may be scheduled before the one ahead of it on the stream has
// finished, and must wait for it (griddepcontrol.wait) before it reads
// anything that kernel wrote.
template <typename... KArgs, typename... Args>
cudaError_t launch_ex(bool pdl, void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                      Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}
// kernels that follow a short or usually idle kernel are launched this way
constexpr bool kPdlTail = true;

// rows of at most this many scores run on the resident path (one block per
// row, the row held in shared memory)
constexpr int64_t kResidentMaxN = 16384;
constexpr int kResidentThreads = 256;
constexpr int kResidentBlocksPerSm = 4;  // one-block forward rows resident per SM (its launch bound)

// Sparse output of a forward pass: the entries with p >= eps as (index, p)
// pairs, row r at r * cap; count[r] receives the number of such entries
// (which may exceed cap: then only cap of them are written).  idx == null
// means the dense output p.
struct SparseOut {
  float eps;
  int32_t* idx;
  float* val;
  int64_t cap;
  uint64_t* count;
};

struct ResidentFwd {
  const float* scores;
  int64_t rows, n, stride;
  double k, alpha;
  float* p_out;
  double* b_out;
  double* sumf_out;
  uint32_t* status_out;
  lapsum_row_stats* stats;
  // localization plan (identical for every row)
  int m;                 // sample size
  int rank_lo, rank_hi;  // ascending sample ranks of a_L and a_R
  int valid_lo, valid_hi;
  int widen_delta;       // rank distance of one widening
  int max_widen;
  int bcap;              // band capacity
  uint64_t seed;
  int force_fallback;
  int force_timeout;     // test knob: odd rows wait on a barrier no copy completes
  uint32_t spin_limit;   // polls of a bounded wait; 0 = kSpinLimitDefault
  int vec;               // scores and p_out start at the same address mod 16
  // workspace
  uint32_t* ws_status;   // [rows]
  uint32_t* fb_count;    // [1]
  int32_t* fb_list;      // [rows]
  SparseOut sp;          // sparse output instead of p_out (sp.idx != null)
  double alpha_p;        // scale of the memberships (alpha except for DFTopK)
  int dftopk;            // memberships around a threshold solved at a tiny alpha:
                         // sum f is taken in the membership pass at alpha_p
  double* sump_out;      // [rows] sum p (may be null)
  // per-row budget and scale (device [rows], or null: k and alpha above for
  // every row); the ranks are then computed per row from z and m
  const double* k_rows;
  const double* alpha_rows;
  double z;
};

size_t resident_fwd_smem(const ResidentFwd& a);
size_t resident_fallback_smem(int64_t n);
cudaError_t launch_resident_fwd(const ResidentFwd& a, int sm_count, cudaStream_t st);

struct RowBwd {
  const float* scores;
  const float* grad_p;
  const double* b;
  int64_t rows, n, stride;
  double alpha;
  float* grad;
  double* grad_k;
  int vec;             // scores, grad_p and grad start at the same address mod 16
  double* grad_alpha;  // dL/dalpha per row, or null
  const double* alpha_rows;  // per-row alpha (device [rows]) or null
};
cudaError_t launch_resident_bwd(const RowBwd& a, int sm_count, cudaStream_t st);

// ---- multi-block (streaming) path ---------------------------------------
struct StreamPlan {
  int64_t rows, n, stride;
  double k, alpha;
  int m;
  int rank_lo, rank_hi, valid_lo, valid_hi;
  int widen_delta, max_widen;
  int64_t band_cap;      // band slots per row
  uint64_t seed;
  int force_fallback;
  int force_timeout;     // test knob: odd rows go to the recovery kernel, whose
                         // barrier then waits for one block more than it has
  uint32_t spin_limit;   // polls of a bounded wait; 0 = kSpinLimitDefault
  int vec;               // scores and p_out start at the same address mod 16
  int Gs, Gf, Gm, Gr;    // grids: sampling, filter, membership, recovery
  int band_cs;           // CTAs in the cluster that solves one row's band
  // workspace pieces
  void* ctl;             // RowCtl[rows] followed by the zeroed per-row block
  size_t zero_bytes;     // bytes to clear at the start of each forward
  uint32_t* hist1;       // [rows][2048]
  uint32_t* hist2;       // [rows][2][2048]
  uint32_t* hist3;       // [rows][2][1024]
  uint32_t* samp;        // [rows][m]
  uint32_t* cand;        // [rows][m] sample keys of the two level-1 bins picked
  void* fpart;           // filter partials [rows][Gf]
  float* band;           // [rows][band_cap], unsorted
  void* mpart;           // membership partials [rows][Gm]
  uint32_t* fb_keys;     // [n] keys for the full-sort fallback
  uint32_t* fb_keys2;    // [n] its second buffer when there is no dense p to borrow
  void* fb_aggs;         // GroupAgg [n / kFallbackGroup + 1]
  uint32_t* rcount;      // radix counts [256 * Gr] (+ scan space)
  SparseOut sp;          // sparse output instead of p (sp.idx != null)
  int Gms;               // grid of the sparse membership pass
  double alpha_p;        // scale of the memberships (alpha except for DFTopK)
  int dftopk;            // sum f taken in the membership pass at alpha_p
  double* sump_out;      // [rows] sum p (may be null)
  const double* k_rows;      // per-row k (device [rows]) or null
  const double* alpha_rows;  // per-row alpha (device [rows]) or null
  double z;                  // rank half-width in standard deviations
  // sharded rows (shard != 0): this GPU holds scores [shard_lo, shard_lo + n)
  // of rows n_total long; the sample and the band solve see the whole row,
  // the streaming passes the shard
  int shard;
  int64_t n_total, shard_lo;
};

constexpr int kFallbackGroup = 4096;   // full-sort fallback: sorted values per group
constexpr int kBucketMax = 8192;       // keys of the fallback's shared-memory tiles
constexpr int kMaxGridPerRow = 4096;   // partial-sum slots per row
constexpr int kStreamThreads = 256;
constexpr int kBandValuesPerCta = 16384;  // band values one CTA of the band cluster bins

cudaError_t launch_stream_fwd(const StreamPlan& P, const float* scores, float* p_out, double* b_out,
                              double* sumf_out, uint32_t* status_out, lapsum_row_stats* stats,
                              int sm_count, cudaStream_t st);

struct StreamBwd {
  const float* scores;
  const float* grad_p;
  const double* b;
  int64_t rows, n, stride;
  double alpha;
  float* grad;
  double* grad_k;
  double* grad_alpha;  // dL/dalpha per row, or null
  const double* alpha_rows;  // per-row alpha (device [rows]) or null
  int vec;           // scores, grad_p and grad start at the same address mod 16
  int parts_only;    // sharded rows: the reduction only writes this shard's partials
  int Gb, Ga;        // grids of the reduction and elementwise passes
  void* part;        // [rows][kMaxGridPerRow] partials (48 bytes each)
  uint32_t* done;    // [rows] counters (zeroed by the launcher)
  double* lam;       // [rows]
};
cudaError_t launch_stream_bwd(const StreamBwd& a, cudaStream_t st);

// ---- sharded rows: the streaming pipeline split at its three exchanges ----
// Exchange 1 (sum over GPUs): the sample keys (P.samp; 0 where another GPU
// holds the sampled score) and the level-1 histogram (P.hist1).
// Exchange 2 (gather): per GPU and row, kShardMeta words (band count, largest
// key, complement of the smallest key, flags, filter grid), the filter
// partials (P.fpart, kMaxGridPerRow slots per row) and the band (P.band,
// band_cap values per row).
// Backward exchange (gather): the reduction partials, kMaxGridPerRow slots of
// 48 bytes per row; slot 0 carries the number of valid slots.
constexpr int kShardMeta = 8;
cudaError_t launch_shard_sample(const StreamPlan& P, const float* scores, cudaStream_t st);
cudaError_t launch_shard_filter(const StreamPlan& P, const float* scores, uint32_t* meta, cudaStream_t st);
// Pb: the plan of the band step (local workspace for fpart and band)
cudaError_t launch_shard_finish(const StreamPlan& P, const StreamPlan& Pb, const float* scores, float* p_out,
                                double* b_out, double* sumf_out, uint32_t* status_out, int world,
                                const void* g_fpart, const uint32_t* g_meta, const float* g_band, cudaStream_t st);
cudaError_t launch_shard_bwd_partials(const StreamBwd& a, bool with_alpha, cudaStream_t st);
cudaError_t launch_shard_bwd_finish(const StreamBwd& a, const void* parts_all, int world, cudaStream_t st);

// occupancy facts of the streaming kernels on the current device
struct StreamOcc {
  int filter_blocks;    // resident blocks per SM of the filter pass
  int memb_blocks;      // of the membership pass
  int reduce_blocks;    // of the backward reduction
  int apply_blocks;     // of the backward elementwise pass
  int memb_sparse_blocks;  // of the sparse membership pass
  int recover_blocks;   // of the cooperative recovery kernel
  int band_max_cluster; // largest cluster of band CTAs (power of two, <= 16)
};
cudaError_t stream_occupancy(StreamOcc* out);

}  // namespace lapsum
