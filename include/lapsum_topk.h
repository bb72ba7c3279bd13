/*
 * lapsum_topk.h -- C ABI of the B200 exact-budget LapSum soft top-k.
 *
 * The operator ("Fast LapSum: Exact Differentiable Top-k at Million Scale",
 * Technical Summary section 2.1): for one row of scores r_1..r_n, a budget
 * k (0 < k < n) and a Laplace scale alpha > 0,
 *
 *     p_i = F((r_i - b) / alpha),   F(z) = exp(z)/2 (z < 0), 1 - exp(-z)/2 (z >= 0),
 *
 * with the threshold b fixed by the exact budget  sum_i p_i = k.  The
 * backward pass (same section: an analytic vector-Jacobian product) is
 *
 *     grad_j = f_j (g_j - lambda),  f_j = exp(-|r_j - b|/alpha) / (2 alpha),
 *     lambda = sum_i g_i f_i / sum_i f_i   (which is also dL/dk).
 *
 * How b is found (section 2.2 of the same page, and the arXiv abstract of
 * Fast LapSum): a sample of Laplace-noised scores and binomial order
 * statistics give a bracket [a_L, a_R); one streaming pass keeps the scores
 * inside it (the band) and folds the others into tail sums; the band is sorted
 * and the budget equation is solved in closed form on it; a certification
 * step proves b lies in the bracket, widening it once and falling back to a
 * full sort of the row when it does not.
 *
 * Conventions for every entry point:
 *   - All array pointers are DEVICE pointers owned by the caller.  The library
 *     allocates no memory: scratch space is the caller's `workspace` (or,
 *     for lapsum_topk_fwd_noalloc, a static array inside the library).
 *   - Scores are fp32, `rows` rows of `n` values, row i starting at
 *     scores + i * row_stride (row-major when row_stride == n).  Outputs use
 *     the same layout.  Outputs may not overlap inputs.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).  All
 *     work is enqueued on it; no entry point synchronises the host.
 *   - Arguments are validated on the host before anything is launched; a
 *     non-zero return code means nothing was enqueued.  Device-side outcomes
 *     are reported per row in `row_status` (see LAPSUM_ROW_*), readable after
 *     the stream has been synchronised.
 *   - k and alpha are shared by all rows, except in the *_rows entry points,
 *     which take one of each per row.  alpha must lie in [1e-30, 1e30] (the
 *     fp32 exponent arithmetic needs 1/alpha finite).
 *   - The first call on a device queries its properties and sets kernel
 *     attributes; later calls on that device do not.  That set-up is kept
 *     for the life of the process: after cudaDeviceReset, do not call the
 *     library again in that process.
 */
#ifndef LAPSUM_TOPK_H
#define LAPSUM_TOPK_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define LAPSUM_API __attribute__((visibility("default")))
#else
#define LAPSUM_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* ---- synchronous return codes ---------------------------------------- */
#define LAPSUM_OK 0
#define LAPSUM_EINVAL 1       /* null pointer, rows/n < 1, row_stride < n,
                                 misaligned or overlapping buffers */
#define LAPSUM_EBADK 2        /* k not finite or not in (0, n) */
#define LAPSUM_EBADALPHA 3    /* alpha not finite or outside [1e-30, 1e30] */
#define LAPSUM_EWORKSPACE 4   /* workspace NULL or smaller than required */
#define LAPSUM_ECUDA 5        /* a CUDA call or launch failed */
#define LAPSUM_ETOOLARGE 6    /* rows or n above the limits of
                                 lapsum_topk_fwd_noalloc */

/* ---- per-row status bits (asynchronous, in row_status) ---------------- */
#define LAPSUM_ROW_CERTIFIED 0x01u  /* b proven inside the final bracket */
#define LAPSUM_ROW_WIDENED 0x02u    /* first bracket missed; widened once */
#define LAPSUM_ROW_FALLBACK 0x04u   /* solved by the full-sort fallback */
#define LAPSUM_ROW_NONFINITE 0x08u  /* NaN or +-inf in the row: outputs of
                                       this row are unspecified */
#define LAPSUM_ROW_TIMEOUT 0x10u    /* a bounded device wait gave up: the
                                       row's p, b and sum f are NaN */
#define LAPSUM_ROW_OVERFLOW 0x20u   /* informational: the band outgrew its
                                       capacity (the row then took the fallback) */
#define LAPSUM_ROW_TRUNCATED 0x40u  /* sparse forward: the row has more entries
                                       with p >= eps than the capacity; its
                                       count is still the full number */
#define LAPSUM_ROW_BADARG 0x80u    /* per-row k or alpha out of range
                                      (lapsum_topk_fwd_rows): outputs NaN */

/* ---- tuning and test knobs --------------------------------------------- */
typedef struct lapsum_params {
    uint32_t sample_m;      /* localization sample size m; 0 = automatic */
    uint32_t force_path;    /* 0 = normal; OR of LAPSUM_FORCE_* (tests) */
    double z;               /* bracket half-width in binomial sigmas; 0 = 4 */
    uint64_t seed;          /* seed of the sampling generator (splitmix64) */
    int64_t band_capacity;  /* band slots per row; 0 = automatic */
    int32_t max_widen;      /* widenings before the full sort: 0 or 1;
                               negative = automatic (1) */
    int32_t spin_limit;     /* polls before a bounded device wait gives up
                               and sets LAPSUM_ROW_TIMEOUT; 0 or negative =
                               the default (2^22 polls, about a second) */
} lapsum_params;

#define LAPSUM_FORCE_NONE 0u
#define LAPSUM_FORCE_FALLBACK 1u   /* solve every row by the full-sort fallback */
#define LAPSUM_FORCE_STREAMING 2u  /* use the multi-block path even for rows
                                      that fit one block's shared memory */
/* Test knob: on every odd-numbered row, make one bounded device wait run out
 * (pair it with a small spin_limit).  A one-block row that is copied into
 * shared memory (n <= 4096) waits on a bulk-copy barrier that no copy
 * targets (when scores and p start at the same address mod 16, as the copy
 * needs).  On a streaming row numbered 1 mod 4 every filter block issues no
 * bulk copy for its first chunk and its barrier wait for that chunk runs out
 * (the block first waits, bounded, for its other copies in flight); any
 * other odd streaming row (or one with no whole chunk of 4096 scores) is
 * sent to the recovery kernel, whose first grid barrier then waits for one
 * block more than the grid holds.  Such a row ends with LAPSUM_ROW_TIMEOUT
 * and NaN outputs (p, b, sum f); on the streaming path every later row that
 * needs the recovery kernel in that call ends the same way, since the kernel
 * stops at its first timed-out barrier.
 * Even-numbered rows are solved as usual, and the next call starts afresh.
 * Nothing waits forever and no fault is raised.  Rows of 4097..16384 scores
 * on the one-block path have no such wait and are not affected. */
#define LAPSUM_FORCE_TIMEOUT 4u

/* Fill *p with the defaults (all automatic, seed 0). */
LAPSUM_API void lapsum_default_params(lapsum_params* p);

/* ---- optional per-row diagnostics (device array of `rows` entries) ----- */
typedef struct lapsum_row_stats {
    float a_L, a_R;          /* final bracket; -inf / +inf when open */
    int64_t n_L, n_R;        /* scores below a_L / at or above a_R */
    int64_t band;            /* scores inside [a_L, a_R) */
    double S_L, S_R;         /* sum exp((r - a_L)/alpha) over r < a_L and
                                sum exp((a_R - r)/alpha) over r >= a_R */
    double b;                /* the threshold */
    double sum_p;            /* sum of the written p, accumulated in fp64 */
    double sum_f;            /* sum_i f_i */
    int32_t sample_m;        /* sample size used */
    int32_t buckets;         /* band key bins used (all levels; 0 when the
                                band was sorted whole), or groups of the
                                full-sort fallback */
    uint32_t status;         /* same bits as row_status */
    int32_t reserved;
} lapsum_row_stats;

/*
 * Bytes of workspace that lapsum_topk_fwd / lapsum_topk_bwd need for this
 * shape and these parameters (params may be NULL for the defaults).  The
 * value does not depend on the device.  Returns 0 for invalid shapes.
 */
LAPSUM_API size_t lapsum_topk_workspace_size(int64_t rows, int64_t n, const lapsum_params* params);

/*
 * Forward pass: threshold b and memberships p for every row.
 *
 *   scores      in   fp32 [rows, row_stride], at least 4-byte aligned
 *   rows, n     in   rows >= 1, n >= 1, row_stride >= n (elements)
 *   k, alpha    in   0 < k < n, alpha in [1e-30, 1e30]
 *   p_out       out  fp32 [rows, row_stride] (only the first n of a row)
 *   b_out       out  fp64 [rows]  threshold b of each row
 *   sumf_out    out  fp64 [rows]  sum_i f_i of each row (may be NULL)
 *   row_status  out  uint32 [rows] LAPSUM_ROW_* bits (may be NULL)
 *   stats       out  lapsum_row_stats [rows] (may be NULL)
 *   workspace   in   device scratch of workspace_bytes bytes, >= the size
 *                    lapsum_topk_workspace_size returns; 256-byte aligned;
 *                    contents on entry are ignored; may be reused by the next
 *                    call on the same stream
 *   params      in   host pointer or NULL
 *   stream      in   cudaStream_t
 * Returns LAPSUM_OK or an error code (nothing enqueued on error).
 * Speed, not results: every pass reads and writes rows 16 bytes at a time
 * after a head of 0-3 scores, which needs scores and p_out to start at the
 * same address mod 16 (contiguous tensors of one shape always do); when they
 * do not, p is written one score at a time.
 */
LAPSUM_API int lapsum_topk_fwd(const float* scores, int64_t rows, int64_t n, int64_t row_stride,
                    double k, double alpha, float* p_out, double* b_out, double* sumf_out,
                    uint32_t* row_status, lapsum_row_stats* stats, void* workspace,
                    size_t workspace_bytes, const lapsum_params* params, void* stream);

/*
 * Sparse forward pass: the same threshold b, but instead of the dense p only
 * the entries with p_i >= eps, as (index, p_i) pairs.  Downstream top-k uses
 * need about k + O(alpha * density) such entries per row instead of n, and
 * the membership pass then writes those instead of 4n bytes per row.
 *
 *   eps         in   0 < eps <= 1 (e.g. 2^-24: every p_i below it is dropped)
 *   idx_out     out  int32 [rows, capacity]: row-local indices, row r at
 *                    r * capacity; ascending when the row takes the
 *                    one-block path (n <= 16384), in unspecified order otherwise
 *   val_out     out  fp32 [rows, capacity]: p at those indices
 *   capacity    in   entries per row of idx_out / val_out (>= 0)
 *   count_out   out  uint64 [rows]: the number of entries with p >= eps.  If it
 *                    exceeds capacity, only capacity of them are written (which
 *                    ones is unspecified) and the row gets LAPSUM_ROW_TRUNCATED
 *   workspace   in   at least lapsum_topk_sparse_workspace_size() bytes
 * The other arguments are those of lapsum_topk_fwd (there is no p_out).
 * Returns LAPSUM_OK or an error code (nothing enqueued on error).
 */
LAPSUM_API int lapsum_topk_fwd_sparse(const float* scores, int64_t rows, int64_t n, int64_t row_stride,
                                      double k, double alpha, float eps, int32_t* idx_out, float* val_out,
                                      int64_t capacity, uint64_t* count_out, double* b_out, double* sumf_out,
                                      uint32_t* row_status, lapsum_row_stats* stats, void* workspace,
                                      size_t workspace_bytes, const lapsum_params* params, void* stream);

/*
 * Batched forward with a budget and a scale per row.  The method is stated
 * for one vector with one k and one alpha (Fast LapSum technical summary,
 * section 2.1); here row r is solved with k[r] and alpha[r], read by the
 * kernels from device memory, so the values may come straight from an earlier
 * kernel or an autograd graph without a host round trip.
 *
 *   k           in   fp64 [rows], device, 8-byte aligned: 0 < k[r] < n
 *   alpha       in   fp64 [rows], device, 8-byte aligned: 1e-30 <= alpha[r] <= 1e30
 * A row whose k[r] or alpha[r] is out of range (or NaN) is not an error of the
 * call: it gets LAPSUM_ROW_BADARG and NaN outputs, the other rows are solved.
 * Every row's sample is drawn with the sample size the one-block path picks
 * for k = n/2 (the widest bracket), so a row's b can differ from that of a
 * lapsum_topk_fwd call with the same k and alpha by rounding (both are the
 * exact root to fp64 accuracy); on the streaming path (n > 16384) the sample
 * and the ranks are the same as there.
 * The other arguments, the workspace size and the per-row status are those of
 * lapsum_topk_fwd.  Returns LAPSUM_OK or an error code (nothing enqueued on
 * error).
 */
LAPSUM_API int lapsum_topk_fwd_rows(const float* scores, int64_t rows, int64_t n, int64_t row_stride,
                                    const double* k, const double* alpha, float* p_out, double* b_out,
                                    double* sumf_out, uint32_t* row_status, lapsum_row_stats* stats,
                                    void* workspace, size_t workspace_bytes, const lapsum_params* params,
                                    void* stream);

/*
 * Backward of lapsum_topk_fwd_rows: lapsum_topk_bwd with alpha[r] (fp64
 * [rows], device) for row r.  A row whose alpha[r] is out of range gets NaN
 * in grad_scores, grad_k and grad_alpha.
 */
LAPSUM_API int lapsum_topk_bwd_rows(const float* scores, const float* grad_p, const double* b, int64_t rows,
                                    int64_t n, int64_t row_stride, const double* alpha, float* grad_scores,
                                    double* grad_k, double* grad_alpha, void* workspace, size_t workspace_bytes,
                                    void* stream);

/*
 * DFTopK relaxation (Fast LapSum technical summary, section 2.3 "Relation to
 * DFTopK"): the threshold is not solved for the budget at alpha but fixed at
 * the midpoint of the k-th and (k+1)-th largest scores of the row, which is
 * the zero-temperature limit of the LapSum threshold; the memberships are the
 * same Laplace CDF around it at scale alpha, so their mass sum_i p_i is free
 * to drift away from k.  Computed as the LapSum threshold at alpha = 1e-30
 * (exactly the midpoint at fp64 resolution for fp32 scores), then one
 * membership pass at the caller's alpha.
 *
 *   k           in   integer, 1 <= k <= n - 1
 *   alpha       in   membership scale, [1e-30, 1e30]
 *   b_out       out  fp64 [rows]  the midpoint threshold
 *   sumf_out    out  fp64 [rows]  sum_i f_i at alpha (may be NULL)
 *   mass_out    out  fp64 [rows]  sum_i p_i, the drifted mass (may be NULL)
 * The other arguments, the workspace size (lapsum_topk_workspace_size) and
 * the per-row status are those of lapsum_topk_fwd.  lapsum_topk_bwd with this
 * b and alpha is NOT the gradient of this map (its threshold does not move
 * with the scores the way the budget constraint makes it move).
 * Returns LAPSUM_OK or an error code (nothing enqueued on error).
 */
LAPSUM_API int lapsum_dftopk_fwd(const float* scores, int64_t rows, int64_t n, int64_t row_stride, int64_t k,
                                 double alpha, float* p_out, double* b_out, double* sumf_out, double* mass_out,
                                 uint32_t* row_status, lapsum_row_stats* stats, void* workspace,
                                 size_t workspace_bytes, const lapsum_params* params, void* stream);

/* Workspace bytes of lapsum_topk_fwd_sparse: that of the dense forward plus,
   for rows longer than 16384 scores, 4n bytes the full-sort fallback uses in
   place of the dense p row. */
LAPSUM_API size_t lapsum_topk_sparse_workspace_size(int64_t rows, int64_t n, const lapsum_params* params);

/*
 * Backward pass (vector-Jacobian product) for the b a forward pass returned.
 *
 *   scores      in   fp32 [rows, row_stride], the forward's input
 *   grad_p      in   fp32 [rows, row_stride], upstream gradient dL/dp
 *   b           in   fp64 [rows], the forward's b_out
 *   alpha       in   the forward's alpha
 *   grad_scores out  fp32 [rows, row_stride] dL/dr
 *   grad_k      out  fp64 [rows] dL/dk = lambda (may be NULL)
 *   grad_alpha  out  fp64 [rows] dL/dalpha (may be NULL; costs two more sums
 *                    in the reduction pass).  With z_j = (r_j - b)/alpha the
 *                    threshold moves as db/dalpha = -sum f z / sum f, and
 *                    dL/dalpha = -(1/alpha) sum_j (r_j - b) grad_j.
 *   workspace   in   as for the forward (the same buffer may be passed)
 * sum_i f_i is not an input: the reduction pass forms sum g f and sum f
 * together, relative to the score nearest b, so that neither underflows.
 * Returns LAPSUM_OK or an error code (nothing enqueued on error).
 * As for the forward, scores, grad_p and grad_scores take the 16-byte path
 * when they start at the same address mod 16.
 */
LAPSUM_API int lapsum_topk_bwd(const float* scores, const float* grad_p, const double* b, int64_t rows,
                               int64_t n, int64_t row_stride, double alpha, float* grad_scores,
                               double* grad_k, double* grad_alpha, void* workspace, size_t workspace_bytes,
                               void* stream);

/*
 * Forward pass that allocates nothing and takes no workspace.  The paper has
 * no counterpart: this entry point exists for callers that cannot allocate
 * device memory when they run the operator -- an inference engine whose
 * plugins get a fixed arena, a host that has reserved all device memory for
 * its own pool, or a framework that must not risk the implicit
 * synchronisation of cudaMalloc in the middle of a step.
 *
 * Arguments, results and per-row status are those of lapsum_topk_fwd, for
 * the one-block-per-row path only:
 *   rows <= LAPSUM_NOALLOC_MAX_ROWS and n <= LAPSUM_NOALLOC_MAX_N, else
 *   LAPSUM_ETOOLARGE (nothing enqueued); LAPSUM_FORCE_STREAMING in params is
 *   rejected with LAPSUM_EINVAL.
 * Scratch: a static device array of 2 * 4 * LAPSUM_NOALLOC_MAX_ROWS + 256
 * bytes (512.25 KiB) inside the library, which every GPU that loads the
 * library holds until the process exits.  It is shared by all calls on a
 * device and keeps the last call's contents; each call clears what must start
 * at zero on its own stream.  Calls that overlap on the GPU (two streams, or
 * two host threads) race on that array and may return wrong results:
 * serialise them.
 * The first call on a device looks up the array's device address and sets
 * kernel attributes; make it before any stream capture on that device.  The
 * library keeps both for the life of the process: after cudaDeviceReset on
 * that device they are stale, so do not call the library again in that
 * process (this holds for every entry point, which cache the same per-device
 * set-up).
 * Calls no cudaMalloc, cudaFree or other allocating routine.
 */
#define LAPSUM_NOALLOC_MAX_ROWS 65536
#define LAPSUM_NOALLOC_MAX_N 16384
LAPSUM_API int lapsum_topk_fwd_noalloc(const float* scores, int64_t rows, int64_t n, int64_t row_stride,
                                       double k, double alpha, float* p_out, double* b_out,
                                       double* sumf_out, uint32_t* row_status, lapsum_row_stats* stats,
                                       const lapsum_params* params, void* stream);

/*
 * ---- sharded rows -----------------------------------------------------------
 * One long row split over G GPUs in contiguous shards (GPU g holds scores
 * [shard_lo, shard_lo + n) of a row n_total long; every GPU passes the same
 * rows, n_total, k, alpha and params).  The probabilistic bracketing of the
 * Fast LapSum technical summary (section 2.2) needs only small exchanges
 * between the GPUs, which the caller makes between the calls below (NCCL
 * through torch.distributed, for instance); no call waits on another GPU:
 *
 *   1. lapsum_shard_fwd_sample      writes x_sample, x_hist
 *      SUM-reduce x_sample and x_hist over the GPUs, in place (int32 or
 *      uint32 sums: every sample slot is non-zero on at most one GPU)
 *   2. lapsum_shard_fwd_filter      reads them; writes x_meta, x_fpart, x_band
 *      GATHER x_meta, x_fpart, x_band of all GPUs, GPU-major, into g_meta,
 *      g_fpart, g_band (G times the size of each)
 *   3. lapsum_shard_fwd_finish      every GPU solves the same band for the
 *      same b, then writes the memberships of its shard
 *
 * The sample is the one a single GPU would draw for the whole row.  A row the
 * band does not certify (its row_status lacks LAPSUM_ROW_CERTIFIED) is not
 * widened here: the caller solves it again from the whole row.  The workspace
 * keeps state from call 1 to call 3 and must not be shared meanwhile.
 *
 * Backward (analytic VJP, section 2.1): lapsum_shard_bwd_partials writes this
 * shard's reduction partials into x_parts; GATHER them GPU-major into g_parts;
 * lapsum_shard_bwd_finish forms lambda (and dL/dalpha when with_alpha was set
 * in the partials call) from all of them and writes dL/dr of its shard.
 *
 * Exchange buffers are device memory, 16-byte aligned, of the sizes
 * lapsum_shard_layout_get returns (per GPU; the gathered ones G times that).
 */
typedef struct lapsum_shard_layout {
    int32_t sample_m;        /* localization sample size */
    int32_t reserved;
    int64_t band_cap;        /* band slots per row and GPU */
    size_t sample_bytes;     /* x_sample: uint32 [rows][sample_m]  (summed) */
    size_t hist_bytes;       /* x_hist:   uint32 [rows][2048]      (summed) */
    size_t meta_bytes;       /* x_meta:   uint32 [rows][8]         (gathered) */
    size_t fpart_bytes;      /* x_fpart:  [rows][4096] x 32 bytes  (gathered) */
    size_t band_bytes;       /* x_band:   fp32 [rows][band_cap]    (gathered) */
    size_t parts_bytes;      /* x_parts:  [rows][4096] x 48 bytes  (gathered) */
    size_t workspace_bytes;  /* workspace of the forward and backward calls */
} lapsum_shard_layout;

/* Sizes for rows of n_total scores (zeros for an invalid shape). */
LAPSUM_API void lapsum_shard_layout_get(int64_t rows, int64_t n_total, const lapsum_params* params,
                                        lapsum_shard_layout* out);

LAPSUM_API int lapsum_shard_fwd_sample(const float* scores, int64_t rows, int64_t n, int64_t row_stride,
                                       int64_t shard_lo, int64_t n_total, double k, double alpha,
                                       uint32_t* x_sample, uint32_t* x_hist, void* workspace,
                                       size_t workspace_bytes, const lapsum_params* params, void* stream);

LAPSUM_API int lapsum_shard_fwd_filter(const float* scores, int64_t rows, int64_t n, int64_t row_stride,
                                       int64_t shard_lo, int64_t n_total, double k, double alpha,
                                       const uint32_t* x_sample, const uint32_t* x_hist, uint32_t* x_meta,
                                       void* x_fpart, float* x_band, void* workspace, size_t workspace_bytes,
                                       const lapsum_params* params, void* stream);

/* p_out: fp32 [rows, row_stride], this shard's memberships; b_out, sumf_out:
   fp64 [rows], the same on every GPU; row_status as for lapsum_topk_fwd. */
LAPSUM_API int lapsum_shard_fwd_finish(const float* scores, int64_t rows, int64_t n, int64_t row_stride,
                                       int64_t shard_lo, int64_t n_total, double k, double alpha, int world,
                                       const uint32_t* g_meta, const void* g_fpart, const float* g_band,
                                       float* p_out, double* b_out, double* sumf_out, uint32_t* row_status,
                                       void* workspace, size_t workspace_bytes, const lapsum_params* params,
                                       void* stream);

LAPSUM_API int lapsum_shard_bwd_partials(const float* scores, const float* grad_p, const double* b, int64_t rows,
                                         int64_t n, int64_t row_stride, double alpha, int with_alpha,
                                         void* x_parts, void* stream);

/* grad_scores: this shard's dL/dr; grad_k, grad_alpha (may be NULL): fp64
   [rows], the same on every GPU. */
LAPSUM_API int lapsum_shard_bwd_finish(const float* scores, const float* grad_p, const double* b, int64_t rows,
                                       int64_t n, int64_t row_stride, double alpha, int world,
                                       const void* g_parts, float* grad_scores, double* grad_k,
                                       double* grad_alpha, void* workspace, size_t workspace_bytes,
                                       void* stream);

/* Text of the CUDA error behind the last LAPSUM_ECUDA returned on the
   calling host thread ("no error" if none). */
LAPSUM_API const char* lapsum_last_cuda_error(void);

/* Static English text for a return code. */
LAPSUM_API const char* lapsum_status_string(int code);

/* Number of kernels this library has launched in this process (all devices,
   all streams).  Used to count launches inside a timed region. */
LAPSUM_API uint64_t lapsum_launch_count(void);

/*
 * Kernel timing without a profiler.  While enabled (on != 0), every kernel
 * launch is bracketed by two CUDA events recorded on its stream; this adds two
 * event records per launch and nothing else.  lapsum_trace_collect waits for
 * the recorded events, writes a JSON object
 *     {"<kernel>": [launches, total_milliseconds], ...}
 * into buf (truncated to len-1 bytes, NUL-terminated), clears the record, and
 * returns the number of bytes written, or -1 if a CUDA call fails.  With
 * buf == NULL it returns the size needed and keeps the record.  Both
 * functions are thread-safe.
 */
LAPSUM_API void lapsum_trace_enable(int on);
LAPSUM_API int lapsum_trace_collect(char* buf, size_t len);

#ifdef __cplusplus
}
#endif

#endif /* LAPSUM_TOPK_H */
