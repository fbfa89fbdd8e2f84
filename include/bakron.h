/*
 * bakron.h -- C ABI of the B200 (sm_100a) BaKron two-sided adaptive-rounding
 * solver.
 *
 * Method: "BaKron: Efficient Quantization with Kronecker-Factored Hessians"
 * (arXiv 2608.06291; called "FastKron" in the arXiv abstract).  A weight
 * matrix W (m x n; row i = output channel, column j = input channel) is
 * rounded to a per-row integer grid so as to keep the proxy loss
 *     l(V) = vec(W-V)^T (A (x) B) vec(W-V) = tr((W-V)^T B (W-V) A)
 * small, where A (n x n, input side) and B (m x m, output side) are the SPD
 * Kronecker factors of the Hessian.  GPTQ applied to vec(W) with that Hessian
 * (the paper's Algorithm 2) is reorganised into anti-diagonal rounding steps
 * and batched rank updates (Proposition 3.1, Theorem 3.2, Algorithm 6), for
 * O(m+n) sequential depth and O(mn(m+n)) work.
 *
 * Conventions for every entry point
 *   - All matrices are dense, row-major, float32 unless stated.  Pointers
 *     named *_dev are CUDA device pointers, *_host are host pointers.  Every
 *     device pointer must be 16-byte aligned (else BAKRON_ERR_ALIGNMENT).
 *   - The caller owns every buffer.  The library never allocates device or
 *     pinned memory buffers, never frees or retains caller memory; all scratch
 *     lives in the caller's workspace, whose size the *_workspace_size query
 *     gives.  (Exceptions, all driver-side: bakron_solve_noalloc's fixed
 *     scratch array, reserved on a device by the first call there; and in
 *     CUDA graph mode a private stream per calling thread and the cached
 *     executable graphs.)
 *   - Calls are stream-ordered and asynchronous on `stream` (a cudaStream_t;
 *     NULL = legacy default stream).  Argument errors are returned at once and
 *     nothing is enqueued.  Errors found on the device (non-SPD pivot,
 *     non-finite input, factor with non-positive diagonal, timed-out wait) are
 *     recorded in a status block in the first 256 bytes of the workspace;
 *     every call clears that block (stream-ordered) before its kernels run, so
 *     bakron_get_status() reports the latest call on that workspace.  A fresh
 *     workspace needs no initialisation.
 *   - A workspace must not be used by two calls that overlap on the GPU.
 *     Distinct workspaces on distinct streams are independent.
 *   - The library uses the current CUDA device; buffers must live on it.
 */
#ifndef BAKRON_H
#define BAKRON_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *bakron_stream_t; /* same type as cudaStream_t */

typedef enum {
    BAKRON_OK = 0,
    BAKRON_ERR_INVALID_ARG = 1,    /* bad size, null pointer, bad grid, bad config */
    BAKRON_ERR_ALIGNMENT = 2,      /* a device pointer is not 16-byte aligned */
    BAKRON_ERR_NOT_SPD = 3,        /* (device) a Cholesky pivot was <= 0 or not finite */
    BAKRON_ERR_NONFINITE = 4,      /* (device) W, A or B holds NaN or Inf */
    BAKRON_ERR_DEVICE_TIMEOUT = 5, /* (device) a bounded wait gave up */
    BAKRON_ERR_CUDA = 6,           /* a CUDA runtime/driver call failed */
    BAKRON_ERR_WORKSPACE = 7,      /* workspace null or smaller than the query */
    BAKRON_ERR_BAD_FACTOR = 8      /* (device) LA or LB has a non-positive or non-finite diagonal */
} bakron_status_t;

/* Fixed per-row integer grid (the base quantizer; the method is modular in
 * it, per the arXiv abstract).  Row i has step s_i and codes in [qmin, qmax];
 * the rounding decision is clamp(rint(Wt_ij / s_i)) in fp32, ties to even.
 *   bits        2..8.
 *   qmin,qmax   both 0 selects the symmetric range qmax = 2^(bits-1)-1,
 *               qmin = -qmax; otherwise -128 <= qmin < qmax <= 127.
 *   row_scale   NULL: steps computed on the device (below).  Non-NULL: device
 *               pointer to m positive finite steps, used as given.
 *   shrink_grid 0: s_i = max_j |W_ij| / qmax (fp32, IEEE division; a row of
 *               zeros gets s_i = 1).  G in [2, 1024]: s_i is searched for the
 *               least round-to-nearest error of row i ("per-row scaling factor
 *               (shrink) up to factor 2, MSE search", the review's list of free
 *               parameters): over c_k = 1 - fp32(k/2) / fp32(G-1), k = 0..G-1,
 *               the step fp32(fp32(c_k * absmax_i) / qmax) whose error
 *               sum_j (W_ij - s q_ij)^2, q_ij = clamp(rint(fp32(W_ij / s))),
 *               summed in FP64, is smallest (the first k on equal errors).
 *               Ignored when row_scale is given. */
typedef struct {
    int32_t bits;
    int32_t qmin;
    int32_t qmax;
    const float *row_scale;
    int32_t shrink_grid;
} bakron_quantizer_t;

/* Solver configuration (NULL = defaults; zero fields take defaults).
 * The environment can change the defaults of five fields: BAKRON_LEAF (0..8),
 * BAKRON_GEMM (0..1), BAKRON_TIMEOUT_MS (1..600000), BAKRON_GRAPH (0..1,
 * ignored when profile = 1) and BAKRON_FUSE (1..65535, the default
 * fuse_width); a non-zero field set by the caller wins.  A
 * variable that is set but not an integer in its range makes every call that
 * reads a config return BAKRON_ERR_INVALID_ARG.
 *   tile        side T of the square tiles whose anti-diagonals the recursion
 *               cuts on: 128 (default; the only supported value).
 *   gemm        0 = tcgen05 tensor-core 3xTF32 band GEMMs (default),
 *               1 = FP32 CUDA-core band GEMMs (cross-check).
 *   use_graph   1: capture the solve's launches for this argument set
 *               (every pointer, size, quantizer and config field, device) into
 *               a CUDA graph on the first call, on a private stream of the
 *               calling thread, and replay it on `stream` in later calls
 *               (the programmatic launches become programmatic graph edges;
 *               a replay reads the buffers' current contents).  Up to 64
 *               graphs are kept per process, oldest dropped first.  Not with
 *               profile = 1 (BAKRON_ERR_INVALID_ARG).  0: launch directly.
 *   timeout_ms  limit for device-side bounded waits (default 200).
 *   wt_out      optional device pointer, m x n fp32: if not NULL it receives
 *               every entry's pre-rounding value Wt_ij (diagnostics). */
typedef struct {
    int32_t tile;
    int32_t gemm;
    int32_t use_graph;
    int32_t timeout_ms;
    float *wt_out;
    int32_t profile;  /* 1: time every kernel class with CUDA events on `stream`;
                         the call then synchronises `stream` before returning and
                         the durations are read with bakron_get_profile(). */
    int32_t leaf;     /* leaf sweep structure: 0 = default (6); 1 = each tile as
                         2 x 2 sub-tiles of 64 swept by the whole CTA; 2 = one
                         anti-diagonal sweep over the whole 128 x 128 tile; 3 =
                         4 x 4 sub-tiles of 32, each swept by three warps; 4 =
                         2 x 2 sub-tiles of 64, each swept by six warps; 5 = as
                         3 with each tile on a cluster of four CTAs, one per
                         row block of sub-tiles; 6 = as 5 with a fourth warp
                         per CTA forming the older product terms of the next
                         sub-tile during each sweep; 7 = as 6 with the two
                         tile diagonals of every width-2 range of the
                         recursion in one launch: the second diagonal's tiles
                         wait (bounded, device flags) for their neighbours on
                         the first and apply that node's updates themselves;
                         8 = each CTA of the cluster rounds its 32-row strip
                         in one continuous sweep, 48 steps behind the CTA
                         above (no sub-tile phases; the CTA above pushes its
                         rounded residuals and its progress into the CTA
                         below, bounded waits)
                         (bakron_tune_leaf picks one by measurement). */
    int32_t b_identity; /* 1: B = I (one-sided GPTQ with Hessian A, the case the
                           two-sided solve reduces to when B = I).  LB_dev may be
                           NULL and is not read; rows are independent, so the
                           solve runs over 128-column blocks (the recursion over
                           column blocks with a one-sided leaf and update)
                           instead of tile diagonals.  The leaf and gemm
                           fields are ignored (the update always runs on the
                           tensor cores, 3xTF32). */
    int32_t fuse_width; /* recursion nodes at most this many tile diagonals
                           wide run both band products in one launch, one CTA
                           per target tile, with X kept in tensor memory
                           (stage 1 and stage 2 fused); wider nodes run them as
                           two launches.  0 = default (2), 1 = never fuse,
                           2..65535 = that width.  Ignored with gemm = 1 and on
                           the one-sided path. */
    int32_t self_test_omit; /* self-test of the bounded waits of leaf structure
                               7 only; 0 = off.  v > 0: the first-diagonal tile
                               with row-major tile index v - 1 never raises its
                               flag, so its neighbours' waits run out after
                               timeout_ms and record BAKRON_ERR_DEVICE_TIMEOUT
                               (the results are then not the solve's). */
} bakron_config_t;

/* Per-kernel-class device time of the latest profiled bakron_solve on the
 * calling host thread (sums of CUDA-event intervals around each launch).  On
 * the one-sided path (b_identity = 1) the leaf fields count the column-block
 * leaves and the stage 1 fields the tensor-core updates; stage 2 stays 0. */
typedef struct {
    double prep_ms, leaf_ms, stage1_ms, stage2_ms, total_ms;
    int64_t prep_launches, leaf_launches, stage1_launches, stage2_launches;
    double fused_ms;        /* nodes whose two band products ran as one launch */
    int64_t fused_launches;
} bakron_profile_t;
bakron_status_t bakron_get_profile(bakron_profile_t *out);

/* One launch of the latest profiled bakron_solve on the calling host thread,
 * in launch order: kind 0 prep (the four preparation kernels together), 1 leaf
 * sweep of tile diagonal k, 2 / 3 stage 1 / stage 2 band product of the
 * recursion node over tile diagonals [k, k+l) split at k+h, 4 both band
 * products of such a node in one fused launch; ms its
 * CUDA-event interval; flops the algorithmic FLOPs of a band product (2 T^3
 * per 128 x 128 x 128 tile product, both products for kind 4; 0 for other
 * kinds).  One-sided path:
 * kind 1 is the leaf of column block k, kind 2 the update of column blocks
 * [k+h, k+l) by blocks [k, k+h). */
typedef struct {
    int32_t kind, k, h, l;
    double ms, flops;
    double structural_flops; /* flops without the structurally zero upper
                                triangles of the diagonal factor tiles */
} bakron_profile_launch_t;
/* Copies min(count, cap) records to `out` (may be NULL) and returns count. */
int64_t bakron_get_profile_launches(bakron_profile_launch_t *out, int64_t cap);

/* ------------------------------------------------------------------ gram */
/* The Kronecker factor from calibration samples, the step before
 * bakron_factor (the pages build A and B as expectations of a a^T over
 * activation / gradient samples, regularised by a multiple of the mean
 * diagonal: "Assumptions & free parameters", Gram matrix regularisation):
 *   A_dev (d x d) <- X^T X / N + damping * mean_i (X^T X / N)_ii * I
 * for X_dev (N x d, row-major samples).  The product runs on the tensor cores
 * in 3xTF32 (lower tiles), each FP32 sum / N rounded once; A is written in
 * full (symmetric).  damping >= 0.  Device errors: BAKRON_ERR_NONFINITE (X).
 * Workspace: bakron_gram_workspace_size(N, d) bytes (X^T split, the product). */
size_t bakron_gram_workspace_size(int64_t N, int64_t d);
bakron_status_t bakron_gram(const float *X_dev, int64_t N, int64_t d, float damping, float *A_dev, void *ws_dev,
                            size_t ws_bytes, bakron_stream_t stream);

/* ---------------------------------------------------------------- factor */
/* Bytes of workspace bakron_factor needs for factors of sizes n and m. */
size_t bakron_factor_workspace_size(int64_t n, int64_t m);

/* Lower Cholesky factors of the inverted Hessian factors ("What carries the
 * argument": L^(A), L^(B) with L L^T = A^{-1}, B^{-1}):
 *   LA_dev (n x n) <- chol(A^{-1}),  LB_dev (m x m) <- chol(B^{-1}),
 * both lower triangular with positive diagonal; the strict upper triangle is
 * written with zeros.  A_dev (n x n) and B_dev (m x m) are SPD; only their
 * lower triangles are read.  Computed in FP64 (blocked Cholesky of the
 * reversed matrix J A J with the trailing updates as FP64 GEMMs, recursive
 * triangular inverse whose merges are FP64 GEMMs, L = J C^{-T} J), rounded
 * to fp32.  Either side may be skipped by passing n = 0 (resp. m = 0) and
 * NULL pointers.  Device errors: BAKRON_ERR_NOT_SPD, BAKRON_ERR_NONFINITE. */
bakron_status_t bakron_factor(const float *A_dev, int64_t n, const float *B_dev, int64_t m,
                              float *LA_dev, float *LB_dev, void *ws_dev, size_t ws_bytes,
                              bakron_stream_t stream);

/* ----------------------------------------------------------------- solve */
/* Bytes of workspace bakron_solve needs for an m x n solve. */
size_t bakron_solve_workspace_size(int64_t m, int64_t n, const bakron_config_t *cfg);

/* The BaKron solve (Algorithm 6 with Proposition 3.1's updates).
 *   W_dev      m x n weights (read only).
 *   LA_dev     n x n raw lower factor of A^{-1} (as bakron_factor writes it).
 *   LB_dev     m x m raw lower factor of B^{-1}.  The solver normalises both
 *              to unit diagonal itself; only lower triangles are read.
 *   q          grid (see bakron_quantizer_t); host pointer.
 *   V_dev      m x n out: quantised weights, V_ij = s_i * codes_ij (fp32).
 *   codes_dev  m x n out: int8 codes.
 *   scales_dev m out: the steps s_i used.
 * Result: the unique code matrix of Theorem 3.2's intended output, computed
 * with FP32 leaf arithmetic and 3xTF32 (or FP32) band updates.  m, n >= 1.
 * Device errors: BAKRON_ERR_NONFINITE (W), BAKRON_ERR_BAD_FACTOR,
 * BAKRON_ERR_DEVICE_TIMEOUT. */
bakron_status_t bakron_solve(const float *W_dev, int64_t m, int64_t n, const float *LA_dev,
                             const float *LB_dev, const bakron_quantizer_t *q, float *V_dev,
                             int8_t *codes_dev, float *scales_dev, void *ws_dev, size_t ws_bytes,
                             const bakron_config_t *cfg, bakron_stream_t stream);

/* Leaf structure picked by measurement (the schedule's leaf size: 4 x 4
 * sub-tiles of 32, 2 x 2 of 64, or the whole 128 x 128 tile per sweep; one
 * CTA or a cluster of four per tile).  Runs
 * bakron_solve on the caller's problem once per structure after one warm-up
 * solve, timing each with CUDA events on `stream` (the call synchronises
 * `stream`), and writes the fastest structure (a bakron_config_t.leaf value,
 * 1..8) to *leaf_out and the eight times in ms to ms_out[0..7] (leaf 1..8;
 * ms_out may be NULL).  Arguments as for bakron_solve; cfg->leaf is ignored
 * and cfg->profile must be 0.  V, codes and scales hold the last solve's
 * results (all structures give the same codes up to rounding ties).  Device
 * errors are read with bakron_get_status as after bakron_solve. */
bakron_status_t bakron_tune_leaf(const float *W_dev, int64_t m, int64_t n, const float *LA_dev,
                                 const float *LB_dev, const bakron_quantizer_t *q, float *V_dev,
                                 int8_t *codes_dev, float *scales_dev, void *ws_dev, size_t ws_bytes,
                                 const bakron_config_t *cfg, bakron_stream_t stream, int32_t *leaf_out,
                                 double *ms_out);

/* Several independent solves (for instance the weight matrices of a model's
 * layers), solve i enqueued on streams[i % nstreams].  One solve keeps few SMs
 * busy while its leaf sweeps run (one CTA per tile of a tile diagonal), so
 * solves on different streams overlap.  Every item needs its own workspace
 * (and its own outputs); all items share the grid and the config.  All
 * arguments are checked before anything is enqueued: the first invalid item's
 * status is returned and nothing runs.  cfg->profile must be 0. */
typedef struct {
    const float *W_dev;
    int64_t m, n;
    const float *LA_dev, *LB_dev;
    float *V_dev;
    int8_t *codes_dev;
    float *scales_dev;
    void *ws_dev;
    size_t ws_bytes;
} bakron_batch_item_t;
bakron_status_t bakron_solve_batch(const bakron_batch_item_t *items, int32_t count, const bakron_quantizer_t *q,
                                   const bakron_config_t *cfg, const bakron_stream_t *streams, int32_t nstreams);

/* Bytes of device workspace bakron_solve_host needs (solve workspace plus
 * device staging for W, LA, LB, V, codes and scales). */
size_t bakron_solve_host_workspace_size(int64_t m, int64_t n, const bakron_config_t *cfg);

/* bakron_solve on HOST buffers: copies W_host, LA_host, LB_host to device
 * staging inside ws_dev, solves, and copies V, codes and scales back, all
 * ordered on `stream` (pinned host memory makes the copies asynchronous;
 * the results are valid after the stream is synchronised).  In the
 * two-sided solve each 128-row block of V and codes is copied back as soon
 * as the tile diagonal that completes it has been rounded, on a copy stream
 * of the library's own that `stream` waits for at the end, so those copies
 * overlap the rest of the solve; the launches are then always direct
 * (cfg->use_graph is ignored).  q->row_scale, if not NULL, is a HOST pointer
 * here. */
bakron_status_t bakron_solve_host(const float *W_host, int64_t m, int64_t n, const float *LA_host,
                                  const float *LB_host, const bakron_quantizer_t *q, float *V_host,
                                  int8_t *codes_host, float *scales_host, void *ws_dev,
                                  size_t ws_bytes, const bakron_config_t *cfg,
                                  bakron_stream_t stream);

/* ------------------------------------------------ allocation-free solve */
/* No counterpart in the paper: this is a service of the library, not a step
 * of the method.
 *
 * Some callers may not allocate device memory at the moment they need a
 * solve: plug-ins whose execution hook must not allocate (an inference
 * engine's enqueue step, for example), and services that reserve all their
 * memory at start-up and forbid allocation afterwards so that their footprint
 * stays fixed.  They cannot obtain the workspace bakron_solve asks for.  This
 * entry point runs the same solve with its workspace in a device array that
 * the library itself declares: BAKRON_NOALLOC_SCRATCH_BYTES bytes per GPU,
 * held until the process exits.
 *
 *   Arguments as bakron_solve, without ws/ws_bytes.  The problem must fit
 *   the array: bakron_solve_workspace_size(m, n, cfg) <=
 *   BAKRON_NOALLOC_SCRATCH_BYTES (true for any m, n <= 512); larger problems
 *   return BAKRON_ERR_WORKSPACE and nothing is enqueued.  cfg->profile must be
 *   0 (BAKRON_ERR_INVALID_ARG otherwise).  The kernels are always launched
 *   directly: cfg->use_graph and BAKRON_GRAPH are ignored here, since graph
 *   capture and instantiation make the driver allocate.
 *   device_status_host: NULL keeps the call asynchronous (device-detected
 *   errors are then not reported); otherwise the call synchronises `stream`
 *   and stores the device status (a bakron_status_t value) there, and a
 *   `stream` that is being captured into a graph is refused with
 *   BAKRON_ERR_INVALID_ARG before anything is enqueued.
 *   Set-up on the first call on each device: the library looks up the array's
 *   device address (once per device, with that device current).  Under CUDA's
 *   default lazy module loading that first call is also when the driver loads
 *   the array's code module and reserves the array on that device (at library
 *   load only with CUDA_MODULE_LOADING=EAGER), so it can fail with
 *   BAKRON_ERR_CUDA if the device's memory is already full.  Make one call on
 *   every device at start-up, before the caller fixes its memory and before
 *   any stream capture.  After that the library calls no cudaMalloc or
 *   cudaFree here.
 *   Every call on a device shares the one array and leaves its contents
 *   behind; the solve clears what must start at zero.  Calls that overlap on
 *   the GPU (other streams, other host threads) race on the array: issue them
 *   one after another. */
#define BAKRON_NOALLOC_SCRATCH_BYTES ((size_t)16 << 20)
bakron_status_t bakron_solve_noalloc(const float *W_dev, int64_t m, int64_t n, const float *LA_dev,
                                     const float *LB_dev, const bakron_quantizer_t *q, float *V_dev,
                                     int8_t *codes_dev, float *scales_dev, const bakron_config_t *cfg,
                                     bakron_stream_t stream, int32_t *device_status_host);

/* ------------------------------------------------------------ proxy loss */
/* Bytes of workspace bakron_proxy_loss needs: the status block, TF32 hi / lo
 * parts of W - V (both orientations), A and B padded to whole 128 x 128
 * tiles, the two products (fp32) and 592 FP64 partial sums; about
 * 4 (6 Mp Np + 2 Mp^2 + 2 Np^2) bytes, Mp, Np = m, n rounded up to 128. */
size_t bakron_proxy_loss_workspace_size(int64_t m, int64_t n);

/* Proxy loss l = tr((W-V)^T B (W-V) A) = ||B^{1/2}(V-W)A^{1/2}||_F^2
 * (Corollary 3.4's distortion; the review's "||vec(W)-vec(V)||_H^2",
 * H = A (x) B).  W_dev, V_dev m x n; A_dev n x n (symmetric: its rows serve as
 * the columns of A); B_dev m x m.  Computed as sum_ij (B E)_ij (E A)_ij,
 * E = W - V: both products on the tensor cores in 3xTF32 (about FP32
 * accuracy), the elementwise products and their sum in FP64, each of 592
 * fixed shares of the entries summed in index order and the shares added in
 * index order, so repeated calls give bit-identical results.  The result is
 * written to *out_dev (a device double) and, if out_host is not NULL, also
 * to *out_host, in which case the call synchronises `stream`.  The
 * workspace must be 1024-byte aligned. */
bakron_status_t bakron_proxy_loss(const float *W_dev, const float *V_dev, const float *A_dev,
                                  const float *B_dev, int64_t m, int64_t n, double *out_dev,
                                  double *out_host, void *ws_dev, size_t ws_bytes,
                                  bakron_stream_t stream);

/* ---------------------------------------------------------- diagnostics */
/* Synchronises `stream` and returns the first device-detected error of the
 * latest call on this workspace (BAKRON_OK if none), then clears it. */
bakron_status_t bakron_get_status(void *ws_dev, size_t ws_bytes, bakron_stream_t stream);

/* Failure-detection self-test: launches one thread that waits, with the same
 * bounded-wait helper and deadline as the band-product kernels, on an
 * mbarrier that nothing ever completes; after timeout_ms (1..10000) it gives
 * up, records BAKRON_ERR_DEVICE_TIMEOUT in the status word at the start of
 * ws_dev (>= 256 bytes, 16-byte aligned; cleared first) and returns, so the
 * context stays usable.  Asynchronous on `stream`: read the result with
 * bakron_get_status.  Returns BAKRON_ERR_INVALID_ARG for a timeout out of
 * range, BAKRON_ERR_WORKSPACE / _ALIGNMENT for a bad workspace. */
bakron_status_t bakron_selftest_wait_timeout(int32_t timeout_ms, void *ws_dev, size_t ws_bytes,
                                             bakron_stream_t stream);

/* Failure-detection self-test of the band-product kernel's abort path: runs
 * the stage-1 band kernel (the tcgen05 3xTF32 product, two CTAs) on a small
 * problem laid out in ws_dev with its copy-issuing thread told to issue
 * nothing, so the MMA issuer's and the epilogue's bounded waits run out after
 * timeout_ms (1..10000).  The kernel then takes the path a real timeout takes:
 * records BAKRON_ERR_DEVICE_TIMEOUT in the status word at the start of ws_dev
 * (where = 2001 for the MMA issuer, 3001 for the epilogue; cleared first),
 * stops, drains what it issued (nothing), frees its tensor memory and exits,
 * leaving the context usable.  ws_dev: at least
 * bakron_selftest_band_abort_workspace_size() bytes, 16-byte aligned; its
 * contents are not read.  Asynchronous on `stream`: read the result with
 * bakron_get_status. */
size_t bakron_selftest_band_abort_workspace_size(void);
bakron_status_t bakron_selftest_band_abort(int32_t timeout_ms, void *ws_dev, size_t ws_bytes,
                                           bakron_stream_t stream);

/* Static description of a status code. */
const char *bakron_status_string(bakron_status_t status);

/* Schedule statistics of an m x n solve with the given config: number of
 * recursion nodes, leaf launches, and the algorithmic update FLOPs (2 x the
 * structurally non-zero multiply-adds of the band products over the tile
 * cut; the leaves' in-tile work excluded).  With cfg->b_identity = 1 they
 * describe the one-sided schedule (column blocks; its updates are counted as
 * stage 1, stage 2 is 0).  Host only; enqueues nothing. */
typedef struct {
    int64_t tiles_m, tiles_n, tile_diagonals;
    int64_t nodes, leaves;
    double update_flops;   /* algorithmic (tile-dense) FLOPs of all band products */
    double stage1_flops, stage2_flops;
    double structural_flops; /* 2 x the structurally non-zero multiply-adds of
                                all band products: a product with the factor
                                tile on the diagonal (lower triangular) counts
                                T^2 (T+1)/2 of them instead of T^3 */
    double leaf_update_flops; /* leaf structure 7: FLOPs of the width-2 nodes'
                                 updates formed inside the leaf launches (2 T^3
                                 per neighbour product); 0 otherwise */
} bakron_plan_stats_t;
bakron_status_t bakron_plan_stats(int64_t m, int64_t n, const bakron_config_t *cfg,
                                  bakron_plan_stats_t *out);

/* Library version string. */
const char *bakron_version(void);

#ifdef __cplusplus
}
#endif
#endif /* BAKRON_H */
