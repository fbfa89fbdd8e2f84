// kernels.cuh -- launch interfaces between the C-ABI layer and the kernels.
#pragma once

#include <cuda.h>

#include "common.cuh"

namespace bakron {

struct LeafArgs {
    const float *LA32, *LB32, *scales;
    float *Wt, *Dhi, *Dlo, *V;
    int8_t *codes;
    int64_t m, n, Mp, Np;
    int Mt, Nt, qmin, qmax;
    DeviceStatus *st;
    float *wt_out;  // optional m x n pre-rounding values
    // two tile diagonals per launch (leaf structure 7)
    float *Rx;          // Mp x Np: each first-diagonal tile's in-tile R (read by its right neighbour)
    int32_t *flags;     // Mt x Nt: CTAs of a first-diagonal tile that have published their outputs
    int32_t *tickets;   // one counter per launch: clusters in the order they started
    int timeout_ms;     // limit of the bounded waits on flags
    int omit_flag;      // self-test only: first-diagonal tile (linear index + 1) that never publishes
};

// Operands of the band products.  Stage 1: A = LtA (Np x Np), B = Delta
// (Mp x Np), out = X^T (Np x Mp, hi/lo).  Stage 2: A = LtB (Mp x Mp),
// B = X^T (Np x Mp), out = Wt (Mp x Np) -= D.
struct GemmArgs {
    const float *Ahi, *Alo, *Bhi, *Blo;
    int64_t lda, ldb;    // row strides (elements) of A and B
    float *out_hi, *out_lo;  // stage 1 outputs (ld = ldo)
    float *out_acc;          // stage 2 output (ld = ldo), out -= D
    int64_t ldo;
    DeviceStatus *st;
    int timeout_ms;
    int test_no_tma;  // self-test only: the producer issues no copies, so the waits run out
};

cudaError_t launch_prep(const float *W, int64_t m, int64_t n, const float *LA, const float *LB, int qmin,
                        int qmax, const float *user_scales, int shrink_grid, float *scales, const SolveLayout &L,
                        char *ws, cudaStream_t stream);

cudaError_t leaf_configure();
cudaError_t launch_leaf(const LeafArgs &p, int K, int variant, cudaStream_t stream);
// Leaf with one tile per cluster of four CTAs (leaf_cluster.cu); overlap:
// a fourth warp forms the older product terms during the sweeps.
cudaError_t leaf_cluster_configure();
cudaError_t launch_leaf_cluster(const LeafArgs &p, int K, int I_lo, int tiles, bool overlap, cudaStream_t stream);
// Tile diagonals K and K+1 in one launch (leaf structure 7): ticket counter
// `slot`; the second diagonal's clusters wait for their neighbours' flags.
cudaError_t launch_leaf_pair(const LeafArgs &p, int K, int slot, cudaStream_t stream);

// FP32 CUDA-core band products (reference kernels for the tensor-core path).
cudaError_t launch_band_simt(int stage, const NodeParams &np, const GemmArgs &g, cudaStream_t stream);

// tcgen05 3xTF32 band products.  The TMA descriptors of a stage's four
// operand parts depend only on the workspace, so they are encoded once per
// solve.
struct TcMaps {
    CUtensorMap a_hi, a_lo, b_hi, b_lo;  // operands, boxes of 128 rows x 32 fp32
    CUtensorMap o0, o1;                  // outputs: stage 1 X^T hi / lo; stage 2 Wt (o0 only)
};
cudaError_t band_tc_configure();
bool make_tc_maps(int stage, int Mt, int Nt, const GemmArgs &g, TcMaps *maps);
cudaError_t launch_band_tc(int stage, const NodeParams &np, const GemmArgs &g, const TcMaps &maps,
                           cudaStream_t stream);

// Both band products of a node in one launch (band_fused.cu): m1 = the
// stage-1 maps (LtA, Delta), m2 = the stage-2 maps (LtB, output Wt).
cudaError_t band_fused_configure();
cudaError_t launch_band_fused(const NodeParams &np, const GemmArgs &g, const TcMaps &m1, const TcMaps &m2,
                              cudaStream_t stream);

// One-sided (B = I) path: the leaf over a 128-column block and the update.
cudaError_t leaf_gptq_configure();
cudaError_t launch_leaf_gptq(const LeafArgs &p, int Jb, cudaStream_t stream);
bool make_gptq_maps(const GemmArgs &g, int64_t Mp, int64_t Np, TcMaps *m);
cudaError_t launch_gptq_tc(const NodeParams &np, const GemmArgs &g, const TcMaps &maps, cudaStream_t stream);

// Gram matrix G = X^T X on the tensor cores (lower tiles), see band_tc.cu.
bool make_gram_maps(const float *xt_hi, const float *xt_lo, float *G, int64_t Dp, int64_t Ns, TcMaps *m);
cudaError_t launch_gram_tc(const NodeParams &np, const GemmArgs &g, const TcMaps &maps, cudaStream_t stream);
cudaError_t launch_gram_prep(const float *X, int64_t N, int64_t d, int64_t Dp, int64_t Ns, float *xt_hi,
                             float *xt_lo, DeviceStatus *st, cudaStream_t stream);
cudaError_t launch_gram_finish(const float *G, int64_t d, int64_t Dp, int64_t N, float damping, float *A,
                               cudaStream_t stream);

// Full GEMM tiles on the tensor cores (band_tc.cu, stage 5): D = A B^T.
bool make_full_maps(const float *a_hi, const float *a_lo, const float *b_hi, const float *b_lo, float *D, int64_t Mo,
                    int64_t No, int64_t K, TcMaps *m);
cudaError_t launch_full_tc(int64_t Mo, int64_t No, int64_t K, const GemmArgs &g, const TcMaps &maps,
                           cudaStream_t stream);

// Proxy loss tr((W-V)^T B (W-V) A) (proxy_loss.cu): the two products on the
// tensor cores in 3xTF32, the elementwise dot in FP64 with a fixed order.
struct ProxyLayout {
    int64_t m, n, Mp, Np;
    size_t status, Ehi, Elo, EThi, ETlo, Bhi, Blo, Ahi, Alo, P, Q, parts, total;
    void compute(int64_t m_, int64_t n_);
};
cudaError_t launch_proxy_loss(const float *W, const float *V, const float *A, const float *B, const ProxyLayout &L,
                              char *ws, double *out, cudaStream_t stream);

// FP64 factorisation: L (n x n, fp32) = chol(A^{-1}); work holds
// factor_work_doubles(n) doubles.
size_t factor_work_doubles(int64_t n);
cudaError_t launch_factor(const float *A, int64_t n, float *L, double *work, DeviceStatus *st,
                          cudaStream_t stream);

// bakron_solve with direct launches only: never the CUDA graph path, whatever
// cfg->use_graph or BAKRON_GRAPH ask for (graph capture and instantiation make
// the driver allocate).  Arguments and checks as bakron_solve.
bakron_status_t solve_direct(const float *W, int64_t m, int64_t n, const float *LA, const float *LB,
                             const bakron_quantizer_t *q, float *V, int8_t *codes, float *scales, void *ws,
                             size_t ws_bytes, const bakron_config_t *cfg, cudaStream_t stream);

// One thread waits on an mbarrier nothing completes, with the band kernel's
// bounded-wait helper; records BAKRON_ERR_DEVICE_TIMEOUT when it gives up.
cudaError_t launch_wait_timeout_selftest(DeviceStatus *st, int timeout_ms, cudaStream_t stream);

// The stage-1 band kernel on a 256 x 256 problem laid out in `buf` (six
// 256 x 256 fp32 arrays, 16-byte aligned) with its producer issuing no copies:
// the MMA and epilogue waits run out, record BAKRON_ERR_DEVICE_TIMEOUT and the
// kernel takes its abort path (nothing is in flight).
constexpr size_t kBandAbortBufBytes = (size_t)6 * 256 * 256 * sizeof(float);
cudaError_t launch_band_abort_selftest(DeviceStatus *st, float *buf, int timeout_ms, cudaStream_t stream);

}  // namespace bakron
