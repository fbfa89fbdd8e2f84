// gram.cu -- Kronecker factor A = X^T X / N + damping * mean(diag) * I from
// calibration samples X (N x d), the estimate the pages' K-FAC factors are
// built from (expectation of a a^T, "Assumptions & free parameters": Gram
// matrix regularisation).  The product runs on the tensor cores (3xTF32,
// band_tc_kernel<3>); this file holds the transpose-and-split before it and
// the symmetrise / scale / damp pass after it.
#include "common.cuh"
#include "kernels.cuh"

namespace bakron {

// XT hi / lo (Dp x Ns, row stride Ns) <- TF32 split of X^T, zero padded;
// 32 x 32 tiles through shared memory so both sides are coalesced.
__global__ void gram_transpose_kernel(const float *__restrict__ X, int64_t N, int64_t d, int64_t Dp, int64_t Ns,
                                      float *__restrict__ xt_hi, float *__restrict__ xt_lo, DeviceStatus *st)
{
    pdl_wait();
    pdl_trigger();
    __shared__ float tile[32][33];
    const int64_t s0 = (int64_t)blockIdx.x * 32, f0 = (int64_t)blockIdx.y * 32;
    const int tx = threadIdx.x, ty = threadIdx.y;  // 32 x 8
    bool finite = true;
    for (int r = ty; r < 32; r += 8) {
        const int64_t s = s0 + r, f = f0 + tx;
        float v = 0.f;
        if (s < N && f < d) {
            v = X[s * d + f];
            finite &= isfinite(v);
        }
        tile[r][tx] = v;
    }
    if (!finite) record_error(st, BAKRON_ERR_NONFINITE, (int)(f0 + tx));
    __syncthreads();
    for (int r = ty; r < 32; r += 8) {
        const int64_t f = f0 + r, s = s0 + tx;
        float hi, lo;
        split_tf32(tile[tx][r], hi, lo);
        xt_hi[f * Ns + s] = hi;
        xt_lo[f * Ns + s] = lo;
    }
}

// A (d x d) <- G / N from G's lower triangle (G padded Dp x Dp), plus
// damping * mean(diag(G / N)) on the diagonal.  Every CTA forms the diagonal
// mean itself (FP64 sum, same order in each), then a grid-stride share of the
// entries.
__global__ void gram_finish_kernel(const float *__restrict__ G, int64_t d, int64_t Dp, int64_t N, float damping,
                                   float *__restrict__ A)
{
    pdl_wait();
    pdl_trigger();
    __shared__ double part[32];
    __shared__ float add_sh;
    const float fN = (float)N;
    double sum = 0.0;
    for (int64_t i = threadIdx.x; i < d; i += blockDim.x) sum += (double)__fdiv_rn(G[i * Dp + i], fN);
    for (int o = 16; o; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = sum;
    __syncthreads();
    if (threadIdx.x == 0) {
        double t = 0.0;
        for (int w = 0; w < (int)(blockDim.x >> 5); ++w) t += part[w];
        add_sh = (float)((double)damping * (t / (double)d));
    }
    __syncthreads();
    const float add = add_sh;
    for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < d * d;
         idx += (int64_t)gridDim.x * blockDim.x) {
        const int64_t i = idx / d, j = idx - i * d;
        const float g = i >= j ? G[i * Dp + j] : G[j * Dp + i];
        float v = __fdiv_rn(g, fN);
        if (i == j) v = __fadd_rn(v, add);
        A[idx] = v;
    }
}

cudaError_t launch_gram_prep(const float *X, int64_t N, int64_t d, int64_t Dp, int64_t Ns, float *xt_hi,
                             float *xt_lo, DeviceStatus *st, cudaStream_t stream)
{
    return launch_pdl(gram_transpose_kernel, dim3((unsigned)(Ns / 32), (unsigned)(Dp / 32)), dim3(32, 8), 0, stream,
                      X, N, d, Dp, Ns, xt_hi, xt_lo, st);
}

cudaError_t launch_gram_finish(const float *G, int64_t d, int64_t Dp, int64_t N, float damping, float *A,
                               cudaStream_t stream)
{
    int64_t blocks = (d * d + 1023) / 1024;
    if (blocks > 148 * 4) blocks = 148 * 4;
    return launch_pdl(gram_finish_kernel, dim3((unsigned)blocks), dim3(1024), 0, stream, G, d, Dp, N, damping, A);
}

}  // namespace bakron
