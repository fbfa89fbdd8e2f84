// band_simt.cu -- FP32 CUDA-core band products of Algorithm 6's postponed
// updates ("two dense matmuls per level"): the cross-check kernels for the
// tensor-core path.  Operands are read as hi + lo, which reconstructs the
// fp32 value to within one TF32 rounding of the low part.
#include "common.cuh"
#include "kernels.cuh"

namespace bakron {

namespace {
constexpr int T = kTile;
constexpr int BK = 16;
}

template <int STAGE>
__global__ void __launch_bounds__(256) band_simt_kernel(NodeParams np, GemmArgs g)
{
    const Item it = STAGE == 1 ? stage1_item(np, blockIdx.x, blockIdx.y)
                               : stage2_item(np, blockIdx.x, blockIdx.y);
    if (!it.valid) return;
    pdl_wait();
    __shared__ float As[BK][T + 4];
    __shared__ float Bs[BK][T + 4];
    const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
    const int64_t arow = (int64_t)it.ra * T, brow = (int64_t)it.rb * T;
    float acc[8][8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;

    const int lr = tid >> 1, lc = (tid & 1) * 8;
    for (int64_t kk = (int64_t)it.k0 * T; kk < (int64_t)it.k1 * T; kk += BK) {
        const int64_t ao = (arow + lr) * g.lda + kk + lc, bo = (brow + lr) * g.ldb + kk + lc;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            As[lc + c][lr] = g.Ahi[ao + c] + g.Alo[ao + c];
            Bs[lc + c][lr] = g.Bhi[bo + c] + g.Blo[bo + c];
        }
        __syncthreads();
#pragma unroll
        for (int k = 0; k < BK; ++k) {
            float a[8], b[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) a[i] = As[k][ty * 8 + i];
#pragma unroll
            for (int j = 0; j < 8; ++j) b[j] = Bs[k][tx * 8 + j];
#pragma unroll
            for (int i = 0; i < 8; ++i)
#pragma unroll
                for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int64_t o = (arow + ty * 8 + i) * g.ldo + brow + tx * 8;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            if (STAGE == 1) {
                float hi, lo;
                split_tf32(acc[i][j], hi, lo);
                g.out_hi[o + j] = hi;
                g.out_lo[o + j] = lo;
            } else {
                g.out_acc[o + j] -= acc[i][j];
            }
        }
    }
}

cudaError_t launch_band_simt(int stage, const NodeParams &np, const GemmArgs &g, cudaStream_t stream)
{
    if (stage == 1) return launch_pdl(band_simt_kernel<1>, dim3(np.l, np.Mt), dim3(256), 0, stream, np, g);
    return launch_pdl(band_simt_kernel<2>, dim3(np.l - np.h, np.Mt), dim3(256), 0, stream, np, g);
}

// --------------------------------------------------------------------------
// Proxy loss l = sum_ij (B E)_ij (E A)_ij with E = W - V (Corollary 3.4's
// ||B^{1/2}(V-W)A^{1/2}||_F^2 written as tr(E^T B E A)).  One CTA per 64 x 64
// output tile computes both products in FP32 and reduces their elementwise
// product in FP64 into its own slot of `part`; one more CTA adds the slots in
// a fixed order, so the result does not depend on the order the CTAs finish.
__global__ void __launch_bounds__(256) proxy_loss_kernel(const float *__restrict__ W,
                                                        const float *__restrict__ V,
                                                        const float *__restrict__ A,
                                                        const float *__restrict__ B, int64_t m,
                                                        int64_t n, double *tile_sums)
{
    constexpr int TB = 64, KB = 16;
    __shared__ float Xs[KB][TB + 4];
    __shared__ float Ys[KB][TB + 4];
    __shared__ double red[8];
    const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
    const int64_t i0 = (int64_t)blockIdx.y * TB, j0 = (int64_t)blockIdx.x * TB;
    float P[4][4], Q[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) P[i][j] = Q[i][j] = 0.f;

    // P = B[i0:, :] * E[:, j0:]   (K = m)
    for (int64_t k0 = 0; k0 < m; k0 += KB) {
        for (int idx = tid; idx < KB * TB; idx += 256) {
            int kk = idx / TB, r = idx % TB;
            int64_t i = i0 + r, k = k0 + kk, j = j0 + r;
            // Xs[kk][r] = B[i][k] = B[k][i] (B symmetric), Ys[kk][r] = E[k][j]
            Xs[kk][r] = (i < m && k < m) ? B[k * m + i] : 0.f;
            Ys[kk][r] = (k < m && j < n) ? W[k * n + j] - V[k * n + j] : 0.f;
        }
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < KB; ++kk)
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) P[i][j] = fmaf(Xs[kk][ty * 4 + i], Ys[kk][tx * 4 + j], P[i][j]);
        __syncthreads();
    }
    // Q = E[i0:, :] * A[:, j0:]   (K = n)
    for (int64_t k0 = 0; k0 < n; k0 += KB) {
        for (int idx = tid; idx < KB * TB; idx += 256) {
            {   // Xs[kk][r] = E[i0+r][k0+kk]: consecutive threads walk k
                int r = idx / KB, kk = idx % KB;
                int64_t i = i0 + r, k = k0 + kk;
                Xs[kk][r] = (i < m && k < n) ? W[i * n + k] - V[i * n + k] : 0.f;
            }
            int kk = idx / TB, r = idx % TB;
            int64_t k = k0 + kk, j = j0 + r;
            Ys[kk][r] = (k < n && j < n) ? A[k * n + j] : 0.f;
        }
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < KB; ++kk)
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) Q[i][j] = fmaf(Xs[kk][ty * 4 + i], Ys[kk][tx * 4 + j], Q[i][j]);
        __syncthreads();
    }
    double part = 0.0;
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j)
            if (i0 + ty * 4 + i < m && j0 + tx * 4 + j < n) part += (double)P[i][j] * (double)Q[i][j];
    for (int o = 16; o; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
    if ((tid & 31) == 0) red[tid >> 5] = part;
    __syncthreads();
    if (tid == 0) {
        double s = 0.0;
        for (int w = 0; w < 8; ++w) s += red[w];
        tile_sums[(int64_t)blockIdx.y * gridDim.x + blockIdx.x] = s;
    }
}

// out = sum of the per-tile partial sums: each thread adds a strided subset in
// index order, then a fixed tree over the threads.
__global__ void __launch_bounds__(256) proxy_loss_finish_kernel(const double *__restrict__ part, int64_t count,
                                                               double *out)
{
    __shared__ double red[256];
    double s = 0.0;
    for (int64_t i = threadIdx.x; i < count; i += 256) s += part[i];
    red[threadIdx.x] = s;
    __syncthreads();
    for (int w = 128; w; w >>= 1) {
        if ((int)threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
        __syncthreads();
    }
    if (threadIdx.x == 0) *out = red[0];
}

int64_t proxy_loss_parts(int64_t m, int64_t n) { return ((n + 63) / 64) * ((m + 63) / 64); }

cudaError_t launch_proxy_loss(const float *W, const float *V, const float *A, const float *B,
                              int64_t m, int64_t n, double *out, double *part, cudaStream_t stream)
{
    dim3 grid((unsigned)((n + 63) / 64), (unsigned)((m + 63) / 64));
    proxy_loss_kernel<<<grid, 256, 0, stream>>>(W, V, A, B, m, n, part);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    proxy_loss_finish_kernel<<<1, 256, 0, stream>>>(part, proxy_loss_parts(m, n), out);
    return cudaGetLastError();
}

}  // namespace bakron
