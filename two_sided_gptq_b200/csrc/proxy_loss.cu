// proxy_loss.cu -- the proxy loss l = tr(E^T B E A), E = W - V (Corollary 3.4's
// distortion ||B^{1/2}(V-W)A^{1/2}||_F^2; the review's ||vec(W)-vec(V)||_H^2
// with H = A (x) B), written as l = sum_ij P_ij Q_ij with P = B E and
// Q = E A.  Both products run on the tensor cores in 3xTF32 (the band
// kernel's full-tile stage); this file holds the split of the operands into
// TF32 hi / lo parts before them (zero padded to whole tiles, E also
// transposed so that every operand is K-major) and the FP64 dot after them.
#include "common.cuh"
#include "kernels.cuh"

namespace bakron {

namespace {
constexpr int T = kTile;
constexpr int kDotBlocks = 148 * 4;  // fixed, so the summation order depends on (m, n) only
}

void ProxyLayout::compute(int64_t m_, int64_t n_)
{
    m = m_; n = n_;
    Mp = (m + T - 1) / T * T; Np = (n + T - 1) / T * T;
    size_t o = 0;
    auto take = [&](size_t bytes) { size_t at = o; o = align_up(o + bytes); return at; };
    const size_t mn = (size_t)Mp * Np * sizeof(float);
    status = take(kStatusBytes);
    Ehi = take(mn); Elo = take(mn); EThi = take(mn); ETlo = take(mn);
    Bhi = take((size_t)Mp * Mp * sizeof(float)); Blo = take((size_t)Mp * Mp * sizeof(float));
    Ahi = take((size_t)Np * Np * sizeof(float)); Alo = take((size_t)Np * Np * sizeof(float));
    P = take(mn); Q = take(mn);
    parts = take((size_t)kDotBlocks * sizeof(double));
    total = o;
}

// out (Rp x Cp, hi / lo) <- TF32 split of X - Y (Y may be null; X, Y rows x
// cols, row stride cols), transposed when `trans` (then out is Cp x Rp and
// holds (X - Y)^T), zero outside the matrix.  32 x 32 tiles through shared
// memory so reads and writes are both coalesced; grid (Cp / 32, Rp / 32) in
// the source's orientation.
__global__ void split_pad_kernel(const float *__restrict__ X, const float *__restrict__ Y, int64_t rows, int64_t cols,
                                 int64_t Rp, int64_t Cp, bool trans, float *__restrict__ hi, float *__restrict__ lo)
{
    __shared__ float tile[32][33];
    const int64_t r0 = (int64_t)blockIdx.y * 32, c0 = (int64_t)blockIdx.x * 32;
    const int tx = threadIdx.x, ty = threadIdx.y;  // 32 x 8
    for (int r = ty; r < 32; r += 8) {
        const int64_t i = r0 + r, j = c0 + tx;
        float v = 0.f;
        if (i < rows && j < cols) v = Y ? X[i * cols + j] - Y[i * cols + j] : X[i * cols + j];
        tile[r][tx] = v;
    }
    __syncthreads();
    for (int r = ty; r < 32; r += 8) {
        float h, l;
        if (trans) {  // out[c0 + r][r0 + tx] = tile[tx][r]
            split_tf32(tile[tx][r], h, l);
            const int64_t o = (c0 + r) * Rp + r0 + tx;
            hi[o] = h;
            lo[o] = l;
        } else {
            split_tf32(tile[r][tx], h, l);
            const int64_t o = (r0 + r) * Cp + c0 + tx;
            hi[o] = h;
            lo[o] = l;
        }
    }
}

// parts[b] = sum over this block's fixed share of the entries of P * Q (FP64):
// each thread adds its grid-strided entries in index order, then a fixed
// tree over the block.
__global__ void __launch_bounds__(256) dot_parts_kernel(const float *__restrict__ P, const float *__restrict__ Q,
                                                        int64_t count, double *__restrict__ parts)
{
    __shared__ double red[256];
    double s = 0.0;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < count; i += stride)
        s = fma((double)P[i], (double)Q[i], s);
    red[threadIdx.x] = s;
    __syncthreads();
    for (int w = 128; w; w >>= 1) {
        if ((int)threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
        __syncthreads();
    }
    if (threadIdx.x == 0) parts[blockIdx.x] = red[0];
}

// *out = the parts added in index order.
__global__ void dot_finish_kernel(const double *__restrict__ parts, int count, double *out)
{
    if (threadIdx.x != 0) return;
    double s = 0.0;
    for (int i = 0; i < count; ++i) s += parts[i];
    *out = s;
}

cudaError_t launch_proxy_loss(const float *W, const float *V, const float *A, const float *B, const ProxyLayout &L,
                              char *ws, double *out, cudaStream_t stream)
{
    float *Ehi = (float *)(ws + L.Ehi), *Elo = (float *)(ws + L.Elo);
    float *EThi = (float *)(ws + L.EThi), *ETlo = (float *)(ws + L.ETlo);
    float *Bhi = (float *)(ws + L.Bhi), *Blo = (float *)(ws + L.Blo);
    float *Ahi = (float *)(ws + L.Ahi), *Alo = (float *)(ws + L.Alo);
    float *P = (float *)(ws + L.P), *Q = (float *)(ws + L.Q);
    double *parts = (double *)(ws + L.parts);
    const dim3 blk(32, 8);
    const dim3 g_e((unsigned)(L.Np / 32), (unsigned)(L.Mp / 32));
    split_pad_kernel<<<g_e, blk, 0, stream>>>(W, V, L.m, L.n, L.Mp, L.Np, false, Ehi, Elo);
    split_pad_kernel<<<g_e, blk, 0, stream>>>(W, V, L.m, L.n, L.Mp, L.Np, true, EThi, ETlo);
    split_pad_kernel<<<dim3((unsigned)(L.Mp / 32), (unsigned)(L.Mp / 32)), blk, 0, stream>>>(B, nullptr, L.m, L.m,
                                                                                            L.Mp, L.Mp, false, Bhi, Blo);
    split_pad_kernel<<<dim3((unsigned)(L.Np / 32), (unsigned)(L.Np / 32)), blk, 0, stream>>>(A, nullptr, L.n, L.n,
                                                                                            L.Np, L.Np, false, Ahi, Alo);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    DeviceStatus *st = (DeviceStatus *)(ws + L.status);
    const GemmArgs g{nullptr, nullptr, nullptr, nullptr, 0, 0, nullptr, nullptr, nullptr, 0, st, 200, 0};
    // P = B E: A operand B (rows of B, K = m), B operand E^T (rows = columns of E)
    TcMaps mp, mq;
    if (!make_full_maps(Bhi, Blo, EThi, ETlo, P, L.Mp, L.Np, L.Mp, &mp)) return cudaErrorInvalidValue;
    // Q = E A: A operand E (K = n), B operand rows of A^T = A (symmetric)
    if (!make_full_maps(Ehi, Elo, Ahi, Alo, Q, L.Mp, L.Np, L.Np, &mq)) return cudaErrorInvalidValue;
    if ((e = launch_full_tc(L.Mp, L.Np, L.Mp, g, mp, stream)) != cudaSuccess) return e;
    if ((e = launch_full_tc(L.Mp, L.Np, L.Np, g, mq, stream)) != cudaSuccess) return e;
    dot_parts_kernel<<<kDotBlocks, 256, 0, stream>>>(P, Q, L.Mp * L.Np, parts);
    dot_finish_kernel<<<1, 32, 0, stream>>>(parts, kDotBlocks, out);
    return cudaGetLastError();
}

}  // namespace bakron
