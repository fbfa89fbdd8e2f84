// factor.cu -- L = chol(A^{-1}) in FP64 ("What carries the argument": the
// lower-triangular Cholesky factors L^(A), L^(B) of A^{-1}, B^{-1}).
//
// With J the exchange matrix, let J A J = C C^T (lower Cholesky).  Then
// A = (J C J)(J C J)^T with J C J upper triangular, so
// A^{-1} = (J C^{-T} J)(J C^{-T} J)^T and J C^{-T} J is lower triangular with
// positive diagonal: by uniqueness it is chol(A^{-1}).  Element-wise,
// L[i][j] = Cinv[n-1-j][n-1-i].  This needs one Cholesky and one triangular
// inverse and never forms A^{-1} explicitly.
//
// Blocked right-looking Cholesky (panel factor, panel solve, trailing
// symmetric update) and a blocked triangular inverse swept by block
// diagonals; all FP64 on CUDA cores, 64 x 64 blocks.
#include "common.cuh"
#include "kernels.cuh"

namespace bakron {

namespace {
constexpr int NB = 64;
}

// X (lower) <- J A J from A's lower triangle; checks finiteness.
__global__ void rev_copy_kernel(const float *__restrict__ A, int64_t n, double *__restrict__ X,
                                DeviceStatus *st)
{
    int64_t total = n * n;
    for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
         idx += (int64_t)gridDim.x * blockDim.x) {
        int64_t i = idx / n, j = idx - i * n;
        double v = 0.0;
        if (j <= i) {
            float a = A[(n - 1 - j) * n + (n - 1 - i)];  // (JAJ)[i][j] = A[n-1-i][n-1-j] = A[n-1-j][n-1-i]
            if (!isfinite(a)) record_error(st, BAKRON_ERR_NONFINITE, (int)i);
            v = a;
        }
        X[idx] = v;
    }
}

// Unblocked Cholesky of the diagonal block [kb, kb+bs) in shared memory.
__global__ void __launch_bounds__(256) potrf_block_kernel(double *X, int64_t n, int64_t kb, int bs,
                                                          DeviceStatus *st)
{
    __shared__ double a[NB][NB + 1];
    const int tid = threadIdx.x;
    for (int idx = tid; idx < bs * bs; idx += 256) {
        int r = idx / bs, c = idx % bs;
        a[r][c] = c <= r ? X[(kb + r) * n + kb + c] : 0.0;
    }
    __syncthreads();
    for (int j = 0; j < bs; ++j) {
        if (tid == 0) {
            double d = a[j][j];
            if (!(d > 0.0) || !isfinite(d)) {
                record_error(st, BAKRON_ERR_NOT_SPD, (int)(kb + j));
                d = 1.0;
            }
            a[j][j] = sqrt(d);
        }
        __syncthreads();
        const double piv = a[j][j];
        for (int i = j + 1 + tid; i < bs; i += 256) a[i][j] /= piv;
        __syncthreads();
        const int w = bs - j - 1;
        for (int idx = tid; idx < w * w; idx += 256) {
            int i = j + 1 + idx / w, k = j + 1 + idx % w;
            if (k <= i) a[i][k] -= a[i][j] * a[k][j];
        }
        __syncthreads();
    }
    for (int idx = tid; idx < bs * bs; idx += 256) {
        int r = idx / bs, c = idx % bs;
        if (c <= r) X[(kb + r) * n + kb + c] = a[r][c];
    }
}

// Rows below the diagonal block: X[r][kb:kb+bs] <- X[r][kb:kb+bs] * C_kk^{-T}.
__global__ void __launch_bounds__(128) trsm_panel_kernel(double *X, int64_t n, int64_t kb, int bs)
{
    __shared__ double c[NB][NB + 1];
    for (int idx = threadIdx.x; idx < bs * bs; idx += blockDim.x) {
        int r = idx / bs, cc = idx % bs;
        c[r][cc] = cc <= r ? X[(kb + r) * n + kb + cc] : 0.0;
    }
    __syncthreads();
    const int64_t r = kb + bs + (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (r >= n) return;
    double x[NB];
#pragma unroll
    for (int j = 0; j < NB; ++j) x[j] = j < bs ? X[r * n + kb + j] : 0.0;
#pragma unroll
    for (int j = 0; j < NB; ++j) {
        if (j < bs) {
            double v = x[j];
#pragma unroll
            for (int t = 0; t < j; ++t) v -= x[t] * c[j][t];
            x[j] = v / c[j][j];
        }
    }
#pragma unroll
    for (int j = 0; j < NB; ++j)
        if (j < bs) X[r * n + kb + j] = x[j];
}

// Trailing update of the lower triangle: X[i][j] -= sum_t P[i][t] P[j][t] for
// i >= j >= kb+bs, P = X[:, kb:kb+bs].  One CTA per 64 x 64 block (ti >= tj).
__global__ void __launch_bounds__(256) syrk_update_kernel(double *X, int64_t n, int64_t kb, int bs)
{
    const int ti = blockIdx.y, tj = blockIdx.x;
    if (tj > ti) return;
    __shared__ double Pi[NB][33];
    __shared__ double Pj[NB][33];
    const int64_t base = kb + bs, r0 = base + (int64_t)ti * NB, c0 = base + (int64_t)tj * NB;
    const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
    double acc[4][4] = {};
    for (int t0 = 0; t0 < bs; t0 += 32) {
        for (int idx = tid; idx < NB * 32; idx += 256) {
            int rr = idx / 32, tt = idx % 32;
            int64_t ri = r0 + rr, rj = c0 + rr;
            bool ok = t0 + tt < bs;
            Pi[rr][tt] = (ok && ri < n) ? X[ri * n + kb + t0 + tt] : 0.0;
            Pj[rr][tt] = (ok && rj < n) ? X[rj * n + kb + t0 + tt] : 0.0;
        }
        __syncthreads();
#pragma unroll 8
        for (int t = 0; t < 32; ++t) {
            double a[4], b[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) a[i] = Pi[ty * 4 + i][t];
#pragma unroll
            for (int j = 0; j < 4; ++j) b[j] = Pj[tx * 4 + j][t];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fma(a[i], b[j], acc[i][j]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            int64_t r = r0 + ty * 4 + i, c = c0 + tx * 4 + j;
            if (r < n && c <= r) X[r * n + c] -= acc[i][j];
        }
}

// Inverse of every diagonal block of C (lower): Y[ib][ib] = C[ib][ib]^{-1}.
// Thread c solves C_bb y = e_c by forward substitution.
__global__ void __launch_bounds__(NB) trinv_diag_kernel(const double *C, double *Y, int64_t n)
{
    __shared__ double c[NB][NB + 1];
    const int64_t b0 = (int64_t)blockIdx.x * NB;
    const int bs = (int)min64(NB, n - b0);
    for (int idx = threadIdx.x; idx < NB * NB; idx += NB) {
        int r = idx / NB, cc = idx % NB;
        c[r][cc] = (r < bs && cc <= r) ? C[(b0 + r) * n + b0 + cc] : 0.0;
    }
    __syncthreads();
    const int col = threadIdx.x;
    if (col >= bs) return;
    double y[NB];
#pragma unroll
    for (int r = 0; r < NB; ++r) {
        double v = r == col ? 1.0 : 0.0;
#pragma unroll
        for (int t = 0; t < r; ++t) v -= c[r][t] * y[t];
        y[r] = r < bs ? v / c[r][r] : 0.0;
    }
#pragma unroll
    for (int r = 0; r < NB; ++r)
        if (r < bs) Y[(b0 + r) * n + b0 + col] = r >= col ? y[r] : 0.0;
}

// Off-diagonal blocks at block distance `dist`: for jb = blockIdx.x,
// ib = jb + dist: Y[ib][jb] = -Y[ib][ib] * sum_{kb=jb}^{ib-1} C[ib][kb] Y[kb][jb].
__global__ void __launch_bounds__(256) trinv_offdiag_kernel(const double *C, double *Y, int64_t n,
                                                            int dist)
{
    // phase 1 uses As/Bs, phase 2 uses Ts/A2 (42 KB, under the static limit)
    __shared__ union {
        struct { double As[NB][33]; double Bs[32][NB + 1]; } p1;
        struct { double Ts[NB][NB + 1]; double A2[NB][17]; } p2;
    } sh;
    auto &As = sh.p1.As;
    auto &Bs = sh.p1.Bs;
    auto &Ts = sh.p2.Ts;
    auto &A2 = sh.p2.A2;
    const int jb = blockIdx.x, ib = jb + dist;
    const int64_t r0 = (int64_t)ib * NB, c0 = (int64_t)jb * NB;
    const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
    double acc[4][4] = {};
    // T = sum_{kb} C[ib][kb] * Y[kb][jb]  (K runs over columns [c0, r0))
    for (int64_t k0 = c0; k0 < r0; k0 += 32) {
        for (int idx = tid; idx < NB * 32; idx += 256) {
            int rr = idx / 32, kk = idx % 32;
            int64_t r = r0 + rr, k = k0 + kk;
            As[rr][kk] = (r < n && k < n) ? C[r * n + k] : 0.0;
            int kk2 = idx / NB, cc = idx % NB;
            int64_t k2 = k0 + kk2, c = c0 + cc;
            Bs[kk2][cc] = (k2 < n && c < n && c <= k2) ? Y[k2 * n + c] : 0.0;
        }
        __syncthreads();
#pragma unroll 8
        for (int kk = 0; kk < 32; ++kk) {
            double a[4], b[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) a[i] = As[ty * 4 + i][kk];
#pragma unroll
            for (int j = 0; j < 4; ++j) b[j] = Bs[kk][tx * 4 + j];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fma(a[i], b[j], acc[i][j]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) Ts[ty * 4 + i][tx * 4 + j] = acc[i][j];
    // Y[ib][jb] = -Y[ib][ib] * T
    double out[4][4] = {};
    for (int k0 = 0; k0 < NB; k0 += 16) {
        for (int idx = tid; idx < NB * 16; idx += 256) {
            int rr = idx / 16, kk = idx % 16;
            int64_t r = r0 + rr, k = r0 + k0 + kk;
            A2[rr][kk] = (r < n && k < n && k <= r) ? Y[r * n + k] : 0.0;
        }
        __syncthreads();
#pragma unroll 8
        for (int kk = 0; kk < 16; ++kk) {
            double a[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) a[i] = A2[ty * 4 + i][kk];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) out[i][j] = fma(a[i], Ts[k0 + kk][tx * 4 + j], out[i][j]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            int64_t r = r0 + ty * 4 + i, c = c0 + tx * 4 + j;
            if (r < n && c < n) Y[r * n + c] = -out[i][j];
        }
}

// L[i][j] = Y[n-1-j][n-1-i] for j <= i, 0 above; fp32.
__global__ void write_factor_kernel(const double *__restrict__ Y, int64_t n, float *__restrict__ L)
{
    int64_t total = n * n;
    for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
         idx += (int64_t)gridDim.x * blockDim.x) {
        int64_t i = idx / n, j = idx - i * n;
        L[idx] = j <= i ? (float)Y[(n - 1 - j) * n + (n - 1 - i)] : 0.f;
    }
}

cudaError_t launch_factor(const float *A, int64_t n, float *L, double *work, DeviceStatus *st,
                          cudaStream_t stream)
{
    if (n <= 0) return cudaSuccess;
    double *C = work, *Y = work + n * n;
    int64_t elems = n * n;
    int g = (int)min64((elems + 255) / 256, 148 * 16);
    rev_copy_kernel<<<g, 256, 0, stream>>>(A, n, C, st);
    for (int64_t kb = 0; kb < n; kb += NB) {
        int bs = (int)min64(NB, n - kb);
        potrf_block_kernel<<<1, 256, 0, stream>>>(C, n, kb, bs, st);
        int64_t rest = n - kb - bs;
        if (rest > 0) {
            trsm_panel_kernel<<<(unsigned)((rest + 127) / 128), 128, 0, stream>>>(C, n, kb, bs);
            unsigned nt = (unsigned)((rest + NB - 1) / NB);
            syrk_update_kernel<<<dim3(nt, nt), 256, 0, stream>>>(C, n, kb, bs);
        }
    }
    const int nblk = (int)((n + NB - 1) / NB);
    trinv_diag_kernel<<<nblk, NB, 0, stream>>>(C, Y, n);
    for (int dist = 1; dist < nblk; ++dist)
        trinv_offdiag_kernel<<<nblk - dist, 256, 0, stream>>>(C, Y, n, dist);
    write_factor_kernel<<<g, 256, 0, stream>>>(Y, n, L);
    return cudaGetLastError();
}

}  // namespace bakron
