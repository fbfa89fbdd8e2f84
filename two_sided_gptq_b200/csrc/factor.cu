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
// Blocked right-looking Cholesky on 64-wide panels (the diagonal block's
// factor and its inverse in one CTA; the panel solve and the trailing
// symmetric update as GEMMs) and a recursive triangular
// inverse, inv([[A, 0], [B, C]]) = [[A^-1, 0], [-C^-1 B A^-1, C^-1]], whose
// merges are two GEMMs each; all FP64 on the CUDA cores.  The GEMM is one
// register-blocked kernel (128 x 128 or 64 x 64 output tiles) that skips the
// zero halves of triangular operands.
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

// 1/sqrt(d) to FP64 accuracy by Newton's iteration for the reciprocal square
// root, y <- y + y (1 - d y^2) / 2, from the single-precision estimate: each
// step squares the relative error (about 2^-22, 2^-44, then FP64 rounding).
// Pivots outside the range where the single-precision estimate is safe take
// the IEEE square root and division.
__device__ __forceinline__ double rsqrt_fp64(double d)
{
    if (!(d > 1e-30 && d < 1e30)) return 1.0 / sqrt(d);
    double y = (double)rsqrtf((float)d);
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const double h = d * y;
        const double r = fma(-h, y, 1.0);
        y = fma(0.5 * y, r, y);
    }
    return y;
}

// Diagonal block [kb, kb+bs): its Cholesky factor C_kk into X and C_kk^-1
// into Y (both lower; Y's block gets explicit zeros above the diagonal).  256
// threads, each holding a 4 x 4 set of the 64 x 64 block in registers (rows
// ty + 16 r, columns tx + 16 c); a block shorter than 64 is padded with the
// identity.  Right-looking in both loops with one barrier per step: the
// column (Cholesky) or row (inverse) that the next step needs is published to
// a double-buffered shared array by its owners as soon as they have updated
// it, and every thread scales its own copy by the pivot.
__global__ void __launch_bounds__(256) potrf_inv_kernel(double *X, double *Y, int64_t n, int64_t kb, int bs,
                                                        DeviceStatus *st)
{
    __shared__ double vec[2][NB];
    __shared__ double cf[NB][NB + 1];
    __shared__ double rdiag[NB];  // 1 / C_kk[j][j]
    const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
    double a[4][4];
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const int i = ty + 16 * r, k = tx + 16 * c;
            a[r][c] = (i < bs && k <= i) ? X[(kb + i) * n + kb + k] : (i == k ? 1.0 : 0.0);
        }
    if (tx == 0)
#pragma unroll
        for (int r = 0; r < 4; ++r) vec[0][ty + 16 * r] = a[r][0];
    __syncthreads();
    for (int j = 0; j < NB; ++j) {
        const double *cj = vec[j & 1];
        double d = cj[j];
        if (!(d > 0.0) || !isfinite(d)) {
            if (tid == 0) record_error(st, BAKRON_ERR_NOT_SPD, (int)(kb + j));
            d = 1.0;
        }
        const double rp = rsqrt_fp64(d), piv = d * rp;
        if (tid == 0) rdiag[j] = rp;
        double li[4], lk[4];
#pragma unroll
        for (int r = 0; r < 4; ++r) li[r] = ty + 16 * r > j ? cj[ty + 16 * r] * rp : 0.0;
#pragma unroll
        for (int c = 0; c < 4; ++c) lk[c] = tx + 16 * c > j ? cj[tx + 16 * c] * rp : 0.0;
#pragma unroll
        for (int r = 0; r < 4; ++r)
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const int i = ty + 16 * r, k = tx + 16 * c;
                if (k == j) {
                    if (i == j) a[r][c] = piv;
                    else if (i > j) a[r][c] = li[r];
                } else if (k > j && k <= i) {
                    a[r][c] -= li[r] * lk[c];
                }
            }
        if (j + 1 < NB && tx == ((j + 1) & 15)) {
            const int cs = (j + 1) >> 4;  // selects, not an indexed read (keeps a[][] in registers)
#pragma unroll
            for (int r = 0; r < 4; ++r)
                vec[(j + 1) & 1][ty + 16 * r] = cs == 0 ? a[r][0] : cs == 1 ? a[r][1] : cs == 2 ? a[r][2] : a[r][3];
        }
        __syncthreads();
    }
    // the factor to shared memory (read by column in the inverse) and X
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const int i = ty + 16 * r, k = tx + 16 * c;
            cf[i][k] = k <= i ? a[r][c] : 0.0;
            if (i < bs && k <= i) X[(kb + i) * n + kb + k] = a[r][c];
        }
    // inverse: Y = I; for each t, row t /= C[t][t], then rows below lose
    // C[i][t] times it.  a[][] now holds Y.
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int c = 0; c < 4; ++c) a[r][c] = (ty + 16 * r == tx + 16 * c) ? 1.0 : 0.0;
    if (ty == 0)
#pragma unroll
        for (int c = 0; c < 4; ++c) vec[0][tx + 16 * c] = a[0][c];
    __syncthreads();
    for (int t = 0; t < NB; ++t) {
        const double *yt = vec[t & 1];
        const double rd = rdiag[t];
        double v[4], ci[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) v[c] = yt[tx + 16 * c] * rd;
#pragma unroll
        for (int r = 0; r < 4; ++r) ci[r] = cf[ty + 16 * r][t];
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            const int i = ty + 16 * r;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                if (i == t) a[r][c] = v[c];
                else if (i > t) a[r][c] -= ci[r] * v[c];
            }
        }
        if (t + 1 < NB && ty == ((t + 1) & 15)) {
            const int rs = (t + 1) >> 4;
#pragma unroll
            for (int c = 0; c < 4; ++c)
                vec[(t + 1) & 1][tx + 16 * c] = rs == 0 ? a[0][c] : rs == 1 ? a[1][c] : rs == 2 ? a[2][c] : a[3][c];
        }
        __syncthreads();
    }
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const int i = ty + 16 * r, k = tx + 16 * c;
            if (i < bs && k < bs) Y[(kb + i) * n + kb + k] = k <= i ? a[r][c] : 0.0;
        }
}

// C[i][j] = alpha sum_k A[i][k] B'[k][j] + beta C[i][j] for an M x N output,
// with A row-major (lda) and B' = B row-major K x N (ldb) or, with
// B_KMAJOR, B' = B^T for B row-major N x K.  flags: kLowerOut computes and
// writes only entries with j <= i (tiles above the diagonal are skipped);
// kLowerA (A[i][k] = 0 for k > i) and kLowerB (B'[k][j] = 0 for j > k) shorten
// each tile's contraction range to the part that can be non-zero.  256 threads
// per 16R x 16R tile, R x R outputs each (rows ty + 16 r, columns tx + 16 c),
// K in steps of 16 through shared memory, the next step's tiles fetched into
// registers while the current one is consumed.  Every CTA reads all the A
// rows it writes before its first store (the last barrier of the K loop
// separates them), so C may be A itself when N fits one tile column.
namespace {
constexpr int GK = 16;
constexpr int kLowerOut = 1, kLowerA = 2, kLowerB = 4;
}

template <bool B_KMAJOR, int R>
__global__ void __launch_bounds__(256) dgemm_kernel(int M, int N, int K, const double *A, int64_t lda,
                                                    const double *__restrict__ B, int64_t ldb, double *C,
                                                    int64_t ldc, double alpha, double beta, int flags)
{
    constexpr int GT = 16 * R;
    const int i0 = blockIdx.y * GT, j0 = blockIdx.x * GT;
    if ((flags & kLowerOut) && j0 > i0 + GT - 1) return;
    int k_lo = 0, k_hi = K;
    if (flags & kLowerB) k_lo = j0;                          // B'[k][j] = 0 for k < j
    if (flags & kLowerA) k_hi = min(K, i0 + GT);             // A[i][k] = 0 for k > i
    k_lo = (k_lo / GK) * GK;
    __shared__ double As[GK][GT + 2];
    __shared__ double Bs[GK][GT + 2];
    const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
    double acc[R][R];
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
        for (int c = 0; c < R; ++c) acc[r][c] = 0.0;
    // tile loads: A rows (i0 + lr, k0 + lk .. + R-1), one R-wide strip per thread
    const int lr = tid / (GK / R), lk = (tid % (GK / R)) * R;
    double ra[R], rb[R];
    auto fetch = [&](int k0) {
#pragma unroll
        for (int u = 0; u < R; ++u) {
            const int i = i0 + lr, k = k0 + lk + u;
            ra[u] = (i < M && k < k_hi) ? A[(int64_t)i * lda + k] : 0.0;
        }
        if (B_KMAJOR) {
#pragma unroll
            for (int u = 0; u < R; ++u) {
                const int j = j0 + lr, k = k0 + lk + u;
                rb[u] = (j < N && k < k_hi) ? B[(int64_t)j * ldb + k] : 0.0;
            }
        } else {
            // B rows k0 + (tid >> 4), columns j0 + (tid & 15) * R .. + R-1
            const int k = k0 + (tid >> 4), jb = j0 + (tid & 15) * R;
#pragma unroll
            for (int u = 0; u < R; ++u)
                rb[u] = (k < k_hi && jb + u < N) ? B[(int64_t)k * ldb + jb + u] : 0.0;
        }
    };
    auto stash = [&]() {
#pragma unroll
        for (int u = 0; u < R; ++u) As[lk + u][lr] = ra[u];
        if (B_KMAJOR) {
#pragma unroll
            for (int u = 0; u < R; ++u) Bs[lk + u][lr] = rb[u];
        } else {
#pragma unroll
            for (int u = 0; u < R; ++u) Bs[tid >> 4][(tid & 15) * R + u] = rb[u];
        }
    };
    if (k_lo < k_hi) fetch(k_lo);
    for (int k0 = k_lo; k0 < k_hi; k0 += GK) {
        stash();
        __syncthreads();
        if (k0 + GK < k_hi) fetch(k0 + GK);  // in flight while this step is consumed
#pragma unroll
        for (int kk = 0; kk < GK; ++kk) {
            double a[R], b[R];
#pragma unroll
            for (int r = 0; r < R; ++r) a[r] = As[kk][ty + 16 * r];
#pragma unroll
            for (int c = 0; c < R; ++c) b[c] = Bs[kk][tx + 16 * c];
#pragma unroll
            for (int r = 0; r < R; ++r)
#pragma unroll
                for (int c = 0; c < R; ++c) acc[r][c] = fma(a[r], b[c], acc[r][c]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
        for (int c = 0; c < R; ++c) {
            const int i = i0 + ty + 16 * r, j = j0 + tx + 16 * c;
            if (i >= M || j >= N) continue;
            if ((flags & kLowerOut) && j > i) continue;
            double *o = C + (int64_t)i * ldc + j;
            *o = beta == 0.0 ? alpha * acc[r][c] : fma(alpha, acc[r][c], beta * *o);
        }
}

namespace {
template <int R>
cudaError_t dgemm_r(int M, int N, int K, const double *A, int64_t lda, const double *B, int64_t ldb, bool b_kmajor,
                    double *C, int64_t ldc, double alpha, double beta, int flags, cudaStream_t stream)
{
    if (M <= 0 || N <= 0) return cudaSuccess;
    constexpr int GT = 16 * R;
    const dim3 grid((unsigned)((N + GT - 1) / GT), (unsigned)((M + GT - 1) / GT));
    if (b_kmajor)
        dgemm_kernel<true, R><<<grid, 256, 0, stream>>>(M, N, K, A, lda, B, ldb, C, ldc, alpha, beta, flags);
    else
        dgemm_kernel<false, R><<<grid, 256, 0, stream>>>(M, N, K, A, lda, B, ldb, C, ldc, alpha, beta, flags);
    return cudaGetLastError();
}

// 128 x 128 tiles where the output fills enough of them, 64 x 64 otherwise
cudaError_t dgemm(int M, int N, int K, const double *A, int64_t lda, const double *B, int64_t ldb, bool b_kmajor,
                  double *C, int64_t ldc, double alpha, double beta, int flags, cudaStream_t stream)
{
    const int64_t big = (int64_t)((M + 127) / 128) * ((N + 127) / 128);
    if (big >= 148 && N > 64)
        return dgemm_r<8>(M, N, K, A, lda, B, ldb, b_kmajor, C, ldc, alpha, beta, flags, stream);
    return dgemm_r<4>(M, N, K, A, lda, B, ldb, b_kmajor, C, ldc, alpha, beta, flags, stream);
}
}  // namespace

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

namespace {
// Y[i0:i0+len, i0:i0+len] = C[...]^-1 (lower) given the inverses of its
// 64 x 64 diagonal blocks in Y: split at a multiple of 64 near the middle,
// invert both halves, then Y21 = -Y22 (C21 Y11) through T.
cudaError_t trinv_rec(const double *C, double *Y, double *T, int64_t ld, int64_t i0, int64_t len,
                      cudaStream_t stream)
{
    if (len <= NB) return cudaSuccess;
    const int64_t h = ((len + 2 * NB - 1) / (2 * NB)) * NB;
    cudaError_t e = trinv_rec(C, Y, T, ld, i0, h, stream);
    if (e == cudaSuccess) e = trinv_rec(C, Y, T, ld, i0 + h, len - h, stream);
    if (e != cudaSuccess) return e;
    const int m2 = (int)(len - h), m1 = (int)h;
    e = dgemm(m2, m1, m1, C + (i0 + h) * ld + i0, ld, Y + i0 * ld + i0, ld, false, T, m1, 1.0, 0.0, kLowerB, stream);
    if (e != cudaSuccess) return e;
    return dgemm(m2, m1, m2, Y + (i0 + h) * ld + (i0 + h), ld, T, m1, false, Y + (i0 + h) * ld + i0, ld, -1.0, 0.0,
                 kLowerA, stream);
}
}  // namespace

size_t factor_work_doubles(int64_t n) { return (size_t)n * n * 2 + (size_t)(n / 2 + NB) * (n / 2 + NB); }

cudaError_t launch_factor(const float *A, int64_t n, float *L, double *work, DeviceStatus *st,
                          cudaStream_t stream)
{
    if (n <= 0) return cudaSuccess;
    double *C = work, *Y = work + n * n, *T = work + 2 * n * n;
    int64_t elems = n * n;
    int g = (int)min64((elems + 255) / 256, 148 * 16);
    rev_copy_kernel<<<g, 256, 0, stream>>>(A, n, C, st);
    // Y's zeros above the diagonal blocks are read by the inverse's merges
    cudaError_t e = cudaMemsetAsync(Y, 0, (size_t)n * n * sizeof(double), stream);
    if (e != cudaSuccess) return e;
    for (int64_t kb = 0; kb < n; kb += NB) {
        const int bs = (int)min64(NB, n - kb);
        potrf_inv_kernel<<<1, 256, 0, stream>>>(C, Y, n, kb, bs, st);
        const int64_t rest = n - kb - bs;
        if (rest > 0) {
            // panel P = C[kb+bs:, kb:kb+bs] <- P C_kk^-T, in place
            double *P = C + (kb + bs) * n + kb;
            e = dgemm((int)rest, bs, bs, P, n, Y + kb * n + kb, n, true, P, n, 1.0, 0.0, 0, stream);
            // C22 -= P P^T on the lower triangle
            if (e == cudaSuccess)
                e = dgemm((int)rest, (int)rest, bs, P, n, P, n, true, C + (kb + bs) * n + kb + bs, n, -1.0, 1.0,
                          kLowerOut, stream);
            if (e != cudaSuccess) return e;
        }
    }
    // Y = C^-1 from the diagonal blocks' inverses
    if ((e = trinv_rec(C, Y, T, n, 0, n, stream)) != cudaSuccess) return e;
    write_factor_kernel<<<g, 256, 0, stream>>>(Y, n, L);
    return cudaGetLastError();
}

}  // namespace bakron
