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
// symmetric update as GEMMs) and a triangular inverse built bottom-up from
// the diagonal blocks' inverses, inv([[A, 0], [B, C]]) = [[A^-1, 0],
// [-C^-1 B A^-1, C^-1]], each level's merges two batched GEMMs; all FP64.
// The GEMM runs on the FP64 tensor cores (128 x 128 or 64 x 64 output tiles)
// and skips the zero halves of triangular operands.
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
// with A row-major (lda) and B' = B row-major K x N (ldb) or, with B_KMAJOR,
// B' = B^T for B row-major N x K; on the FP64 tensor cores
// (mma.sync.m8n8k4.f64).  flags: kLowerOut computes and writes only entries
// with j <= i (tiles above the diagonal are skipped); kLowerA
// (A[i][k] = 0 for k > i) and kLowerB (B'[k][j] = 0 for j > k) shorten each
// tile's contraction range to the part that can be non-zero.  Batched over
// blockIdx.z: problem z reads A + z sA, B + z sB and writes C + z sC, the last
// one with M_last rows and contraction length K_last.  256 threads per
// TM x TN tile as 2 x 4 warps; K in steps of 16 through shared memory (k-major
// rows padded by 8 doubles so the fragment loads take two wavefronts), the
// next step's tiles fetched into registers while the current one is
// consumed.  Every CTA reads all the A rows it writes before its first store
// (the last barrier of the K loop separates them), so C may be A itself when
// N fits one tile column.
namespace {
constexpr int GK = 16;
constexpr int kLowerOut = 1, kLowerA = 2, kLowerB = 4;

struct GemmD {
    int M, N, K, M_last, K_last;
    const double *A;
    int64_t lda, sA;
    const double *B;
    int64_t ldb, sB;
    double *C;
    int64_t ldc, sC;
    double alpha, beta;
    int flags;
};

__device__ __forceinline__ void dmma(double (&c)[2], double a, double b)
{
    asm volatile("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0, %1}, {%2}, {%3}, {%0, %1};"
                 : "+d"(c[0]), "+d"(c[1])
                 : "d"(a), "d"(b));
}
}  // namespace

template <bool B_KMAJOR, int TM, int TN>
__global__ void __launch_bounds__(256) dgemm_kernel(GemmD g)
{
    constexpr int WTM = TM / 2, WTN = TN / 4, MT = WTM / 8, NT = WTN / 8;
    constexpr int EA = TM / 16, EB = TN / 16;  // elements per thread of an A / B step tile
    const int z = blockIdx.z;
    const bool last = z == (int)gridDim.z - 1;
    const int M = last ? g.M_last : g.M, N = g.N, K = last ? g.K_last : g.K;
    const double *A = g.A + z * g.sA, *B = g.B + z * g.sB;
    double *C = g.C + z * g.sC;
    const int i0 = blockIdx.y * TM, j0 = blockIdx.x * TN;
    if (i0 >= M) return;
    if ((g.flags & kLowerOut) && j0 > i0 + TM - 1) return;
    int k_lo = 0, k_hi = K;
    if (g.flags & kLowerB) k_lo = j0;                  // B'[k][j] = 0 for k < j
    if (g.flags & kLowerA) k_hi = min(K, i0 + TM);     // A[i][k] = 0 for k > i
    k_lo = (k_lo / GK) * GK;
    __shared__ double As[GK][TM + 8];
    __shared__ double Bs[GK][TN + 8];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int wm = warp >> 2, wn = warp & 3;
    double acc[MT][NT][2];
#pragma unroll
    for (int a = 0; a < MT; ++a)
#pragma unroll
        for (int b = 0; b < NT; ++b) acc[a][b][0] = acc[a][b][1] = 0.0;
    // step tiles: A rows (i0 + lr, k0 + lk .. + EA-1) per thread; B likewise
    const int lr = tid / (GK / EA), lk = (tid % (GK / EA)) * EA;
    const int br = tid / (GK / EB), bk = (tid % (GK / EB)) * EB;
    double ra[EA], rb[EB];
    auto fetch = [&](int k0) {
#pragma unroll
        for (int u = 0; u < EA; ++u) {
            const int i = i0 + lr, k = k0 + lk + u;
            ra[u] = (i < M && k < k_hi) ? A[(int64_t)i * g.lda + k] : 0.0;
        }
        if (B_KMAJOR) {
#pragma unroll
            for (int u = 0; u < EB; ++u) {
                const int j = j0 + br, k = k0 + bk + u;
                rb[u] = (j < N && k < k_hi) ? B[(int64_t)j * g.ldb + k] : 0.0;
            }
        } else {
            // B rows k0 + (tid >> 4), columns j0 + (tid & 15) * EB .. + EB-1
            const int k = k0 + (tid >> 4), jb = j0 + (tid & 15) * EB;
#pragma unroll
            for (int u = 0; u < EB; ++u)
                rb[u] = (k < k_hi && jb + u < N) ? B[(int64_t)k * g.ldb + jb + u] : 0.0;
        }
    };
    auto stash = [&]() {
#pragma unroll
        for (int u = 0; u < EA; ++u) As[lk + u][lr] = ra[u];
        if (B_KMAJOR) {
#pragma unroll
            for (int u = 0; u < EB; ++u) Bs[bk + u][br] = rb[u];
        } else {
#pragma unroll
            for (int u = 0; u < EB; ++u) Bs[tid >> 4][(tid & 15) * EB + u] = rb[u];
        }
    };
    // fragment coordinates: A (8 x 4) row lane/4, column lane%4; B (4 x 8)
    // row lane%4, column lane/4; C (8 x 8) row lane/4, columns 2 (lane%4) + e
    const int fr = lane >> 2, fk = lane & 3;
    if (k_lo < k_hi) fetch(k_lo);
    for (int k0 = k_lo; k0 < k_hi; k0 += GK) {
        stash();
        __syncthreads();
        if (k0 + GK < k_hi) fetch(k0 + GK);  // in flight while this step is consumed
#pragma unroll
        for (int kk = 0; kk < GK; kk += 4) {
            double af[MT], bf[NT];
#pragma unroll
            for (int a = 0; a < MT; ++a) af[a] = As[kk + fk][wm * WTM + a * 8 + fr];
#pragma unroll
            for (int b = 0; b < NT; ++b) bf[b] = Bs[kk + fk][wn * WTN + b * 8 + fr];
#pragma unroll
            for (int a = 0; a < MT; ++a)
#pragma unroll
                for (int b = 0; b < NT; ++b) dmma(acc[a][b], af[a], bf[b]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int a = 0; a < MT; ++a)
#pragma unroll
        for (int b = 0; b < NT; ++b)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int i = i0 + wm * WTM + a * 8 + fr, j = j0 + wn * WTN + b * 8 + 2 * fk + e;
                if (i >= M || j >= N) continue;
                if ((g.flags & kLowerOut) && j > i) continue;
                double *o = C + (int64_t)i * g.ldc + j;
                *o = g.beta == 0.0 ? g.alpha * acc[a][b][e] : fma(g.alpha, acc[a][b][e], g.beta * *o);
            }
}

namespace {
template <int TM, int TN>
cudaError_t dgemm_t(const GemmD &g, bool b_kmajor, int nz, cudaStream_t stream)
{
    const int Mmax = max(g.M, g.M_last);
    if (Mmax <= 0 || g.N <= 0 || nz <= 0) return cudaSuccess;
    const dim3 grid((unsigned)((g.N + TN - 1) / TN), (unsigned)((Mmax + TM - 1) / TM), (unsigned)nz);
    if (b_kmajor)
        dgemm_kernel<true, TM, TN><<<grid, 256, 0, stream>>>(g);
    else
        dgemm_kernel<false, TM, TN><<<grid, 256, 0, stream>>>(g);
    return cudaGetLastError();
}

// 128 x 128 tiles where the outputs fill enough of them, 64 x 64 otherwise
cudaError_t dgemm_batched(const GemmD &g, bool b_kmajor, int nz, cudaStream_t stream)
{
    const int64_t big = (int64_t)nz * ((g.M + 127) / 128) * ((g.N + 127) / 128);
    if (big >= 148 && g.N > 64) return dgemm_t<128, 128>(g, b_kmajor, nz, stream);
    return dgemm_t<64, 64>(g, b_kmajor, nz, stream);
}

cudaError_t dgemm(int M, int N, int K, const double *A, int64_t lda, const double *B, int64_t ldb, bool b_kmajor,
                  double *C, int64_t ldc, double alpha, double beta, int flags, cudaStream_t stream)
{
    const GemmD g{M, N, K, M, K, A, lda, 0, B, ldb, 0, C, ldc, 0, alpha, beta, flags};
    return dgemm_batched(g, b_kmajor, 1, stream);
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
// Y = C^-1 (lower, n x n, leading dimension n) given the inverses of C's
// 64 x 64 diagonal blocks in Y, bottom-up: at block size s every pair of
// neighbouring blocks [i0, i0+s), [i0+s, min(i0+2s, n)) with i0 a multiple of
// 2s is merged, Y21 = -Y22 (C21 Y11), all merges of a level in one batched
// launch per product (T holds C21 Y11, s x s per merge).
cudaError_t trinv_levels(const double *C, double *Y, double *T, int64_t n, cudaStream_t stream)
{
    for (int64_t s = NB; s < n; s *= 2) {
        const int nz = (int)((n - s + 2 * s - 1) / (2 * s));
        const int m2_last = (int)min64(s, n - ((int64_t)(nz - 1) * 2 * s + s));
        const int64_t step = 2 * s * (n + 1);  // from one merge's block to the next
        const int si = (int)s;
        const GemmD g1{si, si, si, m2_last, si, C + s * n, n, step, Y, n, step, T, s, s * s, 1.0, 0.0, kLowerB};
        cudaError_t e = dgemm_batched(g1, false, nz, stream);
        if (e != cudaSuccess) return e;
        const GemmD g2{si, si, si, m2_last, m2_last, Y + s * n + s, n, step, T, s, s * s, Y + s * n, n, step,
                       -1.0, 0.0, kLowerA};
        if ((e = dgemm_batched(g2, false, nz, stream)) != cudaSuccess) return e;
    }
    return cudaSuccess;
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
    if ((e = trinv_levels(C, Y, T, n, stream)) != cudaSuccess) return e;
    write_factor_kernel<<<g, 256, 0, stream>>>(Y, n, L);
    return cudaGetLastError();
}

}  // namespace bakron
