// prep.cu -- per-solve preparation: grid steps, padded working copy of W, and
// the normalised factors (unit diagonal, "normalized Cholesky factors" of the
// review's circularity check) with their TF32 hi/lo split.
#include "common.cuh"
#include "kernels.cuh"

namespace bakron {

// One warp per row: s_i = max_j |W_ij| / qmax (IEEE fp32 division), 1 for a
// zero row; or the caller's step, checked positive and finite.
__global__ void scales_kernel(const float *__restrict__ W, int64_t m, int64_t n, int qmax,
                              const float *__restrict__ user, float *__restrict__ s,
                              DeviceStatus *st)
{
    pdl_wait();
    pdl_trigger();
    int64_t row = (int64_t)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
    int lane = threadIdx.x & 31;
    if (row >= m) return;
    const float *w = W + row * n;
    float amax = 0.f;
    bool finite = true;
    for (int64_t j = lane; j < n; j += 32) {
        float x = w[j];
        finite &= isfinite(x);
        amax = fmaxf(amax, fabsf(x));
    }
    for (int o = 16; o; o >>= 1) {
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        finite = __all_sync(0xffffffffu, finite);
    }
    if (lane == 0) {
        if (!finite) record_error(st, BAKRON_ERR_NONFINITE, (int)row);
        float sv;
        if (user) {
            sv = user[row];
            if (!(sv > 0.f) || !isfinite(sv)) {
                record_error(st, BAKRON_ERR_INVALID_ARG, (int)row);
                sv = 1.f;
            }
        } else {
            sv = amax > 0.f ? __fdiv_rn(amax, (float)qmax) : 1.f;
        }
        s[row] = sv;
    }
}

// Steps searched for the least round-to-nearest error of each row (the
// review's free parameter "per-row scaling factor (shrink) up to factor 2,
// MSE search"): one CTA per row; candidates c_k = 1 - fp32(k/2)/fp32(G-1),
// s_k = fp32(fp32(c_k * absmax) / qmax); error sum_j (W_ij - s_k q_ij)^2 with
// q = clamp(rint(fp32(W_ij / s_k))) summed in FP64; the first k with the
// smallest error wins.  Eight candidates share each pass over the row.
constexpr int kMseThreads = 256;
constexpr int kMseBatch = 8;
__global__ void __launch_bounds__(kMseThreads) scales_mse_kernel(const float *__restrict__ W, int64_t m, int64_t n,
                                                                  int qmin, int qmax, int grid,
                                                                  float *__restrict__ s, DeviceStatus *st)
{
    pdl_wait();
    pdl_trigger();
    __shared__ float red_f[kMseThreads / 32];
    __shared__ double red_d[kMseThreads / 32][kMseBatch];
    __shared__ int bad_sh;
    const int64_t row = blockIdx.x;
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    if (row >= m) return;
    const float *w = W + row * n;
    float amax = 0.f;
    bool finite = true;
    for (int64_t j = tid; j < n; j += kMseThreads) {
        const float x = w[j];
        finite &= isfinite(x);
        amax = fmaxf(amax, fabsf(x));
    }
    for (int o = 16; o; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const int any_bad = __syncthreads_or(!finite);
    if (lane == 0) red_f[wid] = amax;
    __syncthreads();
    if (tid == 0) {
        float a = 0.f;
        for (int i = 0; i < kMseThreads / 32; ++i) a = fmaxf(a, red_f[i]);
        red_f[0] = a;
        bad_sh = any_bad;
    }
    __syncthreads();
    amax = red_f[0];
    if (bad_sh) {
        if (tid == 0) {
            record_error(st, BAKRON_ERR_NONFINITE, (int)row);
            s[row] = 1.f;
        }
        return;
    }
    if (!(amax > 0.f)) {
        if (tid == 0) s[row] = 1.f;
        return;
    }
    const float fqmin = (float)qmin, fqmax = (float)qmax, fq = (float)qmax, gm1 = (float)(grid - 1);
    double best = 0.0;
    float best_s = 1.f;
    for (int k0 = 0; k0 < grid; k0 += kMseBatch) {
        float sk[kMseBatch], rk[kMseBatch];
        bool ieee = false;
#pragma unroll
        for (int b = 0; b < kMseBatch; ++b) {
            const int k = min(k0 + b, grid - 1);
            const float c = __fsub_rn(1.f, __fdiv_rn(0.5f * (float)k, gm1));
            sk[b] = __fdiv_rn(__fmul_rn(c, amax), fq);
            rk[b] = __frcp_rn(sk[b]);
            ieee |= !(sk[b] >= 0x1p-60f && sk[b] <= 0x1p60f);
        }
        double e[kMseBatch] = {};
        for (int64_t j = tid; j < n; j += kMseThreads) {
            const float x = w[j];
            const double xd = (double)x;
#pragma unroll
            for (int b = 0; b < kMseBatch; ++b) {
                const float qf = ieee ? __fdiv_rn(x, sk[b]) : div_rn_recip(x, sk[b], rk[b]);
                const float c = fminf(fmaxf(rintf(qf), fqmin), fqmax);
                const double d = xd - (double)sk[b] * (double)c;
                e[b] = fma(d, d, e[b]);
            }
        }
#pragma unroll
        for (int b = 0; b < kMseBatch; ++b) {
            double v = e[b];
            for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
            if (lane == 0) red_d[wid][b] = v;
        }
        __syncthreads();
        if (tid == 0) {
            for (int b = 0; b < kMseBatch && k0 + b < grid; ++b) {
                double v = 0.0;
                for (int i = 0; i < kMseThreads / 32; ++i) v += red_d[i][b];
                if (k0 + b == 0 || v < best) {
                    best = v;
                    best_s = sk[b];
                }
            }
        }
        __syncthreads();
    }
    if (tid == 0) s[row] = best_s;
}

// Wt (Mp x Np) <- W zero-padded; Dhi, Dlo <- 0.
__global__ void pad_copy_kernel(const float *__restrict__ W, int64_t m, int64_t n, int64_t Np,
                                int64_t Mp, float *__restrict__ Wt, float *__restrict__ Dhi,
                                float *__restrict__ Dlo)
{
    pdl_wait();
    pdl_trigger();
    int64_t total = Mp * Np;
    for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
         idx += (int64_t)gridDim.x * blockDim.x) {
        int64_t r = idx / Np, c = idx - r * Np;
        Wt[idx] = (r < m && c < n) ? W[r * n + c] : 0.f;
        Dhi[idx] = 0.f;
        Dlo[idx] = 0.f;
    }
}

// Lt (Np x Np) <- L * diag(L)^{-1} on the lower triangle (exact 1 on the
// diagonal), zero elsewhere and in the padding; plus its TF32 hi/lo split.
__global__ void normalize_split_kernel(const float *__restrict__ L, int64_t n, int64_t Np,
                                       float *__restrict__ L32, float *__restrict__ Lhi,
                                       float *__restrict__ Llo, DeviceStatus *st)
{
    pdl_wait();
    pdl_trigger();
    int64_t total = Np * Np;
    for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
         idx += (int64_t)gridDim.x * blockDim.x) {
        int64_t r = idx / Np, c = idx - r * Np;
        float v = 0.f;
        if (r < n && c < n && c <= r) {
            float d = L[c * n + c];
            if (r == c) {
                if (!(d > 0.f) || !isfinite(d)) record_error(st, BAKRON_ERR_BAD_FACTOR, (int)c);
                v = 1.f;
            } else {
                v = __fdiv_rn(L[r * n + c], d);
            }
        }
        float hi, lo;
        split_tf32(v, hi, lo);
        L32[idx] = v;
        Lhi[idx] = hi;
        Llo[idx] = lo;
    }
}

static int grid_for(int64_t total, int threads)
{
    int64_t b = (total + threads - 1) / threads;
    if (b > 148 * 16) b = 148 * 16;
    return (int)(b < 1 ? 1 : b);
}

cudaError_t launch_prep(const float *W, int64_t m, int64_t n, const float *LA, const float *LB, int qmin,
                        int qmax, const float *user_scales, int shrink_grid, float *scales, const SolveLayout &L,
                        char *ws, cudaStream_t stream)
{
    DeviceStatus *st = (DeviceStatus *)(ws + L.status);
    cudaError_t e;
    if (shrink_grid >= 2 && !user_scales)
        e = launch_pdl(scales_mse_kernel, dim3((unsigned)m), dim3(kMseThreads), 0, stream, W, m, n, qmin, qmax,
                       shrink_grid, scales, st);
    else
        e = launch_pdl(scales_kernel, dim3((unsigned)((m + 7) / 8)), dim3(256), 0, stream, W, m, n, qmax,
                       user_scales, scales, st);
    if (e != cudaSuccess) return e;
    if ((e = launch_pdl(pad_copy_kernel, dim3(grid_for(L.Mp * L.Np, 256)), dim3(256), 0, stream, W, m, n, L.Np,
                        L.Mp, (float *)(ws + L.Wt), (float *)(ws + L.Dhi), (float *)(ws + L.Dlo))) != cudaSuccess)
        return e;
    if ((e = launch_pdl(normalize_split_kernel, dim3(grid_for(L.Np * L.Np, 256)), dim3(256), 0, stream, LA, n,
                        L.Np, (float *)(ws + L.LA32), (float *)(ws + L.LAhi), (float *)(ws + L.LAlo), st)) !=
        cudaSuccess)
        return e;
    if (!LB) return cudaSuccess;  // the one-sided path (B = I) has no output-side factor
    return launch_pdl(normalize_split_kernel, dim3(grid_for(L.Mp * L.Mp, 256)), dim3(256), 0, stream, LB, m, L.Mp,
                      (float *)(ws + L.LB32), (float *)(ws + L.LBhi), (float *)(ws + L.LBlo), st);
}

}  // namespace bakron
