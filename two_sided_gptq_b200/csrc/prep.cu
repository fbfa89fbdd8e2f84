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

cudaError_t launch_prep(const float *W, int64_t m, int64_t n, const float *LA, const float *LB,
                        int qmax, const float *user_scales, float *scales, const SolveLayout &L,
                        char *ws, cudaStream_t stream)
{
    DeviceStatus *st = (DeviceStatus *)(ws + L.status);
    cudaError_t e;
    if ((e = launch_pdl(scales_kernel, dim3((unsigned)((m + 7) / 8)), dim3(256), 0, stream, W, m, n, qmax,
                        user_scales, scales, st)) != cudaSuccess)
        return e;
    if ((e = launch_pdl(pad_copy_kernel, dim3(grid_for(L.Mp * L.Np, 256)), dim3(256), 0, stream, W, m, n, L.Np,
                        L.Mp, (float *)(ws + L.Wt), (float *)(ws + L.Dhi), (float *)(ws + L.Dlo))) != cudaSuccess)
        return e;
    if ((e = launch_pdl(normalize_split_kernel, dim3(grid_for(L.Np * L.Np, 256)), dim3(256), 0, stream, LA, n,
                        L.Np, (float *)(ws + L.LA32), (float *)(ws + L.LAhi), (float *)(ws + L.LAlo), st)) !=
        cudaSuccess)
        return e;
    return launch_pdl(normalize_split_kernel, dim3(grid_for(L.Mp * L.Mp, 256)), dim3(256), 0, stream, LB, m, L.Mp,
                      (float *)(ws + L.LB32), (float *)(ws + L.LBhi), (float *)(ws + L.LBlo), st);
}

}  // namespace bakron
