// Checks div_rn_recip (the division used by the rounding decisions) against
// CUDA's IEEE division __fdiv_rn on random and adversarial fp32 pairs with b in
// [2^-60, 2^60]: quotients next to half-integers (the rounding decision's
// midpoints) for every significand of b in [1, 2), random pairs over the
// normal range, and weight-like magnitudes.  The quotient must match bit for
// bit when |a| >= 2^-100, and rint(quotient) must match for every pair.
#include <cstdio>
#include <cstdint>

#include "common.cuh"

__device__ __forceinline__ uint64_t mix64(uint64_t z)  // splitmix64 finaliser
{
    z += 0x9E3779B97F4A7C15ull;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

__global__ void check_kernel(uint64_t n, int mode, unsigned long long *bad, float *first, unsigned long long *bad_dec)
{
    for (uint64_t i = blockIdx.x * (uint64_t)blockDim.x + threadIdx.x; i < n; i += (uint64_t)gridDim.x * blockDim.x) {
        const uint64_t h = mix64(i * 4 + mode);
        float a, b;
        if (mode == 0) {
            // b: every significand in [1, 2) (n = 2^23 * k), times a random power of two
            const uint32_t sig = (uint32_t)(i & 0x7FFFFFu);
            const int e = (int)((h >> 8) % 121) - 60;
            b = ldexpf(__uint_as_float(0x3F800000u | sig), e);
            // a: b times (c + 1/2), nudged by a few ulps
            const float c = (float)((int)(h % 17) - 8) + 0.5f;
            const int nudge = (int)((h >> 40) % 9) - 4;
            a = __uint_as_float(__float_as_uint(b * c) + nudge);
        } else if (mode == 1) {
            // random signs, significands and exponents over the normal range
            // b over [2^-60, 2^60], a over the whole normal range
            b = __uint_as_float((uint32_t)(h & 0x807FFFFFu) | ((uint32_t)(127 - 60 + (h >> 32) % 121) << 23));
            a = __uint_as_float((uint32_t)((h >> 23) & 0x807FFFFFu) | ((uint32_t)(1 + (h >> 48) % 254) << 23));
            const float qq = __fdiv_rn(a, b);
            if (!(fabsf(qq) < 0x1p100f)) continue;  // far beyond any grid: every decision clamps
        } else {
            // weight-like magnitudes: steps around 1e-4..1e-1, quotients within +-40
            b = ldexpf(__uint_as_float(0x3F800000u | (uint32_t)(h & 0x7FFFFFu)), -(int)(3 + (h >> 24) % 12));
            const float t = (float)((int64_t)((h >> 32) % 80001) - 40000) * 1e-3f;
            a = __uint_as_float(__float_as_uint(b * t) + (int)((h >> 60) % 5) - 2);
        }
        if (a != a) continue;  // a nudged below zero's bit pattern
        const float rb = __frcp_rn(b);
        const float q0 = __fdiv_rn(a, b);
        const float q1 = bakron::div_rn_recip(a, b, rb);
        if (rintf(q0) != rintf(q1)) atomicAdd(bad_dec, 1ull);
        if (fabsf(a) >= 0x1p-100f && __float_as_uint(q0) != __float_as_uint(q1)) {
            if (atomicAdd(bad, 1ull) == 0) {
                first[0] = a;
                first[1] = b;
                first[2] = q0;
                first[3] = q1;
            }
        }
    }
}

int main()
{
    unsigned long long *bad, *bad_dec;
    float *first;
    cudaMalloc(&bad, sizeof(unsigned long long));
    cudaMalloc(&bad_dec, sizeof(unsigned long long));
    cudaMalloc(&first, 4 * sizeof(float));
    const uint64_t counts[3] = {(uint64_t)1 << 23 << 5, (uint64_t)1 << 28, (uint64_t)1 << 28};
    int rc = 0;
    for (int mode = 0; mode < 3; ++mode) {
        cudaMemset(bad, 0, sizeof(unsigned long long));
        cudaMemset(bad_dec, 0, sizeof(unsigned long long));
        check_kernel<<<148 * 8, 256>>>(counts[mode], mode, bad, first, bad_dec);
        if (cudaDeviceSynchronize() != cudaSuccess) {
            printf("cuda error\n");
            return 2;
        }
        unsigned long long nb = 0, nd = 0;
        float f[4] = {0, 0, 0, 0};
        cudaMemcpy(&nb, bad, sizeof(nb), cudaMemcpyDeviceToHost);
        cudaMemcpy(&nd, bad_dec, sizeof(nd), cudaMemcpyDeviceToHost);
        cudaMemcpy(f, first, sizeof(f), cudaMemcpyDeviceToHost);
        printf("mode %d pairs %llu mismatches %llu decision_mismatches %llu", mode, (unsigned long long)counts[mode], nb, nd);
        if (nb) printf(" first a=%.9g b=%.9g ieee=%.9g recip=%.9g", f[0], f[1], f[2], f[3]);
        printf("\n");
        if (nb || nd) rc = 1;
    }
    return rc;
}
