// leaf_common.cuh -- device helpers shared by the leaf sweep kernels: named
// barriers, packed FP32 fused multiply-adds, the 3xTF32 mma.sync block
// product, 16-byte asynchronous copies and the code byte.
#pragma once

#include <stdint.h>

#include "common.cuh"

namespace bakron {
namespace leafk {

__device__ __forceinline__ void group_sync(int id, int nthreads)
{
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// Two FP32 fused multiply-adds in one packed instruction (sm_100), each
// rounded to nearest like fmaf.
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c)
{
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
        "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
    return d;
}

__device__ __forceinline__ void mma_tf32(float (&c)[4], const uint32_t (&a)[4], const uint32_t (&b)[2])
{
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

// acc (a 16 x 8*NT block at (i0, j0) of a 32 x 32 product) += sum_{k<K} A[i][k] Bm[j][k]
template <int NT>
__device__ __forceinline__ void mma_block(float (&acc)[NT][4], const float *A, int lda, const float *Bm, int ldb,
                                          int K, int i0, int j0)
{
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
#pragma unroll 4
    for (int k0 = 0; k0 < K; k0 += 8) {
        const float af[4] = {A[(i0 + g) * lda + k0 + t], A[(i0 + g + 8) * lda + k0 + t],
                             A[(i0 + g) * lda + k0 + t + 4], A[(i0 + g + 8) * lda + k0 + t + 4]};
        uint32_t ahi[4], alo[4];
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            float h, l;
            split_tf32(af[r], h, l);
            ahi[r] = __float_as_uint(h);
            alo[r] = __float_as_uint(l);
        }
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const int j = j0 + nt * 8 + g;
            const float bf[2] = {Bm[j * ldb + k0 + t], Bm[j * ldb + k0 + t + 4]};
            uint32_t bhi[2], blo[2];
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                float h, l;
                split_tf32(bf[r], h, l);
                bhi[r] = __float_as_uint(h);
                blo[r] = __float_as_uint(l);
            }
            mma_tf32(acc[nt], alo, bhi);
            mma_tf32(acc[nt], ahi, blo);
            mma_tf32(acc[nt], ahi, bhi);
        }
    }
}

// The 32 x 32 product blocks of a row block's three warps: warps 0 and 1 take
// rows 0-15 / 16-31 of columns 0-23 (three 8-wide column tiles), warp 2 the
// last column tile for all 32 rows.
template <int NT>
__device__ __forceinline__ void store_block(const float (&acc)[NT][4], float *o, int ldo, int i0, int j0)
{
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        const int j = j0 + nt * 8 + 2 * t;
        o[(i0 + g) * ldo + j] = acc[nt][0];
        o[(i0 + g) * ldo + j + 1] = acc[nt][1];
        o[(i0 + g + 8) * ldo + j] = acc[nt][2];
        o[(i0 + g + 8) * ldo + j + 1] = acc[nt][3];
    }
}

// W0 = Wt - acc - S into the slot o (which holds S when has_s), and R's block
// rq (which holds Wt) becomes S.
template <int NT>
__device__ __forceinline__ void finish_w0(const float (&acc)[NT][4], float *o, int ldo, float *rq, int ldr, int i0,
                                          int j0, bool has_s)
{
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int h = 0; h < 4; ++h) {
            const int i = i0 + g + 8 * (h >> 1), j = j0 + nt * 8 + 2 * t + (h & 1);
            const float sv = has_s ? o[i * ldo + j] : 0.f;
            const float wt = rq[i * ldr + j];
            o[i * ldo + j] = wt - acc[nt][h] - sv;
            rq[i * ldr + j] = sv;
        }
}

// acc = A (32 x K) Bm (32 x K)^T over a row block's three warps (role 0..2):
// the split of store_block / finish_w0.  K may be 0 (acc stays zero).
struct Block3 {
    float a3[3][4];
    float a1[2][1][4];
};
__device__ __forceinline__ void product3(Block3 &b, int role, const float *A, int lda, const float *Bm, int ldb, int K)
{
#pragma unroll
    for (int i = 0; i < 3; ++i)
#pragma unroll
        for (int c = 0; c < 4; ++c) b.a3[i][c] = 0.f;
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
        for (int c = 0; c < 4; ++c) b.a1[i][0][c] = 0.f;
    if (K <= 0) return;
    if (role < 2) {
        mma_block<3>(b.a3, A, lda, Bm, ldb, K, 16 * role, 0);
    } else {
        mma_block<1>(b.a1[0], A, lda, Bm, ldb, K, 0, 24);
        mma_block<1>(b.a1[1], A, lda, Bm, ldb, K, 16, 24);
    }
}
__device__ __forceinline__ void store3(const Block3 &b, int role, float *o, int ldo)
{
    if (role < 2) {
        store_block<3>(b.a3, o, ldo, 16 * role, 0);
    } else {
        store_block<1>(b.a1[0], o, ldo, 0, 24);
        store_block<1>(b.a1[1], o, ldo, 16, 24);
    }
}
__device__ __forceinline__ void finish3(const Block3 &b, int role, float *o, int ldo, float *rq, int ldr, bool has_s)
{
    if (role < 2) {
        finish_w0<3>(b.a3, o, ldo, rq, ldr, 16 * role, 0, has_s);
    } else {
        finish_w0<1>(b.a1[0], o, ldo, rq, ldr, 0, 24, has_s);
        finish_w0<1>(b.a1[1], o, ldo, rq, ldr, 16, 24, has_s);
    }
}

// Byte of an integer-valued float in [-128, 127] (two's complement) without a
// conversion instruction: adding 1.5 * 2^23 puts the integer in the low
// mantissa bits.
__device__ __forceinline__ int8_t code_byte(float c)
{
    return (int8_t)(__float_as_int(c + 12582912.0f) & 0xFF);
}

__device__ __forceinline__ void cp_async16(void *dst, const void *src)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"((uint32_t)__cvta_generic_to_shared(dst)),
                 "l"(src)
                 : "memory");
}

}  // namespace leafk
}  // namespace bakron
