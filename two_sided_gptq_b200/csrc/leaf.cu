// leaf.cu -- the leaf sweep: rounds every entry of one tile diagonal.
//
// Tiles (I, J) with I + J = K are mutually incomparable in the product order
// (I < I' forces J > J'), so one CTA per tile runs independently.  Every
// contribution from outside the tile has already been subtracted from Wt by
// the band products; what remains is the tile's own share of Proposition
// 3.1's updates.
//
// Inside the T x T tile the same divide-and-conquer is applied once more:
// the tile is cut into 2 x 2 sub-tiles of S = T/2, processed in sub-tile
// diagonal order (0,0) -> {(0,1), (1,0)} -> (1,1) (again a linear extension of
// the product order), with the cross-sub-tile contributions applied as small
// S^3 products between the phases.  Within a sub-tile the entries are rounded
// one entry anti-diagonal per step (2S-1 steps), in the "pull" form
//     Wt_ab = W0_ab - sum_{b'<b} R_ab' LtA[b,b'] - sum_{a'<a} LtB[a,a'] D_a'b,
//     R_ab  = sum_{a'<=a} LtB[a,a'] D_a'b,
// where a, b index the sub-tile's rows and columns and the factor blocks are
// its diagonal blocks.  R (sub-tile local) is stored over W0 entry by entry.
//
// Cross-sub-tile terms (Sxy = LtB[1,0] D[0,y], blocks of the tile):
//   (0,1) -= R00 LtA[1,0]^T
//   (1,0) -= S10 LtA[0,0]^T
//   (1,1) -= (R10 + S10) LtA[1,0]^T + S11 LtA[1,1]^T
// computed with mma.sync m16n8k8 TF32 in 3xTF32 form (lo*hi + hi*lo + hi*hi).
#include "common.cuh"
#include "kernels.cuh"

namespace bakron {

namespace {
constexpr int T = kTile;           // 128
constexpr int S = T / 2;           // 64: sub-tile side of the two-level variant
constexpr int RS = T + 16;         // row stride of sR / sDt, two-level variant; RS/4 = 4 mod 8
constexpr int RS1 = T + 4;         // row stride of sR / sDt / sLB, single-level variant
constexpr int BS = S + 16;         // row stride of the LtB diagonal sub-blocks
constexpr int ZS = S + 4;          // row stride of the S-block scratch
constexpr int kThreads = 512;
constexpr size_t kSmemNested = ((size_t)2 * T * RS + 2 * S * BS + S * ZS + 2 * T) * sizeof(float);
constexpr size_t kSmemSingle = ((size_t)3 * T * RS1 + 2 * T) * sizeof(float);
static_assert(kSmemNested <= 232448 && kSmemSingle <= 232448, "leaf shared memory");

__device__ __forceinline__ void group_sync(int id, int nthreads)
{
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

__device__ __forceinline__ float4 mask4(float4 v, int len)  // keep the first len (<= 4) components
{
    v.x = len > 0 ? v.x : 0.f;
    v.y = len > 1 ? v.y : 0.f;
    v.z = len > 2 ? v.z : 0.f;
    v.w = len > 3 ? v.w : 0.f;
    return v;
}
__device__ __forceinline__ float dot4(const float4 a, const float4 b, float acc)
{
    acc = fmaf(a.x, b.x, acc);
    acc = fmaf(a.y, b.y, acc);
    acc = fmaf(a.z, b.z, acc);
    return fmaf(a.w, b.w, acc);
}

// Rounding decision clamp(rint(wt / s)) with the IEEE fp32 quotient.  Fast
// path: q = wt * (1/s) is within 2 ulp of the IEEE quotient; whenever q is
// not within 0.002 of a half-integer (and |q| <= 2^12, beyond which every
// grid clamps) both round to the same integer.  Otherwise the exact IEEE
// division decides.
__device__ __forceinline__ float decide(float wt, float s, float rs, float qmin, float qmax)
{
    const float q = wt * rs;
    float c = rintf(q);
    if (fabsf(q - c) > 0.498f && fabsf(q) <= 4096.f) c = rintf(__fdiv_rn(wt, s));
    return fminf(fmaxf(c, qmin), qmax);
}
}  // namespace

// Sweep one SS x SS sub-tile at tile offset (r0, c0) with TPC threads per
// column.  Thread (bl, q) owns column bl; its dot products cover the float4
// chunks ch = q + TPC*j of the SS-long rows.  `LB` is the sub-tile's LtB
// diagonal block in smem (row stride LBS); row bl of the LtA diagonal block
// sits in registers.  R and Dt live in smem with row stride RSS.  Codes go
// straight to global memory; V and the residual split are written after the
// last sweep from smem.
template <int SS, int TPC, int RSS, int LBS>
__device__ void sweep_subtile(const LeafArgs &p, float *sR, float *sDt, const float *LB, const float *scale,
                              const float *rcp, int r0, int c0, int64_t grow0, int64_t gcol0, int mr, int nc,
                              int gtid, int bar_id)
{
    constexpr int NT = SS * TPC;        // threads of this group
    constexpr int NCH = SS / 4 / TPC;   // chunks per thread
    constexpr int COLS_PER_WARP = 32 / TPC;
    const int bl = gtid / TPC, q = gtid % TPC;
    const int warp_bl0 = (gtid / 32) * COLS_PER_WARP;  // first column of this warp
    float4 la[NCH];
#pragma unroll
    for (int j = 0; j < NCH; ++j) {
        const int ch = q + TPC * j;
        la[j] = *(const float4 *)(p.LA32 + (gcol0 + c0 + bl) * p.Np + gcol0 + c0 + 4 * ch);
    }
    const unsigned gmask = (TPC >= 32) ? 0xFFFFFFFFu : (((1u << TPC) - 1u) << (threadIdx.x & (32 - TPC)));
    const float *Dcol = sDt + (c0 + bl) * RSS + r0;
    const int bmax = warp_bl0 + COLS_PER_WARP - 1;  // largest column of the warp
    const float fqmin = (float)p.qmin, fqmax = (float)p.qmax;
    for (int d = 0; d < 2 * SS - 1; ++d) {
        const int a = d - bl;
        const int amax = min(d - warp_bl0, SS - 1);  // largest row of the warp at this step
        if (a >= 0 && a < SS) {
            const float *Rrow = sR + (r0 + a) * RSS + c0;
            const float *Brow = LB + a * LBS;
            float u0 = 0.f, u1 = 0.f, s0 = 0.f, s1 = 0.f;
#pragma unroll
            for (int j = 0; j < NCH; ++j) {
                const int base = 4 * (q + TPC * j);
                if (4 * TPC * j < bmax) {  // warp-uniform: some thread of the warp needs chunk j
                    const float4 rv = mask4(*(const float4 *)(Rrow + base), bl - base);
                    if (j & 1) u1 = dot4(rv, la[j], u1); else u0 = dot4(rv, la[j], u0);
                }
                if (4 * TPC * j < amax) {  // warp-uniform
                    const float4 bv = mask4(*(const float4 *)(Brow + base), a - base);
                    const float4 dv = *(const float4 *)(Dcol + base);
                    if (j & 1) s1 = dot4(bv, dv, s1); else s0 = dot4(bv, dv, s0);
                }
            }
            float u = u0 + u1, sc = s0 + s1;
#pragma unroll
            for (int o = 1; o < TPC; o <<= 1) {
                u += __shfl_xor_sync(gmask, u, o);
                sc += __shfl_xor_sync(gmask, sc, o);
            }
            const int ta = r0 + a, tb = c0 + bl;  // tile-local entry
            if (q == 0 && ta < mr && tb < nc) {
                const float wt = sR[ta * RSS + tb] - u - sc;
                const float s = scale[ta];
                const float c = decide(wt, s, rcp[ta], fqmin, fqmax);
                const float dl = fmaf(-s, c, wt);
                sR[ta * RSS + tb] = sc + dl;
                sDt[tb * RSS + ta] = dl;
                const int64_t gidx = (grow0 + ta) * p.n + gcol0 + tb;
                p.codes[gidx] = (int8_t)c;
                if (p.wt_out) p.wt_out[gidx] = wt;
            }
        }
        group_sync(bar_id, NT);
    }
}

// V = s * code and the residual's TF32 split for the tile's valid entries.
template <int RSS>
__device__ void write_outputs(const LeafArgs &p, const float *sDt, const float *scale, int64_t row0, int64_t col0,
                              int mr, int nc)
{
    for (int idx = threadIdx.x; idx < T * T; idx += kThreads) {
        const int r = idx / T, c = idx % T;
        if (r >= mr || c >= nc) continue;
        const int64_t gi = row0 + r, gj = col0 + c;
        const float code = (float)p.codes[gi * p.n + gj];
        p.V[gi * p.n + gj] = scale[r] * code;
        float hi, lo;
        split_tf32(sDt[c * RSS + r], hi, lo);
        p.Dhi[gi * p.Np + gj] = hi;
        p.Dlo[gi * p.Np + gj] = lo;
    }
}

// ---------------------------------------------------------------- products
// D (S x S) += sum_k A[i][k] Bm[j][k] over k in [0, S), both operands row-major
// with K contiguous (generic pointers into smem or global memory).  16 warps,
// each owning a 16 x 16 block of D as two m16n8 tiles; mma.sync m16n8k8 TF32
// in 3xTF32 form.
__device__ __forceinline__ void mma_tf32(float (&c)[4], const uint32_t (&a)[4], const uint32_t (&b)[2])
{
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

__device__ void accumulate_product(float (&acc)[2][4], const float *a, int lda, const float *b, int ldb)
{
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int i0 = (warp >> 2) * 16, j0 = (warp & 3) * 16;
    const int g = lane >> 2, t = lane & 3;
#pragma unroll 2
    for (int k0 = 0; k0 < S; k0 += 8) {
        const float af[4] = {a[(i0 + g) * lda + k0 + t], a[(i0 + g + 8) * lda + k0 + t],
                             a[(i0 + g) * lda + k0 + t + 4], a[(i0 + g + 8) * lda + k0 + t + 4]};
        uint32_t ahi[4], alo[4];
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            float h, l;
            split_tf32(af[r], h, l);
            ahi[r] = __float_as_uint(h);
            alo[r] = __float_as_uint(l);
        }
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            const int j = j0 + nt * 8 + g;
            const float bf[2] = {b[j * ldb + k0 + t], b[j * ldb + k0 + t + 4]};
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

// out (stride ldo) -= acc (subtract) or = acc
__device__ void apply_product(const float (&acc)[2][4], float *out, int ldo, bool subtract)
{
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int i0 = (warp >> 2) * 16, j0 = (warp & 3) * 16;
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
        const int j = j0 + nt * 8 + 2 * t;
        float *o0 = out + (i0 + g) * ldo + j, *o1 = out + (i0 + g + 8) * ldo + j;
        if (subtract) {
            o0[0] -= acc[nt][0]; o0[1] -= acc[nt][1]; o1[0] -= acc[nt][2]; o1[1] -= acc[nt][3];
        } else {
            o0[0] = acc[nt][0]; o0[1] = acc[nt][1]; o1[0] = acc[nt][2]; o1[1] = acc[nt][3];
        }
    }
}

__device__ void load_scales(const LeafArgs &p, float *scale, float *rcp, int64_t row0, int mr)
{
    if (threadIdx.x < T) {
        const float s = threadIdx.x < mr ? p.scales[row0 + threadIdx.x] : 1.f;
        scale[threadIdx.x] = s;
        rcp[threadIdx.x] = __frcp_rn(s);
    }
}

// Two-level variant: 2 x 2 sub-tiles of 64.
__global__ void __launch_bounds__(kThreads, 1) leaf_nested_kernel(LeafArgs p, int K, int I_lo)
{
    extern __shared__ __align__(16) float smem_f[];
    float *sR = smem_f;                  // T x RS: Wt, overwritten by sub-tile-local R
    float *sDt = sR + T * RS;            // T x RS: D transposed
    float *sLB0 = sDt + T * RS;          // S x BS: LtB tile block (0,0)
    float *sLB1 = sLB0 + S * BS;         // S x BS: LtB tile block (1,1)
    float *sZ = sLB1 + S * BS;           // S x ZS: S10 / S11
    float *scale = sZ + S * ZS;          // T
    float *rcp = scale + T;              // T

    const int I = I_lo + blockIdx.x, J = K - I;
    const int64_t row0 = (int64_t)I * T, col0 = (int64_t)J * T;
    const int mr = (int)min64(T, p.m - row0), nc = (int)min64(T, p.n - col0);
    const int tid = threadIdx.x;
    pdl_wait();

    for (int idx = tid; idx < T * T / 4; idx += kThreads) {
        const int r = idx / (T / 4), c4 = (idx % (T / 4)) * 4;
        *(float4 *)(sR + r * RS + c4) = *(const float4 *)(p.Wt + (row0 + r) * p.Np + col0 + c4);
        *(float4 *)(sDt + r * RS + c4) = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    for (int idx = tid; idx < S * S / 4; idx += kThreads) {
        const int r = idx / (S / 4), c4 = (idx % (S / 4)) * 4;
        *(float4 *)(sLB0 + r * BS + c4) = *(const float4 *)(p.LB32 + (row0 + r) * p.Mp + row0 + c4);
        *(float4 *)(sLB1 + r * BS + c4) = *(const float4 *)(p.LB32 + (row0 + S + r) * p.Mp + row0 + S + c4);
    }
    load_scales(p, scale, rcp, row0, mr);
    __syncthreads();

    // factor blocks used by the products (global, L1/L2 cached)
    const float *LA00 = p.LA32 + col0 * p.Np + col0;
    const float *LA10 = LA00 + S * p.Np;
    const float *LA11 = LA10 + S;
    const float *LB10 = p.LB32 + (row0 + S) * p.Mp + row0;
    const int lda_g = (int)p.Np, ldb_g = (int)p.Mp;

    // phase 0: sub-tile (0,0), all threads
    sweep_subtile<S, 8, RS, BS>(p, sR, sDt, sLB0, scale, rcp, 0, 0, row0, col0, mr, nc, tid, 1);
    __syncthreads();

    // cross terms into (0,1) and (1,0)
    {
        float acc[2][4] = {};
        accumulate_product(acc, sR, RS, LA10, lda_g);           // R00 LtA10^T
        apply_product(acc, sR + S, RS, true);
    }
    {
        float acc[2][4] = {};
        accumulate_product(acc, LB10, ldb_g, sDt, RS);          // S10 = LtB10 D00
        apply_product(acc, sZ, ZS, false);
    }
    __syncthreads();
    {
        float acc[2][4] = {};
        accumulate_product(acc, sZ, ZS, LA00, lda_g);           // S10 LtA00^T
        apply_product(acc, sR + S * RS, RS, true);
    }
    __syncthreads();

    // phase 1: (0,1) by threads [0, 256), (1,0) by threads [256, 512)
    if (tid < 256)
        sweep_subtile<S, 4, RS, BS>(p, sR, sDt, sLB0, scale, rcp, 0, S, row0, col0, mr, nc, tid, 1);
    else
        sweep_subtile<S, 4, RS, BS>(p, sR, sDt, sLB1, scale, rcp, S, 0, row0, col0, mr, nc, tid - 256, 2);
    __syncthreads();

    // R10 += S10 (column sums over all earlier rows of the tile), then the
    // cross terms into (1,1)
    for (int idx = tid; idx < S * S; idx += kThreads) {
        const int r = idx / S, c = idx % S;
        sR[(S + r) * RS + c] += sZ[r * ZS + c];
    }
    __syncthreads();
    {
        float acc[2][4] = {};
        accumulate_product(acc, LB10, ldb_g, sDt + S * RS, RS);  // S11 = LtB10 D01
        apply_product(acc, sZ, ZS, false);
    }
    __syncthreads();
    {
        float acc[2][4] = {};
        accumulate_product(acc, sR + S * RS, RS, LA10, lda_g);   // R10 LtA10^T
        accumulate_product(acc, sZ, ZS, LA11, lda_g);            // S11 LtA11^T
        apply_product(acc, sR + S * RS + S, RS, true);
    }
    __syncthreads();

    // phase 2: sub-tile (1,1), all threads
    sweep_subtile<S, 8, RS, BS>(p, sR, sDt, sLB1, scale, rcp, S, S, row0, col0, mr, nc, tid, 1);
    pdl_trigger();
    __syncthreads();
    write_outputs<RS>(p, sDt, scale, row0, col0, mr, nc);
}

// Single-level variant: the whole 128 x 128 tile in one anti-diagonal sweep.
__global__ void __launch_bounds__(kThreads, 1) leaf_single_kernel(LeafArgs p, int K, int I_lo)
{
    extern __shared__ __align__(16) float smem_f[];
    float *sR = smem_f;                  // T x RS1
    float *sDt = sR + T * RS1;           // T x RS1
    float *sLB = sDt + T * RS1;          // T x RS1: LtB diagonal block
    float *scale = sLB + T * RS1;        // T
    float *rcp = scale + T;              // T
    const int I = I_lo + blockIdx.x, J = K - I;
    const int64_t row0 = (int64_t)I * T, col0 = (int64_t)J * T;
    const int mr = (int)min64(T, p.m - row0), nc = (int)min64(T, p.n - col0);
    const int tid = threadIdx.x;
    pdl_wait();
    for (int idx = tid; idx < T * T / 4; idx += kThreads) {
        const int r = idx / (T / 4), c4 = (idx % (T / 4)) * 4;
        *(float4 *)(sR + r * RS1 + c4) = *(const float4 *)(p.Wt + (row0 + r) * p.Np + col0 + c4);
        *(float4 *)(sLB + r * RS1 + c4) = *(const float4 *)(p.LB32 + (row0 + r) * p.Mp + row0 + c4);
        *(float4 *)(sDt + r * RS1 + c4) = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    load_scales(p, scale, rcp, row0, mr);
    __syncthreads();
    sweep_subtile<T, 4, RS1, RS1>(p, sR, sDt, sLB, scale, rcp, 0, 0, row0, col0, mr, nc, tid, 1);
    pdl_trigger();
    __syncthreads();
    write_outputs<RS1>(p, sDt, scale, row0, col0, mr, nc);
}

// ------------------------------------------------------------------------
// Warp-per-sub-tile variant: 4 x 4 sub-tiles of 32, processed in sub-tile
// diagonal order e = 0..6.  Before phase e, the cross-sub-tile terms of every
// sub-tile (p, q) with p + q = e are applied left-looking with all 16 warps:
//     S[p,q] = sum_{p'<p} LtB[p,p'] D[p',q],
//     Wt[p,q] -= sum_{q'<q} R[p,q'] LtA[q,q']^T + S[p,q] LtA[q,q]^T,
// where R[p,q'] = sum_{p'<=p} LtB[p,p'] D[p',q'] is complete for q' < q.  Then
// warp p sweeps sub-tile (p, q) alone (lane = column, 63 warp-synchronous
// steps), and finally R[p,q] = S[p,q] + (the sweep's in-sub-tile R).
// sR and sDt start at zero, so entries not yet rounded contribute nothing to
// the sweep's dot products and no masking is needed.
namespace {
constexpr int S3 = 32;             // sub-tile side
constexpr int RS3 = T + 4;         // row stride of sR / sDt: 33 float4 per row
constexpr int WS3 = S3 + 4;        // row stride of the per-row-block slots
constexpr size_t kSmemWarp = ((size_t)2 * T * RS3 + 3 * 4 * S3 * WS3 + 2 * T) * sizeof(float) + (size_t)T * T;
static_assert(kSmemWarp <= 232448, "leaf shared memory");
}  // namespace

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

constexpr int kThreadsW = 256;  // warp variant: 4 sweeping warps, 2 product warps per row block

__global__ void __launch_bounds__(kThreadsW, 1) leaf_warp_kernel(LeafArgs p, int K, int I_lo)
{
    extern __shared__ __align__(16) float smem_f[];
    float *sR = smem_f;                 // T x RS3: R (full for finished sub-tiles), 0 elsewhere
    float *sDt = sR + T * RS3;          // T x RS3: D transposed, 0 where not rounded yet
    float *sW = sDt + T * RS3;          // 4 slots of S3 x WS3: Wt of the sub-tile being swept per row block
    float *sS = sW + 4 * S3 * WS3;      // 4 slots: S[p,q]
    float *sLB = sS + 4 * S3 * WS3;     // 4 slots: LtB[p,p]
    float *scale = sLB + 4 * S3 * WS3;  // T
    float *rcp = scale + T;             // T
    int8_t *sCode = (int8_t *)(rcp + T); // T x T codes

    const int I = I_lo + blockIdx.x, J = K - I;
    const int64_t row0 = (int64_t)I * T, col0 = (int64_t)J * T;
    const int mr = (int)min64(T, p.m - row0), nc = (int)min64(T, p.n - col0);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // Warm L2 with the tile's two factor diagonal blocks (read by the products
    // and the sweeps; each leaf launch uses blocks no earlier launch touched).
    // A prefetch is only a hint, so it may run before the dependency wait.
    for (int idx = tid; idx < 2 * T * (T / 32); idx += kThreadsW) {
        const int which = idx / (T * (T / 32)), r = (idx / (T / 32)) % T, seg = idx % (T / 32);
        const float *ptr = which == 0 ? p.LA32 + (col0 + r) * p.Np + col0 + 32 * seg
                                      : p.LB32 + (row0 + r) * p.Mp + row0 + 32 * seg;
        asm volatile("prefetch.global.L2 [%0];" ::"l"(ptr));
    }
    pdl_wait();  // every global input (Wt, factors, steps) comes from earlier kernels

    for (int idx = tid; idx < T * RS3 / 4; idx += kThreadsW) {
        ((float4 *)sR)[idx] = make_float4(0.f, 0.f, 0.f, 0.f);
        ((float4 *)sDt)[idx] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    for (int idx = tid; idx < 4 * S3 * S3; idx += kThreadsW) {  // LtB diagonal sub-blocks (prep output)
        const int blk = idx / (S3 * S3), r = (idx / S3) % S3, c = idx % S3;
        sLB[blk * S3 * WS3 + r * WS3 + c] = p.LB32[(row0 + blk * S3 + r) * p.Mp + row0 + blk * S3 + c];
    }
    load_scales(p, scale, rcp, row0, mr);
    __syncthreads();

    const float *LAt = p.LA32 + col0 * p.Np + col0;  // LtA diagonal block of the tile (global)
    const float *LBt = p.LB32 + row0 * p.Mp + row0;  // LtB diagonal block of the tile (global)
    const int lda_g = (int)p.Np, ldb_g = (int)p.Mp;
    const float fqmin = (float)p.qmin, fqmax = (float)p.qmax;
    const int wp = warp >> 1;                          // products: warp -> (row block, 16 x 32 half)
    const int i0 = (warp & 1) * 16, j0 = 0;

    for (int e = 0; e < 7; ++e) {
        const int p_lo = max(0, e - 3), p_hi = min(3, e);
        const bool mine = wp >= p_lo && wp <= p_hi;  // this warp's row block has a sub-tile in phase e
        const int qv = e - wp;
        // S[p,q] = LtB[p, 0:p] D[0:p, q]
        if (mine) {
            float acc[4][4] = {};
            if (wp > 0)
                mma_block<4>(acc, LBt + (wp * S3) * ldb_g, ldb_g, sDt + (qv * S3) * RS3, RS3, wp * S3, i0, j0);
            const int g = lane >> 2, t = lane & 3;
            float *o = sS + wp * S3 * WS3;
#pragma unroll
            for (int nt = 0; nt < 4; ++nt) {
                const int j = j0 + nt * 8 + 2 * t;
                o[(i0 + g) * WS3 + j] = acc[nt][0];
                o[(i0 + g) * WS3 + j + 1] = acc[nt][1];
                o[(i0 + g + 8) * WS3 + j] = acc[nt][2];
                o[(i0 + g + 8) * WS3 + j + 1] = acc[nt][3];
            }
        }
        __syncthreads();
        // Wt[p,q] = Wt_global - (R[p, 0:q] LtA[q, 0:q]^T + S[p,q] LtA[q,q]^T)
        if (mine) {
            float acc[4][4] = {};
            const float *LAq = LAt + (qv * S3) * lda_g;
            if (qv > 0) mma_block<4>(acc, sR + (wp * S3) * RS3, RS3, LAq, lda_g, qv * S3, i0, j0);
            mma_block<4>(acc, sS + wp * S3 * WS3, WS3, LAq + qv * S3, lda_g, S3, i0, j0);
            const int g = lane >> 2, t = lane & 3;
            float *o = sW + wp * S3 * WS3;
            const float *wg = p.Wt + (row0 + wp * S3) * p.Np + col0 + qv * S3;
#pragma unroll
            for (int nt = 0; nt < 4; ++nt) {
                const int j = j0 + nt * 8 + 2 * t;
                o[(i0 + g) * WS3 + j] = wg[(i0 + g) * p.Np + j] - acc[nt][0];
                o[(i0 + g) * WS3 + j + 1] = wg[(i0 + g) * p.Np + j + 1] - acc[nt][1];
                o[(i0 + g + 8) * WS3 + j] = wg[(i0 + g + 8) * p.Np + j] - acc[nt][2];
                o[(i0 + g + 8) * WS3 + j + 1] = wg[(i0 + g + 8) * p.Np + j + 1] - acc[nt][3];
            }
        }
        __syncthreads();
        // sweep: warp p takes sub-tile (p, e - p), lane = column
        if (warp <= 3 && warp >= p_lo && warp <= p_hi) {
            const int pp = warp, q = e - pp, b = lane;
            float4 la[S3 / 4];  // LtA[q,q] row b, strictly lower part
#pragma unroll
            for (int c = 0; c < S3 / 4; ++c) {
                float4 v = *(const float4 *)(LAt + (q * S3 + b) * lda_g + q * S3 + 4 * c);
                v.x = 4 * c + 0 < b ? v.x : 0.f;
                v.y = 4 * c + 1 < b ? v.y : 0.f;
                v.z = 4 * c + 2 < b ? v.z : 0.f;
                v.w = 4 * c + 3 < b ? v.w : 0.f;
                la[c] = v;
            }
            const float *LBp = sLB + pp * S3 * WS3;
            const float *Wp = sW + pp * S3 * WS3;
            // newest-term coefficient LtA[b, b-1] (0 for b = 0)
            const float la_new = b > 0 ? LAt[(q * S3 + b) * lda_g + q * S3 + b - 1] : 0.f;
            // Software pipeline over the anti-diagonal steps.  At the start of step
            // d every entry on diagonals <= d-1 is final and every entry on
            // diagonal d is still zero in smem, so the dot products of this lane's
            // NEXT entry (row a+1) read now automatically leave out exactly the
            // two terms that become final during step d; those are added at step
            // d+1 from R[a+1][b-1] (written by lane b-1) and this lane's own D.
            // The lane's own column of D lives in registers (dcol[k] holds rows
            // 4k..4k+3), so each step streams only one row of R and one row of
            // LtB from smem, and only the chunks the lane needs.
            float4 dcol[S3 / 4];
#pragma unroll
            for (int c = 0; c < S3 / 4; ++c) dcol[c] = make_float4(0.f, 0.f, 0.f, 0.f);
            float pu = 0.f, ps = 0.f;  // partial sums for the current entry
            float d_prev = 0.f;        // D[a-1][b]
            const float4 zero4 = make_float4(0.f, 0.f, 0.f, 0.f);
            for (int d = 0; d < 2 * S3 - 1; ++d) {
                const int a = d - b;
                const bool active = a >= 0 && a < S3;
                const int ac = min(max(a, 0), S3 - 1);
                const int an = min(max(a + 1, 0), S3 - 1);  // next entry's row (clamped)
                // (1) critical loads first: they must not queue behind the bulk
                const float r_new = b > 0 ? sR[(pp * S3 + ac) * RS3 + q * S3 + b - 1] : 0.f;
                const float lb_new = ac > 0 ? LBp[ac * WS3 + ac - 1] : 0.f;
                const float w0 = Wp[ac * WS3 + b];
                const int ta = pp * S3 + a, tb = q * S3 + b;
                const float s = scale[ac + pp * S3], rs = rcp[ac + pp * S3];
                // (2) bulk loads for the next entry (before any store of this step);
                // a chunk is loaded only by lanes that need an index in it
                const float *Rn = sR + (pp * S3 + an) * RS3 + q * S3;
                const float *Bn = LBp + an * WS3;
                float4 rv[S3 / 4], bv[S3 / 4];
#pragma unroll
                for (int c = 0; c < S3 / 4; ++c) {
                    rv[c] = zero4;
                    bv[c] = zero4;
                    if (4 * c < b) rv[c] = *(const float4 *)(Rn + 4 * c);
                    if (4 * c <= a) bv[c] = *(const float4 *)(Bn + 4 * c);
                }
                // (3) the current entry
                const float uu = fmaf(r_new, la_new, pu), sc = fmaf(lb_new, d_prev, ps);
                float dl = 0.f;
                if (active && ta < mr && tb < nc) {
                    const float wt = w0 - uu - sc;
                    const float c = decide(wt, s, rs, fqmin, fqmax);
                    dl = fmaf(-s, c, wt);
                    sR[ta * RS3 + tb] = sc + dl;
                    sDt[tb * RS3 + ta] = dl;
                    sCode[ta * T + tb] = (int8_t)c;
                    if (p.wt_out) p.wt_out[(row0 + ta) * p.n + col0 + tb] = wt;
                }
                // (4) partial sums of the next entry (dcol does not yet hold D[a][b])
                float u4[4] = {0.f, 0.f, 0.f, 0.f}, s4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int c = 0; c < S3 / 4; ++c) {
                    u4[c & 3] = dot4(rv[c], la[c], u4[c & 3]);
                    s4[c & 3] = dot4(bv[c], dcol[c], s4[c & 3]);
                }
                pu = (u4[0] + u4[1]) + (u4[2] + u4[3]);
                ps = (s4[0] + s4[1]) + (s4[2] + s4[3]);
                // (5) D[a][b] into the register column
                d_prev = dl;
                {
                    // branch-free insert: compare the row against each register slot
                    const int row = active ? a : -1;
#pragma unroll
                    for (int c = 0; c < S3 / 4; ++c) {
                        dcol[c].x = row == 4 * c + 0 ? dl : dcol[c].x;
                        dcol[c].y = row == 4 * c + 1 ? dl : dcol[c].y;
                        dcol[c].z = row == 4 * c + 2 ? dl : dcol[c].z;
                        dcol[c].w = row == 4 * c + 3 ? dl : dcol[c].w;
                    }
                }
                __syncwarp();
            }
        }
        __syncthreads();
        // R[p,q] = S[p,q] + in-sub-tile R
        for (int idx = tid; idx < (p_hi - p_lo + 1) * S3 * S3; idx += kThreadsW) {
            const int pp = p_lo + idx / (S3 * S3), r = (idx / S3) % S3, c = idx % S3;
            sR[(pp * S3 + r) * RS3 + (e - pp) * S3 + c] += sS[pp * S3 * WS3 + r * WS3 + c];
        }
        __syncthreads();
    }
    pdl_trigger();
    for (int idx = tid; idx < T * T; idx += kThreadsW) {  // V = s * code, residual split
        const int r = idx / T, c = idx % T;
        if (r >= mr || c >= nc) continue;
        const int64_t gi = row0 + r, gj = col0 + c;
        const int8_t code = sCode[r * T + c];
        p.codes[gi * p.n + gj] = code;
        p.V[gi * p.n + gj] = scale[r] * (float)code;
        float hi, lo;
        split_tf32(sDt[c * RS3 + r], hi, lo);
        p.Dhi[gi * p.Np + gj] = hi;
        p.Dlo[gi * p.Np + gj] = lo;
    }
}

cudaError_t leaf_configure()
{
    cudaError_t e = cudaFuncSetAttribute(leaf_nested_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kSmemNested);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(leaf_warp_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemWarp);
    if (e != cudaSuccess) return e;
    return cudaFuncSetAttribute(leaf_single_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemSingle);
}

cudaError_t launch_leaf(const LeafArgs &p, int K, int variant, cudaStream_t stream)
{
    int I_lo = max(0, K - (p.Nt - 1)), I_hi = min(p.Mt - 1, K);
    if (I_hi < I_lo) return cudaSuccess;
    if (variant == 2)
        return launch_pdl(leaf_warp_kernel, dim3(I_hi - I_lo + 1), dim3(kThreadsW), kSmemWarp, stream, p, K, I_lo);
    if (variant == 1)
        return launch_pdl(leaf_single_kernel, dim3(I_hi - I_lo + 1), dim3(kThreads), kSmemSingle, stream, p, K, I_lo);
    return launch_pdl(leaf_nested_kernel, dim3(I_hi - I_lo + 1), dim3(kThreads), kSmemNested, stream, p, K, I_lo);
}

}  // namespace bakron
