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
#include <type_traits>

#include "common.cuh"
#include "kernels.cuh"
#include "leaf_wave.cuh"
#include "leaf_common.cuh"

namespace bakron {

using namespace leafk;

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

// Steps and their correctly rounded reciprocals; returns true for a thread
// whose step lies outside [2^-60, 2^60], where the decisions take the IEEE
// division instead of the reciprocal-based one (div_rn_recip).
__device__ bool load_scales(const LeafArgs &p, float *scale, float *rcp, int64_t row0, int mr)
{
    if (threadIdx.x < T) {
        const float s = threadIdx.x < mr ? p.scales[row0 + threadIdx.x] : 1.f;
        scale[threadIdx.x] = s;
        rcp[threadIdx.x] = __frcp_rn(s);
        return !(s >= 0x1p-60f && s <= 0x1p60f);
    }
    return false;
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
// Warp variant (the default): 4 x 4 sub-tiles of 32, processed in sub-tile
// diagonal order e = 0..6, three warps per row block of sub-tiles.  Phase e,
// for every sub-tile (p, q) with p + q = e:
//     S[p,q]  = sum_{p'<p} LtB[p,p'] D[p',q]              (written into R[p,q]),
//     W0[p,q] = Wt[p,q] - sum_{q'<q} R[p,q'] LtA[q,q']^T - S[p,q],
// where R[p,q'] = sum_{p'<=p} LtB[p,p'] D[p',q'] is complete for q' < q; then
// the three warps of row block p sweep the sub-tile (63 entry anti-diagonal
// steps, one 96-thread barrier each).  Entry (a, b) of the sub-tile needs
//     Wt_ab = W0_ab - sum_{c<b} R_ac LtA[b,c] - sum_{r<a} LtB[a,r] D_rb,
// with R holding S plus the sub-tile's own terms, so the S terms of the
// row-side sum come in through R:
//   * the entry warp (lane = column b) rounds the entries and writes
//     R_ab = S_ab + sum_{r<=a} LtB[a,r] D_rb;
//   * the row-side warp (lane = column b) forms sum_{c<=b-2} R_ac LtA[b,c]
//     from its LtA row (registers) and rows of R (smem);
//   * the column-side warp (lane = row rho) forms sum_{r<=rho-2} LtB[rho,r] D_rb
//     from its LtB row (registers) and columns of D (smem);
// both sums a step ahead without their newest term, which the entry warp adds
// from the values the previous step produced.  The Wt blocks and LtA strips of
// the next phase are staged into shared memory by asynchronous copies while the
// current phase sweeps.  sR and sDt start at zero.
namespace {
constexpr int S3 = 32;             // sub-tile side
constexpr int RS3 = T + 4;         // row stride of sR / sDt: 33 float4 per row
constexpr int WS3 = S3 + 4;        // row stride of the per-row-block slots
constexpr int kLAStage = S3 * (3 * S3 * 2 + 4 * 3);  // largest phase: strips for q = 3, 2, 1
constexpr size_t kSmemWarp =
    ((size_t)2 * (T + 1) * RS3 + 4 * S3 * WS3 + 2 * kLAStage + 4 * S3 + 2 * T + 2 * 4 * 2 * S3) * sizeof(float) +
    (size_t)T * T + 32;
static_assert(kSmemWarp <= 232448, "leaf shared memory");
}  // namespace

constexpr int kThreadsW = 384;  // warp variant: 3 warps per row block of sub-tiles

__global__ void __launch_bounds__(kThreadsW, 1) leaf_warp_kernel(LeafArgs p, int K, int I_lo)
{
    extern __shared__ __align__(16) float smem_f[];
    float *sR = smem_f;                  // T x RS3 (+1 spare row): R, S before the sweep, 0 before that
    float *sDt = sR + (T + 1) * RS3;     // T x RS3 (+1 spare row): D transposed, 0 where not rounded yet
    float *sW = sDt + (T + 1) * RS3;     // 4 slots of S3 x WS3: S, then W0 of the sub-tile being swept, then Wt
    float *sLA = sW + 4 * S3 * WS3;      // LtA[q, 0:q] strips of the next phase (staged during the sweep)
    float *sLBs = sLA + kLAStage;        // LtB[p, 0:p] strips of the next phase (staged during the sweep)
    float *sLBd = sLBs + kLAStage;       // 4 x S3: LtB sub-diagonal LtB[r][r-1] per row block
    float *scale = sLBd + 4 * S3;        // T
    float *rcp = scale + T;              // T
    float *sPS = rcp + T;                // 4 x 2 x S3: column-side partial sums by column
    float *sPU = sPS + 4 * 2 * S3;       // 4 x 2 x S3: row-side partial sums by column
    int8_t *sCode = (int8_t *)(sPU + 4 * 2 * S3);  // T x T codes (+32 spare bytes)

    const int I = I_lo + blockIdx.x, J = K - I;
    const int64_t row0 = (int64_t)I * T, col0 = (int64_t)J * T;
    const int mr = (int)min64(T, p.m - row0), nc = (int)min64(T, p.n - col0);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const float *LAt = p.LA32 + col0 * p.Np + col0;  // LtA diagonal block of the tile (global)
    const float *LBt = p.LB32 + row0 * p.Mp + row0;  // LtB diagonal block of the tile (global)
    const int lda_g = (int)p.Np, ldb_g = (int)p.Mp;
    // Warm L2 with the tile's two factor diagonal blocks (read by the products
    // and the sweeps; each leaf launch uses blocks no earlier launch touched).
    // A prefetch is only a hint, so it may run before the dependency wait.
    for (int idx = tid; idx < 2 * T * (T / 32); idx += kThreadsW) {
        const int which = idx / (T * (T / 32)), r = (idx / (T / 32)) % T, seg = idx % (T / 32);
        const float *ptr = which == 0 ? LAt + r * lda_g + 32 * seg : LBt + r * ldb_g + 32 * seg;
        asm volatile("prefetch.global.L2 [%0];" ::"l"(ptr));
    }
    // Zeroing R and D touches no global memory, so it overlaps the previous
    // kernel's tail.
    for (int idx = tid; idx < (T + 1) * RS3 / 4; idx += kThreadsW) {
        ((float4 *)sR)[idx] = make_float4(0.f, 0.f, 0.f, 0.f);
        ((float4 *)sDt)[idx] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    __syncthreads();  // R is zero before the first staged block lands in it
    pdl_wait();  // every global input (Wt, factors, steps) comes from earlier kernels

    // Stage, for the sub-tiles (p, q = e - p) of phase e: the tile's Wt block
    // into R's (p,q) block (untouched until then), the strip LtA[q, 0:q] (32
    // rows x 32 q columns, row stride 32 q + 4) and the strip LtB[p, 0:p] (32
    // rows x 32 p columns, row stride 32 p + 4), strips laid out back to back
    // in row-block order.  Every thread issues a share of 16-byte asynchronous
    // copies and commits them as one group.
    auto stage_phase = [&](int e) {
        if (e > 6) return;
        int off = 0, offb = 0;
        for (int pp = max(0, e - 3); pp <= min(3, e); ++pp) {
            const int q = e - pp;
            if (q > 0) {
                const int ld = S3 * q + 4, c4 = 8 * q;
                for (int c = tid; c < S3 * c4; c += kThreadsW) {
                    const int j = c / c4, k4 = c - j * c4;
                    cp_async16(sLA + off + j * ld + 4 * k4, LAt + (q * S3 + j) * lda_g + 4 * k4);
                }
                off += S3 * ld;
            }
            if (pp > 0) {
                const int ld = S3 * pp + 4, c4 = 8 * pp;
                for (int c = tid; c < S3 * c4; c += kThreadsW) {
                    const int i = c / c4, k4 = c - i * c4;
                    cp_async16(sLBs + offb + i * ld + 4 * k4, LBt + (pp * S3 + i) * ldb_g + 4 * k4);
                }
                offb += S3 * ld;
            }
            for (int c = tid; c < S3 * 8; c += kThreadsW) {
                const int i = c >> 3, k4 = c & 7;
                cp_async16(sR + (pp * S3 + i) * RS3 + q * S3 + 4 * k4,
                           p.Wt + (row0 + pp * S3 + i) * p.Np + col0 + q * S3 + 4 * k4);
            }
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
    };
    // offsets of row block pp's LtA and LtB strips in phase e
    auto la_offset = [](int e, int pp) {
        int off = 0;
        for (int p2 = max(0, e - 3); p2 < pp; ++p2)
            if (e - p2 > 0) off += S3 * (S3 * (e - p2) + 4);
        return off;
    };
    auto lb_offset = [](int e, int pp) {
        int off = 0;
        for (int p2 = max(0, e - 3); p2 < pp; ++p2)
            if (p2 > 0) off += S3 * (S3 * p2 + 4);
        return off;
    };
    stage_phase(0);
    if (tid < T) {
        const int blk = tid / S3, r = tid % S3;
        sLBd[tid] = r > 0 ? LBt[(blk * S3 + r) * ldb_g + blk * S3 + r - 1] : 0.f;
    }
    const float fqmin = (float)p.qmin, fqmax = (float)p.qmax;
    const int wp = warp / 3, role = warp - 3 * wp;  // row block of sub-tiles; 0 entries, 1 row side, 2 column side
    // column-side warp: its LtB[p,p] row rho (columns <= rho-2), fixed for the kernel
    float2 lbr[S3 / 2];
    if (role == 2) {
#pragma unroll
        for (int c = 0; c < S3 / 2; ++c) {
            float2 v = *(const float2 *)(LBt + (wp * S3 + lane) * ldb_g + wp * S3 + 2 * c);
            v.x = 2 * c + 0 <= lane - 2 ? v.x : 0.f;
            v.y = 2 * c + 1 <= lane - 2 ? v.y : 0.f;
            lbr[c] = v;
        }
    }
    // steps outside the range of the reciprocal-based division switch the
    // whole tile to the IEEE division (a tile-uniform choice)
    const bool exact_div = __syncthreads_or(load_scales(p, scale, rcp, row0, mr)) != 0;

    for (int e = 0; e < 7; ++e) {
        const int p_lo = max(0, e - 3), p_hi = min(3, e);
        const bool mine = wp >= p_lo && wp <= p_hi;  // this warp's row block has a sub-tile in phase e
        const int qv = e - wp;
        asm volatile("cp.async.wait_all;" ::: "memory");  // this phase's staged Wt blocks and strips
        __syncthreads();
        // S[p,q] = LtB[p, 0:p] D[0:p, q] into the row block's slot (three warps)
        if (mine && wp > 0) {
            Block3 b;
            product3(b, role, sLBs + lb_offset(e, wp), S3 * wp + 4, sDt + (qv * S3) * RS3, RS3, wp * S3);
            store3(b, role, sW + wp * S3 * WS3, WS3);
        }
        // row-side warp: LtA[q,q] row b (columns <= b-2); entry warp: LtA[b][b-1]
        float2 la[S3 / 2];
        float la_new = 0.f;
        if (mine && role == 1) {
#pragma unroll
            for (int c = 0; c < S3 / 2; ++c) {
                float2 v = *(const float2 *)(LAt + (qv * S3 + lane) * lda_g + qv * S3 + 2 * c);
                v.x = 2 * c + 0 <= lane - 2 ? v.x : 0.f;
                v.y = 2 * c + 1 <= lane - 2 ? v.y : 0.f;
                la[c] = v;
            }
        }
        if (mine && role == 0 && lane > 0) la_new = LAt[(qv * S3 + lane) * lda_g + qv * S3 + lane - 1];
        __syncthreads();
        // W0[p,q] = Wt[p,q] - R[p, 0:q] LtA[q, 0:q]^T - S[p,q] into the slot; R's
        // (p,q) block (holding the staged Wt) becomes S: the sweep adds the S terms
        // of the row-side sums through R
        if (mine) {  // three warps
            Block3 b;
            product3(b, role, sR + (wp * S3) * RS3, RS3, sLA + la_offset(e, wp), S3 * qv + 4, qv * S3);
            finish3(b, role, sW + wp * S3 * WS3, WS3, sR + (wp * S3) * RS3 + qv * S3, RS3, wp > 0);
        }
        __syncthreads();
        stage_phase(e + 1);  // lands while this phase sweeps
        // sweep: warps 3p, 3p+1, 3p+2 take sub-tile (p, e - p) together, one
        // barrier of the three per entry anti-diagonal step
        if (mine) {
            const int pp = wp, q = qv;
            float *ps_buf = sPS + pp * 2 * S3;  // [2][S3]: column-side sums, by column
            float *pu_buf = sPU + pp * 2 * S3;  // [2][S3]: row-side sums, by column
            float *Wp = sW + pp * S3 * WS3;
            const float *LBd = sLBd + pp * S3;
            const int bar_id = 1 + pp;
            if (role == 0) {
                // ---- entry warp (lane = column b): rounds entry (d - b, b) at step d
                const int b = lane, tb = q * S3 + b;
                // row-dependent values of an entry, loaded a step before it is rounded
                auto row_consts = [&](int a, float &w0, float &lbn, float &sv, float &rv_, float &s0) {
                    const int ac = min(max(a, 0), S3 - 1);
                    w0 = Wp[ac * WS3 + b];
                    lbn = LBd[ac];
                    sv = scale[pp * S3 + ac];
                    rv_ = rcp[pp * S3 + ac];
                    s0 = sR[(pp * S3 + ac) * RS3 + tb];  // S[a][b] until this entry overwrites it
                };
                auto sweep = [&](auto ieee_tag) {
                    constexpr bool kIeee = decltype(ieee_tag)::value;
                    float w0, lb_new, sc_s, sc_r, s_ab;
                    row_consts(-b, w0, lb_new, sc_s, sc_r, s_ab);
                    float d_prev = 0.f;
#pragma unroll 2
                    for (int d = 0; d < 2 * S3 - 1; ++d) {
                        const int a = d - b;
                        const int ac = min(max(a, 0), S3 - 1);
                        // the values the previous step produced (the other warps' sums
                        // leave out the newest row and column terms, added here)
                        const float ps_in = d > 0 ? ps_buf[(d & 1) * S3 + b] : 0.f;
                        const float pu_in = d > 0 ? pu_buf[(d & 1) * S3 + b] : 0.f;
                        const float r_new = b > 0 ? sR[(pp * S3 + ac) * RS3 + tb - 1] : 0.f;
                        float w0n, lbn_n, sn, rn, s_n;
                        row_consts(a + 1, w0n, lbn_n, sn, rn, s_n);
                        const float sc = fmaf(lb_new, d_prev, ps_in);
                        const float wt = w0 - fmaf(r_new, la_new, pu_in) - sc;
                        // clamp(rint(wt / s)) with the correctly rounded fp32 quotient
                        const float qf = kIeee ? __fdiv_rn(wt, sc_s) : div_rn_recip(wt, sc_s, sc_r);
                        const float cq = fminf(fmaxf(rintf(qf), fqmin), fqmax);
                        const int ta = pp * S3 + a;
                        const bool valid = a >= 0 && a < S3 && ta < mr && tb < nc;
                        const float dl = valid ? fmaf(-sc_s, cq, wt) : 0.f;
                        // invalid lanes write to spare slots instead of branching
                        const int iR = valid ? ta * RS3 + tb : T * RS3 + lane;
                        const int iD = valid ? tb * RS3 + ta : T * RS3 + lane;
                        const int iC = valid ? ta * T + tb : T * T + lane;
                        const int iW = valid ? a * WS3 + b : ac * WS3 + S3 + (lane & 3);  // row padding
                        sR[iR] = s_ab + sc + dl;
                        sDt[iD] = dl;
                        sCode[iC] = code_byte(cq);
                        Wp[iW] = wt;  // pre-rounding value, copied out when requested
                        d_prev = dl;
                        w0 = w0n; lb_new = lbn_n; sc_s = sn; sc_r = rn; s_ab = s_n;
                        group_sync(bar_id, 96);
                    }
                };
                if (exact_div)
                    sweep(std::true_type{});
                else
                    sweep(std::false_type{});
            } else if (role == 1) {
                // ---- row-side warp (lane = column b): sum_{c <= b-2} R[a+1][c] LtA[b][c]
                // for the entry warp's next entry (a+1, b).  Column b-1 of that R
                // row is written during this step; its coefficient here is zero.
                const int b = lane;
                float4 rv[S3 / 4];  // chunks this lane never loads stay zero
#pragma unroll
                for (int c = 0; c < S3 / 4; ++c) rv[c] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 2
                for (int d = 0; d < 2 * S3 - 1; ++d) {
                    const int an = min(max(d - b + 1, 0), S3 - 1);
                    const float *Rn = sR + (pp * S3 + an) * RS3 + q * S3;
#pragma unroll
                    for (int c = 0; c < S3 / 4; ++c)
                        if (4 * c <= b - 2) rv[c] = *(const float4 *)(Rn + 4 * c);
                    float2 u0 = make_float2(0.f, 0.f), u1 = make_float2(0.f, 0.f);
                    float2 u2 = make_float2(0.f, 0.f), u3 = make_float2(0.f, 0.f);
#pragma unroll
                    for (int c = 0; c < S3 / 4; c += 2) {
                        u0 = ffma2(make_float2(rv[c].x, rv[c].y), la[2 * c], u0);
                        u1 = ffma2(make_float2(rv[c].z, rv[c].w), la[2 * c + 1], u1);
                        u2 = ffma2(make_float2(rv[c + 1].x, rv[c + 1].y), la[2 * c + 2], u2);
                        u3 = ffma2(make_float2(rv[c + 1].z, rv[c + 1].w), la[2 * c + 3], u3);
                    }
                    pu_buf[((d + 1) & 1) * S3 + b] = ((u0.x + u1.x) + (u2.x + u3.x)) + ((u0.y + u1.y) + (u2.y + u3.y));
                    group_sync(bar_id, 96);
                }
            } else {
                // ---- column-side warp (lane = row rho): sum_{r <= rho-2} LtB[rho][r] D[r][b]
                // for the entry warp's entry (rho, b = d+1-rho) at step d+1.  Row
                // rho-1 of that D column is written during this step; its
                // coefficient here is zero.
                const int rho = lane;
                float4 dv[S3 / 4];
#pragma unroll
                for (int c = 0; c < S3 / 4; ++c) dv[c] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 2
                for (int d = 0; d < 2 * S3 - 1; ++d) {
                    const int b = d + 1 - rho;
                    const int bc = min(max(b, 0), S3 - 1);
                    const float *Dc = sDt + (q * S3 + bc) * RS3 + pp * S3;
#pragma unroll
                    for (int c = 0; c < S3 / 4; ++c)
                        if (4 * c <= rho - 2) dv[c] = *(const float4 *)(Dc + 4 * c);
                    float2 s0 = make_float2(0.f, 0.f), s1 = make_float2(0.f, 0.f);
                    float2 s2 = make_float2(0.f, 0.f), s3 = make_float2(0.f, 0.f);
#pragma unroll
                    for (int c = 0; c < S3 / 4; c += 2) {
                        s0 = ffma2(make_float2(dv[c].x, dv[c].y), lbr[2 * c], s0);
                        s1 = ffma2(make_float2(dv[c].z, dv[c].w), lbr[2 * c + 1], s1);
                        s2 = ffma2(make_float2(dv[c + 1].x, dv[c + 1].y), lbr[2 * c + 2], s2);
                        s3 = ffma2(make_float2(dv[c + 1].z, dv[c + 1].w), lbr[2 * c + 3], s3);
                    }
                    if (b == bc)
                        ps_buf[((d + 1) & 1) * S3 + b] = ((s0.x + s1.x) + (s2.x + s3.x)) + ((s0.y + s1.y) + (s2.y + s3.y));
                    group_sync(bar_id, 96);
                }
            }
        }
        __syncthreads();
        if (p.wt_out) {  // the pre-rounding values of this phase's sub-tiles
            for (int idx = tid; idx < (p_hi - p_lo + 1) * S3 * S3; idx += kThreadsW) {
                const int pp = p_lo + idx / (S3 * S3), r = (idx / S3) % S3, c = idx % S3;
                const int ta = pp * S3 + r, tb = (e - pp) * S3 + c;
                if (ta < mr && tb < nc) p.wt_out[(row0 + ta) * p.n + col0 + tb] = sW[pp * S3 * WS3 + r * WS3 + c];
            }
        }
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

// ------------------------------------------------------------------------
// Wide variant: 2 x 2 sub-tiles of 64 in three sub-tile-diagonal phases (fewer
// dependent steps than the 4 x 4 split: 3 x 127 instead of 7 x 63, and three
// product phases instead of seven), six warps per row block of sub-tiles: two
// entry warps (columns 0-31 / 32-63 of the sub-tile), two row-side warps (same
// columns) and two column-side warps (rows 0-31 / 32-63), one 192-thread
// barrier per step.  Phase e, sub-tile (p, q = e - p):
//     S[p,q]  = LtB[1,0] D[0,q] for p = 1 (written into R's (1,q) block),
//     W0[p,q] = Wt[p,q] - R[p,0] LtA[1,0]^T (q = 1) - S[p,q],
// then the sweep as in the warp variant.  Wt blocks are staged by cp.async
// into three slots (phase 0 uses slot 0; phase 1 slots 1, 2; phase 2 slot 0
// again, staged during phase 1), LtA[1,0] once at the start.
namespace {
constexpr int SW = 64;                 // sub-tile side
constexpr int LDW = SW + 4;            // row stride of slots and the LtA block
constexpr int kThreadsWide = 384;
constexpr size_t kSmemWide = ((size_t)2 * (T + 1) * RS3 + 4 * SW * LDW + 2 * T + T + 2 * 2 * 2 * SW) * sizeof(float) +
                             (size_t)T * T + 32;
static_assert(kSmemWide <= 232448, "wide leaf shared memory");
}  // namespace

__global__ void __launch_bounds__(kThreadsWide, 1) leaf_wide_kernel(LeafArgs p, int K, int I_lo)
{
    extern __shared__ __align__(16) float smem_f[];
    float *sR = smem_f;                  // T x RS3 (+1 spare row): R, S before the sweep, 0 before that
    float *sDt = sR + (T + 1) * RS3;     // T x RS3 (+1 spare row): D transposed
    float *sSlot = sDt + (T + 1) * RS3;  // 3 slots of SW x LDW: Wt, then W0, then the pre-rounding values
    float *sLA = sSlot + 3 * SW * LDW;   // LtA[1,0] block of the tile (SW x LDW)
    float *scale = sLA + SW * LDW;       // T
    float *rcp = scale + T;              // T
    float *sLBd = rcp + T;               // T: LtB[r][r-1] inside each diagonal sub-block (0 on its first row)
    float *sPS = sLBd + T;               // 2 x 2 x SW: column-side partial sums by column
    float *sPU = sPS + 2 * 2 * SW;       // 2 x 2 x SW: row-side partial sums by column
    int8_t *sCode = (int8_t *)(sPU + 2 * 2 * SW);  // T x T codes (+32 spare bytes)

    const int I = I_lo + blockIdx.x, J = K - I;
    const int64_t row0 = (int64_t)I * T, col0 = (int64_t)J * T;
    const int mr = (int)min64(T, p.m - row0), nc = (int)min64(T, p.n - col0);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const float *LAt = p.LA32 + col0 * p.Np + col0;
    const float *LBt = p.LB32 + row0 * p.Mp + row0;
    const int lda_g = (int)p.Np, ldb_g = (int)p.Mp;
    for (int idx = tid; idx < 2 * T * (T / 32); idx += kThreadsWide) {
        const int which = idx / (T * (T / 32)), r = (idx / (T / 32)) % T, seg = idx % (T / 32);
        const float *ptr = which == 0 ? LAt + r * lda_g + 32 * seg : LBt + r * ldb_g + 32 * seg;
        asm volatile("prefetch.global.L2 [%0];" ::"l"(ptr));
    }
    pdl_wait();

    // Wt block of sub-tile (pp, q) into a slot
    auto stage_wt = [&](int pp, int q, int slot) {
        for (int c = tid; c < SW * (SW / 4); c += kThreadsWide) {
            const int i = c / (SW / 4), k4 = c % (SW / 4);
            cp_async16(sSlot + slot * SW * LDW + i * LDW + 4 * k4,
                       p.Wt + (row0 + pp * SW + i) * p.Np + col0 + q * SW + 4 * k4);
        }
    };
    stage_wt(0, 0, 0);
    for (int c = tid; c < SW * (SW / 4); c += kThreadsWide) {  // LtA[1,0]
        const int j = c / (SW / 4), k4 = c % (SW / 4);
        cp_async16(sLA + j * LDW + 4 * k4, LAt + (SW + j) * lda_g + 4 * k4);
    }
    asm volatile("cp.async.commit_group;" ::: "memory");

    for (int idx = tid; idx < (T + 1) * RS3 / 4; idx += kThreadsWide) {
        ((float4 *)sR)[idx] = make_float4(0.f, 0.f, 0.f, 0.f);
        ((float4 *)sDt)[idx] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    if (tid < T) {
        const int blk = tid / SW, r = tid % SW;
        sLBd[tid] = r > 0 ? LBt[(blk * SW + r) * ldb_g + blk * SW + r - 1] : 0.f;
    }
    const float fqmin = (float)p.qmin, fqmax = (float)p.qmax;
    const int wp = warp / 6, wr = warp % 6, role = wr >> 1, half = wr & 1;
    const bool exact_div = __syncthreads_or(load_scales(p, scale, rcp, row0, mr)) != 0;

    for (int e = 0; e < 3; ++e) {
        const int p_lo = max(0, e - 1), p_hi = min(1, e);
        const bool mine = wp >= p_lo && wp <= p_hi;
        const int qv = e - wp;
        const int slot = e == 1 ? 1 + wp : 0;
        // S[1,q] = LtB[1,0] D[0,q] into R's (1,q) block: four warps, 16 rows each
        if (mine && wp == 1 && wr < 4) {
            float acc[8][4] = {};
            mma_block<8>(acc, LBt + SW * ldb_g, ldb_g, sDt + (qv * SW) * RS3, RS3, SW, wr * 16, 0);
            const int g = lane >> 2, t = lane & 3;
            float *o = sR + SW * RS3 + qv * SW;
#pragma unroll
            for (int nt = 0; nt < 8; ++nt) {
                const int j = nt * 8 + 2 * t;
                o[(wr * 16 + g) * RS3 + j] = acc[nt][0];
                o[(wr * 16 + g) * RS3 + j + 1] = acc[nt][1];
                o[(wr * 16 + g + 8) * RS3 + j] = acc[nt][2];
                o[(wr * 16 + g + 8) * RS3 + j + 1] = acc[nt][3];
            }
        }
        // the sums' coefficient rows, columns <= (own index) - 2: row-side warps
        // LtA[q,q] row b, column-side warps LtB[p,p] row rho (one register array
        // serves either role); entry warps: LtA[b][b-1]
        float2 coef[SW / 2];
        float la_new = 0.f;
        if (mine && role >= 1) {
            const int x = half * 32 + lane;
            const float *row = role == 1 ? LAt + (qv * SW + x) * lda_g + qv * SW : LBt + (wp * SW + x) * ldb_g + wp * SW;
#pragma unroll
            for (int c = 0; c < SW / 2; ++c) {
                float2 v = make_float2(0.f, 0.f);
                if (2 * c <= x - 2) v = *(const float2 *)(row + 2 * c);
                v.y = 2 * c + 1 <= x - 2 ? v.y : 0.f;
                coef[c] = v;
            }
        }
        if (mine && role == 0) {
            const int b = half * 32 + lane;
            if (b > 0) la_new = LAt[(qv * SW + b) * lda_g + qv * SW + b - 1];
        }
        asm volatile("cp.async.wait_all;" ::: "memory");
        __syncthreads();
        // W0[p,q] = Wt[p,q] - R[p,0] LtA[1,0]^T (q = 1) - S[p,q], in place in the slot
        if (mine && wr < 4) {
            float acc[8][4] = {};
            if (qv == 1) mma_block<8>(acc, sR + (wp * SW) * RS3, RS3, sLA, LDW, SW, wr * 16, 0);
            const int g = lane >> 2, t = lane & 3;
            float *o = sSlot + slot * SW * LDW;
            const float *sq = sR + (wp * SW) * RS3 + qv * SW;
#pragma unroll
            for (int nt = 0; nt < 8; ++nt) {
                const int j = nt * 8 + 2 * t, i = wr * 16 + g;
                o[i * LDW + j] -= acc[nt][0] + sq[i * RS3 + j];
                o[i * LDW + j + 1] -= acc[nt][1] + sq[i * RS3 + j + 1];
                o[(i + 8) * LDW + j] -= acc[nt][2] + sq[(i + 8) * RS3 + j];
                o[(i + 8) * LDW + j + 1] -= acc[nt][3] + sq[(i + 8) * RS3 + j + 1];
            }
        }
        __syncthreads();
        if (e == 0) {  // phase 1's blocks, while phase 0 sweeps
            stage_wt(0, 1, 1);
            stage_wt(1, 0, 2);
            asm volatile("cp.async.commit_group;" ::: "memory");
        } else if (e == 1) {  // phase 2's block into the slot phase 0 used
            stage_wt(1, 1, 0);
            asm volatile("cp.async.commit_group;" ::: "memory");
        }
        if (mine) {
            const int pp = wp, q = qv;
            float *ps_buf = sPS + pp * 2 * SW;
            float *pu_buf = sPU + pp * 2 * SW;
            float *Wp = sSlot + slot * SW * LDW;
            const float *LBd = sLBd + pp * SW;
            const int bar_id = 1 + pp;
            if (role == 0) {
                const int b = half * 32 + lane, tb = q * SW + b;
                auto row_consts = [&](int a, float &w0, float &lbn, float &sv, float &rv_, float &s0) {
                    const int ac = min(max(a, 0), SW - 1);
                    w0 = Wp[ac * LDW + b];
                    lbn = LBd[ac];
                    sv = scale[pp * SW + ac];
                    rv_ = rcp[pp * SW + ac];
                    s0 = sR[(pp * SW + ac) * RS3 + tb];
                };
                auto sweep = [&](auto ieee_tag) {
                    constexpr bool kIeee = decltype(ieee_tag)::value;
                    float w0, lb_new, sc_s, sc_r, s_ab;
                    row_consts(-b, w0, lb_new, sc_s, sc_r, s_ab);
                    float d_prev = 0.f;
#pragma unroll 2
                    for (int d = 0; d < 2 * SW - 1; ++d) {
                        const int a = d - b;
                        const int ac = min(max(a, 0), SW - 1);
                        const float ps_in = d > 0 ? ps_buf[(d & 1) * SW + b] : 0.f;
                        const float pu_in = d > 0 ? pu_buf[(d & 1) * SW + b] : 0.f;
                        const float r_new = b > 0 ? sR[(pp * SW + ac) * RS3 + tb - 1] : 0.f;
                        float w0n, lbn_n, sn, rn, s_n;
                        row_consts(a + 1, w0n, lbn_n, sn, rn, s_n);
                        const float sc = fmaf(lb_new, d_prev, ps_in);
                        const float wt = w0 - fmaf(r_new, la_new, pu_in) - sc;
                        const float qf = kIeee ? __fdiv_rn(wt, sc_s) : div_rn_recip(wt, sc_s, sc_r);
                        const float cq = fminf(fmaxf(rintf(qf), fqmin), fqmax);
                        const int ta = pp * SW + a;
                        const bool valid = a >= 0 && a < SW && ta < mr && tb < nc;
                        const float dl = valid ? fmaf(-sc_s, cq, wt) : 0.f;
                        const int iR = valid ? ta * RS3 + tb : T * RS3 + lane;
                        const int iD = valid ? tb * RS3 + ta : T * RS3 + lane;
                        const int iC = valid ? ta * T + tb : T * T + lane;
                        const int iW = valid ? a * LDW + b : ac * LDW + SW + (lane & 3);
                        sR[iR] = s_ab + sc + dl;
                        sDt[iD] = dl;
                        sCode[iC] = code_byte(cq);
                        Wp[iW] = wt;
                        d_prev = dl;
                        w0 = w0n; lb_new = lbn_n; sc_s = sn; sc_r = rn; s_ab = s_n;
                        group_sync(bar_id, 192);
                    }
                };
                if (exact_div)
                    sweep(std::true_type{});
                else
                    sweep(std::false_type{});
            } else if (role == 1) {
                // row-side sums sum_{c <= b-2} R[a+1][c] LtA[b][c]
                const int b = half * 32 + lane;
                float4 rv[SW / 4];
#pragma unroll
                for (int c = 0; c < SW / 4; ++c) rv[c] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 2
                for (int d = 0; d < 2 * SW - 1; ++d) {
                    const int an = min(max(d - b + 1, 0), SW - 1);
                    const float *Rn = sR + (pp * SW + an) * RS3 + q * SW;
#pragma unroll
                    for (int c = 0; c < SW / 4; ++c)
                        if (4 * c <= b - 2) rv[c] = *(const float4 *)(Rn + 4 * c);
                    float2 u0 = make_float2(0.f, 0.f), u1 = make_float2(0.f, 0.f);
                    float2 u2 = make_float2(0.f, 0.f), u3 = make_float2(0.f, 0.f);
#pragma unroll
                    for (int c = 0; c < SW / 4; c += 2) {
                        u0 = ffma2(make_float2(rv[c].x, rv[c].y), coef[2 * c], u0);
                        u1 = ffma2(make_float2(rv[c].z, rv[c].w), coef[2 * c + 1], u1);
                        u2 = ffma2(make_float2(rv[c + 1].x, rv[c + 1].y), coef[2 * c + 2], u2);
                        u3 = ffma2(make_float2(rv[c + 1].z, rv[c + 1].w), coef[2 * c + 3], u3);
                    }
                    pu_buf[((d + 1) & 1) * SW + b] = ((u0.x + u1.x) + (u2.x + u3.x)) + ((u0.y + u1.y) + (u2.y + u3.y));
                    group_sync(bar_id, 192);
                }
            } else {
                // column-side sums sum_{r <= rho-2} LtB[rho][r] D[r][b], b = d+1-rho
                const int rho = half * 32 + lane;
                float4 dv[SW / 4];
#pragma unroll
                for (int c = 0; c < SW / 4; ++c) dv[c] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 2
                for (int d = 0; d < 2 * SW - 1; ++d) {
                    const int b = d + 1 - rho;
                    const int bc = min(max(b, 0), SW - 1);
                    const float *Dc = sDt + (q * SW + bc) * RS3 + pp * SW;
#pragma unroll
                    for (int c = 0; c < SW / 4; ++c)
                        if (4 * c <= rho - 2) dv[c] = *(const float4 *)(Dc + 4 * c);
                    float2 s0 = make_float2(0.f, 0.f), s1 = make_float2(0.f, 0.f);
                    float2 s2 = make_float2(0.f, 0.f), s3 = make_float2(0.f, 0.f);
#pragma unroll
                    for (int c = 0; c < SW / 4; c += 2) {
                        s0 = ffma2(make_float2(dv[c].x, dv[c].y), coef[2 * c], s0);
                        s1 = ffma2(make_float2(dv[c].z, dv[c].w), coef[2 * c + 1], s1);
                        s2 = ffma2(make_float2(dv[c + 1].x, dv[c + 1].y), coef[2 * c + 2], s2);
                        s3 = ffma2(make_float2(dv[c + 1].z, dv[c + 1].w), coef[2 * c + 3], s3);
                    }
                    if (b == bc)
                        ps_buf[((d + 1) & 1) * SW + b] = ((s0.x + s1.x) + (s2.x + s3.x)) + ((s0.y + s1.y) + (s2.y + s3.y));
                    group_sync(bar_id, 192);
                }
            }
        }
        __syncthreads();
        if (p.wt_out) {
            for (int idx = tid; idx < (p_hi - p_lo + 1) * SW * SW; idx += kThreadsWide) {
                const int pp = p_lo + idx / (SW * SW), r = (idx / SW) % SW, c = idx % SW;
                const int sl = e == 1 ? 1 + pp : 0;
                const int ta = pp * SW + r, tb = (e - pp) * SW + c;
                if (ta < mr && tb < nc) p.wt_out[(row0 + ta) * p.n + col0 + tb] = sSlot[sl * SW * LDW + r * LDW + c];
            }
        }
    }
    pdl_trigger();
    for (int idx = tid; idx < T * T; idx += kThreadsWide) {
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
    e = cudaFuncSetAttribute(leaf_wide_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemWide);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(leaf_single_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemSingle);
    if (e != cudaSuccess) return e;
    if ((e = leaf_cluster_configure()) != cudaSuccess) return e;
    return leaf_wave_configure();
}

cudaError_t launch_leaf(const LeafArgs &p, int K, int variant, cudaStream_t stream)
{
    int I_lo = max(0, K - (p.Nt - 1)), I_hi = min(p.Mt - 1, K);
    if (I_hi < I_lo) return cudaSuccess;
    if (variant == 7) return launch_leaf_wave(p, K, I_lo, I_hi - I_lo + 1, stream);
    if (variant == 4 || variant == 5)
        return launch_leaf_cluster(p, K, I_lo, I_hi - I_lo + 1, variant == 5, stream);
    if (variant == 3)
        return launch_pdl(leaf_wide_kernel, dim3(I_hi - I_lo + 1), dim3(kThreadsWide), kSmemWide, stream, p, K, I_lo);
    if (variant == 2)
        return launch_pdl(leaf_warp_kernel, dim3(I_hi - I_lo + 1), dim3(kThreadsW), kSmemWarp, stream, p, K, I_lo);
    if (variant == 1)
        return launch_pdl(leaf_single_kernel, dim3(I_hi - I_lo + 1), dim3(kThreads), kSmemSingle, stream, p, K, I_lo);
    return launch_pdl(leaf_nested_kernel, dim3(I_hi - I_lo + 1), dim3(kThreads), kSmemNested, stream, p, K, I_lo);
}

}  // namespace bakron
