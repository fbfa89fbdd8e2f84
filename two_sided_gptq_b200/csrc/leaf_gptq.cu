// leaf_gptq.cu -- the leaf of the one-sided path (B = I): with B the identity
// the output side couples nothing, rows are independent, and the product
// order reduces to GPTQ's column order (the review's check that the two-sided
// solve reduces to one-sided GPTQ when B = I).  The recursion then runs over
// 128-column blocks; this kernel rounds one block.
//
// One warp per 32 rows, lane = row.  The block is rounded in column order in
// steps of 8 columns, in the pull form
//     Wt_j = W_j - sum_{j' < j} Delta_j' LtA[j, j'] :
// for the next 8 columns, the terms of all earlier columns of the block come
// from one loop over 4-column chunks (16-byte reads of the lane's own residuals
// and broadcast reads of the 8 factor rows, 8 independent sums), then the 8
// columns are rounded in order with the terms among themselves applied as
// each residual appears.  Every code path is a short loop, so the kernel runs
// from the instruction cache; W and the residuals share one row per lane in
// shared memory (a column's W is replaced by its residual).  Codes, V and the
// residual's TF32 split are staged in shared memory and written row-coalesced
// at the end.
#include "common.cuh"
#include "kernels.cuh"

namespace bakron {

namespace {
constexpr int GB = 128;      // column block
constexpr int GS = 8;        // columns per step
constexpr int LDL = GB + 4;  // row stride of the LtA diagonal block in smem (16-byte rows)
constexpr int LDX = GB + 4;  // row stride of the W / residual rows (16-byte rows; 8 lanes cover the banks)
constexpr int LDO = GB + 1;  // row stride of the staged V and codes (odd: a lane per row hits its own bank)
constexpr size_t kSmemGptq =
    ((size_t)GB * LDL + (size_t)32 * LDX + (size_t)32 * LDO) * sizeof(float) + (size_t)32 * LDO + 32;
static_assert(kSmemGptq <= 232448, "one-sided leaf shared memory");

__device__ __forceinline__ void cp_async16_g(float *dst, const float *src)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"((uint32_t)__cvta_generic_to_shared(dst)),
                 "l"(src)
                 : "memory");
}

__device__ __forceinline__ int8_t code_byte1(float c)
{
    return (int8_t)(__float_as_int(c + 12582912.0f) & 0xFF);
}

// Round the block's columns in steps of GS; x = the lane's row (W, replaced
// column by column by the residual), sLA = the factor's diagonal block.
template <bool IEEE>
__device__ __forceinline__ void gptq_block(float *x, const float *sLA, float s, float rs, float fqmin, float fqmax,
                                           float *dV, int8_t *dC, int ncols, float *wt_row)
{
    const float4 *x4 = (const float4 *)x;
#pragma unroll 1
    for (int c0 = 0; c0 < GB; c0 += GS) {
        // terms of the columns before c0
        float acc[GS];
#pragma unroll
        for (int r = 0; r < GS; ++r) acc[r] = 0.f;
#pragma unroll 2
        for (int g = 0; g < c0 / 4; ++g) {
            const float4 dv = x4[g];
#pragma unroll
            for (int r = 0; r < GS; ++r) {
                const float4 c = *(const float4 *)(sLA + (c0 + r) * LDL + 4 * g);
                acc[r] = fmaf(dv.x, c.x, acc[r]);
                acc[r] = fmaf(dv.y, c.y, acc[r]);
                acc[r] = fmaf(dv.z, c.z, acc[r]);
                acc[r] = fmaf(dv.w, c.w, acc[r]);
            }
        }
        // the step's own columns, in order
        float w[GS];
#pragma unroll
        for (int q = 0; q < GS / 4; ++q) {
            const float4 v = x4[c0 / 4 + q];
            w[4 * q] = v.x - acc[4 * q];
            w[4 * q + 1] = v.y - acc[4 * q + 1];
            w[4 * q + 2] = v.z - acc[4 * q + 2];
            w[4 * q + 3] = v.w - acc[4 * q + 3];
        }
        float cf[GS][GS];  // cf[r][r2] = LtA[c0 + r, c0 + r2], r2 < r
#pragma unroll
        for (int r = 1; r < GS; ++r)
#pragma unroll
            for (int r2 = 0; r2 < r; ++r2) cf[r][r2] = sLA[(c0 + r) * LDL + c0 + r2];
#pragma unroll
        for (int r = 0; r < GS; ++r) {
            const float wt = w[r];
            const float qf = IEEE ? __fdiv_rn(wt, s) : div_rn_recip(wt, s, rs);
            const float cq = fminf(fmaxf(rintf(qf), fqmin), fqmax);
            const float d = fmaf(-s, cq, wt);
#pragma unroll
            for (int r2 = r + 1; r2 < GS; ++r2) w[r2] = fmaf(-d, cf[r2][r], w[r2]);
            x[c0 + r] = d;
            dV[c0 + r] = s * cq;
            dC[c0 + r] = code_byte1(cq);
            if (wt_row && c0 + r < ncols) wt_row[c0 + r] = wt;
        }
    }
}
}  // namespace

__global__ void __launch_bounds__(32, 1) leaf_gptq_kernel(LeafArgs p, int Jb)
{
    extern __shared__ __align__(16) float smem_g[];
    float *sLA = smem_g;          // GB x LDL: LtA[col0 + j, col0 + 0..127] in row j
    float *sX = sLA + GB * LDL;   // 32 x LDX: the lanes' rows of W, then of the residuals
    float *sV = sX + 32 * LDX;    // 32 x LDO: V
    int8_t *sC = (int8_t *)(sV + 32 * LDO);  // 32 x LDO: codes
    const int lane = threadIdx.x;
    const int64_t row = (int64_t)blockIdx.x * 32 + lane;
    const int64_t col0 = (int64_t)Jb * GB;
    const bool live = row < p.m;
    const int64_t rowc = live ? row : p.m - 1;
    const float *LAt = p.LA32 + col0 * p.Np + col0;
    pdl_wait();
    // the factor's diagonal block (rows coalesced) and the lane's row of Wt
#pragma unroll 8
    for (int r = 0; r < GB; ++r) cp_async16_g(sLA + r * LDL + 4 * lane, LAt + (int64_t)r * p.Np + 4 * lane);
    float *x = sX + lane * LDX;
#pragma unroll 8
    for (int c4 = 0; c4 < GB / 4; ++c4) cp_async16_g(x + 4 * c4, p.Wt + rowc * p.Np + col0 + 4 * c4);
    asm volatile("cp.async.commit_group;" ::: "memory");
    const float s = p.scales[rowc], rs = __frcp_rn(s);
    const bool ieee = __any_sync(0xffffffffu, !(s >= 0x1p-60f && s <= 0x1p60f));
    asm volatile("cp.async.wait_all;" ::: "memory");
    __syncwarp();
    const float fqmin = (float)p.qmin, fqmax = (float)p.qmax;
    float *dV = sV + lane * LDO;
    int8_t *dC = sC + lane * LDO;
    float *wt_row = p.wt_out && live ? p.wt_out + row * p.n + col0 : nullptr;
    const int ncols = (int)min64(GB, p.n - col0);
    if (ieee)
        gptq_block<true>(x, sLA, s, rs, fqmin, fqmax, dV, dC, ncols, wt_row);
    else
        gptq_block<false>(x, sLA, s, rs, fqmin, fqmax, dV, dC, ncols, wt_row);
    __syncwarp();
    pdl_trigger();
    // row-coalesced writes: the warp walks its 32 rows, lanes along the columns
    for (int r = 0; r < 32; ++r) {
        const int64_t gr = (int64_t)blockIdx.x * 32 + r;
        if (gr >= p.m) break;
        for (int c = lane; c < GB; c += 32) {
            const int64_t gc = col0 + c;
            float hi, lo;
            split_tf32(sX[r * LDX + c], hi, lo);
            p.Dhi[gr * p.Np + gc] = hi;
            p.Dlo[gr * p.Np + gc] = lo;
            if (gc < p.n) {
                p.codes[gr * p.n + gc] = sC[r * LDO + c];
                p.V[gr * p.n + gc] = sV[r * LDO + c];
            }
        }
    }
}

cudaError_t leaf_gptq_configure()
{
    return cudaFuncSetAttribute(leaf_gptq_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemGptq);
}

cudaError_t launch_leaf_gptq(const LeafArgs &p, int Jb, cudaStream_t stream)
{
    return launch_pdl(leaf_gptq_kernel, dim3((unsigned)(p.Mp / 32)), dim3(32), kSmemGptq, stream, p, Jb);
}

}  // namespace bakron
