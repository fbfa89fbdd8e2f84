// leaf_gptq.cu -- the leaf of the one-sided path (B = I): with B the identity
// the output side couples nothing, rows are independent, and the product
// order reduces to GPTQ's column order (the review's check that the two-sided
// solve reduces to one-sided GPTQ when B = I).  The recursion then runs over
// 128-column blocks; this kernel rounds one block.
//
// One warp per 32 rows, lane = row.  The row's 128 block entries live in
// registers; the block is rounded column by column in two halves of 64 in
// GPTQ's push form: after rounding column j, every later column j' of the
// half loses Delta_j LtA[j', j], and after the first half its 64 residuals are
// pushed into the second half.  The coefficients come from the block's
// transposed copy (prepared once per solve), so the ones a column pushes are
// contiguous: one asynchronous 64 KB copy into shared memory, then 16-byte
// broadcast reads.  Codes, V and the residual's TF32 split are staged in
// shared memory and written row-coalesced at the end.
#include "common.cuh"
#include "kernels.cuh"

namespace bakron {

namespace {
constexpr int GB = 128;        // column block
constexpr int GH = 64;         // half block
constexpr int LDL = GB + 4;    // row stride of the transposed diagonal block in smem (16-byte rows)
constexpr int LDO = GB + 1;    // row stride of the staged outputs (odd: a lane per row hits its own bank)
constexpr size_t kSmemGptq = ((size_t)GB * LDL + 2 * 32 * LDO + 32) * sizeof(float) + (size_t)32 * LDO + 32;
static_assert(kSmemGptq <= 232448, "one-sided leaf shared memory");

__device__ __forceinline__ void cp_async16_g(float *dst, const float *src)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"((uint32_t)__cvta_generic_to_shared(dst)),
                 "l"(src)
                 : "memory");
}

// w[C0 + jj] -= d * LtA[C0 + jj, C0 + j] for jj in (j, 64): the coefficients
// are row C0 + j of the transposed block, read four at a time.  Called with j
// a constant (inside fully unrolled loops), so every bound folds away.
template <int C0>
__device__ __forceinline__ void push_half(float (&w)[GB], const float *crow, float d, int j)
{
#pragma unroll
    for (int g = 0; g < GH / 4; ++g) {
        if (4 * g + 3 > j) {
            const float4 c = *(const float4 *)(crow + C0 + 4 * g);
            const float cc[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
            for (int e = 0; e < 4; ++e)
                if (4 * g + e > j) w[C0 + 4 * g + e] = fmaf(-d, cc[e], w[C0 + 4 * g + e]);
        }
    }
}

__device__ __forceinline__ int8_t code_byte1(float c)
{
    return (int8_t)(__float_as_int(c + 12582912.0f) & 0xFF);
}

// Round the 64 columns [c0, c0 + 64) of the lane's row: push form inside the
// half; residual, V and code of each column go to the staging rows (columns
// at or beyond n are zero padding: their value, code and residual are 0).
template <bool IEEE, int C0>
__device__ __forceinline__ void gptq_half(float (&w)[GB], const float *sLA, float s, float rs, float fqmin,
                                          float fqmax, float *dD, float *dV, int8_t *dC, int ncols, float *wt_row)
{
#pragma unroll
    for (int j = 0; j < GH; ++j) {
        const float wt = w[C0 + j];
        const float qf = IEEE ? __fdiv_rn(wt, s) : div_rn_recip(wt, s, rs);
        const float cq = fminf(fmaxf(rintf(qf), fqmin), fqmax);
        const float d = fmaf(-s, cq, wt);
        push_half<C0>(w, sLA + (C0 + j) * LDL, d, j);
        dD[C0 + j] = d;
        dV[C0 + j] = s * cq;
        dC[C0 + j] = code_byte1(cq);
        if (wt_row && C0 + j < ncols) wt_row[C0 + j] = wt;
    }
}
}  // namespace

__global__ void __launch_bounds__(32, 1) leaf_gptq_kernel(LeafArgs p, int Jb)
{
    extern __shared__ __align__(16) float smem_g[];
    float *sLA = smem_g;                     // GB x LDL: row j = LtA[col0 + 0..127, col0 + j]
    float *sD = sLA + GB * LDL;              // 32 x LDO: residuals of the warp's rows
    float *sV = sD + 32 * LDO;               // 32 x LDO: V
    float *sWt = sV + 32 * LDO;              // 32 floats spare (alignment)
    int8_t *sC = (int8_t *)(sWt + 32);       // 32 x LDO: codes
    const int lane = threadIdx.x;
    const int64_t row = (int64_t)blockIdx.x * 32 + lane;
    const int64_t col0 = (int64_t)Jb * GB;
    const float *LAt = p.LAdT + col0 * GB;  // transposed diagonal block Jb, contiguous
    pdl_wait();
#pragma unroll 8
    for (int r = 0; r < GB; ++r) cp_async16_g(sLA + r * LDL + 4 * lane, LAt + r * GB + 4 * lane);
    asm volatile("cp.async.commit_group;" ::: "memory");
    const bool live = row < p.m;
    const int64_t rowc = live ? row : p.m - 1;
    float w[GB];
#pragma unroll
    for (int c4 = 0; c4 < GB / 4; ++c4) {
        const float4 v = *(const float4 *)(p.Wt + rowc * p.Np + col0 + 4 * c4);
        w[4 * c4] = v.x; w[4 * c4 + 1] = v.y; w[4 * c4 + 2] = v.z; w[4 * c4 + 3] = v.w;
    }
    const float s = p.scales[rowc], rs = __frcp_rn(s);
    const bool ieee = __any_sync(0xffffffffu, !(s >= 0x1p-60f && s <= 0x1p60f));
    asm volatile("cp.async.wait_all;" ::: "memory");
    __syncwarp();
    const float fqmin = (float)p.qmin, fqmax = (float)p.qmax;
    float *dD = sD + lane * LDO, *dV = sV + lane * LDO;
    int8_t *dC = sC + lane * LDO;
    float *wt_row = p.wt_out && live ? p.wt_out + row * p.n + col0 : nullptr;
    const int ncols = (int)min64(GB, p.n - col0);
    if (ieee)
        gptq_half<true, 0>(w, sLA, s, rs, fqmin, fqmax, dD, dV, dC, ncols, wt_row);
    else
        gptq_half<false, 0>(w, sLA, s, rs, fqmin, fqmax, dD, dV, dC, ncols, wt_row);
    // the first half's residuals reach the second half
#pragma unroll 2
    for (int j = 0; j < GH; ++j) {
        const float d = dD[j];
        const float *crow = sLA + j * LDL + GH;
#pragma unroll
        for (int g = 0; g < GH / 4; ++g) {
            const float4 c = *(const float4 *)(crow + 4 * g);
            w[GH + 4 * g] = fmaf(-d, c.x, w[GH + 4 * g]);
            w[GH + 4 * g + 1] = fmaf(-d, c.y, w[GH + 4 * g + 1]);
            w[GH + 4 * g + 2] = fmaf(-d, c.z, w[GH + 4 * g + 2]);
            w[GH + 4 * g + 3] = fmaf(-d, c.w, w[GH + 4 * g + 3]);
        }
    }
    if (ieee)
        gptq_half<true, GH>(w, sLA, s, rs, fqmin, fqmax, dD, dV, dC, ncols, wt_row);
    else
        gptq_half<false, GH>(w, sLA, s, rs, fqmin, fqmax, dD, dV, dC, ncols, wt_row);
    __syncwarp();
    pdl_trigger();
    // row-coalesced writes: the warp walks its 32 rows, lanes along the columns
    for (int r = 0; r < 32; ++r) {
        const int64_t gr = (int64_t)blockIdx.x * 32 + r;
        if (gr >= p.m) break;
        for (int c = lane; c < GB; c += 32) {
            const int64_t gc = col0 + c;
            float hi, lo;
            split_tf32(sD[r * LDO + c], hi, lo);
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
