// leaf_gptq.cu -- the leaf of the one-sided path (B = I): with B the identity
// the output side couples nothing, rows are independent, and the product
// order reduces to GPTQ's column order (the review's check that the two-sided
// solve reduces to one-sided GPTQ when B = I).  The recursion then runs over
// 128-column blocks; this kernel rounds one block.
//
// One CTA of four warps per 32 rows, lane = row in every warp.  The block is
// rounded in column order, 8 columns per step k, in the pull form
//     Wt_j = W_j - sum_{j' < j} Delta_j' LtA[j, j'] .
// Warp 0 rounds; warps 1-3 work one step ahead: during step k they form, for
// step k+1's 8 columns, the sums over the columns before step k (4-column
// chunks split three ways: 16-byte reads of the lane's own residuals,
// broadcast reads of 8 factor rows, 8 independent sums each).  At step k warp
// 0 adds the three partial sums and the two chunks of step k-1 (its own, just
// written), then rounds the 8 columns in order, applying the terms among them
// as each residual appears.  One CTA barrier per step; every loop is short,
// so the kernel runs from the instruction cache.  W and the residuals share
// one row per lane in shared memory (a column's W is replaced by its
// residual).  Codes, V and the residual's TF32 split are staged in shared
// memory and written row-coalesced at the end by all four warps.
#include "common.cuh"
#include "kernels.cuh"

namespace bakron {

namespace {
constexpr int GB = 128;          // column block
constexpr int GS = 8;            // columns per step
constexpr int NSTEP = GB / GS;   // 16 steps
constexpr int NHELP = 3;         // warps forming the next step's sums
constexpr int kThreadsG = 32 * (1 + NHELP);
constexpr int LDL = GB + 4;      // row stride of the LtA diagonal block in smem (16-byte rows)
constexpr int LDX = GB + 4;      // row stride of the W / residual rows (16-byte rows; 8 lanes cover the banks)
constexpr int LDO = GB + 1;      // row stride of the staged V and codes (odd: a lane per row hits its own bank)
constexpr int LDP = 12;          // per-lane stride of the partial sums (16-byte aligned, 8 lanes cover the banks)
constexpr size_t kSmemGptq = ((size_t)GB * LDL + (size_t)32 * LDX + (size_t)32 * LDO +
                              (size_t)2 * NHELP * 32 * LDP) * sizeof(float) + (size_t)32 * LDO + 32;
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

// acc[r] += sum over 4-column chunk g of x[4g + t] * LtA[c0 + r, 4g + t]
__device__ __forceinline__ void add_chunk(float (&acc)[GS], const float *x, const float *sLA, int c0, int g)
{
    const float4 dv = ((const float4 *)x)[g];
#pragma unroll
    for (int r = 0; r < GS; ++r) {
        const float4 c = *(const float4 *)(sLA + (c0 + r) * LDL + 4 * g);
        acc[r] = fmaf(dv.x, c.x, acc[r]);
        acc[r] = fmaf(dv.y, c.y, acc[r]);
        acc[r] = fmaf(dv.z, c.z, acc[r]);
        acc[r] = fmaf(dv.w, c.w, acc[r]);
    }
}

// Warp 0, step k: the 8 columns [8k, 8k + 8) of the lane's row.
template <bool IEEE>
__device__ __forceinline__ void round_step(int k, float *x, const float *sLA, const float *part, float s, float rs,
                                           float fqmin, float fqmax, float *dV, int8_t *dC, int ncols,
                                           float *wt_row)
{
    const int c0 = k * GS, lane = threadIdx.x & 31;
    float acc[GS];
#pragma unroll
    for (int r = 0; r < GS; ++r) acc[r] = 0.f;
    if (k >= 2) {  // the helpers' sums over the columns before step k-1
#pragma unroll
        for (int h = 0; h < NHELP; ++h) {
            const float4 a = *(const float4 *)(part + (h * 32 + lane) * LDP);
            const float4 b = *(const float4 *)(part + (h * 32 + lane) * LDP + 4);
            acc[0] += a.x; acc[1] += a.y; acc[2] += a.z; acc[3] += a.w;
            acc[4] += b.x; acc[5] += b.y; acc[6] += b.z; acc[7] += b.w;
        }
    }
    if (k >= 1) {  // the columns of step k-1
        add_chunk(acc, x, sLA, c0, 2 * k - 2);
        add_chunk(acc, x, sLA, c0, 2 * k - 1);
    }
    float w[GS];
#pragma unroll
    for (int q = 0; q < GS / 4; ++q) {
        const float4 v = ((const float4 *)x)[c0 / 4 + q];
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
}  // namespace

__global__ void __launch_bounds__(kThreadsG, 1) leaf_gptq_kernel(LeafArgs p, int Jb)
{
    extern __shared__ __align__(16) float smem_g[];
    float *sLA = smem_g;                 // GB x LDL: LtA[col0 + j, col0 + 0..127] in row j
    float *sX = sLA + GB * LDL;          // 32 x LDX: the rows of W, then of the residuals
    float *sV = sX + 32 * LDX;           // 32 x LDO: V
    float *sP = sV + 32 * LDO;           // 2 x NHELP x 32 x LDP: the helpers' partial sums (double buffered)
    int8_t *sC = (int8_t *)(sP + 2 * NHELP * 32 * LDP);  // 32 x LDO: codes
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t row = (int64_t)blockIdx.x * 32 + lane;
    const int64_t col0 = (int64_t)Jb * GB;
    const bool live = row < p.m;
    const int64_t rowc = live ? row : p.m - 1;
    const float *LAt = p.LA32 + col0 * p.Np + col0;
    pdl_wait();
    // the factor's diagonal block (rows coalesced) and the 32 rows of Wt
    for (int i = tid; i < GB * (GB / 4); i += kThreadsG) {
        const int r = i / (GB / 4), c4 = i % (GB / 4);
        cp_async16_g(sLA + r * LDL + 4 * c4, LAt + (int64_t)r * p.Np + 4 * c4);
    }
    for (int i = tid; i < 32 * (GB / 4); i += kThreadsG) {
        const int r = i / (GB / 4), c4 = i % (GB / 4);
        const int64_t gr = min64((int64_t)blockIdx.x * 32 + r, p.m - 1);
        cp_async16_g(sX + r * LDX + 4 * c4, p.Wt + gr * p.Np + col0 + 4 * c4);
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
    const float s = p.scales[rowc], rs = __frcp_rn(s);
    const bool ieee = __any_sync(0xffffffffu, !(s >= 0x1p-60f && s <= 0x1p60f));
    asm volatile("cp.async.wait_all;" ::: "memory");
    __syncthreads();
    const float fqmin = (float)p.qmin, fqmax = (float)p.qmax;
    float *x = sX + lane * LDX;
    const int ncols = (int)min64(GB, p.n - col0);
    for (int k = 0; k < NSTEP; ++k) {
        if (warp == 0) {
            const float *part = sP + (k & 1) * NHELP * 32 * LDP;
            float *wt_row = p.wt_out && live ? p.wt_out + row * p.n + col0 : nullptr;
            if (ieee)
                round_step<true>(k, x, sLA, part, s, rs, fqmin, fqmax, sV + lane * LDO, sC + lane * LDO, ncols,
                                 wt_row);
            else
                round_step<false>(k, x, sLA, part, s, rs, fqmin, fqmax, sV + lane * LDO, sC + lane * LDO, ncols,
                                  wt_row);
        } else if (k + 1 < NSTEP) {
            // step k+1's sums over the columns before step k (chunks g < 2k), split three ways
            const int h = warp - 1, c1 = (k + 1) * GS;
            float acc[GS];
#pragma unroll
            for (int r = 0; r < GS; ++r) acc[r] = 0.f;
            for (int g = h; g < 2 * k; g += NHELP) add_chunk(acc, x, sLA, c1, g);
            float *o = sP + ((k + 1) & 1) * NHELP * 32 * LDP + (h * 32 + lane) * LDP;
            *(float4 *)o = make_float4(acc[0], acc[1], acc[2], acc[3]);
            *(float4 *)(o + 4) = make_float4(acc[4], acc[5], acc[6], acc[7]);
        }
        __syncthreads();  // step k's residuals and step k+1's partial sums are in place
    }
    pdl_trigger();
    // row-coalesced writes: each warp walks every fourth row, lanes along the columns
    for (int r = warp; r < 32; r += kThreadsG / 32) {
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
    return launch_pdl(leaf_gptq_kernel, dim3((unsigned)(p.Mp / 32)), dim3(kThreadsG), kSmemGptq, stream, p, Jb);
}

}  // namespace bakron
