// band_simt.cu -- FP32 CUDA-core band products of Algorithm 6's postponed
// updates ("two dense matmuls per level"): the cross-check kernels for the
// tensor-core path.  Operands are read as hi + lo, which reconstructs the
// fp32 value to within one TF32 rounding of the low part.
#include "common.cuh"
#include "kernels.cuh"

namespace bakron {

namespace {
constexpr int T = kTile;
constexpr int BK = 16;
}

template <int STAGE>
__global__ void __launch_bounds__(256) band_simt_kernel(NodeParams np, GemmArgs g)
{
    const Item it = STAGE == 1 ? stage1_item(np, blockIdx.x, blockIdx.y)
                               : stage2_item(np, blockIdx.x, blockIdx.y);
    if (!it.valid) return;
    pdl_wait();
    __shared__ float As[BK][T + 4];
    __shared__ float Bs[BK][T + 4];
    const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
    const int64_t arow = (int64_t)it.ra * T, brow = (int64_t)it.rb * T;
    float acc[8][8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;

    const int lr = tid >> 1, lc = (tid & 1) * 8;
    for (int64_t kk = (int64_t)it.k0 * T; kk < (int64_t)it.k1 * T; kk += BK) {
        const int64_t ao = (arow + lr) * g.lda + kk + lc, bo = (brow + lr) * g.ldb + kk + lc;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            As[lc + c][lr] = g.Ahi[ao + c] + g.Alo[ao + c];
            Bs[lc + c][lr] = g.Bhi[bo + c] + g.Blo[bo + c];
        }
        __syncthreads();
#pragma unroll
        for (int k = 0; k < BK; ++k) {
            float a[8], b[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) a[i] = As[k][ty * 8 + i];
#pragma unroll
            for (int j = 0; j < 8; ++j) b[j] = Bs[k][tx * 8 + j];
#pragma unroll
            for (int i = 0; i < 8; ++i)
#pragma unroll
                for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int64_t o = (arow + ty * 8 + i) * g.ldo + brow + tx * 8;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            if (STAGE == 1) {
                float hi, lo;
                split_tf32(acc[i][j], hi, lo);
                g.out_hi[o + j] = hi;
                g.out_lo[o + j] = lo;
            } else {
                g.out_acc[o + j] -= acc[i][j];
            }
        }
    }
}

cudaError_t launch_band_simt(int stage, const NodeParams &np, const GemmArgs &g, cudaStream_t stream)
{
    if (stage == 1) return launch_pdl(band_simt_kernel<1>, dim3(np.l, np.Mt), dim3(256), 0, stream, np, g);
    return launch_pdl(band_simt_kernel<2>, dim3(np.l - np.h, np.Mt), dim3(256), 0, stream, np, g);
}

}  // namespace bakron
