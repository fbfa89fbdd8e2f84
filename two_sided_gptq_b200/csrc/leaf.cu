// leaf.cu -- the leaf sweep: rounds every entry of one tile diagonal.
//
// Tiles (I, J) with I + J = K are mutually incomparable in the product order
// (I < I' forces J > J'), so one CTA per tile runs independently.  Inside a
// T x T tile the entries are rounded one entry anti-diagonal per step
// (entries on a diagonal are independent, Theorem 3.2's anti-diagonal
// parallelism), 2T-1 steps.  All contributions from outside the tile were
// already subtracted from Wt by the band products; inside the tile the
// intended output of Proposition 3.1 is accumulated in "pull" form:
//     Wt_ab = W0_ab - sum_{b'<b} R_ab' LtA[b,b'] - S_ab,
//     S_ab  = sum_{a'<a} LtB[a,a'] D_a'b,     R_ab = S_ab + D_ab,
// where a, b are local row/column indices and LtA, LtB are the diagonal
// blocks of the normalised factors.
#include "common.cuh"
#include "kernels.cuh"

namespace bakron {

namespace {
constexpr int T = kTile;
constexpr int S = T + 4;  // padded smem row stride: rows a..a+7 land 4 banks apart
constexpr int kLeafThreads = 4 * T;
constexpr size_t kLeafSmem = (size_t)3 * T * S * sizeof(float) + T * sizeof(float);
}  // namespace

// Thread (b, q) = (tid / 4, tid % 4) owns column b; the four threads of a
// column split the two dot products over interleaved indices 4t + q.
__global__ void __launch_bounds__(kLeafThreads, 1)
leaf_pull_kernel(LeafArgs p, int K, int I_lo)
{
    extern __shared__ float sm[];
    float *sR = sm;             // T x S: W0 on entry, overwritten by R entry by entry
    float *sDt = sR + T * S;    // T x S: sDt[b*S + a] = D_ab
    float *sLB = sDt + T * S;   // T x S: LtB diagonal block, row-major
    float *sScale = sLB + T * S;

    const int I = I_lo + blockIdx.x, J = K - I;
    const int64_t row0 = (int64_t)I * T, col0 = (int64_t)J * T;
    const int mr = (int)min64(T, p.m - row0), nc = (int)min64(T, p.n - col0);
    const int tid = threadIdx.x;

    for (int idx = tid; idx < T * T; idx += kLeafThreads) {
        int r = idx / T, c = idx % T;
        sR[r * S + c] = p.Wt[(row0 + r) * p.Np + col0 + c];
        sLB[r * S + c] = p.LB32[(row0 + r) * p.Mp + row0 + c];
        sDt[r * S + c] = 0.f;
    }
    if (tid < T) sScale[tid] = tid < mr ? p.scales[row0 + tid] : 1.f;

    const int b = tid >> 2, q = tid & 3;
    float la[T / 4];
#pragma unroll
    for (int t = 0; t < T / 4; ++t) la[t] = p.LA32[(col0 + b) * p.Np + col0 + 4 * t + q];
    __syncthreads();

    const unsigned gmask = 0xFu << (threadIdx.x & 28);
    for (int d = 0; d < 2 * T - 1; ++d) {
        const int a = d - b;
        if (a >= 0 && a < T) {
            const float *Rrow = sR + a * S;
            const float *Brow = sLB + a * S;
            const float *Dcol = sDt + b * S;
            float u = 0.f, sc = 0.f;
#pragma unroll
            for (int t = 0; t < T / 4; ++t) {
                const int idx = 4 * t + q;
                float rv = Rrow[idx], bv = Brow[idx], dv = Dcol[idx];
                u = fmaf(idx < b ? rv : 0.f, la[t], u);
                sc = fmaf(idx < a ? bv : 0.f, dv, sc);
            }
            u += __shfl_xor_sync(gmask, u, 1);
            sc += __shfl_xor_sync(gmask, sc, 1);
            u += __shfl_xor_sync(gmask, u, 2);
            sc += __shfl_xor_sync(gmask, sc, 2);
            if (q == 0 && a < mr && b < nc) {
                const float w0 = sR[a * S + b];
                const float wt = w0 - u - sc;
                const float s = sScale[a];
                float c = rintf(__fdiv_rn(wt, s));
                c = fminf(fmaxf(c, (float)p.qmin), (float)p.qmax);
                const float dl = fmaf(-s, c, wt);
                sR[a * S + b] = sc + dl;
                sDt[b * S + a] = dl;
                const int64_t gi = row0 + a, gj = col0 + b;
                p.codes[gi * p.n + gj] = (int8_t)c;
                if (p.wt_out) p.wt_out[gi * p.n + gj] = wt;
                p.V[gi * p.n + gj] = s * c;
                float hi, lo;
                split_tf32(dl, hi, lo);
                p.Dhi[gi * p.Np + gj] = hi;
                p.Dlo[gi * p.Np + gj] = lo;
            }
        }
        __syncthreads();
    }
}

cudaError_t leaf_configure()
{
    return cudaFuncSetAttribute(leaf_pull_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)kLeafSmem);
}

cudaError_t launch_leaf(const LeafArgs &p, int K, cudaStream_t stream)
{
    int I_lo = max(0, K - (p.Nt - 1)), I_hi = min(p.Mt - 1, K);
    if (I_hi < I_lo) return cudaSuccess;
    leaf_pull_kernel<<<I_hi - I_lo + 1, kLeafThreads, kLeafSmem, stream>>>(p, K, I_lo);
    return cudaGetLastError();
}

}  // namespace bakron
