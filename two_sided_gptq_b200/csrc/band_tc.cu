// band_tc.cu -- the band products of Algorithm 6 on the 5th-generation tensor
// cores (tcgen05, sm_100a), 3xTF32.
//
// Each CTA computes one T x T output tile D = sum_k A[ra rows, k] B[rb rows, k]^T
// over a contiguous range of tile columns (stage 1: X^T = LtA . Delta^T,
// stage 2: Wt -= LtB . X).  Both operands are K-major in global memory, so
// TMA loads 128-row x 32-column fp32 boxes with 128-byte swizzle straight into
// the canonical UMMA layout.  Operands are pre-split into TF32 hi/lo parts;
// every K=8 step issues hi*hi + hi*lo + lo*hi into one FP32 TMEM accumulator
// (the low*low term is below FP32 resolution).
//
// Warp roles (192 threads): warp 0 lane 0 issues TMA into a 3-stage ring;
// warp 1 owns TMEM and lane 0 issues the MMAs; warps 2..5 read the
// accumulator back (tcgen05.ld, 32 lanes each), write their rows of the
// finished tile into the then idle stage buffers in the swizzled box layout,
// and hand each 32 x 32 box to TMA: a tile store for stage 1 (X^T hi and lo),
// a tile add-reduction of -D into Wt for stage 2 (each Wt tile has one writer
// per launch, so the single rounding of Wt + (-D) equals a read-modify-write).
// Every mbarrier wait is bounded by a %globaltimer deadline; on expiry the
// kernel records BAKRON_ERR_DEVICE_TIMEOUT, drains what it issued and exits.
#include <cuda.h>

#include "common.cuh"
#include "kernels.cuh"
#include "tcgen05.cuh"

namespace bakron {

using namespace tc;

namespace {
constexpr int T = kTile;
constexpr int KB = 32;                    // fp32 columns per stage (128 bytes)
constexpr int kStages = 3;
constexpr int kTileBytes = T * KB * 4;    // 16 KB per operand part
constexpr int kBoxBytes = 32 * KB * 4;    // 4 KB: one 32 x 32 output box
constexpr int kStageBytes = 4 * kTileBytes;
constexpr int kThreads = 192;
constexpr size_t kSmem = (size_t)kStages * kStageBytes + 1024 /*align*/ + 256 /*barriers*/;
constexpr uint32_t kTmemCols = 2 * T;  // two accumulator buffers

// Instruction descriptor: D fp32, A/B tf32, K-major both, N = 128, M = 128.
constexpr uint32_t kIdesc = (1u << 4) | (2u << 7) | (2u << 10) | ((uint32_t)(T >> 3) << 17) |
                            ((uint32_t)(T >> 4) << 24);

}  // namespace

template <int STAGE>
__global__ void __launch_bounds__(kThreads, 1)
band_tc_kernel(const __grid_constant__ TcMaps maps, NodeParams np, GemmArgs g)
{
    // STAGE 1, 2: the band products; 3: Gram tiles; 4: the one-sided update;
    // 5: full GEMM tiles (the proxy loss's products).  With np.lpt the band
    // products run on a (row tile, key offset) grid with the key offset
    // descending along y: CTAs are dispatched x-fastest, so the items with
    // the longest contractions (the largest offsets) start first and the
    // short ones fill the tail of the last wave.
    const bool lpt = STAGE <= 2 && np.lpt;
    const int bx = lpt ? (int)(gridDim.y - 1 - blockIdx.y) : (int)blockIdx.x;
    const int by = lpt ? (int)blockIdx.x : (int)blockIdx.y;
    const Item it = STAGE == 1   ? stage1_item(np, bx, by)
                    : STAGE == 2 ? stage2_item(np, bx, by)
                    : STAGE == 3 ? gram_item(np, blockIdx.x, blockIdx.y)
                    : STAGE == 4 ? gptq_item(np, blockIdx.x, blockIdx.y)
                                 : full_item(np, blockIdx.x, blockIdx.y);
    if (!it.valid) return;

    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint64_t *bars = (uint64_t *)(smem + kStages * kStageBytes);
    // bars: [0,S) stage full, [S,2S) stage empty, 2S+{0,1} accumulator full,
    // 2S+{2,3} accumulator empty, 2S+4 drain
    __shared__ uint32_t tmem_base_sh;
    __shared__ int abort_sh;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t bar0 = smem_u32(bars);
    auto full_bar = [&](int s) { return bar0 + 8u * s; };
    auto empty_bar = [&](int s) { return bar0 + 8u * (kStages + s); };
    auto accf_bar = [&](int b) { return bar0 + 8u * (2 * kStages + b); };
    auto acce_bar = [&](int b) { return bar0 + 8u * (2 * kStages + 2 + b); };
    const uint32_t drain_bar = bar0 + 8u * (2 * kStages + 4);

    if (threadIdx.x == 0) {
        asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)&maps.a_hi) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)&maps.a_lo) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)&maps.b_hi) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)&maps.b_lo) : "memory");
        for (int s = 0; s < kStages; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty_bar(s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(accf_bar(b), 1);
            mbar_init(acce_bar(b), 4);  // one arrive per epilogue warp
        }
        mbar_init(drain_bar, 1);
        abort_sh = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(&tmem_base_sh)),
                     "r"(kTmemCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = tmem_base_sh;
    if (threadIdx.x == 0) {
        // The factor operand (A in the band products and the Gram, B in the
        // one-sided update) was written by the preparation kernels long
        // before: warm L2 with its first boxes while the previous kernel
        // finishes (a prefetch is only a hint).
        const CUtensorMap *f_hi = STAGE == 4 ? &maps.b_hi : &maps.a_hi;
        const CUtensorMap *f_lo = STAGE == 4 ? &maps.b_lo : &maps.a_lo;
        const int f_row = (STAGE == 4 ? it.rb : it.ra) * T;
        const int nk_pre = min((it.k1 - it.k0) * (T / KB), 8);
        for (int kb = 0; kb < nk_pre; ++kb) {
            tma_prefetch_2d(f_hi, it.k0 * T + kb * KB, f_row);
            tma_prefetch_2d(f_lo, it.k0 * T + kb * KB, f_row);
        }
    }
    pdl_wait();  // operands and the output tile were written by earlier kernels

    // The contraction runs over nchunk chunks of one tile (T = 128 columns) each.
    // Chunk c accumulates from zero in TMEM buffer c & 1 (columns 128 (c&1) ..);
    // the epilogue warps add every finished chunk into FP32 registers, which
    // keeps the tensor cores' accumulation to 128-long sums.
    constexpr int KB_PER_CHUNK = T / KB;
    const int nchunk = it.k1 - it.k0;
    const int nk = nchunk * KB_PER_CHUNK;
    const int kbase = it.k0 * T;
    const uint64_t deadline = now_ns() + (uint64_t)g.timeout_ms * 1000000ull;

    if (warp == 0 && lane == 0) {
        // ---------------- TMA producer
        int issued = 0;
        for (int kb = 0; kb < (g.test_no_tma ? 0 : nk); ++kb) {
            const int s = kb % kStages;
            if (kb >= kStages && !mbar_wait(empty_bar(s), ((kb / kStages) - 1) & 1, deadline)) {
                record_error(g.st, BAKRON_ERR_DEVICE_TIMEOUT, 1000 + STAGE);
                atomicExch(&abort_sh, 1);
                break;
            }
            if (*(volatile int *)&abort_sh) break;
            const uint32_t base = smem_u32(smem + s * kStageBytes);
            mbar_expect_tx(full_bar(s), kStageBytes);
            const int x = kbase + kb * KB;
            tma_load_2d(base, &maps.a_hi, x, it.ra * T, full_bar(s));
            tma_load_2d(base + kTileBytes, &maps.a_lo, x, it.ra * T, full_bar(s));
            tma_load_2d(base + 2 * kTileBytes, &maps.b_hi, x, it.rb * T, full_bar(s));
            tma_load_2d(base + 3 * kTileBytes, &maps.b_lo, x, it.rb * T, full_bar(s));
            issued = kb + 1;
        }
        pdl_trigger();
        // make sure every issued copy has landed before the CTA can exit
        for (int kb = max(0, issued - kStages); kb < issued; ++kb)
            mbar_wait(full_bar(kb % kStages), (kb / kStages) & 1, deadline + 50000000ull);
    } else if (warp == 1 && lane == 0) {
        // ---------------- MMA issuer
        bool ok = true;
        for (int c = 0; c < nchunk && ok; ++c) {
            const int buf = c & 1;
            if (c >= 2 && !mbar_wait(acce_bar(buf), ((c >> 1) - 1) & 1, deadline)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t tmem_d = tmem_base + (uint32_t)(buf * T);
            for (int kc = 0; kc < KB_PER_CHUNK; ++kc) {
                const int kb = c * KB_PER_CHUNK + kc;
                const int s = kb % kStages;
                if (!mbar_wait(full_bar(s), (kb / kStages) & 1, deadline)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t base = smem_u32(smem + s * kStageBytes);
#pragma unroll
                for (int k8 = 0; k8 < KB / 8; ++k8) {
                    const uint32_t off = k8 * 32;  // 8 tf32 = 32 bytes along K inside the swizzle atom
                    const uint64_t ah = umma_desc(base + off), al = umma_desc(base + kTileBytes + off);
                    const uint64_t bh = umma_desc(base + 2 * kTileBytes + off),
                                   bl = umma_desc(base + 3 * kTileBytes + off);
                    umma_tf32(tmem_d, al, bh, kIdesc, (kc | k8) != 0);
                    umma_tf32(tmem_d, ah, bl, kIdesc, 1);
                    umma_tf32(tmem_d, ah, bh, kIdesc, 1);
                }
                umma_commit(empty_bar(s));
            }
            if (ok) umma_commit(accf_bar(buf));
        }
        if (!ok) {
            record_error(g.st, BAKRON_ERR_DEVICE_TIMEOUT, 2000 + STAGE);
            atomicExch(&abort_sh, 1);
            umma_commit(drain_bar);  // let issued MMAs finish before TMEM is released
            mbar_wait(drain_bar, 0, deadline + 50000000ull);
        }
        pdl_trigger();
    } else if (warp < 2) {
        pdl_trigger();  // idle lanes of the producer and MMA warps
    } else {
        // ---------------- epilogue: per-chunk promotion TMEM -> FP32 registers, then store
        const int quad = warp & 3;  // TMEM lanes [32 quad, 32 quad + 32)
        const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
        float acc[T];
#pragma unroll
        for (int i = 0; i < T; ++i) acc[i] = 0.f;
        bool good = true;
        for (int c = 0; c < nchunk; ++c) {
            const int buf = c & 1;
            int go = 0;
            if (lane == 0) {
                const bool ok = mbar_wait(accf_bar(buf), (c >> 1) & 1, deadline);
                if (!ok) {
                    record_error(g.st, BAKRON_ERR_DEVICE_TIMEOUT, 3000 + STAGE);
                    atomicExch(&abort_sh, 1);
                }
                go = ok && !*(volatile int *)&abort_sh;
            }
            go = __shfl_sync(0xffffffffu, go, 0);  // warp-uniform: tcgen05.ld is .sync.aligned
            if (!go) {
                good = false;
                break;
            }
            tc_fence_after();
#pragma unroll
            for (int c0 = 0; c0 < T; c0 += 32) {
                float v[32];
                tmem_ld32(tmem_base + lane_off + (uint32_t)(buf * T + c0), v);
#pragma unroll
                for (int i = 0; i < 32; ++i) acc[c0 + i] += v[i];
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(acce_bar(buf)) : "memory");
        }
        pdl_trigger();
        // Each epilogue warp stages its 32 rows one column block (32 columns)
        // at a time and hands each 32 x 32 box to TMA at once, so staging and
        // storing overlap.  Row r of a box is 128 bytes whose 16-byte chunk c
        // sits at chunk position c ^ (r & 7) (128-byte swizzle).
        uint8_t *wbuf = smem + quad * (2 * T / 32) * kBoxBytes;  // this warp's boxes
        const int y = it.ra * T + quad * 32;
        const bool store = good && !*(volatile int *)&abort_sh;
#pragma unroll
        for (int cb = 0; cb < T / 32; ++cb) {
            if (store) {
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const int col = cb * 32 + 4 * c;
                    const uint32_t off = (uint32_t)(lane * 128 + ((c ^ (lane & 7)) << 4));
                    if (STAGE == 1) {
                        float4 h, l;
                        split_tf32(acc[col + 0], h.x, l.x);
                        split_tf32(acc[col + 1], h.y, l.y);
                        split_tf32(acc[col + 2], h.z, l.z);
                        split_tf32(acc[col + 3], h.w, l.w);
                        *(float4 *)(wbuf + (2 * cb) * kBoxBytes + off) = h;
                        *(float4 *)(wbuf + (2 * cb + 1) * kBoxBytes + off) = l;
                    } else if (STAGE == 2 || STAGE == 4) {
                        *(float4 *)(wbuf + cb * kBoxBytes + off) =
                            make_float4(-acc[col + 0], -acc[col + 1], -acc[col + 2], -acc[col + 3]);
                    } else {
                        *(float4 *)(wbuf + cb * kBoxBytes + off) =
                            make_float4(acc[col + 0], acc[col + 1], acc[col + 2], acc[col + 3]);
                    }
                }
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            }
            __syncwarp();
            if (store && lane == 0) {
                const int x = it.rb * T + cb * 32;
                if (STAGE == 1) {
                    tma_store_2d(&maps.o0, x, y, smem_u32(wbuf + (2 * cb) * kBoxBytes));
                    tma_store_2d(&maps.o1, x, y, smem_u32(wbuf + (2 * cb + 1) * kBoxBytes));
                } else if (STAGE == 2 || STAGE == 4) {
                    tma_add_2d(&maps.o0, x, y, smem_u32(wbuf + cb * kBoxBytes));
                } else {
                    tma_store_2d(&maps.o0, x, y, smem_u32(wbuf + cb * kBoxBytes));
                }
            }
        }
        if (store && lane == 0) bulk_commit_and_wait_read();
        __syncwarp();
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(kTmemCols));
    }
}

// Self-test of the bounded wait: one thread waits, with the band kernel's own
// helper and deadline, on an mbarrier that no thread ever arrives on; when the
// deadline passes it records BAKRON_ERR_DEVICE_TIMEOUT (where = 9000) and the
// kernel returns, leaving the context usable.
__global__ void wait_timeout_selftest_kernel(DeviceStatus *st, int timeout_ms)
{
    __shared__ __align__(8) uint64_t bar;
    const uint32_t b = smem_u32(&bar);
    if (threadIdx.x == 0) {
        mbar_init(b, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        const uint64_t deadline = now_ns() + (uint64_t)timeout_ms * 1000000ull;
        if (!mbar_wait(b, 0, deadline)) record_error(st, BAKRON_ERR_DEVICE_TIMEOUT, 9000);
    }
}

// ------------------------------------------------------------------ host side
namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode()
{
    static EncodeTiledFn fn = nullptr;
    static bool tried = false;
    if (!tried) {
        tried = true;
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = (EncodeTiledFn)p;
    }
    return fn;
}

// rows x cols fp32 row-major matrix with row stride ld (elements); boxes of
// box_rows rows x 32 columns.
bool make_map(CUtensorMap *map, const float *base, int64_t rows, int64_t cols, int64_t ld, int box_rows = T)
{
    EncodeTiledFn enc = get_encode();
    if (!enc) return false;
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)ld * 4};
    cuuint32_t box[2] = {(cuuint32_t)KB, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, (void *)base, dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

cudaError_t band_tc_configure()
{
    cudaError_t e = cudaFuncSetAttribute(band_tc_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmem);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(band_tc_kernel<3>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmem);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(band_tc_kernel<4>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmem);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(band_tc_kernel<5>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmem);
    if (e != cudaSuccess) return e;
    return cudaFuncSetAttribute(band_tc_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmem);
}

// Gram products: A = B = X^T hi / lo (Dp x Ns, K-major), output G (Dp x Dp).
bool make_gram_maps(const float *xt_hi, const float *xt_lo, float *G, int64_t Dp, int64_t Ns, TcMaps *m)
{
    return make_map(&m->a_hi, xt_hi, Dp, Ns, Ns) && make_map(&m->a_lo, xt_lo, Dp, Ns, Ns) &&
           make_map(&m->b_hi, xt_hi, Dp, Ns, Ns) && make_map(&m->b_lo, xt_lo, Dp, Ns, Ns) &&
           make_map(&m->o0, G, Dp, Dp, Dp, 32) && make_map(&m->o1, G, Dp, Dp, Dp, 32);
}

// One-sided update: A = Delta hi / lo (Mp x Np), B = LtA hi / lo (Np x Np),
// output Wt (Mp x Np, add-reduction of -D).
bool make_gptq_maps(const GemmArgs &g, int64_t Mp, int64_t Np, TcMaps *m)
{
    return make_map(&m->a_hi, g.Ahi, Mp, Np, Np) && make_map(&m->a_lo, g.Alo, Mp, Np, Np) &&
           make_map(&m->b_hi, g.Bhi, Np, Np, Np) && make_map(&m->b_lo, g.Blo, Np, Np, Np) &&
           make_map(&m->o0, g.out_acc, Mp, Np, Np, 32) && make_map(&m->o1, g.out_acc, Mp, Np, Np, 32);
}

cudaError_t launch_gptq_tc(const NodeParams &np, const GemmArgs &g, const TcMaps &maps, cudaStream_t stream)
{
    return launch_pdl(band_tc_kernel<4>, dim3(np.l - np.h, np.Mt), dim3(kThreads), kSmem, stream, maps, np, g);
}

cudaError_t launch_wait_timeout_selftest(DeviceStatus *st, int timeout_ms, cudaStream_t stream)
{
    wait_timeout_selftest_kernel<<<1, 32, 0, stream>>>(st, timeout_ms);
    return cudaGetLastError();
}

cudaError_t launch_band_abort_selftest(DeviceStatus *st, float *buf, int timeout_ms, cudaStream_t stream)
{
    // stage 1 of node (k 0, h 1, l 2) on a 2 x 2 tile grid: two valid items
    // (X^T tiles (0, 0) and (1, 0)), each with one chunk of contraction
    constexpr int64_t n2 = 256;
    float *a_hi = buf, *a_lo = buf + n2 * n2, *b_hi = buf + 2 * n2 * n2, *b_lo = buf + 3 * n2 * n2;
    float *o_hi = buf + 4 * n2 * n2, *o_lo = buf + 5 * n2 * n2;
    GemmArgs g{a_hi, a_lo, b_hi, b_lo, n2, n2, o_hi, o_lo, nullptr, n2, st, timeout_ms, 1};
    TcMaps maps;
    if (!make_tc_maps(1, 2, 2, g, &maps)) return cudaErrorInvalidValue;
    const NodeParams np{0, 1, 2, 2, 2};
    return launch_band_tc(1, np, g, maps, stream);
}

// Full GEMM D (Mo x No) = A (Mo x K) B (No x K)^T, operands as TF32 hi / lo
// parts, K-major with row stride K; D stored with row stride No.  All sizes
// multiples of the tile.
bool make_full_maps(const float *a_hi, const float *a_lo, const float *b_hi, const float *b_lo, float *D, int64_t Mo,
                    int64_t No, int64_t K, TcMaps *m)
{
    return make_map(&m->a_hi, a_hi, Mo, K, K) && make_map(&m->a_lo, a_lo, Mo, K, K) &&
           make_map(&m->b_hi, b_hi, No, K, K) && make_map(&m->b_lo, b_lo, No, K, K) &&
           make_map(&m->o0, D, Mo, No, No, 32) && make_map(&m->o1, D, Mo, No, No, 32);
}

cudaError_t launch_full_tc(int64_t Mo, int64_t No, int64_t K, const GemmArgs &g, const TcMaps &maps,
                           cudaStream_t stream)
{
    const NodeParams np{0, 0, (int)(K / T), (int)(Mo / T), (int)(No / T)};
    return launch_pdl(band_tc_kernel<5>, dim3((unsigned)np.Nt, (unsigned)np.Mt), dim3(kThreads), kSmem, stream, maps,
                      np, g);
}

cudaError_t launch_gram_tc(const NodeParams &np, const GemmArgs &g, const TcMaps &maps, cudaStream_t stream)
{
    return launch_pdl(band_tc_kernel<3>, dim3(np.Mt, np.Mt), dim3(kThreads), kSmem, stream, maps, np, g);
}

bool make_tc_maps(int stage, int Mt, int Nt, const GemmArgs &g, TcMaps *maps)
{
    // stage 1: A = LtA (Np x Np), B = Delta (Mp x Np); stage 2: A = LtB (Mp x Mp),
    // B = X^T (Np x Mp).  In both, an operand's column count equals its row stride.
    const int64_t Mp = (int64_t)Mt * T, Np = (int64_t)Nt * T;
    const int64_t a_rows = stage == 1 ? Np : Mp, b_rows = stage == 1 ? Mp : Np;
    // outputs: stage 1 X^T (Np x Mp), stage 2 Wt (Mp x Np); row stride ldo
    const int64_t o_rows = stage == 1 ? Np : Mp;
    const bool outs = stage == 1 ? make_map(&maps->o0, g.out_hi, o_rows, g.ldo, g.ldo, 32) &&
                                       make_map(&maps->o1, g.out_lo, o_rows, g.ldo, g.ldo, 32)
                                 : make_map(&maps->o0, g.out_acc, o_rows, g.ldo, g.ldo, 32) &&
                                       make_map(&maps->o1, g.out_acc, o_rows, g.ldo, g.ldo, 32);
    return outs && make_map(&maps->a_hi, g.Ahi, a_rows, g.lda, g.lda) &&
           make_map(&maps->a_lo, g.Alo, a_rows, g.lda, g.lda) && make_map(&maps->b_hi, g.Bhi, b_rows, g.ldb, g.ldb) &&
           make_map(&maps->b_lo, g.Blo, b_rows, g.ldb, g.ldb);
}

cudaError_t launch_band_tc(int stage, const NodeParams &np, const GemmArgs &g, const TcMaps &maps,
                           cudaStream_t stream)
{
    // Longest-first order measured faster for nodes up to 40 tile diagonals
    // wide (levels 32 and 16 at 4096^2, 36 and 18 at 14336 x 4096) and slower
    // for the widest, whose row-tile-major order keeps operands in L2.
    NodeParams q = np;
    q.lpt = np.l <= 40;
    const unsigned nx = (unsigned)(stage == 1 ? np.l : np.l - np.h);
    const dim3 grid = q.lpt ? dim3((unsigned)np.Mt, nx) : dim3(nx, (unsigned)np.Mt);
    if (stage == 1) return launch_pdl(band_tc_kernel<1>, grid, dim3(kThreads), kSmem, stream, maps, q, g);
    return launch_pdl(band_tc_kernel<2>, grid, dim3(kThreads), kSmem, stream, maps, q, g);
}

}  // namespace bakron
