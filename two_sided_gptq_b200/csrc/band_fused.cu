// band_fused.cu -- both band products of a small recursion node in one launch
// (Algorithm 6's postponed update, referee report: "two matrix
// multiplications" per level), on the 5th-generation tensor cores, 3xTF32.
//
// One CTA per target tile (I', J') of node (k, h, l) (target keys
// [k+h, k+l)).  For every source row I of the target (the range stage 2
// contracts over) the CTA forms
//     X^T[J', I] = sum_J LtA[J', J] Delta[I, J]^T     (stage 1, J over the
//                  source tiles of row I at or left of J')
// in tensor memory, splits it into TF32 hi/lo parts in tensor memory, and
// accumulates
//     D^T[J', I'] += sum_i X^T[J', i] LtB[I', i]     (stage 2)
// with X^T as the A operand read straight from tensor memory and LtB rows as
// the B operand from shared memory.  Finally Wt[I', J'] -= D by a TMA
// add-reduction (one writer per Wt tile).  X never leaves the SM, and the
// node costs one launch instead of two; in exchange, X tiles shared by several
// targets are formed by each of them, so the kernel is used for narrow nodes,
// where launch and pipeline latency, not FLOPs, set the time.
//
// Warp roles (320 threads): warp 0 lane 0 issues TMA loads into a 3-slot ring
// (stage-1 slots: LtA hi/lo + Delta hi/lo boxes of 128 rows x 32 fp32;
// stage-2 slots: LtB hi/lo); warp 1 owns the 512 TMEM columns (stage-1
// accumulator, X^T hi, X^T lo, stage-2 accumulator) and lane 0 issues the
// MMAs; warps 2..9 are the epilogue, two per TMEM lane quarter, 64 columns
// each.  Each 128-long chunk of a contraction accumulates from zero in TMEM
// and is added into FP32 registers (per-chunk promotion, as in band_tc.cu).
// Every wait is bounded by a %globaltimer deadline; on expiry the kernel
// records BAKRON_ERR_DEVICE_TIMEOUT, drains what it issued and exits.
#include <cuda.h>

#include "common.cuh"
#include "kernels.cuh"
#include "tcgen05.cuh"

namespace bakron {

using namespace tc;

namespace {
constexpr int T = kTile;
constexpr int KB = 32;                  // fp32 columns per K block (128 bytes)
constexpr int kStages = 3;
constexpr int kPart = T * KB * 4;       // 16 KB: one operand part of a K block
constexpr int kSlot = 4 * kPart;        // 64 KB: a stage-1 K block (stage 2 uses half)
constexpr int kBox = 32 * 32 * 4;       // 4 KB: one 32 x 32 output box
constexpr int kThreads = 320;
constexpr size_t kSmem = (size_t)kStages * kSlot + 1024 /*align*/ + 256 /*barriers*/;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kAcc1 = 0, kXhi = 128, kXlo = 256, kAcc2 = 384;  // TMEM column offsets

// Instruction descriptor: D fp32, A/B tf32, K-major both, N = 128, M = 128.
constexpr uint32_t kIdesc = (1u << 4) | (2u << 7) | (2u << 10) | ((uint32_t)(T >> 3) << 17) |
                            ((uint32_t)(T >> 4) << 24);
}  // namespace

__global__ void __launch_bounds__(kThreads, 1)
band_fused_kernel(const __grid_constant__ TcMaps m1, const __grid_constant__ TcMaps m2, NodeParams np, GemmArgs g)
{
    // target tile and its source rows [I0, I1): the stage-2 item of the node
    const Item it = stage2_item(np, blockIdx.x, blockIdx.y);
    if (!it.valid) return;
    const int Ip = it.ra, Jp = it.rb, I0 = it.k0, I1 = it.k1;
    // source tiles of row I that reach J': [jlo(I), jend(I))
    auto jlo = [&](int I) { return max(0, np.k - I); };
    auto jend = [&](int I) { return min(min(np.Nt, np.k + np.h - I), Jp + 1); };

    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint64_t *bars = (uint64_t *)(smem + kStages * kSlot);
    __shared__ uint32_t tmem_base_sh;
    __shared__ int abort_sh;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t bar0 = smem_u32(bars);
    auto full_bar = [&](int s) { return bar0 + 8u * s; };
    auto empty_bar = [&](int s) { return bar0 + 8u * (kStages + s); };
    const uint32_t acc1_full = bar0 + 8u * (2 * kStages + 0);   // stage-1 chunk in TMEM (commit)
    const uint32_t acc1_empty = bar0 + 8u * (2 * kStages + 1);  // chunk read back (8 epilogue warps)
    const uint32_t x_ready = bar0 + 8u * (2 * kStages + 2);     // X^T hi/lo of a row written (8 warps)
    const uint32_t s2_done = bar0 + 8u * (2 * kStages + 3);     // stage-2 chunk in TMEM, X^T free (commit)
    const uint32_t acc2_empty = bar0 + 8u * (2 * kStages + 4);  // stage-2 chunk read back (8 warps)
    const uint32_t drain_bar = bar0 + 8u * (2 * kStages + 5);

    if (threadIdx.x == 0) {
        asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)&m1.a_hi) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)&m1.a_lo) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)&m1.b_hi) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)&m1.b_lo) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)&m2.a_hi) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)&m2.a_lo) : "memory");
        for (int s = 0; s < kStages; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty_bar(s), 1);
        }
        mbar_init(acc1_full, 1);
        mbar_init(acc1_empty, 8);
        mbar_init(x_ready, 8);
        mbar_init(s2_done, 1);
        mbar_init(acc2_empty, 8);
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
        // The factor rows this tile reads were written by the preparation
        // kernels long before: warm L2 with their first boxes while the
        // previous kernel finishes (a hint only).
        const int j0 = jlo(I0);
        for (int kb = 0; kb < T / KB; ++kb) {
            tma_prefetch_2d(&m1.a_hi, j0 * T + kb * KB, Jp * T);
            tma_prefetch_2d(&m1.a_lo, j0 * T + kb * KB, Jp * T);
            tma_prefetch_2d(&m2.a_hi, I0 * T + kb * KB, Ip * T);
            tma_prefetch_2d(&m2.a_lo, I0 * T + kb * KB, Ip * T);
        }
    }
    pdl_wait();  // Delta and Wt were written by earlier kernels
    const uint64_t deadline = now_ns() + (uint64_t)g.timeout_ms * 1000000ull;

    if (warp == 0 && lane == 0) {
        // ---------------- TMA producer: per source row, its stage-1 K blocks
        // then its stage-2 K blocks, in the order the MMA issuer takes them
        int r = 0;
        bool ok = true;
        auto next_slot = [&](uint32_t bytes) -> int {
            const int s = r % kStages;
            if (r >= kStages && !mbar_wait(empty_bar(s), ((r / kStages) - 1) & 1, deadline)) {
                record_error(g.st, BAKRON_ERR_DEVICE_TIMEOUT, 1005);
                atomicExch(&abort_sh, 1);
                return -1;
            }
            if (*(volatile int *)&abort_sh) return -1;
            mbar_expect_tx(full_bar(s), bytes);
            return s;
        };
        for (int I = I0; I < I1 && ok; ++I) {
            for (int J = jlo(I); J < jend(I) && ok; ++J)
                for (int kb = 0; kb < T / KB; ++kb) {
                    const int s = next_slot(kSlot);
                    if (s < 0) { ok = false; break; }
                    const uint32_t base = smem_u32(smem + s * kSlot);
                    const int x = J * T + kb * KB;
                    tma_load_2d(base, &m1.a_hi, x, Jp * T, full_bar(s));
                    tma_load_2d(base + kPart, &m1.a_lo, x, Jp * T, full_bar(s));
                    tma_load_2d(base + 2 * kPart, &m1.b_hi, x, I * T, full_bar(s));
                    tma_load_2d(base + 3 * kPart, &m1.b_lo, x, I * T, full_bar(s));
                    ++r;
                }
            for (int kb = 0; kb < T / KB && ok; ++kb) {
                const int s = next_slot(2 * kPart);
                if (s < 0) { ok = false; break; }
                const uint32_t base = smem_u32(smem + s * kSlot);
                const int x = I * T + kb * KB;
                tma_load_2d(base, &m2.a_hi, x, Ip * T, full_bar(s));
                tma_load_2d(base + kPart, &m2.a_lo, x, Ip * T, full_bar(s));
                ++r;
            }
        }
        pdl_trigger();
        // every issued copy lands before the CTA can exit
        for (int q = max(0, r - kStages); q < r; ++q)
            mbar_wait(full_bar(q % kStages), (q / kStages) & 1, deadline + 50000000ull);
    } else if (warp == 1 && lane == 0) {
        // ---------------- MMA issuer
        int r = 0, c1 = 0, ii = 0;
        bool ok = true;
        const uint32_t acc1 = tmem_base + kAcc1, acc2 = tmem_base + kAcc2;
        const uint32_t xhi = tmem_base + kXhi, xlo = tmem_base + kXlo;
        for (int I = I0; I < I1 && ok; ++I, ++ii) {
            const int nj = jend(I) - jlo(I);
            for (int jc = 0; jc < nj && ok; ++jc) {
                if (c1 > 0 && !mbar_wait(acc1_empty, (c1 - 1) & 1, deadline)) { ok = false; break; }
                tc_fence_after();
                for (int kb = 0; kb < T / KB; ++kb) {
                    const int s = r % kStages;
                    if (!mbar_wait(full_bar(s), (r / kStages) & 1, deadline)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t base = smem_u32(smem + s * kSlot);
#pragma unroll
                    for (int k8 = 0; k8 < KB / 8; ++k8) {
                        const uint32_t off = k8 * 32;  // 8 tf32 = 32 bytes along K inside the swizzle atom
                        const uint64_t ah = umma_desc(base + off), al = umma_desc(base + kPart + off);
                        const uint64_t bh = umma_desc(base + 2 * kPart + off), bl = umma_desc(base + 3 * kPart + off);
                        umma_tf32(acc1, al, bh, kIdesc, (kb | k8) != 0);
                        umma_tf32(acc1, ah, bl, kIdesc, 1);
                        umma_tf32(acc1, ah, bh, kIdesc, 1);
                    }
                    umma_commit(empty_bar(s));
                    ++r;
                }
                if (!ok) break;
                umma_commit(acc1_full);
                ++c1;
            }
            if (!ok) break;
            // stage 2 of source row I: X^T (TMEM, hi/lo) against LtB[I', I] rows
            if (!mbar_wait(x_ready, ii & 1, deadline)) { ok = false; break; }
            if (ii > 0 && !mbar_wait(acc2_empty, (ii - 1) & 1, deadline)) { ok = false; break; }
            tc_fence_after();
            for (int kb = 0; kb < T / KB; ++kb) {
                const int s = r % kStages;
                if (!mbar_wait(full_bar(s), (r / kStages) & 1, deadline)) { ok = false; break; }
                tc_fence_after();
                const uint32_t base = smem_u32(smem + s * kSlot);
#pragma unroll
                for (int k8 = 0; k8 < KB / 8; ++k8) {
                    const uint32_t off = k8 * 32;
                    const uint32_t col = (uint32_t)(kb * KB + k8 * 8);  // K = i: eight TMEM columns per MMA
                    const uint64_t bh = umma_desc(base + off), bl = umma_desc(base + kPart + off);
                    umma_tf32_ts(acc2, xlo + col, bh, kIdesc, (kb | k8) != 0);
                    umma_tf32_ts(acc2, xhi + col, bl, kIdesc, 1);
                    umma_tf32_ts(acc2, xhi + col, bh, kIdesc, 1);
                }
                umma_commit(empty_bar(s));
                ++r;
            }
            if (ok) umma_commit(s2_done);
        }
        if (!ok) {
            record_error(g.st, BAKRON_ERR_DEVICE_TIMEOUT, 2005);
            atomicExch(&abort_sh, 1);
            umma_commit(drain_bar);  // let issued MMAs finish before TMEM is released
            mbar_wait(drain_bar, 0, deadline + 50000000ull);
        }
        pdl_trigger();
    } else if (warp < 2) {
        pdl_trigger();  // idle lanes of the producer and MMA warps
    } else {
        // ---------------- epilogue: warps 2..9, TMEM lane quarter warp % 4,
        // columns [64 hf, 64 hf + 64) of every 128-column region
        const int quad = warp & 3, hf = (warp - 2) >> 2;
        const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
        const uint32_t my = tmem_base + lane_off + (uint32_t)(hf * 64);
        float xacc[64], dacc[64];
#pragma unroll
        for (int i = 0; i < 64; ++i) dacc[i] = 0.f;
        bool good = true;
        // warp-uniform bounded wait on `bar` (lane 0 polls)
        auto wait_all = [&](uint32_t bar, uint32_t parity) -> bool {
            int go = 0;
            if (lane == 0) {
                const bool ok = mbar_wait(bar, parity, deadline);
                if (!ok) {
                    record_error(g.st, BAKRON_ERR_DEVICE_TIMEOUT, 3005);
                    atomicExch(&abort_sh, 1);
                }
                go = ok && !*(volatile int *)&abort_sh;
            }
            return __shfl_sync(0xffffffffu, go, 0) != 0;  // tcgen05.ld/st are .sync.aligned
        };
        auto arrive = [&](uint32_t bar) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
        };
        int c1 = 0, ii = 0;
        for (int I = I0; I < I1 && good; ++I, ++ii) {
#pragma unroll
            for (int i = 0; i < 64; ++i) xacc[i] = 0.f;
            const int nj = jend(I) - jlo(I);
            for (int jc = 0; jc < nj; ++jc, ++c1) {
                if (!wait_all(acc1_full, c1 & 1)) { good = false; break; }
                tc_fence_after();
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    float v[32];
                    tmem_ld32(my + kAcc1 + hh * 32, v);
#pragma unroll
                    for (int i = 0; i < 32; ++i) xacc[hh * 32 + i] += v[i];
                }
                arrive(acc1_empty);
            }
            if (!good) break;
            if (ii > 0) {  // the previous row's stage 2 is complete: its sum, and X^T is free
                if (!wait_all(s2_done, (ii - 1) & 1)) { good = false; break; }
                tc_fence_after();
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    float v[32];
                    tmem_ld32(my + kAcc2 + hh * 32, v);
#pragma unroll
                    for (int i = 0; i < 32; ++i) dacc[hh * 32 + i] += v[i];
                }
                arrive(acc2_empty);
            }
            // this lane's row j' of X^T into TMEM as TF32 hi and lo parts
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                float hi[32], lo[32];
#pragma unroll
                for (int i = 0; i < 32; ++i) split_tf32(xacc[hh * 32 + i], hi[i], lo[i]);
                tmem_st32(my + kXhi + hh * 32, hi);
                tmem_st32(my + kXlo + hh * 32, lo);
            }
            tmem_st_wait();
            arrive(x_ready);
        }
        if (good && wait_all(s2_done, (ii - 1) & 1)) {
            tc_fence_after();
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                float v[32];
                tmem_ld32(my + kAcc2 + hh * 32, v);
#pragma unroll
                for (int i = 0; i < 32; ++i) dacc[hh * 32 + i] += v[i];
            }
        } else {
            good = false;
        }
        pdl_trigger();
        // dacc holds D^T[j'][i'] for j' = 32 quad + lane and i' in [64 hf, 64 hf + 64).
        // Every MMA has completed (the last stage-2 commit covers all of them)
        // and every copy has been consumed, so the ring is free for staging.
        // Box b (rows i' in [64 hf + 32 b, +32), columns j' in [32 quad, +32)):
        // row r is 128 bytes whose 16-byte chunk c sits at chunk position
        // c ^ (r & 7) (128-byte swizzle); lane = column.
        uint8_t *wbuf = smem + (warp - 2) * 2 * kBox;
        const bool store = good && !*(volatile int *)&abort_sh;
#pragma unroll
        for (int b = 0; b < 2; ++b) {
            if (store) {
#pragma unroll
                for (int r = 0; r < 32; ++r) {
                    const uint32_t off = (uint32_t)(r * 128 + (((lane >> 2) ^ (r & 7)) << 4) + (lane & 3) * 4);
                    *(float *)(wbuf + b * kBox + off) = -dacc[b * 32 + r];
                }
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            }
            __syncwarp();
            if (store && lane == 0)
                tma_add_2d(&m2.o0, Jp * T + quad * 32, Ip * T + hf * 64 + b * 32, smem_u32(wbuf + b * kBox));
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

cudaError_t band_fused_configure()
{
    return cudaFuncSetAttribute(band_fused_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmem);
}

cudaError_t launch_band_fused(const NodeParams &np, const GemmArgs &g, const TcMaps &m1, const TcMaps &m2,
                              cudaStream_t stream)
{
    return launch_pdl(band_fused_kernel, dim3(np.l - np.h, np.Mt), dim3(kThreads), kSmem, stream, m1, m2, np, g);
}

}  // namespace bakron
