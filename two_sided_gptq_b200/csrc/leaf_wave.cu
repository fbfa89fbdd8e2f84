// leaf_wave.cu -- the leaf sweep of one tile diagonal as a continuous strip
// sweep (leaf structure 8): each tile on a cluster of four CTAs, CTA p owning
// row block p (32 rows x 128 columns), every CTA rounding its whole strip in
// one sweep of 159 entry anti-diagonals (Proposition 3.1's updates inside the
// tile; entries of one entry anti-diagonal in parallel, Theorem 3.2).
//
// Lane b of the entry warp walks down column b of sub-tile 0, then column b
// of sub-tile 1, and so on: at step s it rounds entry (a, c) with
// a = (s - b) mod 32, c = b + 32 floor((s - b) / 32), so the sub-tiles of a row
// block follow each other without a phase boundary.  CTA p starts 48 steps
// after CTA p-1, and a tile takes 3 x 48 + 159 dependent steps instead of the
// 7 x 63 of the sub-tile phases.  The sums an entry needs,
//     Wt[a][c] - sum_{(r,c') before (a,c) in the tile} LtB[a][r] D[r][c'] LtA[c][c'],
// are split by where their terms come from:
//   row side   sum_{c' < c} R[a][c'] LtA[c][c']:  the current sub-tile's columns
//              (side warp 1, without the newest c-1), the previous sub-tile's
//              32 columns (side warp 2; both read R and LtA rows from shared
//              memory each step), the older sub-tiles (the product warp,
//              per half sub-tile, subtracted from the staged Wt), and R[a][c-1]
//              (the entry warp, from the lane to its left);
//   column side sum_{r < a} LtB[a][r] D[r][c] over this row block (side warp 3,
//              without the newest a-1, which the entry warp adds from its own
//              previous result), the row block above (side warp 4, from the
//              D values the CTA above pushes into this CTA's shared memory as
//              it rounds them), and the older row blocks (the product warp, per sub-tile,
//              from the other CTAs' shared memory);
// with R[a][c] = (all column-side terms) + D[a][c].  The side warps form step
// s+1's sums during step s; the five sweep warps meet at one named barrier per
// step.  Cross-CTA hand-offs stay off that barrier: a push warp follows the
// sweep's progress, copies the D values of the steps done since its last pass
// into the CTA below and then publishes the progress (one cluster-scope
// release per pass, however many steps it covers) to every CTA below.  The
// waits on progress and on the product warp's flags are bounded by a
// %globaltimer deadline (an expired wait records BAKRON_ERR_DEVICE_TIMEOUT,
// where = 6000 + 10 role + row block, and every later wait returns at once).
#include <cooperative_groups.h>

#include <type_traits>

#include "common.cuh"
#include "kernels.cuh"
#include "leaf_wave.cuh"
#include "leaf_common.cuh"

namespace cg = cooperative_groups;

namespace bakron {

using namespace leafk;

namespace {
constexpr int T = kTile;
constexpr int S3 = 32;
constexpr int kSteps = T + S3 - 1;   // 159 entry anti-diagonals of a 32 x 128 strip
constexpr int kLag = 48;             // steps between the starts of CTA p-1 and CTA p
constexpr int kNeed = 33;            // CTA p's step s needs CTA p-1's steps < s + kNeed
constexpr int kSweep = 160;          // entry and four side warps
constexpr int kThreadsW = 224;       // + the product warp and the push warp
constexpr int RSC = T + 4;           // row stride of sR, sW0, sOS, sLB (32 x 128 blocks)
constexpr int DSC = S3 + 4;          // row stride of sDt, sDab (128 columns x 32 rows)
constexpr int LAS = T + 4;           // row stride of the LtA tile
constexpr int LSC = 3 * S3 + 4;      // row stride of sDr (D of the older row blocks, by column)
constexpr size_t kSmemWaveFloats = (size_t)(S3 + 1) * RSC   // sR
                                   + (size_t)(T + 1) * DSC  // sDt
                                   + (size_t)(S3 + 1) * RSC // sW0
                                   + (size_t)S3 * RSC       // sOS
                                   + (size_t)T * LAS        // sLA
                                   + (size_t)S3 * RSC       // sLB
                                   + (size_t)(T + 1) * DSC  // sDab
                                   + (size_t)S3 * LSC       // sDr
                                   + 4 * 2 * S3             // sums
                                   + 4 * S3                 // row constants
                                   + T;                     // LtA sub-diagonal
constexpr size_t kSmemWave = kSmemWaveFloats * sizeof(float) + (size_t)S3 * T + 32 + 16 * sizeof(int);
static_assert(kSmemWave <= 232448, "wave leaf shared memory");

__device__ __forceinline__ uint64_t wave_now()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
__device__ __forceinline__ int ld_acquire_cluster(const int *p)
{
    int v;
    asm volatile("ld.acquire.cluster.shared::cta.b32 %0, [%1];" : "=r"(v) : "r"((uint32_t)__cvta_generic_to_shared(p))
                 : "memory");
    return v;
}
}  // namespace

__global__ void __cluster_dims__(4, 1, 1) __launch_bounds__(kThreadsW, 1)
leaf_wave_kernel(LeafArgs p, int K, int I_lo)
{
    cg::cluster_group cluster = cg::this_cluster();
    const int pp = (int)cluster.block_rank();  // row block of the tile

    extern __shared__ __align__(16) float smem_f[];
    float *sR = smem_f;                          // (S3+1) x RSC: R (row S3: spare slots)
    float *sDt = sR + (S3 + 1) * RSC;            // (T+1) x DSC: D transposed (column-major), 0 until rounded
    float *sW0 = sDt + (T + 1) * DSC;            // (S3+1) x RSC: staged Wt minus the older terms; then Wt pre-rounding
    float *sOS = sW0 + (S3 + 1) * RSC;           // S3 x RSC: column-side terms of the older row blocks
    float *sLA = sOS + S3 * RSC;                 // T x LAS: the tile's LtA diagonal block
    float *sLB = sLA + T * LAS;                  // S3 x RSC: LtB rows of this row block, columns 0..127
    float *sDab = sLB + S3 * RSC;                // (T+1) x DSC: D of the row block above, pushed by that CTA
    float *sDr = sDab + (T + 1) * DSC;           // S3 x LSC: D of the older row blocks, one sub-tile's columns
    float *sSum = sDr + S3 * LSC;                // 4 x 2 x S3: side sums by entry lane, double-buffered
    float4 *sRowC = (float4 *)(sSum + 4 * 2 * S3);  // S3: {LtB[a][a-1], step, 1/step, 0}
    float *sLAsub = (float *)(sRowC + S3);       // T: LtA[c][c-1]
    int8_t *sCode = (int8_t *)(sLAsub + T);      // S3 x T codes (+32 spare bytes)
    int *sInt = (int *)(sCode + S3 * T + 32);    // [0..3] progress of CTA p' (steps done), [4..11] flags, [12] abort
    int *sProg = sInt, *sFlag = sInt + 4, *sAbort = sInt + 12;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int I = I_lo + (int)(blockIdx.x / 4), J = K - I;
    const int64_t row0 = (int64_t)I * T, col0 = (int64_t)J * T;
    const int64_t brow0 = row0 + pp * S3;
    const int mr = (int)min64(T, p.m - row0), nc = (int)min64(T, p.n - col0);
    const int mrb = max(0, min(S3, mr - pp * S3));
    const float *LAt = p.LA32 + col0 * p.Np + col0;
    const float *LBr = p.LB32 + brow0 * p.Mp + row0;  // LtB rows of this row block, tile columns
    const float fqmin = (float)p.qmin, fqmax = (float)p.qmax;

    // ---- prologue: zero what must start at zero; the factors come from the
    // preparation kernel (complete before this kernel's predecessor passed its
    // own dependency wait), so they load before this kernel's wait
    for (int idx = tid; idx < (S3 + 1) * RSC; idx += kThreadsW) sR[idx] = 0.f;
    for (int idx = tid; idx < (T + 1) * DSC; idx += kThreadsW) sDt[idx] = sDab[idx] = 0.f;
    for (int idx = tid; idx < S3 * RSC; idx += kThreadsW) sOS[idx] = 0.f;
    for (int idx = tid; idx < 4 * 2 * S3; idx += kThreadsW) sSum[idx] = 0.f;
    if (tid < 16) sInt[tid] = 0;
    for (int c = tid; c < T * (T / 4); c += kThreadsW) {
        const int r = c / (T / 4), k4 = c % (T / 4);
        cp_async16(sLA + r * LAS + 4 * k4, LAt + (int64_t)r * p.Np + 4 * k4);
    }
    for (int c = tid; c < S3 * (T / 4); c += kThreadsW) {
        const int r = c / (T / 4), k4 = c % (T / 4);
        cp_async16(sLB + r * RSC + 4 * k4, LBr + (int64_t)r * p.Mp + 4 * k4);
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
    bool out_of_range = false;
    float step_s = 1.f;
    if (tid < S3) {
        step_s = tid < mrb ? p.scales[brow0 + tid] : 1.f;
        out_of_range = !(step_s >= 0x1p-60f && step_s <= 0x1p60f);
    }
    asm volatile("cp.async.wait_all;" ::: "memory");
    const bool exact_div = __syncthreads_or(out_of_range) != 0;
    if (tid < S3) {
        const int r = pp * S3 + tid;  // row within the tile
        sRowC[tid] = make_float4(tid > 0 ? sLB[tid * RSC + r - 1] : 0.f, step_s, __frcp_rn(step_s), 0.f);
    }
    for (int c = tid; c < T; c += kThreadsW) {
        sLAsub[c] = c > 0 ? sLA[c * LAS + c - 1] : 0.f;
        // the row side's sums leave out the newest column (the entry warp's
        // term) and never need the diagonal: both zero in the staged block
        if (c > 0) sLA[c * LAS + c - 1] = 0.f;
        sLA[c * LAS + c] = 0.f;
    }
    // the other CTAs write into this one's shared memory from here on
    cluster.sync();
    pdl_wait();  // Wt comes from the previous kernel
    for (int c = tid; c < S3 * (T / 4); c += kThreadsW) {
        const int r = c / (T / 4), k4 = c % (T / 4);
        cp_async16(sW0 + r * RSC + 4 * k4, p.Wt + (brow0 + r) * p.Np + col0 + 4 * k4);
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
    asm volatile("cp.async.wait_all;" ::: "memory");
    __syncthreads();

    const int role = warp;  // 0 entries, 1 row side (current sub-tile), 2 row side (previous),
                            // 3 column side (this row block), 4 column side (block above), 5 products,
                            // 6 pushes to the CTAs below
    const uint64_t deadline_ns = (uint64_t)p.timeout_ms * 1000000ull;
    // bounded wait until *ctr >= target (acquire at cluster scope); returns
    // the last value read
    auto wait_ge = [&](const int *ctr, int target, int where) {
        int v = ld_acquire_cluster(ctr);
        if (v >= target) return v;
        const uint64_t t_end = wave_now() + deadline_ns;
        while ((v = ld_acquire_cluster(ctr)) < target) {
            if (*(volatile int *)sAbort) return v;
            if (wave_now() > t_end) {
                if (atomicExch(sAbort, 1) == 0) record_error(p.st, BAKRON_ERR_DEVICE_TIMEOUT, where);
                return v;
            }
            __nanosleep(32);
        }
        return v;
    };

    if (role == 6) {
        // ---- push warp (lane = row rho): the D values of steps last .. P-1
        // into the CTA below, then progress P to every CTA below
        const int rho = lane;
        int last = 0;
        while (pp < 3 && last < kSteps) {
            const int P = min(wait_ge(sProg + pp, last + 1, 6060 + pp), kSteps);
            __syncwarp();
            if (P <= last) continue;  // only after an expired wait: the sweep still ends
            float *dst = cluster.map_shared_rank(sDab, pp + 1);
            for (int st = last; st < P; ++st) {
                const int c = st - rho;
                if (c >= 0 && c < T) dst[c * DSC + rho] = sDt[c * DSC + rho];
            }
            asm volatile("fence.acq_rel.cluster;" ::: "memory");
            __syncwarp();
            if (lane < 3 - pp) {
                int *pdst = cluster.map_shared_rank(sProg + pp, pp + 1 + lane);
                asm volatile("st.relaxed.cluster.shared::cluster.b32 [%0], %1;"
                             ::"r"((uint32_t)__cvta_generic_to_shared(pdst)), "r"(P)
                             : "memory");
            }
            last = P;
        }
    } else if (role == 5) {
        // ---- product warp: the older terms, per half sub-tile in the order
        // the entry warp needs them; sW0 -= O_U + O_S, sOS = O_S, then the flag
        const float *sLBs = sLB;  // LtB[p, 0:p-1]: columns 0 .. 32(p-1)-1 of this CTA's rows
        for (int q = 0; q < 4; ++q) {
            if (pp >= 2) {
                // D[0:p-1, q] of the older row blocks (complete at their step 32q + 62)
                for (int pr = 0; pr <= pp - 2; ++pr)
                    wait_ge(sProg + pr, min(32 * q + 63, kSteps), 6050 + pp);
                __syncwarp();
                for (int c = lane; c < (pp - 1) * S3 * 8; c += 32) {
                    const int pr = c / (S3 * 8), j = (c >> 3) % S3, r4 = c & 7;
                    const float *src = cluster.map_shared_rank(sDt, pr) + (q * S3 + j) * DSC + 4 * r4;
                    *(float4 *)(sDr + j * LSC + pr * S3 + 4 * r4) = *(const float4 *)src;
                }
                __syncwarp();
            }
            for (int h = 0; h < 2; ++h) {
                float os[4][4] = {}, ou[4][4] = {};
                if (pp >= 2) mma_block<4>(os, sLBs, RSC, sDr, LSC, S3 * (pp - 1), 16 * h, 0);
                if (q >= 2) {
                    // rows 16h .. 16h+15 have finished sub-tile q-2 (own progress)
                    wait_ge(sProg + pp, 32 * q + 16 * h - 17, 6050 + pp);
                    __syncwarp();
                    mma_block<4>(ou, sR, RSC, sLA + q * S3 * LAS, LAS, S3 * (q - 1), 16 * h, 0);
                }
                if (pp >= 2 || q >= 2) {
                    const int g = lane >> 2, t = lane & 3;
#pragma unroll
                    for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int i = 16 * h + g + 8 * (e >> 1), j = q * S3 + nt * 8 + 2 * t + (e & 1);
                            sOS[i * RSC + j] = os[nt][e];
                            sW0[i * RSC + j] -= ou[nt][e] + os[nt][e];
                        }
                }
                __syncwarp();
                if (lane == 0) {
                    __threadfence_block();
                    *(volatile int *)(sFlag + 2 * q + h) = 1;
                }
            }
        }
    } else if (role == 0) {
        // ---- entry warp
        const int b = lane;
        auto entry = [&](int s, int &a, int &c, bool &live) {
            const int act = s - b;
            live = act >= 0 && act < T;
            const int ac = min(max(act, 0), T - 1);
            a = ac & (S3 - 1);
            c = b + S3 * (ac >> 5);
        };
        auto consts = [&](int s, float &w0, float &os, float4 &rc, float &la) {
            int a, c;
            bool live;
            entry(s, a, c, live);
            w0 = sW0[a * RSC + c];
            os = sOS[a * RSC + c];
            rc = sRowC[a];
            la = sLAsub[c];
        };
        auto sweep = [&](auto ieee_tag) {
            constexpr bool kIeee = decltype(ieee_tag)::value;
            wait_ge(sFlag + 0, 1, 6000 + pp);
            __syncwarp();
            float w0, os, la;
            float4 rc;
            consts(0, w0, os, rc, la);
            float d_prev = 0.f;
            for (int s = -1; s < kSteps; ++s) {
                if (s >= 0) {
                    int a, c;
                    bool live;
                    entry(s, a, c, live);
                    const float *sb = sSum + (s & 1) * S3;
                    const float w1 = sb[b], w2 = sb[2 * S3 + b], w3 = sb[4 * S3 + b], w4 = sb[6 * S3 + b];
                    const float r_left = c > 0 ? sR[a * RSC + c - 1] : 0.f;
                    // the next step's constants, after the product warp's flag
                    // for the half sub-tile the lanes reach first
                    if (((s + 1) & 15) == 0 && s + 1 < T) {
                        wait_ge(sFlag + ((s + 1) >> 4), 1, 6000 + pp);
                        __syncwarp();
                    }
                    float w0n, osn, lan;
                    float4 rcn;
                    consts(s + 1, w0n, osn, rcn, lan);
                    const float cs = fmaf(rc.x, d_prev, w3) + w4;
                    const float wt = w0 - fmaf(la, r_left, w1 + w2) - cs;
                    const float qf = kIeee ? __fdiv_rn(wt, rc.y) : div_rn_recip(wt, rc.y, rc.z);
                    const float cq = fminf(fmaxf(rintf(qf), fqmin), fqmax);
                    const bool valid = live && a < mrb && c < nc;
                    const float dl = valid ? fmaf(-rc.y, cq, wt) : 0.f;
                    // invalid lanes write to spare slots instead of branching
                    const int iR = valid ? a * RSC + c : S3 * RSC + lane;
                    const int iD = valid ? c * DSC + a : T * DSC + lane;
                    const int iC = valid ? a * T + c : S3 * T + lane;
                    sR[iR] = (os + cs) + dl;
                    sDt[iD] = dl;
                    sCode[iC] = code_byte(cq);
                    sW0[iR] = wt;  // pre-rounding value (W0 of this entry is no longer read)
                    d_prev = dl;
                    w0 = w0n; os = osn; rc = rcn; la = lan;
                }
                group_sync(1, kSweep);
            }
        };
        if (exact_div)
            sweep(std::true_type{});
        else
            sweep(std::false_type{});
    } else if (role == 1 || role == 2) {
        // ---- row side (lane = entry lane b): role 1 the current sub-tile's
        // columns, role 2 the previous sub-tile's 32 columns, both rows (R row
        // a and LtA row c) read from shared memory each step.  The staged LtA
        // block holds zeros on its diagonal and sub-diagonal (the newest
        // column c-1 is the entry warp's term, written during this step) and
        // above the diagonal, and R is still zero from column c on, so no
        // lane masks its operands and none branches when it moves on to the
        // next sub-tile; role 1 skips the 4-column groups past c-2
        const int b = lane;
        const int off = role == 1 ? 0 : 1;
        const int lim = role == 1 ? b - 2 : S3 - 1;  // last column of the block with a term
        for (int s = -1; s < kSteps; ++s) {
            const int act = s + 1 - b;
            const bool live = s + 1 < kSteps && act >= 0 && act < T;
            const int ac = min(max(act, 0), T - 1);
            const int a1 = ac & (S3 - 1), q1 = ac >> 5, qb = q1 - off;
            float sum = 0.f;
            if (live && qb >= 0) {
                const float *Rn = sR + a1 * RSC + S3 * qb;
                const float *Ln = sLA + (b + S3 * q1) * LAS + S3 * qb;
                float4 rv[S3 / 4], lv[S3 / 4];
#pragma unroll
                for (int k = 0; k < S3 / 4; ++k) {
                    const bool use = 4 * k <= lim;
                    rv[k] = use ? *(const float4 *)(Rn + 4 * k) : make_float4(0.f, 0.f, 0.f, 0.f);
                    lv[k] = use ? *(const float4 *)(Ln + 4 * k) : make_float4(0.f, 0.f, 0.f, 0.f);
                }
                float2 u0 = make_float2(0.f, 0.f), u1 = make_float2(0.f, 0.f);
                float2 u2 = make_float2(0.f, 0.f), u3 = make_float2(0.f, 0.f);
#pragma unroll
                for (int k = 0; k < S3 / 4; k += 2) {
                    u0 = ffma2(make_float2(rv[k].x, rv[k].y), make_float2(lv[k].x, lv[k].y), u0);
                    u1 = ffma2(make_float2(rv[k].z, rv[k].w), make_float2(lv[k].z, lv[k].w), u1);
                    u2 = ffma2(make_float2(rv[k + 1].x, rv[k + 1].y), make_float2(lv[k + 1].x, lv[k + 1].y), u2);
                    u3 = ffma2(make_float2(rv[k + 1].z, rv[k + 1].w), make_float2(lv[k + 1].z, lv[k + 1].w), u3);
                }
                sum = ((u0.x + u1.x) + (u2.x + u3.x)) + ((u0.y + u1.y) + (u2.y + u3.y));
            }
            sSum[(role == 1 ? 0 : 2 * S3) + ((s + 1) & 1) * S3 + b] = sum;
            group_sync(1, kSweep);
        }
    } else {
        // ---- column side (lane = row rho): role 3 this row block's rows
        // <= rho-2, role 4 the 32 rows of the block above (pushed D columns);
        // the entry of row rho at step s+1 has column c = s + 1 - rho
        const int rho = lane;
        float2 lb[S3 / 2];
        const int base = role == 3 ? pp * S3 : (pp - 1) * S3;
        const int lim = role == 3 ? rho - 2 : S3 - 1;
#pragma unroll
        for (int k = 0; k < S3 / 2; ++k) {
            float2 v = make_float2(0.f, 0.f);
            if (role == 3 || pp > 0) {
                v = *(const float2 *)(sLB + rho * RSC + base + 2 * k);
                v.x = 2 * k + 0 <= lim ? v.x : 0.f;
                v.y = 2 * k + 1 <= lim ? v.y : 0.f;
            }
            lb[k] = v;
        }
        const float *Dsrc = role == 3 ? sDt : sDab;
        int seen = 0;  // role 4: last progress of the CTA above read
        float4 dv[S3 / 4];
#pragma unroll
        for (int k = 0; k < S3 / 4; ++k) dv[k] = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int s = -1; s < kSteps; ++s) {
            if (role == 3 && s >= 0 && lane == 0) {
                // steps < s are done: this CTA's progress, for its product and
                // push warps
                __threadfence_block();
                *(volatile int *)(sProg + pp) = s;
            }
            if (role == 4 && pp > 0 && s + 1 < kSteps) {
                // column c3 of the block above is complete after its step 31 + c3;
                // the first step also waits for the start lag
                const int need = s < 0 ? kLag : min(s + 1 + kNeed, kSteps);
                if (seen < need) seen = wait_ge(sProg + pp - 1, need, 6040 + pp);
                __syncwarp();
            }
            const int c3 = s + 1 - rho;
            const bool live = s + 1 < kSteps && c3 >= 0 && c3 < T && (role == 3 || pp > 0);
            if (live) {
                const float *Dc = Dsrc + c3 * DSC;
#pragma unroll
                for (int k = 0; k < S3 / 4; ++k)
                    if (4 * k <= lim) dv[k] = *(const float4 *)(Dc + 4 * k);
                float2 s0 = make_float2(0.f, 0.f), s1 = make_float2(0.f, 0.f);
                float2 s2 = make_float2(0.f, 0.f), s3 = make_float2(0.f, 0.f);
#pragma unroll
                for (int k = 0; k < S3 / 4; k += 2) {
                    s0 = ffma2(make_float2(dv[k].x, dv[k].y), lb[2 * k], s0);
                    s1 = ffma2(make_float2(dv[k].z, dv[k].w), lb[2 * k + 1], s1);
                    s2 = ffma2(make_float2(dv[k + 1].x, dv[k + 1].y), lb[2 * k + 2], s2);
                    s3 = ffma2(make_float2(dv[k + 1].z, dv[k + 1].w), lb[2 * k + 3], s3);
                }
                sSum[(role == 3 ? 4 * S3 : 6 * S3) + ((s + 1) & 1) * S3 + (c3 & (S3 - 1))] =
                    ((s0.x + s1.x) + (s2.x + s3.x)) + ((s0.y + s1.y) + (s2.y + s3.y));
            }
            group_sync(1, kSweep);
        }
        if (role == 3 && lane == 0) {
            __threadfence_block();
            *(volatile int *)(sProg + pp) = kSteps;
        }
    }
    __syncthreads();
    pdl_trigger();
    for (int idx = tid; idx < S3 * T; idx += kThreadsW) {  // V = s * code, residual split
        const int r = idx / T, c = idx % T;
        if (r >= mrb || c >= nc) continue;
        const int64_t gi = brow0 + r, gj = col0 + c;
        const int8_t code = sCode[r * T + c];
        p.codes[gi * p.n + gj] = code;
        p.V[gi * p.n + gj] = sRowC[r].y * (float)code;
        float hi, lo;
        split_tf32(sDt[c * DSC + r], hi, lo);
        p.Dhi[gi * p.Np + gj] = hi;
        p.Dlo[gi * p.Np + gj] = lo;
        if (p.wt_out) p.wt_out[gi * p.n + gj] = sW0[r * RSC + c];
    }
    // the CTAs below may still read this CTA's D (older-block products)
    cluster.sync();
}

cudaError_t leaf_wave_configure()
{
    return cudaFuncSetAttribute(leaf_wave_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemWave);
}

cudaError_t launch_leaf_wave(const LeafArgs &p, int K, int I_lo, int tiles, cudaStream_t stream)
{
    return launch_pdl(leaf_wave_kernel, dim3(4 * tiles), dim3(kThreadsW), kSmemWave, stream, p, K, I_lo);
}

}  // namespace bakron
