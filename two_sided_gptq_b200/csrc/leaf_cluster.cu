// leaf_cluster.cu -- the leaf sweep of one tile diagonal with each tile on a
// cluster of four CTAs (Proposition 3.1's updates inside the tile, entries of
// one entry anti-diagonal rounded in parallel: Theorem 3.2).
//
// The warp variant (leaf.cu) keeps a whole 128 x 128 tile in one CTA, cut into
// 4 x 4 sub-tiles of 32 processed in sub-tile-diagonal phases; in the middle
// phases up to four sub-tile sweeps share one SM's issue slots and
// shared-memory bandwidth, and each dependent step gets slower.  Here CTA p of
// a four-CTA cluster owns row block p of the tile: its R rows, its columns of
// D, its sub-tiles (p, q), q = 0..3, swept in phase e = p + q by its three
// warps exactly as the warp variant sweeps one sub-tile:
//     S[p,q]  = sum_{p'<p} LtB[p,p'] D[p',q],
//     W0[p,q] = Wt[p,q] - sum_{q'<q} R[p,q'] LtA[q,q']^T - S[p,q],
// then 63 entry anti-diagonal steps (entry warp, row-side warp, column-side
// warp; one 96-thread barrier per step).  The only data that crosses CTAs is
// D[p',q] of the row blocks above, which the S product reads from their
// shared memory (distributed shared memory) after the cluster barrier that
// opens each phase; R and everything else stays local.  Every CTA passes the
// same eight cluster barriers, so the waits are those of a hardware barrier
// with equal trip counts.
//
// Overlapped form (kOverlap, structure 6): of the two products only the
// newest 32-deep terms, LtB[p,p-1] D[p-1,q] and R[p,q-1] LtA[q,q-1]^T, depend
// on the phase just finished.  A fourth warp per CTA forms the older terms
// of the CTA's next sub-tile,
//     O_S = sum_{p' <= p-2} LtB[p,p'] D[p',q+1],
//     O_U = sum_{q' <= q-1} R[p,q'] LtA[q+1,q']^T,
// while the three sweep warps round the current one (it also stages the next
// sub-tile's Wt block and LtA strip and fetches the older D blocks from the
// other CTAs), so between two sweeps only the newest terms remain, shared by
// all four warps.
//
// Two tile diagonals per launch (kPair, structure 7): clusters take tickets
// from a counter in the order they start; the first tickets take the tiles of
// diagonal K, the rest those of K + 1, so a cluster only ever waits for
// clusters that are already running.  A diagonal-K tile runs as above, then
// exports its in-tile R (rows of its CTAs) and raises its flag (one increment
// per CTA, after a device-scope fence).  A diagonal-(K+1) tile (I', J') waits,
// bounded by a %globaltimer deadline, for the flags of its neighbours on K --
// left (I', J'-1) and upper (I'-1, J') -- and then applies their share of
// Proposition 3.1's updates itself, which for a width-2 node takes two plain
// products instead of two chained ones:
//     left:  sum_{r<=a, c} LtB[a,r] D_rc LtA[b,c] = (R_left LtA[J',J'-1]^T)[a,b],
//            R_left the left tile's in-tile R, subtracted from Wt;
//     upper: sum_{r, c<=b} LtB[a,r] D_rc LtA[b,c] = sum_{c<=b} S_up[a,c] LtA[b,c],
//            S_up = LtB[I',I'-1] D_up, which enters the sweep's pull form
//            exactly like the in-tile S (added into S before each sub-tile).
// Both products run in FP32 on the CUDA cores of the tile's four CTAs (each
// its own 32 rows) before the first phase.
#include <cooperative_groups.h>

#include <type_traits>

#include "common.cuh"
#include "kernels.cuh"
#include "leaf_common.cuh"

namespace cg = cooperative_groups;

namespace bakron {

using namespace leafk;

namespace {
constexpr int T = kTile;
constexpr int S3 = 32;            // sub-tile side
constexpr int kSweepThreads = 96;  // entry, row-side and column-side warps
constexpr int RSC = T + 4;        // row stride of sR (32 rows x 128 columns)
constexpr int DSC = S3 + 4;       // row stride of sDt (128 columns x 32 rows)
constexpr int WSC = S3 + 4;       // row stride of the sub-tile slot
constexpr int LSC = 3 * S3 + 4;   // row stride of strips of up to three 32-wide blocks
constexpr size_t kSmemC = ((size_t)(S3 + 1) * RSC + (size_t)(T + 1) * DSC + (size_t)3 * S3 * WSC +
                           (size_t)3 * S3 * LSC + 3 * S3 + 4 * S3) * sizeof(float) +
                          (size_t)S3 * T + 32;
// Requested per CTA so that two CTAs never share an SM: the point of the
// variant is one sub-tile sweep per SM.
constexpr size_t kSmemCLaunch = 120 * 1024;
static_assert(kSmemC <= kSmemCLaunch && 2 * kSmemCLaunch > 228 * 1024, "cluster leaf shared memory");
// pair form: S_up rows (S3 x SUPS) and one staging chunk of the neighbour
// products (R_left 32 x 32, LtA 128 x 32, LtB 32 x 32, D_up 32 x 128)
constexpr int SUPS = T + 4;
constexpr int CKS = 36;  // row stride of the staged 32-wide chunks
constexpr size_t kSmemPairExtra = ((size_t)S3 * SUPS + 2 * S3 * CKS + (size_t)T * CKS + (size_t)S3 * T) * sizeof(float);
constexpr size_t kSmemPairLaunch = align_up(kSmemC, 16) + kSmemPairExtra;
static_assert(kSmemPairLaunch <= 232448, "pair leaf shared memory");

// Bounded wait for a device-scope counter to reach `target`; false if the
// deadline passed first.
__device__ __forceinline__ bool wait_counter(const int32_t *ctr, int target, uint64_t deadline)
{
    for (;;) {
        int v;
        asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(ctr) : "memory");
        if (v >= target) return true;
        uint64_t t;
        asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
        if (t > deadline) return false;
        __nanosleep(64);
    }
}
}  // namespace

template <bool kOverlap, bool kPair>
__global__ void __cluster_dims__(4, 1, 1) __launch_bounds__(kOverlap ? 128 : 96, 1)
leaf_cluster_kernel(LeafArgs p, int K, int I_lo, int slot)
{
    constexpr int kThreadsC = kOverlap ? 128 : 96;
    cg::cluster_group cluster = cg::this_cluster();
    const int pp = (int)cluster.block_rank();  // row block of sub-tiles

    extern __shared__ __align__(16) float smem_f[];
    float *sR = smem_f;                       // (S3+1) x RSC: R of this row block (S before a sweep, Wt staged)
    float *sDt = sR + (S3 + 1) * RSC;         // (T+1) x DSC: D transposed, this row block's rows, 0 until rounded
    float *sW = sDt + (T + 1) * DSC;          // S3 x WSC: S, then W0 of the sub-tile being swept
    float *sOS = sW + S3 * WSC;               // S3 x WSC: older column-side terms O_S of the next sub-tile
    float *sOU = sOS + S3 * WSC;              // S3 x WSC: older row-side terms O_U of the next sub-tile
    float *sLA = sOU + S3 * WSC;              // LtA[q, 0:q] strip, row stride 32 q + 4 (staged a phase ahead)
    float *sLBs = sLA + S3 * LSC;             // LtB[p, 0:p] strip, row stride 32 p + 4 (loaded once)
    float *sDr = sLBs + S3 * LSC;             // D[0:p, q] of the row blocks above: [column][32 p' + row], LSC
    float *sLBd = sDr + S3 * LSC;             // S3: LtB[r][r-1] inside the row block (0 for r = 0)
    float *scale = sLBd + S3;                 // S3
    float *rcp = scale + S3;                  // S3
    float *sPS = rcp + S3;                    // 2 x S3: column-side partial sums by column
    float *sPU = sPS + 2 * S3;                // 2 x S3: row-side partial sums by column
    int8_t *sCode = (int8_t *)(sPU + 2 * S3); // S3 x T codes (+32 spare bytes)
    // pair form: S_up rows of this row block, then the staging chunk
    float *sSup = (float *)((uint8_t *)smem_f + align_up(kSmemC, 16));  // S3 x SUPS
    float *cR = sSup + S3 * SUPS;             // S3 x CKS: R_left rows, 32-wide chunk
    float *cB = cR + S3 * CKS;                // S3 x CKS: LtB[I', I'-1] rows, chunk
    float *cA = cB + S3 * CKS;                // T x CKS: LtA[J', J'-1] rows, chunk
    float *cD = cA + T * CKS;                 // S3 x T: D_up rows of the chunk

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // the cluster's tile: by launch position, or (pair form) by ticket
    int Kd = K, I = I_lo + (int)(blockIdx.x / 4);
    bool consumer = false;  // pair form: a tile of the second diagonal
    if (kPair) {
        __shared__ int ticket_sh;
        pdl_wait();  // the ticket counter was cleared before this solve's first kernel
        if (pp == 0 && tid == 0) ticket_sh = atomicAdd(&p.tickets[slot], 1);
        cluster.sync();
        const int tk = *cluster.map_shared_rank(&ticket_sh, 0);
        const int lo0 = max(0, K - (p.Nt - 1)), n0 = min(p.Mt - 1, K) - lo0 + 1;
        const int lo1 = max(0, K + 1 - (p.Nt - 1));
        consumer = tk >= n0;
        Kd = consumer ? K + 1 : K;
        I = consumer ? lo1 + (tk - n0) : lo0 + tk;
    }
    const int J = Kd - I;
    const int64_t row0 = (int64_t)I * T, col0 = (int64_t)J * T;
    const int64_t brow0 = row0 + pp * S3;  // first row of this row block
    const int mr = (int)min64(T, p.m - row0), nc = (int)min64(T, p.n - col0);
    const int mrb = max(0, min(S3, mr - pp * S3));  // rows of this row block inside the matrix
    const float *LAt = p.LA32 + col0 * p.Np + col0;  // LtA diagonal block of the tile (global)
    const float *LBt = p.LB32 + row0 * p.Mp + row0;  // LtB diagonal block of the tile (global)
    const int lda_g = (int)p.Np, ldb_g = (int)p.Mp;
    // Warm L2 with the factor rows this CTA reads (a hint; it may precede the
    // dependency wait): all of the LtA diagonal block, this row block's LtB rows.
    for (int idx = tid; idx < (T + S3) * (T / 32); idx += kThreadsC) {
        const int r = idx / (T / 32), seg = idx % (T / 32);
        const float *ptr = r < T ? LAt + r * lda_g + 32 * seg : LBt + (pp * S3 + r - T) * ldb_g + 32 * seg;
        asm volatile("prefetch.global.L2 [%0];" ::"l"(ptr));
    }
    for (int idx = tid; idx < (S3 + 1) * RSC / 4; idx += kThreadsC)
        ((float4 *)sR)[idx] = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int idx = tid; idx < (T + 1) * DSC / 4; idx += kThreadsC)
        ((float4 *)sDt)[idx] = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int idx = tid; idx < 2 * S3 * WSC / 4; idx += kThreadsC)  // O_S, O_U
        ((float4 *)sOS)[idx] = make_float4(0.f, 0.f, 0.f, 0.f);
    // The factors and the steps come from the preparation kernel at the start
    // of the solve, which has completed before this kernel's predecessor
    // passed its own dependency wait: they are read before this kernel's
    // wait, overlapping the predecessor's tail.  Only Wt (and the pair form's
    // neighbour data) depend on the predecessor.
    if (pp > 0) {  // LtB[p, 0:p], fixed for the kernel
        const int ld = S3 * pp + 4, c4 = 8 * pp;
        for (int c = tid; c < S3 * c4; c += kThreadsC) {
            const int i = c / c4, k4 = c - i * c4;
            cp_async16(sLBs + i * ld + 4 * k4, LBt + (pp * S3 + i) * ldb_g + 4 * k4);
        }
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
    if (tid < S3) sLBd[tid] = tid > 0 ? LBt[(pp * S3 + tid) * ldb_g + pp * S3 + tid - 1] : 0.f;
    const float fqmin = (float)p.qmin, fqmax = (float)p.qmax;
    const int role = warp;  // 0 entries, 1 row side, 2 column side, 3 (overlapped form) older products
    // column-side warp: its LtB[p,p] row rho (columns <= rho-2), fixed for the kernel
    float2 lbr[S3 / 2];
    if (role == 2) {
#pragma unroll
        for (int c = 0; c < S3 / 2; ++c) {
            float2 v = *(const float2 *)(LBt + (pp * S3 + lane) * ldb_g + pp * S3 + 2 * c);
            v.x = 2 * c + 0 <= lane - 2 ? v.x : 0.f;
            v.y = 2 * c + 1 <= lane - 2 ? v.y : 0.f;
            lbr[c] = v;
        }
    }
    // Steps of this row block and their correctly rounded reciprocals; a step
    // outside [2^-60, 2^60] switches the row block to the IEEE division (both
    // give the correctly rounded quotient, so the choice never shows).
    bool out_of_range = false;
    if (tid < S3) {
        const float s = tid < mrb ? p.scales[brow0 + tid] : 1.f;
        scale[tid] = s;
        rcp[tid] = __frcp_rn(s);
        out_of_range = !(s >= 0x1p-60f && s <= 0x1p60f);
    }
    // (this barrier also orders the zeroing above before the first staged block)
    const bool exact_div = __syncthreads_or(out_of_range) != 0;

    // row-side warp: LtA[q,q] row b (used for columns <= b-2, masked when its
    // sweep starts, so no instruction waits for these loads before then);
    // entry warp: LtA[b][b-1].  Loaded for the CTA's next sub-tile as soon as
    // the previous sweep ends, so the L2 latency overlaps the phase change.
    float2 la[S3 / 2];
    float la_new = 0.f;
    auto load_la = [&](int q) {
        if (q < 0 || q > 3) return;
        if (role == 1) {
#pragma unroll
            for (int c = 0; c < S3 / 2; ++c) la[c] = *(const float2 *)(LAt + (q * S3 + lane) * lda_g + q * S3 + 2 * c);
        }
        if (role == 0 && lane > 0) la_new = LAt[(q * S3 + lane) * lda_g + q * S3 + lane - 1];
    };
    load_la(0 - pp);
    pdl_wait();  // Wt comes from the previous kernel
    const bool has_left = kPair && consumer && J >= 1;  // neighbours on the first diagonal
    const bool has_up = kPair && consumer && I >= 1;
    if (kPair && consumer) {
        // wait for the neighbours' outputs (bounded), then their share of the
        // updates: P = R_left LtA[J',J'-1]^T off Wt, S_up = LtB[I',I'-1] D_up
        if (tid == 0) {
            const uint64_t deadline = [] { uint64_t t; asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t)); return t; }() +
                                      (uint64_t)p.timeout_ms * 1000000ull;
            bool ok = true;
            if (has_left) ok = wait_counter(p.flags + (int64_t)I * p.Nt + (J - 1), 4, deadline);
            if (ok && has_up) ok = wait_counter(p.flags + (int64_t)(I - 1) * p.Nt + J, 4, deadline);
            if (!ok) record_error(p.st, BAKRON_ERR_DEVICE_TIMEOUT, 4000 + pp);
            __threadfence();
        }
        __syncthreads();
        // thread t: column j = t of P and S_up, rows a of this row block in pairs
        float2 pa[S3 / 2], sa[S3 / 2];
#pragma unroll
        for (int i = 0; i < S3 / 2; ++i) pa[i] = sa[i] = make_float2(0.f, 0.f);
        const int jj = tid;  // 128 threads = 128 columns
        for (int kc = 0; kc < T / 32; ++kc) {
            // stage the chunk of 32 contraction indices (L2-coherent loads)
            const int64_t kx = (int64_t)kc * 32;
            if (has_left) {
                for (int c = tid; c < S3 * 8; c += kThreadsC) {
                    const int r = c >> 3, k4 = c & 7;
                    *(float4 *)(cR + r * CKS + 4 * k4) =
                        __ldcg((const float4 *)(p.Rx + (brow0 + r) * p.Np + (col0 - T) + kx + 4 * k4));
                }
                for (int c = tid; c < T * 8; c += kThreadsC) {
                    const int r = c >> 3, k4 = c & 7;
                    *(float4 *)(cA + r * CKS + 4 * k4) =
                        *(const float4 *)(p.LA32 + (col0 + r) * p.Np + (col0 - T) + kx + 4 * k4);
                }
            }
            if (has_up) {
                for (int c = tid; c < S3 * 8; c += kThreadsC) {
                    const int r = c >> 3, k4 = c & 7;
                    *(float4 *)(cB + r * CKS + 4 * k4) =
                        *(const float4 *)(p.LB32 + (brow0 + r) * p.Mp + (row0 - T) + kx + 4 * k4);
                }
                for (int r = 0; r < S3; ++r) {
                    const int64_t g = (row0 - T + kx + r) * p.Np + col0 + jj;
                    cD[r * T + jj] = __ldcg(p.Dhi + g) + __ldcg(p.Dlo + g);
                }
            }
            __syncthreads();
#pragma unroll 2
            for (int k = 0; k < 32; k += 4) {
                if (has_left) {
                    const float4 la4 = *(const float4 *)(cA + jj * CKS + k);
#pragma unroll
                    for (int i = 0; i < S3 / 2; ++i) {
                        const float4 r0 = *(const float4 *)(cR + (2 * i) * CKS + k);
                        const float4 r1 = *(const float4 *)(cR + (2 * i + 1) * CKS + k);
                        pa[i] = ffma2(make_float2(r0.x, r1.x), make_float2(la4.x, la4.x), pa[i]);
                        pa[i] = ffma2(make_float2(r0.y, r1.y), make_float2(la4.y, la4.y), pa[i]);
                        pa[i] = ffma2(make_float2(r0.z, r1.z), make_float2(la4.z, la4.z), pa[i]);
                        pa[i] = ffma2(make_float2(r0.w, r1.w), make_float2(la4.w, la4.w), pa[i]);
                    }
                }
                if (has_up) {
                    const float d0 = cD[(k + 0) * T + jj], d1 = cD[(k + 1) * T + jj];
                    const float d2 = cD[(k + 2) * T + jj], d3 = cD[(k + 3) * T + jj];
#pragma unroll
                    for (int i = 0; i < S3 / 2; ++i) {
                        const float4 b0 = *(const float4 *)(cB + (2 * i) * CKS + k);
                        const float4 b1 = *(const float4 *)(cB + (2 * i + 1) * CKS + k);
                        sa[i] = ffma2(make_float2(b0.x, b1.x), make_float2(d0, d0), sa[i]);
                        sa[i] = ffma2(make_float2(b0.y, b1.y), make_float2(d1, d1), sa[i]);
                        sa[i] = ffma2(make_float2(b0.z, b1.z), make_float2(d2, d2), sa[i]);
                        sa[i] = ffma2(make_float2(b0.w, b1.w), make_float2(d3, d3), sa[i]);
                    }
                }
            }
            __syncthreads();  // the chunk buffers are refilled next
        }
        // Wt rows of this row block lose P (no other CTA reads them until this
        // CTA stages them below); S_up waits in shared memory for the sweeps
#pragma unroll
        for (int i = 0; i < S3 / 2; ++i) {
            if (has_left) {
                float *w0 = p.Wt + (brow0 + 2 * i) * p.Np + col0 + jj;
                w0[0] -= pa[i].x;
                w0[p.Np] -= pa[i].y;
            }
            sSup[(2 * i) * SUPS + jj] = sa[i].x;
            sSup[(2 * i + 1) * SUPS + jj] = sa[i].y;
        }
        __syncthreads();
    }

    // Stage the sub-tile (pp, q) -- its Wt block into R's block (untouched
    // until then) and the strip LtA[q, 0:q] -- with threads [t0, t0 + nt).
    auto stage_subtile = [&](int q, int t0, int nt) {
        if (q < 0 || q > 3) return;
        if (q > 0) {
            const int ld = S3 * q + 4, c4 = 8 * q;
            for (int c = tid - t0; c < S3 * c4; c += nt) {
                const int j = c / c4, k4 = c - j * c4;
                cp_async16(sLA + j * ld + 4 * k4, LAt + (q * S3 + j) * lda_g + 4 * k4);
            }
        }
        for (int c = tid - t0; c < S3 * 8; c += nt) {
            const int i = c >> 3, k4 = c & 7;
            cp_async16(sR + i * RSC + q * S3 + 4 * k4, p.Wt + (brow0 + i) * p.Np + col0 + q * S3 + 4 * k4);
        }
    };
    // D[p', q] of CTA p' (rows of row block p') into sDr, transposed, for
    // p' in [p0, p1), with threads [t0, t0 + nt)
    auto gather_d = [&](int q, int p0, int p1, int t0, int nt) {
        for (int c = tid - t0; c < (p1 - p0) * S3 * 8; c += nt) {
            const int pr = p0 + c / (S3 * 8), j = (c >> 3) % S3, r4 = c & 7;
            const float *src = cluster.map_shared_rank(sDt, pr) + (q * S3 + j) * DSC + 4 * r4;
            *(float4 *)(sDr + j * LSC + pr * S3 + 4 * r4) = *(const float4 *)src;
        }
    };
    // V = s * code and the residual's TF32 split for columns [c0, c1) of this
    // row block, with threads [t0, t0 + nt)
    auto write_out = [&](int c0, int c1, int t0, int nt) {
        const int w = c1 - c0;
        for (int idx = tid - t0; idx < S3 * w; idx += nt) {
            const int r = idx / w, c = c0 + idx % w;
            if (r >= mrb || c >= nc) continue;
            const int64_t gi = brow0 + r, gj = col0 + c;
            const int8_t code = sCode[r * T + c];
            p.codes[gi * p.n + gj] = code;
            p.V[gi * p.n + gj] = scale[r] * (float)code;
            float hi, lo;
            split_tf32(sDt[c * DSC + r], hi, lo);
            p.Dhi[gi * p.Np + gj] = hi;
            p.Dlo[gi * p.Np + gj] = lo;
        }
    };
    stage_subtile(0 - pp, 0, kThreadsC);

    for (int e = 0; e < 7; ++e) {
        const int q = e - pp;
        const bool mine = q >= 0 && q <= 3;
        // Every CTA of the cluster has finished phase e - 1, so the D blocks
        // it rounded are final and visible (release / acquire at cluster scope).
        // Overlapped form: the barrier is split; between arriving and waiting
        // the CTA forms the newest row-side term R[p,q-1] LtA[q,q-1]^T, which
        // needs only its own R (final since the last CTA barrier) and the LtA
        // strip the product warp staged and waited for.
        float au[2][4] = {};
        if (kOverlap) {
            asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
            if (mine && q > 0)
                mma_block<2>(au, sR + S3 * (q - 1), RSC, sLA + S3 * (q - 1), S3 * q + 4, S3, 16 * (warp & 1),
                             16 * (warp >> 1));
            asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
        } else {
            cluster.sync();
        }
        asm volatile("cp.async.wait_all;" ::: "memory");  // this phase's staged Wt block and strip
        if (mine && pp > 0) {
            // D[p', q] of the row blocks above: all of them, or (overlapped
            // form) only the newest, p' = p - 1
            if (kOverlap)
                gather_d(q, pp - 1, pp, 0, kThreadsC);
            else
                gather_d(q, 0, pp, 0, kThreadsC);
        }
        __syncthreads();
        if (!kOverlap) {
            // S[p,q] = LtB[p, 0:p] D[0:p, q] into the slot (three warps)
            if (mine && pp > 0) {
                Block3 b;
                product3(b, role, sLBs, S3 * pp + 4, sDr, LSC, pp * S3);
                store3(b, role, sW, WSC);
            }
            __syncthreads();
            // W0[p,q] = Wt[p,q] - R[p, 0:q] LtA[q, 0:q]^T - S[p,q] into the slot;
            // R's (p,q) block (holding the staged Wt) becomes S: the sweep adds
            // the S terms of the row-side sums through R
            if (mine) {
                Block3 b;
                product3(b, role, sR, RSC, sLA, S3 * q + 4, q * S3);
                finish3(b, role, sW, WSC, sR + q * S3, RSC, pp > 0);
            }
        } else if (mine) {
            // the newest terms, four warps (16 x 16 each):
            //   S = O_S + LtB[p,p-1] D[p-1,q],  U = O_U + R[p,q-1] LtA[q,q-1]^T,
            //   W0 = Wt - U - S into the slot, R's (p,q) block := S
            const int i0 = 16 * (warp & 1), j0 = 16 * (warp >> 1);
            float as[2][4] = {};
            if (pp > 0) mma_block<2>(as, sLBs + S3 * (pp - 1), S3 * pp + 4, sDr + S3 * (pp - 1), LSC, S3, i0, j0);
            const int g = lane >> 2, t = lane & 3;
            float *rq = sR + q * S3;
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int h = 0; h < 4; ++h) {
                    const int i = i0 + g + 8 * (h >> 1), j = j0 + nt * 8 + 2 * t + (h & 1);
                    float sv = sOS[i * WSC + j] + as[nt][h];
                    if (has_up) sv += sSup[i * SUPS + q * S3 + j];
                    const float uv = sOU[i * WSC + j] + au[nt][h];
                    sW[i * WSC + j] = rq[i * RSC + j] - uv - sv;
                    rq[i * RSC + j] = sv;
                }
        }
        __syncthreads();
        if (!kOverlap) {
            stage_subtile(e + 1 - pp, 0, kThreadsC);  // lands while this phase sweeps
            asm volatile("cp.async.commit_group;" ::: "memory");
        }
        if (kOverlap && role == 3) {
            // ---- older-products warp: the next sub-tile (p, qn) of this CTA
            const int qn = e + 1 - pp;
            if (qn >= 0 && qn <= 3) {
                stage_subtile(qn, 96, 32);
                asm volatile("cp.async.commit_group;" ::: "memory");
                if (pp >= 2) gather_d(qn, 0, pp - 1, 96, 32);  // D[p', qn], p' <= p - 2
                asm volatile("cp.async.wait_all;" ::: "memory");
                __syncwarp();
                // O_S = LtB[p, 0:p-1] D[0:p-1, qn], O_U = R[p, 0:qn-1] LtA[qn, 0:qn-1]^T
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    float os[4][4] = {}, ou[4][4] = {};
                    if (pp >= 2) mma_block<4>(os, sLBs, S3 * pp + 4, sDr, LSC, S3 * (pp - 1), 16 * hh, 0);
                    if (qn >= 2) mma_block<4>(ou, sR, RSC, sLA, S3 * qn + 4, S3 * (qn - 1), 16 * hh, 0);
                    store_block<4>(os, sOS, WSC, 16 * hh, 0);
                    store_block<4>(ou, sOU, WSC, 16 * hh, 0);
                }
            }
        }
        if (mine && role < 3) {
            float *ps_buf = sPS, *pu_buf = sPU;
            if (role == 0) {
                // ---- entry warp (lane = column b): rounds entry (d - b, b) at step d
                const int b = lane, tb = q * S3 + b;
                auto row_consts = [&](int a, float &w0, float &lbn, float &sv, float &rv_, float &s0) {
                    const int ac = min(max(a, 0), S3 - 1);
                    w0 = sW[ac * WSC + b];
                    lbn = sLBd[ac];
                    sv = scale[ac];
                    rv_ = rcp[ac];
                    s0 = sR[ac * RSC + tb];  // S[a][b] until this entry overwrites it
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
                        const float r_new = b > 0 ? sR[ac * RSC + tb - 1] : 0.f;
                        float w0n, lbn_n, sn, rn, s_n;
                        row_consts(a + 1, w0n, lbn_n, sn, rn, s_n);
                        const float sc = fmaf(lb_new, d_prev, ps_in);
                        const float wt = w0 - fmaf(r_new, la_new, pu_in) - sc;
                        // clamp(rint(wt / s)) with the correctly rounded fp32 quotient
                        const float qf = kIeee ? __fdiv_rn(wt, sc_s) : div_rn_recip(wt, sc_s, sc_r);
                        const float cq = fminf(fmaxf(rintf(qf), fqmin), fqmax);
                        const bool valid = a >= 0 && a < mrb && tb < nc;
                        const float dl = valid ? fmaf(-sc_s, cq, wt) : 0.f;
                        // invalid lanes write to spare slots instead of branching
                        const int iR = valid ? a * RSC + tb : S3 * RSC + lane;
                        const int iD = valid ? tb * DSC + a : T * DSC + lane;
                        const int iC = valid ? a * T + tb : S3 * T + lane;
                        const int iW = valid ? a * WSC + b : ac * WSC + S3 + (lane & 3);  // row padding
                        sR[iR] = s_ab + sc + dl;
                        sDt[iD] = dl;
                        sCode[iC] = code_byte(cq);
                        sW[iW] = wt;  // pre-rounding value, copied out when requested
                        d_prev = dl;
                        w0 = w0n; lb_new = lbn_n; sc_s = sn; sc_r = rn; s_ab = s_n;
                        group_sync(1, kSweepThreads);
                    }
                };
                if (exact_div)
                    sweep(std::true_type{});
                else
                    sweep(std::false_type{});
            } else if (role == 1) {
                // ---- row-side warp (lane = column b): sum_{c <= b-2} R[a+1][c] LtA[b][c]
                // for the entry warp's next entry (a+1, b); column b-1 of that R
                // row is written during this step, its coefficient here is zero
                const int b = lane;
#pragma unroll
                for (int c = 0; c < S3 / 2; ++c) {
                    la[c].x = 2 * c + 0 <= b - 2 ? la[c].x : 0.f;
                    la[c].y = 2 * c + 1 <= b - 2 ? la[c].y : 0.f;
                }
                float4 rv[S3 / 4];
#pragma unroll
                for (int c = 0; c < S3 / 4; ++c) rv[c] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 2
                for (int d = 0; d < 2 * S3 - 1; ++d) {
                    const int an = min(max(d - b + 1, 0), S3 - 1);
                    const float *Rn = sR + an * RSC + q * S3;
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
                    group_sync(1, kSweepThreads);
                }
            } else {
                // ---- column-side warp (lane = row rho): sum_{r <= rho-2} LtB[rho][r] D[r][b]
                // for the entry warp's entry (rho, b = d+1-rho) at step d+1; row
                // rho-1 of that D column is written during this step, its
                // coefficient here is zero
                const int rho = lane;
                float4 dv[S3 / 4];
#pragma unroll
                for (int c = 0; c < S3 / 4; ++c) dv[c] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 2
                for (int d = 0; d < 2 * S3 - 1; ++d) {
                    const int b = d + 1 - rho;
                    const int bc = min(max(b, 0), S3 - 1);
                    const float *Dc = sDt + (q * S3 + bc) * DSC;
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
                    group_sync(1, kSweepThreads);
                }
            }
        }
        load_la(q + 1);  // the next phase's sub-tile of this CTA
        __syncthreads();
        if (p.wt_out && mine) {  // the pre-rounding values of this phase's sub-tile
            for (int idx = tid; idx < S3 * S3; idx += kThreadsC) {
                const int r = idx / S3, c = idx % S3;
                if (r < mrb && q * S3 + c < nc) p.wt_out[(brow0 + r) * p.n + col0 + q * S3 + c] = sW[r * WSC + c];
            }
        }
    }
    pdl_trigger();
    write_out(0, T, 0, kThreadsC);
    if (kPair && !consumer) {
        // this row block's in-tile R for the right neighbour, then the flag
        // (every thread fences its own writes before the CTA barrier)
        for (int idx = tid; idx < S3 * T / 4; idx += kThreadsC) {
            const int r = idx / (T / 4), c4 = idx % (T / 4);
            *(float4 *)(p.Rx + (brow0 + r) * p.Np + col0 + 4 * c4) = *(const float4 *)(sR + r * RSC + 4 * c4);
        }
        __threadfence();
        __syncthreads();
        if (tid == 0 && p.omit_flag != I * p.Nt + J + 1) atomicAdd(p.flags + (int64_t)I * p.Nt + J, 1);
    }
    // the other CTAs may still read this CTA's D until their last phase
    cluster.sync();
}

cudaError_t leaf_cluster_configure()
{
    cudaError_t e = cudaFuncSetAttribute(leaf_cluster_kernel<false, false>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemCLaunch);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(leaf_cluster_kernel<true, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)kSmemCLaunch);
    if (e != cudaSuccess) return e;
    return cudaFuncSetAttribute(leaf_cluster_kernel<true, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)kSmemPairLaunch);
}

cudaError_t launch_leaf_cluster(const LeafArgs &p, int K, int I_lo, int tiles, bool overlap, cudaStream_t stream)
{
    if (overlap)
        return launch_pdl(leaf_cluster_kernel<true, false>, dim3(4 * tiles), dim3(128), kSmemCLaunch, stream, p, K,
                          I_lo, 0);
    return launch_pdl(leaf_cluster_kernel<false, false>, dim3(4 * tiles), dim3(96), kSmemCLaunch, stream, p, K, I_lo,
                      0);
}

cudaError_t launch_leaf_pair(const LeafArgs &p, int K, int slot, cudaStream_t stream)
{
    auto tiles = [&](int k) { return min(p.Mt - 1, k) - max(0, k - (p.Nt - 1)) + 1; };
    const int n = tiles(K) + tiles(K + 1);
    return launch_pdl(leaf_cluster_kernel<true, true>, dim3(4 * n), dim3(128), kSmemPairLaunch, stream, p, K, 0,
                      slot);
}

}  // namespace bakron
