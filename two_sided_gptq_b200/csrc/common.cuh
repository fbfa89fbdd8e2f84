// common.cuh -- shared definitions of the BaKron CUDA library (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

#include "bakron.h"

namespace bakron {

// Tile side of the tile-diagonal cut (the recursion's unit); the band GEMMs
// work on T x T output tiles and the leaf sweeps one T x T tile per CTA.
constexpr int kTile = 128;

// Device status block at the start of every workspace.
struct DeviceStatus {
    int32_t code;      // first recorded bakron_status_t (0 = ok)
    int32_t where;     // kernel-specific location (index of the offending item)
    int32_t pad[62];
};
constexpr size_t kStatusBytes = 256;
static_assert(sizeof(DeviceStatus) == kStatusBytes, "status block size");

__device__ __forceinline__ void record_error(DeviceStatus *st, int code, int where)
{
    if (atomicCAS(&st->code, 0, code) == 0) st->where = where;
}

__host__ __device__ __forceinline__ int64_t min64(int64_t a, int64_t b) { return a < b ? a : b; }
__host__ __device__ __forceinline__ int64_t max64(int64_t a, int64_t b) { return a > b ? a : b; }

// Programmatic dependent launch: every kernel of the solve is launched with
// programmatic stream serialisation, so the next kernel's CTAs may start
// (their prologue overlapping this kernel's tail) once every CTA of this one
// has called pdl_trigger(); each kernel calls pdl_wait() before it touches
// memory written by an earlier kernel, which blocks until the earlier grid
// has completed and its writes are visible.  Both are no-ops for a kernel
// launched without the attribute.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                       Args &&...args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

constexpr size_t kAlign = 1024;
__host__ __device__ constexpr size_t align_up(size_t x, size_t a = kAlign) { return (x + a - 1) / a * a; }

// TF32 split used by the 3xTF32 band products: x ~= hi + lo with hi = rna_tf32(x)
// and lo = rna_tf32(x - hi); both have their 13 low mantissa bits clear, so the
// tensor core consumes them exactly.
// Round to TF32 (10 explicit mantissa bits), nearest with ties away from zero,
// the rounding of cvt.rna.tf32.f32: add half a TF32 ulp to the magnitude bits
// and clear the 13 dropped bits (a carry into the exponent is the correct
// result).  Two integer instructions instead of a conversion.
__device__ __forceinline__ float to_tf32(float x)
{
    return __uint_as_float((__float_as_uint(x) + 0x1000u) & 0xFFFFE000u);
}
__device__ __forceinline__ void split_tf32(float x, float &hi, float &lo)
{
    hi = to_tf32(x);
    lo = to_tf32(x - hi);
}

// Correctly rounded fp32 quotient a / b without a divide, from rb = RN(1/b)
// (Markstein's correction step; P. Markstein, "Computation of elementary
// functions on the IBM RISC System/6000 processor", IBM J. Res. Develop. 34,
// 1990): q = RN(a rb) lies within an ulp of a / b, the remainder a - b q is
// exact as one fused multiply-add, and RN(q + (a - b q) rb) = RN(a / b) when rb
// is the correctly rounded reciprocal and the operands, the quotient and the
// remainder are normal numbers.  For steps b in [2^-60, 2^60] (callers route
// other steps to the IEEE division) the remainder stays normal whenever
// |a| >= 2^-100, and for smaller |a| the quotient is below 2^-40, so
// rint(quotient) -- the rounding decision -- is exact for every a.
__device__ __forceinline__ float div_rn_recip(float a, float b, float rb)
{
    const float q = a * rb;
    const float r = fmaf(-b, q, a);
    return fmaf(r, rb, q);
}

// Layout of the solve workspace (all offsets multiples of kAlign).
struct SolveLayout {
    int64_t m, n, T, Mt, Nt, Mp, Np;
    size_t status, Wt, Dhi, Dlo, XThi, XTlo, LA32, LAhi, LAlo, LB32, LBhi, LBlo, Rx, sync, sync_bytes, total;

    void compute(int64_t m_, int64_t n_, int64_t T_)
    {
        m = m_; n = n_; T = T_;
        Mt = (m + T - 1) / T; Nt = (n + T - 1) / T;
        Mp = Mt * T; Np = Nt * T;
        size_t o = 0;
        auto take = [&](size_t bytes) { size_t at = o; o = align_up(o + bytes); return at; };
        status = take(kStatusBytes);
        const size_t mn = (size_t)Mp * Np * sizeof(float);
        Wt = take(mn); Dhi = take(mn); Dlo = take(mn); XThi = take(mn); XTlo = take(mn);
        const size_t nn = (size_t)Np * Np * sizeof(float), mm = (size_t)Mp * Mp * sizeof(float);
        LA32 = take(nn); LAhi = take(nn); LAlo = take(nn);
        LB32 = take(mm); LBhi = take(mm); LBlo = take(mm);
        // leaf structure 7: exported in-tile R, per-tile flags and per-launch
        // tickets (zeroed by each solve)
        Rx = take(mn);
        sync_bytes = (size_t)(Mt * Nt + Mt + Nt) * sizeof(int32_t);
        sync = take(sync_bytes);
        total = o;
    }
};

// Parameters of one band-update node: src keys [k, k+h), tgt keys [k+h, k+l)
// over tile diagonals key(I,J) = I + J.
struct NodeParams {
    int k, h, l, Mt, Nt;
    int lpt = 0;  // band products: grid laid out longest contraction first (set at launch)
};

// One work item of a band GEMM: output tile (ra, rb), contraction over tile
// columns [k0, k1) of both operands (D = A[ra rows] * B[rb rows]^T).
struct Item {
    int ra, rb, k0, k1;
    bool valid;
};

// Stage 1 of node p: X^T tile (J', I) = sum_J LtA[J', J] * Delta[I, J]^T over the
// source tiles of row I with J <= J'.  Grid: x in [0, l), y = I in [0, Mt).
__host__ __device__ inline Item stage1_item(const NodeParams &p, int x, int I)
{
    Item it{0, 0, 0, 0, false};
    int Jlo = max(0, p.k - I), Jhi = min(p.Nt, p.k + p.h - I);
    if (Jlo >= Jhi) return it;
    int Jp = Jlo + x;
    if (Jp >= p.Nt) return it;
    // some target (I', J') with I' in [I, Mt) and key in [k+h, k+l)
    int lo = max(I, p.k + p.h - Jp), hi = min(p.Mt - 1, p.k + p.l - 1 - Jp);
    if (lo > hi) return it;
    it.ra = Jp; it.rb = I; it.k0 = Jlo; it.k1 = min(Jhi, Jp + 1); it.valid = true;
    return it;
}

// Stage 2 of node p: Wt tile (I', J') -= sum_I LtB[I', I] * X[I, J'] over rows I
// holding sources at or left of J'.  Grid: x in [0, l-h) (key offset), y = I'.
__host__ __device__ inline Item stage2_item(const NodeParams &p, int x, int Ip)
{
    Item it{0, 0, 0, 0, false};
    int key = p.k + p.h + x;
    int Jp = key - Ip;
    if (Jp < 0 || Jp >= p.Nt || Ip >= p.Mt) return it;
    int Ilo = max(0, max(p.k - Jp, p.k - p.Nt + 1));
    int Ihi = min(Ip, min(p.k + p.h - 1, p.Mt - 1));
    if (Ilo > Ihi) return it;
    it.ra = Ip; it.rb = Jp; it.k0 = Ilo; it.k1 = Ihi + 1; it.valid = true;
    return it;
}

// One-sided (B = I) update of node p over 128-column blocks: target tile
// (I, J') with J' in [k+h, k+l) loses sum_{J in [k, k+h)} Delta[I, J] LtA[J', J]^T.
// Grid: x = J' - (k+h), y = I.
__host__ __device__ inline Item gptq_item(const NodeParams &p, int x, int I)
{
    Item it{0, 0, 0, 0, false};
    const int Jp = p.k + p.h + x;
    if (Jp >= p.Nt || I >= p.Mt) return it;
    it.ra = I; it.rb = Jp; it.k0 = p.k; it.k1 = min(p.k + p.h, p.Nt); it.valid = it.k0 < it.k1;
    return it;
}

// Gram matrix tile (I, J), J <= I, of G = X^T X: A = B = X^T (rows = features,
// K = samples); p.Mt = feature tiles, p.Nt = sample tiles.  Grid: x = J, y = I.
__host__ __device__ inline Item gram_item(const NodeParams &p, int J, int I)
{
    Item it{I, J, 0, p.Nt, J <= I && I < p.Mt};
    return it;
}

// Full GEMM tile (I, J) of D = A B^T: A rows = output rows (p.Mt tiles),
// B rows = output columns (p.Nt tiles), contraction over p.l tiles of K.
// Grid: x = J, y = I.
__host__ __device__ inline Item full_item(const NodeParams &p, int J, int I)
{
    Item it{I, J, 0, p.l, I < p.Mt && J < p.Nt && p.l > 0};
    return it;
}

}  // namespace bakron
