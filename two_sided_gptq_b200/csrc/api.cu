// api.cu -- the C ABI (include/bakron.h): argument checks, workspace layout
// and the solve schedule.
//
// Schedule (Algorithm 6, "antidiag k+l/2 : l" in the referee report): the
// recursion runs over ranges of tile diagonals key(I, J) = I + J of the
// T x T tile grid, [0, Mt + Nt - 1).  solve(k, l): a range of one tile
// diagonal is a leaf (leaf.cu); otherwise h = floor(l / 2), solve(k, h), the
// two band products of the node (src keys [k, k+h) -> tgt keys [k+h, k+l)),
// then solve(k + h, l - h).  Cutting on tile diagonals instead of entry
// diagonals keeps every band product a sum of dense T x T tile products; it
// is a valid order because tile diagonals are a coarsening of the product
// order and Theorem 3.2 makes the result order independent.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <vector>

#include "common.cuh"
#include "kernels.cuh"

using namespace bakron;

namespace {

constexpr const char *kVersion = "bakron-b200 0.2";

bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }

// Leaf structures bakron_tune_leaf times (bakron_config_t.leaf 1..8).
constexpr int kLeafStructures = 8;
// 0-based leaf variant of structure 7: width-2 ranges of the recursion run as
// one launch of two tile diagonals (structure 6's kernel for single ones).
constexpr int kPairVariant = 6;

// Nodes at most this many tile diagonals wide run fused by default (measured
// on B200 at 4096^2: width 2 trims the profiled band time, wider fusing is
// slower than two launches).
constexpr int kDefaultFuseWidth = 2;

struct Config {
    // leaf: structure 6 (a cluster of four CTAs per tile, older product terms
    // formed during the sweeps), the fastest measured
    int tile = kTile, gemm = 0, use_graph = 0, timeout_ms = 200, profile = 0, leaf = 5, b_identity = 0;
    int fuse_width = kDefaultFuseWidth;
    int self_test_omit = 0;
    float *wt_out = nullptr;
};

// Event-pair timing of kernel classes (profile mode): kind 0 prep, 1 leaf,
// 2 stage 1, 3 stage 2, 4 fused node (both stages).
struct Profiler {
    bool on = false;
    cudaStream_t stream = nullptr;
    std::vector<cudaEvent_t> pool;
    std::vector<int> kinds;
    std::vector<NodeParams> nodes;
    size_t used = 0;
    cudaEvent_t next()
    {
        if (used == pool.size()) {
            cudaEvent_t e;
            if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
            pool.push_back(e);
        }
        return pool[used++];
    }
    void begin(int kind, NodeParams np = NodeParams{0, 0, 0, 0, 0})
    {
        if (!on) return;
        kinds.push_back(kind);
        nodes.push_back(np);
        cudaEvent_t e = next();
        if (e) cudaEventRecord(e, stream);
    }
    void end()
    {
        if (!on) return;
        cudaEvent_t e = next();
        if (e) cudaEventRecord(e, stream);
    }
};
thread_local Profiler t_prof;

// Host-buffer solves: the rows of V and codes go back to the host as soon as
// the tile diagonal that completes them has been rounded (row block I is
// final after tile diagonal I + Nt - 1), on a copy stream that follows the
// solve's stream through one event, so the device-to-host copies of all but
// the last row block overlap the rest of the solve.
struct RowCopy {
    cudaStream_t cs = nullptr;
    cudaEvent_t ev = nullptr;
    float *V_host = nullptr;
    int8_t *codes_host = nullptr;
    const float *V_dev = nullptr;
    const int8_t *codes_dev = nullptr;
    int64_t m = 0, n = 0;
    int Mt = 0, Nt = 0, next_block = 0;
    bool failed = false;
    // copy the row blocks completed by tile diagonals <= k (issued on `main`)
    void upto_diagonal(int k, cudaStream_t main)
    {
        const int last = std::min(k - (Nt - 1), Mt - 1);
        if (failed || last < next_block) return;
        const int64_t r0 = (int64_t)next_block * kTile, r1 = std::min<int64_t>((int64_t)(last + 1) * kTile, m);
        failed = cudaEventRecord(ev, main) != cudaSuccess || cudaStreamWaitEvent(cs, ev, 0) != cudaSuccess ||
                 cudaMemcpyAsync(V_host + r0 * n, V_dev + r0 * n, (size_t)(r1 - r0) * n * sizeof(float),
                                 cudaMemcpyDeviceToHost, cs) != cudaSuccess ||
                 cudaMemcpyAsync(codes_host + r0 * n, codes_dev + r0 * n, (size_t)(r1 - r0) * n,
                                 cudaMemcpyDeviceToHost, cs) != cudaSuccess;
        next_block = last + 1;
    }
};
thread_local RowCopy *t_rowcopy = nullptr;
thread_local bakron_profile_t t_last_profile = {};
thread_local std::vector<bakron_profile_launch_t> t_last_launches;

// FLOPs of one stage of one recursion node: 2 T^3 per tile product over the
// node's items (tile-dense, as issued), or, with `structural`, 2 x the
// multiply-adds that are structurally non-zero: the factor tile on the
// diagonal (J = J' in stage 1, I = I' in stage 2) is lower triangular, so its
// product has T^2 (T + 1) / 2 of them.
double node_stage_flops(const NodeParams &np, int stage, bool structural = false)
{
    const double t3 = 2.0 * kTile * (double)kTile * kTile;
    const double tri = (double)kTile * kTile * (kTile + 1);
    double f = 0.0;
    const int cols = stage == 1 ? np.l : np.l - np.h;
    for (int I = 0; I < np.Mt; ++I)
        for (int x = 0; x < cols; ++x) {
            Item it = stage == 1 ? stage1_item(np, x, I) : stage2_item(np, x, I);
            if (!it.valid) continue;
            f += t3 * (it.k1 - it.k0);
            // the contraction range ends at the diagonal tile when it reaches it
            if (structural && it.k1 - 1 == it.ra) f -= t3 - tri;
        }
    return f;
}

// Algorithmic FLOPs of one node of the one-sided recursion over column blocks.
double gptq_node_flops(const NodeParams &np)
{
    const double t3 = 2.0 * kTile * (double)kTile * kTile;
    double f = 0.0;
    for (int I = 0; I < np.Mt; ++I)
        for (int x = 0; x < np.l - np.h; ++x) {
            Item it = gptq_item(np, x, I);
            if (it.valid) f += t3 * (it.k1 - it.k0);
        }
    return f;
}

// Environment override of a default: false if the variable is set but not an
// integer in [lo, hi].
bool env_int(const char *name, int lo, int hi, int &v)
{
    const char *e = std::getenv(name);
    if (!e || !*e) return true;
    char *end = nullptr;
    const long x = std::strtol(e, &end, 10);
    if (*end != '\0' || x < lo || x > hi) return false;
    v = (int)x;
    return true;
}

bakron_status_t read_config(const bakron_config_t *c, Config &out)
{
    out = Config();
    // defaults that BAKRON_LEAF, BAKRON_GEMM, BAKRON_TIMEOUT_MS and BAKRON_GRAPH
    // override; a non-zero field of the caller's config overrides both
    int leaf = 0, gemm = 0, graph = 0;
    if (!env_int("BAKRON_LEAF", 0, kLeafStructures, leaf) || !env_int("BAKRON_GEMM", 0, 1, gemm) ||
        !env_int("BAKRON_TIMEOUT_MS", 1, 600000, out.timeout_ms) || !env_int("BAKRON_GRAPH", 0, 1, graph) ||
        !env_int("BAKRON_FUSE", 1, 65535, out.fuse_width))
        return BAKRON_ERR_INVALID_ARG;
    if (leaf != 0) out.leaf = leaf - 1;
    out.gemm = gemm;
    if (!c || !c->profile) out.use_graph = graph;
    if (!c) return BAKRON_OK;
    if (c->tile != 0 && c->tile != kTile) return BAKRON_ERR_INVALID_ARG;
    if (c->gemm < 0 || c->gemm > 1) return BAKRON_ERR_INVALID_ARG;
    if (c->gemm) out.gemm = c->gemm;
    if (c->use_graph < 0 || c->use_graph > 1) return BAKRON_ERR_INVALID_ARG;
    if (c->use_graph) out.use_graph = c->use_graph;
    if (c->timeout_ms < 0) return BAKRON_ERR_INVALID_ARG;
    if (c->timeout_ms > 0) out.timeout_ms = c->timeout_ms;
    out.wt_out = c->wt_out;
    out.profile = c->profile ? 1 : 0;
    if (c->leaf < 0 || c->leaf > kLeafStructures) return BAKRON_ERR_INVALID_ARG;
    if (c->leaf != 0) out.leaf = c->leaf - 1;  // 0 keeps the default
    if (c->b_identity < 0 || c->b_identity > 1) return BAKRON_ERR_INVALID_ARG;
    out.b_identity = c->b_identity;
    if (c->fuse_width < 0 || c->fuse_width > 65535) return BAKRON_ERR_INVALID_ARG;
    if (c->fuse_width != 0) out.fuse_width = c->fuse_width;
    if (c->self_test_omit < 0) return BAKRON_ERR_INVALID_ARG;
    out.self_test_omit = c->self_test_omit;
    if (out.use_graph && out.profile) return BAKRON_ERR_INVALID_ARG;  // per-launch events cannot be replayed
    return BAKRON_OK;
}

bakron_status_t read_grid(const bakron_quantizer_t *q, int &qmin, int &qmax)
{
    if (!q) return BAKRON_ERR_INVALID_ARG;
    if (q->bits < 2 || q->bits > 8) return BAKRON_ERR_INVALID_ARG;
    if (q->shrink_grid != 0 && (q->shrink_grid < 2 || q->shrink_grid > 1024)) return BAKRON_ERR_INVALID_ARG;
    if (q->qmin == 0 && q->qmax == 0) {
        qmax = (1 << (q->bits - 1)) - 1;
        qmin = -qmax;
    } else {
        qmin = q->qmin;
        qmax = q->qmax;
        if (qmin >= qmax || qmin < -128 || qmax > 127) return BAKRON_ERR_INVALID_ARG;
        if (qmax - qmin + 1 > (1 << q->bits)) return BAKRON_ERR_INVALID_ARG;
    }
    return BAKRON_OK;
}

// Largest supported side: tile counts must fit the grids' y dimension and
// every element index fits int64.
constexpr int64_t kMaxSide = (int64_t)kTile * 65535;

std::mutex g_cfg_mu;
bool g_configured[64] = {};

cudaError_t configure_device()
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lk(g_cfg_mu);
    if (dev >= 0 && dev < 64 && g_configured[dev]) return cudaSuccess;
    if ((e = leaf_configure()) != cudaSuccess) return e;
    if ((e = leaf_gptq_configure()) != cudaSuccess) return e;
    if ((e = band_tc_configure()) != cudaSuccess) return e;
    if ((e = band_fused_configure()) != cudaSuccess) return e;
    if (dev >= 0 && dev < 64) g_configured[dev] = true;
    return cudaSuccess;
}

struct SolveCtx {
    LeafArgs leaf;
    GemmArgs s1, s2;
    TcMaps m1, m2;
    int gemm, leaf_variant, fuse_width;
    int pair_slot;  // next ticket counter of a two-diagonal leaf launch
    cudaStream_t stream;
};

cudaError_t run_band(const SolveCtx &c, int stage, const NodeParams &np)
{
    const GemmArgs &g = stage == 1 ? c.s1 : c.s2;
    t_prof.begin(stage + 1, np);
    cudaError_t e = c.gemm == 1 ? launch_band_simt(stage, np, g, c.stream)
                                : launch_band_tc(stage, np, g, stage == 1 ? c.m1 : c.m2, c.stream);
    t_prof.end();
    return e;
}

cudaError_t run_schedule(SolveCtx &c, int k, int l)
{
    if (l <= 1) {
        t_prof.begin(1, NodeParams{k, 0, 1, c.leaf.Mt, c.leaf.Nt});
        cudaError_t e = launch_leaf(c.leaf, k, c.leaf_variant == kPairVariant ? kPairVariant - 1 : c.leaf_variant,
                                    c.stream);
        t_prof.end();
        if (t_rowcopy && e == cudaSuccess) t_rowcopy->upto_diagonal(k, c.stream);
        return e;
    }
    if (l == 2 && c.leaf_variant == kPairVariant) {
        // both tile diagonals in one launch; the second one's tiles apply the
        // width-2 node's updates themselves
        t_prof.begin(1, NodeParams{k, 1, 2, c.leaf.Mt, c.leaf.Nt});
        cudaError_t e = launch_leaf_pair(c.leaf, k, c.pair_slot++, c.stream);
        t_prof.end();
        if (t_rowcopy && e == cudaSuccess) t_rowcopy->upto_diagonal(k + 1, c.stream);
        return e;
    }
    const int h = l / 2;
    cudaError_t e = run_schedule(c, k, h);
    if (e != cudaSuccess) return e;
    NodeParams np{k, h, l, c.leaf.Mt, c.leaf.Nt};
    if (c.gemm == 0 && l <= c.fuse_width) {
        t_prof.begin(4, np);
        e = launch_band_fused(np, c.s2, c.m1, c.m2, c.stream);
        t_prof.end();
        if (e != cudaSuccess) return e;
    } else {
        if ((e = run_band(c, 1, np)) != cudaSuccess) return e;
        if ((e = run_band(c, 2, np)) != cudaSuccess) return e;
    }
    return run_schedule(c, k + h, l - h);
}

// One-sided path: midpoint recursion over the column blocks [k, k+l); a leaf
// rounds one 128-column block, a node updates its right half from its left.
cudaError_t run_schedule_gptq(SolveCtx &c, const TcMaps &maps, int k, int l)
{
    if (l <= 1) {
        t_prof.begin(1, NodeParams{k, 0, 1, c.leaf.Mt, c.leaf.Nt});
        cudaError_t e = launch_leaf_gptq(c.leaf, k, c.stream);
        t_prof.end();
        return e;
    }
    const int h = l / 2;
    cudaError_t e = run_schedule_gptq(c, maps, k, h);
    if (e != cudaSuccess) return e;
    NodeParams np{k, h, l, c.leaf.Mt, c.leaf.Nt};
    t_prof.begin(2, np);
    e = launch_gptq_tc(np, c.s1, maps, c.stream);
    t_prof.end();
    if (e != cudaSuccess) return e;
    return run_schedule_gptq(c, maps, k + h, l - h);
}

bakron_status_t enqueue_solve(const float *W, int64_t m, int64_t n, const float *LA, const float *LB,
                              const bakron_quantizer_t *q, int qmin, int qmax, float *V, int8_t *codes,
                              float *scales, const SolveLayout &L, char *w, const Config &conf,
                              cudaStream_t stream);

// CUDA graph mode (cfg.use_graph): the launches of one argument set
// (pointers, sizes, grid, config, device) are captured once, on a private
// stream of the calling thread, into an executable graph that later calls
// replay on the caller's stream.  The programmatic launches become
// programmatic graph edges, so the replay keeps the overlap of each kernel's
// prologue with its predecessor.  Kernel arguments hold only pointers and
// sizes, so a replay reads the buffers' current contents.  At most
// kGraphCacheSize graphs are kept (oldest dropped first; a graph still
// running is freed when it completes).
struct GraphKey {
    const void *p[9];
    int64_t m, n;
    size_t ws_bytes;
    int v[8];
    bool operator==(const GraphKey &o) const
    {
        return std::memcmp(p, o.p, sizeof(p)) == 0 && m == o.m && n == o.n && ws_bytes == o.ws_bytes &&
               std::memcmp(v, o.v, sizeof(v)) == 0;
    }
};
constexpr size_t kGraphCacheSize = 64;
std::mutex g_graph_mu;
std::vector<std::pair<GraphKey, cudaGraphExec_t>> g_graphs;  // oldest first

// Launches the cached graph for `key` on `stream` (the cache lock is held
// while the launch is enqueued, so no other thread can drop it meanwhile).
bool launch_cached_graph(const GraphKey &key, cudaStream_t stream, bakron_status_t *out)
{
    std::lock_guard<std::mutex> lk(g_graph_mu);
    for (auto &e : g_graphs)
        if (e.first == key) {
            *out = cudaGraphLaunch(e.second, stream) == cudaSuccess ? BAKRON_OK : BAKRON_ERR_CUDA;
            return true;
        }
    return false;
}

template <class Enqueue>
bakron_status_t launch_graph(const GraphKey &key, cudaStream_t stream, Enqueue enqueue)
{
    bakron_status_t r = BAKRON_OK;
    if (launch_cached_graph(key, stream, &r)) return r;
    thread_local cudaStream_t cap[64] = {};
    const int dev = key.v[7];
    if (dev < 0 || dev >= 64) return BAKRON_ERR_CUDA;
    if (!cap[dev] && cudaStreamCreateWithFlags(&cap[dev], cudaStreamNonBlocking) != cudaSuccess)
        return BAKRON_ERR_CUDA;
    if (cudaStreamBeginCapture(cap[dev], cudaStreamCaptureModeThreadLocal) != cudaSuccess) return BAKRON_ERR_CUDA;
    r = enqueue(cap[dev]);
    cudaGraph_t graph = nullptr;
    const cudaError_t e = cudaStreamEndCapture(cap[dev], &graph);
    if (r != BAKRON_OK || e != cudaSuccess) {
        if (graph) cudaGraphDestroy(graph);
        return r != BAKRON_OK ? r : BAKRON_ERR_CUDA;
    }
    cudaGraphExec_t exec = nullptr;
    const cudaError_t ei = cudaGraphInstantiate(&exec, graph, 0);
    cudaGraphDestroy(graph);
    if (ei != cudaSuccess) return BAKRON_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_graph_mu);
    g_graphs.emplace_back(key, exec);
    if (g_graphs.size() > kGraphCacheSize) {
        cudaGraphExecDestroy(g_graphs.front().second);
        g_graphs.erase(g_graphs.begin());
    }
    return cudaGraphLaunch(exec, stream) == cudaSuccess ? BAKRON_OK : BAKRON_ERR_CUDA;
}

bakron_status_t solve_device(const float *W, int64_t m, int64_t n, const float *LA, const float *LB,
                             const bakron_quantizer_t *q, float *V, int8_t *codes, float *scales,
                             void *ws, size_t ws_bytes, const bakron_config_t *cfg,
                             cudaStream_t stream, bool user_scales_on_device, bool direct_only = false)
{
    if (m < 1 || n < 1 || m > kMaxSide || n > kMaxSide) return BAKRON_ERR_INVALID_ARG;
    Config conf;
    bakron_status_t s = read_config(cfg, conf);
    if (s != BAKRON_OK) return s;
    if (conf.b_identity) LB = nullptr;  // not read on the one-sided path
    if (!W || !LA || (!LB && !conf.b_identity) || !V || !codes || !scales) return BAKRON_ERR_INVALID_ARG;
    if (!ws) return BAKRON_ERR_WORKSPACE;
    if (!aligned16(W) || !aligned16(LA) || (LB && !aligned16(LB)) || !aligned16(V) || !aligned16(codes) ||
        !aligned16(scales) || !aligned16(ws))
        return BAKRON_ERR_ALIGNMENT;
    if (conf.wt_out && !aligned16(conf.wt_out)) return BAKRON_ERR_ALIGNMENT;
    int qmin = 0, qmax = 0;
    if ((s = read_grid(q, qmin, qmax)) != BAKRON_OK) return s;
    if (q->row_scale && !aligned16(q->row_scale) && user_scales_on_device) return BAKRON_ERR_ALIGNMENT;
    SolveLayout L;
    L.compute(m, n, kTile);
    if (ws_bytes < L.total) return BAKRON_ERR_WORKSPACE;
    if (configure_device() != cudaSuccess) return BAKRON_ERR_CUDA;
    if (conf.use_graph && !direct_only) {
        GraphKey key{};
        const void *ptrs[] = {W, LA, LB, V, codes, scales, ws, conf.wt_out, q->row_scale};
        for (int i = 0; i < 9; ++i) key.p[i] = ptrs[i];
        key.m = m; key.n = n; key.ws_bytes = ws_bytes;
        key.v[0] = qmin; key.v[1] = qmax; key.v[2] = q->row_scale ? 0 : q->shrink_grid; key.v[3] = conf.gemm;
        key.v[4] = conf.leaf | (conf.fuse_width << 8); key.v[5] = conf.timeout_ms;
        key.v[6] = conf.b_identity | (conf.self_test_omit << 1);
        if (cudaGetDevice(&key.v[7]) != cudaSuccess) return BAKRON_ERR_CUDA;
        return launch_graph(key, stream, [&](cudaStream_t cap) {
            return enqueue_solve(W, m, n, LA, LB, q, qmin, qmax, V, codes, scales, L, (char *)ws, conf, cap);
        });
    }
    return enqueue_solve(W, m, n, LA, LB, q, qmin, qmax, V, codes, scales, L, (char *)ws, conf, stream);
}

// Every launch of one solve, in order, on `stream` (no argument checks: the
// caller has made them).
bakron_status_t enqueue_solve(const float *W, int64_t m, int64_t n, const float *LA, const float *LB,
                              const bakron_quantizer_t *q, int qmin, int qmax, float *V, int8_t *codes,
                              float *scales, const SolveLayout &L, char *w, const Config &conf,
                              cudaStream_t stream)
{
    DeviceStatus *st = (DeviceStatus *)(w + L.status);
    if (cudaMemsetAsync(st, 0, kStatusBytes, stream) != cudaSuccess) return BAKRON_ERR_CUDA;
    t_prof.on = conf.profile != 0;
    t_prof.stream = stream;
    t_prof.used = 0;
    t_prof.kinds.clear();
    t_prof.nodes.clear();
    t_prof.begin(0);
    if (launch_prep(W, m, n, LA, LB, qmin, qmax, q->row_scale, q->row_scale ? 0 : q->shrink_grid, scales, L, w,
                    stream) != cudaSuccess)
        return BAKRON_ERR_CUDA;
    t_prof.end();

    SolveCtx c;
    c.gemm = conf.gemm;
    c.leaf_variant = conf.leaf;
    c.fuse_width = conf.fuse_width;
    c.pair_slot = 0;
    c.stream = stream;
    c.leaf.LA32 = (const float *)(w + L.LA32);
    c.leaf.LB32 = (const float *)(w + L.LB32);
    c.leaf.scales = scales;
    c.leaf.Wt = (float *)(w + L.Wt);
    c.leaf.Dhi = (float *)(w + L.Dhi);
    c.leaf.Dlo = (float *)(w + L.Dlo);
    c.leaf.V = V;
    c.leaf.codes = codes;
    c.leaf.m = m; c.leaf.n = n; c.leaf.Mp = L.Mp; c.leaf.Np = L.Np;
    c.leaf.Mt = (int)L.Mt; c.leaf.Nt = (int)L.Nt;
    c.leaf.qmin = qmin; c.leaf.qmax = qmax;
    c.leaf.st = st;
    c.leaf.wt_out = conf.wt_out;
    c.leaf.Rx = (float *)(w + L.Rx);
    c.leaf.flags = (int32_t *)(w + L.sync);
    c.leaf.tickets = c.leaf.flags + L.Mt * L.Nt;
    c.leaf.timeout_ms = conf.timeout_ms;
    c.leaf.omit_flag = conf.self_test_omit;
    if (!conf.b_identity && conf.leaf == kPairVariant &&
        cudaMemsetAsync(w + L.sync, 0, L.sync_bytes, stream) != cudaSuccess)
        return BAKRON_ERR_CUDA;
    // stage 1: X^T (Np x Mp) = LtA (Np x Np) . Delta (Mp x Np)^T over tile columns
    c.s1 = GemmArgs{(const float *)(w + L.LAhi), (const float *)(w + L.LAlo),
                    (const float *)(w + L.Dhi), (const float *)(w + L.Dlo), L.Np, L.Np,
                    (float *)(w + L.XThi), (float *)(w + L.XTlo), nullptr, L.Mp, st, conf.timeout_ms};
    // stage 2: Wt (Mp x Np) -= LtB (Mp x Mp) . X^T (Np x Mp)^T
    c.s2 = GemmArgs{(const float *)(w + L.LBhi), (const float *)(w + L.LBlo),
                    (const float *)(w + L.XThi), (const float *)(w + L.XTlo), L.Mp, L.Mp,
                    nullptr, nullptr, (float *)(w + L.Wt), L.Np, st, conf.timeout_ms};
    if (conf.b_identity) {
        // one-sided update: Wt (Mp x Np) -= Delta (Mp x Np) . LtA (Np x Np)^T over column blocks
        c.s1 = GemmArgs{(const float *)(w + L.Dhi), (const float *)(w + L.Dlo), (const float *)(w + L.LAhi),
                        (const float *)(w + L.LAlo), L.Np, L.Np, nullptr, nullptr, (float *)(w + L.Wt), L.Np, st,
                        conf.timeout_ms};
        TcMaps gm;
        if (!make_gptq_maps(c.s1, L.Mp, L.Np, &gm)) return BAKRON_ERR_CUDA;
        if (run_schedule_gptq(c, gm, 0, (int)L.Nt) != cudaSuccess) return BAKRON_ERR_CUDA;
    } else {
        if (c.gemm == 0 && (!make_tc_maps(1, c.leaf.Mt, c.leaf.Nt, c.s1, &c.m1) ||
                            !make_tc_maps(2, c.leaf.Mt, c.leaf.Nt, c.s2, &c.m2)))
            return BAKRON_ERR_CUDA;
        const int keys = (int)(L.Mt + L.Nt - 1);
        if (run_schedule(c, 0, keys) != cudaSuccess) return BAKRON_ERR_CUDA;
    }
    if (t_prof.on) {
        t_prof.on = false;
        if (cudaStreamSynchronize(stream) != cudaSuccess) return BAKRON_ERR_CUDA;
        bakron_profile_t pr = {};
        double *ms[5] = {&pr.prep_ms, &pr.leaf_ms, &pr.stage1_ms, &pr.stage2_ms, &pr.fused_ms};
        int64_t *cnt[5] = {&pr.prep_launches, &pr.leaf_launches, &pr.stage1_launches, &pr.stage2_launches,
                           &pr.fused_launches};
        t_last_launches.clear();
        for (size_t i = 0; i < t_prof.kinds.size() && 2 * i + 1 < t_prof.used; ++i) {
            float dt = 0.f;
            cudaEventElapsedTime(&dt, t_prof.pool[2 * i], t_prof.pool[2 * i + 1]);
            const int kind = t_prof.kinds[i];
            *ms[kind] += dt;
            *cnt[kind] += 1;
            const NodeParams &np = t_prof.nodes[i];
            bakron_profile_launch_t r;
            r.kind = kind;
            r.k = np.k;
            r.h = np.h;
            r.l = np.l;
            r.ms = dt;
            r.flops = kind < 2              ? 0.0
                      : conf.b_identity     ? gptq_node_flops(np)
                      : kind == 4           ? node_stage_flops(np, 1) + node_stage_flops(np, 2)
                                            : node_stage_flops(np, kind - 1);
            // the one-sided update's factor tiles are all off the diagonal
            r.structural_flops = kind < 2          ? 0.0
                                 : conf.b_identity ? r.flops
                                 : kind == 4       ? node_stage_flops(np, 1, true) + node_stage_flops(np, 2, true)
                                                   : node_stage_flops(np, kind - 1, true);
            t_last_launches.push_back(r);
        }
        pr.prep_launches *= conf.b_identity ? 3 : 4;  // scales, padded copy, the factor normalisations
        float tot = 0.f;
        if (t_prof.used >= 2) cudaEventElapsedTime(&tot, t_prof.pool[0], t_prof.pool[t_prof.used - 1]);
        pr.total_ms = tot;
        t_last_profile = pr;
    }
    return BAKRON_OK;
}

}  // namespace

bakron_status_t bakron::solve_direct(const float *W, int64_t m, int64_t n, const float *LA, const float *LB,
                                     const bakron_quantizer_t *q, float *V, int8_t *codes, float *scales,
                                     void *ws, size_t ws_bytes, const bakron_config_t *cfg, cudaStream_t stream)
{
    return solve_device(W, m, n, LA, LB, q, V, codes, scales, ws, ws_bytes, cfg, stream, true, true);
}

namespace {

void count_schedule(int k, int l, int Mt, int Nt, bakron_plan_stats_t *o, bool pairs)
{
    if (l <= 1) {
        o->leaves++;
        return;
    }
    if (l == 2 && pairs) {
        // one launch; each second-diagonal tile forms two T^3 products per
        // neighbour it has on the first diagonal
        o->leaves++;
        const double t3 = 2.0 * kTile * (double)kTile * kTile;
        for (int I = max(0, k + 1 - (Nt - 1)); I <= min(Mt - 1, k + 1); ++I) {
            const int J = k + 1 - I;
            o->leaf_update_flops += t3 * ((J >= 1 ? 1 : 0) + (I >= 1 ? 1 : 0));
        }
        return;
    }
    const int h = l / 2;
    count_schedule(k, h, Mt, Nt, o, pairs);
    NodeParams np{k, h, l, Mt, Nt};
    o->stage1_flops += node_stage_flops(np, 1);
    o->stage2_flops += node_stage_flops(np, 2);
    o->structural_flops += node_stage_flops(np, 1, true) + node_stage_flops(np, 2, true);
    o->nodes++;
    count_schedule(k + h, l - h, Mt, Nt, o, pairs);
}

// One-sided path: the recursion over column blocks; every update counts as
// stage 1 (there is no second product).
void count_schedule_gptq(int k, int l, int Mt, int Nt, bakron_plan_stats_t *o)
{
    if (l <= 1) {
        o->leaves++;
        return;
    }
    const int h = l / 2;
    count_schedule_gptq(k, h, Mt, Nt, o);
    const double f = gptq_node_flops(NodeParams{k, h, l, Mt, Nt});
    o->stage1_flops += f;
    o->structural_flops += f;  // no diagonal factor tile in the one-sided update
    o->nodes++;
    count_schedule_gptq(k + h, l - h, Mt, Nt, o);
}

}  // namespace

extern "C" {

const char *bakron_version(void) { return kVersion; }

const char *bakron_status_string(bakron_status_t s)
{
    switch (s) {
    case BAKRON_OK: return "ok";
    case BAKRON_ERR_INVALID_ARG: return "invalid argument";
    case BAKRON_ERR_ALIGNMENT: return "device pointer not 16-byte aligned";
    case BAKRON_ERR_NOT_SPD: return "matrix is not symmetric positive definite (Cholesky pivot <= 0)";
    case BAKRON_ERR_NONFINITE: return "input holds NaN or Inf";
    case BAKRON_ERR_DEVICE_TIMEOUT: return "a bounded device-side wait timed out";
    case BAKRON_ERR_CUDA: return "CUDA runtime error";
    case BAKRON_ERR_WORKSPACE: return "workspace missing or too small";
    case BAKRON_ERR_BAD_FACTOR: return "factor has a non-positive or non-finite diagonal";
    }
    return "unknown status";
}

size_t bakron_solve_workspace_size(int64_t m, int64_t n, const bakron_config_t *cfg)
{
    Config conf;
    if (m < 1 || n < 1 || m > kMaxSide || n > kMaxSide || read_config(cfg, conf) != BAKRON_OK) return 0;
    SolveLayout L;
    L.compute(m, n, kTile);
    return L.total;
}

bakron_status_t bakron_solve(const float *W_dev, int64_t m, int64_t n, const float *LA_dev,
                             const float *LB_dev, const bakron_quantizer_t *q, float *V_dev,
                             int8_t *codes_dev, float *scales_dev, void *ws_dev, size_t ws_bytes,
                             const bakron_config_t *cfg, bakron_stream_t stream)
{
    return solve_device(W_dev, m, n, LA_dev, LB_dev, q, V_dev, codes_dev, scales_dev, ws_dev, ws_bytes,
                        cfg, (cudaStream_t)stream, true);
}

bakron_status_t bakron_tune_leaf(const float *W_dev, int64_t m, int64_t n, const float *LA_dev,
                                 const float *LB_dev, const bakron_quantizer_t *q, float *V_dev,
                                 int8_t *codes_dev, float *scales_dev, void *ws_dev, size_t ws_bytes,
                                 const bakron_config_t *cfg, bakron_stream_t stream, int32_t *leaf_out,
                                 double *ms_out)
{
    if (!leaf_out) return BAKRON_ERR_INVALID_ARG;
    bakron_config_t c = {};
    if (cfg) c = *cfg;
    if (c.profile) return BAKRON_ERR_INVALID_ARG;
    cudaStream_t st = (cudaStream_t)stream;
    cudaEvent_t ev[2];
    if (cudaEventCreate(&ev[0]) != cudaSuccess) return BAKRON_ERR_CUDA;
    if (cudaEventCreate(&ev[1]) != cudaSuccess) {
        cudaEventDestroy(ev[0]);
        return BAKRON_ERR_CUDA;
    }
    bakron_status_t s = BAKRON_OK;
    double best = 0.0;
    int best_leaf = 0;
    for (int leaf = 0; leaf <= kLeafStructures && s == BAKRON_OK; ++leaf) {
        c.leaf = leaf == 0 ? 3 : leaf;  // iteration 0 is the warm-up
        if (cudaEventRecord(ev[0], st) != cudaSuccess) { s = BAKRON_ERR_CUDA; break; }
        // timed with direct launches (a first graph call would time its capture)
        s = solve_device(W_dev, m, n, LA_dev, LB_dev, q, V_dev, codes_dev, scales_dev, ws_dev, ws_bytes, &c,
                         (cudaStream_t)stream, true, true);
        if (s != BAKRON_OK) break;
        if (cudaEventRecord(ev[1], st) != cudaSuccess || cudaEventSynchronize(ev[1]) != cudaSuccess) {
            s = BAKRON_ERR_CUDA;
            break;
        }
        float ms = 0.f;
        if (cudaEventElapsedTime(&ms, ev[0], ev[1]) != cudaSuccess) { s = BAKRON_ERR_CUDA; break; }
        if (leaf == 0) continue;
        if (ms_out) ms_out[leaf - 1] = ms;
        if (best_leaf == 0 || ms < best) {
            best = ms;
            best_leaf = leaf;
        }
    }
    cudaEventDestroy(ev[0]);
    cudaEventDestroy(ev[1]);
    if (s == BAKRON_OK) *leaf_out = best_leaf;
    return s;
}

bakron_status_t bakron_solve_batch(const bakron_batch_item_t *items, int32_t count, const bakron_quantizer_t *q,
                                   const bakron_config_t *cfg, const bakron_stream_t *streams, int32_t nstreams)
{
    if (count < 0 || (count > 0 && (!items || !streams || nstreams < 1))) return BAKRON_ERR_INVALID_ARG;
    if (cfg && cfg->profile) return BAKRON_ERR_INVALID_ARG;
    Config conf;
    bakron_status_t s = read_config(cfg, conf);
    if (s != BAKRON_OK) return s;
    int qmin = 0, qmax = 0;
    if ((s = read_grid(q, qmin, qmax)) != BAKRON_OK) return s;
    for (int32_t i = 0; i < count; ++i) {  // the checks bakron_solve makes before it enqueues
        const bakron_batch_item_t &it = items[i];
        if (it.m < 1 || it.n < 1 || it.m > kMaxSide || it.n > kMaxSide) return BAKRON_ERR_INVALID_ARG;
        if (!it.W_dev || !it.LA_dev || !it.LB_dev || !it.V_dev || !it.codes_dev || !it.scales_dev)
            return BAKRON_ERR_INVALID_ARG;
        if (!it.ws_dev) return BAKRON_ERR_WORKSPACE;
        if (!aligned16(it.W_dev) || !aligned16(it.LA_dev) || !aligned16(it.LB_dev) || !aligned16(it.V_dev) ||
            !aligned16(it.codes_dev) || !aligned16(it.scales_dev) || !aligned16(it.ws_dev))
            return BAKRON_ERR_ALIGNMENT;
        SolveLayout L;
        L.compute(it.m, it.n, kTile);
        if (it.ws_bytes < L.total) return BAKRON_ERR_WORKSPACE;
    }
    for (int32_t i = 0; i < count; ++i) {
        const bakron_batch_item_t &it = items[i];
        s = bakron_solve(it.W_dev, it.m, it.n, it.LA_dev, it.LB_dev, q, it.V_dev, it.codes_dev, it.scales_dev,
                         it.ws_dev, it.ws_bytes, cfg, streams[i % nstreams]);
        if (s != BAKRON_OK) return s;
    }
    return BAKRON_OK;
}

namespace {
struct GramLayout {
    int64_t Dt, Nt, Dp, Ns;
    size_t status, xt_hi, xt_lo, G, total;
    void compute(int64_t N, int64_t d)
    {
        Dt = (d + kTile - 1) / kTile; Nt = (N + kTile - 1) / kTile;
        Dp = Dt * kTile; Ns = Nt * kTile;
        size_t o = 0;
        auto take = [&](size_t bytes) { size_t at = o; o = align_up(o + bytes); return at; };
        status = take(kStatusBytes);
        xt_hi = take((size_t)Dp * Ns * sizeof(float));
        xt_lo = take((size_t)Dp * Ns * sizeof(float));
        G = take((size_t)Dp * Dp * sizeof(float));
        total = o;
    }
};
}  // namespace

size_t bakron_gram_workspace_size(int64_t N, int64_t d)
{
    if (N < 1 || d < 1 || N > kMaxSide || d > kMaxSide) return 0;
    GramLayout L;
    L.compute(N, d);
    return L.total;
}

bakron_status_t bakron_gram(const float *X_dev, int64_t N, int64_t d, float damping, float *A_dev, void *ws_dev,
                            size_t ws_bytes, bakron_stream_t stream)
{
    if (N < 1 || d < 1 || N > kMaxSide || d > kMaxSide) return BAKRON_ERR_INVALID_ARG;
    if (!X_dev || !A_dev || !(damping >= 0.f) || !isfinite(damping)) return BAKRON_ERR_INVALID_ARG;
    if (!ws_dev) return BAKRON_ERR_WORKSPACE;
    if (!aligned16(X_dev) || !aligned16(A_dev) || !aligned16(ws_dev)) return BAKRON_ERR_ALIGNMENT;
    GramLayout L;
    L.compute(N, d);
    if (ws_bytes < L.total) return BAKRON_ERR_WORKSPACE;
    if (configure_device() != cudaSuccess) return BAKRON_ERR_CUDA;
    cudaStream_t st = (cudaStream_t)stream;
    char *w = (char *)ws_dev;
    DeviceStatus *status = (DeviceStatus *)(w + L.status);
    if (cudaMemsetAsync(status, 0, kStatusBytes, st) != cudaSuccess) return BAKRON_ERR_CUDA;
    float *xt_hi = (float *)(w + L.xt_hi), *xt_lo = (float *)(w + L.xt_lo), *G = (float *)(w + L.G);
    if (launch_gram_prep(X_dev, N, d, L.Dp, L.Ns, xt_hi, xt_lo, status, st) != cudaSuccess) return BAKRON_ERR_CUDA;
    TcMaps maps;
    if (!make_gram_maps(xt_hi, xt_lo, G, L.Dp, L.Ns, &maps)) return BAKRON_ERR_CUDA;
    const NodeParams np{0, 0, 0, (int)L.Dt, (int)L.Nt};
    GemmArgs g{xt_hi, xt_lo, xt_hi, xt_lo, L.Ns, L.Ns, G, nullptr, nullptr, L.Dp, status, 200};
    if (launch_gram_tc(np, g, maps, st) != cudaSuccess) return BAKRON_ERR_CUDA;
    if (launch_gram_finish(G, d, L.Dp, N, damping, A_dev, st) != cudaSuccess) return BAKRON_ERR_CUDA;
    return BAKRON_OK;
}

// Host-buffer variant: staging buffers follow the solve workspace.
namespace {
struct HostLayout {
    size_t solve, W, LA, LB, V, codes, scales, uscales, total;
    void compute(int64_t m, int64_t n, size_t solve_bytes)
    {
        size_t o = 0;
        auto take = [&](size_t bytes) { size_t at = o; o = align_up(o + bytes); return at; };
        solve = take(solve_bytes);
        W = take((size_t)m * n * 4); LA = take((size_t)n * n * 4); LB = take((size_t)m * m * 4);
        V = take((size_t)m * n * 4); codes = take((size_t)m * n); scales = take((size_t)m * 4);
        uscales = take((size_t)m * 4);
        total = o;
    }
};
}  // namespace

size_t bakron_solve_host_workspace_size(int64_t m, int64_t n, const bakron_config_t *cfg)
{
    size_t s = bakron_solve_workspace_size(m, n, cfg);
    if (!s) return 0;
    HostLayout H;
    H.compute(m, n, s);
    return H.total;
}

bakron_status_t bakron_solve_host(const float *W_host, int64_t m, int64_t n, const float *LA_host,
                                  const float *LB_host, const bakron_quantizer_t *q, float *V_host,
                                  int8_t *codes_host, float *scales_host, void *ws_dev,
                                  size_t ws_bytes, const bakron_config_t *cfg,
                                  bakron_stream_t stream)
{
    const bool one_sided = cfg && cfg->b_identity == 1;
    if (!W_host || !LA_host || (!LB_host && !one_sided) || !V_host || !codes_host || !scales_host || !q)
        return BAKRON_ERR_INVALID_ARG;
    size_t sb = bakron_solve_workspace_size(m, n, cfg);
    if (!sb) return BAKRON_ERR_INVALID_ARG;
    if (!ws_dev) return BAKRON_ERR_WORKSPACE;
    if (!aligned16(ws_dev)) return BAKRON_ERR_ALIGNMENT;
    HostLayout H;
    H.compute(m, n, sb);
    if (ws_bytes < H.total) return BAKRON_ERR_WORKSPACE;
    cudaStream_t s = (cudaStream_t)stream;
    char *w = (char *)ws_dev;
    auto h2d = [&](size_t off, const void *src, size_t bytes) {
        return cudaMemcpyAsync(w + off, src, bytes, cudaMemcpyHostToDevice, s) == cudaSuccess;
    };
    if (!h2d(H.W, W_host, (size_t)m * n * 4) || !h2d(H.LA, LA_host, (size_t)n * n * 4) ||
        (!one_sided && !h2d(H.LB, LB_host, (size_t)m * m * 4)))
        return BAKRON_ERR_CUDA;
    bakron_quantizer_t qd = *q;
    if (q->row_scale) {
        if (!h2d(H.uscales, q->row_scale, (size_t)m * 4)) return BAKRON_ERR_CUDA;
        qd.row_scale = (const float *)(w + H.uscales);
    }
    if (one_sided) {
        // rows are final only at the end of the column-block recursion
        bakron_status_t r = solve_device((const float *)(w + H.W), m, n, (const float *)(w + H.LA),
                                         (const float *)(w + H.LB), &qd, (float *)(w + H.V),
                                         (int8_t *)(w + H.codes), (float *)(w + H.scales), w + H.solve, sb,
                                         cfg, s, true);
        if (r != BAKRON_OK) return r;
        if (cudaMemcpyAsync(V_host, w + H.V, (size_t)m * n * 4, cudaMemcpyDeviceToHost, s) != cudaSuccess ||
            cudaMemcpyAsync(codes_host, w + H.codes, (size_t)m * n, cudaMemcpyDeviceToHost, s) != cudaSuccess ||
            cudaMemcpyAsync(scales_host, w + H.scales, (size_t)m * 4, cudaMemcpyDeviceToHost, s) != cudaSuccess)
            return BAKRON_ERR_CUDA;
        return BAKRON_OK;
    }
    // two-sided: row blocks stream back during the solve (direct launches)
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return BAKRON_ERR_CUDA;
    thread_local cudaStream_t copy_stream[64] = {};
    thread_local cudaEvent_t copy_event[64] = {};
    if (!copy_stream[dev] && cudaStreamCreateWithFlags(&copy_stream[dev], cudaStreamNonBlocking) != cudaSuccess)
        return BAKRON_ERR_CUDA;
    if (!copy_event[dev] && cudaEventCreateWithFlags(&copy_event[dev], cudaEventDisableTiming) != cudaSuccess)
        return BAKRON_ERR_CUDA;
    RowCopy rc;
    rc.cs = copy_stream[dev];
    rc.ev = copy_event[dev];
    rc.V_host = V_host;
    rc.codes_host = codes_host;
    rc.V_dev = (const float *)(w + H.V);
    rc.codes_dev = (const int8_t *)(w + H.codes);
    rc.m = m;
    rc.n = n;
    rc.Mt = (int)((m + kTile - 1) / kTile);
    rc.Nt = (int)((n + kTile - 1) / kTile);
    t_rowcopy = &rc;
    bakron_status_t r = solve_device((const float *)(w + H.W), m, n, (const float *)(w + H.LA),
                                     (const float *)(w + H.LB), &qd, (float *)(w + H.V),
                                     (int8_t *)(w + H.codes), (float *)(w + H.scales), w + H.solve, sb,
                                     cfg, s, true, true);
    t_rowcopy = nullptr;
    // whatever was issued, `s` ends after the copy stream's work: the rows not
    // yet copied and the steps follow the last kernel
    rc.upto_diagonal(rc.Mt + rc.Nt - 2, s);
    const bool ok = !rc.failed && r == BAKRON_OK &&
                    cudaMemcpyAsync(scales_host, w + H.scales, (size_t)m * 4, cudaMemcpyDeviceToHost, rc.cs) ==
                        cudaSuccess;
    if (cudaEventRecord(rc.ev, rc.cs) != cudaSuccess || cudaStreamWaitEvent(s, rc.ev, 0) != cudaSuccess)
        return BAKRON_ERR_CUDA;
    if (r != BAKRON_OK) return r;
    return ok ? BAKRON_OK : BAKRON_ERR_CUDA;
}

size_t bakron_factor_workspace_size(int64_t n, int64_t m)
{
    if (n < 0 || m < 0 || (n == 0 && m == 0)) return 0;
    int64_t d = std::max(n, m);
    return align_up(kStatusBytes) + align_up(factor_work_doubles(d) * sizeof(double));
}

bakron_status_t bakron_factor(const float *A_dev, int64_t n, const float *B_dev, int64_t m,
                              float *LA_dev, float *LB_dev, void *ws_dev, size_t ws_bytes,
                              bakron_stream_t stream)
{
    if (n < 0 || m < 0 || (n == 0 && m == 0) || n > kMaxSide || m > kMaxSide) return BAKRON_ERR_INVALID_ARG;
    if ((n > 0 && (!A_dev || !LA_dev)) || (m > 0 && (!B_dev || !LB_dev))) return BAKRON_ERR_INVALID_ARG;
    if (!ws_dev) return BAKRON_ERR_WORKSPACE;
    if ((n > 0 && (!aligned16(A_dev) || !aligned16(LA_dev))) ||
        (m > 0 && (!aligned16(B_dev) || !aligned16(LB_dev))) || !aligned16(ws_dev))
        return BAKRON_ERR_ALIGNMENT;
    if (ws_bytes < bakron_factor_workspace_size(n, m)) return BAKRON_ERR_WORKSPACE;
    char *w = (char *)ws_dev;
    DeviceStatus *st = (DeviceStatus *)w;
    double *work = (double *)(w + align_up(kStatusBytes));
    cudaStream_t s = (cudaStream_t)stream;
    if (cudaMemsetAsync(st, 0, kStatusBytes, s) != cudaSuccess) return BAKRON_ERR_CUDA;
    if (n > 0 && launch_factor(A_dev, n, LA_dev, work, st, s) != cudaSuccess) return BAKRON_ERR_CUDA;
    if (m > 0 && launch_factor(B_dev, m, LB_dev, work, st, s) != cudaSuccess) return BAKRON_ERR_CUDA;
    return BAKRON_OK;
}

size_t bakron_proxy_loss_workspace_size(int64_t m, int64_t n)
{
    if (m < 1 || n < 1 || m > kMaxSide || n > kMaxSide) return 0;
    ProxyLayout L;
    L.compute(m, n);
    return L.total;
}

bakron_status_t bakron_proxy_loss(const float *W_dev, const float *V_dev, const float *A_dev,
                                  const float *B_dev, int64_t m, int64_t n, double *out_dev,
                                  double *out_host, void *ws_dev, size_t ws_bytes,
                                  bakron_stream_t stream)
{
    if (m < 1 || n < 1 || m > kMaxSide || n > kMaxSide) return BAKRON_ERR_INVALID_ARG;
    if (!W_dev || !V_dev || !A_dev || !B_dev || !out_dev) return BAKRON_ERR_INVALID_ARG;
    if (!ws_dev || ws_bytes < bakron_proxy_loss_workspace_size(m, n)) return BAKRON_ERR_WORKSPACE;
    if (!aligned16(W_dev) || !aligned16(V_dev) || !aligned16(A_dev) || !aligned16(B_dev) ||
        ((uintptr_t)ws_dev & (kAlign - 1)) || ((uintptr_t)out_dev & 7u))
        return BAKRON_ERR_ALIGNMENT;
    if (configure_device() != cudaSuccess) return BAKRON_ERR_CUDA;
    cudaStream_t s = (cudaStream_t)stream;
    ProxyLayout L;
    L.compute(m, n);
    if (cudaMemsetAsync(ws_dev, 0, kStatusBytes, s) != cudaSuccess) return BAKRON_ERR_CUDA;
    if (launch_proxy_loss(W_dev, V_dev, A_dev, B_dev, L, (char *)ws_dev, out_dev, s) != cudaSuccess)
        return BAKRON_ERR_CUDA;
    if (out_host) {
        if (cudaMemcpyAsync(out_host, out_dev, sizeof(double), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
            cudaStreamSynchronize(s) != cudaSuccess)
            return BAKRON_ERR_CUDA;
    }
    return BAKRON_OK;
}

bakron_status_t bakron_selftest_wait_timeout(int32_t timeout_ms, void *ws_dev, size_t ws_bytes,
                                             bakron_stream_t stream)
{
    if (timeout_ms < 1 || timeout_ms > 10000) return BAKRON_ERR_INVALID_ARG;
    if (!ws_dev || ws_bytes < kStatusBytes) return BAKRON_ERR_WORKSPACE;
    if (!aligned16(ws_dev)) return BAKRON_ERR_ALIGNMENT;
    cudaStream_t s = (cudaStream_t)stream;
    if (cudaMemsetAsync(ws_dev, 0, kStatusBytes, s) != cudaSuccess) return BAKRON_ERR_CUDA;
    if (launch_wait_timeout_selftest((DeviceStatus *)ws_dev, timeout_ms, s) != cudaSuccess) return BAKRON_ERR_CUDA;
    return BAKRON_OK;
}

size_t bakron_selftest_band_abort_workspace_size(void) { return align_up(kStatusBytes) + kBandAbortBufBytes; }

bakron_status_t bakron_selftest_band_abort(int32_t timeout_ms, void *ws_dev, size_t ws_bytes, bakron_stream_t stream)
{
    if (timeout_ms < 1 || timeout_ms > 10000) return BAKRON_ERR_INVALID_ARG;
    if (!ws_dev || ws_bytes < bakron_selftest_band_abort_workspace_size()) return BAKRON_ERR_WORKSPACE;
    if (!aligned16(ws_dev)) return BAKRON_ERR_ALIGNMENT;
    if (configure_device() != cudaSuccess) return BAKRON_ERR_CUDA;
    cudaStream_t s = (cudaStream_t)stream;
    char *w = (char *)ws_dev;
    if (cudaMemsetAsync(w, 0, kStatusBytes, s) != cudaSuccess) return BAKRON_ERR_CUDA;
    if (launch_band_abort_selftest((DeviceStatus *)w, (float *)(w + align_up(kStatusBytes)), timeout_ms, s) !=
        cudaSuccess)
        return BAKRON_ERR_CUDA;
    return BAKRON_OK;
}

bakron_status_t bakron_get_status(void *ws_dev, size_t ws_bytes, bakron_stream_t stream)
{
    if (!ws_dev || ws_bytes < kStatusBytes) return BAKRON_ERR_WORKSPACE;
    cudaStream_t s = (cudaStream_t)stream;
    if (cudaStreamSynchronize(s) != cudaSuccess) return BAKRON_ERR_CUDA;
    DeviceStatus h;
    if (cudaMemcpy(&h, ws_dev, sizeof(h), cudaMemcpyDeviceToHost) != cudaSuccess) return BAKRON_ERR_CUDA;
    if (h.code != 0 && cudaMemset(ws_dev, 0, sizeof(h)) != cudaSuccess) return BAKRON_ERR_CUDA;
    return (bakron_status_t)h.code;
}

int64_t bakron_get_profile_launches(bakron_profile_launch_t *out, int64_t cap)
{
    const int64_t n = (int64_t)t_last_launches.size();
    if (out)
        for (int64_t i = 0; i < n && i < cap; ++i) out[i] = t_last_launches[(size_t)i];
    return n;
}

bakron_status_t bakron_get_profile(bakron_profile_t *out)
{
    if (!out) return BAKRON_ERR_INVALID_ARG;
    *out = t_last_profile;
    return BAKRON_OK;
}

bakron_status_t bakron_plan_stats(int64_t m, int64_t n, const bakron_config_t *cfg, bakron_plan_stats_t *out)
{
    Config conf;
    if (!out || m < 1 || n < 1 || m > kMaxSide || n > kMaxSide) return BAKRON_ERR_INVALID_ARG;
    if (read_config(cfg, conf) != BAKRON_OK) return BAKRON_ERR_INVALID_ARG;
    std::memset(out, 0, sizeof(*out));
    out->tiles_m = (m + kTile - 1) / kTile;
    out->tiles_n = (n + kTile - 1) / kTile;
    out->tile_diagonals = out->tiles_m + out->tiles_n - 1;
    if (conf.b_identity)
        count_schedule_gptq(0, (int)out->tiles_n, (int)out->tiles_m, (int)out->tiles_n, out);
    else
        count_schedule(0, (int)out->tile_diagonals, (int)out->tiles_m, (int)out->tiles_n, out,
                       conf.leaf == kPairVariant);
    out->update_flops = out->stage1_flops + out->stage2_flops;
    return BAKRON_OK;
}

}  // extern "C"
