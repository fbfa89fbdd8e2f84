// solve_static.cu -- bakron_solve_noalloc: the solve with its workspace in a
// fixed device array that the library owns, for callers that may not
// allocate device memory themselves (see include/bakron.h).
//
// The array is a file-scope __device__ variable.  This file is its own code
// module, and under CUDA's lazy module loading (the default) the driver loads
// the module, and so reserves the array on a device, at the first use of the
// array's address on that device; with CUDA_MODULE_LOADING=EAGER it is
// reserved when the library loads.  It stays reserved until the process
// exits.  Host code cannot use the array's name as a device address: the
// address is looked up once per device with cudaGetSymbolAddress, with that
// device current, and cached.
#include <mutex>

#include "common.cuh"
#include "kernels.cuh"

namespace {

constexpr size_t kScratchBytes = BAKRON_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

std::mutex g_scratch_mu;
void *g_scratch_addr[kMaxDevices] = {};

// Device address of the scratch array on the current device (set-up on the
// first call per device).
cudaError_t scratch_address(void **out)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lk(g_scratch_mu);
    if (!g_scratch_addr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return cudaSuccess;
}

}  // namespace

extern "C" bakron_status_t bakron_solve_noalloc(const float *W_dev, int64_t m, int64_t n,
                                                const float *LA_dev, const float *LB_dev,
                                                const bakron_quantizer_t *q, float *V_dev,
                                                int8_t *codes_dev, float *scales_dev,
                                                const bakron_config_t *cfg, bakron_stream_t stream,
                                                int32_t *device_status_host)
{
    // event-based profiling creates CUDA events; this entry point stays away from it
    if (cfg && cfg->profile) return BAKRON_ERR_INVALID_ARG;
    const size_t need = bakron_solve_workspace_size(m, n, cfg);
    if (need == 0) return BAKRON_ERR_INVALID_ARG;
    if (need > kScratchBytes) return BAKRON_ERR_WORKSPACE;
    cudaStream_t st = (cudaStream_t)stream;
    if (device_status_host) {
        // reading the status back synchronises the stream, which a stream
        // being captured into a graph does not allow
        cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
        if (cudaStreamIsCapturing(st, &cs) != cudaSuccess) return BAKRON_ERR_CUDA;
        if (cs != cudaStreamCaptureStatusNone) return BAKRON_ERR_INVALID_ARG;
    }
    void *ws = nullptr;
    if (scratch_address(&ws) != cudaSuccess) return BAKRON_ERR_CUDA;
    // Direct launches only: the graph mode (cfg->use_graph, BAKRON_GRAPH)
    // creates a stream and executable graphs, which allocate.  The solve
    // clears the status block and rewrites every other part of the workspace
    // it reads (the residual buffers are zeroed by its preparation step), so
    // nothing left by an earlier call leaks into this one.
    bakron_status_t s = bakron::solve_direct(W_dev, m, n, LA_dev, LB_dev, q, V_dev, codes_dev, scales_dev, ws,
                                             kScratchBytes, cfg, st);
    if (s != BAKRON_OK) return s;
    if (device_status_host) {
        int32_t code = 0;
        if (cudaMemcpyAsync(&code, ws, sizeof(code), cudaMemcpyDeviceToHost, st) != cudaSuccess ||
            cudaStreamSynchronize(st) != cudaSuccess)
            return BAKRON_ERR_CUDA;
        *device_status_host = code;
    }
    return BAKRON_OK;
}
