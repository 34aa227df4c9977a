// gdn_chunk_fwd_noalloc: the chunkwise forward for callers that cannot allocate
// device memory.  Some callers cannot call cudaMalloc at the point where they
// run the layer: engines that plan every buffer once at start-up and forbid
// allocation afterwards, code paths where cudaMalloc's implicit device-wide
// synchronisation is not acceptable, and hosts that own the device's memory
// and hand the library none.  For them the workspace lives in a fixed array
// compiled into this library instead of a buffer they pass in.
//
// The array is a file-scope __device__ array of kScratchBytes (8 MiB); every
// GPU that loads the library holds it until the process exits.  Its device
// address is looked up once per device (the first call on that device, with
// that device current), so that first call must come before any stream capture.
// All calls share the one array and it keeps the last call's contents.  The
// two paths that use it write their scratch before reading it (the CUDA-core
// path's per-chunk T, P and gate sums; the tcgen05 path's [T'; T''] tiles, and
// with the prologue flags off there is nothing else), so nothing needs
// clearing; calls whose work overlaps on the GPU (different streams, or
// threads) race on it and must be serialised by the caller.  The address is
// cached for the life of the process: after a cudaDeviceReset the cached value
// is stale, and the entry point must not be used on that device again.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/gdn.h"

namespace {

constexpr size_t kScratchBytes = size_t(8) << 20;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

void *g_scratch_addr[kMaxDevices];
std::mutex g_scratch_mu;

// Device address of g_noalloc_scratch on the current device.
cudaError_t scratch_address(void **out) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
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

extern "C" gdn_status_t gdn_chunk_fwd_noalloc(const void *q, const void *k, const void *v,
                                              const float *log_alpha, const float *beta,
                                              const float *S0, void *o, float *S_T, int B, int T,
                                              int H, int Dk, int Dv, int chunk,
                                              gdn_dtype_t dtype, void *stream) {
    // 0 for invalid sizes too: gdn_chunk_fwd then reports the exact error.
    const size_t need = gdn_chunk_fwd_workspace_size(B, T, H, Dk, Dv, chunk, dtype);
    if (need > kScratchBytes) return GDN_ERR_UNSUPPORTED;
    void *ws = nullptr;
    if (need > 0 && scratch_address(&ws) != cudaSuccess) return GDN_ERR_CUDA;
    return gdn_chunk_fwd(q, k, v, log_alpha, beta, S0, o, S_T, B, T, H, Dk, Dv, chunk, dtype, ws,
                         need > 0 ? kScratchBytes : 0, stream);
}
