// noalloc.cu -- mi_vs_index_static: the Vertical-Slash index with its scratch
// in a fixed device array instead of a caller-provided workspace.
//
// Some callers cannot hand the library a workspace: an inference server that
// reserves almost all HBM for its KV-cache pool up front and forbids new
// allocations on the request path, or host code on a latency-critical path
// where cudaMalloc's implicit device synchronisation is not acceptable.  This
// entry point computes exactly what mi_vs_index computes (same kernels, same
// results) but keeps its scratch in g_vs_scratch below, a file-scope device
// array of kStaticScratchBytes that every GPU loading the library holds until
// the process exits.  It calls no cudaMalloc, cudaFree or allocating library
// routine.
#include <mutex>

#include "internal.h"

namespace minfer {

namespace {

constexpr size_t kStaticScratchBytes = size_t(16) << 20;  // 16 MiB
constexpr int kMaxDevices = 64;

// The scratch itself.  Host code must not pass `g_vs_scratch` to a kernel:
// in host code that name is only a host-side stand-in; the device address
// comes from cudaGetSymbolAddress below.
__device__ __align__(256) unsigned char g_vs_scratch[kStaticScratchBytes];

std::mutex g_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of g_vs_scratch on the current device.  The first call on a
// device looks it up (cudaGetSymbolAddress, with that device current) and
// caches it; that first call should therefore happen before any stream
// capture on that device.  A device reset (cudaDeviceReset) unloads the
// library's module on that device, so the cached address is no longer the
// array's: after a reset this entry point must not be used in that process.
cudaError_t scratch_address(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_mutex);
    if (!g_scratch_ptr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_vs_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return cudaSuccess;
}

}  // namespace

}  // namespace minfer

using namespace minfer;

extern "C" int mi_vs_index_static(const mi_bf16* q, const mi_bf16* k, int Hq, int Hkv, int N,
                                  int d, float scale, int last_q, int vertical_size,
                                  int slash_size, const int32_t* heads, int n_heads,
                                  int32_t* v_idx, int32_t* s_idx, float* v_score,
                                  float* s_score, void* stream) {
    // Argument checks first, with mi_vs_index's own rules: without a workspace
    // it stops at the workspace check (MI_ERR_WORKSPACE) and launches nothing,
    // or returns the argument error, or MI_OK when there is nothing to do.
    int rc = mi_vs_index(q, k, Hq, Hkv, N, d, scale, last_q, vertical_size, slash_size, heads,
                         n_heads, v_idx, s_idx, v_score, s_score, nullptr, 0, stream);
    if (rc != MI_ERR_WORKSPACE) return rc;
    const size_t need = mi_workspace_bytes(MI_OP_VS_INDEX, Hq, Hkv, N, d, heads ? n_heads : Hq,
                                           last_q, vertical_size, slash_size, 0);
    if (need > kStaticScratchBytes) return MI_ERR_UNSUPPORTED;
    void* scratch = nullptr;
    rc = cuda_status(scratch_address(&scratch));
    if (rc != MI_OK) return rc;
    // Nothing in the scratch has to start at zero: every byte the index
    // kernels read is written earlier in the same call, so whatever the last
    // call left there is harmless.
    rc = mi_vs_index(q, k, Hq, Hkv, N, d, scale, last_q, vertical_size, slash_size, heads,
                     n_heads, v_idx, s_idx, v_score, s_score, scratch, kStaticScratchBytes, stream);
    // The capacity check above and mi_vs_index size the scratch the same way;
    // should they ever disagree, a call that does not fit still reads as one.
    return rc == MI_ERR_WORKSPACE ? MI_ERR_UNSUPPORTED : rc;
}
