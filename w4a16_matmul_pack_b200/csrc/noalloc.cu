// noalloc.cu -- w4a16_gemv_noalloc: the decode GEMV for callers that cannot
// allocate device memory themselves.
//
// Some callers run inside a host framework that owns every device allocation
// (an inference engine's plugin interface, an embedded runtime with a fixed
// memory budget, a C program that only ever receives input and output
// buffers).  They can hand the GEMV its x and y, but they cannot provide the
// split-K scratch that w4a16_gemv takes as `workspace`.  This entry point
// supplies that scratch from a file-scope device array instead, so the call
// allocates nothing.
//
// The array is part of the library image: every GPU that loads the library
// holds W4_NOALLOC_SCRATCH_BYTES of it until the process exits.  All calls on a
// device share the one array, so calls whose work overlaps on that GPU (two
// streams, or two host threads) race on it and must be serialised by the
// caller.  The GEMV writes every scratch word it later reads within the same
// call, so nothing in the array has to start at zero and stale contents from an
// earlier call are never read.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/w4a16.h"

namespace {

__device__ __align__(256) unsigned char g_noalloc_scratch[W4_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
void *g_scratch_addr[kMaxDevices];
std::mutex g_scratch_mu;

// Device address of g_noalloc_scratch on the current device.  In host code the
// symbol itself is only a host-side stand-in, so the address is queried once
// per device (with that device current) and cached.
w4_status scratch_address(void **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return W4_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_scratch_mu);
    if (!g_scratch_addr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return W4_ERR_CUDA;
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return W4_OK;
}

}  // namespace

extern "C" w4_status w4a16_gemv_noalloc(const w4_weights *w, const void *x, int M, float *y, void *stream) {
    const size_t need = w4a16_workspace_bytes(w, M);
    if (need > (size_t)W4_NOALLOC_SCRATCH_BYTES) return W4_ERR_WORKSPACE;
    void *scratch = nullptr;
    const w4_status s = scratch_address(&scratch);
    if (s != W4_OK) return s;
    return w4a16_gemv(w, x, M, y, scratch, (size_t)W4_NOALLOC_SCRATCH_BYTES, stream);
}
