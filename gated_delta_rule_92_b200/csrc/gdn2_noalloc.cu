// gdn2_noalloc.cu -- gdn2_chunk_fwd_host for callers that cannot allocate
// device memory.
//
// gdn2_chunk_fwd_host stages each slice of sequences in a device workspace
// that the caller allocates.  Some callers cannot do that: a plug-in that
// only gets host buffers and a CUDA context it does not own, or a serving
// process whose device memory is all handed out to another allocator at
// start-up and that may not call cudaMalloc afterwards.  For them the
// workspace below is one file-scope device array of fixed size, reserved
// when this file's device code is loaded and kept until the process exits.
// Nothing here calls cudaMalloc, cudaFree or any allocating routine.
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "../../include/gdn2.h"

namespace {

// The staging workspace.  In host code this name stands for the device
// object only symbolically: it is not a device address, and a kernel or copy
// given it would touch the wrong memory (or fault).  Its device address comes
// from cudaGetSymbolAddress, looked up once per device below.
__device__ __align__(256) unsigned char g_noalloc_workspace[GDN2_NOALLOC_WORKSPACE_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_setup_lock;
void *g_workspace_ptr[kMaxDevices] = {};

// Device address of the array on the current device; looked up on the first
// call on that device (with it current) and cached afterwards.
gdn2_status_t workspace_on_current_device(void **ptr) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return GDN2_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return GDN2_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> guard(g_setup_lock);
    if (g_workspace_ptr[dev] == nullptr) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_workspace) != cudaSuccess || p == nullptr) return GDN2_ERR_CUDA;
        g_workspace_ptr[dev] = p;
    }
    *ptr = g_workspace_ptr[dev];
    return GDN2_OK;
}

}  // namespace

extern "C" gdn2_status_t gdn2_chunk_fwd_host_noalloc(const void *q, const void *k, const void *v,
                                                     const void *log_alpha, const void *b, const void *w,
                                                     const float *S0, void *o, float *S_T, int B, int T, int H,
                                                     int d_k, int d_v, int chunk, gdn2_io_t io, void *stream) {
    size_t need = 0;
    gdn2_status_t s = gdn2_chunk_fwd_host_workspace(B, T, H, d_k, d_v, io, &need);
    if (s != GDN2_OK) return s;
    if (need > (size_t)GDN2_NOALLOC_WORKSPACE_BYTES) return GDN2_ERR_UNSUPPORTED;
    void *ws = nullptr;
    if ((s = workspace_on_current_device(&ws)) != GDN2_OK) return s;
    // Every input is copied into the workspace before the kernel reads it, the
    // kernel writes every o row and S_T element it copies back, and a null S0
    // is never read from it: no part of the array has to start at zero, so the
    // previous call's contents are simply overwritten.
    return gdn2_chunk_fwd_host(q, k, v, log_alpha, b, w, S0, o, S_T, B, T, H, d_k, d_v, chunk, io, ws,
                               (size_t)GDN2_NOALLOC_WORKSPACE_BYTES, stream);
}
