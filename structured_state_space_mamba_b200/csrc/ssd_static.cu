// ssd_static.cu -- ssd_forward_static: the forward scan on a fixed, statically
// sized device scratch area, with no allocation of any kind.
//
// Who needs it: callers that cannot provide a workspace and must not allocate.
// Examples are code whose device memory is entirely held by another allocator
// (a framework's caching pool that leaves no room for cudaMallocAsync), and
// latency-critical loops where a cudaMalloc, with its implicit device-wide
// synchronisation, or a pool growth is not acceptable.
//
// How: one file-scope __device__ array of SSD_STATIC_SCRATCH_BYTES per device,
// placed in its own translation unit so that, under lazy module loading, only
// the callers of this entry point pay for it.  Its device address is looked up
// with cudaGetSymbolAddress once per device, on the first call on that device
// (set-up), and cached; that first call must therefore come before any stream
// capture on the device.  The call then runs exactly the ssd_forward_ws path on
// that scratch area.
//
// Nothing in the scratch needs to start at zero: every byte the kernels read
// there is written earlier in the same call.  All calls on one device share the
// one scratch area, so two calls that overlap in time (different streams, or
// different host threads without ordering) race on it; calls issued in order on
// one stream do not.
#include <cuda_runtime.h>

#include <mutex>

#include "ssd.h"

namespace {

constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_ssd_static_scratch[SSD_STATIC_SCRATCH_BYTES];

std::mutex g_setup_mu;
void *g_scratch_ptr[kMaxDevices] = {};

// Device address of this device's scratch array, or nullptr on a CUDA error.
void *static_scratch(int dev) {
    std::lock_guard<std::mutex> lock(g_setup_mu);
    if (!g_scratch_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_ssd_static_scratch) != cudaSuccess) {
            cudaGetLastError();
            return nullptr;
        }
        g_scratch_ptr[dev] = p;
    }
    return g_scratch_ptr[dev];
}

}  // namespace

extern "C" {

ssd_status_t ssd_forward_static(const ssd_dims_t *dims, const void *x, const float *dt,
                                const float *A, const void *Bm, const void *Cm, const float *D,
                                int chunk_len, const float *init_state, void *y_out,
                                float *final_state_out, void *stream) {
    // sizes first: a workload too large for the scratch is refused before any
    // CUDA call
    ssd_workspace_layout_t lay;
    ssd_status_t s = ssd_workspace_layout(dims, chunk_len, &lay);
    if (s != SSD_OK) return s;
    if (lay.total_bytes > SSD_STATIC_SCRATCH_BYTES) return SSD_ERR_WORKSPACE;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return SSD_ERR_CUDA;
    }
    if (dev < 0 || dev >= kMaxDevices) return SSD_ERR_UNSUPPORTED;
    void *ws = static_scratch(dev);
    if (!ws) return SSD_ERR_CUDA;
    return ssd_forward_ws(dims, x, dt, A, Bm, Cm, D, chunk_len, init_state, y_out,
                          final_state_out, ws, SSD_STATIC_SCRATCH_BYTES, stream);
}

}  // extern "C"
