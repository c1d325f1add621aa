// ssd_api.cu -- the C ABI of libssd.so (declared in include/ssd.h).
//
// Argument validation, workspace layout and the launch sequence
//   ssd_chunk_cumsum -> ssd_chunk_state -> ssd_state_passing -> ssd_chunk_scan
// of the chunked SSD algorithm (aifetchly blog "Mamba-2 Architecture: State
// Space Duality Explained", "The Chunked SSD Algorithm").  Every error is
// detected before the first launch.
#include <cuda_runtime.h>

#include <cstdlib>
#include <cstring>
#include <mutex>

#include "../../include/ssd.h"
#include "common.cuh"
#include "kernels.h"

// Device word set by tensor-core kernels whose bounded waits expired.
__device__ unsigned int g_ssd_device_error;

namespace {

using ssd::Dims;

constexpr int kMaxDevices = 64;
unsigned int *g_err_ptr[kMaxDevices];  // per-device address of g_ssd_device_error
std::once_flag g_err_once[kMaxDevices];

// Address of the error word on the current device (NULL if unavailable).
unsigned int *device_error_word() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        cudaGetLastError();
        return nullptr;
    }
    std::call_once(g_err_once[dev], [dev] {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_ssd_device_error) == cudaSuccess)
            g_err_ptr[dev] = static_cast<unsigned int *>(p);
        else
            cudaGetLastError();
    });
    return g_err_ptr[dev];
}

constexpr size_t kAlign = 256;

size_t align_up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }

bool misaligned(const void *p) { return p && (reinterpret_cast<uintptr_t>(p) & 15u); }

constexpr int kB200Sms = 148;

struct Plan {
    Dims d;
    bool bf16;
    bool tc_state;  // tcgen05 chunk state
    bool tc_scan;   // tcgen05 chunk scan (consumes bf16 s_in)
    bool fused;     // chunk_state + state_passing in one kernel (no states buffer)
    bool scan5;     // chunk-wide scan, steep tiles finished by the block-factored scan
    size_t steep_offset;  // scan5: item counter (256 bytes) + packed steep items
    size_t gq_offset;     // scan5: per-token column factors [B,H,nc,chunk_gq(Q)]
    ssd_workspace_layout_t ws;
};

ssd_status_t make_plan(const ssd_dims_t *dims, int chunk_len, Plan *plan) {
    if (!dims || !plan) return SSD_ERR_NULL_ARG;
    const ssd_dims_t &a = *dims;
    if (a.batch <= 0 || a.seqlen <= 0 || a.nheads <= 0 || a.headdim <= 0 || a.dstate <= 0 ||
        a.ngroups <= 0 || a.reserved != 0)
        return SSD_ERR_INVALID_DIM;
    if (a.dtype != SSD_F32 && a.dtype != SSD_BF16) return SSD_ERR_UNSUPPORTED;
    if (a.nheads % a.ngroups != 0) return SSD_ERR_INVALID_DIM;
    if (chunk_len != 32 && chunk_len != 64 && chunk_len != 128 && chunk_len != 256)
        return SSD_ERR_UNSUPPORTED;
    if (a.seqlen % chunk_len != 0) return SSD_ERR_INVALID_DIM;
    if (a.headdim > 256 || a.dstate > 256) return SSD_ERR_UNSUPPORTED;
    if (a.dtype == SSD_BF16 && (a.headdim % 8 != 0 || a.dstate % 8 != 0)) return SSD_ERR_UNSUPPORTED;
    // grid limits (blockIdx.y / .z <= 65535) and 32-bit token indices
    const int64_t nc = a.seqlen / chunk_len;
    if (a.seqlen > (int64_t(1) << 30) || nc > 65535 || a.batch * a.nheads > 65535 ||
        a.batch > 65535 || a.nheads > 65535)
        return SSD_ERR_UNSUPPORTED;

    Dims d;
    d.B = int(a.batch); d.T = int(a.seqlen); d.H = int(a.nheads); d.P = int(a.headdim);
    d.N = int(a.dstate); d.G = int(a.ngroups); d.Q = chunk_len; d.nc = int(nc);
    d.r = d.H / d.G;
    plan->d = d;
    plan->bf16 = a.dtype == SSD_BF16;
    plan->tc_state = plan->bf16 && ssd::tc_chunk_state_supported(d);
    plan->tc_scan = plan->bf16 && ssd::tc_chunk_scan_supported(d);
    // the fused state kernel walks each (b, head pair) over all chunks: used when
    // those units fill most of the GPU's 148 SMs in one wave
    plan->fused = plan->tc_state && plan->tc_scan && ssd::tc_state_fused_supported(d, kB200Sms);
    plan->scan5 = plan->tc_scan && ssd::tc_chunk_scan5_supported(d) && ssd::tc_chunk_scan4_supported(d);

    ssd_workspace_layout_t &w = plan->ws;
    std::memset(&w, 0, sizeof(w));
    const size_t lq = size_t(d.B) * d.H * d.nc * d.Q * sizeof(float);
    const size_t al = size_t(d.B) * d.H * d.nc * sizeof(float);
    const size_t st = size_t(d.B) * d.nc * d.H * d.P * d.N;
    size_t off = 0;
    w.l_offset = off; off = align_up(off + lq);
    w.w_offset = off; off = align_up(off + lq);
    w.dtq_offset = off; off = align_up(off + lq);
    w.beta_offset = off; off = align_up(off + lq);
    w.alpha_offset = off; off = align_up(off + al);
    w.states_offset = off;
    w.states_dtype = plan->tc_state ? SSD_BF16 : SSD_F32;
    if (!plan->fused) off = align_up(off + st * (plan->tc_state ? 2 : 4));
    w.s_in_offset = off;
    w.s_in_dtype = plan->tc_scan ? SSD_BF16 : SSD_F32;
    off = align_up(off + st * (plan->tc_scan ? 2 : 4));
    plan->steep_offset = off;
    if (plan->scan5) off = align_up(off + kAlign + sizeof(long long) * size_t(ssd::chunk_scan5_max_steep(d)));
    plan->gq_offset = off;
    if (plan->scan5) off = align_up(off + al * ssd::chunk_gq(d.Q));
    w.total_bytes = off;
    w.tensor_core = (plan->tc_state || plan->tc_scan) ? 1 : 0;
    w.launches = (plan->fused ? 3 : 4) + (plan->scan5 ? 1 : 0);
    w.fused_state = plan->fused ? 1 : 0;
    return SSD_OK;
}

ssd_status_t check_tensors(const Plan &pl, const void *x, const float *dt, const float *A,
                           const void *Bm, const void *Cm, const float *D,
                           const float *init_state, const void *y, const float *fin) {
    if (!x || !dt || !A || !Bm || !Cm || !y) return SSD_ERR_NULL_ARG;
    const void *ptrs[] = {x, dt, A, Bm, Cm, D, init_state, y, fin};
    for (const void *p : ptrs)
        if (misaligned(p)) return SSD_ERR_MISALIGNED;
    (void)pl;
    return SSD_OK;
}

bool inject_launch_failure() {
    // Host-side fault injection for tests of the error path: with
    // SSD_FAULT_INJECT=launch the call fails as a launch failure would,
    // before anything is launched.
    const char *v = std::getenv("SSD_FAULT_INJECT");
    return v && std::strcmp(v, "launch") == 0;
}

ssd_status_t run(const Plan &pl, const void *x, const float *dt, const float *A, const void *Bm,
                 const void *Cm, const float *D, const float *init_state, void *y,
                 float *fin, char *ws, cudaStream_t stream, int only_stage = -1) {
    if (inject_launch_failure()) return SSD_ERR_CUDA;
    const Dims &d = pl.d;
    unsigned int *err = nullptr;
    if (pl.tc_state || pl.tc_scan) {
        err = device_error_word();
        if (!err) return SSD_ERR_CUDA;
    }
    float *l = reinterpret_cast<float *>(ws + pl.ws.l_offset);
    float *w = reinterpret_cast<float *>(ws + pl.ws.w_offset);
    float *dtq = reinterpret_cast<float *>(ws + pl.ws.dtq_offset);
    float *beta = reinterpret_cast<float *>(ws + pl.ws.beta_offset);
    float *alpha = reinterpret_cast<float *>(ws + pl.ws.alpha_offset);
    void *states = ws + pl.ws.states_offset;
    void *s_in = ws + pl.ws.s_in_offset;
    int *nsteep = reinterpret_cast<int *>(ws + pl.steep_offset);
    long long *steep_items = reinterpret_cast<long long *>(ws + pl.steep_offset + kAlign);
    float *gq = pl.scan5 ? reinterpret_cast<float *>(ws + pl.gq_offset) : nullptr;
    for (int stage = 0; stage < 4; ++stage) {
        if (only_stage >= 0 && stage != only_stage) continue;
        cudaError_t e = cudaSuccess;
        switch (stage) {
            case SSD_STAGE_CHUNK_CUMSUM:
                // also empties the chunk-wide scan's steep-tile list
                e = ssd::launch_chunk_cumsum(d, dt, A, l, w, dtq, beta, alpha, gq,
                                             pl.scan5 ? nsteep : nullptr, stream);
                break;
            case SSD_STAGE_CHUNK_STATE:
                e = pl.fused ? ssd::launch_state_fused(d, x, Bm, w, alpha, init_state, s_in, fin, err, stream)
                    : pl.tc_state ? ssd::launch_chunk_state_tc(d, x, Bm, w, states, err, stream)
                                : ssd::launch_chunk_state_simt(d, pl.bf16, x, Bm, w,
                                                               static_cast<float *>(states), stream);
                break;
            case SSD_STAGE_STATE_PASSING:
                if (pl.fused) break;  // done by the fused chunk_state kernel
                e = ssd::launch_state_passing(d, states, pl.tc_state, alpha, init_state, s_in,
                                              pl.tc_scan, fin, stream);
                break;
            case SSD_STAGE_CHUNK_SCAN:
                if (pl.scan5) {
                    // chunk-wide scan, then the block-factored scan over the tiles
                    // it listed as steep (an empty list costs one short launch)
                    e = ssd::launch_chunk_scan_tc5(d, x, gq, Bm, Cm, D, l, s_in, y, nsteep,
                                                   steep_items, err, stream);
                    if (e == cudaSuccess)
                        e = ssd::launch_chunk_scan_tc4(d, x, dtq, beta, Bm, Cm, D, l, s_in, y,
                                                       steep_items, nsteep,
                                                       ssd::chunk_scan5_max_steep(d), err, stream);
                } else {
                    e = pl.tc_scan
                            ? (ssd::tc_chunk_scan4_supported(d)
                                   ? ssd::launch_chunk_scan_tc4(d, x, dtq, beta, Bm, Cm, D, l, s_in, y,
                                                                nullptr, nullptr, 0, err, stream)
                                   : ssd::launch_chunk_scan_tc(d, x, dt, Bm, Cm, D, l, s_in, y, err, stream))
                            : ssd::launch_chunk_scan_simt(d, pl.bf16, x, dt, Bm, Cm, D, l,
                                                          static_cast<const float *>(s_in), y, stream);
                }
                break;
        }
        if (e != cudaSuccess) return SSD_ERR_CUDA;
    }
    return SSD_OK;
}

}  // namespace

extern "C" {

size_t ssd_workspace_bytes(const ssd_dims_t *dims, int chunk_len) {
    Plan pl;
    if (make_plan(dims, chunk_len, &pl) != SSD_OK) return 0;
    return pl.ws.total_bytes;
}

ssd_status_t ssd_workspace_layout(const ssd_dims_t *dims, int chunk_len,
                                  ssd_workspace_layout_t *out) {
    if (!out) return SSD_ERR_NULL_ARG;
    Plan pl;
    ssd_status_t s = make_plan(dims, chunk_len, &pl);
    if (s != SSD_OK) return s;
    *out = pl.ws;
    return SSD_OK;
}

ssd_status_t ssd_forward_ws(const ssd_dims_t *dims, const void *x, const float *dt,
                            const float *A, const void *Bm, const void *Cm, const float *D,
                            int chunk_len, const float *init_state, void *y_out,
                            float *final_state_out, void *workspace, size_t workspace_bytes,
                            void *stream) {
    Plan pl;
    ssd_status_t s = make_plan(dims, chunk_len, &pl);
    if (s != SSD_OK) return s;
    s = check_tensors(pl, x, dt, A, Bm, Cm, D, init_state, y_out, final_state_out);
    if (s != SSD_OK) return s;
    if (!workspace || workspace_bytes < pl.ws.total_bytes ||
        (reinterpret_cast<uintptr_t>(workspace) & (kAlign - 1)))
        return SSD_ERR_WORKSPACE;
    return run(pl, x, dt, A, Bm, Cm, D, init_state, y_out, final_state_out,
               static_cast<char *>(workspace), static_cast<cudaStream_t>(stream));
}

ssd_status_t ssd_forward_stage(int stage, const ssd_dims_t *dims, const void *x,
                               const float *dt, const float *A, const void *Bm, const void *Cm,
                               const float *D, int chunk_len, const float *init_state,
                               void *y_out, float *final_state_out, void *workspace,
                               size_t workspace_bytes, void *stream) {
    if (stage < 0 || stage > 3) return SSD_ERR_INVALID_DIM;
    Plan pl;
    ssd_status_t s = make_plan(dims, chunk_len, &pl);
    if (s != SSD_OK) return s;
    s = check_tensors(pl, x, dt, A, Bm, Cm, D, init_state, y_out, final_state_out);
    if (s != SSD_OK) return s;
    if (!workspace || workspace_bytes < pl.ws.total_bytes ||
        (reinterpret_cast<uintptr_t>(workspace) & (kAlign - 1)))
        return SSD_ERR_WORKSPACE;
    return run(pl, x, dt, A, Bm, Cm, D, init_state, y_out, final_state_out,
               static_cast<char *>(workspace), static_cast<cudaStream_t>(stream), stage);
}

ssd_status_t ssd_forward(const ssd_dims_t *dims, const void *x, const float *dt, const float *A,
                         const void *Bm, const void *Cm, const float *D, int chunk_len,
                         const float *init_state, void *y_out, float *final_state_out,
                         void *stream) {
    Plan pl;
    ssd_status_t s = make_plan(dims, chunk_len, &pl);
    if (s != SSD_OK) return s;
    s = check_tensors(pl, x, dt, A, Bm, Cm, D, init_state, y_out, final_state_out);
    if (s != SSD_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    void *ws = nullptr;
    if (cudaMallocAsync(&ws, pl.ws.total_bytes, st) != cudaSuccess) {
        cudaGetLastError();
        return SSD_ERR_WORKSPACE;
    }
    s = run(pl, x, dt, A, Bm, Cm, D, init_state, y_out, final_state_out,
            static_cast<char *>(ws), st);
    if (cudaFreeAsync(ws, st) != cudaSuccess && s == SSD_OK) s = SSD_ERR_CUDA;
    return s;
}

const char *ssd_status_string(ssd_status_t status) {
    switch (status) {
        case SSD_OK: return "SSD_OK: success";
        case SSD_ERR_NULL_ARG: return "SSD_ERR_NULL_ARG: a required pointer is NULL";
        case SSD_ERR_INVALID_DIM: return "SSD_ERR_INVALID_DIM: invalid dimensions";
        case SSD_ERR_UNSUPPORTED: return "SSD_ERR_UNSUPPORTED: sizes outside the supported set";
        case SSD_ERR_MISALIGNED: return "SSD_ERR_MISALIGNED: pointer not 16-byte aligned";
        case SSD_ERR_CUDA: return "SSD_ERR_CUDA: CUDA call or kernel launch failed";
        case SSD_ERR_DEVICE_TIMEOUT: return "SSD_ERR_DEVICE_TIMEOUT: device-side wait expired";
        case SSD_ERR_WORKSPACE: return "SSD_ERR_WORKSPACE: workspace missing, too small or unallocatable";
    }
    return "SSD_ERR_UNKNOWN: unknown status code";
}

ssd_status_t ssd_device_status(void *stream) {
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(st) != cudaSuccess) {
        cudaGetLastError();
        return SSD_ERR_CUDA;
    }
    unsigned int *err = device_error_word();
    if (!err) return SSD_ERR_CUDA;
    unsigned int v = 0;
    if (cudaMemcpy(&v, err, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return SSD_ERR_CUDA;
    if (v) {
        const unsigned int zero = 0;
        if (cudaMemcpy(err, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess)
            return SSD_ERR_CUDA;
        return SSD_ERR_DEVICE_TIMEOUT;
    }
    return SSD_OK;
}

const char *ssd_version(void) { return "ssd-b200 0.1.0 sm_100a"; }

}  // extern "C"
