// k_state_passing.cu -- ssd_state_passing: the sequential inter-chunk recurrence.
//
//   s_in[0]   = h0 (or 0)
//   s_in[c+1] = alpha_c * s_in[c] + S_c          for c = 0 .. nc-1
//   final     = s_in[nc]
//
// the "inter-chunk recurrence (state hand-off)" of the chunked SSD algorithm
// (aifetchly blog "Mamba-2 Architecture", "The Chunked SSD Algorithm", step 2:
// h_k = a_k h_{k-1} + h_chunk,k), with a_k the whole-chunk decay alpha_c.
//
// Every element of the P x N state is an independent scalar recurrence, so the
// kernel is parallel over (b, h, element) and sequential only over chunks.
// Each thread owns 8 consecutive elements; the loads of S_c do not depend on
// the running state, so they are issued several chunks ahead and the loop is
// bound by HBM bandwidth rather than by latency.  The running sum stays fp32
// in registers; s_in is stored as fp32 or bf16 (the tensor-core scan consumes
// bf16).
#include "common.cuh"
#include "kernels.h"
#include "tma_host.h"

namespace ssd {

namespace {

constexpr int kThreads = 256;
constexpr int kVec = 8;  // state elements per thread (one 16-byte bf16 load)

// kVec consecutive fp32 values in registers
struct V8 {
    float v[kVec];
};

__device__ __forceinline__ void load8(const float *p, V8 &o) {
    const float4 a = __ldcs(reinterpret_cast<const float4 *>(p));
    const float4 b = __ldcs(reinterpret_cast<const float4 *>(p) + 1);
    o.v[0] = a.x; o.v[1] = a.y; o.v[2] = a.z; o.v[3] = a.w;
    o.v[4] = b.x; o.v[5] = b.y; o.v[6] = b.z; o.v[7] = b.w;
}
__device__ __forceinline__ void load8(const __nv_bfloat16 *p, V8 &o) {
    const uint4 u = __ldcs(reinterpret_cast<const uint4 *>(p));
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        o.v[2 * i] = __uint_as_float(w[i] << 16);
        o.v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
}
__device__ __forceinline__ void store8(float *p, const V8 &s) {
    reinterpret_cast<float4 *>(p)[0] = make_float4(s.v[0], s.v[1], s.v[2], s.v[3]);
    reinterpret_cast<float4 *>(p)[1] = make_float4(s.v[4], s.v[5], s.v[6], s.v[7]);
}
__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
    __nv_bfloat162 t = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&t);
}
__device__ __forceinline__ void store8(__nv_bfloat16 *p, const V8 &s) {
    *reinterpret_cast<uint4 *>(p) = make_uint4(pack2(s.v[0], s.v[1]), pack2(s.v[2], s.v[3]),
                                               pack2(s.v[4], s.v[5]), pack2(s.v[6], s.v[7]));
}

// Scalar fallback for state sizes that are not a multiple of kVec.
template <typename ST, typename SinT>
__global__ void __launch_bounds__(kThreads)
state_passing_scalar_kernel(Dims d, const ST *__restrict__ states, const float *__restrict__ alpha,
                            const float *__restrict__ h0, SinT *__restrict__ s_in,
                            float *__restrict__ final_state) {
    const int64_t PN = int64_t(d.P) * d.N;
    const int64_t e = int64_t(blockIdx.x) * kThreads + threadIdx.x;
    const int bh = blockIdx.y;
    const int b = bh / d.H, h = bh % d.H;
    if (e >= PN) return;
    float cur = h0 ? h0[int64_t(bh) * PN + e] : 0.f;
    const float *al = alpha + off_alpha(d, b, h, 0);
    for (int c = 0; c < d.nc; ++c) {
        const float sc = to_f32(states[off_state(d, b, c, h) + e]);
        s_in[off_state(d, b, c, h) + e] = from_f32<SinT>(cur);
        cur = fmaf(__ldg(al + c), cur, sc);
    }
    if (final_state) final_state[int64_t(bh) * PN + e] = cur;
}

// kPrefetch chunks are loaded ahead: 4 with three CTAs per SM when the grid
// fills the GPU, 16 with one CTA per SM when it does not (few (b, h) chains,
// long sequences), so that enough bytes are in flight either way.
template <typename ST, typename SinT, int kPrefetch, int kMinBlocks>
__global__ void __launch_bounds__(kThreads, kMinBlocks)
state_passing_kernel(Dims d, const ST *__restrict__ states, const float *__restrict__ alpha,
                     const float *__restrict__ h0, SinT *__restrict__ s_in,
                     float *__restrict__ final_state) {
    const int64_t PN = int64_t(d.P) * d.N;
    const int64_t e = (int64_t(blockIdx.x) * kThreads + threadIdx.x) * kVec;
    const int bh = blockIdx.y;
    const int b = bh / d.H, h = bh % d.H;
    if (e >= PN) return;
    V8 cur;
    if (h0) load8(h0 + int64_t(bh) * PN + e, cur);
    else
#pragma unroll
        for (int i = 0; i < kVec; ++i) cur.v[i] = 0.f;
    const float *al = alpha + off_alpha(d, b, h, 0);
    const int64_t cstride = int64_t(d.H) * PN;  // elements between consecutive chunks
    const ST *sp = states + off_state(d, b, 0, h) + e;
    SinT *op = s_in + off_state(d, b, 0, h) + e;
    for (int c0 = 0; c0 < d.nc; c0 += kPrefetch) {
        V8 buf[kPrefetch];
        float a[kPrefetch];
#pragma unroll
        for (int k = 0; k < kPrefetch; ++k) {
            if (c0 + k < d.nc) {
                load8(sp + k * cstride, buf[k]);
                a[k] = __ldg(al + c0 + k);
            }
        }
#pragma unroll
        for (int k = 0; k < kPrefetch; ++k) {
            if (c0 + k < d.nc) {
                store8(op + k * cstride, cur);
#pragma unroll
                for (int i = 0; i < kVec; ++i) cur.v[i] = fmaf(a[k], cur.v[i], buf[k].v[i]);
            }
        }
        sp += kPrefetch * cstride;
        op += kPrefetch * cstride;
    }
    if (final_state) store8(final_state + int64_t(bh) * PN + e, cur);
}

template <typename ST, typename SinT>
cudaError_t launch_sp(const Dims &d, const ST *states, const float *alpha, const float *h0,
                      SinT *s_in, float *final_state, cudaStream_t stream) {
    const int64_t PN = int64_t(d.P) * d.N;
    if (PN % kVec == 0) {
        dim3 grid(unsigned((PN / kVec + kThreads - 1) / kThreads), unsigned(d.B * d.H));
        const int64_t threads = int64_t(grid.x) * grid.y * kThreads;
        if (threads >= int64_t(device_sm_count()) * 3 * kThreads)
            state_passing_kernel<ST, SinT, 4, 3><<<grid, kThreads, 0, stream>>>(
                d, states, alpha, h0, s_in, final_state);
        else
            state_passing_kernel<ST, SinT, 16, 1><<<grid, kThreads, 0, stream>>>(
                d, states, alpha, h0, s_in, final_state);
    } else {
        dim3 grid(unsigned((PN + kThreads - 1) / kThreads), unsigned(d.B * d.H));
        state_passing_scalar_kernel<ST, SinT><<<grid, kThreads, 0, stream>>>(d, states, alpha, h0,
                                                                             s_in, final_state);
    }
    return cudaGetLastError();
}

template <typename ST>
cudaError_t dispatch_out(const Dims &d, const ST *states, const float *alpha, const float *h0,
                         void *s_in, bool s_in_bf16, float *final_state, cudaStream_t stream) {
    if (s_in_bf16)
        return launch_sp(d, states, alpha, h0, static_cast<__nv_bfloat16 *>(s_in), final_state, stream);
    return launch_sp(d, states, alpha, h0, static_cast<float *>(s_in), final_state, stream);
}

}  // namespace

cudaError_t launch_state_passing(const Dims &d, const void *states, bool states_bf16,
                                 const float *alpha, const float *init_state, void *s_in,
                                 bool s_in_bf16, float *final_state, cudaStream_t stream) {
    if (states_bf16)
        return dispatch_out(d, static_cast<const __nv_bfloat16 *>(states), alpha, init_state, s_in,
                            s_in_bf16, final_state, stream);
    return dispatch_out(d, static_cast<const float *>(states), alpha, init_state, s_in, s_in_bf16,
                        final_state, stream);
}

}  // namespace ssd
