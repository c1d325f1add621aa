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
// Each thread owns VEC consecutive elements; the loads of S_c do not depend on
// the running state, so they are issued kPrefetch chunks ahead and the loop is
// bound by HBM bandwidth rather than by latency.  The running sum stays fp32
// in registers; s_in is stored as fp32 or bf16 (the tensor-core scan consumes
// bf16).
#include "common.cuh"
#include "kernels.h"

namespace ssd {

namespace {

constexpr int kThreads = 256;
constexpr int kPrefetch = 8;

template <int VEC> struct VecF;
template <> struct VecF<4> { using T = float4; };
template <> struct VecF<1> { using T = float; };

__device__ __forceinline__ void fma_vec(float4 &s, float a, const float4 &v) {
    s.x = fmaf(a, s.x, v.x); s.y = fmaf(a, s.y, v.y);
    s.z = fmaf(a, s.z, v.z); s.w = fmaf(a, s.w, v.w);
}
__device__ __forceinline__ void fma_vec(float &s, float a, const float &v) { s = fmaf(a, s, v); }

__device__ __forceinline__ void store_vec(float *p, const float4 &v) {
    *reinterpret_cast<float4 *>(p) = v;
}
__device__ __forceinline__ void store_vec(float *p, const float &v) { *p = v; }
__device__ __forceinline__ void store_vec(__nv_bfloat16 *p, const float4 &v) {
    __nv_bfloat162 lo = __floats2bfloat162_rn(v.x, v.y);
    __nv_bfloat162 hi = __floats2bfloat162_rn(v.z, v.w);
    uint2 u;
    u.x = *reinterpret_cast<uint32_t *>(&lo);
    u.y = *reinterpret_cast<uint32_t *>(&hi);
    *reinterpret_cast<uint2 *>(p) = u;
}
__device__ __forceinline__ void store_vec(__nv_bfloat16 *p, const float &v) {
    *p = __float2bfloat16_rn(v);
}

__device__ __forceinline__ float4 load_vec(const float4 *p) { return __ldcs(p); }
__device__ __forceinline__ float load_vec(const float *p) { return __ldcs(p); }
__device__ __forceinline__ void zero(float4 &v) { v = make_float4(0.f, 0.f, 0.f, 0.f); }
__device__ __forceinline__ void zero(float &v) { v = 0.f; }

template <int VEC, typename SinT>
__global__ void __launch_bounds__(kThreads)
state_passing_kernel(Dims d, const float *__restrict__ states, const float *__restrict__ alpha,
                     const float *__restrict__ h0, SinT *__restrict__ s_in,
                     float *__restrict__ final_state) {
    using V = typename VecF<VEC>::T;
    const int64_t PN = int64_t(d.P) * d.N;
    const int64_t e = (int64_t(blockIdx.x) * kThreads + threadIdx.x) * VEC;
    const int bh = blockIdx.y;
    const int b = bh / d.H, h = bh % d.H;
    if (e >= PN) return;
    V cur;
    if (h0) cur = *reinterpret_cast<const V *>(h0 + int64_t(bh) * PN + e);
    else zero(cur);
    const float *al = alpha + off_alpha(d, b, h, 0);
    for (int c0 = 0; c0 < d.nc; c0 += kPrefetch) {
        V buf[kPrefetch];
        float a[kPrefetch];
#pragma unroll
        for (int k = 0; k < kPrefetch; ++k) {
            if (c0 + k < d.nc) {
                buf[k] = load_vec(reinterpret_cast<const V *>(states + off_state(d, b, c0 + k, h) + e));
                a[k] = __ldg(al + c0 + k);
            }
        }
#pragma unroll
        for (int k = 0; k < kPrefetch; ++k) {
            if (c0 + k < d.nc) {
                store_vec(s_in + off_state(d, b, c0 + k, h) + e, cur);
                fma_vec(cur, a[k], buf[k]);
            }
        }
    }
    if (final_state) store_vec(final_state + int64_t(bh) * PN + e, cur);
}

template <int VEC, typename SinT>
cudaError_t launch_sp(const Dims &d, const float *states, const float *alpha, const float *h0,
                      SinT *s_in, float *final_state, cudaStream_t stream) {
    const int64_t PN = int64_t(d.P) * d.N;
    dim3 grid(unsigned((PN / VEC + kThreads - 1) / kThreads), unsigned(d.B * d.H));
    state_passing_kernel<VEC, SinT><<<grid, kThreads, 0, stream>>>(d, states, alpha, h0, s_in,
                                                                  final_state);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_state_passing(const Dims &d, const float *states, const float *alpha,
                                 const float *init_state, void *s_in, bool s_in_bf16,
                                 float *final_state, cudaStream_t stream) {
    const bool vec4 = ((int64_t(d.P) * d.N) % 4) == 0;
    if (s_in_bf16) {
        auto *p = static_cast<__nv_bfloat16 *>(s_in);
        return vec4 ? launch_sp<4>(d, states, alpha, init_state, p, final_state, stream)
                    : launch_sp<1>(d, states, alpha, init_state, p, final_state, stream);
    }
    auto *p = static_cast<float *>(s_in);
    return vec4 ? launch_sp<4>(d, states, alpha, init_state, p, final_state, stream)
                : launch_sp<1>(d, states, alpha, init_state, p, final_state, stream);
}

}  // namespace ssd
