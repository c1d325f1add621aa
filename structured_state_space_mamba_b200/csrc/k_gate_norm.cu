// k_gate_norm.cu -- the output side of the Mamba-2 block around the scan: the
// silu gate and RMSNorm over each token's H * P values (aifetchly blog "Mamba-2
// Architecture: State Space Duality Explained", "Step 2: Full Mamba-2 Block
// with Gated Projections": y * silu(z), then RMSNorm over d_inner;
// akillness.github.io "State Space Duality and Mamba-2", the block diagram).
//
// Per token (b, t), over its E = H * P values:
//   g    = y * silu(z)                    (y when there is no gate)
//   rstd = 1 / sqrt(mean(g^2) + eps)
//   out  = g * rstd * w    (apply)   or   g * w    (deferred: the caller applies
//                                         the per-token rstd, e.g. to the rows of
//                                         the next projection's output)
// in place on y.  HBM-bound: one CTA per token reads its y (and z) row once
// from HBM; the second pass over the row finds it in L1 / L2.
#include "common.cuh"
#include "kernels.h"

namespace ssd {

namespace {

constexpr int kThreads = 256;

template <typename T>
__device__ __forceinline__ float gate_value(const T *y, const T *z, int64_t i) {
    const float v = to_f32<T>(y[i]);
    if (!z) return v;
    const float zz = to_f32<T>(z[i]);
    return v * (zz / (1.f + __expf(-zz)));
}

template <typename T>
__global__ void __launch_bounds__(kThreads)
gate_norm_kernel(T *__restrict__ y, const T *__restrict__ z, const float *__restrict__ w, float eps,
                 int apply, int E, float *__restrict__ rstd_out) {
    const int64_t tok = blockIdx.x;
    T *row = y + tok * E;
    const T *zr = z ? z + tok * E : nullptr;
    __shared__ float red[kThreads / 32];
    float rs = 1.f;
    if (w) {
        float ss = 0.f;
        for (int i = threadIdx.x; i < E; i += kThreads) {
            const float g = gate_value<T>(row, zr, i);
            ss = fmaf(g, g, ss);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
        if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
        __syncthreads();
        if (threadIdx.x < 32) {
            float v = threadIdx.x < kThreads / 32 ? red[threadIdx.x] : 0.f;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
            if (threadIdx.x == 0) red[0] = v;
        }
        __syncthreads();
        rs = rsqrtf(red[0] / float(E) + eps);
        if (rstd_out && threadIdx.x == 0) rstd_out[tok] = rs;
    }
    const float scale = (w && apply) ? rs : 1.f;
    for (int i = threadIdx.x; i < E; i += kThreads) {
        float g = gate_value<T>(row, zr, i);
        if (w) g *= scale * __ldg(w + i);
        row[i] = from_f32<T>(g);
    }
}

}  // namespace

cudaError_t launch_gate_norm(const Dims &d, bool bf16, void *y, const void *z, const float *w, float eps,
                             bool apply, float *rstd_out, cudaStream_t stream) {
    const int64_t tokens = int64_t(d.B) * d.T;
    const int E = d.H * d.P;
    if (tokens <= 0 || tokens > 0x7fffffff) return cudaErrorInvalidValue;
    const dim3 grid(static_cast<unsigned>(tokens), 1, 1);
    if (bf16)
        gate_norm_kernel<__nv_bfloat16><<<grid, kThreads, 0, stream>>>(
            static_cast<__nv_bfloat16 *>(y), static_cast<const __nv_bfloat16 *>(z), w, eps, apply ? 1 : 0, E,
            rstd_out);
    else
        gate_norm_kernel<float><<<grid, kThreads, 0, stream>>>(static_cast<float *>(y),
                                                                static_cast<const float *>(z), w, eps,
                                                                apply ? 1 : 0, E, rstd_out);
    return cudaGetLastError();
}

}  // namespace ssd
