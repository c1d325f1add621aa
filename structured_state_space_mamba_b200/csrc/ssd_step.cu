// ssd_step.cu -- ssd_step: one token of the SSD recurrence for every (batch,
// head), the decode step.
//
// Per batch b, head h, group g = h / (H / G):
//     h'  = exp(dt A_h) h + dt x B^T      (state P x N, updated in place)
//     y   = h' C + D_h x
// -- the recurrent (linear) form of the scalar-identity SSM (akillness.github.io
// "State Space Duality and Mamba-2: Unifying Transformers and Semiseparable
// Matrices", "Mathematical Foundations: From State Spaces to Semiseparable
// Matrices"), with the step size dt on the decay and on the input as in the
// forward scan of this library; it is the dual of the chunked scan that a
// generation loop runs once per new token.
//
// HBM-bound on the fp32 state (read and written once, 8 P N bytes per (b, h));
// x, B, C and y are a few hundred bytes.  One CTA per (b, h): B_t, C_t and x_t
// go to shared memory as fp32; each state row (N fp32) is covered by a group of
// lanes with 16-byte loads and stores, four rows' loads in flight per thread
// before any arithmetic, and y_p is reduced across the row's lanes by shuffles.
// Shapes whose rows are not a power of two of 16-byte vectors (or an unaligned
// state) take a scalar kernel with one thread per row.
#include <cuda_runtime.h>

#include <cstdint>

#include "../../include/ssd.h"
#include "common.cuh"

namespace {

constexpr int kThreads = 256;

struct StepDims {
    int B, H, P, N, G, r;
};

__device__ __forceinline__ float ld_f32(const float *p) { return __ldg(p); }
__device__ __forceinline__ float ld_f32(const __nv_bfloat16 *p) { return __bfloat162float(*p); }

// B_t, C_t of the head's group and x_t of the head into shared memory as fp32.
template <typename T>
__device__ __forceinline__ void load_vectors(const StepDims &d, int b, int h, const T *x, const T *Bm,
                                             const T *Cm, float *sB, float *sC, float *sx) {
    const int g = h / d.r;
    const int64_t bg = (int64_t(b) * d.G + g) * d.N;
    for (int i = threadIdx.x; i < d.N; i += kThreads) {
        sB[i] = ld_f32(Bm + bg + i);
        sC[i] = ld_f32(Cm + bg + i);
    }
    const int64_t bh = (int64_t(b) * d.H + h) * d.P;
    for (int i = threadIdx.x; i < d.P; i += kThreads) sx[i] = ld_f32(x + bh + i);
}

// F = N / 4 sixteen-byte vectors per state row (a power of two, 4 .. 64).
template <typename T, int F>
__global__ void __launch_bounds__(kThreads)
step_vec_kernel(StepDims d, const T *__restrict__ x, const float *__restrict__ dt,
                const float *__restrict__ A, const T *__restrict__ Bm, const T *__restrict__ Cm,
                const float *__restrict__ D, float *__restrict__ state, T *__restrict__ y) {
    constexpr int kTpr = F < 32 ? F : 32;   // lanes per row (divides 32)
    constexpr int kPer = F / kTpr;          // vectors per lane and row
    constexpr int kRpp = kThreads / kTpr;   // rows per pass
    constexpr int kPass = 4;                // passes whose loads are issued together
    __shared__ float sB[4 * F], sC[4 * F], sx[256];
    const int bh = blockIdx.x;
    const int b = bh / d.H, h = bh % d.H;
    load_vectors(d, b, h, x, Bm, Cm, sB, sC, sx);
    const float dth = __ldg(dt + bh);
    const float a = expf(dth * __ldg(A + h));
    const float Dh = D ? __ldg(D + h) : 0.f;
    __syncthreads();
    const int lr = threadIdx.x % kTpr, row0 = threadIdx.x / kTpr;
    float4 *S = reinterpret_cast<float4 *>(state) + int64_t(bh) * d.P * F;
    T *yh = y + int64_t(bh) * d.P;
    for (int pb = 0; pb < d.P; pb += kPass * kRpp) {
        float4 v[kPass][kPer];
#pragma unroll
        for (int j = 0; j < kPass; ++j) {
            const int p = pb + j * kRpp + row0;
            if (p < d.P)
#pragma unroll
                for (int k = 0; k < kPer; ++k) v[j][k] = S[int64_t(p) * F + k * kTpr + lr];
        }
#pragma unroll
        for (int j = 0; j < kPass; ++j) {
            const int p = pb + j * kRpp + row0;
            const bool act = p < d.P;
            float part = 0.f;
            if (act) {
                const float u = dth * sx[p];
#pragma unroll
                for (int k = 0; k < kPer; ++k) {
                    const int f = k * kTpr + lr, n = 4 * f;
                    float4 s = v[j][k];
                    s.x = fmaf(a, s.x, u * sB[n]);
                    s.y = fmaf(a, s.y, u * sB[n + 1]);
                    s.z = fmaf(a, s.z, u * sB[n + 2]);
                    s.w = fmaf(a, s.w, u * sB[n + 3]);
                    S[int64_t(p) * F + f] = s;
                    part += s.x * sC[n] + s.y * sC[n + 1] + s.z * sC[n + 2] + s.w * sC[n + 3];
                }
            }
            // every lane of the warp takes part in the row reductions
#pragma unroll
            for (int o = kTpr / 2; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
            if (act && lr == 0) yh[p] = ssd::from_f32<T>(part + Dh * sx[p]);
        }
    }
}

// Any N and alignment: one thread per state row.
template <typename T>
__global__ void __launch_bounds__(kThreads)
step_scalar_kernel(StepDims d, const T *__restrict__ x, const float *__restrict__ dt,
                   const float *__restrict__ A, const T *__restrict__ Bm, const T *__restrict__ Cm,
                   const float *__restrict__ D, float *__restrict__ state, T *__restrict__ y) {
    __shared__ float sB[256], sC[256], sx[256];
    const int bh = blockIdx.x;
    const int b = bh / d.H, h = bh % d.H;
    load_vectors(d, b, h, x, Bm, Cm, sB, sC, sx);
    const float dth = __ldg(dt + bh);
    const float a = expf(dth * __ldg(A + h));
    const float Dh = D ? __ldg(D + h) : 0.f;
    __syncthreads();
    for (int p = threadIdx.x; p < d.P; p += kThreads) {
        float *row = state + (int64_t(bh) * d.P + p) * d.N;
        const float u = dth * sx[p];
        float acc = 0.f;
        for (int n = 0; n < d.N; ++n) {
            const float s = fmaf(a, row[n], u * sB[n]);
            row[n] = s;
            acc += s * sC[n];
        }
        y[int64_t(bh) * d.P + p] = ssd::from_f32<T>(acc + Dh * sx[p]);
    }
}

template <typename T>
cudaError_t launch_step(const StepDims &d, const void *x, const float *dt, const float *A, const void *Bm,
                        const void *Cm, const float *D, float *state, void *y, cudaStream_t stream) {
    const T *xt = static_cast<const T *>(x), *bt = static_cast<const T *>(Bm), *ct = static_cast<const T *>(Cm);
    T *yt = static_cast<T *>(y);
    const dim3 grid(unsigned(d.B * d.H));
    const bool vec = (reinterpret_cast<uintptr_t>(state) & 15u) == 0;
    if (vec) {
        switch (d.N) {
            case 16: step_vec_kernel<T, 4><<<grid, kThreads, 0, stream>>>(d, xt, dt, A, bt, ct, D, state, yt); return cudaGetLastError();
            case 32: step_vec_kernel<T, 8><<<grid, kThreads, 0, stream>>>(d, xt, dt, A, bt, ct, D, state, yt); return cudaGetLastError();
            case 64: step_vec_kernel<T, 16><<<grid, kThreads, 0, stream>>>(d, xt, dt, A, bt, ct, D, state, yt); return cudaGetLastError();
            case 128: step_vec_kernel<T, 32><<<grid, kThreads, 0, stream>>>(d, xt, dt, A, bt, ct, D, state, yt); return cudaGetLastError();
            case 256: step_vec_kernel<T, 64><<<grid, kThreads, 0, stream>>>(d, xt, dt, A, bt, ct, D, state, yt); return cudaGetLastError();
            default: break;
        }
    }
    step_scalar_kernel<T><<<grid, kThreads, 0, stream>>>(d, xt, dt, A, bt, ct, D, state, yt);
    return cudaGetLastError();
}

}  // namespace

extern "C" {

ssd_status_t ssd_step(const ssd_dims_t *dims, const void *x_t, const float *dt_t, const float *A,
                      const void *B_t, const void *C_t, const float *D, float *state, void *y_t,
                      void *stream) {
    if (!dims || !x_t || !dt_t || !A || !B_t || !C_t || !state || !y_t) return SSD_ERR_NULL_ARG;
    const ssd_dims_t &a = *dims;
    if (a.batch <= 0 || a.nheads <= 0 || a.headdim <= 0 || a.dstate <= 0 || a.ngroups <= 0 ||
        a.seqlen != 1 || a.reserved != 0)
        return SSD_ERR_INVALID_DIM;
    if (a.dtype != SSD_F32 && a.dtype != SSD_BF16) return SSD_ERR_UNSUPPORTED;
    if (a.nheads % a.ngroups != 0) return SSD_ERR_INVALID_DIM;
    if (a.headdim > 256 || a.dstate > 256) return SSD_ERR_UNSUPPORTED;
    if (a.batch * a.nheads > 0x7fffffff) return SSD_ERR_UNSUPPORTED;
    StepDims d;
    d.B = int(a.batch);
    d.H = int(a.nheads);
    d.P = int(a.headdim);
    d.N = int(a.dstate);
    d.G = int(a.ngroups);
    d.r = d.H / d.G;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const cudaError_t e = a.dtype == SSD_BF16
                              ? launch_step<__nv_bfloat16>(d, x_t, dt_t, A, B_t, C_t, D, state, y_t, st)
                              : launch_step<float>(d, x_t, dt_t, A, B_t, C_t, D, state, y_t, st);
    return e == cudaSuccess ? SSD_OK : SSD_ERR_CUDA;
}

}  // extern "C"
