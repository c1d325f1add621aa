// common.cuh -- small device helpers shared by the SSD kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace ssd {

// Problem description passed by value to every kernel (all sizes in elements).
struct Dims {
    int B, T, H, P, N, G;
    int Q;   // chunk length
    int nc;  // T / Q
    int r;   // heads per group, H / G
};

template <typename T> __device__ __forceinline__ float to_f32(T v);
template <> __device__ __forceinline__ float to_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 v) {
    return __bfloat162float(v);
}

template <typename T> __device__ __forceinline__ T from_f32(float v);
template <> __device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) {
    return __float2bfloat16_rn(v);
}

// Offsets into the row-major tensors (64-bit: the long-context layer has
// more than 2^31 elements in some tensors).
__device__ __forceinline__ int64_t off_x(const Dims &d, int b, int t, int h) {
    return ((int64_t(b) * d.T + t) * d.H + h) * d.P;
}
__device__ __forceinline__ int64_t off_bc(const Dims &d, int b, int t, int g) {
    return ((int64_t(b) * d.T + t) * d.G + g) * d.N;
}
__device__ __forceinline__ int64_t off_dt(const Dims &d, int b, int t) {
    return (int64_t(b) * d.T + t) * d.H;
}
// [B, H, nc, Q] (cumsum, weights) and [B, H, nc] (chunk decay)
__device__ __forceinline__ int64_t off_lq(const Dims &d, int b, int h, int c) {
    return ((int64_t(b) * d.H + h) * d.nc + c) * d.Q;
}
__device__ __forceinline__ int64_t off_alpha(const Dims &d, int b, int h, int c) {
    return (int64_t(b) * d.H + h) * d.nc + c;
}
// [B, nc, H, P, N] chunk states and incoming states
__device__ __forceinline__ int64_t off_state(const Dims &d, int b, int c, int h) {
    return ((int64_t(b) * d.nc + c) * d.H + h) * int64_t(d.P) * d.N;
}

}  // namespace ssd
