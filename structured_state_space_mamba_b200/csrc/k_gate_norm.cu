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
// in place on y.  HBM-bound: y and z are read from HBM once and y written once.
// One CTA of 128 threads per token; each thread takes 16-byte vectors of the
// row (8 bf16 or 4 fp32) at a stride of the block, forms the block-wide sum of
// squares, then reads its vectors again (from L1 / L2), scales and stores
// them.  Rows that are not a whole number of vectors take a scalar loop.
#include "common.cuh"
#include "kernels.h"

namespace ssd {

namespace {

constexpr int kThreads = 256;    // the scalar two-pass kernel
constexpr int kVecThreads = 128; // the vector kernel

template <typename T>
struct Vec;
template <>
struct Vec<__nv_bfloat16> {
    static constexpr int n = 8;
    __device__ static void load(const __nv_bfloat16 *p, float (&v)[8]) {
        const uint4 u = *reinterpret_cast<const uint4 *>(p);
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            v[2 * i] = __uint_as_float(w[i] << 16);
            v[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
        }
    }
    __device__ static void store(__nv_bfloat16 *p, const float (&v)[8]) {
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
            w[i] = *reinterpret_cast<const uint32_t *>(&h);
        }
        *reinterpret_cast<uint4 *>(p) = make_uint4(w[0], w[1], w[2], w[3]);
    }
};
template <>
struct Vec<float> {
    static constexpr int n = 4;
    __device__ static void load(const float *p, float (&v)[4]) {
        const float4 u = *reinterpret_cast<const float4 *>(p);
        v[0] = u.x; v[1] = u.y; v[2] = u.z; v[3] = u.w;
    }
    __device__ static void store(float *p, const float (&v)[4]) {
        *reinterpret_cast<float4 *>(p) = make_float4(v[0], v[1], v[2], v[3]);
    }
};

// y * silu(z) = y * z / (1 + e^-z).  The kernel is bound by its instruction
// issue, not by HBM (ncu on the 2.7B-shaped block: issue slots 76 % busy, DRAM
// 37 %), and an IEEE division costs several times the rest of the gate, so it
// takes the approximate division (2 ulp; for z below about -88, e^-z is inf
// and the quotient 0, the limit of silu).
__device__ __forceinline__ float silu_gate(float y, float z) { return y * __fdividef(z, 1.f + __expf(-z)); }

// block-wide sum over NT threads (every thread gets the result)
template <int NT = kThreads>
__device__ __forceinline__ float block_sum(float v, float *red) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
    __syncthreads();
    float t = threadIdx.x < NT / 32 ? red[threadIdx.x] : 0.f;
    if (threadIdx.x < 32) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
        if (threadIdx.x == 0) red[NT / 32] = t;
    }
    __syncthreads();
    return red[NT / 32];
}

// rows of whole 16-byte vectors: two passes over the row, the second finding
// it in L1 / L2, with nothing but the running sum held between them (about 40
// registers), NT threads per token.  Measured on the 2.7B-shaped block (16384
// tokens of 5120 values), with the gate's IEEE division: 144 us with 128
// threads, 154 us with 256, 148 us with 64; holding the row's g in registers
// between the passes (two or three tokens per SM in flight) took 177 us, one
// warp per token 182 us.  With the approximate division: 95 us (128 threads).
template <typename T, int NT>
__global__ void __launch_bounds__(NT)
gate_norm_vec2_kernel(T *__restrict__ y, const T *__restrict__ z, const float *__restrict__ w, float eps,
                      int apply, int E, float *__restrict__ rstd_out) {
    constexpr int V = Vec<T>::n;
    __shared__ float red[NT / 32 + 1];
    const int64_t tok = blockIdx.x;
    T *row = y + tok * E;
    const T *zr = z ? z + tok * E : nullptr;
    const int nv = E / V;
    float scale = 1.f;
    if (w) {
        float ss = 0.f;
#pragma unroll 2
        for (int v = threadIdx.x; v < nv; v += NT) {
            float g[V], zz[V];
            Vec<T>::load(row + v * V, g);
            if (zr) Vec<T>::load(zr + v * V, zz);
#pragma unroll
            for (int e = 0; e < V; ++e) {
                if (zr) g[e] = silu_gate(g[e], zz[e]);
                ss = fmaf(g[e], g[e], ss);
            }
        }
        const float rs = rsqrtf(block_sum<NT>(ss, red) / float(E) + eps);
        if (rstd_out && threadIdx.x == 0) rstd_out[tok] = rs;
        if (apply) scale = rs;
    }
#pragma unroll 2
    for (int v = threadIdx.x; v < nv; v += NT) {
        float g[V], zz[V];
        Vec<T>::load(row + v * V, g);
        if (zr) Vec<T>::load(zr + v * V, zz);
#pragma unroll
        for (int e = 0; e < V; ++e)
            if (zr) g[e] = silu_gate(g[e], zz[e]);
        if (w) {
#pragma unroll
            for (int e = 0; e < V; e += 4) {
                const float4 q = __ldg(reinterpret_cast<const float4 *>(w + v * V + e));
                g[e] *= scale * q.x;
                g[e + 1] *= scale * q.y;
                g[e + 2] *= scale * q.z;
                g[e + 3] *= scale * q.w;
            }
        }
        Vec<T>::store(row + v * V, g);
    }
}

// any row: two passes over it (the second finds it in L1 / L2)
template <typename T>
__global__ void __launch_bounds__(kThreads)
gate_norm_kernel(T *__restrict__ y, const T *__restrict__ z, const float *__restrict__ w, float eps,
                 int apply, int E, float *__restrict__ rstd_out) {
    __shared__ float red[kThreads / 32 + 1];
    const int64_t tok = blockIdx.x;
    T *row = y + tok * E;
    const T *zr = z ? z + tok * E : nullptr;
    float scale = 1.f;
    if (w) {
        float ss = 0.f;
        for (int i = threadIdx.x; i < E; i += kThreads) {
            const float v = to_f32<T>(row[i]);
            const float g = zr ? silu_gate(v, to_f32<T>(zr[i])) : v;
            ss = fmaf(g, g, ss);
        }
        const float rs = rsqrtf(block_sum(ss, red) / float(E) + eps);
        if (rstd_out && threadIdx.x == 0) rstd_out[tok] = rs;
        if (apply) scale = rs;
    }
    for (int i = threadIdx.x; i < E; i += kThreads) {
        const float v = to_f32<T>(row[i]);
        float g = zr ? silu_gate(v, to_f32<T>(zr[i])) : v;
        if (w) g *= scale * __ldg(w + i);
        row[i] = from_f32<T>(g);
    }
}

template <typename T>
cudaError_t launch_typed(int64_t tokens, int E, void *y, const void *z, const float *w, float eps, bool apply,
                         float *rstd_out, cudaStream_t stream) {
    const dim3 grid(static_cast<unsigned>(tokens), 1, 1);
    constexpr int V = Vec<T>::n;
    // the vector path needs whole 16-byte vectors: E % V == 0 keeps every row
    // (and the weight) 16-byte aligned, the tensors themselves being aligned
    if (E % V == 0)
        gate_norm_vec2_kernel<T, kVecThreads><<<grid, kVecThreads, 0, stream>>>(
            static_cast<T *>(y), static_cast<const T *>(z), w, eps, apply ? 1 : 0, E, rstd_out);
    else
        gate_norm_kernel<T><<<grid, kThreads, 0, stream>>>(static_cast<T *>(y), static_cast<const T *>(z), w, eps,
                                                           apply ? 1 : 0, E, rstd_out);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gate_norm(const Dims &d, bool bf16, void *y, const void *z, const float *w, float eps,
                             bool apply, float *rstd_out, cudaStream_t stream) {
    const int64_t tokens = int64_t(d.B) * d.T;
    const int E = d.H * d.P;
    if (tokens <= 0 || tokens > 0x7fffffff) return cudaErrorInvalidValue;
    return bf16 ? launch_typed<__nv_bfloat16>(tokens, E, y, z, w, eps, apply, rstd_out, stream)
                : launch_typed<float>(tokens, E, y, z, w, eps, apply, rstd_out, stream);
}

}  // namespace ssd
