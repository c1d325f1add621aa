// k_tail.cu -- the last T mod chunk_len tokens of a sequence whose length is
// not a multiple of chunk_len, as the recurrence itself:
//     h_t = exp(dt_t A_h) h_{t-1} + dt_t x_t B_t^T,   y_t = h_t C_t + D_h x_t
// (akillness.github.io "State Space Duality and Mamba-2", "Mathematical
// Foundations": the recurrent form -- the chunked form's last, partial chunk is
// the same operation), starting from the state the chunked kernels leave after
// the last full chunk (or from the initial state when there is none).
//
// One CTA per (b, h).  The fp32 state lives in registers: thread i owns row
// p = i / TPR and the EPT columns starting at (i % TPR) * EPT (EPT = min(64, N),
// TPR = N / EPT threads per row, consecutive lanes, so a row's readout is a
// shuffle reduction).  The tail's x, dt, B and C are staged through shared
// memory 32 tokens at a time; the token steps then read only shared memory.
// Latency-bound (at most chunk_len - 1 sequential steps), and only on lengths
// that are not a multiple of chunk_len.
#include "common.cuh"
#include "kernels.h"

namespace ssd {

namespace {

constexpr int kBlockTok = 32;

template <typename T, int EPT>
__global__ void __launch_bounds__(1024)
tail_kernel(Dims d, int t_begin, const T *__restrict__ x, const float *__restrict__ dt,
            const float *__restrict__ dt_bias, int dt_softplus, const float *__restrict__ A, const T *__restrict__ Bm, const T *__restrict__ Cm,
            const float *__restrict__ D, const float *__restrict__ h_in, T *__restrict__ y,
            float *__restrict__ fin) {
    extern __shared__ float sm[];
    const int h = blockIdx.x % d.H, b = blockIdx.x / d.H;
    const int g = h / d.r;
    const int tpr = d.N / EPT;
    const int i = threadIdx.x;
    const int p = i / tpr, n0 = (i % tpr) * EPT;
    const bool active = p < d.P;
    float *sB = sm;                        // [kBlockTok][N]
    float *sC = sB + kBlockTok * d.N;      // [kBlockTok][N]
    float *sX = sC + kBlockTok * d.N;      // [kBlockTok][P]
    float *sDt = sX + kBlockTok * d.P;     // [kBlockTok]
    const float a_h = __ldg(A + h);
    const float Dh = D ? __ldg(D + h) : 0.f;
    float s[EPT];
    const int64_t srow = ((int64_t(b) * d.H + h) * d.P + (active ? p : 0)) * d.N + n0;
#pragma unroll
    for (int e = 0; e < EPT; ++e) s[e] = (active && h_in) ? h_in[srow + e] : 0.f;
    for (int tb = t_begin; tb < d.T; tb += kBlockTok) {
        const int nt = min(kBlockTok, d.T - tb);
        __syncthreads();  // the previous block's reads are done
        for (int k = i; k < nt * d.N; k += blockDim.x) {
            const int tt = k / d.N, nn = k % d.N;
            sB[tt * d.N + nn] = to_f32<T>(Bm[off_bc(d, b, tb + tt, g) + nn]);
            sC[tt * d.N + nn] = to_f32<T>(Cm[off_bc(d, b, tb + tt, g) + nn]);
        }
        for (int k = i; k < nt * d.P; k += blockDim.x) {
            const int tt = k / d.P, pp = k % d.P;
            sX[tt * d.P + pp] = to_f32<T>(x[off_x(d, b, tb + tt, h) + pp]);
        }
        for (int k = i; k < nt; k += blockDim.x) {
            // the block's dt transform, as in the cumsum kernel: softplus(dt + dt_bias)
            float v = __ldg(dt + off_dt(d, b, tb + k) + h) + (dt_bias ? __ldg(dt_bias + h) : 0.f);
            if (dt_softplus) v = fmaxf(v, 0.f) + log1pf(expf(-fabsf(v)));
            sDt[k] = v;
        }
        __syncthreads();
        for (int tt = 0; tt < nt; ++tt) {
            const float dtt = sDt[tt];
            const float a = __expf(dtt * a_h);
            const float xin = active ? dtt * sX[tt * d.P + p] : 0.f;
            const float *bt = sB + tt * d.N + n0;
            const float *ct = sC + tt * d.N + n0;
            float part = 0.f;
#pragma unroll
            for (int e = 0; e < EPT; ++e) {
                s[e] = fmaf(a, s[e], xin * bt[e]);
                part = fmaf(s[e], ct[e], part);
            }
            // the row's tpr threads are consecutive lanes (tpr divides 32)
            for (int o = tpr >> 1; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o, tpr);
            if (active && (i % tpr) == 0)
                y[off_x(d, b, tb + tt, h) + p] = from_f32<T>(part + Dh * sX[tt * d.P + p]);
        }
    }
    if (active && fin) {
#pragma unroll
        for (int e = 0; e < EPT; ++e) fin[srow + e] = s[e];
    }
}

template <typename T, int EPT>
cudaError_t launch_tail_t(const Dims &d, int t_begin, const void *x, const float *dt, const float *dt_bias,
                          int dt_softplus, const float *A,
                          const void *Bm, const void *Cm, const float *D, const float *h_in, void *y,
                          float *fin, cudaStream_t stream) {
    const int tpr = d.N / EPT;
    int threads = d.P * tpr;
    threads = (threads + 31) / 32 * 32;
    const size_t smem = (size_t(2) * kBlockTok * d.N + size_t(kBlockTok) * d.P + kBlockTok) * sizeof(float);
    if (smem > 48 * 1024 &&
        cudaFuncSetAttribute(tail_kernel<T, EPT>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)) !=
            cudaSuccess)
        return cudaErrorInvalidValue;
    tail_kernel<T, EPT><<<d.B * d.H, threads, smem, stream>>>(
        d, t_begin, static_cast<const T *>(x), dt, dt_bias, dt_softplus, A, static_cast<const T *>(Bm), static_cast<const T *>(Cm), D,
        h_in, static_cast<T *>(y), fin);
    return cudaGetLastError();
}

template <typename T>
cudaError_t launch_tail_typed(const Dims &d, int t_begin, const void *x, const float *dt, const float *dt_bias,
                              int dt_softplus, const float *A,
                              const void *Bm, const void *Cm, const float *D, const float *h_in, void *y,
                              float *fin, cudaStream_t stream) {
    // EPT = N for N <= 64 (one thread per row), else 64 (N / 64 threads per row)
    switch (d.N <= 64 ? d.N : 64) {
        case 8: return launch_tail_t<T, 8>(d, t_begin, x, dt, dt_bias, dt_softplus, A, Bm, Cm, D, h_in, y, fin, stream);
        case 16: return launch_tail_t<T, 16>(d, t_begin, x, dt, dt_bias, dt_softplus, A, Bm, Cm, D, h_in, y, fin, stream);
        case 32: return launch_tail_t<T, 32>(d, t_begin, x, dt, dt_bias, dt_softplus, A, Bm, Cm, D, h_in, y, fin, stream);
        case 64: return launch_tail_t<T, 64>(d, t_begin, x, dt, dt_bias, dt_softplus, A, Bm, Cm, D, h_in, y, fin, stream);
        default: break;
    }
    return cudaErrorInvalidValue;
}

}  // namespace

bool tail_supported(const Dims &d) {
    // the state row split into equal per-thread pieces: N <= 64 one of 8/16/32/64,
    // else a multiple of 64; at most 1024 threads
    const bool n_ok = d.N == 8 || d.N == 16 || d.N == 32 || d.N == 64 || (d.N > 64 && d.N % 64 == 0);
    const int tpr = d.N <= 64 ? 1 : d.N / 64;
    return n_ok && d.P * tpr <= 1024;
}

cudaError_t launch_tail(const Dims &d, bool bf16, int t_begin, const void *x, const float *dt,
                        const float *dt_bias, int dt_softplus, const float *A, const void *Bm, const void *Cm,
                        const float *D, const float *h_in, void *y, float *fin, cudaStream_t stream) {
    if (t_begin >= d.T) return cudaSuccess;
    return bf16 ? launch_tail_typed<__nv_bfloat16>(d, t_begin, x, dt, dt_bias, dt_softplus, A, Bm, Cm, D, h_in, y,
                                                   fin, stream)
                : launch_tail_typed<float>(d, t_begin, x, dt, dt_bias, dt_softplus, A, Bm, Cm, D, h_in, y, fin,
                                           stream);
}

}  // namespace ssd
