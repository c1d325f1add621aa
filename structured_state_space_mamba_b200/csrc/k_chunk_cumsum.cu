// k_chunk_cumsum.cu -- ssd_chunk_cumsum: the per-chunk cumulative log-decay.
//
// For chunk c of batch b and head h (tokens t = cQ + i, i in [0, Q)):
//   l[i]    = sum_{k<=i} dt_{cQ+k} * A_h        (inclusive, restarts every chunk)
//   alpha   = exp(l[Q-1])                       (decay across the whole chunk)
//   w[i]    = exp(l[Q-1] - l[i]) * dt_{cQ+i}    (weight of token i in the chunk state)
// The decay between tokens s <= t of one chunk is exp(l[t] - l[s]): the
// segment-sum mask L of akillness.github.io "State Space Duality and Mamba-2",
// "The Scalar-Identity Structural Constraint" (product of the a_k = exp(s_j - s_i)).
// L itself is never stored; ssd_chunk_scan rebuilds it on chip from l.
//
// HBM-bound: reads dt once (coalesced over heads), writes l and w once per
// token-head and alpha once per chunk-head.
#include "common.cuh"
#include "kernels.h"

namespace ssd {

namespace {

constexpr int kThreads = 256;
constexpr int kHeadTile = 32;

template <int E>  // E = Q / 32 values per lane
__global__ void __launch_bounds__(kThreads)
chunk_cumsum_kernel(Dims d, const float *__restrict__ dt, const float *__restrict__ A,
                    float *__restrict__ l_out, float *__restrict__ w_out,
                    float *__restrict__ alpha_out) {
    constexpr int Q = 32 * E;
    __shared__ float s_dt[Q][kHeadTile + 1];
    const int c = blockIdx.x, b = blockIdx.z;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int t0 = c * Q;
    {
        const int h0 = blockIdx.y * kHeadTile;
        // coalesced load of dt[b, t0:t0+Q, h0:h0+32]; all loads issued before
        // the first store so that they are in flight together
        {
            constexpr int kIters = Q / (kThreads / 32);
            const int h = h0 + lane;
            float v[kIters];
#pragma unroll
            for (int k = 0; k < kIters; ++k) {
                const int i = warp + k * (kThreads / 32);
                v[k] = h < d.H ? __ldg(dt + off_dt(d, b, t0 + i) + h) : 0.f;
            }
#pragma unroll
            for (int k = 0; k < kIters; ++k) s_dt[warp + k * (kThreads / 32)][lane] = v[k];
        }
        __syncthreads();
        for (int j = warp; j < kHeadTile; j += kThreads / 32) {
            const int h = h0 + j;
            if (h >= d.H) break;  // warp-uniform
            const float a = __ldg(A + h);
            float v[E], dts[E];
            float run = 0.f;
#pragma unroll
            for (int e = 0; e < E; ++e) {
                dts[e] = s_dt[lane * E + e][j];
                run += dts[e] * a;
                v[e] = run;
            }
            // exclusive scan of the lane totals
            float incl = run;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float n = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += n;
            }
            const float excl = incl - run;
            const float last = __shfl_sync(0xffffffffu, incl, 31);
            float *lp = l_out + off_lq(d, b, h, c) + lane * E;
            float *wp = w_out + off_lq(d, b, h, c) + lane * E;
#pragma unroll
            for (int e = 0; e < E; ++e) {
                const float li = v[e] + excl;
                lp[e] = li;
                wp[e] = __expf(last - li) * dts[e];
            }
            if (lane == 0) alpha_out[off_alpha(d, b, h, c)] = __expf(last);
        }
        __syncthreads();
    }
}

}  // namespace

cudaError_t launch_chunk_cumsum(const Dims &d, const float *dt, const float *A, float *l,
                                float *w, float *alpha, cudaStream_t stream) {
    dim3 grid(d.nc, (d.H + kHeadTile - 1) / kHeadTile, d.B);
    switch (d.Q) {
        case 32: chunk_cumsum_kernel<1><<<grid, kThreads, 0, stream>>>(d, dt, A, l, w, alpha); break;
        case 64: chunk_cumsum_kernel<2><<<grid, kThreads, 0, stream>>>(d, dt, A, l, w, alpha); break;
        case 128: chunk_cumsum_kernel<4><<<grid, kThreads, 0, stream>>>(d, dt, A, l, w, alpha); break;
        case 256: chunk_cumsum_kernel<8><<<grid, kThreads, 0, stream>>>(d, dt, A, l, w, alpha); break;
        default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

}  // namespace ssd
