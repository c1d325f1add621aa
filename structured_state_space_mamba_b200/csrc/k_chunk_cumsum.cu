// k_chunk_cumsum.cu -- ssd_chunk_cumsum: the per-chunk cumulative log-decay.
//
// For chunk c of batch b and head h (tokens t = cQ + i, i in [0, Q)):
//   l[i]    = sum_{k<=i} dt_{cQ+k} * A_h        (inclusive, restarts every chunk)
//   alpha   = exp(l[Q-1])                       (decay across the whole chunk)
//   w[i]    = exp(l[Q-1] - l[i]) * dt_{cQ+i}    (weight of token i in the chunk state)
//   dtq[i]  = dt_{cQ+i}                         (dt regrouped per chunk and head)
//   beta[i] = exp(l[32k+31] - l[i]) * dt_{cQ+i}, k = i / 32
//                                               (source factor of the factored decay
//                                                used by the block-factored scan)
//   gq      = the chunk-wide scan's token factors (chunk_len 128 or 256 only):
//             gq[i] = exp(r - l[i]) dt_i (exponent clamped at 80), then one flag
//             per 128-token tile k (1 when r - l[128k+127] >= kScanSteep or a dt
//             of the tile is 0, below 1e-30: such tiles are computed by the
//             block-factored scan), then r.  The reference r is 0, or l[127]
//             when -l[Q-1] reaches kScanSteep but neither tile's own decay
//             range does; dtq and beta are then written only for chunks with a
//             flagged tile (the block-factored scan reads no others)
//   fused mode (the single-pass kernel of k_tc_chunk_fused.cu): the same gq
//             layout with a reference that also keeps the chunk state exact --
//             r = 0 or l[127] as above, otherwise r = l[Q-1] (then every
//             g_s <= dt_s); a tile is flagged only when a factor it needs,
//             u_t = exp(l_t - r) or g_s, would reach e^kScanSteep (a zero dt
//             is handled by the scan itself); w and alpha are written only
//             when w is given (the presolved single pass reads them), dtq and
//             beta only for chunks with a flagged tile (the block-factored
//             scan reads them); the pairs' chain flags are reset to 0
// With a dt bias or softplus requested (the Mamba-2 block's dt preprocessing),
// every use above takes dt_eff = softplus(dt + dt_bias) (or dt + dt_bias), and
// dt_eff is also written in dt's layout for the scans that read dt directly.
// The decay between tokens s <= t of one chunk is exp(l[t] - l[s]): the
// segment-sum mask L of akillness.github.io "State Space Duality and Mamba-2",
// "The Scalar-Identity Structural Constraint" (the product of the a_k is
// exp(s_j - s_i)).  L itself is never stored; ssd_chunk_scan rebuilds it on
// chip from l.
//
// HBM-bound: one CTA per (chunk, 8 heads, batch) reads dt for its 8 heads in
// 32-byte row segments; one warp scans one head.  Lane j holds tokens j,
// j+32, j+64, ..., so every store instruction writes 128 contiguous bytes and
// a 32-token block is exactly one warp-wide row of the scan.
#include "common.cuh"
#include "kernels.h"

namespace ssd {

namespace {

constexpr int kThreads = 256;
constexpr int kHeads = 8;  // heads per CTA = warps per CTA

template <int E>  // E = Q / 32 rows of 32 tokens
__global__ void __launch_bounds__(kThreads)
chunk_cumsum_kernel(Dims d, const float *__restrict__ dt, const float *__restrict__ A,
                    float *__restrict__ l_out, float *__restrict__ w_out,
                    float *__restrict__ dtq_out, float *__restrict__ beta_out,
                    float *__restrict__ alpha_out, float *__restrict__ gq_out,
                    int *__restrict__ nsteep, unsigned int *__restrict__ chain_flags,
                    const float *__restrict__ dt_bias, int dt_softplus, float *__restrict__ dt_eff) {
    constexpr int Q = 32 * E;
    const bool fused = chain_flags != nullptr;
    // the chunk-wide scan's steep-tile list starts empty (that kernel runs after
    // this one in stream order)
    if (nsteep && (blockIdx.x | blockIdx.y | blockIdx.z | threadIdx.x) == 0) *nsteep = 0;
    // fused mode: the chain flags of this CTA's 4 head pairs start at 0
    if (fused && blockIdx.x == 0 && threadIdx.x < kHeads / 2) {
        const int pair = blockIdx.y * (kHeads / 2) + threadIdx.x;
        if (pair < d.H / 2) chain_flags[int64_t(blockIdx.z) * (d.H / 2) + pair] = 0u;
    }
    __shared__ float s_dt[Q][kHeads + 1];
    const int c = blockIdx.x, b = blockIdx.z;
    const int h0 = blockIdx.y * kHeads;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int t0 = c * Q;
    // dt[b, t0:t0+Q, h0:h0+8]: each row is one 32-byte segment; all loads are
    // issued before the first shared-memory store
    {
        constexpr int kIters = Q * kHeads / kThreads;
        const int j = threadIdx.x % kHeads;
        const int i0 = threadIdx.x / kHeads;
        float v[kIters];
        const float bias = (dt_bias && h0 + j < d.H) ? __ldg(dt_bias + h0 + j) : 0.f;
#pragma unroll
        for (int k = 0; k < kIters; ++k) {
            const int i = i0 + k * (kThreads / kHeads);
            v[k] = h0 + j < d.H ? __ldg(dt + off_dt(d, b, t0 + i) + h0 + j) : 0.f;
        }
        if (dt_bias || dt_softplus) {
            // the step size the scan uses: softplus(dt + dt_bias), written as
            // max(v, 0) + log1p(e^-|v|) (no overflow for large v)
#pragma unroll
            for (int k = 0; k < kIters; ++k) {
                if (h0 + j >= d.H) continue;
                float e = v[k] + bias;
                if (dt_softplus) e = fmaxf(e, 0.f) + log1pf(expf(-fabsf(e)));
                v[k] = e;
                if (dt_eff) dt_eff[off_dt(d, b, t0 + i0 + k * (kThreads / kHeads)) + h0 + j] = e;
            }
        }
#pragma unroll
        for (int k = 0; k < kIters; ++k) s_dt[i0 + k * (kThreads / kHeads)][j] = v[k];
    }
    __syncthreads();
    const int h = h0 + warp;
    if (h >= d.H) return;
    const float a = __ldg(A + h);
    const int64_t base = off_lq(d, b, h, c);
    float lv[E], dts[E], bend[E];
    float carry = 0.f;
#pragma unroll
    for (int k = 0; k < E; ++k) {
        dts[k] = s_dt[32 * k + lane][warp];
        float incl = dts[k] * a;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float n = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += n;
        }
        lv[k] = carry + incl;
        bend[k] = __shfl_sync(0xffffffffu, lv[k], 31);  // l at token 32k+31
        l_out[base + 32 * k + lane] = lv[k];
        carry = bend[k];
    }
    const float last = carry;  // l[Q-1]
    if (fused && E >= 4) {
        float *g = gq_out + ((int64_t(b) * d.H + h) * d.nc + c) * chunk_gq(Q);
        // r = 0, or l[127] when only the whole chunk's decay reaches the limit,
        // else l[Q-1] (every g_s <= dt_s: the chunk state stays exact)
        const float l127 = __shfl_sync(0xffffffffu, lv[3], 31);
        float r;
        if (-last < kScanSteep) r = 0.f;
        else if (E == 8 && -l127 < kScanSteep && l127 - last < kScanSteep) r = l127;
        else r = last;
        bool any = false;
#pragma unroll
        for (int k = 0; k < E; ++k) {
            g[32 * k + lane] = __expf(fminf(r - lv[k], 80.f)) * dts[k];
            if ((k & 3) == 3) {  // last 32 tokens of a 128-token tile
                const float lfirst = __shfl_sync(0xffffffffu, lv[k - 3], 0);
                const bool steep = lfirst - r >= kScanSteep || r - bend[k] >= kScanSteep;
                any |= steep;
                if (lane == 0) g[Q + (k >> 2)] = steep ? 1.f : 0.f;
            }
        }
        if (lane == 0) {
            if (E == 4) g[Q + 1] = 0.f;
            g[Q + 2] = r;
            g[Q + 3] = 0.f;
        }
        if (any) {  // the block-factored scan recomputes this chunk's flagged tiles
#pragma unroll
            for (int k = 0; k < E; ++k) {
                dtq_out[base + 32 * k + lane] = dts[k];
                beta_out[base + 32 * k + lane] = __expf(bend[k] - lv[k]) * dts[k];
            }
        }
        if (w_out) {  // presolved ranges: their pass over x and B takes w and alpha
#pragma unroll
            for (int k = 0; k < E; ++k) w_out[base + 32 * k + lane] = __expf(last - lv[k]) * dts[k];
            if (lane == 0) alpha_out[off_alpha(d, b, h, c)] = __expf(last);
        }
        return;
    }
    bool flagged = false;  // a tile of this (chunk, head) is left to the block-factored scan
    if (gq_out && E >= 4) {
        float *g = gq_out + ((int64_t(b) * d.H + h) * d.nc + c) * chunk_gq(Q);
        // reference r of the chunk-wide factors: 0, or l[127] when the decay over
        // the whole chunk reaches kScanSteep but neither 128-token tile's does
        const float l127 = __shfl_sync(0xffffffffu, lv[3], 31);
        const bool shift = E == 8 && -last >= kScanSteep && -l127 < kScanSteep && l127 - last < kScanSteep;
        const float r = shift ? l127 : 0.f;
        bool zero = false;
#pragma unroll
        for (int k = 0; k < E; ++k) {
            g[32 * k + lane] = __expf(fminf(r - lv[k], 80.f)) * dts[k];
            zero |= dts[k] < 1e-30f;
            if ((k & 3) == 3) {  // last 32 tokens of a 128-token tile
                const bool any0 = __any_sync(0xffffffffu, zero);
                const float lend = __shfl_sync(0xffffffffu, lv[k], 31);
                const bool steep = r - lend >= kScanSteep || any0;
                flagged |= steep;
                if (lane == 0) g[Q + (k >> 2)] = steep ? 1.f : 0.f;
                zero = false;
            }
        }
        if (lane == 0) g[Q + 2] = r;
        if (lane == 0 && E == 4) g[Q + 1] = 0.f;
        if (lane == 0) g[Q + 3] = 0.f;
    }
    // dtq and beta feed the block-factored scan: every chunk when it is the
    // scan, only the chunks with a flagged tile when it finishes the chunk-wide
    // scan's list (the plans that take gq)
    const bool factored = !gq_out || flagged;
#pragma unroll
    for (int k = 0; k < E; ++k) {
        if (factored) {
            dtq_out[base + 32 * k + lane] = dts[k];
            beta_out[base + 32 * k + lane] = __expf(bend[k] - lv[k]) * dts[k];
        }
        w_out[base + 32 * k + lane] = __expf(last - lv[k]) * dts[k];
    }
    if (lane == 0) alpha_out[off_alpha(d, b, h, c)] = __expf(last);
}

}  // namespace

cudaError_t launch_chunk_cumsum(const Dims &d, const float *dt, const float *A, float *l,
                                float *w, float *dtq, float *beta, float *alpha, float *gq,
                                int *nsteep, unsigned int *chain_flags, const float *dt_bias,
                                int dt_softplus, float *dt_eff, cudaStream_t stream) {
    if (chain_flags && (d.Q < 128 || !gq)) return cudaErrorInvalidValue;
    dim3 grid(d.nc, (d.H + kHeads - 1) / kHeads, d.B);
    switch (d.Q) {
        case 32: chunk_cumsum_kernel<1><<<grid, kThreads, 0, stream>>>(d, dt, A, l, w, dtq, beta, alpha, gq, nsteep, chain_flags, dt_bias, dt_softplus, dt_eff); break;
        case 64: chunk_cumsum_kernel<2><<<grid, kThreads, 0, stream>>>(d, dt, A, l, w, dtq, beta, alpha, gq, nsteep, chain_flags, dt_bias, dt_softplus, dt_eff); break;
        case 128: chunk_cumsum_kernel<4><<<grid, kThreads, 0, stream>>>(d, dt, A, l, w, dtq, beta, alpha, gq, nsteep, chain_flags, dt_bias, dt_softplus, dt_eff); break;
        case 256: chunk_cumsum_kernel<8><<<grid, kThreads, 0, stream>>>(d, dt, A, l, w, dtq, beta, alpha, gq, nsteep, chain_flags, dt_bias, dt_softplus, dt_eff); break;
        default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

}  // namespace ssd
