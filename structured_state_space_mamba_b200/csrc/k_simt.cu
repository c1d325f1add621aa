// k_simt.cu -- CUDA-core (FFMA) ssd_chunk_state and ssd_chunk_scan.
//
// These kernels serve every shape the tensor-core kernels do not (the fp32
// path and bf16 shapes outside P == 64): fp32 arithmetic throughout, inputs
// widened on load.  They follow the chunk equations directly:
//
//   chunk state (aifetchly blog "Mamba-2 Architecture", "The Chunked SSD
//   Algorithm", step 2, with the decay weights and dt the page leaves out):
//       S_c[p, n] = sum_{s in chunk} w_s x_s[p] B_s[n],  w_s = exp(l_last - l_s) dt_s
//
//   chunk scan (same page, step 1, the intra-chunk product (C B^T o L) X, plus
//   the contribution of the incoming state and the skip term):
//       y_t[p] = exp(l_t) sum_n C_t[n] s_in[p, n]
//              + sum_{s <= t} exp(l_t - l_s) dt_s (C_t . B_s) x_s[p] + D_h x_t[p]
#include "common.cuh"
#include "kernels.h"

namespace ssd {

namespace {

constexpr int kThreads = 256;  // 16 x 16 threads, 4 x 4 outputs each -> 64 x 64 tiles
constexpr int kTile = 64;
constexpr int kK = 16;

// ---------------------------------------------------------------------------
// chunk state: one block per (c, h, b); loops over 64 x 64 tiles of P x N.
// ---------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(kThreads)
chunk_state_simt_kernel(Dims d, const T *__restrict__ x, const T *__restrict__ Bm,
                        const float *__restrict__ w, float *__restrict__ states) {
    __shared__ float xs[kK][kTile + 4];  // [token][p], weighted by w
    __shared__ float bs[kK][kTile + 4];  // [token][n]
    const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int g = h / d.r;
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
    const int t0 = c * d.Q;
    const float *wc = w + off_lq(d, b, h, c);
    float *Sc = states + off_state(d, b, c, h);
    for (int p0 = 0; p0 < d.P; p0 += kTile)
        for (int n0 = 0; n0 < d.N; n0 += kTile) {
            float acc[4][4] = {};
            for (int k0 = 0; k0 < d.Q; k0 += kK) {
                for (int i = threadIdx.x; i < kK * kTile; i += kThreads) {
                    const int kk = i / kTile, j = i % kTile;
                    const int t = t0 + k0 + kk;
                    const bool tin = (k0 + kk) < d.Q;
                    const float wt = tin ? __ldg(wc + k0 + kk) : 0.f;
                    xs[kk][j] = (tin && p0 + j < d.P) ? wt * to_f32(x[off_x(d, b, t, h) + p0 + j]) : 0.f;
                    bs[kk][j] = (tin && n0 + j < d.N) ? to_f32(Bm[off_bc(d, b, t, g) + n0 + j]) : 0.f;
                }
                __syncthreads();
#pragma unroll
                for (int kk = 0; kk < kK; ++kk) {
                    float xv[4], bv[4];
#pragma unroll
                    for (int i = 0; i < 4; ++i) xv[i] = xs[kk][ty * 4 + i];
#pragma unroll
                    for (int j = 0; j < 4; ++j) bv[j] = bs[kk][tx * 4 + j];
#pragma unroll
                    for (int i = 0; i < 4; ++i)
#pragma unroll
                        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(xv[i], bv[j], acc[i][j]);
                }
                __syncthreads();
            }
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int p = p0 + ty * 4 + i;
                if (p >= d.P) continue;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int n = n0 + tx * 4 + j;
                    if (n < d.N) Sc[int64_t(p) * d.N + n] = acc[i][j];
                }
            }
        }
}

// ---------------------------------------------------------------------------
// chunk scan: one block per (64-row tile of the chunk, c, b*H + h).
// ---------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(kThreads)
chunk_scan_simt_kernel(Dims d, const T *__restrict__ x, const float *__restrict__ dt,
                       const T *__restrict__ Bm, const T *__restrict__ Cm,
                       const float *__restrict__ Dskip, const float *__restrict__ l,
                       const float *__restrict__ s_in, T *__restrict__ y) {
    __shared__ float cs[kTile][kK + 1];     // C rows of this tile, one K slice
    __shared__ float ks[kTile][kK + 1];     // B rows (scores) or s_in rows (state term)
    __shared__ float gs[kTile][kTile + 1];  // masked scores [t][s]
    __shared__ float vs[kTile][kTile + 1];  // x rows [s][p]
    __shared__ float lt[kTile], ls[kTile], dts[kTile];
    const int mt = blockIdx.x, c = blockIdx.y;
    const int b = blockIdx.z / d.H, h = blockIdx.z % d.H;
    const int g = h / d.r;
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
    const int t0 = c * d.Q;        // first token of the chunk
    const int r0 = mt * kTile;     // first row (within the chunk) of this tile
    const int rows = min(kTile, d.Q - r0);
    const float *lc = l + off_lq(d, b, h, c);
    const float *sc = s_in + off_state(d, b, c, h);
    const float Dh = Dskip ? __ldg(Dskip + h) : 0.f;
    if (threadIdx.x < kTile) lt[threadIdx.x] = threadIdx.x < rows ? __ldg(lc + r0 + threadIdx.x) : 0.f;
    __syncthreads();

    for (int p0 = 0; p0 < d.P; p0 += kTile) {
        float acc[4][4] = {};
        // ---- state term: exp(l_t) * C_t . s_in[p, :] -------------------------
        for (int k0 = 0; k0 < d.N; k0 += kK) {
            for (int i = threadIdx.x; i < kTile * kK; i += kThreads) {
                const int row = i / kK, kk = i % kK;
                const int n = k0 + kk;
                cs[row][kk] = (row < rows && n < d.N) ? to_f32(Cm[off_bc(d, b, t0 + r0 + row, g) + n]) : 0.f;
                ks[row][kk] = (p0 + row < d.P && n < d.N) ? __ldg(sc + int64_t(p0 + row) * d.N + n) : 0.f;
            }
            __syncthreads();
#pragma unroll
            for (int kk = 0; kk < kK; ++kk) {
                float cv[4], sv[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) cv[i] = cs[ty * 4 + i][kk];
#pragma unroll
                for (int j = 0; j < 4; ++j) sv[j] = ks[tx * 4 + j][kk];
#pragma unroll
                for (int i = 0; i < 4; ++i)
#pragma unroll
                    for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(cv[i], sv[j], acc[i][j]);
            }
            __syncthreads();
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float e = __expf(lt[ty * 4 + i]);
#pragma unroll
            for (int j = 0; j < 4; ++j) acc[i][j] *= e;
        }
        // ---- intra-chunk term, 64 source tokens at a time --------------------
        for (int s0 = 0; s0 < r0 + rows; s0 += kTile) {
            const int srows = min(kTile, d.Q - s0);
            if (threadIdx.x < kTile) {
                const int s = threadIdx.x;
                ls[s] = s < srows ? __ldg(lc + s0 + s) : 0.f;
                dts[s] = s < srows ? __ldg(dt + off_dt(d, b, t0 + s0 + s) + h) : 0.f;
            }
            // scores G[t][s] = C_t . B_s
            float sco[4][4] = {};
            for (int k0 = 0; k0 < d.N; k0 += kK) {
                for (int i = threadIdx.x; i < kTile * kK; i += kThreads) {
                    const int row = i / kK, kk = i % kK;
                    const int n = k0 + kk;
                    cs[row][kk] = (row < rows && n < d.N) ? to_f32(Cm[off_bc(d, b, t0 + r0 + row, g) + n]) : 0.f;
                    ks[row][kk] = (row < srows && n < d.N) ? to_f32(Bm[off_bc(d, b, t0 + s0 + row, g) + n]) : 0.f;
                }
                __syncthreads();
#pragma unroll
                for (int kk = 0; kk < kK; ++kk) {
                    float cv[4], bv[4];
#pragma unroll
                    for (int i = 0; i < 4; ++i) cv[i] = cs[ty * 4 + i][kk];
#pragma unroll
                    for (int j = 0; j < 4; ++j) bv[j] = ks[tx * 4 + j][kk];
#pragma unroll
                    for (int i = 0; i < 4; ++i)
#pragma unroll
                        for (int j = 0; j < 4; ++j) sco[i][j] = fmaf(cv[i], bv[j], sco[i][j]);
                }
                __syncthreads();
            }
            // mask and decay: L[t][s] = exp(l_t - l_s) for s <= t, times dt_s
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int t = ty * 4 + i;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int s = tx * 4 + j;
                    const bool keep = (s0 + s <= r0 + t) && (s < srows) && (t < rows);
                    gs[t][s] = keep ? sco[i][j] * __expf(lt[t] - ls[s]) * dts[s] : 0.f;
                }
            }
            for (int i = threadIdx.x; i < kTile * kTile; i += kThreads) {
                const int s = i / kTile, p = i % kTile;
                vs[s][p] = (s < srows && p0 + p < d.P) ? to_f32(x[off_x(d, b, t0 + s0 + s, h) + p0 + p]) : 0.f;
            }
            __syncthreads();
#pragma unroll 4
            for (int s = 0; s < kTile; ++s) {
                float gv[4], xv[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) gv[i] = gs[ty * 4 + i][s];
#pragma unroll
                for (int j = 0; j < 4; ++j) xv[j] = vs[s][tx * 4 + j];
#pragma unroll
                for (int i = 0; i < 4; ++i)
#pragma unroll
                    for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(gv[i], xv[j], acc[i][j]);
            }
            __syncthreads();
        }
        // ---- skip term and store ---------------------------------------------
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int t = ty * 4 + i;
            if (t >= rows) continue;
            const int64_t base = off_x(d, b, t0 + r0 + t, h);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int p = p0 + tx * 4 + j;
                if (p >= d.P) continue;
                const float xv = to_f32(x[base + p]);
                y[base + p] = from_f32<T>(fmaf(Dh, xv, acc[i][j]));
            }
        }
    }
}

}  // namespace

cudaError_t launch_chunk_state_simt(const Dims &d, bool bf16, const void *x, const void *Bm,
                                    const float *w, float *states, cudaStream_t stream) {
    dim3 grid(d.nc, d.H, d.B);
    if (bf16)
        chunk_state_simt_kernel<__nv_bfloat16><<<grid, kThreads, 0, stream>>>(
            d, static_cast<const __nv_bfloat16 *>(x), static_cast<const __nv_bfloat16 *>(Bm), w, states);
    else
        chunk_state_simt_kernel<float><<<grid, kThreads, 0, stream>>>(
            d, static_cast<const float *>(x), static_cast<const float *>(Bm), w, states);
    return cudaGetLastError();
}

cudaError_t launch_chunk_scan_simt(const Dims &d, bool bf16, const void *x, const float *dt,
                                   const void *Bm, const void *Cm, const float *D,
                                   const float *l, const float *s_in, void *y,
                                   cudaStream_t stream) {
    dim3 grid((d.Q + kTile - 1) / kTile, d.nc, d.B * d.H);
    if (bf16)
        chunk_scan_simt_kernel<__nv_bfloat16><<<grid, kThreads, 0, stream>>>(
            d, static_cast<const __nv_bfloat16 *>(x), dt, static_cast<const __nv_bfloat16 *>(Bm),
            static_cast<const __nv_bfloat16 *>(Cm), D, l, s_in, static_cast<__nv_bfloat16 *>(y));
    else
        chunk_scan_simt_kernel<float><<<grid, kThreads, 0, stream>>>(
            d, static_cast<const float *>(x), dt, static_cast<const float *>(Bm),
            static_cast<const float *>(Cm), D, l, s_in, static_cast<float *>(y));
    return cudaGetLastError();
}

}  // namespace ssd
