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
#include "tma_host.h"

namespace ssd {

namespace {

constexpr int kThreads = 256;  // 16 x 16 threads, 4 x 4 outputs each -> 64 x 64 tiles
constexpr int kTile = 64;
constexpr int kK = 16;

// ---------------------------------------------------------------------------
// chunk state: one block per (c, h, b); loops over 64 x 64 tiles of P x N.
// K (the chunk's tokens) runs in slices of kK through two shared-memory
// buffers: the next slice's global loads are in flight in registers while the
// current one is multiplied (16-byte operand loads, one barrier per slice).
// ---------------------------------------------------------------------------
constexpr int kLd = kTile + 4;  // row stride (floats) of the [k][i] operand tiles

__device__ __forceinline__ void fma44(float (&acc)[4][4], const float4 a, const float4 b) {
    const float av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
}

template <typename T>
__global__ void __launch_bounds__(kThreads)
chunk_state_simt_kernel(Dims d, const T *__restrict__ x, const T *__restrict__ Bm,
                        const float *__restrict__ w, float *__restrict__ states) {
    __shared__ __align__(16) float xs[2][kK][kLd];  // [token][p], weighted by w
    __shared__ __align__(16) float bs[2][kK][kLd];  // [token][n]
    constexpr int kPer = kK * kTile / kThreads;     // staged elements per thread and operand
    const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int g = h / d.r;
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
    const int t0 = c * d.Q;
    const float *wc = w + off_lq(d, b, h, c);
    float *Sc = states + off_state(d, b, c, h);
    for (int p0 = 0; p0 < d.P; p0 += kTile)
        for (int n0 = 0; n0 < d.N; n0 += kTile) {
            float acc[4][4] = {};
            float px[kPer], pb[kPer];
            // this thread stages column j of rows kb, kb + 4, ... of each slice
            const int j = threadIdx.x % kTile, kb = threadIdx.x / kTile;
            const bool pin = p0 + j < d.P, nin = n0 + j < d.N;
            const T *xcol = x + off_x(d, b, t0, h) + p0 + j;
            const T *bcol = Bm + off_bc(d, b, t0, g) + n0 + j;
            const int64_t xstride = int64_t(d.H) * d.P, bstride = int64_t(d.G) * d.N;
            auto fetch = [&](int k0) {
#pragma unroll
                for (int q = 0; q < kPer; ++q) {
                    const int kk = k0 + kb + q * (kThreads / kTile);
                    const bool tin = kk < d.Q;
                    const float wt = tin ? __ldg(wc + kk) : 0.f;
                    px[q] = (tin && pin) ? wt * to_f32(xcol[kk * xstride]) : 0.f;
                    pb[q] = (tin && nin) ? to_f32(bcol[kk * bstride]) : 0.f;
                }
            };
            auto put = [&](int buf) {
#pragma unroll
                for (int q = 0; q < kPer; ++q) {
                    xs[buf][kb + q * (kThreads / kTile)][j] = px[q];
                    bs[buf][kb + q * (kThreads / kTile)][j] = pb[q];
                }
            };
            __syncthreads();  // the previous tile's last slice is no longer read
            fetch(0);
            put(0);
            __syncthreads();
            int buf = 0;
            for (int k0 = 0; k0 < d.Q; k0 += kK) {
                const bool more = k0 + kK < d.Q;
                if (more) fetch(k0 + kK);
#pragma unroll
                for (int kk = 0; kk < kK; ++kk)
                    fma44(acc, *reinterpret_cast<const float4 *>(&xs[buf][kk][ty * 4]),
                          *reinterpret_cast<const float4 *>(&bs[buf][kk][tx * 4]));
                if (more) put(buf ^ 1);
                __syncthreads();
                buf ^= 1;
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
// chunk scan: one block per (64-row tile of the chunk, c, b, block of hpc heads
// of one group).  The scores C_t . B_s do not depend on the head, so they are
// computed once per block into shared memory (scores[s][t]); per head and per
// 64-column slice of P, the state term and the masked, decayed product follow.
// Every shared-memory operand is laid out [k][i] with rows of kLd floats, so
// each thread's four values of a k step are one 16-byte load (one of the two
// operands is the same for the 16 threads of a half-warp: a broadcast).
// ---------------------------------------------------------------------------
struct ScanSmemSimt {
    int scores, pt, xs, ak, bk, lt, ls, dts, total;  // float offsets
};
__host__ __device__ inline ScanSmemSimt simt_scan_smem(int Q) {
    ScanSmemSimt m;
    m.scores = 0;                     // [Q][64]    C_t . B_s as [s][t] (whole-row float4 access: no padding)
    m.pt = m.scores + Q * kTile;      // [64][kLd]  masked, decayed scores of one source block, [s][t]
    m.xs = m.pt + kTile * kLd;        // [64][kLd]  x rows of one source block, [s][p]
    m.ak = m.xs + kTile * kLd;        // [kK][kLd]  C slice, [n][t]
    m.bk = m.ak + kK * kLd;           // [kK][kLd]  B slice [n][s] or s_in slice [n][p]
    m.lt = m.bk + kK * kLd;           // [64]       l of the tile's rows
    m.ls = m.lt + kTile;              // [Q]        l of the sources
    m.dts = m.ls + Q;                 // [Q]        dt of the sources
    m.total = m.dts + Q;
    return m;
}

// A kK-column slice [k0, k0 + kK) of `nrows` rows (row r at src + r * stride,
// columns < ncols; zero outside), staged transposed into dst[k][r]: thread i
// takes row i / 4 and four consecutive columns.  fetch_slice loads them into
// registers (so the loads of the next slice are in flight during a multiply),
// put_slice stores them.
template <typename T>
__device__ __forceinline__ void fetch_slice(float (&r)[4], const T *src, int64_t stride, int nrows, int k0,
                                            int ncols) {
    const int row = threadIdx.x >> 2, kq = (threadIdx.x & 3) * 4;
    const T *p = src + int64_t(row) * stride;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const int n = k0 + kq + j;
        r[j] = (row < nrows && n < ncols) ? to_f32(p[n]) : 0.f;
    }
}
__device__ __forceinline__ void put_slice(float *dst, const float (&r)[4]) {
    const int row = threadIdx.x >> 2, kq = (threadIdx.x & 3) * 4;
#pragma unroll
    for (int j = 0; j < 4; ++j) dst[(kq + j) * kLd + row] = r[j];
}

// three blocks per SM where shared memory allows (64-token chunks: 60 KB each;
// two at chunk length 256, 109 KB each): 80 registers, 3 % faster on the
// backward's 64-token scans than two blocks with 128
template <typename T>
__global__ void __launch_bounds__(kThreads, 3)
chunk_scan_simt_kernel(Dims d, int hpc, const T *__restrict__ x, const float *__restrict__ dt,
                       const T *__restrict__ Bm, const T *__restrict__ Cm,
                       const float *__restrict__ Dskip, const float *__restrict__ l,
                       const float *__restrict__ s_in, T *__restrict__ y) {
    extern __shared__ float4 smem_f4[];
    float *sm = reinterpret_cast<float *>(smem_f4);
    const int Q = d.Q;
    const ScanSmemSimt L = simt_scan_smem(Q);
    float *scores = sm + L.scores, *pt = sm + L.pt, *xs = sm + L.xs, *ak = sm + L.ak, *bk = sm + L.bk;
    float *lt = sm + L.lt, *ls = sm + L.ls, *dts = sm + L.dts;
    const int mt = blockIdx.x, c = blockIdx.y;
    const int nhb = d.H / hpc;
    const int b = blockIdx.z / nhb, hfirst = (blockIdx.z % nhb) * hpc;
    const int g = hfirst / d.r;
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
    const int t0 = c * Q;          // first token of the chunk
    const int r0 = mt * kTile;     // first row (within the chunk) of this tile
    const int rows = min(kTile, Q - r0);
    const int s_len = r0 + rows;   // sources [0, s_len) of the chunk
    const int64_t bc_stride = int64_t(d.G) * d.N;
    const T *crow = Cm + off_bc(d, b, t0 + r0, g);  // C of the tile's first row

    // ---- 1. scores[s][t] = C_t . B_s, t <- tx, s <- ty ----------------------
    float ra[4], rb[4];  // the next slice, in flight
    for (int s0 = 0; s0 < s_len; s0 += kTile) {
        const int scols = min(kTile, s_len - s0);
        const T *brow = Bm + off_bc(d, b, t0 + s0, g);
        float acc[4][4] = {};
        fetch_slice(ra, crow, bc_stride, rows, 0, d.N);
        fetch_slice(rb, brow, bc_stride, scols, 0, d.N);
        for (int k0 = 0; k0 < d.N; k0 += kK) {
            put_slice(ak, ra);
            put_slice(bk, rb);
            __syncthreads();
            if (k0 + kK < d.N) {
                fetch_slice(ra, crow, bc_stride, rows, k0 + kK, d.N);
                fetch_slice(rb, brow, bc_stride, scols, k0 + kK, d.N);
            }
#pragma unroll
            for (int kk = 0; kk < kK; ++kk)
                fma44(acc, *reinterpret_cast<const float4 *>(ak + kk * kLd + tx * 4),
                      *reinterpret_cast<const float4 *>(bk + kk * kLd + ty * 4));
            __syncthreads();
        }
#pragma unroll
        for (int j = 0; j < 4; ++j)
            if (ty * 4 + j < scols)
                *reinterpret_cast<float4 *>(scores + (s0 + ty * 4 + j) * kTile + tx * 4) =
                    make_float4(acc[0][j], acc[1][j], acc[2][j], acc[3][j]);
    }

    for (int hi = 0; hi < hpc; ++hi) {
        const int h = hfirst + hi;
        const float *lc = l + off_lq(d, b, h, c);
        const float *sc = s_in + off_state(d, b, c, h);
        const float Dh = Dskip ? __ldg(Dskip + h) : 0.f;
        __syncthreads();  // the previous head's l / dt are no longer read
        for (int i = threadIdx.x; i < s_len; i += kThreads) {
            ls[i] = __ldg(lc + i);
            dts[i] = __ldg(dt + off_dt(d, b, t0 + i) + h);
        }
        if (threadIdx.x < kTile) lt[threadIdx.x] = threadIdx.x < rows ? __ldg(lc + r0 + threadIdx.x) : 0.f;
        __syncthreads();
        for (int p0 = 0; p0 < d.P; p0 += kTile) {
            const int pcols = min(kTile, d.P - p0);
            float acc[4][4] = {};  // t <- ty, p <- tx
            // ---- 2. state term: exp(l_t) C_t . s_in[p, :] -----------------------
            const float *srow = sc + int64_t(p0) * d.N;
            fetch_slice(ra, crow, bc_stride, rows, 0, d.N);
            fetch_slice(rb, srow, int64_t(d.N), pcols, 0, d.N);
            for (int k0 = 0; k0 < d.N; k0 += kK) {
                put_slice(ak, ra);
                put_slice(bk, rb);
                __syncthreads();
                if (k0 + kK < d.N) {
                    fetch_slice(ra, crow, bc_stride, rows, k0 + kK, d.N);
                    fetch_slice(rb, srow, int64_t(d.N), pcols, k0 + kK, d.N);
                }
#pragma unroll
                for (int kk = 0; kk < kK; ++kk)
                    fma44(acc, *reinterpret_cast<const float4 *>(ak + kk * kLd + ty * 4),
                          *reinterpret_cast<const float4 *>(bk + kk * kLd + tx * 4));
                __syncthreads();
            }
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float e = __expf(lt[ty * 4 + i]);
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] *= e;
            }
            // ---- 3. intra-chunk term, 64 source tokens at a time ------------------
            // this thread's x values of a source block: s = e / 64, p = e % 64 for
            // e = threadIdx.x + kThreads q; the next block's are loaded during
            // the current block's multiply
            constexpr int kXPer = kTile * kTile / kThreads;
            float rx[kXPer];
            auto fetch_x = [&](int s0) {
                const int scols = min(kTile, s_len - s0);
#pragma unroll
                for (int q = 0; q < kXPer; ++q) {
                    const int e = threadIdx.x + q * kThreads;
                    const int s = e >> 6, p = e & 63;
                    rx[q] = (s < scols && p < pcols) ? to_f32(x[off_x(d, b, t0 + s0 + s, h) + p0 + p]) : 0.f;
                }
            };
            fetch_x(0);
            for (int s0 = 0; s0 < s_len; s0 += kTile) {
                const int scols = min(kTile, s_len - s0);
                // masked, decayed scores: exp(l_t - l_s) dt_s (C_t . B_s) for s <= t
                for (int e = threadIdx.x; e < kTile * (kTile / 4); e += kThreads) {
                    const int s = e >> 4, tq = (e & 15) * 4;
                    const float4 v = s < scols ? *reinterpret_cast<const float4 *>(scores + (s0 + s) * kTile + tq)
                                               : make_float4(0.f, 0.f, 0.f, 0.f);
                    const float vv[4] = {v.x, v.y, v.z, v.w};
                    float o[4];
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const int t = tq + q;
                        const bool keep = s < scols && s0 + s <= r0 + t && t < rows;
                        o[q] = keep ? vv[q] * __expf(lt[t] - ls[s0 + s]) * dts[s0 + s] : 0.f;
                    }
                    *reinterpret_cast<float4 *>(pt + s * kLd + tq) = make_float4(o[0], o[1], o[2], o[3]);
                }
#pragma unroll
                for (int q = 0; q < kXPer; ++q) {
                    const int e = threadIdx.x + q * kThreads;
                    xs[(e >> 6) * kLd + (e & 63)] = rx[q];
                }
                __syncthreads();
                if (s0 + kTile < s_len) fetch_x(s0 + kTile);
#pragma unroll 8
                for (int s = 0; s < kTile; ++s)
                    fma44(acc, *reinterpret_cast<const float4 *>(pt + s * kLd + ty * 4),
                          *reinterpret_cast<const float4 *>(xs + s * kLd + tx * 4));
                __syncthreads();
            }
            // ---- 4. skip term and store ---------------------------------------
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int t = ty * 4 + i;
                if (t >= rows) continue;
                const int64_t base = off_x(d, b, t0 + r0 + t, h) + p0;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int p = tx * 4 + j;
                    if (p >= pcols) continue;
                    y[base + p] = from_f32<T>(fmaf(Dh, to_f32(x[base + p]), acc[i][j]));
                }
            }
        }
    }
}

// heads per block of the CUDA-core scan: the largest divisor of H / G up to 8
int simt_heads_per_block(const Dims &d) {
    int best = 1;
    for (int k = 1; k <= 8; ++k)
        if (d.r % k == 0) best = k;
    return best;
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
    const int hpc = simt_heads_per_block(d);
    dim3 grid((d.Q + kTile - 1) / kTile, d.nc, d.B * (d.H / hpc));
    const int smem = simt_scan_smem(d.Q).total * int(sizeof(float));
    if (bf16) {
        if (!smem_attr_once(reinterpret_cast<const void *>(chunk_scan_simt_kernel<__nv_bfloat16>), smem))
            return cudaErrorInvalidValue;
        chunk_scan_simt_kernel<__nv_bfloat16><<<grid, kThreads, smem, stream>>>(
            d, hpc, static_cast<const __nv_bfloat16 *>(x), dt, static_cast<const __nv_bfloat16 *>(Bm),
            static_cast<const __nv_bfloat16 *>(Cm), D, l, s_in, static_cast<__nv_bfloat16 *>(y));
    } else {
        if (!smem_attr_once(reinterpret_cast<const void *>(chunk_scan_simt_kernel<float>), smem))
            return cudaErrorInvalidValue;
        chunk_scan_simt_kernel<float><<<grid, kThreads, smem, stream>>>(
            d, hpc, static_cast<const float *>(x), dt, static_cast<const float *>(Bm),
            static_cast<const float *>(Cm), D, l, s_in, static_cast<float *>(y));
    }
    return cudaGetLastError();
}

}  // namespace ssd
