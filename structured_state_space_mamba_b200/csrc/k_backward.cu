// k_backward.cu -- the element-wise and prefix-sum kernels of the backward
// pass (ssd_backward in ssd_api.cu, which runs the scans themselves).
//
// Reverse mode of h_t = a_t h_{t-1} + dt_t x_t B_t^T, y_t = h_t C_t + D x_t
// (a_t = exp(dt_t A_h)), per (b, h) with G_t = dL/dh_t and K_t = a_t G_t =
// dL/dh_{t-1}:
//   K_t = a_t K_{t+1} + a_t dy_t C_t^T,  K_T = dfinal,  dh0 = K_0
//   dx_t = dt_t G_t B_t + D dy_t,   dB_t = sum_h dt_t G_t^T x_t,   dC_t = sum_h h_t^T dy_t
//   ddt_t = x_t . (G_t B_t) + A R_t,   dA = sum dt_t R_t,   dD = sum dy_t . x_t
// with R_t = K_t : h_{t-1}, which obeys R_0 = dh0 : h0 and
//   R_{t+1} = R_t + c_t - r_t,  c_t = dt_t x_t . (G_t B_t),  r_t = dy_t . (h_t C_t)
// (expand K_{t+1} = K_t / a_t - dy_t C_t^T and h_t = a_t h_{t-1} + dt_t x_t B_t^T
// in K_{t+1} : h_t).  K is the forward recurrence run backwards in time with
// input a_t dy_t / dt_t against C_t (read out against B_t); its transpose gives
// dB; h^T read out against dy gives dC.  These kernels build the scans' inputs
// (reversed in time where needed), and turn the scans' outputs into the
// gradients.  All of them are HBM-bound element-wise passes; the prefix over
// tokens is one warp per (b, h).
#include "common.cuh"
#include "kernels.h"

namespace ssd {

namespace {

constexpr int kThreads = 256;

template <typename T>
__device__ __forceinline__ float ld(const T *p, int64_t i) { return to_f32<T>(p[i]); }

// kVec consecutive elements at a 16-byte aligned address, widened to fp32 on
// load and rounded to the element type on store (the same conversions as the
// scalar ld / from_f32, so either path gives the same values)
constexpr int kVec = 8;
__device__ __forceinline__ void ld8(const float *p, float (&v)[kVec]) {
    const float4 a = __ldg(reinterpret_cast<const float4 *>(p)), b = __ldg(reinterpret_cast<const float4 *>(p) + 1);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}
__device__ __forceinline__ void ld8(const __nv_bfloat16 *p, float (&v)[kVec]) {
    const uint4 a = __ldg(reinterpret_cast<const uint4 *>(p));
    const __nv_bfloat16 *e = reinterpret_cast<const __nv_bfloat16 *>(&a);
#pragma unroll
    for (int i = 0; i < kVec; ++i) v[i] = __bfloat162float(e[i]);
}
__device__ __forceinline__ void ld2(const float *p, float (&v)[2]) {
    const float2 a = *reinterpret_cast<const float2 *>(p);
    v[0] = a.x; v[1] = a.y;
}
__device__ __forceinline__ void ld2(const __nv_bfloat16 *p, float (&v)[2]) {
    const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162 *>(p);
    v[0] = __low2float(a); v[1] = __high2float(a);
}
__device__ __forceinline__ void st2(float *p, const float (&v)[2]) {
    *reinterpret_cast<float2 *>(p) = make_float2(v[0], v[1]);
}
__device__ __forceinline__ void st2(__nv_bfloat16 *p, const float (&v)[2]) {
    __nv_bfloat162 a;
    a.x = __float2bfloat16_rn(v[0]);
    a.y = __float2bfloat16_rn(v[1]);
    *reinterpret_cast<__nv_bfloat162 *>(p) = a;
}
__device__ __forceinline__ void st8(float *p, const float (&v)[kVec]) {
    reinterpret_cast<float4 *>(p)[0] = make_float4(v[0], v[1], v[2], v[3]);
    reinterpret_cast<float4 *>(p)[1] = make_float4(v[4], v[5], v[6], v[7]);
}
__device__ __forceinline__ void st8(__nv_bfloat16 *p, const float (&v)[kVec]) {
    uint4 a;
    __nv_bfloat16 *e = reinterpret_cast<__nv_bfloat16 *>(&a);
#pragma unroll
    for (int i = 0; i < kVec; ++i) e[i] = __float2bfloat16_rn(v[i]);
    *reinterpret_cast<uint4 *>(p) = a;
}

// The row kernels below take one (b, t) row per block, blocks striding over
// the B*T rows; inside a row the indices are 32-bit (a row holds H*N or H*P
// elements).

// scan K (reversed): xr[b,tau,h,p] = a_t dy[b,t,h,p] / dt_t, dtr[b,tau,h] = dt_t,
// and (per group) Br = C, Cr = B, all at tau = T-1-t
template <typename T, typename TS>
__global__ void __launch_bounds__(kThreads)
prep_k_kernel(Dims d, const T *__restrict__ dy, const float *__restrict__ dt, const float *__restrict__ A,
              const T *__restrict__ Bm, const T *__restrict__ Cm, TS *__restrict__ xr, float *__restrict__ dtr,
              TS *__restrict__ Br, TS *__restrict__ Cr, bool vec) {
    for (int64_t row = blockIdx.x; row < int64_t(d.B) * d.T; row += gridDim.x) {
        const int b = int(row / d.T), t = int(row % d.T);
        const int tau = d.T - 1 - t;
        const int64_t sdt = off_dt(d, b, t), ddt_ = off_dt(d, b, tau);
        const int64_t sx = off_x(d, b, t, 0), dx_ = off_x(d, b, tau, 0);
        const int HP = d.H * d.P;
        const int GN = d.G * d.N;
        const int64_t sbc = off_bc(d, b, t, 0), dbc = off_bc(d, b, tau, 0);
        if (vec) {  // headdim and dstate multiples of kVec: whole vectors of one head / group
            for (int k = threadIdx.x * kVec; k < HP; k += blockDim.x * kVec) {
                const int h = k / d.P;
                const float dtt = __ldg(dt + sdt + h);
                const float f = __expf(dtt * __ldg(A + h));
                float v[kVec];
                ld8(dy + sx + k, v);
#pragma unroll
                for (int e = 0; e < kVec; ++e) v[e] = f * v[e] / dtt;
                st8(xr + dx_ + k, v);
            }
            for (int k = threadIdx.x * kVec; k < GN; k += blockDim.x * kVec) {
                float v[kVec];
                ld8(Cm + sbc + k, v);
                st8(Br + dbc + k, v);
                ld8(Bm + sbc + k, v);
                st8(Cr + dbc + k, v);
            }
        } else {
            for (int k = threadIdx.x; k < HP; k += blockDim.x) {
                const int h = k / d.P;
                const float dtt = __ldg(dt + sdt + h);
                xr[dx_ + k] = from_f32<TS>(__expf(dtt * __ldg(A + h)) * ld(dy, sx + k) / dtt);
            }
            for (int k = threadIdx.x; k < GN; k += blockDim.x) {
                Br[dbc + k] = from_f32<TS>(ld(Cm, sbc + k));
                Cr[dbc + k] = from_f32<TS>(ld(Bm, sbc + k));
            }
        }
        for (int h = threadIdx.x; h < d.H; h += blockDim.x) dtr[ddt_ + h] = __ldg(dt + sdt + h);
    }
}

// fp32 copies in the same layout (the scans of the backward run in fp32)
template <typename T>
__global__ void to_f32_kernel(const T *__restrict__ src, float *__restrict__ dst, int64_t n) {
    for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < n; i += int64_t(gridDim.x) * blockDim.x)
        dst[i] = ld(src, i);
}

// the transposed scans' inputs, one value per (b, t, h, n):
//   reversed (dB): xb[b,tau,h,n] = a_t C[b,t,g,n] / dt_t
//   forward  (dC): xc[b,t,h,n]   = B[b,t,g,n]
// and the per-head rows of the reversed ones:
//   dyr[b,tau,h,p] = dy[b,t,h,p],  xrr[b,tau,h,p] = x[b,t,h,p]
template <typename T, typename TS>
__global__ void __launch_bounds__(kThreads)
prep_t_kernel(Dims d, int W, const T *__restrict__ x, const T *__restrict__ dy, const float *__restrict__ dt,
              const float *__restrict__ A, const T *__restrict__ Bm, const T *__restrict__ Cm,
              TS *__restrict__ xb, TS *__restrict__ xc, TS *__restrict__ dyr, TS *__restrict__ xrr, bool vec) {
    // xb and xc are split along dstate into slices of W columns, slice-major:
    // slice s holds [B, T, H, W] (each slice is one transposed scan's x)
    extern __shared__ float f_h[];  // a_t / dt_t of this row, per head
    const int64_t slice = int64_t(d.B) * d.T * d.H * W;
    for (int64_t row = blockIdx.x; row < int64_t(d.B) * d.T; row += gridDim.x) {
        const int b = int(row / d.T), t = int(row % d.T);
        const int tau = d.T - 1 - t;
        const int64_t sdt = off_dt(d, b, t), sbc = off_bc(d, b, t, 0);
        const int64_t rowr = off_dt(d, b, tau) * W, rowf = off_dt(d, b, t) * W;  // (b, t', h = 0) * W
        __syncthreads();  // the previous row's factors are no longer read
        for (int h = threadIdx.x; h < d.H; h += blockDim.x) {
            const float dtt = __ldg(dt + sdt + h);
            f_h[h] = __expf(dtt * __ldg(A + h)) / dtt;
        }
        __syncthreads();
        const int HN = d.H * d.N;
        const int HP = d.H * d.P;
        const int64_t sx = off_x(d, b, t, 0), dx_ = off_x(d, b, tau, 0);
        if (vec) {  // headdim, dstate and W multiples of kVec: a vector stays in one head and slice
            for (int k = threadIdx.x * kVec; k < HN; k += blockDim.x * kVec) {
                const int h = k / d.N, n = k - h * d.N;
                const int g = h / d.r;
                const int sl = n / W, nn = n - sl * W;
                const int64_t o = sl * slice + int64_t(h) * W + nn;
                const float f = f_h[h];
                float v[kVec];
                ld8(Cm + sbc + g * d.N + n, v);
#pragma unroll
                for (int e = 0; e < kVec; ++e) v[e] *= f;
                st8(xb + o + rowr, v);
                ld8(Bm + sbc + g * d.N + n, v);
                st8(xc + o + rowf, v);
            }
            for (int k = threadIdx.x * kVec; k < HP; k += blockDim.x * kVec) {
                float v[kVec];
                ld8(dy + sx + k, v);
                st8(dyr + dx_ + k, v);
                ld8(x + sx + k, v);
                st8(xrr + dx_ + k, v);
            }
            continue;
        }
        for (int k = threadIdx.x; k < HN; k += blockDim.x) {
            const int h = k / d.N, n = k - h * d.N;
            const int g = h / d.r;
            const int sl = n / W, nn = n - sl * W;
            const int64_t o = sl * slice + int64_t(h) * W + nn;
            xb[o + rowr] = from_f32<TS>(f_h[h] * ld(Cm, sbc + g * d.N + n));
            xc[o + rowf] = from_f32<TS>(ld(Bm, sbc + g * d.N + n));
        }
        for (int k = threadIdx.x; k < HP; k += blockDim.x) {
            dyr[dx_ + k] = from_f32<TS>(ld(dy, sx + k));
            xrr[dx_ + k] = from_f32<TS>(ld(x, sx + k));
        }
    }
}

// [B, H, P, N] -> slices of [B, H, W, P] (a state as the transposed scans
// hold it, dstate split into slices of W rows, slice-major)
__global__ void transpose_state_kernel(int64_t BH, int P, int N, int W, const float *__restrict__ s,
                                       float *__restrict__ st) {
    const int64_t total = BH * P * N;
    for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < total;
         i += int64_t(gridDim.x) * blockDim.x) {
        const int n = int(i % N);
        const int64_t r = i / N;
        const int p = int(r % P);
        const int64_t bh = r / P;
        const int sl = n / W, nn = n % W;
        st[sl * BH * W * P + (bh * W + nn) * P + p] = s[i];
    }
}

// one warp per (b, t, h): u = G_t B_t = yk / a_t (yk from the reversed scan),
// dx = dt u + D dy, xu = x . u, c = dt xu, r = dy . yh (yh = h_t C_t), and the
// row's share of dD, dd = dy . x
template <typename T, typename TS>
__global__ void post_k_kernel(Dims d, const T *__restrict__ x, const T *__restrict__ dy,
                              const float *__restrict__ dt, const float *__restrict__ A,
                              const float *__restrict__ D, const TS *__restrict__ yk,
                              const TS *__restrict__ yh, T *__restrict__ dx, float *__restrict__ xu,
                              float *__restrict__ cc, float *__restrict__ rr, float *__restrict__ dd,
                              bool pairs) {
    const int lane = threadIdx.x & 31;
    const int64_t nw = int64_t(d.B) * d.T * d.H;
    for (int64_t w = (blockIdx.x * int64_t(blockDim.x) + threadIdx.x) >> 5; w < nw;
         w += (int64_t(gridDim.x) * blockDim.x) >> 5) {
        const int h = int(w % d.H);
        const int64_t bt = w / d.H;
        const int t = int(bt % d.T), b = int(bt / d.T);
        const int64_t idt = off_dt(d, b, t) + h;
        const float dtt = dt[idt];
        const float inv_a = __expf(-dtt * A[h]);
        const float Dh = D ? D[h] : 0.f;
        const int64_t row = off_x(d, b, t, h);
        const int64_t rowr = off_x(d, b, d.T - 1 - t, h);
        float sx = 0.f, sr = 0.f, sd = 0.f;
        if (pairs) {
            // two adjacent elements per lane (headdim even: 8- and 4-byte aligned pairs)
            for (int p = 2 * lane; p < d.P; p += 64) {
                float uk[2], dyv[2], xv[2], yv[2];
                ld2(yk + rowr + p, uk);
                ld2(dy + row + p, dyv);
                ld2(x + row + p, xv);
                ld2(yh + row + p, yv);
                float o[2];
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const float u = uk[e] * inv_a;
                    o[e] = dtt * u + Dh * dyv[e];
                    sx = fmaf(xv[e], u, sx);
                    sr = fmaf(dyv[e], yv[e], sr);
                    sd = fmaf(dyv[e], xv[e], sd);
                }
                st2(dx + row + p, o);
            }
        } else {
            for (int p = lane; p < d.P; p += 32) {
                const float u = ld(yk, rowr + p) * inv_a;
                const float dyp = ld(dy, row + p), xp = ld(x, row + p);
                dx[row + p] = from_f32<T>(dtt * u + Dh * dyp);
                sx = fmaf(xp, u, sx);
                sr = fmaf(dyp, ld(yh, row + p), sr);
                sd = fmaf(dyp, xp, sd);
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            sx += __shfl_xor_sync(0xffffffffu, sx, o);
            sr += __shfl_xor_sync(0xffffffffu, sr, o);
            sd += __shfl_xor_sync(0xffffffffu, sd, o);
        }
        if (lane == 0) {
            xu[idt] = sx;
            cc[idt] = dtt * sx;
            rr[idt] = sr;
            dd[idt] = sd;
        }
    }
}

// one block per (b, h): R0 = dh0 : h0 (0 without an initial state)
__global__ void r0_kernel(int64_t BH, int PN, const float *__restrict__ dh0, const float *__restrict__ h0,
                          float *__restrict__ R0) {
    __shared__ float red[kThreads / 32];
    const int64_t bh = blockIdx.x;
    float s = 0.f;
    if (h0)
        for (int i = threadIdx.x; i < PN; i += blockDim.x) s = fmaf(dh0[bh * PN + i], h0[bh * PN + i], s);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = s;
    __syncthreads();
    if (threadIdx.x == 0) {
        float t = 0.f;
        for (int i = 0; i < kThreads / 32; ++i) t += red[i];
        R0[bh] = t;
    }
}

// one warp per (b, h): R over the tokens in blocks of 32 (a warp prefix sum of
// c - r), ddt_t = xu_t + A R_t, and this (b, h)'s shares of dA = sum dt_t R_t
// and of dD = sum dd_t
__global__ void prefix_kernel(Dims d, const float *__restrict__ dt, const float *__restrict__ A,
                              const float *__restrict__ R0, const float *__restrict__ xu,
                              const float *__restrict__ cc, const float *__restrict__ rr,
                              const float *__restrict__ dd, float *__restrict__ ddt, float *__restrict__ dA_part,
                              float *__restrict__ dD_part) {
    const int lane = threadIdx.x & 31;
    const int64_t nw = int64_t(d.B) * d.H;
    for (int64_t w = (blockIdx.x * int64_t(blockDim.x) + threadIdx.x) >> 5; w < nw;
         w += (int64_t(gridDim.x) * blockDim.x) >> 5) {
        const int h = int(w % d.H), b = int(w / d.H);
        const float a_h = A[h];
        float R = R0[w];  // R at the first token of the block
        float sA = 0.f, sD = 0.f;
        for (int t0 = 0; t0 < d.T; t0 += 32) {
            const int t = t0 + lane;
            const bool in = t < d.T;
            const int64_t i = off_dt(d, b, in ? t : 0) + h;
            const float step = in ? cc[i] - rr[i] : 0.f;
            // exclusive prefix of the steps: R_t = R + sum_{t0 <= k < t} (c_k - r_k)
            float incl = step;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float nb = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += nb;
            }
            const float Rt = R + incl - step;
            if (in) {
                ddt[i] = xu[i] + a_h * Rt;
                sA = fmaf(dt[i], Rt, sA);
                sD += dd[i];
            }
            R += __shfl_sync(0xffffffffu, incl, 31);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            sA += __shfl_xor_sync(0xffffffffu, sA, o);
            sD += __shfl_xor_sync(0xffffffffu, sD, o);
        }
        if (lane == 0) {
            dA_part[w] = sA;
            dD_part[w] = sD;
        }
    }
}

// dA[h] = sum_b dA_part[b, h]; dD[h] = sum_b dD_part[b, h]   (one thread per head)
__global__ void head_sums_kernel(Dims d, const float *__restrict__ dA_part, const float *__restrict__ dD_part,
                                 float *__restrict__ dA, float *__restrict__ dD) {
    const int h = blockIdx.x * blockDim.x + threadIdx.x;
    if (h >= d.H) return;
    float a = 0.f, s = 0.f;
    for (int b = 0; b < d.B; ++b) {
        a += dA_part[int64_t(b) * d.H + h];
        s += dD_part[int64_t(b) * d.H + h];
    }
    dA[h] = a;
    if (dD) dD[h] = s;
}

// dB[b,t,g,n] = sum_{h in g} (dt_t / a_t) yb[b,T-1-t,h,n];  dC[b,t,g,n] = sum_{h in g} yc[b,t,h,n]
// the heads of a group are split over kParts threads per output (partial sums
// combined in shared memory), so each row keeps kThreads loads in flight
constexpr int kParts = 4;
template <typename T, typename TS>
__global__ void __launch_bounds__(kThreads)
group_sums_kernel(Dims d, int W, const float *__restrict__ dt, const float *__restrict__ A,
                  const TS *__restrict__ yb, const TS *__restrict__ yc, T *__restrict__ dB, T *__restrict__ dC,
                  bool vec) {
    constexpr int kCols = kThreads / kParts;  // outputs per pass
    __shared__ float red_b[kParts][kCols], red_c[kParts][kCols];
    __shared__ float4 red8_b[kThreads][2], red8_c[kThreads][2];
    const int64_t slice = int64_t(d.B) * d.T * d.H * W;
    const int col = threadIdx.x % kCols, part = threadIdx.x / kCols;
    for (int64_t row = blockIdx.x; row < int64_t(d.B) * d.T; row += gridDim.x) {
        const int b = int(row / d.T), t = int(row % d.T);
        const int tau = d.T - 1 - t;
        const int64_t sdt = off_dt(d, b, t), obc = off_bc(d, b, t, 0);
        const int64_t rowr = off_dt(d, b, tau) * W, rowf = off_dt(d, b, t) * W;
        const int GN = d.G * d.N;
        if (vec) {
            // kVec consecutive outputs (one group, one slice) per thread; the
            // row's GN / kVec vectors take `cols` threads, the heads of a group
            // are split over `parts` = kThreads / cols of them (partial sums
            // combined in shared memory, in part order)
            const int nv = GN / kVec;
            const int cols = nv < kThreads ? nv : kThreads;
            const int parts = kThreads / cols;
            const int vcol = threadIdx.x % cols, vpart = threadIdx.x / cols;
            for (int v0 = 0; v0 < nv; v0 += cols) {
                const int v = v0 + vcol;
                const bool act = vpart < parts && v < nv;
                float sb[kVec] = {}, sc[kVec] = {};
                if (act) {
                    const int k = v * kVec;
                    const int g = k / d.N, n = k - g * d.N;
                    const int sl = n / W, nn = n - sl * W;
                    const int64_t o = sl * slice + nn;
                    for (int j = vpart; j < d.r; j += parts) {
                        const int h = g * d.r + j;
                        const float dtt = __ldg(dt + sdt + h);
                        const float f = dtt * __expf(-dtt * __ldg(A + h));
                        float vb[kVec], vc[kVec];
                        ld8(yb + o + rowr + int64_t(h) * W, vb);
                        ld8(yc + o + rowf + int64_t(h) * W, vc);
#pragma unroll
                        for (int e = 0; e < kVec; ++e) {
                            sb[e] = fmaf(f, vb[e], sb[e]);
                            sc[e] += vc[e];
                        }
                    }
                }
                red8_b[threadIdx.x][0] = make_float4(sb[0], sb[1], sb[2], sb[3]);
                red8_b[threadIdx.x][1] = make_float4(sb[4], sb[5], sb[6], sb[7]);
                red8_c[threadIdx.x][0] = make_float4(sc[0], sc[1], sc[2], sc[3]);
                red8_c[threadIdx.x][1] = make_float4(sc[4], sc[5], sc[6], sc[7]);
                __syncthreads();
                if (vpart == 0 && v < nv) {
                    float tb[kVec] = {}, tc[kVec] = {};
                    for (int q = 0; q < parts; ++q)
#pragma unroll
                        for (int hh = 0; hh < 2; ++hh) {
                            const float4 b4 = red8_b[q * cols + vcol][hh], c4 = red8_c[q * cols + vcol][hh];
                            tb[4 * hh] += b4.x; tb[4 * hh + 1] += b4.y; tb[4 * hh + 2] += b4.z; tb[4 * hh + 3] += b4.w;
                            tc[4 * hh] += c4.x; tc[4 * hh + 1] += c4.y; tc[4 * hh + 2] += c4.z; tc[4 * hh + 3] += c4.w;
                        }
                    st8(dB + obc + int64_t(v) * kVec, tb);
                    st8(dC + obc + int64_t(v) * kVec, tc);
                }
                __syncthreads();
            }
            continue;
        }
        for (int k0 = 0; k0 < GN; k0 += kCols) {
            const int k = k0 + col;
            float sb = 0.f, sc = 0.f;
            if (k < GN) {
                const int g = k / d.N, n = k - g * d.N;
                const int sl = n / W, nn = n - sl * W;
                const int64_t o = sl * slice + nn;
                for (int j = part; j < d.r; j += kParts) {
                    const int h = g * d.r + j;
                    const float dtt = __ldg(dt + sdt + h);
                    const float f = dtt * __expf(-dtt * __ldg(A + h));
                    sb = fmaf(f, ld(yb, o + rowr + int64_t(h) * W), sb);
                    sc += ld(yc, o + rowf + int64_t(h) * W);
                }
            }
            red_b[part][col] = sb;
            red_c[part][col] = sc;
            __syncthreads();
            if (part == 0 && k < GN) {
                float tb = 0.f, tc = 0.f;
#pragma unroll
                for (int q = 0; q < kParts; ++q) {
                    tb += red_b[q][col];
                    tc += red_c[q][col];
                }
                dB[obc + k] = from_f32<T>(tb);
                dC[obc + k] = from_f32<T>(tc);
            }
            __syncthreads();
        }
    }
}

unsigned grid_for(int64_t n) {
    const int64_t g = (n + kThreads - 1) / kThreads;
    return unsigned(g < 148 * 32 ? (g < 1 ? 1 : g) : 148 * 32);
}
// blocks for the row kernels (one row per block, striding)
unsigned grid_rows(const Dims &d) {
    const int64_t rows = int64_t(d.B) * d.T;
    return unsigned(rows < 148 * 64 ? (rows < 1 ? 1 : rows) : 148 * 64);
}

template <typename T, typename TS>
cudaError_t backward_prep_t(const Dims &d, const void *x, const void *dy, const float *dt, const float *A,
                            const void *Bm, const void *Cm, const BackwardBuffers &w, cudaStream_t s) {
    const T *xx = static_cast<const T *>(x), *dyy = static_cast<const T *>(dy);
    const T *bb = static_cast<const T *>(Bm), *cc = static_cast<const T *>(Cm);
    const int64_t nx = int64_t(d.B) * d.T * d.H * d.P, nbc = int64_t(d.B) * d.T * d.G * d.N;
    // whole 16-byte vectors where every row, head and slice starts on one
    const bool vec = d.P % kVec == 0 && d.N % kVec == 0 && w.W % kVec == 0;
    prep_k_kernel<T, float><<<grid_rows(d), kThreads, 0, s>>>(d, dyy, dt, A, bb, cc, w.xk, w.dtr, w.bk,
                                                                    w.ck, vec);
    prep_t_kernel<T, TS><<<grid_rows(d), kThreads, size_t(d.H) * sizeof(float), s>>>(d, w.W, xx, dyy, dt, A, bb, cc,
                                                                static_cast<TS *>(w.xb), static_cast<TS *>(w.xc),
                                                                static_cast<TS *>(w.dyr), static_cast<TS *>(w.xrr),
                                                                vec);
    if (w.xf) to_f32_kernel<T><<<grid_for(nx), kThreads, 0, s>>>(xx, w.xf, nx);
    if (w.dyf) to_f32_kernel<T><<<grid_for(nx), kThreads, 0, s>>>(dyy, w.dyf, nx);
    if (w.bf) to_f32_kernel<T><<<grid_for(nbc), kThreads, 0, s>>>(bb, w.bf, nbc);
    if (w.cf) to_f32_kernel<T><<<grid_for(nbc), kThreads, 0, s>>>(cc, w.cf, nbc);
    return cudaGetLastError();
}

template <typename T, typename TS>
cudaError_t backward_post_t(const Dims &d, const void *x, const void *dy, const float *dt, const float *A,
                            const float *D, const float *h0, const BackwardBuffers &w, void *dx, float *ddt,
                            float *dA, void *dB, void *dC, float *dD, cudaStream_t s) {
    const T *xx = static_cast<const T *>(x), *dyy = static_cast<const T *>(dy);
    const int64_t nw = int64_t(d.B) * d.T * d.H;
    const int64_t BH = int64_t(d.B) * d.H;
    post_k_kernel<T, float><<<grid_for(nw * 32), kThreads, 0, s>>>(d, xx, dyy, dt, A, D, w.yk, w.yh,
                                                                  static_cast<T *>(dx), w.xu, w.cc, w.rr, w.dd,
                                                                  d.P % 2 == 0);
    r0_kernel<<<unsigned(BH), kThreads, 0, s>>>(BH, d.P * d.N, w.dh0, h0, w.R0);
    prefix_kernel<<<grid_for(BH * 32), kThreads, 0, s>>>(d, dt, A, w.R0, w.xu, w.cc, w.rr, w.dd, ddt, w.dA_part,
                                                         w.dD_part);
    head_sums_kernel<<<unsigned((d.H + kThreads - 1) / kThreads), kThreads, 0, s>>>(d, w.dA_part, w.dD_part, dA,
                                                                                       dD);
    group_sums_kernel<T, TS><<<grid_rows(d), kThreads, 0, s>>>(
        d, w.W, dt, A, static_cast<const TS *>(w.yb), static_cast<const TS *>(w.yc), static_cast<T *>(dB),
        static_cast<T *>(dC), d.N % kVec == 0 && w.W % kVec == 0);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_backward_prep(const Dims &d, bool bf16, const void *x, const void *dy, const float *dt,
                                 const float *A, const void *Bm, const void *Cm, const BackwardBuffers &w,
                                 cudaStream_t stream) {
    if (!bf16) return backward_prep_t<float, float>(d, x, dy, dt, A, Bm, Cm, w, stream);
    return w.scan_bf16 ? backward_prep_t<__nv_bfloat16, __nv_bfloat16>(d, x, dy, dt, A, Bm, Cm, w, stream)
                       : backward_prep_t<__nv_bfloat16, float>(d, x, dy, dt, A, Bm, Cm, w, stream);
}

cudaError_t launch_transpose_state(int64_t BH, int P, int N, int W, const float *s, float *st, cudaStream_t stream) {
    transpose_state_kernel<<<grid_for(BH * P * N), kThreads, 0, stream>>>(BH, P, N, W, s, st);
    return cudaGetLastError();
}

cudaError_t launch_backward_post(const Dims &d, bool bf16, const void *x, const void *dy, const float *dt,
                                 const float *A, const float *D, const float *h0, const BackwardBuffers &w,
                                 void *dx, float *ddt, float *dA, void *dB, void *dC, float *dD,
                                 cudaStream_t stream) {
    if (!bf16) return backward_post_t<float, float>(d, x, dy, dt, A, D, h0, w, dx, ddt, dA, dB, dC, dD, stream);
    return w.scan_bf16
               ? backward_post_t<__nv_bfloat16, __nv_bfloat16>(d, x, dy, dt, A, D, h0, w, dx, ddt, dA, dB, dC, dD,
                                                               stream)
               : backward_post_t<__nv_bfloat16, float>(d, x, dy, dt, A, D, h0, w, dx, ddt, dA, dB, dC, dD, stream);
}

}  // namespace ssd
