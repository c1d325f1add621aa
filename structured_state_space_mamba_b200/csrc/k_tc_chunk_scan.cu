// k_tc_chunk_scan.cu -- ssd_chunk_scan on the 5th-generation tensor cores.
//
// For the rows t of one 128-token tile of chunk c (batch b, head h, group g):
//     y_t[p] = exp(l_t) sum_n C_t[n] s_in[p, n]                      (state term)
//            + sum_{s <= t} exp(l_t - l_s) dt_s (C_t . B_s) x_s[p]     (intra-chunk)
//            + D_h x_t[p]                                              (skip)
// i.e. Y = (L o C B^T)(dt o X) + diag(exp(l)) C s_in^T + D X: the intra-chunk
// "attention-like" product with the 1-semiseparable decay mask
// L[t,s] = exp(l_t - l_s) (akillness.github.io "State Space Duality and
// Mamba-2", "The Scalar-Identity Structural Constraint"; aifetchly blog
// "Mamba-2 Architecture", "The Chunked SSD Algorithm", step 1) plus the
// low-rank contribution of the state carried in from earlier chunks.
//
// One CTA = one 128-row tile x a block of heads sharing a group:
//   1. TMA: C tile [128 x N], B rows [0, s_len) x N (K-major, swizzled).
//   2. UMMA  CB = C B^T  (M=128, N=s_len, K=N) -> tensor memory, once for
//      every head of the block.
//   3. per head: TMA x rows [0, s_len) and s_in [64 x N]; eight warps turn CB
//      (tcgen05.ld) into bf16 scores CB * exp(l_t - l_s) * dt_s (s <= t) in
//      shared memory; UMMA  Y = scores . X (K = s_len) and Z = C s_in^T (K = N)
//      -> tensor memory; epilogue y = Y + exp(l_t) Z + D x, rounded to bf16.
// The scores take exp(l_t - l_s) per element, so every decay range is exact:
// in list mode (one CTA per SM walking packed (b, c, tile, head) items) this
// kernel finishes the tiles that the chunk-wide scan left as steep where the
// block-factored kernel has no shared-memory plan (dstate 256).
#include "common.cuh"
#include "kernels.h"
#include "tc_common.cuh"
#include "tma_host.h"

namespace ssd {

namespace {

using namespace tc;

constexpr int kThreads = 256;
constexpr int kRows = 128;       // rows (tokens t) per tile
constexpr int kTmemCols = 512;
constexpr int kColY = 256, kColZ = 320;

__host__ __device__ constexpr int row_bytes(int n) { return n >= 64 ? 128 : n * 2; }
__host__ __device__ constexpr uint32_t kmajor_swz(int n) { return n >= 64 ? kSw128 : (n == 32 ? kSw64 : kSw32); }

struct ScanSmem {
    uint32_t c_off, r1_off, x_off, s_off, p_off, l_off, dt_off, bar_off, total;
};

__host__ __device__ inline ScanSmem scan_smem(int Q, int N) {
    ScanSmem s;
    const uint32_t size_c = kRows * N * 2;
    const uint32_t size_b = Q * N * 2;
    const uint32_t size_x = Q * 128;
    const uint32_t size_s = 64 * N * 2;
    const uint32_t size_p = kRows * Q * 2;
    const uint32_t r1 = size_b > size_x + size_s + size_p ? size_b : size_x + size_s + size_p;
    s.c_off = 0;
    s.r1_off = size_c;
    s.x_off = s.r1_off;
    s.s_off = s.x_off + size_x;
    s.p_off = s.s_off + size_s;
    s.l_off = s.r1_off + r1;
    s.dt_off = s.l_off + Q * 4;
    s.bar_off = s.dt_off + Q * 4;
    s.total = s.bar_off + 64 + 1024;  // + alignment slack
    return s;
}

// K-major operand descriptor for K step k of a tile whose rows are split
// into 64-column slabs of `rows` rows each (N >= 64), or a single slab of
// narrower rows (N = 16, 32).
__device__ __forceinline__ uint64_t kmajor_desc(uint32_t base, int k, int rows, int n) {
    if (n >= 64)
        return smem_desc(base + (k >> 2) * rows * 128 + (k & 3) * 32, 16, 1024, kSw128);
    return smem_desc(base + k * 32, 16, 8 * row_bytes(n), kmajor_swz(n));
}

template <int N>
__global__ void __launch_bounds__(kThreads, 1)
chunk_scan_tc_kernel(const __grid_constant__ CUtensorMap tm_c, const __grid_constant__ CUtensorMap tm_b,
                     const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_s,
                     Dims d, int hpc, const float *__restrict__ dt, const float *__restrict__ Dskip,
                     const float *__restrict__ lcum, __nv_bfloat16 *__restrict__ y,
                     const long long *__restrict__ items, const int *__restrict__ nitems, int max_items,
                     unsigned int *err) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int Q = d.Q;
    const ScanSmem L = scan_smem(Q, N);
    uint8_t *sC = smem + L.c_off;
    uint8_t *sB = smem + L.r1_off;
    uint8_t *sX = smem + L.x_off;
    uint8_t *sS = smem + L.s_off;
    uint8_t *sP = smem + L.p_off;
    float *sl = reinterpret_cast<float *>(smem + L.l_off);
    float *sdt = reinterpret_cast<float *>(smem + L.dt_off);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L.bar_off);  // ld, cb, x, mma, drain
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(bars + 5);
    __shared__ int s_abort;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int qd = warp & 3, half = warp >> 2;
    const int t_local = qd * 32 + lane;               // this thread's row within the tile
    // units: the grid's one (b, c, tile, head block), or in list mode the listed
    // items blockIdx.x, blockIdx.x + gridDim.x, ... (one head each)
    int nunits = 1;
    if (items) {
        const unsigned int err_word = err ? *reinterpret_cast<const volatile unsigned int *>(err) : 0u;
        const int listed = *nitems;
        if (err_word & 1u) return;
        nunits = min(listed, max_items);
        if (int(blockIdx.x) >= nunits) return;  // uniform: nothing listed for this CTA
        hpc = 1;
    }
    if (device_failed(err)) return;  // an earlier wait expired: skip all work
    if (tid == 0) {
        s_abort = 0;
        for (int i = 0; i < 5; ++i) mbar_init(&bars[i], 1);
        fence_mbar_init();
        tma_prefetch_desc(&tm_c);
        tma_prefetch_desc(&tm_b);
        tma_prefetch_desc(&tm_x);
        tma_prefetch_desc(&tm_s);
    }
    if (warp == 0) tmem_alloc(tmem_holder, kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;
    const uint32_t lane_base = uint32_t(qd * 32) << 16;
    // phases: bars[0] and bars[1] complete once per unit, bars[2] and bars[3] once per head
    uint32_t jc = 0, hc = 0;
    // thread 0: phase parity of the last C / B and x / s_in loads it issued (-1: none)
    int ld0_par = -1, ld2_par = -1;

    for (int unit = items ? int(blockIdx.x) : 0; unit < nunits && s_abort == 0;
         unit += items ? int(gridDim.x) : 1, ++jc) {
        int mt, c, b, hfirst;
        if (items) {
            const long long v = items[unit];
            b = int(v >> 40);
            c = int((v >> 24) & 0xFFFF);
            mt = int((v >> 16) & 0xFF);
            hfirst = int(v & 0xFFFF);
        } else {
            const int nhb = d.H / hpc;
            mt = blockIdx.x;
            c = blockIdx.y;
            b = blockIdx.z / nhb;
            hfirst = (blockIdx.z % nhb) * hpc;
        }
        const int g = hfirst / d.r;
        const int s_len = (mt + 1) * kRows;              // source tokens [0, s_len) of the chunk
        const int trow0 = b * d.T + c * Q;                // first token row of the chunk in [B*T]
        const int t = mt * kRows + t_local;               // this thread's row within the chunk
        const uint32_t jpar = jc & 1;

        // ---- 1. C tile and B rows --------------------------------------------
        if (tid == 0) {
            constexpr int slabs = N >= 64 ? N / 64 : 1;
            const uint32_t bytes = uint32_t(kRows) * N * 2 + uint32_t(s_len) * N * 2;
            mbar_expect_tx(&bars[0], bytes);
            ld0_par = int(jpar);
            for (int sl_i = 0; sl_i < slabs; ++sl_i) {
                tma_load_3d(sC + sl_i * kRows * 128, &tm_c, &bars[0], sl_i * 64, g, trow0 + mt * kRows);
                for (int i = 0; i <= mt; ++i)
                    tma_load_3d(sB + sl_i * s_len * 128 + i * kRows * row_bytes(N), &tm_b, &bars[0],
                                sl_i * 64, g, trow0 + i * kRows);
            }
        }
        bool ok = mbar_wait(&bars[0], jpar, err);
        // ---- 2. CB = C B^T into TMEM columns [0, s_len) ----------------------------
        if (tid == 0 && ok) {
            tc_fence_after();
            const uint32_t idesc = idesc_bf16_f32(kRows, s_len, 0, 0);
            const uint32_t ca = smem_u32(sC), ba = smem_u32(sB);
            for (int k = 0; k < N / 16; ++k)
                mma_bf16_ss(tmem, kmajor_desc(ca, k, kRows, N), kmajor_desc(ba, k, s_len, N), idesc,
                            k > 0 ? 1u : 0u);
            mma_commit(&bars[1]);
        }
        if (ok && !mbar_wait(&bars[1], jpar, err)) ok = false;
        tc_fence_after();
        if (!ok) s_abort = 1;
        __syncthreads();

        for (int hi = 0; hi < hpc && s_abort == 0; ++hi, ++hc) {
            const int h = hfirst + hi;
            const uint32_t par = hc & 1;
            // ---- 3a. loads for this head ----------------------------------------
            if (tid == 0) {
                constexpr int slabs = N >= 64 ? N / 64 : 1;
                const uint32_t bytes = uint32_t(s_len) * 128 + 64u * N * 2;
                mbar_expect_tx(&bars[2], bytes);
                ld2_par = int(par);
                for (int i = 0; i <= mt; ++i)
                    tma_load_3d(sX + i * kRows * 128, &tm_x, &bars[2], 0, h, trow0 + i * kRows);
                const int srow = ((b * d.nc + c) * d.H + h) * 64;
                for (int sl_i = 0; sl_i < slabs; ++sl_i)
                    tma_load_2d(sS + sl_i * 64 * 128, &tm_s, &bars[2], sl_i * 64, srow);
            }
            for (int i = tid; i < s_len; i += kThreads) {
                sl[i] = __ldg(lcum + off_lq(d, b, h, c) + i);
                sdt[i] = __ldg(dt + off_dt(d, b, c * Q + i) + h);
            }
            __syncthreads();

            // ---- 3b. scores = CB * exp(l_t - l_s) * dt_s for s <= t -> bf16 smem
            {
                const float lt = sl[t];
                const int cols = s_len / 2;
                const int c0 = half * cols;
                const int tmax = mt * kRows + qd * 32 + 31;  // last row of this warp
#pragma unroll 1
                for (int s0 = c0; s0 < c0 + cols; s0 += 32) {
                    uint32_t pk[16];
                    if (s0 > tmax) {
#pragma unroll
                        for (int e = 0; e < 16; ++e) pk[e] = 0u;
                    } else {
                        float v[32];
                        tmem_ld32(tmem + lane_base + s0, v);
#pragma unroll
                        for (int e = 0; e < 16; ++e) {
                            const int s = s0 + 2 * e;
                            const float a0 = s <= t ? v[2 * e] * __expf(lt - sl[s]) * sdt[s] : 0.f;
                            const float a1 = s + 1 <= t ? v[2 * e + 1] * __expf(lt - sl[s + 1]) * sdt[s + 1] : 0.f;
                            pk[e] = pack_bf16x2(a0, a1);
                        }
                    }
                    uint8_t *slab = sP + (s0 >> 6) * (kRows * 128);
                    const int q0 = (s0 & 63) >> 3;
#pragma unroll
                    for (int qq = 0; qq < 4; ++qq)
                        *reinterpret_cast<uint4 *>(slab + sw128_off(t_local, q0 + qq)) =
                            make_uint4(pk[4 * qq], pk[4 * qq + 1], pk[4 * qq + 2], pk[4 * qq + 3]);
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            __syncthreads();

            // ---- 3c. Y = scores . X,  Z = C . s_in^T -------------------------------
            if (tid == 0) {
                if (!mbar_wait(&bars[2], par, err)) {
                    s_abort = 1;
                } else {
                    tc_fence_after();
                    const uint32_t pa = smem_u32(sP), xa = smem_u32(sX), ca = smem_u32(sC), sa = smem_u32(sS);
                    const uint32_t id1 = idesc_bf16_f32(kRows, 64, 0, 1);
                    for (int k = 0; k < s_len / 16; ++k)
                        mma_bf16_ss(tmem + kColY, kmajor_desc(pa, k, kRows, 64),
                                    smem_desc(xa + k * 2048, 16, 1024, kSw128), id1, k > 0 ? 1u : 0u);
                    const uint32_t id2 = idesc_bf16_f32(kRows, 64, 0, 0);
                    for (int k = 0; k < N / 16; ++k)
                        mma_bf16_ss(tmem + kColZ, kmajor_desc(ca, k, kRows, N), kmajor_desc(sa, k, 64, N),
                                    id2, k > 0 ? 1u : 0u);
                    mma_commit(&bars[3]);
                }
            }
            __syncthreads();
            if (s_abort == 0) {
                // bars[2] (already complete) also makes the TMA-written x rows
                // visible to this thread's epilogue loads
                if (!mbar_wait(&bars[2], par, err) || !mbar_wait(&bars[3], par, err)) s_abort = 1;
            }
            tc_fence_after();
            __syncthreads();

            // ---- 3d. epilogue: y = Y + exp(l_t) Z + D x ------------------------------
            if (s_abort == 0) {
                const int p0 = half * 32;
                float yv[32], zv[32];
                tmem_ld32(tmem + lane_base + kColY + p0, yv);
                tmem_ld32(tmem + lane_base + kColZ + p0, zv);
                const float e = __expf(sl[t]);
                const float Dh = Dskip ? __ldg(Dskip + h) : 0.f;
                uint32_t out[16];
#pragma unroll
                for (int qq = 0; qq < 4; ++qq) {
                    const uint4 xv = *reinterpret_cast<const uint4 *>(sX + sw128_off(t, (p0 >> 3) + qq));
                    const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const int i = qq * 8 + 2 * u;
                        const float o0 = fmaf(Dh, bf16lo(xw[u]), fmaf(e, zv[i], yv[i]));
                        const float o1 = fmaf(Dh, bf16hi(xw[u]), fmaf(e, zv[i + 1], yv[i + 1]));
                        out[qq * 4 + u] = pack_bf16x2(o0, o1);
                    }
                }
                uint4 *dst = reinterpret_cast<uint4 *>(y + off_x(d, b, c * Q + t, h) + p0);
#pragma unroll
                for (int qq = 0; qq < 4; ++qq)
                    dst[qq] = make_uint4(out[4 * qq], out[4 * qq + 1], out[4 * qq + 2], out[4 * qq + 3]);
            }
            tc_fence_before();
            __syncthreads();
        }
    }
    // after an abandoned wait, give the work still in flight a bounded chance
    // to finish before the tensor memory is released: the last C / B and x /
    // s_in loads issued, and every MMA this thread issued (one commit tracks
    // them all)
    if (tid == 0 && s_abort) {
        if (ld0_par >= 0) mbar_wait(&bars[0], uint32_t(ld0_par), nullptr);
        if (ld2_par >= 0) mbar_wait(&bars[2], uint32_t(ld2_par), nullptr);
        mma_commit(&bars[4]);
        mbar_wait(&bars[4], 0, nullptr);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, kTmemCols);
}

template <int N>
cudaError_t launch_n(const Dims &d, const CUtensorMap *maps, int hpc, const float *dt,
                     const float *D, const float *l, __nv_bfloat16 *y, const long long *items,
                     const int *nitems, int max_items, unsigned int *err, cudaStream_t stream) {
    const ScanSmem L = scan_smem(d.Q, N);
    // at least 116 KB so that one CTA (which takes all 512 TMEM columns) runs per SM
    const int smem = int(L.total < 116 * 1024 ? 116 * 1024 : L.total);
    if (!smem_attr_once(reinterpret_cast<const void *>(chunk_scan_tc_kernel<N>), smem))
        return cudaErrorInvalidValue;
    dim3 grid(d.Q / kRows, d.nc, d.B * (d.H / hpc));
    if (items) {
        // one CTA per SM walks the list (most CTAs exit at once when it is short)
        const int sms = device_sm_count();
        grid = dim3(max_items < sms ? max_items : sms, 1, 1);
    }
    chunk_scan_tc_kernel<N><<<grid, kThreads, smem, stream>>>(maps[0], maps[1], maps[2], maps[3], d, hpc,
                                                                dt, D, l, y, items, nitems, max_items, err);
    return cudaGetLastError();
}

int heads_per_cta(const Dims &d) {
    int best = 1;
    for (int k = 1; k <= 8; ++k)
        if (d.r % k == 0) best = k;
    return best;
}

}  // namespace

bool tc_chunk_scan_supported(const Dims &d) {
    const bool n_ok = d.N == 16 || d.N == 32 || d.N == 64 || d.N == 128 || d.N == 256;
    return d.P == 64 && n_ok && (d.Q == 128 || d.Q == 256) &&
           scan_smem(d.Q, d.N).total <= 227 * 1024 && d.B * (d.H / heads_per_cta(d)) <= 65535;
}

cudaError_t launch_chunk_scan_tc(const Dims &d, const void *x, const float *dt, const void *Bm,
                                 const void *Cm, const float *D, const float *l,
                                 const void *s_in_bf16, void *y, const long long *items,
                                 const int *nitems, int max_items, unsigned int *err,
                                 cudaStream_t stream) {
    if (items && max_items <= 0) return cudaSuccess;
    const uint32_t nbox = uint32_t(d.N >= 64 ? 64 : d.N);
    const int rb = row_bytes(d.N);
    const uint64_t bcdims[3] = {uint64_t(d.N), uint64_t(d.G), uint64_t(d.B) * d.T};
    const uint64_t bcstr[2] = {uint64_t(d.N) * 2, uint64_t(d.G) * d.N * 2};
    const uint32_t bcbox[3] = {nbox, 1, uint32_t(kRows)};
    const uint64_t xdims[3] = {uint64_t(d.P), uint64_t(d.H), uint64_t(d.B) * d.T};
    const uint64_t xstr[2] = {uint64_t(d.P) * 2, uint64_t(d.H) * d.P * 2};
    const uint32_t xbox[3] = {64, 1, uint32_t(kRows)};
    const uint64_t sdims[2] = {uint64_t(d.N), uint64_t(d.B) * d.nc * d.H * d.P};
    const uint64_t sstr[1] = {uint64_t(d.N) * 2};
    const uint32_t sbox[2] = {nbox, 64};
    CUtensorMap maps[4];
    if (!make_tmap_bf16(&maps[0], 3, Cm, bcdims, bcstr, bcbox, rb) ||
        !make_tmap_bf16(&maps[1], 3, Bm, bcdims, bcstr, bcbox, rb) ||
        !make_tmap_bf16(&maps[2], 3, x, xdims, xstr, xbox, 128) ||
        !make_tmap_bf16(&maps[3], 2, s_in_bf16, sdims, sstr, sbox, rb))
        return cudaErrorInvalidValue;
    const int hpc = heads_per_cta(d);
    auto *yo = static_cast<__nv_bfloat16 *>(y);
    switch (d.N) {
        case 16: return launch_n<16>(d, maps, hpc, dt, D, l, yo, items, nitems, max_items, err, stream);
        case 32: return launch_n<32>(d, maps, hpc, dt, D, l, yo, items, nitems, max_items, err, stream);
        case 64: return launch_n<64>(d, maps, hpc, dt, D, l, yo, items, nitems, max_items, err, stream);
        case 128: return launch_n<128>(d, maps, hpc, dt, D, l, yo, items, nitems, max_items, err, stream);
        case 256: return launch_n<256>(d, maps, hpc, dt, D, l, yo, items, nitems, max_items, err, stream);
    }
    return cudaErrorInvalidValue;
}

}  // namespace ssd
