// k_tc_state_fused.cu -- ssd_chunk_state and ssd_state_passing as one
// persistent tensor-core kernel.
//
// For batch b and head h (group g), chunk by chunk:
//     S_c       = sum_{s in chunk c} w_s x_s B_s^T,   w_s = exp(l_last - l_s) dt_s
//     s_in[0]   = h0 (or 0),   s_in[c+1] = alpha_c s_in[c] + S_c,   final = s_in[nc]
// (the per-chunk state and the inter-chunk recurrence of the chunked SSD
// algorithm: aifetchly blog "Mamba-2 Architecture: State Space Duality
// Explained", "The Chunked SSD Algorithm", step 2; the weights w and the chunk
// decay alpha come from unrolling h_t = exp(dt_t A) h_{t-1} + dt_t x_t B_t^T).
//
// One work unit = (b, nh heads of one group) walked over ALL its chunks in
// order, so the running state never leaves the SM:
//     * S_c is one UMMA per 16 tokens, D[m, n] = sum_s (w o X)^T[m, s] B[s, n]
//       with m = (head j, p) (M = 128), K = chunk_len, accumulated in one of two
//       TMEM accumulators;
//     * the running state R (fp32, same M x N shape) lives in a third TMEM
//       region; the epilogue warps update R = alpha_c R + S_c and store s_in as
//       bf16 for the chunk scan (and the final state as fp32);
//     * chunk c + 1's MMAs overlap chunk c's update (double-buffered
//       accumulators), and the loads run a ring of up to 6 stages ahead.
// The chunk states S_c are never written to HBM, and the separate state
// passing pass over them disappears.  The kernel needs nc sequential steps per
// unit, so it is used when the (b, head pair) units fill most of the GPU in a
// single wave (a second wave would run nc steps again on a few SMs).
//
// Roles (10 warps): warp 0 TMA producer, warp 1 MMA issuer, warps 2..5 scale x
// rows by w in shared memory, warps 6..9 state update + stores.
//
// Range mode (seg_out != nullptr) serves the presolved single pass: the grid
// splits the (chain = head-pair unit, chunk) items exactly as the single pass
// does (chain_ranges.cuh), and each CTA runs only its range's LAST segment, if
// that ends inside its chain: from h0 when the segment starts a chain, from
// zero otherwise, with no s_in written; its end state goes to seg_out[CTA].
// range_states_kernel (below) then chains those partial states along each
// chain into the state entering every range.
#include "chain_ranges.cuh"
#include "common.cuh"
#include "kernels.h"
#include "tc_common.cuh"
#include "tma_host.h"

namespace ssd {

namespace {

using namespace tc;

constexpr int kThreads = 320;
constexpr int kKS = 64;  // tokens per stage
// stages in flight: as many 64-token stages as shared memory holds (each TMA
// stage takes ~3 us to land when every SM streams, so a deep ring matters)
__host__ __device__ constexpr int num_stages(int ns) { return ns <= 128 ? 6 : 4; }

__host__ __device__ constexpr int acc_cols(int ns) { return ns < 16 ? 16 : ns; }
__host__ __device__ constexpr int alloc_cols(int ns) {
    return 3 * acc_cols(ns) <= 32 ? 32
         : 3 * acc_cols(ns) <= 64 ? 64
         : 3 * acc_cols(ns) <= 128 ? 128
         : 3 * acc_cols(ns) <= 256 ? 256 : 512;
}
__host__ __device__ constexpr int brow_bytes(int ns) { return ns >= 64 ? 128 : ns * 2; }
__host__ __device__ constexpr uint32_t bswz(int ns) { return ns >= 64 ? kSw128 : (ns == 32 ? kSw64 : kSw32); }
__host__ __device__ constexpr uint32_t x_bytes() { return 2 * kKS * 128; }
__host__ __device__ constexpr uint32_t b_bytes(int ns) { return kKS * ns * 2; }
__host__ __device__ constexpr uint32_t w_bytes() { return 2 * kKS * 4; }
__host__ __device__ constexpr uint32_t stage_bytes(int ns) {
    return ((x_bytes() + b_bytes(ns) + w_bytes()) + 1023u) & ~1023u;
}
// Per update warp, two 32 x 32 bf16 staging blocks (64-byte rows) for the TMA
// stores of s_in.
constexpr uint32_t kStgWarpBytes = 2 * 32 * 64;
__host__ __device__ constexpr uint32_t stg_off(int ns) { return uint32_t(num_stages(ns)) * stage_bytes(ns) + 1024; }
size_t fused_smem_bytes(int ns) { return 1024 + stg_off(ns) + 4 * kStgWarpBytes; }

// Work item k of this CTA: unit u over chunks [c0, c1).  Normal mode: units
// blockIdx.x + k gridDim.x over all chunks.  Range mode: at most one item, the
// last segment of the CTA's single-pass range when it ends inside its chain.
struct UnitWork {
    int u, c0, c1;
};
__device__ __forceinline__ bool unit_work(int k, const Dims &d, int units, bool range_mode, UnitWork &w) {
    if (!range_mode) {
        const int u = int(blockIdx.x) + k * int(gridDim.x);
        w.u = u;
        w.c0 = 0;
        w.c1 = d.nc;
        return u < units;
    }
    if (k > 0) return false;
    const ChainRange r = chain_range(units, d.nc, blockIdx.x, gridDim.x);
    w.u = r.cl;
    w.c0 = r.cf == r.cl ? r.cfc : 0;
    w.c1 = r.clc;
    return w.c1 < d.nc;
}

__device__ __forceinline__ void store_bf16_row(__nv_bfloat16 *dst, const float *v, int n) {
    uint4 *o = reinterpret_cast<uint4 *>(dst);
    for (int q = 0; q < n / 8; ++q)
        o[q] = make_uint4(pack_bf16x2(v[8 * q], v[8 * q + 1]), pack_bf16x2(v[8 * q + 2], v[8 * q + 3]),
                          pack_bf16x2(v[8 * q + 4], v[8 * q + 5]), pack_bf16x2(v[8 * q + 6], v[8 * q + 7]));
}

template <int NS>
__global__ void __launch_bounds__(kThreads, 1)
state_fused_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_b,
                   const __grid_constant__ CUtensorMap tm_s, Dims d, int nh, int units,
                   const float *__restrict__ w,
                   const float *__restrict__ alpha, const float *__restrict__ h0,
                   __nv_bfloat16 *__restrict__ s_in, float *__restrict__ fin, float *__restrict__ seg_out,
                   unsigned int *err) {
    constexpr int kAcc = acc_cols(NS);
    constexpr int kStages = num_stages(NS);
    constexpr int kCols = alloc_cols(NS);
    constexpr int kRowB = brow_bytes(NS);
    constexpr int kSeg = NS >= 32 ? 32 : 16;  // TMEM columns per load/store
    if (device_failed(err)) return;  // an earlier wait expired: skip all work
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kStages * stage_bytes(NS));
    uint64_t *full = bars, *scaled = bars + kStages, *empty = bars + 2 * kStages;
    uint64_t *accf = bars + 3 * kStages, *acce = accf + 2, *done = acce + 2;
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(done + 1);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nhp = d.H / nh;
    const int ksteps = d.Q / kKS;
    const bool range_mode = seg_out != nullptr;

    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&scaled[s], 128);
            mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&accf[a], 1);
            mbar_init(&acce[a], 128);
        }
        mbar_init(done, 1);
        fence_mbar_init();
        tma_prefetch_desc(&tm_x);
        tma_prefetch_desc(&tm_b);
    }
    if (warp == 1) tmem_alloc(tmem_holder, kCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;

    if (warp == 0) {
        // ------------------------------ TMA producer ------------------------------
        if (lane == 0) {
            uint32_t it = 0;
            bool ok = true;
            UnitWork W;
            for (int wk = 0; ok && unit_work(wk, d, units, range_mode, W); ++wk) {
                const int u = W.u;
                const int hp = u % nhp, b = u / nhp;
                const int hh = hp * nh, g = hh / d.r;
                for (int c = W.c0; c < W.c1 && ok; ++c) {
                    const int trow = b * d.T + c * d.Q;
                    for (int ks = 0; ks < ksteps; ++ks) {
                        const int s = it % kStages;
                        if (!mbar_wait(&empty[s], ((it / kStages) & 1) ^ 1, err)) { ok = false; break; }
                        uint8_t *sx = smem + s * stage_bytes(NS);
                        uint8_t *sb = sx + x_bytes();
                        float *sw = reinterpret_cast<float *>(sb + b_bytes(NS));
                        mbar_expect_tx(&full[s], uint32_t(nh) * (kKS * 128 + kKS * 4) + b_bytes(NS));
                        for (int j = 0; j < nh; ++j)
                            bulk_load(sw + j * kKS, w + off_lq(d, b, hh + j, c) + ks * kKS, kKS * 4, &full[s]);
                        for (int j = 0; j < nh; ++j)
                            tma_load_3d(sx + j * kKS * 128, &tm_x, &full[s], 0, hh + j, trow + ks * kKS);
                        if (NS >= 64) {
                            for (int sl = 0; sl < NS / 64; ++sl)
                                tma_load_3d(sb + sl * kKS * 128, &tm_b, &full[s], sl * 64, g, trow + ks * kKS);
                        } else {
                            tma_load_3d(sb, &tm_b, &full[s], 0, g, trow + ks * kKS);
                        }
                        ++it;
                    }
                }
            }
            // drain: every stage issued must have landed before the CTA exits
            for (int k = 0; k < kStages && it > 0; ++k, --it) {
                const uint32_t i = it - 1;
                mbar_wait(&full[i % kStages], (i / kStages) & 1, nullptr);
            }
        }
    } else if (warp == 1) {
        // ------------------------------ MMA issuer --------------------------------
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_bf16_f32(128, kAcc, 1, 1);
            uint32_t it = 0, ci = 0;
            bool ok = true;
            UnitWork W;
            for (int wk = 0; ok && unit_work(wk, d, units, range_mode, W); ++wk) {
                for (int c = W.c0; c < W.c1 && ok; ++c, ++ci) {
                    const int a = ci & 1;
                    if (!mbar_wait(&acce[a], ((ci >> 1) & 1) ^ 1, err)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t dacc = tmem + a * kAcc;
                    for (int ks = 0; ks < ksteps; ++ks) {
                        const int s = it % kStages;
                        if (!mbar_wait(&scaled[s], (it / kStages) & 1, err)) { ok = false; break; }
                        tc_fence_after();
                        const uint32_t xa = smem_u32(smem + s * stage_bytes(NS));
                        const uint32_t ba = xa + x_bytes();
#pragma unroll
                        for (int k = 0; k < kKS / 16; ++k) {
                            const uint64_t ad = smem_desc(xa + k * 16 * 128, kKS * 128, 1024, kSw128);
                            const uint64_t bd = smem_desc(ba + k * 16 * kRowB, kKS * 128, 8 * kRowB, bswz(NS));
                            mma_bf16_ss(dacc, ad, bd, idesc, (ks > 0 || k > 0) ? 1u : 0u);
                        }
                        mma_commit(&empty[s]);
                        ++it;
                    }
                    if (ok) mma_commit(&accf[a]);
                }
            }
            mma_commit(done);
            mbar_wait(done, 0, nullptr);
        }
    } else if (warp < 6) {
        // ------------------------------ scale x by w -------------------------------
        // 16-byte chunk i of the stage's x tile belongs to row i / 8 (head
        // j = row / 64, token row % 64); eight consecutive threads share a row,
        // so a warp touches four whole 128-byte rows (no bank conflicts).  The
        // swizzle only permutes chunks within a row, so each chunk takes its
        // row's weight.
        const int st = tid - 64;  // 0..127
        uint32_t it = 0;
        bool ok = true;
        UnitWork W;
        for (int wk = 0; ok && unit_work(wk, d, units, range_mode, W); ++wk) {
            for (int c = W.c0; c < W.c1 && ok; ++c) {
                for (int ks = 0; ks < ksteps; ++ks) {
                    const int s = it % kStages;
                    if (!mbar_wait(&full[s], (it / kStages) & 1, err)) { ok = false; break; }
                    uint8_t *sx = smem + s * stage_bytes(NS);
                    const float *sw = reinterpret_cast<const float *>(sx + x_bytes() + b_bytes(NS));
                    // every load first, then the stores: the shared-memory stores may
                    // alias the loads, so a fused loop would run at load latency
                    constexpr int kPer = (2 * kKS * 8) / 128;
                    uint4 v[kPer];
                    float wv[kPer];
#pragma unroll
                    for (int k = 0; k < kPer; ++k) {
                        const int i = st + k * 128;
                        v[k] = reinterpret_cast<const uint4 *>(sx)[i];
                        wv[k] = sw[i >> 3];
                    }
#pragma unroll
                    for (int k = 0; k < kPer; ++k) {
                        const int i = st + k * 128;
                        if (((i >> 3) >> 6) < nh) {
                            uint4 o;
                            o.x = pack_bf16x2(bf16lo(v[k].x) * wv[k], bf16hi(v[k].x) * wv[k]);
                            o.y = pack_bf16x2(bf16lo(v[k].y) * wv[k], bf16hi(v[k].y) * wv[k]);
                            o.z = pack_bf16x2(bf16lo(v[k].z) * wv[k], bf16hi(v[k].z) * wv[k]);
                            o.w = pack_bf16x2(bf16lo(v[k].w) * wv[k], bf16hi(v[k].w) * wv[k]);
                            reinterpret_cast<uint4 *>(sx)[i] = o;
                        }
                    }
                    fence_proxy_async_smem();
                    mbar_arrive(&scaled[s]);
                    ++it;
                }
            }
        }
    } else {
        // --------------------------- state update + stores --------------------------
        // Thread (lane quarter qd, lane) owns TMEM row m = (head j, p).  For
        // N >= 32 each 32 x 32 block of s_in goes out as bf16 through a swizzled
        // staging block and one 2-D TMA store (coalesced, and off the load/store
        // unit that the scale warps use); N = 16 rows are stored directly.
        const int qd = warp & 3;
        const int m = qd * 32 + lane;
        const int j = m >> 6, p = m & 63;
        const uint32_t lane_base = uint32_t(qd * 32) << 16;
        const uint32_t tR = tmem + lane_base + 2 * kAcc;  // running state
        const bool valid = j < nh;  // warp-uniform
        uint8_t *stg = smem + stg_off(NS) + qd * kStgWarpBytes;
        uint32_t ci = 0, nst = 0;
        bool ok = true;
        UnitWork W;
        for (int wk = 0; ok && unit_work(wk, d, units, range_mode, W); ++wk) {
            const int u = W.u;
            const int hp = u % nhp, b = u / nhp;
            const int h = hp * nh + (valid ? j : 0);
            const int64_t row = (int64_t(b) * d.H + h) * d.P + p;  // row of [B, H, P, N]
            // s_in[b, cc, h, p, n0 .. n0 + kSeg) = bf16(v)
            auto emit = [&](const float *v, int cc, int n0) {
                if (NS >= 32) {
                    if (!valid) return;
                    uint8_t *blk = stg + (nst & 1) * (32 * 64);
                    // the store that used this block two stores ago has read it
                    if (lane == 0) bulk_wait_read_1();
                    __syncwarp();
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        *reinterpret_cast<uint4 *>(blk + sw64_off(lane, q)) =
                            make_uint4(pack_bf16x2(v[8 * q], v[8 * q + 1]), pack_bf16x2(v[8 * q + 2], v[8 * q + 3]),
                                       pack_bf16x2(v[8 * q + 4], v[8 * q + 5]), pack_bf16x2(v[8 * q + 6], v[8 * q + 7]));
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        tma_store_2d(&tm_s, blk, n0, ((b * d.nc + cc) * d.H + h) * 64 + (qd & 1) * 32);
                        bulk_commit();
                    }
                    ++nst;
                } else if (valid) {
                    store_bf16_row(s_in + off_state(d, b, cc, h) + int64_t(p) * NS + n0, v, kSeg);
                }
            };
            // R = h0 (or 0: range mode inside a chain); s_in[0] = R
#pragma unroll 1
            for (int n0 = 0; n0 < NS; n0 += kSeg) {
                float v[32];
#pragma unroll
                for (int e = 0; e < kSeg; ++e) v[e] = 0.f;
                if (h0 && valid && W.c0 == 0) {
                    const float4 *src = reinterpret_cast<const float4 *>(h0 + row * NS + n0);
#pragma unroll
                    for (int q = 0; q < kSeg / 4; ++q) {
                        const float4 t = __ldg(src + q);
                        v[4 * q] = t.x; v[4 * q + 1] = t.y; v[4 * q + 2] = t.z; v[4 * q + 3] = t.w;
                    }
                }
#pragma unroll
                for (int q = 0; q < kSeg / 16; ++q)
                    tmem_st16(tR + n0 + 16 * q, reinterpret_cast<const uint32_t *>(v + 16 * q));
                if (!range_mode) emit(v, 0, n0);
            }
            tmem_wait_st();
            for (int c = W.c0; c < W.c1; ++c, ++ci) {
                const int a = ci & 1;
                if (!mbar_wait(&accf[a], (ci >> 1) & 1, err)) { ok = false; break; }
                tc_fence_after();
                const float al = valid ? __ldg(alpha + off_alpha(d, b, h, c)) : 0.f;
                const bool last = c + 1 == W.c1;
#pragma unroll 1
                for (int n0 = 0; n0 < NS; n0 += kSeg) {
                    uint32_t r[32], sc[32];
                    if (kSeg == 32) {
                        tmem_ld32_nowait(tR + n0, r);
                        tmem_ld32_nowait(tmem + lane_base + a * kAcc + n0, sc);
                    } else {
                        tmem_ld16_nowait(tR + n0, *reinterpret_cast<uint32_t(*)[16]>(r));
                        tmem_ld16_nowait(tmem + lane_base + a * kAcc + n0, *reinterpret_cast<uint32_t(*)[16]>(sc));
                    }
                    tmem_wait_ld();
                    float v[32];
#pragma unroll
                    for (int e = 0; e < kSeg; ++e)
                        v[e] = fmaf(al, __uint_as_float(r[e]), __uint_as_float(sc[e]));
                    if (!last) {
#pragma unroll
                        for (int q = 0; q < kSeg / 16; ++q)
                            tmem_st16(tR + n0 + 16 * q, reinterpret_cast<const uint32_t *>(v + 16 * q));
                        if (!range_mode) emit(v, c + 1, n0);
                    } else if (range_mode) {
                        if (valid) {
                            float4 *o = reinterpret_cast<float4 *>(seg_out + (int64_t(blockIdx.x) * 128 + m) * NS + n0);
#pragma unroll
                            for (int q = 0; q < kSeg / 4; ++q)
                                o[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
                        }
                    } else if (fin && valid) {
                        float4 *o = reinterpret_cast<float4 *>(fin + row * NS + n0);
#pragma unroll
                        for (int q = 0; q < kSeg / 4; ++q)
                            o[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
                    }
                }
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(&acce[a]);
            }
        }
        if (lane == 0) bulk_wait_all();
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) tmem_dealloc(tmem, kCols);
}

template <int NS>
cudaError_t launch_ns(const Dims &d, const CUtensorMap &tx, const CUtensorMap &tb,
                      const CUtensorMap &ts, int nh, const float *w, const float *alpha,
                      const float *h0, __nv_bfloat16 *s_in, float *fin, float *seg_out, int range_grid,
                      unsigned int *err, cudaStream_t stream) {
    const size_t smem = fused_smem_bytes(NS);
    if (!smem_attr_once(reinterpret_cast<const void *>(state_fused_kernel<NS>), int(smem)))
        return cudaErrorInvalidValue;
    const int units = d.B * (d.H / nh);
    const int grid = seg_out ? range_grid : (units < device_sm_count() ? units : device_sm_count());
    state_fused_kernel<NS><<<grid, kThreads, smem, stream>>>(tx, tb, ts, d, nh, units, w, alpha,
                                                             h0, s_in, fin, seg_out, err);
    return cudaGetLastError();
}

// One block per (slice of a head pair's state, chain); four consecutive
// elements e of that state per thread (row m = (head of the pair, p), column n).  The CTAs whose
// single-pass range begins strictly inside the chain are k0 .. k0 + M - 1, in
// order; CTA k - 1's last segment [cp, ck) ends where CTA k's range starts, and
// its partial end state seg[k - 1] started from h0 when cp is 0, from zero
// otherwise, so the state entering CTA k is
//     start[k] = seg[k - 1]                                   (cp == 0)
//     start[k] = (prod_{c in [cp, ck)} alpha_c) start[k - 1] + seg[k - 1]
// The products (one per listed CTA and head) are formed once per block in
// shared memory; each thread (four elements) then walks the list with one
// 16-byte load and store per step.
constexpr int kMaxRangesPerChain = 160;  // >= the grid (148) + 1
__global__ void __launch_bounds__(256)
range_states_kernel(Dims d, int G, const float *__restrict__ alpha, const float *__restrict__ seg,
                    float *__restrict__ start) {
    __shared__ float dec[kMaxRangesPerChain][2];
    __shared__ int s_k0, s_m;
    const int64_t per = int64_t(128) * d.N;
    const int np = d.H / 2;
    const int chain = blockIdx.y;
    const int b = chain / np, hp = chain % np;
    const long long items = (long long)d.B * np * d.nc;
    const long long first = (long long)chain * d.nc, end = first + d.nc;
    if (threadIdx.x == 0) {
        // first CTA whose range begins strictly inside the chain, and how many do
        int k = int(first * G / items);
        while (k < G && chain_range_begin(items, k, G) <= first) ++k;
        int m = 0;
        while (k + m < G && chain_range_begin(items, k + m, G) < end) ++m;
        s_k0 = k;
        s_m = m;
    }
    __syncthreads();
    const int k0 = s_k0, M = s_m;
    // decay over the segment ending where listed CTA i starts (unused for i = 0):
    // one warp per (i, head), the segment's chunks spread over the lanes
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int t = warp; t < 2 * M; t += blockDim.x >> 5) {
        const int i = t >> 1, jh = t & 1;
        const int ck = int(chain_range_begin(items, k0 + i, G) - first);
        const int cp = i == 0 ? ck : int(chain_range_begin(items, k0 + i - 1, G) - first);
        float pr = 1.f;
        for (int c = cp + lane; c < ck; c += 32) pr *= __ldg(alpha + off_alpha(d, b, 2 * hp + jh, c));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) pr *= __shfl_xor_sync(0xffffffffu, pr, o);
        if (lane == 0) dec[i][jh] = pr;
    }
    __syncthreads();
    // four consecutive elements per thread (one row: N is a multiple of 4)
    const int64_t e = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) * 4;
    if (e >= per) return;
    const int jh = int(e / d.N) / 64;
    float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
    for (int i = 0; i < M; ++i) {
        const int k = k0 + i;
        const float4 part = *reinterpret_cast<const float4 *>(seg + (int64_t(k) - 1) * per + e);
        // the first listed CTA follows one whose last segment started the chain
        if (i == 0) {
            s = part;
        } else {
            const float dk = dec[i][jh];
            s = make_float4(fmaf(dk, s.x, part.x), fmaf(dk, s.y, part.y), fmaf(dk, s.z, part.z), fmaf(dk, s.w, part.w));
        }
        *reinterpret_cast<float4 *>(start + int64_t(k) * per + e) = s;
    }
}

int fused_heads_per_unit(const Dims &d) { return d.r % 2 == 0 ? 2 : 1; }

}  // namespace

bool tc_state_fused_supported(const Dims &d, int sms) {
    const bool ns_ok = d.N == 16 || d.N == 32 || d.N == 64 || d.N == 128;
    const int64_t units = int64_t(d.B) * (d.H / fused_heads_per_unit(d));
    // nc sequential steps per unit: worth it when the units fill most SMs in ONE
    // wave (with more units than SMs a second wave repeats all nc steps)
    return d.P == 64 && ns_ok && (d.Q == 64 || d.Q == 128 || d.Q == 256) &&
           fused_smem_bytes(d.N) <= 227 * 1024 && units * 5 >= int64_t(sms) * 3 &&
           units <= sms;
}

cudaError_t launch_state_fused(const Dims &d, const void *x, const void *Bm, const float *w,
                               const float *alpha, const float *h0, void *s_in_bf16, float *fin,
                               unsigned int *err, cudaStream_t stream) {
    // x viewed as [B*T rows][H][P]; box = one head, 64 tokens
    const uint64_t xdims[3] = {uint64_t(d.P), uint64_t(d.H), uint64_t(d.B) * d.T};
    const uint64_t xstr[2] = {uint64_t(d.P) * 2, uint64_t(d.H) * d.P * 2};
    const uint32_t xbox[3] = {64, 1, uint32_t(kKS)};
    const uint32_t nbox = uint32_t(d.N >= 64 ? 64 : d.N);
    const uint64_t bdims[3] = {uint64_t(d.N), uint64_t(d.G), uint64_t(d.B) * d.T};
    const uint64_t bstr[2] = {uint64_t(d.N) * 2, uint64_t(d.G) * d.N * 2};
    const uint32_t bbox[3] = {nbox, 1, uint32_t(kKS)};
    // s_in viewed as [B*nc*H*P rows][N]; box = 32 columns x 32 rows
    const uint64_t sdims[2] = {uint64_t(d.N), uint64_t(d.B) * d.nc * d.H * d.P};
    const uint64_t sstr[1] = {uint64_t(d.N) * 2};
    const uint32_t sbox[2] = {32, 32};
    CUtensorMap tx, tb, ts{};
    if (!make_tmap_bf16(&tx, 3, x, xdims, xstr, xbox, 128) ||
        !make_tmap_bf16(&tb, 3, Bm, bdims, bstr, bbox, brow_bytes(d.N)) ||
        (d.N >= 32 && !make_tmap_bf16(&ts, 2, s_in_bf16, sdims, sstr, sbox, 64)))
        return cudaErrorInvalidValue;
    const int nh = fused_heads_per_unit(d);
    __nv_bfloat16 *s = static_cast<__nv_bfloat16 *>(s_in_bf16);
    switch (d.N) {
        case 16: return launch_ns<16>(d, tx, tb, ts, nh, w, alpha, h0, s, fin, nullptr, 0, err, stream);
        case 32: return launch_ns<32>(d, tx, tb, ts, nh, w, alpha, h0, s, fin, nullptr, 0, err, stream);
        case 64: return launch_ns<64>(d, tx, tb, ts, nh, w, alpha, h0, s, fin, nullptr, 0, err, stream);
        case 128: return launch_ns<128>(d, tx, tb, ts, nh, w, alpha, h0, s, fin, nullptr, 0, err, stream);
    }
    return cudaErrorInvalidValue;
}

bool presolved_ranges_supported(const Dims &d) {
    return d.P == 64 && (d.N == 64 || d.N == 128) && (d.Q == 128 || d.Q == 256) && d.r % 2 == 0 &&
           fused_smem_bytes(d.N) <= 227 * 1024;
}

size_t presolved_state_bytes(int G, const Dims &d) { return size_t(G) * 128 * d.N * sizeof(float); }

cudaError_t launch_presolve_ranges(const Dims &d, int G, const void *x, const void *Bm, const float *w,
                                   const float *alpha, const float *h0, float *seg, float *start,
                                   unsigned int *err, cudaStream_t stream) {
    if (G <= 0 || G >= kMaxRangesPerChain || !presolved_ranges_supported(d)) return cudaErrorInvalidValue;
    const uint64_t xdims[3] = {uint64_t(d.P), uint64_t(d.H), uint64_t(d.B) * d.T};
    const uint64_t xstr[2] = {uint64_t(d.P) * 2, uint64_t(d.H) * d.P * 2};
    const uint32_t xbox[3] = {64, 1, uint32_t(kKS)};
    const uint64_t bdims[3] = {uint64_t(d.N), uint64_t(d.G), uint64_t(d.B) * d.T};
    const uint64_t bstr[2] = {uint64_t(d.N) * 2, uint64_t(d.G) * d.N * 2};
    const uint32_t bbox[3] = {64, 1, uint32_t(kKS)};
    CUtensorMap tx, tb, ts{};
    if (!make_tmap_bf16(&tx, 3, x, xdims, xstr, xbox, 128) ||
        !make_tmap_bf16(&tb, 3, Bm, bdims, bstr, bbox, brow_bytes(d.N)))
        return cudaErrorInvalidValue;
    cudaError_t e = d.N == 64
        ? launch_ns<64>(d, tx, tb, ts, 2, w, alpha, h0, nullptr, nullptr, seg, G, err, stream)
        : launch_ns<128>(d, tx, tb, ts, 2, w, alpha, h0, nullptr, nullptr, seg, G, err, stream);
    if (e != cudaSuccess) return e;
    const int64_t per = int64_t(128) * d.N;
    const dim3 grid(unsigned((per / 4 + 255) / 256), unsigned(d.B * (d.H / 2)));
    range_states_kernel<<<grid, 256, 0, stream>>>(d, G, alpha, seg, start);
    return cudaGetLastError();
}

}  // namespace ssd
