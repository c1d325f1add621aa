// k_tc_chunk_scan4.cu -- ssd_chunk_scan on the tensor cores: persistent, warp
// specialised, double-buffered scores and accumulators (dstate <= 128).
//
// Output, for the rows t of the 128-token tile [t0, t0 + 128) of chunk c:
//     y_t = exp(l_t) C_t s_in^T + sum_{s <= t} exp(l_t - l_s) dt_s (C_t . B_s) x_s + D_h x_t
// (the intra-chunk masked product (L o C B^T)(dt o X) of the chunked SSD
// algorithm -- aifetchly blog "Mamba-2 Architecture", "The Chunked SSD
// Algorithm", step 1; akillness.github.io "State Space Duality and Mamba-2",
// "The Scalar-Identity Structural Constraint" -- plus the state carried in from
// earlier chunks and the skip term).
//
// Split of the source tokens s at the tile start t0, with r = l_{t0-1} (r = 0
// for the first tile) and u_t = exp(l_t - r) <= 1:
//   * s < t0:  exp(l_t - l_s) = u_t exp(r - l_s), both factors <= 1, so
//         sum_{s<t0} = u_t (C B^T)[t, s<t0] (g o X)[s<t0],  g_s = exp(r - l_s) dt_s;
//     the block CBoff = (C B^T)[tile, s<t0] needs no mask and serves every head.
//   * state term:  exp(l_t) C_t s_in = u_t C_t (exp(r) s_in).
//   * t0 <= s <= t:  the 128 x 128 diagonal tile keeps its mask, built per head.
// So  y = Yd + u_t Yoz,  Yd = P Xd,  Yoz = CBoff X' + C S'^T,  with
//   P  = masked diagonal scores in bf16 (+ D_h on the diagonal: the skip term),
//   X' = g o X[s < t0],  S' = exp(r) s_in.
//
// Decay factors inside the diagonal tile, per 32 x 32 block with source block
// k (last token k_e): exp(l_t - l_s) dt_s = exp(l_t - l_{k_e}) beta_s, where
// beta_s = exp(l_{k_e} - l_s) dt_s <= dt_s comes precomputed from the cumsum.
//   * blocks entirely below the diagonal: both factors are <= 1;
//   * blocks on the diagonal: the row factor exp(l_t - l_{k_e}) is >= 1 but at
//     most exp(l_{k_s} - l_{k_e}), so the same factorisation holds when the
//     block's decay range l_{k_s} - l_{k_e} is below 80; otherwise the exact
//     exp(l_t - l_s) per element.
//
// Tensor memory: [0,128) CB diagonal tile (fp32); [128,256) two score buffers
// (bf16; at the start of a unit this range holds CBoff in fp32); [256,512) two
// accumulators {Yd, Yoz}.  Shared memory: C and CBoff (bf16, A operands of the
// Yoz MMAs), the per-head stages {x rows, s_in, l, dt, beta}, and a staging
// tile for y, written back with a TMA store.
//
// Roles (22 warps): warp 0 TMA producer, warp 1 MMA issuer, warps 2..17 scores
// (one 32 x 32 block of the tile each: TMEM lane quarter warp % 4, column block
// (warp - 2) / 4), warps 18..21 epilogue.
#include <cmath>

#include "common.cuh"
#include "kernels.h"
#include "tc_common.cuh"
#include "tc_scan_common.cuh"
#include "tma_host.h"

namespace ssd {

namespace {

using namespace tc;

constexpr int kThreads = 704;
constexpr int kRows = 128;
constexpr int kScoreWarps = 16;
constexpr int kScoreThreads = 32 * kScoreWarps;
constexpr int kEpiWarp0 = 2 + kScoreWarps;
constexpr int kEpiThreads = 128;
constexpr int kTmemCols = 512;
constexpr uint32_t kColCBd = 0, kColP = 128, kColTmp = 128, kColAcc = 256;


struct Smem4 {
    uint32_t c_off, b_off, stage_off, stage_bytes, x_rel, s_rel, l_rel, dt_rel, beta_rel;
    uint32_t y_off, e_off, bar_off, total;
};

__host__ __device__ inline Smem4 scan4_smem(int Q, int N) {
    Smem4 s;
    s.c_off = 0;
    s.b_off = up1k(kRows * N * 2);
    // B rows for the CB MMAs; afterwards CBoff (128 x 128 bf16) in the same place
    s.stage_off = s.b_off + up1k(umax(Q * N * 2, Q > kRows ? kRows * kRows * 2 : 0));
    s.x_rel = 0;
    s.s_rel = Q * 128;
    s.l_rel = s.s_rel + up1k(64 * N * 2);
    s.dt_rel = s.l_rel + Q * 4;
    s.beta_rel = s.dt_rel + Q * 4;
    s.stage_bytes = up1k(s.beta_rel + Q * 4);
    s.y_off = s.stage_off + 2 * s.stage_bytes;
    s.e_off = s.y_off + kRows * 128;
    s.bar_off = s.e_off + 2 * kRows * 4;
    s.total = s.bar_off + 256 + 1024;
    return s;
}


// Work unit u: (b, c, tile mt, first head h0).  Normally units enumerate
// (b, c, mt, head block of hpc heads); in list mode (items != nullptr, hpc = 1)
// unit u is the packed item items[u] = b << 40 | c << 24 | mt << 16 | h.
struct Unit4 {
    int b, c, mt, h0;
};
__device__ __forceinline__ Unit4 unit_at(int u, const Dims &d, int hpc, int ntiles,
                                         const long long *items) {
    Unit4 x;
    if (items) {
        const long long v = items[u];
        x.b = int(v >> 40);
        x.c = int((v >> 24) & 0xFFFF);
        x.mt = int((v >> 16) & 0xFF);
        x.h0 = int(v & 0xFFFF);
    } else {
        const int nhb = d.H / hpc;
        const int rest = u / nhb;
        x.h0 = (u % nhb) * hpc;
        x.mt = rest % ntiles;
        x.c = (rest / ntiles) % d.nc;
        x.b = (rest / ntiles) / d.nc;
    }
    return x;
}

template <int N>
__global__ void __launch_bounds__(kThreads, 1)
chunk_scan4_kernel(const __grid_constant__ CUtensorMap tm_c, const __grid_constant__ CUtensorMap tm_b,
                   const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_s,
                   const __grid_constant__ CUtensorMap tm_y, Dims d, int hpc, int units,
                   const float *__restrict__ dtq, const float *__restrict__ betaq,
                   const float *__restrict__ Dskip, const float *__restrict__ lcum,
                   const long long *__restrict__ items, const int *__restrict__ nitems,
                   unsigned int *err) {
    // both words are read before either is tested (one memory latency, not two:
    // an empty list, the usual case in list mode, then costs one round trip)
    const unsigned int err_word = err ? *reinterpret_cast<const volatile unsigned int *>(err) : 0u;
    const int listed = items ? *nitems : units;  // list mode: the listed (b, c, tile, head) items
    if (err_word & 1u) return;               // an earlier wait expired: skip all work
    units = min(listed, units);
    if (int(blockIdx.x) >= units) return;    // no unit for this CTA (units are strided by the grid)
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int Q = d.Q;
    const Smem4 L = scan4_smem(Q, N);
    uint8_t *sC = smem + L.c_off;
    uint8_t *sB = smem + L.b_off;  // B rows, then CBoff
    uint8_t *sY = smem + L.y_off;
    float *sE = reinterpret_cast<float *>(smem + L.e_off);  // [2][128] row factors u_t
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L.bar_off);
    uint64_t *ld_cb = bars + 0, *cb_full = bars + 1, *cb_smem_free = bars + 2, *cvt_done = bars + 3;
    uint64_t *head_full = bars + 4, *head_free = bars + 6;      // [2]
    uint64_t *scores_ready = bars + 8, *p_free = bars + 10;     // [2]
    uint64_t *acc_full = bars + 12, *acc_free = bars + 14;      // [2]
    uint64_t *y_ready = bars + 16, *y_free = bars + 17, *done = bars + 18;
    uint64_t *scaled_ready = bars + 19;                         // [2]
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(bars + 21);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int ntiles = Q / kRows;
    constexpr int kSlabs = N >= 64 ? N / 64 : 1;
    constexpr int kRB = row_bytes(N);

    if (tid == 0) {
        mbar_init(ld_cb, 1);
        mbar_init(cb_full, 1);
        mbar_init(cb_smem_free, 1);
        mbar_init(cvt_done, kScoreThreads);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&head_full[i], 1);
            mbar_init(&head_free[i], 1);
            mbar_init(&scores_ready[i], kScoreThreads);
            mbar_init(&p_free[i], 1);
            mbar_init(&acc_full[i], 1);
            mbar_init(&acc_free[i], kEpiThreads);
            mbar_init(&scaled_ready[i], kScoreThreads);
        }
        mbar_init(y_ready, kEpiThreads);
        mbar_init(y_free, 1);
        mbar_init(done, 1);
        fence_mbar_init();
        tma_prefetch_desc(&tm_c);
        tma_prefetch_desc(&tm_b);
        tma_prefetch_desc(&tm_x);
        tma_prefetch_desc(&tm_s);
        tma_prefetch_desc(&tm_y);
    }
    if (warp == 1) tmem_alloc(tmem_holder, kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;

    if (warp == 0) {
        // =============================== producer ===============================
        if (lane == 0) {
            uint32_t ui = 0, hit = 0;
            bool ok = true;
            for (int u = blockIdx.x; u < units && ok; u += gridDim.x, ++ui) {
                const Unit4 U = unit_at(u, d, hpc, ntiles, items);
                const int mt = U.mt, c = U.c, b = U.b;
                const int h0 = U.h0, g = h0 / d.r;
                const int s_len = (mt + 1) * kRows;
                const int trow0 = b * d.T + c * Q;
                // C and B of this unit, once the previous unit's MMAs are done
                if (!mbar_wait(cb_smem_free, (ui & 1) ^ 1, err)) break;
                mbar_expect_tx(ld_cb, uint32_t(kRows) * N * 2 + uint32_t(s_len) * N * 2);
                for (int sl = 0; sl < kSlabs; ++sl) {
                    tma_load_3d(sC + sl * kRows * 128, &tm_c, ld_cb, sl * 64, g, trow0 + mt * kRows);
                    for (int i = 0; i <= mt; ++i)
                        tma_load_3d(sB + sl * s_len * 128 + i * kRows * kRB, &tm_b, ld_cb, sl * 64, g,
                                    trow0 + i * kRows);
                }
                for (int hi = 0; hi < hpc; ++hi, ++hit) {
                    const int st = hit & 1;
                    const int h = h0 + hi;
                    if (!mbar_wait(&head_free[st], ((hit >> 1) & 1) ^ 1, err)) { ok = false; break; }
                    uint8_t *stage = smem + L.stage_off + st * L.stage_bytes;
                    mbar_expect_tx(&head_full[st], uint32_t(s_len) * 128 + 64u * N * 2 + 3u * s_len * 4);
                    for (int i = 0; i <= mt; ++i)
                        tma_load_3d(stage + L.x_rel + i * kRows * 128, &tm_x, &head_full[st], 0, h,
                                    trow0 + i * kRows);
                    const int srow = ((b * d.nc + c) * d.H + h) * 64;
                    for (int sl = 0; sl < kSlabs; ++sl)
                        tma_load_2d(stage + L.s_rel + sl * 64 * 128, &tm_s, &head_full[st], sl * 64, srow);
                    const int64_t lo = off_lq(d, b, h, c);
                    bulk_load(stage + L.l_rel, lcum + lo, s_len * 4, &head_full[st]);
                    bulk_load(stage + L.dt_rel, dtq + lo, s_len * 4, &head_full[st]);
                    bulk_load(stage + L.beta_rel, betaq + lo, s_len * 4, &head_full[st]);
                }
            }
            // drain: the last loads issued must have landed before the CTA exits
            if (ui > 0) mbar_wait(ld_cb, (ui - 1) & 1, nullptr);
            for (uint32_t k = 0; k < 2 && k < hit; ++k) {
                const uint32_t i = hit - 1 - k;
                mbar_wait(&head_full[i & 1], (i >> 1) & 1, nullptr);
            }
        }
    } else if (warp == 1) {
        // =============================== MMA issuer =============================
        if (lane == 0) {
            uint32_t ui = 0, hit = 0;
            bool ok = true;
            const uint32_t ca = smem_u32(sC), ba = smem_u32(sB);
            const uint32_t idCB = idesc_bf16_f32(kRows, kRows, 0, 0);
            const uint32_t idX = idesc_bf16_f32(kRows, 64, 0, 1);
            const uint32_t idS = idesc_bf16_f32(kRows, 64, 0, 0);
            for (int u = blockIdx.x; u < units && ok; u += gridDim.x, ++ui) {
                const int mt = unit_at(u, d, hpc, ntiles, items).mt;
                const int s_len = (mt + 1) * kRows;
                if (!mbar_wait(ld_cb, ui & 1, err)) break;
                tc_fence_after();
                // CB on the diagonal tile (B rows [t0, t0 + 128)) and, for t0 > 0,
                // CB of the sources before the tile (B rows [0, 128)) into the score range
                const uint32_t bdiag = ba + mt * kRows * kRB;
                for (int k = 0; k < N / 16; ++k)
                    mma_bf16_ss(tmem + kColCBd, kmajor_desc(ca, k, kRows, N),
                                kmajor_desc(bdiag, k, s_len, N), idCB, k > 0 ? 1u : 0u);
                if (mt > 0)
                    for (int k = 0; k < N / 16; ++k)
                        mma_bf16_ss(tmem + kColTmp, kmajor_desc(ca, k, kRows, N),
                                    kmajor_desc(ba, k, s_len, N), idCB, k > 0 ? 1u : 0u);
                mma_commit(cb_full);
                for (int hi = 0; hi < hpc; ++hi, ++hit) {
                    const int st = hit & 1, pb = hit & 1, ab = hit & 1;
                    // Yoz first: it needs only the scaled operands, so it runs on the
                    // tensor cores while the score warps still build P
                    if (!mbar_wait(&head_full[st], (hit >> 1) & 1, err) ||
                        !mbar_wait(&scaled_ready[st], (hit >> 1) & 1, err) ||
                        !mbar_wait(&acc_free[ab], ((hit >> 1) & 1) ^ 1, err)) { ok = false; break; }
                    tc_fence_after();
                    const uint8_t *stage = smem + L.stage_off + st * L.stage_bytes;
                    const uint32_t xa = smem_u32(stage + L.x_rel);
                    const uint32_t sa = smem_u32(stage + L.s_rel);
                    const uint32_t dYd = tmem + kColAcc + ab * 128, dYo = dYd + 64;
                    // Yoz = CBoff X' + C S'^T
                    if (mt > 0)
                        for (int k = 0; k < kRows / 16; ++k)
                            mma_bf16_ss(dYo, kmajor_desc(ba, k, kRows, kRows),
                                        smem_desc(xa + k * 2048, 16, 1024, kSw128), idX, k > 0 ? 1u : 0u);
                    for (int k = 0; k < N / 16; ++k)
                        mma_bf16_ss(dYo, kmajor_desc(ca, k, kRows, N), kmajor_desc(sa, k, 64, N), idS,
                                    (mt > 0 || k > 0) ? 1u : 0u);
                    // Yd = P Xd
                    if (!mbar_wait(&scores_ready[pb], (hit >> 1) & 1, err)) { ok = false; break; }
                    tc_fence_after();
                    for (int k = 0; k < kRows / 16; ++k)
                        mma_bf16_ts(dYd, tmem + kColP + pb * 64 + k * 8,
                                    smem_desc(xa + mt * kRows * 128 + k * 2048, 16, 1024, kSw128), idX,
                                    k > 0 ? 1u : 0u);
                    mma_commit(&p_free[pb]);
                    mma_commit(&acc_full[ab]);
                    mma_commit(&head_free[st]);
                }
                if (ok) mma_commit(cb_smem_free);
            }
            mma_commit(done);
            mbar_wait(done, 0, nullptr);
        }
    } else if (warp < kEpiWarp0) {
        // ================================ scores ================================
        const int sid = tid - 64;            // 0..511
        const int qd = warp & 3;             // TMEM lane quarter of this warp
        const int cb = (warp - 2) >> 2;      // 32-column block of the tile
        const int t_local = qd * 32 + lane;  // row of the tile
        const int j0 = cb * 32;              // first column of the block
        const uint32_t lane_base = uint32_t(qd * 32) << 16;
        uint32_t ui = 0, hit = 0;
        bool ok = true;
        for (int u = blockIdx.x; u < units && ok; u += gridDim.x, ++ui) {
            const Unit4 U = unit_at(u, d, hpc, ntiles, items);
            const int mt = U.mt;
            const int t0 = mt * kRows;
            if (!mbar_wait(cb_full, ui & 1, err)) break;
            tc_fence_after();
            if (mt > 0) {
                // CBoff fp32 -> bf16, into shared memory as a K-major, 128B-swizzled
                // A operand: this thread packs row t_local, columns [j0, j0 + 32)
                uint8_t *slab = sB + (cb >> 1) * (kRows * 128);
                float v[32];
                tmem_ld32(tmem + lane_base + kColTmp + j0, v);
#pragma unroll
                for (int c4 = 0; c4 < 4; ++c4)
                    *reinterpret_cast<uint4 *>(slab + sw128_off(t_local, (cb & 1) * 4 + c4)) =
                        make_uint4(pack_bf16x2(v[8 * c4], v[8 * c4 + 1]),
                                   pack_bf16x2(v[8 * c4 + 2], v[8 * c4 + 3]),
                                   pack_bf16x2(v[8 * c4 + 4], v[8 * c4 + 5]),
                                   pack_bf16x2(v[8 * c4 + 6], v[8 * c4 + 7]));
                fence_proxy_async_smem();
            }
            // every score thread is done with the CBoff range before any score
            // buffer (same tensor-memory columns) is written
            tc_fence_before();
            mbar_arrive(cvt_done);
            if (!mbar_wait(cvt_done, ui & 1, err)) break;
            tc_fence_after();
            for (int hi = 0; hi < hpc; ++hi, ++hit) {
                const int st = hit & 1, pb = hit & 1, ab = hit & 1;
                const int h = U.h0 + hi;
                uint8_t *stage = smem + L.stage_off + st * L.stage_bytes;
                const float *sl_ = reinterpret_cast<const float *>(stage + L.l_rel);
                const float *sdt = reinterpret_cast<const float *>(stage + L.dt_rel);
                const float *beta = reinterpret_cast<const float *>(stage + L.beta_rel);
                if (!mbar_wait(&head_full[st], (hit >> 1) & 1, err)) { ok = false; break; }
                const float r = t0 > 0 ? sl_[t0 - 1] : 0.f;
                if (t0 > 0) {
                    // X' = g o X for sources before the tile, S' = exp(r) s_in
                    scale_chunks(stage + L.x_rel, t0 * 8, sid, kScoreThreads, [&](int k) {
                        const int s = k >> 3;
                        return __expf(r - sl_[s]) * sdt[s];
                    });
                    const float er = __expf(r);
                    scale_chunks(stage + L.s_rel, 64 * N * 2 / 16, sid, kScoreThreads,
                                 [&](int) { return er; });
                    fence_proxy_async_smem();
                }
                mbar_arrive(&scaled_ready[st]);
                // row factors for the epilogue (its previous use of sE[ab] has ended
                // once accumulator ab is free)
                if (sid < kRows) {
                    if (!mbar_wait(&acc_free[ab], ((hit >> 1) & 1) ^ 1, err)) { ok = false; break; }
                    sE[ab * kRows + sid] = __expf(sl_[t0 + sid] - r);
                }
                if (!mbar_wait(&p_free[pb], ((hit >> 1) & 1) ^ 1, err)) { ok = false; break; }
                tc_fence_after();
                const uint32_t pcol = tmem + lane_base + kColP + pb * 64 + (j0 >> 1);
                if (j0 > qd * 32) {
                    // block above the diagonal
                    uint32_t pk[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e) pk[e] = 0u;
                    tmem_st16(pcol, pk);
                } else if (j0 < qd * 32) {
                    // block entirely below the diagonal
                    float v[32];
                    tmem_ld32(tmem + lane_base + kColCBd + j0, v);
                    const float at = __expf(sl_[t0 + t_local] - sl_[t0 + j0 + 31]);
                    const float4 *b4 = reinterpret_cast<const float4 *>(beta + t0 + j0);
                    uint32_t pk[16];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const float4 bb = b4[e];
                        pk[2 * e] = pack_bf16x2(v[4 * e] * at * bb.x, v[4 * e + 1] * at * bb.y);
                        pk[2 * e + 1] = pack_bf16x2(v[4 * e + 2] * at * bb.z, v[4 * e + 3] * at * bb.w);
                    }
                    tmem_st16(pcol, pk);
                } else {
                    // block on the diagonal (warp-uniform branch), in two 16-column
                    // halves: row lane of the block sees sources 0..lane, and D_h
                    // sits on the diagonal
                    const float Dh = Dskip ? __ldg(Dskip + h) : 0.f;
                    const float lt = sl_[t0 + t_local];
                    const float lke = sl_[t0 + j0 + 31];
                    const bool factored = sl_[t0 + j0] - lke < 80.f;
                    const float at = __expf(lt - lke);
#pragma unroll
                    for (int hf = 0; hf < 2; ++hf) {
                        float v[16];
                        tmem_ld16(tmem + lane_base + kColCBd + j0 + 16 * hf, v);
                        if (factored) {
                            const float4 *b4 = reinterpret_cast<const float4 *>(beta + t0 + j0 + 16 * hf);
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const float4 bb = b4[e];
                                v[4 * e] *= at * bb.x;
                                v[4 * e + 1] *= at * bb.y;
                                v[4 * e + 2] *= at * bb.z;
                                v[4 * e + 3] *= at * bb.w;
                            }
                        } else {
#pragma unroll
                            for (int e = 0; e < 16; ++e) {
                                const int sidx = t0 + j0 + 16 * hf + e;
                                v[e] *= __expf(fminf(lt - sl_[sidx], 0.f)) * sdt[sidx];
                            }
                        }
                        uint32_t pk[8];
#pragma unroll
                        for (int e = 0; e < 16; e += 2) {
                            const int c0 = 16 * hf + e;  // column within the block
                            float p0 = c0 <= lane ? v[e] : 0.f;
                            float p1 = c0 + 1 <= lane ? v[e + 1] : 0.f;
                            if (c0 == lane) p0 += Dh;
                            if (c0 + 1 == lane) p1 += Dh;
                            pk[e >> 1] = pack_bf16x2(p0, p1);
                        }
                        tmem_st8(pcol + 8 * hf, pk);
                    }
                }
                tmem_wait_st();
                fence_proxy_async_smem();
                tc_fence_before();
                mbar_arrive(&scores_ready[pb]);
            }
        }
    } else {
        // =============================== epilogue ===============================
        const int qd = warp & 3;
        const int t_local = qd * 32 + lane;
        const uint32_t lane_base = uint32_t(qd * 32) << 16;
        const bool issuer = (warp == kEpiWarp0 && lane == 0);
        uint32_t hit = 0;
        bool ok = true;
        for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
            const Unit4 U = unit_at(u, d, hpc, ntiles, items);
            const int mt = U.mt, c = U.c, b = U.b;
            for (int hi = 0; hi < hpc; ++hi, ++hit) {
                const int ab = hit & 1;
                const int h = U.h0 + hi;
                if (!mbar_wait(&acc_full[ab], (hit >> 1) & 1, err)) { ok = false; break; }
                // the staging tile is free once the previous TMA store has read it
                if (!mbar_wait(y_free, (hit & 1) ^ 1, err)) { ok = false; break; }
                tc_fence_after();
                const float ut = sE[ab * kRows + t_local];
                // y = Yd + u_t Yoz, 16 columns at a time, staged in shared memory
                // (128B swizzle) for one TMA store of the tile
#pragma unroll
                for (int p0 = 0; p0 < 64; p0 += 16) {
                    uint32_t yd[16], yo[16];
                    tmem_ld16_nowait(tmem + lane_base + kColAcc + ab * 128 + p0, yd);
                    tmem_ld16_nowait(tmem + lane_base + kColAcc + ab * 128 + 64 + p0, yo);
                    tmem_wait_ld();
#pragma unroll
                    for (int q = 0; q < 2; ++q) {
                        uint32_t o[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int i = 8 * q + 2 * e;
                            o[e] = pack_bf16x2(fmaf(ut, __uint_as_float(yo[i]), __uint_as_float(yd[i])),
                                               fmaf(ut, __uint_as_float(yo[i + 1]), __uint_as_float(yd[i + 1])));
                        }
                        *reinterpret_cast<uint4 *>(sY + sw128_off(t_local, p0 / 8 + q)) =
                            make_uint4(o[0], o[1], o[2], o[3]);
                    }
                }
                tc_fence_before();
                mbar_arrive(&acc_free[ab]);
                fence_proxy_async_smem();
                mbar_arrive(y_ready);
                if (issuer) {
                    if (!mbar_wait(y_ready, hit & 1, err)) { ok = false; break; }
                    tma_store_3d(&tm_y, sY, 0, h, b * d.T + c * Q + mt * kRows);
                    bulk_commit();
                    bulk_wait_read();
                    mbar_arrive(y_free);
                }
            }
        }
        if (issuer) bulk_wait_all();
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) tmem_dealloc(tmem, kTmemCols);
}

// Heads per work unit: a divisor of the heads per group, at most 16, chosen so
// that the persistent grid's last round of units is as full as possible.
int heads_per_cta4(const Dims &d, int sms) {
    int best = 1;
    double best_eff = -1.0;
    for (int k = 1; k <= 16; ++k) {
        if (d.r % k) continue;
        const double units = double(d.B) * d.nc * (d.Q / kRows) * (d.H / k);
        const double rounds = std::ceil(units / sms);
        const double eff = units / (rounds * sms);
        if (eff > best_eff + 0.02 || (eff > best_eff - 0.02 && k > best)) {
            if (eff > best_eff) best_eff = eff;
            best = k;
        }
    }
    return best;
}

template <int N>
cudaError_t launch4(const Dims &d, const CUtensorMap *maps, int hpc, const float *dtq,
                    const float *beta, const float *D, const float *l, const long long *items,
                    const int *nitems, int max_items, unsigned int *err, cudaStream_t stream) {
    const Smem4 L = scan4_smem(d.Q, N);
    const int smem = int(L.total < 116 * 1024 ? 116 * 1024 : L.total);
    if (!smem_attr_once(reinterpret_cast<const void *>(chunk_scan4_kernel<N>), smem))
        return cudaErrorInvalidValue;
    const int units = items ? max_items : d.B * d.nc * (d.Q / kRows) * (d.H / hpc);
    const int sms = device_sm_count();
    const int grid = units < sms ? units : sms;
    if (grid == 0) return cudaSuccess;
    chunk_scan4_kernel<N><<<grid, kThreads, smem, stream>>>(maps[0], maps[1], maps[2], maps[3], maps[4],
                                                          d, hpc, units, dtq, beta, D, l, items,
                                                          nitems, err);
    return cudaGetLastError();
}

}  // namespace

bool tc_chunk_scan4_supported(const Dims &d) {
    const bool n_ok = d.N == 16 || d.N == 32 || d.N == 64 || d.N == 128;
    return d.P == 64 && n_ok && (d.Q == 128 || d.Q == 256) &&
           scan4_smem(d.Q, d.N).total <= 227 * 1024 &&
           int64_t(d.B) * d.nc * (d.Q / kRows) * d.H < (int64_t(1) << 31);
}

cudaError_t launch_chunk_scan_tc4(const Dims &d, const void *x, const float *dtq,
                                  const float *beta, const void *Bm, const void *Cm,
                                  const float *D, const float *l, const void *s_in_bf16, void *y,
                                  const long long *items, const int *nitems, int max_items,
                                  unsigned int *err, cudaStream_t stream) {
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
    CUtensorMap maps[5];
    if (!make_tmap_bf16(&maps[0], 3, Cm, bcdims, bcstr, bcbox, rb) ||
        !make_tmap_bf16(&maps[1], 3, Bm, bcdims, bcstr, bcbox, rb) ||
        !make_tmap_bf16(&maps[2], 3, x, xdims, xstr, xbox, 128) ||
        !make_tmap_bf16(&maps[3], 2, s_in_bf16, sdims, sstr, sbox, rb) ||
        !make_tmap_bf16(&maps[4], 3, y, xdims, xstr, xbox, 128))
        return cudaErrorInvalidValue;
    const int hpc = items ? 1 : heads_per_cta4(d, device_sm_count());
    switch (d.N) {
        case 16: return launch4<16>(d, maps, hpc, dtq, beta, D, l, items, nitems, max_items, err, stream);
        case 32: return launch4<32>(d, maps, hpc, dtq, beta, D, l, items, nitems, max_items, err, stream);
        case 64: return launch4<64>(d, maps, hpc, dtq, beta, D, l, items, nitems, max_items, err, stream);
        case 128: return launch4<128>(d, maps, hpc, dtq, beta, D, l, items, nitems, max_items, err, stream);
    }
    return cudaErrorInvalidValue;
}

}  // namespace ssd
