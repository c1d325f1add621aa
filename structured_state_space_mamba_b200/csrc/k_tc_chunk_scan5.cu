// k_tc_chunk_scan5.cu -- ssd_chunk_scan on the tensor cores, one work item per
// (batch, chunk, head) covering the whole chunk (chunk_len 128 or 256).
//
// Output of chunk c, head h:
//     y_t = exp(l_t) C_t s_in^T + sum_{s <= t} exp(l_t - l_s) dt_s (C_t . B_s) x_s + D_h x_t
// (the intra-chunk masked product (L o C B^T)(dt o X) of the chunked SSD
// algorithm -- aifetchly blog "Mamba-2 Architecture: State Space Duality
// Explained", "The Chunked SSD Algorithm", step 1; akillness.github.io "State
// Space Duality and Mamba-2", "The Scalar-Identity Structural Constraint" --
// plus the state carried in from earlier chunks and the skip term).
//
// The chunk is split into 128-row tiles k (one or two).  With the reference
// r_k = l_{128k-1} (r_0 = 0), u_t = exp(l_t - r_k) <= 1 and
// g_s = exp(r_k - l_s) dt_s, every decay factorises exactly as
// exp(l_t - l_s) dt_s = u_t g_s, so each tile needs ONE accumulator:
//     y_t = u_t Y_k[t],
//     Y_0 = P'_0 X_0 + C_0 s_in^T
//     Y_1 = P'_1 X_1 + CBoff X' + C_1 S'^T,
//     P'_k[t, s] = (C_t . B_s) g_s [s <= t] + [s = t] D_h / u_t   (t, s in tile k),
//     X'_s = exp(l_127 - l_s) dt_s x_s (s in tile 0),   S' = exp(l_127) s_in,
// with CBoff = C_1 B_0^T.  g_s and D_h/u_t grow like exp(decay range of the
// tile); a tile whose range r_k - l_{128k+127} reaches kSteep is therefore not
// computed here: its (b, c, k, h) is appended to a list that the block-factored
// kernel of k_tc_chunk_scan4.cu finishes in a second launch.
//
// Work: the (b, c, h) items are split into one contiguous range per CTA
// (persistent grid), walked in order; C and B are loaded, and C B^T computed
// on the tensor cores, once per run of heads of one group in one chunk.  Per
// head the x rows, s_in, l and dt of the chunk are loaded once (double
// buffered) and both tiles are computed from them.
//
// Tensor memory (512 columns): [0,128) C_0 B_0^T and [128,256) C_1 B_1^T (fp32);
// [256,384) the scores P'_0, P'_1 (bf16; at the start of a run this range holds
// CBoff in fp32); [384,512) the accumulators Y_0, Y_1.  With chunk_len 128 the
// two score/accumulator slots alternate between consecutive heads instead.
//
// Roles (22 warps): warp 0 TMA producer, warp 1 MMA issuer, warps 2..17 scores
// (one 32 x 32 block each: lane quarter warp % 4, column block (warp - 2) / 4),
// warps 18..21 epilogue (y = u_t Y, each warp staging its 32 rows in shared
// memory and writing them with its own TMA store).
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
constexpr uint32_t kColCB = 0, kColP = 256, kColTmp = 256, kColAcc = 384;
constexpr int kGStride = 384;  // floats per factor buffer: g0 [0,128), g1 [128,384)
// Tiles whose decay range reaches this go to the block-factored kernel: the
// factors g_s and D_h / u_t here stay below e^64.
constexpr float kSteep = 64.f;

struct Smem5 {
    uint32_t c_off, b_off, stage_off, stage_bytes, x_rel, s_rel, l_rel, dt_rel;
    uint32_t y_off, g_off, e_off, flag_off, bar_off, total;
};

__host__ __device__ inline Smem5 scan5_smem(int Q, int N) {
    Smem5 s;
    s.c_off = 0;
    s.b_off = up1k(Q * N * 2);                                      // C rows of the chunk
    s.stage_off = s.b_off + up1k(umax(kRows * N * 2, kRows * kRows * 2));  // B rows / CBoff
    s.x_rel = 0;
    s.s_rel = Q * 128;
    s.l_rel = s.s_rel + up1k(64 * N * 2);
    s.dt_rel = s.l_rel + Q * 4;
    s.stage_bytes = up1k(s.dt_rel + Q * 4);
    s.y_off = s.stage_off + 2 * s.stage_bytes;  // y staging: 128 rows x 128 bytes
    s.g_off = s.y_off + kRows * 128;
    s.e_off = s.g_off + 2 * kGStride * 4;
    s.flag_off = s.e_off + 2 * kRows * 4;
    s.bar_off = s.flag_off + 16;
    s.total = s.bar_off + 256 + 1024;
    return s;
}

// A operand: rows [128 k, 128 k + 128) of the C tile of Q rows, K step kk.
__device__ __forceinline__ uint64_t c_desc(uint32_t base, int k, int kk, int Q, int n) {
    if (n >= 64)
        return smem_desc(base + (kk >> 2) * Q * 128 + k * kRows * 128 + (kk & 3) * 32, 16, 1024, kSw128);
    return smem_desc(base + k * kRows * row_bytes(n) + kk * 32, 16, 8 * row_bytes(n), kmajor_swz(n));
}

// Items (b, c, h) in order, h fastest; a run = consecutive items of one
// (b, c, group).  Returns the run length starting at item i (< i1).
struct Run {
    int b, c, h, g, len;
};
__device__ __forceinline__ Run run_at(long long i, long long i1, const Dims &d) {
    Run r;
    r.h = int(i % d.H);
    const long long bc = i / d.H;
    r.c = int(bc % d.nc);
    r.b = int(bc / d.nc);
    r.g = r.h / d.r;
    const long long end_g = i + ((r.g + 1) * d.r - r.h);
    r.len = int((end_g < i1 ? end_g : i1) - i);
    return r;
}

template <int N>
__global__ void __launch_bounds__(kThreads, 1)
chunk_scan5_kernel(const __grid_constant__ CUtensorMap tm_c, const __grid_constant__ CUtensorMap tm_b,
                   const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_s,
                   const __grid_constant__ CUtensorMap tm_y, Dims d, const float *__restrict__ dtq,
                   const float *__restrict__ Dskip, const float *__restrict__ lcum,
                   int *__restrict__ nsteep, long long *__restrict__ steep_items, int max_steep,
                   unsigned int *err) {
    if (device_failed(err)) return;  // an earlier wait expired: skip all work
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int Q = d.Q;
    const bool two = Q == 2 * kRows;  // two tiles per chunk
    const Smem5 L = scan5_smem(Q, N);
    uint8_t *sC = smem + L.c_off;
    uint8_t *sB = smem + L.b_off;  // B rows of one tile, then CBoff (bf16)
    uint8_t *sY = smem + L.y_off;  // y staging, 32 rows per epilogue warp
    float *sG = reinterpret_cast<float *>(smem + L.g_off);   // [2][kGStride] per-token factors
    float *sE = reinterpret_cast<float *>(smem + L.e_off);   // [2][128] row factors u_t
    int *sFlag = reinterpret_cast<int *>(smem + L.flag_off);  // [2] tile left to the list
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L.bar_off);
    uint64_t *ld_c = bars + 0, *ld_b1 = bars + 1, *b0_free = bars + 2, *cb_full = bars + 3;
    uint64_t *cvt_done = bars + 4, *cb_smem_free = bars + 5;
    uint64_t *head_full = bars + 6, *head_free = bars + 8, *gsync = bars + 10;  // [2] each
    uint64_t *scores_ready = bars + 12, *p_free = bars + 14;                  // [2] each
    uint64_t *acc_full = bars + 16, *acc_free = bars + 18;                    // [2] each
    uint64_t *scaled_ready = bars + 20, *done = bars + 21;
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(bars + 22);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    constexpr int kSlabs = N >= 64 ? N / 64 : 1;
    constexpr int kRB = row_bytes(N);
    // this CTA's contiguous range of (b, c, h) items
    const long long n_items = (long long)d.B * d.nc * d.H;
    const long long i0 = n_items * blockIdx.x / gridDim.x;
    const long long i1 = n_items * (blockIdx.x + 1) / gridDim.x;

    if (tid == 0) {
        mbar_init(ld_c, 1);
        mbar_init(ld_b1, 1);
        mbar_init(b0_free, 1);
        mbar_init(cb_full, 1);
        mbar_init(cvt_done, kScoreThreads);
        mbar_init(cb_smem_free, 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&head_full[i], 1);
            mbar_init(&head_free[i], 1);
            mbar_init(&gsync[i], kScoreThreads);
            mbar_init(&scores_ready[i], kScoreThreads);
            mbar_init(&p_free[i], 1);
            mbar_init(&acc_full[i], 1);
            mbar_init(&acc_free[i], kEpiThreads);
        }
        mbar_init(scaled_ready, kScoreThreads);
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
            uint32_t si = 0, hit = 0;
            bool ok = true;
            for (long long i = i0; i < i1 && ok; ++si) {
                const Run R = run_at(i, i1, d);
                i += R.len;
                const int trow0 = R.b * d.T + R.c * Q;
                // C of the chunk and B of tile 0, once the previous run's MMAs are done
                if (!mbar_wait(cb_smem_free, (si & 1) ^ 1, err)) break;
                mbar_expect_tx(ld_c, uint32_t(Q) * N * 2 + uint32_t(kRows) * N * 2);
                for (int k = 0; k < Q / kRows; ++k)
                    for (int sl = 0; sl < kSlabs; ++sl)
                        tma_load_3d(sC + sl * Q * 128 + k * kRows * kRB, &tm_c, ld_c, sl * 64, R.g,
                                    trow0 + k * kRows);
                for (int sl = 0; sl < kSlabs; ++sl)
                    tma_load_3d(sB + sl * kRows * 128, &tm_b, ld_c, sl * 64, R.g, trow0);
                if (two) {
                    // B of tile 1 into the same place once the tile-0 products are done
                    if (!mbar_wait(b0_free, si & 1, err)) break;
                    mbar_expect_tx(ld_b1, uint32_t(kRows) * N * 2);
                    for (int sl = 0; sl < kSlabs; ++sl)
                        tma_load_3d(sB + sl * kRows * 128, &tm_b, ld_b1, sl * 64, R.g, trow0 + kRows);
                }
                for (int hi = 0; hi < R.len; ++hi, ++hit) {
                    const int st = hit & 1;
                    const int h = R.h + hi;
                    if (!mbar_wait(&head_free[st], ((hit >> 1) & 1) ^ 1, err)) { ok = false; break; }
                    uint8_t *stage = smem + L.stage_off + st * L.stage_bytes;
                    mbar_expect_tx(&head_full[st], uint32_t(Q) * 128 + 64u * N * 2 + 2u * Q * 4);
                    for (int k = 0; k < Q / kRows; ++k)
                        tma_load_3d(stage + L.x_rel + k * kRows * 128, &tm_x, &head_full[st], 0, h,
                                    trow0 + k * kRows);
                    const int srow = ((R.b * d.nc + R.c) * d.H + h) * 64;
                    for (int sl = 0; sl < kSlabs; ++sl)
                        tma_load_2d(stage + L.s_rel + sl * 64 * 128, &tm_s, &head_full[st], sl * 64, srow);
                    const int64_t lo = off_lq(d, R.b, h, R.c);
                    bulk_load(stage + L.l_rel, lcum + lo, Q * 4, &head_full[st]);
                    bulk_load(stage + L.dt_rel, dtq + lo, Q * 4, &head_full[st]);
                }
            }
            // drain: the last loads issued must have landed before the CTA exits
            for (uint32_t k = 0; k < 2 && k < hit; ++k) {
                const uint32_t i = hit - 1 - k;
                mbar_wait(&head_full[i & 1], (i >> 1) & 1, nullptr);
            }
            if (si > 0) {
                mbar_wait(ld_c, (si - 1) & 1, nullptr);
                if (two) mbar_wait(ld_b1, (si - 1) & 1, nullptr);
            }
        }
    } else if (warp == 1) {
        // =============================== MMA issuer =============================
        if (lane == 0) {
            uint32_t si = 0, hit = 0;
            bool ok = true;
            const uint32_t ca = smem_u32(sC), ba = smem_u32(sB);
            const uint32_t idCB = idesc_bf16_f32(kRows, kRows, 0, 0);
            const uint32_t idX = idesc_bf16_f32(kRows, 64, 0, 1);
            const uint32_t idS = idesc_bf16_f32(kRows, 64, 0, 0);
            for (long long i = i0; i < i1 && ok; ++si) {
                const Run R = run_at(i, i1, d);
                i += R.len;
                if (!mbar_wait(ld_c, si & 1, err)) break;
                tc_fence_after();
                // C_0 B_0^T and, for two tiles, CBoff = C_1 B_0^T (fp32, score range)
                for (int kk = 0; kk < N / 16; ++kk)
                    mma_bf16_ss(tmem + kColCB, c_desc(ca, 0, kk, Q, N), kmajor_desc(ba, kk, kRows, N), idCB,
                                kk > 0 ? 1u : 0u);
                if (two) {
                    for (int kk = 0; kk < N / 16; ++kk)
                        mma_bf16_ss(tmem + kColTmp, c_desc(ca, 1, kk, Q, N), kmajor_desc(ba, kk, kRows, N),
                                    idCB, kk > 0 ? 1u : 0u);
                    mma_commit(b0_free);
                    if (!mbar_wait(ld_b1, si & 1, err)) break;
                    tc_fence_after();
                    for (int kk = 0; kk < N / 16; ++kk)
                        mma_bf16_ss(tmem + kColCB + kRows, c_desc(ca, 1, kk, Q, N),
                                    kmajor_desc(ba, kk, kRows, N), idCB, kk > 0 ? 1u : 0u);
                }
                mma_commit(cb_full);
                for (int hi = 0; hi < R.len; ++hi, ++hit) {
                    const int st = hit & 1;
                    const uint32_t hp = (hit >> 1) & 1;
                    const uint8_t *stage = smem + L.stage_off + st * L.stage_bytes;
                    const uint32_t xa = smem_u32(stage + L.x_rel);
                    const uint32_t sa = smem_u32(stage + L.s_rel);
                    // tile 0 (or, for chunk_len 128, the slot of this head)
                    const int k0 = two ? 0 : st;
                    const uint32_t n0 = two ? (hit & 1) : hp;  // parity of this slot's use
                    if (!mbar_wait(&head_full[st], hp, err) ||
                        !mbar_wait(&acc_free[k0], n0 ^ 1, err)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t acc0 = tmem + kColAcc + k0 * 64;
                    // Y_0 = C_0 s_in^T ...
                    for (int kk = 0; kk < N / 16; ++kk)
                        mma_bf16_ss(acc0, c_desc(ca, 0, kk, Q, N), kmajor_desc(sa, kk, 64, N), idS,
                                    kk > 0 ? 1u : 0u);
                    // ... + P'_0 X_0
                    if (!mbar_wait(&scores_ready[k0], n0, err)) { ok = false; break; }
                    tc_fence_after();
                    for (int kk = 0; kk < kRows / 16; ++kk)
                        mma_bf16_ts(acc0, tmem + kColP + k0 * 64 + kk * 8,
                                    smem_desc(xa + kk * 2048, 16, 1024, kSw128), idX, 1u);
                    mma_commit(&p_free[k0]);
                    mma_commit(&acc_full[k0]);
                    if (two) {
                        const uint32_t acc1 = tmem + kColAcc + 64;
                        if (!mbar_wait(&acc_free[1], (hit & 1) ^ 1, err) ||
                            !mbar_wait(&scores_ready[1], hit & 1, err)) { ok = false; break; }
                        tc_fence_after();
                        // Y_1 = P'_1 X_1 ...
                        for (int kk = 0; kk < kRows / 16; ++kk)
                            mma_bf16_ts(acc1, tmem + kColP + 64 + kk * 8,
                                        smem_desc(xa + kRows * 128 + kk * 2048, 16, 1024, kSw128), idX,
                                        kk > 0 ? 1u : 0u);
                        mma_commit(&p_free[1]);
                        // ... + CBoff X' + C_1 S'^T (operands scaled in place by the score warps)
                        if (!mbar_wait(scaled_ready, hit & 1, err)) { ok = false; break; }
                        tc_fence_after();
                        for (int kk = 0; kk < kRows / 16; ++kk)
                            mma_bf16_ss(acc1, kmajor_desc(ba, kk, kRows, kRows),
                                        smem_desc(xa + kk * 2048, 16, 1024, kSw128), idX, 1u);
                        for (int kk = 0; kk < N / 16; ++kk)
                            mma_bf16_ss(acc1, c_desc(ca, 1, kk, Q, N), kmajor_desc(sa, kk, 64, N), idS, 1u);
                        mma_commit(&acc_full[1]);
                    }
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
        uint32_t si = 0, hit = 0;
        bool ok = true;
        for (long long i = i0; i < i1 && ok; ++si) {
            const Run R = run_at(i, i1, d);
            i += R.len;
            if (!mbar_wait(cb_full, si & 1, err)) break;
            tc_fence_after();
            if (two) {
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
            // (same tensor-memory columns) is written
            tc_fence_before();
            mbar_arrive(cvt_done);
            if (!mbar_wait(cvt_done, si & 1, err)) break;
            tc_fence_after();
            for (int hi = 0; hi < R.len; ++hi, ++hit) {
                const int st = hit & 1;
                const uint32_t hp = (hit >> 1) & 1;
                const int h = R.h + hi;
                uint8_t *stage = smem + L.stage_off + st * L.stage_bytes;
                const float *sl_ = reinterpret_cast<const float *>(stage + L.l_rel);
                const float *sdt = reinterpret_cast<const float *>(stage + L.dt_rel);
                float *gb = sG + st * kGStride;
                if (!mbar_wait(&head_full[st], hp, err)) { ok = false; break; }
                const float l127 = sl_[kRows - 1];
                // per-token factors: g0_s = exp(-l_s) dt_s (tile 0), and for two
                // tiles g1_s = exp(l_127 - l_s) dt_s (s < 128: X' factors; s >= 128:
                // tile-1 column factors).  Exponents are clamped at 80: beyond
                // kSteep the tile is left to the list anyway.
                if (sid < kRows) {
                    gb[sid] = __expf(fminf(-sl_[sid], 80.f)) * sdt[sid];
                } else if (two && sid < 3 * kRows) {
                    const int s = sid - kRows;
                    gb[kRows + s] = __expf(fminf(l127 - sl_[s], 80.f)) * sdt[s];
                }
                mbar_arrive(&gsync[st]);
                if (!mbar_wait(&gsync[st], hp, err)) { ok = false; break; }
                const bool steep0 = -l127 >= kSteep;
                const bool steep1 = two && (l127 - sl_[Q - 1] >= kSteep);
                if ((sid == 0 && steep0) || (sid == 1 && steep1)) {
                    const int idx = atomicAdd(nsteep, 1);
                    if (idx < max_steep)
                        steep_items[idx] = ((long long)R.b << 40) | ((long long)R.c << 24) |
                                           ((long long)sid << 16) | h;
                }
                const float Dh = Dskip ? __ldg(Dskip + h) : 0.f;
                const int ntile = two ? 2 : 1;
                for (int k = 0; k < ntile; ++k) {
                    const int slot = two ? k : st;
                    const uint32_t use = two ? (hit & 1) : hp;
                    const int t0 = k * kRows;
                    const float r = k == 0 ? 0.f : l127;
                    // row factors for the epilogue (its previous use of this slot
                    // has ended once the slot's accumulator is free)
                    if (sid < kRows) {
                        if (!mbar_wait(&acc_free[slot], use ^ 1, err)) { ok = false; break; }
                        sE[slot * kRows + sid] = __expf(sl_[t0 + sid] - r);
                        if (sid == 0) sFlag[slot] = k == 0 ? steep0 : steep1;
                    }
                    if (!mbar_wait(&p_free[slot], use ^ 1, err)) { ok = false; break; }
                    tc_fence_after();
                    const float *gcol = gb + (k == 0 ? 0 : 2 * kRows) + j0;  // factors of this block
                    const uint32_t pcol = tmem + lane_base + kColP + slot * 64 + (j0 >> 1);
                    const uint32_t cbcol = tmem + lane_base + kColCB + k * kRows + j0;
                    if (j0 > qd * 32) {
                        // block above the diagonal
                        uint32_t pk[16];
#pragma unroll
                        for (int e = 0; e < 16; ++e) pk[e] = 0u;
                        tmem_st16(pcol, pk);
                    } else if (j0 < qd * 32) {
                        // block entirely below the diagonal: column factors only
                        float v[32];
                        tmem_ld32(cbcol, v);
                        const float4 *g4 = reinterpret_cast<const float4 *>(gcol);
                        uint32_t pk[16];
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            const float4 gg = g4[e];
                            pk[2 * e] = pack_bf16x2(v[4 * e] * gg.x, v[4 * e + 1] * gg.y);
                            pk[2 * e + 1] = pack_bf16x2(v[4 * e + 2] * gg.z, v[4 * e + 3] * gg.w);
                        }
                        tmem_st16(pcol, pk);
                    } else {
                        // block on the diagonal (warp-uniform branch): row lane of the
                        // block sees sources 0..lane; D_h / u_t sits on the diagonal
                        const float dfac = Dh * __expf(fminf(r - sl_[t0 + t_local], 80.f));
#pragma unroll
                        for (int hf = 0; hf < 2; ++hf) {
                            float v[16];
                            tmem_ld16(cbcol + 16 * hf, v);
                            const float4 *g4 = reinterpret_cast<const float4 *>(gcol + 16 * hf);
                            uint32_t pk[8];
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const float4 gg = g4[e];
                                const int c0 = 16 * hf + 4 * e;  // column within the block
                                float p0 = c0 <= lane ? v[4 * e] * gg.x : 0.f;
                                float p1 = c0 + 1 <= lane ? v[4 * e + 1] * gg.y : 0.f;
                                float p2 = c0 + 2 <= lane ? v[4 * e + 2] * gg.z : 0.f;
                                float p3 = c0 + 3 <= lane ? v[4 * e + 3] * gg.w : 0.f;
                                if (c0 == lane) p0 += dfac;
                                if (c0 + 1 == lane) p1 += dfac;
                                if (c0 + 2 == lane) p2 += dfac;
                                if (c0 + 3 == lane) p3 += dfac;
                                pk[2 * e] = pack_bf16x2(p0, p1);
                                pk[2 * e + 1] = pack_bf16x2(p2, p3);
                            }
                            tmem_st8(pcol + 8 * hf, pk);
                        }
                    }
                    tmem_wait_st();
                    tc_fence_before();
                    mbar_arrive(&scores_ready[slot]);
                }
                if (!ok) break;
                if (two) {
                    // X' = g1 o X_0 and S' = exp(l_127) s_in, in place, once this
                    // head's tile-0 products (which read them unscaled) are done
                    if (!mbar_wait(&p_free[0], hit & 1, err)) { ok = false; break; }
                    scale_chunks(stage + L.x_rel, kRows * 8, sid, kScoreThreads,
                                 [&](int k) { return gb[kRows + (k >> 3)]; });
                    const float el = __expf(l127);
                    scale_chunks(stage + L.s_rel, 64 * N * 2 / 16, sid, kScoreThreads,
                                 [&](int) { return el; });
                    fence_proxy_async_smem();
                    mbar_arrive(scaled_ready);
                }
            }
        }
    } else {
        // =============================== epilogue ===============================
        // y_t = u_t Y[t]: each warp stages its 32 rows (128B swizzle) and writes
        // them with its own TMA store, so the warps never wait on one another
        const int qd = warp & 3;
        const int t_local = qd * 32 + lane;
        const uint32_t lane_base = uint32_t(qd * 32) << 16;
        uint8_t *sYw = sY + qd * 32 * 128;
        uint32_t hit = 0;
        bool ok = true;
        for (long long i = i0; i < i1 && ok;) {
            const Run R = run_at(i, i1, d);
            i += R.len;
            for (int hi = 0; hi < R.len && ok; ++hi, ++hit) {
                const int h = R.h + hi;
                const int ntile = two ? 2 : 1;
                for (int k = 0; k < ntile; ++k) {
                    const int slot = two ? k : (hit & 1);
                    const uint32_t use = two ? (hit & 1) : ((hit >> 1) & 1);
                    if (!mbar_wait(&acc_full[slot], use, err)) { ok = false; break; }
                    tc_fence_after();
                    const bool store = !sFlag[slot];
                    const float ut = sE[slot * kRows + t_local];
                    // this warp's previous TMA store has finished reading the staging rows
                    if (lane == 0) bulk_wait_read();
                    __syncwarp();
#pragma unroll
                    for (int p0 = 0; p0 < 64; p0 += 16) {
                        uint32_t a[16];
                        tmem_ld16_nowait(tmem + lane_base + kColAcc + slot * 64 + p0, a);
                        tmem_wait_ld();
                        uint32_t o[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e)
                            o[e] = pack_bf16x2(ut * __uint_as_float(a[2 * e]), ut * __uint_as_float(a[2 * e + 1]));
                        *reinterpret_cast<uint4 *>(sY + sw128_off(t_local, p0 / 8)) = make_uint4(o[0], o[1], o[2], o[3]);
                        *reinterpret_cast<uint4 *>(sY + sw128_off(t_local, p0 / 8 + 1)) = make_uint4(o[4], o[5], o[6], o[7]);
                    }
                    tc_fence_before();
                    mbar_arrive(&acc_free[slot]);
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0 && store) {
                        tma_store_3d(&tm_y, sYw, 0, h, R.b * d.T + R.c * Q + k * kRows + qd * 32);
                        bulk_commit();
                    }
                }
            }
        }
        if (lane == 0) bulk_wait_all();
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) tmem_dealloc(tmem, kTmemCols);
}

template <int N>
cudaError_t launch5(const Dims &d, const CUtensorMap *maps, const float *dtq, const float *D,
                    const float *l, int *nsteep, long long *items, int max_items,
                    unsigned int *err, cudaStream_t stream) {
    const Smem5 L = scan5_smem(d.Q, N);
    if (!smem_attr_once(reinterpret_cast<const void *>(chunk_scan5_kernel<N>), int(L.total)))
        return cudaErrorInvalidValue;
    const long long n_items = (long long)d.B * d.nc * d.H;
    const int sms = device_sm_count();
    const int grid = n_items < sms ? int(n_items) : sms;
    chunk_scan5_kernel<N><<<grid, kThreads, L.total, stream>>>(
        maps[0], maps[1], maps[2], maps[3], maps[4], d, dtq, D, l, nsteep, items, max_items, err);
    return cudaGetLastError();
}

}  // namespace

bool tc_chunk_scan5_supported(const Dims &d) {
    const bool n_ok = d.N == 16 || d.N == 128;
    return d.P == 64 && n_ok && (d.Q == 128 || d.Q == 256) &&
           scan5_smem(d.Q, d.N).total <= 227 * 1024 && d.H < 65536 && d.nc < 65536 &&
           d.B < 65536;
}

int chunk_scan5_max_steep(const Dims &d) { return d.B * d.nc * d.H * (d.Q / kRows); }

cudaError_t launch_chunk_scan_tc5(const Dims &d, const void *x, const float *dtq, const void *Bm,
                                  const void *Cm, const float *D, const float *l,
                                  const void *s_in_bf16, void *y, int *nsteep, long long *items,
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
    const uint32_t ybox[3] = {64, 1, 32};  // one epilogue warp's 32 rows
    CUtensorMap maps[5];
    if (!make_tmap_bf16(&maps[0], 3, Cm, bcdims, bcstr, bcbox, rb) ||
        !make_tmap_bf16(&maps[1], 3, Bm, bcdims, bcstr, bcbox, rb) ||
        !make_tmap_bf16(&maps[2], 3, x, xdims, xstr, xbox, 128) ||
        !make_tmap_bf16(&maps[3], 2, s_in_bf16, sdims, sstr, sbox, rb) ||
        !make_tmap_bf16(&maps[4], 3, y, xdims, xstr, ybox, 128))
        return cudaErrorInvalidValue;
    const int max_items = chunk_scan5_max_steep(d);
    switch (d.N) {
        case 16: return launch5<16>(d, maps, dtq, D, l, nsteep, items, max_items, err, stream);
        case 128: return launch5<128>(d, maps, dtq, D, l, nsteep, items, max_items, err, stream);
    }
    return cudaErrorInvalidValue;
}

}  // namespace ssd
