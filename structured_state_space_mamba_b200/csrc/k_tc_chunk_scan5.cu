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
// With a reference r per (chunk, head), u_t = exp(l_t - r) and
// g_s = exp(r - l_s) dt_s, every decay factorises exactly as
// exp(l_t - l_s) dt_s = u_t g_s, so the masked scores do not depend on the head:
//     y_t = u_t Y[t] + D_h x_t,   Y = (C B^T o M) X'' + C S'^T,
//     X''_s = g_s x_s,  S' = e^r s_in   (scaled per head, in shared memory),
// with M the causal mask (diagonal included); the epilogue adds the skip term
// D_h x_t = (D_h / g_t) X''_t from the scaled rows.  The chunk is split into
// 128-row tiles k; tile 1 also takes the sources of tile 0 through
// CBoff = C_1 B_0^T:
//     Y_0 = P_0 X''_0 + C_0 S'^T,   Y_1 = P_1 X''_1 + CBoff X''_0 + C_1 S'^T.
// The masked scores P_k = C_k B_k^T o M are built once per run of heads of one
// group in one chunk and shared by all of them; per head only x (and s_in when
// r != 0) is scaled.
// r is 0 (u_t <= 1), or l_127 when the chunk's decay range reaches kScanSteep
// but neither tile's does.  g_s reaches exp(r - l_s): a tile whose
// r - l_{128k+127} reaches kScanSteep, or with a zero dt, is flagged by the
// cumsum kernel; it is not stored here but appended to a list that the
// block-factored kernel of k_tc_chunk_scan4.cu finishes in a second launch.
//
// Work: the (b, c, h) items are split into one contiguous range per CTA
// (persistent grid), walked in order.  Per head the chunk's x rows and s_in
// go through a ring of three stages (l and g through a ring of their own); a
// run's start borrows two stages of the ring for C_0 and the B tiles, so a
// stage is reused three uses later, once the use's products are done and the
// epilogue has read the head's scaled rows.  C_1 stays in its own buffer for
// the run.
//
// Tensor memory (512 columns): [0,128) P_0, P_1 (bf16); [256,384) CBoff and
// C_0 (bf16 A operands of TS products: CBoff in [256,288) and [320,352), C_0 in
// [288,320) and [352,384); with dstate 256, which runs 128-token chunks only,
// C_0 takes all of [256,384)); two accumulator buffers {Y_0, Y_1} at [384,512) and
// [128,256), alternating between heads.  At the start of a run the fp32 C B^T
// tiles pass through them (C_0 B_0^T -> [384,512), C_1 B_1^T -> [128,256),
// CBoff -> [256,384)), so a run starts once the accumulators of the previous
// heads are read.
//
// Roles (14 warps): warp 0 TMA producer, warp 1 MMA issuer, warps 2..9 score /
// scale warps (at the start of a run two 32 x 32 score blocks each -- lane
// quarter warp % 4, column blocks 2 (warp - 2) / 4 + {0, 1} -- and half of
// C_0's row; x scaling per head), warps 10..13 epilogue (y = u_t Y + D_h x,
// each warp staging its 32 rows, 32 columns at a time, and writing them with
// its own TMA stores).
#include <cmath>

#include "common.cuh"
#include "kernels.h"
#include "tc_common.cuh"
#include "tc_scan_common.cuh"
#include "tma_host.h"

namespace ssd {

namespace {

using namespace tc;

constexpr int kThreads = 448;
constexpr int kRows = 128;
constexpr int kScoreWarps = 8;
constexpr int kScoreThreads = 32 * kScoreWarps;
constexpr int kEpiWarp0 = 2 + kScoreWarps;
constexpr int kEpiThreads = 128;
constexpr int kTmemCols = 512;
constexpr int kStages = 3;  // x / s_in stages (a run's start borrows two)
constexpr uint32_t kColP = 0, kColOff = 256;
// packed CBoff: 32-column block cb (16 bf16 pairs) within the fp32 range that
// the two score warps of column blocks {2 (cb / 2), 2 (cb / 2) + 1} read
__device__ __forceinline__ uint32_t off_col(int cb) { return kColOff + (cb >> 1) * 64 + (cb & 1) * 16; }
// accumulator buffer ab of a head (hit & 1)
__device__ __forceinline__ uint32_t acc_col(int ab) { return ab == 0 ? 384u : 128u; }
// C_0 (bf16, A operand of the C_0 S'^T products), K step kk: the second half of
// each score warp pair's CBoff source range, free once CBoff is packed; with
// dstate 256 (128-token chunks only, so no CBoff) the whole range [256,384)
template <int N>
__device__ __forceinline__ uint32_t c0_col(int kk) {
    if (N == 256) return kColOff + kk * 8;
    return kColOff + 32 + (kk >> 2) * 64 + (kk & 3) * 8;
}

struct Smem5 {
    uint32_t c1_off, stage_off, stage_bytes, s_rel, lg_off, lg_bytes, y_off, bar_off, total;
};

// C_1 (tile 1 of C, for the C_1 S'^T products) stays for the whole run; a stage
// holds a head's x rows and s_in, or at a run's start C_0 (first stage) and the
// B tiles (second); l and g ride in a ring of their own.
__host__ __device__ inline Smem5 scan5_smem(int Q, int N) {
    Smem5 s;
    s.c1_off = 0;
    s.stage_off = Q == 2 * kRows ? up1k(kRows * N * 2) : 0;
    s.s_rel = Q * 128;
    s.stage_bytes = umax(up1k(s.s_rel + 64 * N * 2), up1k(kRows * N * 2));
    s.lg_off = s.stage_off + kStages * s.stage_bytes;
    s.lg_bytes = (Q * 4 + chunk_gq(Q) * 4 + 127) & ~127u;  // l (Q floats), then g, flags, r
    s.y_off = up1k(s.lg_off + kStages * s.lg_bytes);  // y staging: 128 rows x 128 bytes
    s.bar_off = s.y_off + kRows * 128;
    s.total = s.bar_off + 256 + 1024;
    return s;
}

// Start-address step (in 16-byte units) of K step kk in a K-major operand of
// `rows` rows, relative to K step 0 (the layouts of kmajor_desc).
template <int N>
__device__ __forceinline__ uint64_t kdesc_step_n(int kk, int rows) {
    if (N >= 64) return uint64_t(((kk >> 2) * rows * 128 + (kk & 3) * 32) >> 4);
    return uint64_t((kk * 32) >> 4);
}

// Items (b, c, h) in order, h fastest; a run = consecutive items of one
// (b, c, group).  Returns the run starting at item i (< i1).
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

// fp32 32 x 32 block (one TMEM row per lane) -> bf16 pairs, all columns or,
// for a block on the diagonal, columns e <= lane only.
template <bool kDiag>
__device__ __forceinline__ void mask_pack(const float (&v)[32], int lane, uint32_t (&pk)[16]) {
#pragma unroll
    for (int e = 0; e < 16; ++e) {
        const float a = (!kDiag || 2 * e <= lane) ? v[2 * e] : 0.f;
        const float b = (!kDiag || 2 * e + 1 <= lane) ? v[2 * e + 1] : 0.f;
        pk[e] = pack_bf16x2(a, b);
    }
}

template <int N>
__global__ void __launch_bounds__(kThreads, 1)
chunk_scan5_kernel(const __grid_constant__ CUtensorMap tm_c, const __grid_constant__ CUtensorMap tm_b,
                   const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_s,
                   const __grid_constant__ CUtensorMap tm_y, Dims d, const float *__restrict__ gq,
                   const float *__restrict__ Dskip, const float *__restrict__ lcum,
                   int *__restrict__ nsteep, long long *__restrict__ steep_items, int max_steep,
                   unsigned int *err) {
    if (device_failed(err)) return;  // an earlier wait expired: skip all work
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int Q = d.Q;
    const bool two = Q == 2 * kRows;  // two tiles per chunk
    const int ntile = two ? 2 : 1;
    const int ngq = chunk_gq(Q);
    const Smem5 L = scan5_smem(Q, N);
    uint8_t *sC1 = smem + L.c1_off;  // C_1 (two tiles only)
    uint8_t *sY = smem + L.y_off;    // y staging, 32 rows per epilogue warp
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L.bar_off);
    uint64_t *ld_c = bars + 0, *ld_b1 = bars + 1, *b0_free = bars + 2, *cb_full = bars + 3;
    uint64_t *cvt_done = bars + 4, *cb_smem_free = bars + 5;
    uint64_t *head_full = bars + 6, *stage_free = bars + 9, *ready = bars + 12;  // [kStages] each
    uint64_t *acc_full = bars + 15, *acc_free = bars + 17;                      // [2] each
    uint64_t *done = bars + 19;
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(bars + 20);
    auto stage_at = [&](uint32_t use) { return smem + L.stage_off + (use % kStages) * L.stage_bytes; };
    auto lg_at = [&](uint32_t use) {
        return reinterpret_cast<float *>(smem + L.lg_off + (use % kStages) * L.lg_bytes);
    };

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
        for (int i = 0; i < kStages; ++i) {
            mbar_init(&head_full[i], 1);
            // the use's products (one commit) and the epilogue, which reads a
            // head's scaled rows
            mbar_init(&stage_free[i], 1 + kEpiThreads);
            mbar_init(&ready[i], kScoreThreads);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&acc_full[i], 1);
            mbar_init(&acc_free[i], kEpiThreads);
        }
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

    // Every role walks the same sequence of stage uses: per run, two for its
    // start (C_0, then the B tiles), then one per head.
    if (warp == 0) {
        // =============================== producer ===============================
        if (lane == 0) {
            uint32_t si = 0, use = 0, nc_issued = 0, nb1_issued = 0;
            bool ok = true;
            for (long long i = i0; i < i1 && ok; ++si) {
                const Run R = run_at(i, i1, d);
                i += R.len;
                const int trow0 = R.b * d.T + R.c * Q;
                // C_0 and B_0 into the next two stages, C_1 into its own buffer
                // once the previous run's products are done
                const uint32_t uc = use, ub = use + 1;
                if (!mbar_wait(&stage_free[uc % kStages], ((uc / kStages) & 1) ^ 1, err) ||
                    !mbar_wait(&stage_free[ub % kStages], ((ub / kStages) & 1) ^ 1, err) ||
                    !mbar_wait(cb_smem_free, (si & 1) ^ 1, err))
                    break;
                uint8_t *sc0 = stage_at(uc), *sb = stage_at(ub);
                // these two uses carry no head: their head_full phases pass at once
                mbar_arrive(&head_full[uc % kStages]);
                mbar_arrive(&head_full[ub % kStages]);
                use += 2;  // counted once armed (the exit drain waits on every counted use)
                mbar_expect_tx(ld_c, uint32_t(ntile + 1) * kRows * N * 2);
                for (int sl = 0; sl < kSlabs; ++sl) {
                    tma_load_3d(sc0 + sl * kRows * 128, &tm_c, ld_c, sl * 64, R.g, trow0);
                    tma_load_3d(sb + sl * kRows * 128, &tm_b, ld_c, sl * 64, R.g, trow0);
                    if (two) tma_load_3d(sC1 + sl * kRows * 128, &tm_c, ld_c, sl * 64, R.g, trow0 + kRows);
                }
                ++nc_issued;
                if (two) {
                    // B of tile 1 into the same place once the tile-0 products are done
                    if (!mbar_wait(b0_free, si & 1, err)) break;
                    mbar_expect_tx(ld_b1, uint32_t(kRows) * N * 2);
                    for (int sl = 0; sl < kSlabs; ++sl)
                        tma_load_3d(sb + sl * kRows * 128, &tm_b, ld_b1, sl * 64, R.g, trow0 + kRows);
                    ++nb1_issued;
                }
                for (int hi = 0; hi < R.len; ++hi, ++use) {
                    const int st = use % kStages;
                    const int h = R.h + hi;
                    if (!mbar_wait(&stage_free[st], ((use / kStages) & 1) ^ 1, err)) { ok = false; break; }
                    uint8_t *stage = stage_at(use);
                    float *lg = lg_at(use);
                    mbar_expect_tx(&head_full[st], uint32_t(Q) * 128 + 64u * N * 2 + uint32_t(Q + ngq) * 4);
                    for (int k = 0; k < ntile; ++k)
                        tma_load_3d(stage + k * kRows * 128, &tm_x, &head_full[st], 0, h, trow0 + k * kRows);
                    const int srow = ((R.b * d.nc + R.c) * d.H + h) * 64;
                    for (int sl = 0; sl < kSlabs; ++sl)
                        tma_load_2d(stage + L.s_rel + sl * 64 * 128, &tm_s, &head_full[st], sl * 64, srow);
                    bulk_load(lg, lcum + off_lq(d, R.b, h, R.c), Q * 4, &head_full[st]);
                    bulk_load(lg + Q, gq + ((int64_t(R.b) * d.H + h) * d.nc + R.c) * ngq, ngq * 4,
                              &head_full[st]);
                }
            }
            // drain: the loads issued have landed before the CTA exits (their own
            // completion barriers, so this holds on the early-out path too, where
            // the consumers stop freeing stages)
            for (uint32_t k = 1; k <= kStages && k <= use; ++k) {
                const uint32_t u = use - k;
                mbar_wait(&head_full[u % kStages], (u / kStages) & 1, nullptr);
            }
            if (nc_issued > 0) mbar_wait(ld_c, (nc_issued - 1) & 1, nullptr);
            if (nb1_issued > 0) mbar_wait(ld_b1, (nb1_issued - 1) & 1, nullptr);
        }
    } else if (warp == 1) {
        // =============================== MMA issuer =============================
        if (lane == 0) {
            uint32_t si = 0, hit = 0, use = 0;
            bool ok = true;
            const uint32_t c1a = smem_u32(sC1);
            const uint64_t c1d = kmajor_desc(c1a, 0, kRows, N);
            const uint32_t idCB = idesc_bf16_f32(kRows, kRows, 0, 0);
            const uint32_t idX = idesc_bf16_f32(kRows, 64, 0, 1);
            const uint32_t idS = idesc_bf16_f32(kRows, 64, 0, 0);
            for (long long i = i0; i < i1 && ok; ++si) {
                const Run R = run_at(i, i1, d);
                i += R.len;
                const uint32_t uc = use, ub = use + 1;
                use += 2;
                const uint32_t c0a = smem_u32(stage_at(uc)), ba = smem_u32(stage_at(ub));
                // the fp32 C B^T tiles pass through the accumulator columns: wait
                // until the epilogue has read the previous heads' accumulators
                for (uint32_t j = 1; j <= 2 && j <= hit && ok; ++j) {
                    const uint32_t hh = hit - j;
                    ok = mbar_wait(&acc_free[hh & 1], (hh >> 1) & 1, err);
                }
                if (!ok || !mbar_wait(ld_c, si & 1, err)) break;
                tc_fence_after();
                // C_0 B_0^T -> [384,512) and, for two tiles, CBoff = C_1 B_0^T -> [256,384)
                for (int kk = 0; kk < N / 16; ++kk)
                    mma_bf16_ss(tmem + acc_col(0), kmajor_desc(c0a, kk, kRows, N), kmajor_desc(ba, kk, kRows, N),
                                idCB, kk > 0 ? 1u : 0u);
                if (two) {
                    for (int kk = 0; kk < N / 16; ++kk)
                        mma_bf16_ss(tmem + kColOff, kmajor_desc(c1a, kk, kRows, N),
                                    kmajor_desc(ba, kk, kRows, N), idCB, kk > 0 ? 1u : 0u);
                    mma_commit(b0_free);
                    if (!mbar_wait(ld_b1, si & 1, err)) break;
                    tc_fence_after();
                    // C_1 B_1^T -> [128,256)
                    for (int kk = 0; kk < N / 16; ++kk)
                        mma_bf16_ss(tmem + acc_col(1), kmajor_desc(c1a, kk, kRows, N),
                                    kmajor_desc(ba, kk, kRows, N), idCB, kk > 0 ? 1u : 0u);
                }
                mma_commit(cb_full);
                // the scores of this run (and C_0 in tensor memory) exist once the
                // score warps have converted them; the run's two stages go back
                if (!mbar_wait(cvt_done, si & 1, err)) break;
                tc_fence_after();
                // (the epilogue does not read them: its share is arrived here; both
                // stages' previous uses were released before C_0 and B landed)
                mma_commit(&stage_free[uc % kStages]);
                mma_commit(&stage_free[ub % kStages]);
                mbar_arrive_cnt(&stage_free[uc % kStages], kEpiThreads);
                mbar_arrive_cnt(&stage_free[ub % kStages], kEpiThreads);
                for (int hi = 0; hi < R.len; ++hi, ++hit, ++use) {
                    const int st = use % kStages, ab = hit & 1;
                    const uint32_t sp = (use / kStages) & 1, hp = (hit >> 1) & 1;
                    const uint8_t *stage = stage_at(use);
                    const uint32_t xa = smem_u32(stage);
                    const uint32_t sa = smem_u32(stage + L.s_rel);
                    if (!mbar_wait(&head_full[st], sp, err) || !mbar_wait(&ready[st], sp, err) ||
                        !mbar_wait(&acc_free[ab], hp ^ 1, err)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t acc = tmem + acc_col(ab);
                    // Y_0 = C_0 S'^T + P_0 X''_0 and Y_1 = C_1 S'^T + CBoff X''_0 + P_1 X''_1.
                    // Descriptors are formed once per head; each K step adds a
                    // constant to the start-address field (no carry: every
                    // address stays inside shared memory).
                    const uint64_t xd = smem_desc(xa, 16, 1024, kSw128);
                    const uint64_t sd = kmajor_desc(sa, 0, 64, N);
#pragma unroll
                    for (int kk = 0; kk < N / 16; ++kk) {
                        mma_bf16_ts(acc, tmem + c0_col<N>(kk), sd + kdesc_step_n<N>(kk, 64), idS, kk > 0 ? 1u : 0u);
                        if (two)
                            mma_bf16_ss(acc + 64, c1d + kdesc_step_n<N>(kk, kRows), sd + kdesc_step_n<N>(kk, 64), idS,
                                        kk > 0 ? 1u : 0u);
                    }
#pragma unroll
                    for (int kk = 0; kk < kRows / 16; ++kk) {
                        const uint64_t x0 = xd + uint64_t(kk * (2048 >> 4));
                        mma_bf16_ts(acc, tmem + kColP + kk * 8, x0, idX, 1u);
                        if (two) mma_bf16_ts(acc + 64, tmem + off_col(kk >> 1) + (kk & 1) * 8, x0, idX, 1u);
                    }
                    if (two) {
#pragma unroll
                        for (int kk = 0; kk < kRows / 16; ++kk)
                            mma_bf16_ts(acc + 64, tmem + kColP + 64 + kk * 8,
                                        xd + uint64_t((kRows * 128 + kk * 2048) >> 4), idX, 1u);
                    }
                    mma_commit(&acc_full[ab]);
                    mma_commit(&stage_free[st]);
                }
                if (ok) mma_commit(cb_smem_free);
            }
            mma_commit(done);
            mbar_wait(done, 0, nullptr);
        }
    } else if (warp < kEpiWarp0) {
        // ============================ scores / scaling ==========================
        const int sid = tid - 64;            // 0..255
        const int qd = warp & 3;             // TMEM lane quarter of this warp
        const int cb0 = 2 * ((warp - 2) >> 2);  // first of its two 32-column blocks
        const uint32_t lane_base = uint32_t(qd * 32) << 16;
        uint32_t si = 0, use = 0;
        bool ok = true;
        for (long long i = i0; i < i1 && ok; ++si) {
            const Run R = run_at(i, i1, d);
            i += R.len;
            const uint32_t uc = use;
            use += 2;
            if (!mbar_wait(cb_full, si & 1, err) || !mbar_wait(ld_c, si & 1, err)) break;
            tc_fence_after();
            // ---- masked scores of this run: fp32 C B^T -> bf16 P_k, CBoff ----
            // block (qd, cb) of a tile: below the diagonal all columns, on it the
            // causal half, above it zeros.  P ([0,128)) overlaps no fp32 source;
            // CBoff is packed in place, each warp within its own source columns.
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                if (k == 1 && !two) break;
                const uint32_t src = acc_col(k);  // C_0 B_0^T, C_1 B_1^T
#pragma unroll
                for (int bb = 0; bb < 2; ++bb) {
                    const int cb = cb0 + bb;
                    uint32_t pk[16];
                    if (cb > qd) {
#pragma unroll
                        for (int e = 0; e < 16; ++e) pk[e] = 0u;
                    } else {
                        float v[32];
                        tmem_ld32(tmem + lane_base + src + cb * 32, v);
                        if (cb < qd) mask_pack<false>(v, lane, pk);
                        else mask_pack<true>(v, lane, pk);
                    }
                    tmem_st16(tmem + lane_base + kColP + k * 64 + cb * 16, pk);
                }
            }
            if (two) {
                // CBoff in place: packed block cb goes to the first half of this
                // warp's own fp32 range (off_col), so no other warp's source is
                // overwritten; one block at a time, each read before it is replaced
#pragma unroll
                for (int bb = 0; bb < 2; ++bb) {
                    float v[32];
                    uint32_t pk[16];
                    tmem_ld32(tmem + lane_base + kColOff + (cb0 + bb) * 32, v);
                    mask_pack<false>(v, lane, pk);
                    tmem_st16(tmem + lane_base + off_col(cb0 + bb), pk);
                }
            }
            // C_0 into tensor memory: row t, K half cb0 / 2 (one 128-byte swizzled
            // slab row per 64 columns of dstate, or the 32-byte row for N = 16)
            {
                const int t = qd * 32 + lane;
                const uint8_t *sc0 = stage_at(uc);
                if (N >= 64) {
                    constexpr int kHalf = kSlabs / 2;  // slabs per K half
#pragma unroll 1
                    for (int j = 0; j < kHalf; ++j) {
                        const int sl = (cb0 >> 1) * kHalf + j;
                        const uint8_t *row = sc0 + sl * kRows * 128 + t * 128;
                        uint32_t cw[32];
#pragma unroll
                        for (int q = 0; q < 8; ++q) {
                            const uint4 v = *reinterpret_cast<const uint4 *>(row + ((q ^ (t & 7)) << 4));
                            cw[4 * q] = v.x;
                            cw[4 * q + 1] = v.y;
                            cw[4 * q + 2] = v.z;
                            cw[4 * q + 3] = v.w;
                        }
                        tmem_st16(tmem + lane_base + c0_col<N>(4 * sl), cw);
                        tmem_st16(tmem + lane_base + c0_col<N>(4 * sl) + 16, cw + 16);
                    }
                } else if (cb0 == 0) {
                    uint32_t cw[8];
#pragma unroll
                    for (int q = 0; q < 2; ++q) {
                        const uint4 v = *reinterpret_cast<const uint4 *>(sc0 + swz_off(t * kRB + q * 16, kRB));
                        cw[4 * q] = v.x;
                        cw[4 * q + 1] = v.y;
                        cw[4 * q + 2] = v.z;
                        cw[4 * q + 3] = v.w;
                    }
                    tmem_st8(tmem + lane_base + c0_col<N>(0), cw);
                }
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(cvt_done);
            // the run's start uses carry no head: their ready phases pass at once
            mbar_arrive(&ready[uc % kStages]);
            mbar_arrive(&ready[(uc + 1) % kStages]);
            if (!mbar_wait(cvt_done, si & 1, err)) break;
            tc_fence_after();
            for (int hi = 0; hi < R.len; ++hi, ++use) {
                const int st = use % kStages;
                const uint32_t sp = (use / kStages) & 1;
                const int h = R.h + hi;
                uint8_t *stage = stage_at(use);
                const float *gb = lg_at(use) + Q;
                if (!mbar_wait(&head_full[st], sp, err)) { ok = false; break; }
                if (sid < ntile && gb[Q + sid] != 0.f) {
                    // steep tile: left to the block-factored scan
                    const int idx = atomicAdd(nsteep, 1);
                    if (idx < max_steep)
                        steep_items[idx] = ((long long)R.b << 40) | ((long long)R.c << 24) |
                                           ((long long)sid << 16) | h;
                }
                // X'' = g o X in place (every row of the chunk) and, for r != 0,
                // S' = e^r s_in, which directly follows x in the stage
                const float r = gb[Q + 2];
                const float er = __expf(r);
                scale_chunks(stage, r != 0.f ? Q * 8 + 8 * N : Q * 8, sid, kScoreThreads,
                             [&](int kc) { return kc < Q * 8 ? gb[kc >> 3] : er; });
                fence_proxy_async_smem();
                mbar_arrive(&ready[st]);
            }
        }
    } else {
        // =============================== epilogue ===============================
        // y_t = u_t Y[t] + (D_h / g_t) X''_t with u_t = exp(l_t - r): the skip term
        // D_h x_t comes from the head's scaled rows (the cumsum kernel flags a
        // tile with a zero dt as steep, so g_t > 0 here).  Per tile, each thread
        // reads its scaled x row, l and g (the stage is released after the last
        // tile's) and its accumulator row in two halves.  Each warp stages
        // its 32 rows and writes them with its own TMA stores, so the warps never
        // wait on one another.
        const int qd = warp & 3;
        const int t_local = qd * 32 + lane;
        const uint32_t lane_base = uint32_t(qd * 32) << 16;
        uint8_t *sYw = sY + qd * 32 * 128;  // two 32 x 32 bf16 blocks per warp
        uint32_t hit = 0, nst = 0, use = 0;
        bool ok = true;
        for (long long i = i0; i < i1 && ok;) {
            const Run R = run_at(i, i1, d);
            i += R.len;
            use += 2;  // the run's start uses: released by the MMA issuer
            for (int hi = 0; hi < R.len && ok; ++hi, ++hit, ++use) {
                const int h = R.h + hi;
                const int ab = hit & 1, st = use % kStages;
                const float Dh = Dskip ? __ldg(Dskip + h) : 0.f;
                if (!mbar_wait(&acc_full[ab], (hit >> 1) & 1, err)) { ok = false; break; }
                tc_fence_after();
                const uint8_t *stage = stage_at(use);
                const float *lb = lg_at(use);
                const float *gb = lb + Q;
#pragma unroll
                for (int k = 0; k < 2; ++k) {
                    if (k == 1 && !two) break;
                    const int t = k * kRows + t_local;
                    // this tile's scaled x row, l and g from the stage; its
                    // accumulator row in two 32-column halves, one wait each
                    const uint8_t *xrow = stage + t * 128;
                    uint4 xr[8];
#pragma unroll
                    for (int q = 0; q < 8; ++q)
                        xr[q] = *reinterpret_cast<const uint4 *>(xrow + ((q ^ (t & 7)) << 4));
                    const float u = __expf(lb[t] - gb[Q + 2]);
                    const bool store = gb[Q + k] == 0.f;
                    const float dg = store ? Dh / gb[t] : 0.f;
                    // the stage goes back to the producer after the last tile's reads
                    if (k == ntile - 1) mbar_arrive(&stage_free[st]);
                    const int row = R.b * d.T + R.c * Q + k * kRows + qd * 32;
#pragma unroll
                    for (int hf = 0; hf < 2; ++hf) {
                        uint32_t a[32];
                        tmem_ld32_nowait(tmem + lane_base + acc_col(ab) + k * 64 + hf * 32, a);
                        tmem_wait_ld();
                        if (k == ntile - 1 && hf == 1) {
                            // the accumulator buffer goes back to the MMAs
                            tc_fence_before();
                            mbar_arrive(&acc_free[ab]);
                        }
                        if (!store) continue;
                        // staged (64-byte swizzle) in one of this warp's two blocks
                        // and written by its own TMA store
                        uint8_t *blk = sYw + (nst & 1) * (32 * 64);
                        // the store that used this block two stores ago has read it
                        if (lane == 0) bulk_wait_read_1();
                        __syncwarp();
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            const uint4 xv = xr[4 * hf + q];
                            const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
                            const uint32_t *ah = a + 8 * q;
                            uint32_t o[4];
#pragma unroll
                            for (int e = 0; e < 4; ++e)
                                o[e] = pack_bf16x2(fmaf(u, __uint_as_float(ah[2 * e]), dg * bf16lo(xw[e])),
                                                   fmaf(u, __uint_as_float(ah[2 * e + 1]), dg * bf16hi(xw[e])));
                            *reinterpret_cast<uint4 *>(blk + sw64_off(lane, q)) = make_uint4(o[0], o[1], o[2], o[3]);
                        }
                        fence_proxy_async_smem();
                        __syncwarp();
                        if (lane == 0) {
                            tma_store_3d(&tm_y, blk, 32 * hf, h, row);
                            bulk_commit();
                        }
                        ++nst;
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
cudaError_t launch5(const Dims &d, const CUtensorMap *maps, const float *gq, const float *D,
                    const float *l, int *nsteep, long long *items, int max_items,
                    unsigned int *err, cudaStream_t stream) {
    const Smem5 L = scan5_smem(d.Q, N);
    if (!smem_attr_once(reinterpret_cast<const void *>(chunk_scan5_kernel<N>), int(L.total)))
        return cudaErrorInvalidValue;
    const long long n_items = (long long)d.B * d.nc * d.H;
    const int sms = device_sm_count();
    const int grid = n_items < sms ? int(n_items) : sms;
    chunk_scan5_kernel<N><<<grid, kThreads, L.total, stream>>>(
        maps[0], maps[1], maps[2], maps[3], maps[4], d, gq, D, l, nsteep, items, max_items, err);
    return cudaGetLastError();
}

}  // namespace

bool tc_chunk_scan5_supported(const Dims &d) {
    // dstate 256: 128-token chunks only (C_0 takes the tensor memory that CBoff
    // would need, and C_1 would not fit in shared memory)
    const bool n_ok = d.N == 16 || d.N == 128 || (d.N == 256 && d.Q == kRows);
    return d.P == 64 && n_ok && (d.Q == 128 || d.Q == 256) &&
           scan5_smem(d.Q, d.N).total <= 227 * 1024 && d.H < 65536 && d.nc < 65536 &&
           d.B < 65536;
}

int chunk_scan5_max_steep(const Dims &d) { return d.B * d.nc * d.H * (d.Q / kRows); }

cudaError_t launch_chunk_scan_tc5(const Dims &d, const void *x, const float *gq, const void *Bm,
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
    const uint32_t ybox[3] = {32, 1, 32};  // 32 columns of one epilogue warp's 32 rows
    CUtensorMap maps[5];
    if (!make_tmap_bf16(&maps[0], 3, Cm, bcdims, bcstr, bcbox, rb) ||
        !make_tmap_bf16(&maps[1], 3, Bm, bcdims, bcstr, bcbox, rb) ||
        !make_tmap_bf16(&maps[2], 3, x, xdims, xstr, xbox, 128) ||
        !make_tmap_bf16(&maps[3], 2, s_in_bf16, sdims, sstr, sbox, rb) ||
        !make_tmap_bf16(&maps[4], 3, y, xdims, xstr, ybox, 64))
        return cudaErrorInvalidValue;
    const int max_items = chunk_scan5_max_steep(d);
    switch (d.N) {
        case 16: return launch5<16>(d, maps, gq, D, l, nsteep, items, max_items, err, stream);
        case 128: return launch5<128>(d, maps, gq, D, l, nsteep, items, max_items, err, stream);
        case 256: return launch5<256>(d, maps, gq, D, l, nsteep, items, max_items, err, stream);
    }
    return cudaErrorInvalidValue;
}

}  // namespace ssd
