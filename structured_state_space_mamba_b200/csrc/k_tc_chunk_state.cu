// k_tc_chunk_state.cu -- ssd_chunk_state on the 5th-generation tensor cores.
//
// For chunk c, batch b and head h (group g):
//     S_c[p, n] = sum_{s in chunk} w_s x_s[p] B_s[n],    w_s = exp(l_last - l_s) dt_s
// (the per-chunk state of the chunked SSD algorithm: aifetchly blog "Mamba-2
// Architecture", "The Chunked SSD Algorithm", step 2, which writes it as
// B_chunk^T X_chunk; the decay weights w and the step dt follow from the
// recurrence h_t = exp(dt_t A) h_{t-1} + dt_t x_t B_t^T unrolled over the chunk).
//
// One work unit = (b, c, a pair of heads of one group): one UMMA
//     D[m, n] = sum_s A[m, s] Bop[s, n],   m = (head j, p) -> M = 128,
//     A = (w o X)^T read MN-major from the x tile [s][p], Bop = B read MN-major
//     from the B tile [s][n], K = Q tokens, D in tensor memory (fp32).
// The kernel is persistent (one CTA per SM walks the units) and warp
// specialised around a ring of 64-token stages:
//     warp 0      TMA producer: x rows of both heads + B rows -> stage
//     warps 2..5  scale each x row by its weight w_s in place (bf16 -> bf16)
//     warp 1      MMA issuer: 4 UMMAs (K = 16 each) per stage into one of two
//                 TMEM accumulators; the commit frees the stage
//     warps 6..9  epilogue: TMEM -> bf16 S_c -> global (overlaps the next unit)
#include "common.cuh"
#include "kernels.h"
#include "tc_common.cuh"
#include "tma_host.h"

namespace ssd {

namespace {

using namespace tc;

constexpr int kThreads = 320;  // 10 warps
constexpr int kKS = 64;        // tokens per stage
// stages in flight: as many 64-token stages as shared memory holds (each TMA
// stage takes ~3 us to land when every SM streams, so a deep ring matters)
__host__ __device__ constexpr int num_stages(int ns) { return ns <= 128 ? 6 : 4; }

__host__ __device__ constexpr int acc_cols(int ns) { return ns < 16 ? 16 : ns; }
__host__ __device__ constexpr int tmem_alloc_cols(int ns) {
    return 2 * acc_cols(ns) <= 32 ? 32 : (2 * acc_cols(ns) <= 64 ? 64 : (2 * acc_cols(ns) <= 128 ? 128 : (2 * acc_cols(ns) <= 256 ? 256 : 512)));
}
__host__ __device__ constexpr int brow_bytes(int ns) { return ns >= 64 ? 128 : ns * 2; }
__host__ __device__ constexpr uint32_t bswz(int ns) { return ns >= 64 ? kSw128 : (ns == 32 ? kSw64 : kSw32); }
__host__ __device__ constexpr uint32_t x_stage_bytes() { return 2 * kKS * 128; }
__host__ __device__ constexpr uint32_t b_stage_bytes(int ns) { return kKS * ns * 2; }
__host__ __device__ constexpr uint32_t w_stage_bytes() { return 2 * kKS * 4; }
__host__ __device__ constexpr uint32_t stage_bytes(int ns) {
    return ((x_stage_bytes() + b_stage_bytes(ns) + w_stage_bytes()) + 1023u) & ~1023u;
}

// Per epilogue warp, two 32 x 32 bf16 staging blocks (64-byte rows) for the
// TMA stores of the chunk states.
constexpr uint32_t kStgWarpBytes = 2 * 32 * 64;
__host__ __device__ constexpr uint32_t stg_off(int ns) { return uint32_t(num_stages(ns)) * stage_bytes(ns) + 1024; }
size_t state_smem_bytes(int NS) { return 1024 + stg_off(NS) + 4 * kStgWarpBytes; }

template <int NS>
__global__ void __launch_bounds__(kThreads, 1)
chunk_state_tc_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_b,
                      const __grid_constant__ CUtensorMap tm_st, Dims d, int nh, int units,
                      const float *__restrict__ w, __nv_bfloat16 *__restrict__ states,
                      unsigned int *err) {
    constexpr int kAcc = acc_cols(NS);
    constexpr int kStages = num_stages(NS);
    constexpr int kCols = tmem_alloc_cols(NS);
    constexpr int kRowB = brow_bytes(NS);
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
            for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
                const int hp = u % nhp, bc = u / nhp;
                const int c = bc % d.nc, b = bc / d.nc;
                const int h0 = hp * nh, g = h0 / d.r;
                const int trow = b * d.T + c * d.Q;
                for (int ks = 0; ks < ksteps; ++ks) {
                    const int s = it % kStages;
                    if (!mbar_wait(&empty[s], ((it / kStages) & 1) ^ 1, err)) { ok = false; break; }
                    uint8_t *sx = smem + s * stage_bytes(NS);
                    uint8_t *sb = sx + x_stage_bytes();
                    mbar_expect_tx(&full[s], uint32_t(nh) * (kKS * 128 + kKS * 4) + b_stage_bytes(NS));
                    float *sw = reinterpret_cast<float *>(sb + b_stage_bytes(NS));
                    for (int j = 0; j < nh; ++j)
                        bulk_load(sw + j * kKS, w + off_lq(d, b, h0 + j, c) + ks * kKS, kKS * 4, &full[s]);
                    for (int j = 0; j < nh; ++j)
                        tma_load_3d(sx + j * kKS * 128, &tm_x, &full[s], 0, h0 + j, trow + ks * kKS);
                    if (NS >= 64) {
                        for (int sl = 0; sl < NS / 64; ++sl)
                            tma_load_3d(sb + sl * kKS * 128, &tm_b, &full[s], sl * 64, g, trow + ks * kKS);
                    } else {
                        tma_load_3d(sb, &tm_b, &full[s], 0, g, trow + ks * kKS);
                    }
                    ++it;
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
            uint32_t it = 0, ui = 0;
            bool ok = true;
            for (int u = blockIdx.x; u < units && ok; u += gridDim.x, ++ui) {
                const int a = ui & 1;
                if (!mbar_wait(&acce[a], ((ui >> 1) & 1) ^ 1, err)) break;
                tc_fence_after();
                const uint32_t dacc = tmem + a * kAcc;
                for (int ks = 0; ks < ksteps; ++ks) {
                    const int s = it % kStages;
                    if (!mbar_wait(&scaled[s], (it / kStages) & 1, err)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t xa = smem_u32(smem + s * stage_bytes(NS));
                    const uint32_t ba = xa + x_stage_bytes();
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
        for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
            for (int ks = 0; ks < ksteps; ++ks) {
                const int s = it % kStages;
                if (!mbar_wait(&full[s], (it / kStages) & 1, err)) { ok = false; break; }
                uint8_t *sx = smem + s * stage_bytes(NS);
                const float *sw = reinterpret_cast<const float *>(sx + x_stage_bytes() + b_stage_bytes(NS));
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
    } else {
        // ------------------------------ epilogue ----------------------------------
        // Warp qd owns TMEM rows m = 32 qd + lane = (head j = qd / 2, p).  For
        // N >= 32 each 32 x 32 block goes out as bf16 through a swizzled staging
        // block and one 2-D TMA store (coalesced, and off the load/store unit
        // that the scale warps use); N = 16 rows are stored directly.
        const int qd = warp & 3;
        const int m = qd * 32 + lane;
        const int j = m >> 6, p = m & 63;
        const bool valid = j < nh;  // warp-uniform
        uint8_t *stg = smem + stg_off(NS) + qd * kStgWarpBytes;
        uint32_t ui = 0, nst = 0;
        for (int u = blockIdx.x; u < units; u += gridDim.x, ++ui) {
            const int a = ui & 1;
            if (!mbar_wait(&accf[a], (ui >> 1) & 1, err)) break;
            tc_fence_after();
            const int hp = u % nhp, bc = u / nhp;
            const int c = bc % d.nc, b = bc / d.nc;
            const int h = hp * nh + (valid ? j : 0);
            const uint32_t taddr = tmem + (uint32_t(qd * 32) << 16) + a * kAcc;
            if (NS >= 32) {
                const int row0 = ((b * d.nc + c) * d.H + h) * 64 + (qd & 1) * 32;
#pragma unroll 1
                for (int n0 = 0; n0 < NS; n0 += 32, ++nst) {
                    float v[32];
                    tmem_ld32(taddr + n0, v);
                    if (valid) {
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
                            tma_store_2d(&tm_st, blk, n0, row0);
                            bulk_commit();
                        }
                    }
                }
            } else {
                float v[16];
                tmem_ld16(taddr, v);
                if (valid) {
                    uint4 *o = reinterpret_cast<uint4 *>(states + off_state(d, b, c, h) + int64_t(p) * NS);
#pragma unroll
                    for (int q = 0; q < 2; ++q)
                        o[q] = make_uint4(pack_bf16x2(v[8 * q], v[8 * q + 1]), pack_bf16x2(v[8 * q + 2], v[8 * q + 3]),
                                          pack_bf16x2(v[8 * q + 4], v[8 * q + 5]), pack_bf16x2(v[8 * q + 6], v[8 * q + 7]));
                }
            }
            tc_fence_before();
            mbar_arrive(&acce[a]);
        }
        if (lane == 0) bulk_wait_all();
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) tmem_dealloc(tmem, kCols);
}

template <int NS>
cudaError_t launch_ns(const Dims &d, const CUtensorMap &tx, const CUtensorMap &tb,
                      const CUtensorMap &tst, int nh,
                      const float *w, __nv_bfloat16 *states, unsigned int *err, cudaStream_t stream) {
    const size_t smem = state_smem_bytes(NS);
    if (!smem_attr_once(reinterpret_cast<const void *>(chunk_state_tc_kernel<NS>), int(smem)))
        return cudaErrorInvalidValue;
    const int units = d.B * d.nc * (d.H / nh);
    const int grid = units < device_sm_count() ? units : device_sm_count();
    chunk_state_tc_kernel<NS><<<grid, kThreads, smem, stream>>>(tx, tb, tst, d, nh, units, w, states, err);
    return cudaGetLastError();
}

}  // namespace

bool tc_chunk_state_supported(const Dims &d) {
    const bool ns_ok = d.N == 16 || d.N == 32 || d.N == 64 || d.N == 128 || d.N == 256;
    return d.P == 64 && ns_ok && (d.Q == 64 || d.Q == 128 || d.Q == 256) &&
           state_smem_bytes(d.N) <= 227 * 1024 && int64_t(d.B) * d.nc * d.H < (int64_t(1) << 31);
}

cudaError_t launch_chunk_state_tc(const Dims &d, const void *x, const void *Bm, const float *w,
                                  void *states_bf16, unsigned int *err, cudaStream_t stream) {
    // x viewed as [B*T rows][H][P]; box = one head, 64 tokens
    const uint64_t xdims[3] = {uint64_t(d.P), uint64_t(d.H), uint64_t(d.B) * d.T};
    const uint64_t xstr[2] = {uint64_t(d.P) * 2, uint64_t(d.H) * d.P * 2};
    const uint32_t xbox[3] = {64, 1, uint32_t(kKS)};
    // B viewed as [B*T rows][G][N]; box = one group, 64 tokens, a 64-wide slab of N
    const uint64_t bdims[3] = {uint64_t(d.N), uint64_t(d.G), uint64_t(d.B) * d.T};
    const uint64_t bstr[2] = {uint64_t(d.N) * 2, uint64_t(d.G) * d.N * 2};
    const uint32_t bbox[3] = {uint32_t(d.N >= 64 ? 64 : d.N), 1, uint32_t(kKS)};
    // states viewed as [B*nc*H*P rows][N]; box = 32 columns x 32 rows
    const uint64_t sdims[2] = {uint64_t(d.N), uint64_t(d.B) * d.nc * d.H * d.P};
    const uint64_t sstr[1] = {uint64_t(d.N) * 2};
    const uint32_t sbox[2] = {32, 32};
    CUtensorMap tx, tb, tst{};
    if (!make_tmap_bf16(&tx, 3, x, xdims, xstr, xbox, 128) ||
        !make_tmap_bf16(&tb, 3, Bm, bdims, bstr, bbox, brow_bytes(d.N)) ||
        (d.N >= 32 && !make_tmap_bf16(&tst, 2, states_bf16, sdims, sstr, sbox, 64)))
        return cudaErrorInvalidValue;
    const int nh = (d.r % 2 == 0) ? 2 : 1;
    auto *st = static_cast<__nv_bfloat16 *>(states_bf16);
    switch (d.N) {
        case 16: return launch_ns<16>(d, tx, tb, tst, nh, w, st, err, stream);
        case 32: return launch_ns<32>(d, tx, tb, tst, nh, w, st, err, stream);
        case 64: return launch_ns<64>(d, tx, tb, tst, nh, w, st, err, stream);
        case 128: return launch_ns<128>(d, tx, tb, tst, nh, w, st, err, stream);
        case 256: return launch_ns<256>(d, tx, tb, tst, nh, w, st, err, stream);
    }
    return cudaErrorInvalidValue;
}

}  // namespace ssd
