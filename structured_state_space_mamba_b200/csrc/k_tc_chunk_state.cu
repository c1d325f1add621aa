// k_tc_chunk_state.cu -- ssd_chunk_state on the 5th-generation tensor cores.
//
// For chunk c, batch b and head h (group g):
//     S_c[p, n] = sum_{s in chunk} w_s x_s[p] B_s[n],    w_s = exp(l_last - l_s) dt_s
// (the per-chunk state of the chunked SSD algorithm: aifetchly blog "Mamba-2
// Architecture", "The Chunked SSD Algorithm", step 2, which writes it as
// B_chunk^T X_chunk; the decay weights w and the step dt follow from the
// recurrence h_t = exp(dt_t A) h_{t-1} + dt_t x_t B_t^T unrolled over the chunk).
//
// As one UMMA per CTA: D[m, n] = sum_s A[m, s] Bop[s, n] with
//   m = (head j, p): two heads of the same group stacked -> M = 128,
//   A   = (w o X)^T  read MN-major from the x tile [s][p] (TMA, 128B swizzle),
//   Bop = B          read MN-major from the B tile [s][n] (TMA),
//   K   = Q tokens, D (fp32) in tensor memory, N = dstate columns.
// The weights are applied in shared memory (bf16 round trip) between the TMA
// load and the MMA.  One thread issues the MMAs; four warps drain TMEM.
#include "common.cuh"
#include "kernels.h"
#include "tc_common.cuh"
#include "tma_host.h"

namespace ssd {

namespace {

using namespace tc;

constexpr int kThreads = 128;

__host__ __device__ constexpr int tmem_cols_for(int n) { return n <= 32 ? 32 : (n <= 64 ? 64 : (n <= 128 ? 128 : 256)); }
__host__ __device__ constexpr int brow_bytes(int ns) { return ns >= 64 ? 128 : ns * 2; }
__host__ __device__ constexpr uint32_t bswz(int ns) { return ns >= 64 ? kSw128 : (ns == 32 ? kSw64 : kSw32); }

size_t state_smem_bytes(int Q, int NS) {
    return 1024 /*align slack*/ + size_t(2) * Q * 128 + size_t(Q) * NS * 2 + size_t(2) * Q * 4 + 64;
}

template <int NS>
__global__ void __launch_bounds__(kThreads, 1)
chunk_state_tc_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_b,
                      Dims d, int nh, const float *__restrict__ w, float *__restrict__ states,
                      unsigned int *err) {
    constexpr int kCols = tmem_cols_for(NS);
    constexpr int kRowB = brow_bytes(NS);
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int Q = d.Q;
    uint8_t *sX = smem;                           // [2][Q][64] bf16, 128B rows, swizzled
    uint8_t *sB = smem + 2 * Q * 128;             // [NS/64][Q][64] (or [Q][NS]) bf16, swizzled
    float *sW = reinterpret_cast<float *>(sB + Q * NS * 2);  // [2][Q]
    uint64_t *bars = reinterpret_cast<uint64_t *>(sW + 2 * Q);
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(bars + 2);
    __shared__ int s_abort;

    const int c = blockIdx.x, b = blockIdx.z;
    const int h0 = blockIdx.y * nh;
    const int g = h0 / d.r;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int trow = b * d.T + c * Q;  // first token row in the [B*T] view

    if (device_failed(err)) return;  // an earlier wait expired: skip all work
    if (tid == 0) {
        s_abort = 0;
        mbar_init(&bars[0], 1);
        mbar_init(&bars[1], 1);
        fence_mbar_init();
        tma_prefetch_desc(&tm_x);
        tma_prefetch_desc(&tm_b);
    }
    if (warp == 0) tmem_alloc(tmem_holder, kCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;

    if (tid == 0) {
        const uint32_t bytes = uint32_t(nh) * Q * 128 + uint32_t(Q) * NS * 2;
        mbar_expect_tx(&bars[0], bytes);
        for (int j = 0; j < nh; ++j) tma_load_3d(sX + j * Q * 128, &tm_x, &bars[0], 0, h0 + j, trow);
        if (NS >= 64) {
            for (int s = 0; s < NS / 64; ++s) tma_load_3d(sB + s * Q * 128, &tm_b, &bars[0], s * 64, g, trow);
        } else {
            tma_load_3d(sB, &tm_b, &bars[0], 0, g, trow);
        }
    }
    for (int i = tid; i < nh * Q; i += kThreads) sW[i] = __ldg(w + off_lq(d, b, h0 + i / Q, c) + i % Q);
    if (nh == 1)
        for (int i = tid; i < Q * 8; i += kThreads)
            reinterpret_cast<uint4 *>(sX + Q * 128)[i] = make_uint4(0u, 0u, 0u, 0u);
    __syncthreads();

    if (!mbar_wait(&bars[0], 0, err)) s_abort = 1;
    // x <- bf16(w_s * x_s): the swizzle permutes 16-byte chunks within a
    // 128-byte row, so every chunk of row (j, s) takes the same weight.
    for (int i = tid; i < nh * Q * 8; i += kThreads) {
        uint4 *p = reinterpret_cast<uint4 *>(sX) + i;
        const float wv = sW[i >> 3];
        uint4 v = *p;
        v.x = pack_bf16x2(bf16lo(v.x) * wv, bf16hi(v.x) * wv);
        v.y = pack_bf16x2(bf16lo(v.y) * wv, bf16hi(v.y) * wv);
        v.z = pack_bf16x2(bf16lo(v.z) * wv, bf16hi(v.z) * wv);
        v.w = pack_bf16x2(bf16lo(v.w) * wv, bf16hi(v.w) * wv);
        *p = v;
    }
    fence_proxy_async_smem();
    __syncthreads();
    const bool go = s_abort == 0;

    if (tid == 0 && go) {
        tc_fence_after();
        constexpr uint32_t idesc = idesc_bf16_f32(128, NS, 1, 1);
        const uint32_t xa = smem_u32(sX), ba = smem_u32(sB);
        for (int k = 0; k < Q / 16; ++k) {
            const uint64_t ad = smem_desc(xa + k * 16 * 128, Q * 128, 1024, kSw128);
            const uint64_t bd = smem_desc(ba + k * 16 * kRowB, Q * 128, 8 * kRowB, bswz(NS));
            mma_bf16_ss(tmem, ad, bd, idesc, k > 0 ? 1u : 0u);
        }
        mma_commit(&bars[1]);
    }
    __syncthreads();
    if (go && !mbar_wait(&bars[1], 0, err)) s_abort = 1;
    tc_fence_after();
    __syncthreads();

    // epilogue: TMEM lane m = 32*warp + lane holds row (head m/64, p = m%64)
    const int m = warp * 32 + lane;
    const int j = m >> 6, p = m & 63;
    if (s_abort == 0) {
        const uint32_t taddr = tmem + (uint32_t(warp * 32) << 16);
        float *dst = states + off_state(d, b, c, h0 + (j < nh ? j : 0)) + int64_t(p) * NS;
        if (NS >= 32) {
#pragma unroll 1
            for (int n0 = 0; n0 < NS; n0 += 32) {
                float v[32];
                tmem_ld32(taddr + n0, v);
                if (j < nh) {
#pragma unroll
                    for (int q = 0; q < 8; ++q)
                        reinterpret_cast<float4 *>(dst + n0)[q] =
                            make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
                }
            }
        } else {
            float v[16];
            tmem_ld16(taddr, v);
            if (j < nh) {
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    reinterpret_cast<float4 *>(dst)[q] =
                        make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
            }
        }
    }
    // on an abandoned wait, give the copies in flight a bounded chance to land
    if (tid == 0 && s_abort) mbar_wait(&bars[0], 0, nullptr);
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, kCols);
}

template <int NS>
cudaError_t launch_ns(const Dims &d, const CUtensorMap &tx, const CUtensorMap &tb, int nh,
                      const float *w, float *states, unsigned int *err, cudaStream_t stream) {
    const size_t smem = state_smem_bytes(d.Q, NS);
    if (cudaFuncSetAttribute(chunk_state_tc_kernel<NS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             int(smem)) != cudaSuccess)
        return cudaGetLastError();
    dim3 grid(d.nc, d.H / nh, d.B);
    chunk_state_tc_kernel<NS><<<grid, kThreads, smem, stream>>>(tx, tb, d, nh, w, states, err);
    return cudaGetLastError();
}

}  // namespace

bool tc_chunk_state_supported(const Dims &d) {
    const bool ns_ok = d.N == 16 || d.N == 32 || d.N == 64 || d.N == 128 || d.N == 256;
    return d.P == 64 && ns_ok && (d.Q == 64 || d.Q == 128 || d.Q == 256) &&
           state_smem_bytes(d.Q, d.N) <= 227 * 1024;
}

cudaError_t launch_chunk_state_tc(const Dims &d, const void *x, const void *Bm, const float *w,
                                  float *states, unsigned int *err, cudaStream_t stream) {
    // x viewed as [B*T rows][H][P]; box = one head, Q tokens
    const uint64_t xdims[3] = {uint64_t(d.P), uint64_t(d.H), uint64_t(d.B) * d.T};
    const uint64_t xstr[2] = {uint64_t(d.P) * 2, uint64_t(d.H) * d.P * 2};
    const uint32_t xbox[3] = {64, 1, uint32_t(d.Q)};
    // B viewed as [B*T rows][G][N]; box = one group, Q tokens, a 64-wide slab of N
    const uint64_t bdims[3] = {uint64_t(d.N), uint64_t(d.G), uint64_t(d.B) * d.T};
    const uint64_t bstr[2] = {uint64_t(d.N) * 2, uint64_t(d.G) * d.N * 2};
    const uint32_t bbox[3] = {uint32_t(d.N >= 64 ? 64 : d.N), 1, uint32_t(d.Q)};
    CUtensorMap tx, tb;
    if (!make_tmap_bf16(&tx, 3, x, xdims, xstr, xbox, 128) ||
        !make_tmap_bf16(&tb, 3, Bm, bdims, bstr, bbox, brow_bytes(d.N)))
        return cudaErrorInvalidValue;
    const int nh = (d.r % 2 == 0) ? 2 : 1;
    switch (d.N) {
        case 16: return launch_ns<16>(d, tx, tb, nh, w, states, err, stream);
        case 32: return launch_ns<32>(d, tx, tb, nh, w, states, err, stream);
        case 64: return launch_ns<64>(d, tx, tb, nh, w, states, err, stream);
        case 128: return launch_ns<128>(d, tx, tb, nh, w, states, err, stream);
        case 256: return launch_ns<256>(d, tx, tb, nh, w, states, err, stream);
    }
    return cudaErrorInvalidValue;
}

}  // namespace ssd
