// ssd_api.cu -- the C ABI of libssd.so (declared in include/ssd.h).
//
// Argument validation, workspace layout and the launch sequence
//   ssd_chunk_cumsum -> ssd_chunk_state -> ssd_state_passing -> ssd_chunk_scan
// of the chunked SSD algorithm (aifetchly blog "Mamba-2 Architecture: State
// Space Duality Explained", "The Chunked SSD Algorithm").  Every error is
// detected before the first launch.
#include <cuda_runtime.h>

#include <cstdlib>
#include <cstring>
#include <mutex>

#include "../../include/ssd.h"
#include "common.cuh"
#include "kernels.h"

// Device word set by tensor-core kernels whose bounded waits expired.
__device__ unsigned int g_ssd_device_error;

namespace {

using ssd::Dims;

constexpr int kMaxDevices = 64;
unsigned int *g_err_ptr[kMaxDevices];  // per-device address of g_ssd_device_error
std::once_flag g_err_once[kMaxDevices];

// Address of the error word on the current device (NULL if unavailable).
unsigned int *device_error_word() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        cudaGetLastError();
        return nullptr;
    }
    std::call_once(g_err_once[dev], [dev] {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_ssd_device_error) == cudaSuccess)
            g_err_ptr[dev] = static_cast<unsigned int *>(p);
        else
            cudaGetLastError();
    });
    return g_err_ptr[dev];
}

// Workspace memory of the entry points that allocate their own: a stream-
// ordered pool per device, private to the library, that keeps what it has
// reserved between calls (release threshold unlimited), so a repeated call
// reuses its memory instead of mapping it again at every synchronisation
// (the default pool returns it; for the backward's 3 GB on the 2.7B-shaped
// layer that mapping cost about a third of the call).  ssd_workspace_trim
// returns the unused part.  Falls back to the device's default pool.
cudaMemPool_t g_pool[kMaxDevices];
std::once_flag g_pool_once[kMaxDevices];

cudaMemPool_t workspace_pool(int dev) {
    std::call_once(g_pool_once[dev], [dev] {
        cudaMemPoolProps props;
        std::memset(&props, 0, sizeof(props));
        props.allocType = cudaMemAllocationTypePinned;
        props.handleTypes = cudaMemHandleTypeNone;
        props.location.type = cudaMemLocationTypeDevice;
        props.location.id = dev;
        cudaMemPool_t pool = nullptr;
        if (cudaMemPoolCreate(&pool, &props) != cudaSuccess) {
            cudaGetLastError();
            return;
        }
        uint64_t keep = ~uint64_t(0);
        if (cudaMemPoolSetAttribute(pool, cudaMemPoolAttrReleaseThreshold, &keep) != cudaSuccess)
            cudaGetLastError();
        g_pool[dev] = pool;
    });
    return g_pool[dev];
}

cudaError_t workspace_alloc(void **p, size_t bytes, cudaStream_t st) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        cudaGetLastError();
        return cudaErrorInvalidDevice;
    }
    cudaMemPool_t pool = workspace_pool(dev);
    return pool ? cudaMallocFromPoolAsync(p, bytes, pool, st) : cudaMallocAsync(p, bytes, st);
}

constexpr size_t kAlign = 256;
// the backward's per-row kernels keep one factor per head in shared memory
constexpr int64_t kMaxBackwardHeads = 12288;
// chunk length of the backward's two fp32 CUDA-core scans (K and h).  Their
// results do not depend on it beyond rounding; 64-token chunks shorten the
// quadratic in-chunk products (about 2x fewer FMAs per token than 256) for 4x
// the chunk states: 9.4 ms against 10.6 ms per call on the 2.7B-shaped layer.
constexpr int kBackwardScanChunk = 64;

size_t align_up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }

bool misaligned(const void *p) { return p && (reinterpret_cast<uintptr_t>(p) & 15u); }

constexpr int kB200Sms = 148;
constexpr int kMinChainNum = 2, kMinChainDen = 5;  // single-pass kernel: chains >= 40% of SMs

struct Plan {
    Dims d;
    bool bf16;
    bool tc_state;  // tcgen05 chunk state
    bool tc_scan;   // tcgen05 chunk scan (consumes bf16 s_in)
    bool fused;     // chunk_state + state_passing in one kernel (no states buffer)
    bool scan5;     // chunk-wide scan, steep tiles finished by the block-factored scan
    bool single;    // the single-pass kernel (chunk state + state passing + scan)
    bool presolved; // single pass whose ranges start from states computed by two passes before it
    int G = 0;      // presolved: CTAs of the single pass (and of its range-state pass)
    bool tile_finish;  // scan5's steep tiles go to the per-tile scan (no block-factored plan)
    int t_full = 0;       // tokens in full chunks; the tail [t_full, T) runs in the tail kernel
    size_t mid_offset = 0;  // tail: fp32 state after the full chunks [B,H,P,N]
    size_t steep_offset;  // scan5 / single: item counter (256 bytes) + packed steep items
    size_t gq_offset;     // scan5 / single: per-token column factors [B,H,nc,chunk_gq(Q)]
    size_t chain_offset;  // single: per-(b, h) fp32 state slots [B,H,P,N]
    size_t flag_offset;   // single: per-(b, head pair) chain flags [B, H/2]
    size_t seg_offset;    // presolved: partial end states of the ranges [G][128][N] fp32
    size_t start_offset;  // presolved: states entering the ranges [G][128][N] fp32
    ssd_workspace_layout_t ws;
};

// The single-pass kernel applies in one of two forms.
//  * Hand-off: (batch, head pair) chains for at least kMinChainNum /
//    kMinChainDen of the SMs; a CTA takes at most one chain's worth of chunks
//    and hands a state to the next CTA at most once.
//  * Presolved (fewer chains): the ranges of a full grid start from states that
//    two passes compute first (one more pass over x and B).  Measured on B200:
//    it pays off when the ranges are long (16 chunks or more each: the long
//    grouped layer, 0.383 -> 0.350 ms) or when the alternative is the
//    block-factored scan (dstate 64: the sweep shape 0.108 -> 0.098 ms); with
//    short ranges at dstate 128 the per-range pipeline refill and the extra
//    pass lose to the four-kernel sequence (0.101 against 0.120 ms).
bool single_pass_supported(const Dims &d) {
    return ssd::tc_chunk_scan_supported(d) && ssd::tc_chunk_scan4_supported(d) && ssd::tc_chunk_fused_supported(d);
}
bool handoff_applies(const Dims &d) {
    return single_pass_supported(d) && int64_t(d.B) * (d.H / 2) * kMinChainDen >= int64_t(kB200Sms) * kMinChainNum;
}
bool presolved_applies(const Dims &d) {
    const long long chains = (long long)d.B * (d.H / 2);
    return single_pass_supported(d) && !handoff_applies(d) && ssd::presolved_ranges_supported(d) &&
           (d.N == 64 || chains * d.nc >= 16ll * kB200Sms);
}
bool single_pass_applies(const Dims &d) { return handoff_applies(d) || presolved_applies(d); }

ssd_status_t make_plan(const ssd_dims_t *dims, int chunk_len, Plan *plan) {
    if (!dims || !plan) return SSD_ERR_NULL_ARG;
    const ssd_dims_t &a = *dims;
    if (a.batch <= 0 || a.seqlen <= 0 || a.nheads <= 0 || a.headdim <= 0 || a.dstate <= 0 ||
        a.ngroups <= 0 || a.reserved != 0)
        return SSD_ERR_INVALID_DIM;
    if (a.dtype != SSD_F32 && a.dtype != SSD_BF16) return SSD_ERR_UNSUPPORTED;
    if (a.nheads % a.ngroups != 0) return SSD_ERR_INVALID_DIM;
    if (chunk_len != 32 && chunk_len != 64 && chunk_len != 128 && chunk_len != 256)
        return SSD_ERR_UNSUPPORTED;
    if (a.headdim > 256 || a.dstate > 256) return SSD_ERR_UNSUPPORTED;
    if (a.dtype == SSD_BF16 && (a.headdim % 8 != 0 || a.dstate % 8 != 0)) return SSD_ERR_UNSUPPORTED;
    // grid limits (blockIdx.y / .z <= 65535) and 32-bit token indices
    const int64_t nc = a.seqlen / chunk_len;
    if (a.seqlen > (int64_t(1) << 30) || nc > 65535 || a.batch * a.nheads > 65535 ||
        a.batch > 65535 || a.nheads > 65535)
        return SSD_ERR_UNSUPPORTED;

    Dims d;
    d.B = int(a.batch); d.T = int(a.seqlen); d.H = int(a.nheads); d.P = int(a.headdim);
    d.N = int(a.dstate); d.G = int(a.ngroups); d.Q = chunk_len; d.nc = int(nc);
    d.r = d.H / d.G;
    // chunk_len 64 on the tensor cores: their tile is 128 rows (the full TMEM
    // lane range of a one-CTA MMA), so the chunked algorithm runs with 128-token
    // chunks -- two of the caller's chunks per tile, whose hand-off then happens
    // inside the tile's masked product.  The result is the same recurrence (the
    // chunk length only sets the blocking); the workspace arrays then describe
    // 128-token chunks.
    if (a.dtype == SSD_BF16 && d.Q == 64 && d.T % 128 == 0) {
        Dims d2 = d;
        d2.Q = 128;
        d2.nc = d.T / 128;
        if (ssd::tc_chunk_state_supported(d2) && ssd::tc_chunk_scan_supported(d2)) d = d2;
    }
    // dstate 256: the chunk-wide tensor-core scan holds one 128-token tile of C
    // (C_0 in tensor memory) but not a second, so the chunks are 128 tokens
    // (the same recurrence, blocked differently; the workspace arrays then
    // describe 128-token chunks), unless that lengthens the ragged tail
    if (a.dtype == SSD_BF16 && d.N == 256 && d.Q != 128 && d.T % 128 <= d.T % chunk_len && d.T / 128 <= 65535) {
        Dims d2 = d;
        d2.Q = 128;
        d2.nc = d.T / 128;
        if (ssd::tc_chunk_state_supported(d2) && ssd::tc_chunk_scan_supported(d2) &&
            ssd::tc_chunk_scan5_supported(d2))
            d = d2;
    }
    // chunk_len 32 / 64 / 128 on the four-kernel tensor-core path or the
    // presolved single pass: 256-token chunks halve the chunk states the
    // four-kernel path writes and reads back (S and s_in; on the dstate-128
    // sweep shape 0.127 -> 0.102 ms per call) and the presolved ranges' chunk
    // count.  Not where the hand-off single pass applies (it keeps its
    // length), for dstate 256 (above), or when the tail kernel would get more
    // tokens (T mod 256 > T mod chunk_len).
    if (a.dtype == SSD_BF16 && d.Q < 256 && d.N != 256 && d.T % 256 <= d.T % chunk_len && !handoff_applies(d)) {
        Dims d2 = d;
        d2.Q = 256;
        d2.nc = d.T / 256;
        if (ssd::tc_chunk_state_supported(d2) && ssd::tc_chunk_scan_supported(d2) && !handoff_applies(d2))
            d = d2;
    }
    // a length that is not a multiple of chunk_len: the chunked kernels take the
    // full chunks (they index rows with the true T), the tail kernel the rest
    plan->t_full = d.nc * d.Q;
    if (plan->t_full < d.T && !ssd::tail_supported(d)) return SSD_ERR_UNSUPPORTED;
    plan->d = d;
    plan->bf16 = a.dtype == SSD_BF16;
    plan->tc_state = plan->bf16 && ssd::tc_chunk_state_supported(d);
    plan->tc_scan = plan->bf16 && ssd::tc_chunk_scan_supported(d);
    // the fused state kernel walks each (b, head pair) over all chunks: used when
    // those units fill most of the GPU's 148 SMs in one wave
    plan->fused = plan->tc_state && plan->tc_scan && ssd::tc_state_fused_supported(d, kB200Sms);
    // the chunk-wide scan leaves steep tiles to the block-factored scan, or (no
    // shared-memory plan there: dstate 256) to the per-tile scan, whose scores
    // take every decay exactly
    plan->scan5 = plan->tc_scan && ssd::tc_chunk_scan5_supported(d);
    plan->tile_finish = plan->scan5 && !ssd::tc_chunk_scan4_supported(d);
    // the single-pass kernel walks each (b, head pair) chain chunk by chunk; the
    // tiles it lists as steep go to the block-factored scan
    plan->single = plan->bf16 && single_pass_applies(d);
    plan->presolved = plan->single && presolved_applies(d);
    if (plan->presolved) {
        const long long items = (long long)d.B * (d.H / 2) * d.nc;
        plan->G = int(items < kB200Sms ? items : kB200Sms);
        // a whole number of CTAs per chain when that keeps 95 % of the SMs: every
        // chain is then cut at the same chunks, so the head pairs of one group
        // read each chunk's B and C at about the same time and the second read
        // hits L2 (long grouped layer, 16 chains on 144 CTAs: 337 -> 314 us)
        const long long chains = (long long)d.B * (d.H / 2);
        const long long aligned = chains * (kB200Sms / chains);
        if (chains <= kB200Sms && aligned * 100 >= 95ll * kB200Sms && aligned <= items) plan->G = int(aligned);
    }
    if (plan->single) plan->fused = false;

    ssd_workspace_layout_t &w = plan->ws;
    std::memset(&w, 0, sizeof(w));
    const size_t lq = size_t(d.B) * d.H * d.nc * d.Q * sizeof(float);
    const size_t al = size_t(d.B) * d.H * d.nc * sizeof(float);
    const size_t st = size_t(d.B) * d.nc * d.H * d.P * d.N;
    size_t off = 0;
    w.l_offset = off; off = align_up(off + lq);
    w.w_offset = off; off = align_up(off + lq);
    w.dtq_offset = off; off = align_up(off + lq);
    w.beta_offset = off; off = align_up(off + lq);
    w.alpha_offset = off; off = align_up(off + al);
    w.states_offset = off;
    w.states_dtype = plan->tc_state ? SSD_BF16 : SSD_F32;
    if (!plan->fused && !plan->single) off = align_up(off + st * (plan->tc_state ? 2 : 4));
    w.s_in_offset = off;
    w.s_in_dtype = plan->tc_scan ? SSD_BF16 : SSD_F32;
    off = align_up(off + st * (plan->tc_scan ? 2 : 4));
    plan->steep_offset = off;
    const bool lists = plan->scan5 || plan->single;  // per-token factors and a steep-tile list
    if (lists) off = align_up(off + kAlign + sizeof(long long) * size_t(ssd::chunk_scan5_max_steep(d)));
    plan->gq_offset = off;
    if (lists) off = align_up(off + al * ssd::chunk_gq(d.Q));
    plan->chain_offset = off;
    if (plan->single) off = align_up(off + ssd::chunk_fused_chain_bytes(d));
    plan->flag_offset = off;
    if (plan->single) off = align_up(off + ssd::chunk_fused_flag_bytes(d));
    plan->seg_offset = off;
    if (plan->presolved) off = align_up(off + ssd::presolved_state_bytes(plan->G, d));
    plan->start_offset = off;
    if (plan->presolved) off = align_up(off + ssd::presolved_state_bytes(plan->G, d));
    plan->mid_offset = off;
    if (plan->t_full < d.T) off = align_up(off + size_t(d.B) * d.H * d.P * d.N * sizeof(float));
    w.total_bytes = off;
    w.tensor_core = (plan->tc_state || plan->tc_scan) ? 1 : 0;
    w.launches = d.nc == 0 ? 0
                 : plan->presolved ? 5
                 : plan->single ? 3 : (plan->fused ? 3 : 4) + (plan->scan5 ? 1 : 0);
    if (plan->t_full < d.T) w.launches += 1;
    w.fused_state = plan->fused ? 1 : 0;
    w.single_pass = plan->single ? 1 : 0;
    w.chunk_len = d.Q;
    w.scan_engine = plan->single ? SSD_ENGINE_SINGLE_PASS
                    : plan->scan5 ? SSD_ENGINE_CHUNK_WIDE
                    : plan->tc_scan ? (ssd::tc_chunk_scan4_supported(d) ? SSD_ENGINE_BLOCK_FACTORED
                                                                        : SSD_ENGINE_TILE)
                                    : SSD_ENGINE_SIMT;
    return SSD_OK;
}

ssd_status_t check_tensors(const Plan &pl, const void *x, const float *dt, const float *A,
                           const void *Bm, const void *Cm, const float *D,
                           const float *init_state, const void *y, const float *fin) {
    if (!x || !dt || !A || !Bm || !Cm || !y) return SSD_ERR_NULL_ARG;
    const void *ptrs[] = {x, dt, A, Bm, Cm, D, init_state, y, fin};
    for (const void *p : ptrs)
        if (misaligned(p)) return SSD_ERR_MISALIGNED;
    (void)pl;
    return SSD_OK;
}

bool inject_launch_failure() {
    // Host-side fault injection for tests of the error path: with
    // SSD_FAULT_INJECT=launch the call fails as a launch failure would,
    // before anything is launched.
    const char *v = std::getenv("SSD_FAULT_INJECT");
    return v && std::strcmp(v, "launch") == 0;
}

// The block neighbours of one call (ssd_forward_block); all off for the plain
// entry points.
struct Neighbours {
    const float *dt_bias = nullptr;
    int softplus = 0;
    const void *z = nullptr;
    const float *norm_w = nullptr;
    float eps = 0.f;
    bool apply = false;
    float *rstd = nullptr;
    float *dt_eff = nullptr;  // workspace copy of the transformed dt, dt's layout
    bool transform() const { return dt_bias || softplus; }
    bool output() const { return z || norm_w; }
};

ssd_status_t run(const Plan &pl, const void *x, const float *dt, const float *A, const void *Bm,
                 const void *Cm, const float *D, const float *init_state, void *y,
                 float *fin, char *ws, cudaStream_t stream, int only_stage = -1,
                 const Neighbours *nb = nullptr) {
    if (inject_launch_failure()) return SSD_ERR_CUDA;
    const Dims &d = pl.d;
    const Neighbours none;
    if (!nb) nb = &none;
    // with a tail, the full chunks' final state goes to the workspace and the
    // tail kernel continues from it
    const bool tail = pl.t_full < d.T;
    float *fin_user = fin;
    float *mid = tail ? reinterpret_cast<float *>(ws + pl.mid_offset) : nullptr;
    if (tail) fin = mid;
    // after the scan: the tail tokens (recurrence from the full chunks' state),
    // then the block's gate and norm over every token
    auto finish_scan = [&]() -> cudaError_t {
        cudaError_t e2 = cudaSuccess;
        if (tail)
            e2 = ssd::launch_tail(d, pl.bf16, pl.t_full, x, dt, nb->dt_bias, nb->softplus, A, Bm, Cm, D,
                                  d.nc > 0 ? mid : init_state, y, fin_user, stream);
        if (e2 == cudaSuccess && nb->output())
            e2 = ssd::launch_gate_norm(d, pl.bf16, y, nb->z, nb->norm_w, nb->eps, nb->apply, nb->rstd, stream);
        return e2;
    };
    // the scans that read dt themselves take the transformed copy
    const float *dt_scan = nb->transform() ? nb->dt_eff : dt;
    unsigned int *err = nullptr;
    if (pl.tc_state || pl.tc_scan) {
        err = device_error_word();
        if (!err) return SSD_ERR_CUDA;
    }
    float *l = reinterpret_cast<float *>(ws + pl.ws.l_offset);
    float *w = reinterpret_cast<float *>(ws + pl.ws.w_offset);
    float *dtq = reinterpret_cast<float *>(ws + pl.ws.dtq_offset);
    float *beta = reinterpret_cast<float *>(ws + pl.ws.beta_offset);
    float *alpha = reinterpret_cast<float *>(ws + pl.ws.alpha_offset);
    void *states = ws + pl.ws.states_offset;
    void *s_in = ws + pl.ws.s_in_offset;
    int *nsteep = reinterpret_cast<int *>(ws + pl.steep_offset);
    long long *steep_items = reinterpret_cast<long long *>(ws + pl.steep_offset + kAlign);
    float *gq = (pl.scan5 || pl.single) ? reinterpret_cast<float *>(ws + pl.gq_offset) : nullptr;
    float *chain = pl.single ? reinterpret_cast<float *>(ws + pl.chain_offset) : nullptr;
    unsigned int *flags = pl.single ? reinterpret_cast<unsigned int *>(ws + pl.flag_offset) : nullptr;
    float *seg = pl.presolved ? reinterpret_cast<float *>(ws + pl.seg_offset) : nullptr;
    float *start = pl.presolved ? reinterpret_cast<float *>(ws + pl.start_offset) : nullptr;
    for (int stage = 0; stage < 4; ++stage) {
        if (only_stage >= 0 && stage != only_stage) continue;
        cudaError_t e = cudaSuccess;
        if (d.nc == 0) {
            // shorter than one chunk: the tail kernel does everything
            if (stage == SSD_STAGE_CHUNK_SCAN) e = finish_scan();
            if (e != cudaSuccess) return SSD_ERR_CUDA;
            continue;
        }
        if (pl.single) {
            // cumsum (fused mode), the single-pass kernel, the block-factored scan
            // over the tiles it listed as steep.  Presolved: the cumsum also
            // writes w and alpha, stage 1 computes the state entering every
            // range of the single pass (two launches), and stage 3 runs the
            // single pass from those states, then the block-factored scan.
            const int max_steep = ssd::chunk_scan5_max_steep(d);
            switch (stage) {
                case SSD_STAGE_CHUNK_CUMSUM:
                    e = ssd::launch_chunk_cumsum(d, dt, A, l, pl.presolved ? w : nullptr, dtq, beta, alpha, gq,
                                                 nsteep, flags, nb->dt_bias, nb->softplus, nullptr, stream);
                    break;
                case SSD_STAGE_CHUNK_STATE:
                    e = pl.presolved
                            ? ssd::launch_presolve_ranges(d, pl.G, x, Bm, w, alpha, init_state, seg, start, err,
                                                          stream)
                            : ssd::launch_chunk_fused(d, x, gq, Bm, Cm, D, l, init_state, y, fin, chain, flags,
                                                      nullptr, 0, s_in, nsteep, steep_items, max_steep, err,
                                                      stream);
                    break;
                case SSD_STAGE_STATE_PASSING:
                    break;
                case SSD_STAGE_CHUNK_SCAN:
                    if (pl.presolved)
                        e = ssd::launch_chunk_fused(d, x, gq, Bm, Cm, D, l, init_state, y, fin, chain, flags, start,
                                                    pl.G, s_in, nsteep, steep_items, max_steep, err, stream);
                    if (e == cudaSuccess)
                        e = ssd::launch_chunk_scan_tc4(d, x, dtq, beta, Bm, Cm, D, l, s_in, y, steep_items, nsteep,
                                                       max_steep, err, stream);
                    if (e == cudaSuccess) e = finish_scan();
                    break;
            }
            if (e != cudaSuccess) return SSD_ERR_CUDA;
            continue;
        }
        switch (stage) {
            case SSD_STAGE_CHUNK_CUMSUM:
                // also empties the chunk-wide scan's steep-tile list
                e = ssd::launch_chunk_cumsum(d, dt, A, l, w, dtq, beta, alpha, gq,
                                             pl.scan5 ? nsteep : nullptr, nullptr, nb->dt_bias,
                                             nb->softplus, nb->transform() ? nb->dt_eff : nullptr, stream);
                break;
            case SSD_STAGE_CHUNK_STATE:
                e = pl.fused ? ssd::launch_state_fused(d, x, Bm, w, alpha, init_state, s_in, fin, err, stream)
                    : pl.tc_state ? ssd::launch_chunk_state_tc(d, x, Bm, w, states, err, stream)
                                : ssd::launch_chunk_state_simt(d, pl.bf16, x, Bm, w,
                                                               static_cast<float *>(states), stream);
                break;
            case SSD_STAGE_STATE_PASSING:
                if (pl.fused) break;  // done by the fused chunk_state kernel
                e = ssd::launch_state_passing(d, states, pl.tc_state, alpha, init_state, s_in,
                                              pl.tc_scan, fin, stream);
                break;
            case SSD_STAGE_CHUNK_SCAN:
                if (pl.scan5) {
                    // chunk-wide scan, then the block-factored scan over the tiles
                    // it listed as steep (an empty list costs one short launch)
                    e = ssd::launch_chunk_scan_tc5(d, x, gq, Bm, Cm, D, l, s_in, y, nsteep,
                                                   steep_items, err, stream);
                    if (e == cudaSuccess)
                        e = pl.tile_finish
                                ? ssd::launch_chunk_scan_tc(d, x, dt_scan, Bm, Cm, D, l, s_in, y, steep_items,
                                                            nsteep, ssd::chunk_scan5_max_steep(d), err, stream)
                                : ssd::launch_chunk_scan_tc4(d, x, dtq, beta, Bm, Cm, D, l, s_in, y,
                                                             steep_items, nsteep,
                                                             ssd::chunk_scan5_max_steep(d), err, stream);
                } else {
                    e = pl.tc_scan
                            ? (ssd::tc_chunk_scan4_supported(d)
                                   ? ssd::launch_chunk_scan_tc4(d, x, dtq, beta, Bm, Cm, D, l, s_in, y,
                                                                nullptr, nullptr, 0, err, stream)
                                   : ssd::launch_chunk_scan_tc(d, x, dt_scan, Bm, Cm, D, l, s_in, y, nullptr,
                                                               nullptr, 0, err, stream))
                            : ssd::launch_chunk_scan_simt(d, pl.bf16, x, dt_scan, Bm, Cm, D, l,
                                                          static_cast<const float *>(s_in), y, stream);
                }
                if (e == cudaSuccess) e = finish_scan();
                break;
        }
        if (e != cudaSuccess) return SSD_ERR_CUDA;
    }
    return SSD_OK;
}

// ---------------------------------------------------------------------------
// varlen: several sequences packed along the token axis of one row
// ---------------------------------------------------------------------------
// Validates the packing and makes one plan per non-empty sequence (nothing is
// launched); `need` gets the largest workspace among them.
ssd_status_t varlen_plans(const ssd_dims_t *dims, const int64_t *cu, int64_t nseq, int chunk_len,
                          size_t *need) {
    if (!dims || !cu) return SSD_ERR_NULL_ARG;
    if (dims->batch != 1 || nseq < 1 || cu[0] != 0 || cu[nseq] != dims->seqlen) return SSD_ERR_INVALID_DIM;
    *need = 0;
    for (int64_t i = 0; i < nseq; ++i) {
        if (cu[i + 1] < cu[i]) return SSD_ERR_INVALID_DIM;
        if (cu[i + 1] == cu[i]) continue;
        ssd_dims_t di = *dims;
        di.seqlen = cu[i + 1] - cu[i];
        Plan pl;
        const ssd_status_t s = make_plan(&di, chunk_len, &pl);
        if (s != SSD_OK) return s;
        if (pl.ws.total_bytes > *need) *need = pl.ws.total_bytes;
    }
    return SSD_OK;
}

}  // namespace

extern "C" {

size_t ssd_workspace_bytes(const ssd_dims_t *dims, int chunk_len) {
    Plan pl;
    if (make_plan(dims, chunk_len, &pl) != SSD_OK) return 0;
    return pl.ws.total_bytes;
}

ssd_status_t ssd_workspace_layout(const ssd_dims_t *dims, int chunk_len,
                                  ssd_workspace_layout_t *out) {
    if (!out) return SSD_ERR_NULL_ARG;
    Plan pl;
    ssd_status_t s = make_plan(dims, chunk_len, &pl);
    if (s != SSD_OK) return s;
    *out = pl.ws;
    return SSD_OK;
}

ssd_status_t ssd_forward_ws(const ssd_dims_t *dims, const void *x, const float *dt,
                            const float *A, const void *Bm, const void *Cm, const float *D,
                            int chunk_len, const float *init_state, void *y_out,
                            float *final_state_out, void *workspace, size_t workspace_bytes,
                            void *stream) {
    Plan pl;
    ssd_status_t s = make_plan(dims, chunk_len, &pl);
    if (s != SSD_OK) return s;
    s = check_tensors(pl, x, dt, A, Bm, Cm, D, init_state, y_out, final_state_out);
    if (s != SSD_OK) return s;
    if (!workspace || workspace_bytes < pl.ws.total_bytes ||
        (reinterpret_cast<uintptr_t>(workspace) & (kAlign - 1)))
        return SSD_ERR_WORKSPACE;
    return run(pl, x, dt, A, Bm, Cm, D, init_state, y_out, final_state_out,
               static_cast<char *>(workspace), static_cast<cudaStream_t>(stream));
}

ssd_status_t ssd_forward_stage(int stage, const ssd_dims_t *dims, const void *x,
                               const float *dt, const float *A, const void *Bm, const void *Cm,
                               const float *D, int chunk_len, const float *init_state,
                               void *y_out, float *final_state_out, void *workspace,
                               size_t workspace_bytes, void *stream) {
    if (stage < 0 || stage > 3) return SSD_ERR_INVALID_DIM;
    Plan pl;
    ssd_status_t s = make_plan(dims, chunk_len, &pl);
    if (s != SSD_OK) return s;
    s = check_tensors(pl, x, dt, A, Bm, Cm, D, init_state, y_out, final_state_out);
    if (s != SSD_OK) return s;
    if (!workspace || workspace_bytes < pl.ws.total_bytes ||
        (reinterpret_cast<uintptr_t>(workspace) & (kAlign - 1)))
        return SSD_ERR_WORKSPACE;
    return run(pl, x, dt, A, Bm, Cm, D, init_state, y_out, final_state_out,
               static_cast<char *>(workspace), static_cast<cudaStream_t>(stream), stage);
}

ssd_status_t ssd_forward(const ssd_dims_t *dims, const void *x, const float *dt, const float *A,
                         const void *Bm, const void *Cm, const float *D, int chunk_len,
                         const float *init_state, void *y_out, float *final_state_out,
                         void *stream) {
    Plan pl;
    ssd_status_t s = make_plan(dims, chunk_len, &pl);
    if (s != SSD_OK) return s;
    s = check_tensors(pl, x, dt, A, Bm, Cm, D, init_state, y_out, final_state_out);
    if (s != SSD_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    void *ws = nullptr;
    if (workspace_alloc(&ws, pl.ws.total_bytes, st) != cudaSuccess) {
        cudaGetLastError();
        return SSD_ERR_WORKSPACE;
    }
    s = run(pl, x, dt, A, Bm, Cm, D, init_state, y_out, final_state_out,
            static_cast<char *>(ws), st);
    if (cudaFreeAsync(ws, st) != cudaSuccess && s == SSD_OK) s = SSD_ERR_CUDA;
    return s;
}

size_t ssd_block_workspace_bytes(const ssd_dims_t *dims, int chunk_len, const ssd_block_opts_t *opts) {
    Plan pl;
    if (make_plan(dims, chunk_len, &pl) != SSD_OK) return 0;
    size_t total = pl.ws.total_bytes;
    if (opts && (opts->dt_bias || opts->dt_softplus))
        total = align_up(total + size_t(pl.d.B) * pl.d.T * pl.d.H * sizeof(float));
    return total;
}

ssd_status_t ssd_forward_block(const ssd_dims_t *dims, const void *x, const float *dt, const float *A,
                               const void *Bm, const void *Cm, const float *D, int chunk_len,
                               const float *init_state, void *y_out, float *final_state_out,
                               const ssd_block_opts_t *opts, void *workspace, size_t workspace_bytes,
                               void *stream) {
    Plan pl;
    ssd_status_t s = make_plan(dims, chunk_len, &pl);
    if (s != SSD_OK) return s;
    s = check_tensors(pl, x, dt, A, Bm, Cm, D, init_state, y_out, final_state_out);
    if (s != SSD_OK) return s;
    Neighbours nb;
    if (opts) {
        if (opts->reserved0 != 0) return SSD_ERR_INVALID_DIM;
        const void *ptrs[] = {opts->dt_bias, opts->z, opts->norm_weight, opts->rstd_out};
        for (const void *p : ptrs)
            if (misaligned(p)) return SSD_ERR_MISALIGNED;
        if (opts->norm_weight && !(opts->norm_eps > 0.f)) return SSD_ERR_INVALID_DIM;
        if (opts->norm_weight && !opts->norm_apply && !opts->rstd_out) return SSD_ERR_NULL_ARG;
        nb.dt_bias = opts->dt_bias;
        nb.softplus = opts->dt_softplus ? 1 : 0;
        nb.z = opts->z;
        nb.norm_w = opts->norm_weight;
        nb.eps = opts->norm_eps;
        nb.apply = opts->norm_apply != 0;
        nb.rstd = opts->norm_weight ? opts->rstd_out : nullptr;
    }
    const size_t need = ssd_block_workspace_bytes(dims, chunk_len, opts);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    void *ws = workspace;
    if (ws) {
        if (workspace_bytes < need || (reinterpret_cast<uintptr_t>(ws) & (kAlign - 1))) return SSD_ERR_WORKSPACE;
    } else if (workspace_alloc(&ws, need, st) != cudaSuccess) {
        cudaGetLastError();
        return SSD_ERR_WORKSPACE;
    }
    if (nb.transform()) nb.dt_eff = reinterpret_cast<float *>(static_cast<char *>(ws) + pl.ws.total_bytes);
    s = run(pl, x, dt, A, Bm, Cm, D, init_state, y_out, final_state_out, static_cast<char *>(ws), st, -1, &nb);
    if (!workspace && cudaFreeAsync(ws, st) != cudaSuccess && s == SSD_OK) s = SSD_ERR_CUDA;
    return s;
}

size_t ssd_varlen_workspace_bytes(const ssd_dims_t *dims, const int64_t *cu_seqlens, int64_t nseq,
                                  int chunk_len) {
    size_t need = 0;
    if (varlen_plans(dims, cu_seqlens, nseq, chunk_len, &need) != SSD_OK) return 0;
    return need;
}

ssd_status_t ssd_forward_varlen(const ssd_dims_t *dims, const int64_t *cu_seqlens, int64_t nseq, const void *x,
                                const float *dt, const float *A, const void *Bm, const void *Cm, const float *D,
                                int chunk_len, const float *init_states, void *y_out, float *final_states_out,
                                void *workspace, size_t workspace_bytes, void *stream) {
    size_t need = 0;
    ssd_status_t s = varlen_plans(dims, cu_seqlens, nseq, chunk_len, &need);
    if (s != SSD_OK) return s;
    if (!x || !dt || !A || !Bm || !Cm || !y_out) return SSD_ERR_NULL_ARG;
    const size_t esz = dims->dtype == SSD_BF16 ? 2 : 4;
    const int64_t H = dims->nheads, P = dims->headdim, N = dims->dstate, G = dims->ngroups;
    const int64_t st_elems = H * P * N;
    // every sequence's slices must keep the 16-byte alignment of the whole tensors
    for (int64_t i = 0; i < nseq; ++i) {
        const int64_t t0 = cu_seqlens[i];
        if (cu_seqlens[i + 1] == t0) continue;
        const char *px = static_cast<const char *>(x) + t0 * H * P * esz;
        const char *pb = static_cast<const char *>(Bm) + t0 * G * N * esz;
        const char *pc = static_cast<const char *>(Cm) + t0 * G * N * esz;
        const char *py = static_cast<const char *>(y_out) + t0 * H * P * esz;
        const float *pdt = dt + t0 * H;
        const void *ptrs[] = {px, pb, pc, py, pdt, A, D, init_states, final_states_out};
        for (const void *p : ptrs)
            if (misaligned(p)) return SSD_ERR_MISALIGNED;
    }
    if (need > 0 && (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & (kAlign - 1))))
        return SSD_ERR_WORKSPACE;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    for (int64_t i = 0; i < nseq; ++i) {
        const int64_t t0 = cu_seqlens[i], len = cu_seqlens[i + 1] - t0;
        const float *h0 = init_states ? init_states + i * st_elems : nullptr;
        float *fin = final_states_out ? final_states_out + i * st_elems : nullptr;
        if (len == 0) {
            // an empty sequence leaves its initial state (or zeros)
            if (fin) {
                const cudaError_t e = h0 ? cudaMemcpyAsync(fin, h0, st_elems * sizeof(float), cudaMemcpyDeviceToDevice, st)
                                         : cudaMemsetAsync(fin, 0, st_elems * sizeof(float), st);
                if (e != cudaSuccess) return SSD_ERR_CUDA;
            }
            continue;
        }
        ssd_dims_t di = *dims;
        di.seqlen = len;
        Plan pl;
        s = make_plan(&di, chunk_len, &pl);
        if (s != SSD_OK) return s;
        // the sequences run one after another on the stream and share the workspace
        s = run(pl, static_cast<const char *>(x) + t0 * H * P * esz, dt + t0 * H, A,
                static_cast<const char *>(Bm) + t0 * G * N * esz, static_cast<const char *>(Cm) + t0 * G * N * esz, D,
                h0, static_cast<char *>(y_out) + t0 * H * P * esz, fin, static_cast<char *>(workspace), st);
        if (s != SSD_OK) return s;
    }
    return SSD_OK;
}

// ---------------------------------------------------------------------------
// backward: the reverse mode, through four fp32 scans of the forward plans and
// the element-wise / prefix kernels of k_backward.cu
// ---------------------------------------------------------------------------
ssd_status_t ssd_backward(const ssd_dims_t *dims, const void *x, const float *dt, const float *A, const void *Bm,
                          const void *Cm, const float *D, int chunk_len, const float *init_state, const void *dy,
                          const float *dfinal_state, void *dx, float *ddt, float *dA, void *dB, void *dC,
                          float *dD, float *dinit_state, void *stream) {
    Plan pf;
    ssd_status_t s = make_plan(dims, chunk_len, &pf);
    if (s != SSD_OK) return s;
    if (!x || !dt || !A || !Bm || !Cm || !dy || !dx || !ddt || !dA || !dB || !dC) return SSD_ERR_NULL_ARG;
    if (dims->nheads > kMaxBackwardHeads) return SSD_ERR_UNSUPPORTED;
    {
        const void *ptrs[] = {x, dt, A, Bm, Cm, D, init_state, dy, dfinal_state, dx, ddt, dA, dB, dC, dD,
                              dinit_state};
        for (const void *p : ptrs)
            if (misaligned(p)) return SSD_ERR_MISALIGNED;
    }
    const ssd_dims_t &a = *dims;
    const bool bf16 = a.dtype == SSD_BF16;
    // The scans of the backward: K (= dL/dh_{t-1}, backwards in time) and h with
    // the forward's shape, in fp32 (their outputs feed the decay terms' prefix
    // sum, where bf16 outputs lose too much to cancellation), and the transposed
    // ones for dB and dC with headdim and dstate swapped and one group per head,
    // dstate split into S slices of W: bf16 on the tensor-core plans when the
    // inputs are bf16 with headdim 64 and dstate a multiple of 64 (W = 64),
    // else fp32 (W = dstate).
    ssd_dims_t dk = a;
    dk.dtype = SSD_F32;
    ssd_dims_t dtp = a;
    dtp.dstate = a.headdim;
    dtp.ngroups = a.nheads;
    bool scan_bf16 = bf16 && a.headdim == 64 && a.dstate % 64 == 0;
    Plan pk, pt;
    // (the caller's chunk length where 64 leaves a ragged tail the tail kernel cannot take)
    if (make_plan(&dk, kBackwardScanChunk, &pk) != SSD_OK && make_plan(&dk, chunk_len, &pk) != SSD_OK)
        return SSD_ERR_UNSUPPORTED;
    if (scan_bf16) {
        dtp.headdim = 64;
        if (make_plan(&dtp, chunk_len, &pt) != SSD_OK || !pt.tc_scan) scan_bf16 = false;
    }
    if (!scan_bf16) {
        dtp.headdim = a.dstate;
        dtp.dtype = SSD_F32;
        if (make_plan(&dtp, chunk_len, &pt) != SSD_OK) return SSD_ERR_UNSUPPORTED;
    }
    const int W = scan_bf16 ? 64 : int(a.dstate);
    const int S = int(a.dstate) / W;
    const size_t es = scan_bf16 ? 2 : 4;  // bytes per scan-buffer element
    const Dims &d = pf.d;
    const size_t nx = size_t(a.batch) * a.seqlen * a.nheads * a.headdim;
    const size_t nn = size_t(a.batch) * a.seqlen * a.nheads * a.dstate;
    const size_t nbc = size_t(a.batch) * a.seqlen * a.ngroups * a.dstate;
    const size_t ntok = size_t(a.batch) * a.seqlen * a.nheads;
    const size_t nst = size_t(a.batch) * a.nheads * a.headdim * a.dstate;
    const size_t nbh = size_t(a.batch) * a.nheads;
    const size_t nsl = size_t(a.batch) * a.seqlen * a.nheads * W;        // one slice of xb, xc, yb, yc
    const size_t nstsl = size_t(a.batch) * a.nheads * W * a.headdim;    // one slice of a transposed state
    // fp32 copies of bf16 inputs: x, B, C for the scan of h; dy for fp32 transposed scans
    const bool copies = bf16;
    const bool dy_copy = bf16 && !scan_bf16;
    // one allocation: the buffers, the transposed states and the scans' workspace
    size_t off = 0;
    auto take = [&](size_t bytes) { const size_t o = off; off = align_up(off + bytes); return o; };
    const size_t o_xk = take(nx * 4), o_dtr = take(ntok * 4), o_bk = take(nbc * 4), o_ck = take(nbc * 4),
                 o_xb = take(nn * es), o_xc = take(nn * es), o_dyr = take(nx * es), o_xrr = take(nx * es);
    const size_t o_xf = copies ? take(nx * 4) : 0, o_dyf = dy_copy ? take(nx * 4) : 0,
                 o_bf = copies ? take(nbc * 4) : 0, o_cf = copies ? take(nbc * 4) : 0;
    const size_t o_yk = take(nx * 4), o_yh = take(nx * 4), o_yb = take(nn * es), o_yc = take(nn * es);
    const size_t o_dh0 = dinit_state ? 0 : take(nst * 4);
    const size_t o_xu = take(ntok * 4), o_cc = take(ntok * 4), o_rr = take(ntok * 4), o_dd = take(ntok * 4),
                 o_R0 = take(nbh * 4), o_dAp = take(nbh * 4), o_dDp = take(nbh * 4);
    const size_t o_ft = dfinal_state ? take(nst * 4) : 0, o_ht = init_state ? take(nst * 4) : 0;
    const size_t o_ws = off;
    off = align_up(off + (pk.ws.total_bytes > pt.ws.total_bytes ? pk.ws.total_bytes : pt.ws.total_bytes));
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    char *buf = nullptr;
    if (workspace_alloc(reinterpret_cast<void **>(&buf), off, st) != cudaSuccess) {
        cudaGetLastError();
        return SSD_ERR_WORKSPACE;
    }
    auto F = [&](size_t o) { return reinterpret_cast<float *>(buf + o); };
    auto V = [&](size_t o) { return static_cast<void *>(buf + o); };
    ssd::BackwardBuffers w;
    w.xk = F(o_xk); w.bk = F(o_bk); w.ck = F(o_ck); w.xb = V(o_xb); w.xc = V(o_xc);
    w.dyr = V(o_dyr); w.xrr = V(o_xrr); w.yk = F(o_yk); w.yh = F(o_yh); w.yb = V(o_yb); w.yc = V(o_yc);
    w.dtr = F(o_dtr);
    w.xf = copies ? F(o_xf) : nullptr; w.dyf = dy_copy ? F(o_dyf) : nullptr;
    w.bf = copies ? F(o_bf) : nullptr; w.cf = copies ? F(o_cf) : nullptr;
    w.dh0 = dinit_state ? dinit_state : F(o_dh0);
    w.xu = F(o_xu); w.cc = F(o_cc); w.rr = F(o_rr); w.dd = F(o_dd); w.R0 = F(o_R0); w.dA_part = F(o_dAp);
    w.dD_part = F(o_dDp);
    w.W = W;
    w.scan_bf16 = scan_bf16;
    float *ft = dfinal_state ? F(o_ft) : nullptr, *ht = init_state ? F(o_ht) : nullptr;
    char *ws = buf + o_ws;
    // the forward-direction scans read the inputs themselves where their dtype fits
    const void *xs = copies ? static_cast<const void *>(w.xf) : x;    // the fp32 scan of h
    const void *bs = copies ? static_cast<const void *>(w.bf) : Bm;
    const void *cs = copies ? static_cast<const void *>(w.cf) : Cm;
    const void *xt = scan_bf16 || !bf16 ? x : static_cast<const void *>(w.xf);  // the transposed scans
    const void *dyt = dy_copy ? static_cast<const void *>(w.dyf) : dy;
    s = SSD_OK;
    if (ssd::launch_backward_prep(d, bf16, x, dy, dt, A, Bm, Cm, w, st) != cudaSuccess) s = SSD_ERR_CUDA;
    if (s == SSD_OK && ft &&
        ssd::launch_transpose_state(int64_t(nbh), int(a.headdim), int(a.dstate), W, dfinal_state, ft, st) !=
            cudaSuccess)
        s = SSD_ERR_CUDA;
    if (s == SSD_OK && ht &&
        ssd::launch_transpose_state(int64_t(nbh), int(a.headdim), int(a.dstate), W, init_state, ht, st) !=
            cudaSuccess)
        s = SSD_ERR_CUDA;
    // K = dL/dh_{t-1}, backwards in time: read out against B, final state dh0
    if (s == SSD_OK) s = run(pk, w.xk, w.dtr, A, w.bk, w.ck, nullptr, dfinal_state, w.yk, w.dh0, ws, st);
    // h_t C_t (the forward without the skip term)
    if (s == SSD_OK) s = run(pk, xs, dt, A, bs, cs, nullptr, init_state, w.yh, nullptr, ws, st);
    for (int sl = 0; sl < S && s == SSD_OK; ++sl) {
        char *xb = static_cast<char *>(w.xb) + sl * nsl * es, *xc = static_cast<char *>(w.xc) + sl * nsl * es;
        char *yb = static_cast<char *>(w.yb) + sl * nsl * es, *yc = static_cast<char *>(w.yc) + sl * nsl * es;
        // K^T read out against x (dB), backwards in time
        s = run(pt, xb, w.dtr, A, w.dyr, w.xrr, nullptr, ft ? ft + sl * nstsl : nullptr, yb, nullptr, ws, st);
        // h^T read out against dy (dC)
        if (s == SSD_OK)
            s = run(pt, xc, dt, A, xt, dyt, nullptr, ht ? ht + sl * nstsl : nullptr, yc, nullptr, ws, st);
    }
    if (s == SSD_OK &&
        ssd::launch_backward_post(d, bf16, x, dy, dt, A, D, init_state, w, dx, ddt, dA, dB, dC, dD, st) != cudaSuccess)
        s = SSD_ERR_CUDA;
    if (cudaFreeAsync(buf, st) != cudaSuccess && s == SSD_OK) s = SSD_ERR_CUDA;
    return s;
}

const char *ssd_status_string(ssd_status_t status) {
    switch (status) {
        case SSD_OK: return "SSD_OK: success";
        case SSD_ERR_NULL_ARG: return "SSD_ERR_NULL_ARG: a required pointer is NULL";
        case SSD_ERR_INVALID_DIM: return "SSD_ERR_INVALID_DIM: invalid dimensions";
        case SSD_ERR_UNSUPPORTED: return "SSD_ERR_UNSUPPORTED: sizes outside the supported set";
        case SSD_ERR_MISALIGNED: return "SSD_ERR_MISALIGNED: pointer not 16-byte aligned";
        case SSD_ERR_CUDA: return "SSD_ERR_CUDA: CUDA call or kernel launch failed";
        case SSD_ERR_DEVICE_TIMEOUT: return "SSD_ERR_DEVICE_TIMEOUT: device-side wait expired";
        case SSD_ERR_WORKSPACE: return "SSD_ERR_WORKSPACE: workspace missing, too small or unallocatable";
    }
    return "SSD_ERR_UNKNOWN: unknown status code";
}

ssd_status_t ssd_device_status(void *stream) {
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(st) != cudaSuccess) {
        cudaGetLastError();
        return SSD_ERR_CUDA;
    }
    unsigned int *err = device_error_word();
    if (!err) return SSD_ERR_CUDA;
    unsigned int v = 0;
    if (cudaMemcpy(&v, err, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return SSD_ERR_CUDA;
    if (v) {
        const unsigned int zero = 0;
        if (cudaMemcpy(err, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess)
            return SSD_ERR_CUDA;
        return SSD_ERR_DEVICE_TIMEOUT;
    }
    return SSD_OK;
}

ssd_status_t ssd_workspace_trim(void) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        cudaGetLastError();
        return SSD_ERR_CUDA;
    }
    cudaMemPool_t pool = workspace_pool(dev);
    if (!pool) return SSD_OK;
    if (cudaDeviceSynchronize() != cudaSuccess || cudaMemPoolTrimTo(pool, 0) != cudaSuccess) {
        cudaGetLastError();
        return SSD_ERR_CUDA;
    }
    return SSD_OK;
}

const char *ssd_version(void) { return "ssd-b200 0.3.1 sm_100a"; }

}  // extern "C"
