// kernels.h -- host-side launchers of the SSD kernels (internal to libssd.so).
#pragma once

#include <cuda_runtime.h>

#include "common.cuh"

namespace ssd {

// ssd_chunk_cumsum: dt, A -> l, w, dtq, beta [B,H,nc,Q], alpha [B,H,nc]; sets
// *nsteep = 0 when nsteep != nullptr; and,
// if gq != nullptr (chunk_len 128 / 256), per (b, h, c) the chunk-wide scan's
// token factors g_s = exp(-l_s) dt_s (Q floats) followed by one steep flag per
// 128-token tile (1.0 when the tile is left to the block-factored scan) and
// padding: chunk_gq(Q) floats in all
__host__ __device__ constexpr int chunk_gq(int Q) { return Q + 4; }
// a 128-token tile k is steep when -l at its last token reaches this (the
// chunk-wide scan's factors exp(-l_s) would exceed e^72), or when one of its
// dt is 0 (the skip term is recovered from the scaled rows as D / g)
constexpr float kScanSteep = 72.f;
// chain_flags != nullptr selects the fused mode (chunk_len 128 / 256, gq
// required): the reference and flags of the single-pass kernel, no w / alpha,
// dtq and beta only for chunks with a flagged tile, and the (b, head pair)
// chain flags [B, H/2] reset to 0.
// dt_bias [H] (or nullptr) and dt_softplus select the block's dt transform,
// softplus(dt + dt_bias); dt_eff (or nullptr) receives it in dt's layout.
cudaError_t launch_chunk_cumsum(const Dims &d, const float *dt, const float *A, float *l,
                                float *w, float *dtq, float *beta, float *alpha, float *gq,
                                int *nsteep, unsigned int *chain_flags, const float *dt_bias,
                                int dt_softplus, float *dt_eff, cudaStream_t stream);

// The block's output side in place on y [B,T,H,P]: g = y * silu(z) (z may be
// nullptr), then with a weight w [H*P] the RMSNorm factor rstd per token
// (written to rstd_out if non-null) and out = g * rstd * w (apply) or g * w.
cudaError_t launch_gate_norm(const Dims &d, bool bf16, void *y, const void *z, const float *w, float eps,
                             bool apply, float *rstd_out, cudaStream_t stream);

// ssd_state_passing: states [B,nc,H,P,N] (fp32 or bf16 per states_bf16), alpha
// -> s_in [B,nc,H,P,N] (fp32 or bf16 per s_in_bf16), final state [B,H,P,N] fp32
// (may be NULL)
cudaError_t launch_state_passing(const Dims &d, const void *states, bool states_bf16,
                                 const float *alpha, const float *init_state, void *s_in,
                                 bool s_in_bf16, float *final_state, cudaStream_t stream);

// CUDA-core (SIMT) chunk state and chunk scan, any supported shape.
// bf16 selects the storage type of x/B/C/y.  s_in is fp32 here.
cudaError_t launch_chunk_state_simt(const Dims &d, bool bf16, const void *x, const void *Bm,
                                    const float *w, float *states, cudaStream_t stream);
cudaError_t launch_chunk_scan_simt(const Dims &d, bool bf16, const void *x, const float *dt,
                                   const void *Bm, const void *Cm, const float *D,
                                   const float *l, const float *s_in, void *y,
                                   cudaStream_t stream);

// Tensor-core (tcgen05) kernels, bf16 storage, P == 64.
bool tc_chunk_state_supported(const Dims &d);
// chunk_state + state_passing as one kernel (units of (b, head pair) walked over
// all chunks); `sms` is the SM count the launch will fill
bool tc_state_fused_supported(const Dims &d, int sms);
// The states entering the ranges of a presolved single pass with G CTAs:
// the fused state kernel in range mode (each CTA's last segment from zero, or
// from h0 at a chain start, into seg [G][128][N] fp32), then those partial
// states chained along every chain into start [G][128][N] (rows = head of the
// pair x P).  Needs w and alpha from the cumsum.
bool presolved_ranges_supported(const Dims &d);
size_t presolved_state_bytes(int G, const Dims &d);
cudaError_t launch_presolve_ranges(const Dims &d, int G, const void *x, const void *Bm, const float *w,
                                   const float *alpha, const float *h0, float *seg, float *start,
                                   unsigned int *err, cudaStream_t stream);
bool tc_chunk_scan_supported(const Dims &d);
// `err` is a device word: bit 0 is set when a bounded wait inside a kernel
// expired (the kernel then skips its remaining work and exits cleanly).
cudaError_t launch_chunk_state_tc(const Dims &d, const void *x, const void *Bm, const float *w,
                                  void *states_bf16, unsigned int *err, cudaStream_t stream);
// writes s_in (bf16, [B, nc, H, P, N]) and, if fin != nullptr, the final state
cudaError_t launch_state_fused(const Dims &d, const void *x, const void *Bm, const float *w,
                               const float *alpha, const float *h0, void *s_in_bf16, float *fin,
                               unsigned int *err, cudaStream_t stream);
// items == nullptr: every (b, c, tile, head block); otherwise list mode: the
// *nitems packed (b, c, tile, head) items (at most max_items) that the
// chunk-wide scan left as steep, walked by one CTA per SM
cudaError_t launch_chunk_scan_tc(const Dims &d, const void *x, const float *dt, const void *Bm,
                                 const void *Cm, const float *D, const float *l,
                                 const void *s_in_bf16, void *y, const long long *items,
                                 const int *nitems, int max_items, unsigned int *err,
                                 cudaStream_t stream);
// Persistent warp-specialised variant (dstate <= 128); dtq and beta come from
// ssd_chunk_cumsum.  Writes y with TMA stores.
bool tc_chunk_scan4_supported(const Dims &d);
// items == nullptr: every (b, c, tile, head); otherwise list mode: the *nitems
// packed (b, c, tile, head) items (at most max_items) that the chunk-wide scan
// left to this kernel
cudaError_t launch_chunk_scan_tc4(const Dims &d, const void *x, const float *dtq,
                                  const float *beta, const void *Bm, const void *Cm,
                                  const float *D, const float *l, const void *s_in_bf16, void *y,
                                  const long long *items, const int *nitems, int max_items,
                                  unsigned int *err, cudaStream_t stream);
// chunk-wide tensor-core scan: masked scores shared by the heads of a group,
// one accumulator per 128-row tile; tiles that the cumsum kernel flagged as
// steep are appended to (nsteep, items) for the kernel above
bool tc_chunk_scan5_supported(const Dims &d);
int chunk_scan5_max_steep(const Dims &d);
cudaError_t launch_chunk_scan_tc5(const Dims &d, const void *x, const float *gq, const void *Bm,
                                  const void *Cm, const float *D, const float *l,
                                  const void *s_in_bf16, void *y, int *nsteep, long long *items,
                                  unsigned int *err, cudaStream_t stream);

// The whole pass after the cumsum in one persistent kernel (bf16, P = 64,
// N in {64, 128}, chunk_len 128 / 256, an even number of heads per group):
// chunk state, state passing through per-(b, h) fp32 slots `chain` [B,H,P,N]
// with flags [B, H/2], and chunk scan.  Tiles flagged steep by the cumsum are
// appended to (nsteep, items) for the block-factored scan, with s_in (bf16
// [B,nc,H,P,N]) written for their chunks.
bool tc_chunk_fused_supported(const Dims &d);
size_t chunk_fused_chain_bytes(const Dims &d);
size_t chunk_fused_flag_bytes(const Dims &d);
// presolved != nullptr: the grid is presolved_grid CTAs (any number), and CTA
// k's range starts from the fp32 state presolved[k] ([128 rows (head of the
// pair, p)][N], computed by the two passes below) instead of waiting for the
// CTA before it; no state is handed on.
cudaError_t launch_chunk_fused(const Dims &d, const void *x, const float *gq, const void *Bm, const void *Cm,
                               const float *D, const float *l, const float *h0, void *y, float *fin,
                               float *chain, unsigned int *flags, const float *presolved, int presolved_grid,
                               void *s_in_bf16, int *nsteep, long long *items, int max_items, unsigned int *err,
                               cudaStream_t stream);

// The last T mod chunk_len tokens of every (b, h) as the recurrence, from
// h_in (the full chunks' final state, or the initial state; nullptr = zeros),
// with the block's dt transform when dt_bias / dt_softplus are given; writes y
// of those tokens and, if fin != nullptr, the final state.
bool tail_supported(const Dims &d);
cudaError_t launch_tail(const Dims &d, bool bf16, int t_begin, const void *x, const float *dt,
                        const float *dt_bias, int dt_softplus, const float *A, const void *Bm, const void *Cm,
                        const float *D, const float *h_in, void *y, float *fin, cudaStream_t stream);

// The backward pass's own kernels (the scans run through the forward plans).
// The scans that feed the decay terms (K and h) run in fp32; the transposed
// ones (dB, dC) hold bf16 when scan_bf16 (they then take the tensor-core
// plans), fp32 otherwise.  Reversed = token t stored at T-1-t:
//   xk [B,T,H,P] a_t dy_t / dt_t reversed;  dtr [B,T,H] dt reversed;
//   bk, ck [B,T,G,N] C and B reversed       (the scan of K = dL/dh_{t-1})
//   xb [S][B,T,H,W] a_t C_t / dt_t reversed, dstate in S slices of W columns;
//   dyr, xrr [B,T,H,P] dy, x reversed       (the transposed scans for dB)
//   xc [S][B,T,H,W] B per head               (the transposed forward scans for dC)
//   xf, bf, cf: fp32 copies of x, B, C for the scan of h (nullptr: fp32 inputs);
//   dyf: fp32 copy of dy for fp32 transposed scans of bf16 inputs
//   yk, yh [B,T,H,P] fp32, yb, yc [S][B,T,H,W]   the scans' outputs
//   dh0 [B,H,P,N]; xu, cc, rr [B,T,H]; R0, dA_part [B,H]
struct BackwardBuffers {
    void *xb, *xc, *dyr, *xrr, *yb, *yc;
    float *xk, *bk, *ck, *yk, *yh;
    float *dtr, *xf, *dyf, *bf, *cf, *dh0, *xu, *cc, *rr, *dd, *R0, *dA_part, *dD_part;
    int W;           // dstate columns per transposed scan
    bool scan_bf16;  // transposed-scan buffers in bf16
};
cudaError_t launch_backward_prep(const Dims &d, bool bf16, const void *x, const void *dy, const float *dt,
                                 const float *A, const void *Bm, const void *Cm, const BackwardBuffers &w,
                                 cudaStream_t stream);
cudaError_t launch_transpose_state(int64_t BH, int P, int N, int W, const float *s, float *st, cudaStream_t stream);
cudaError_t launch_backward_post(const Dims &d, bool bf16, const void *x, const void *dy, const float *dt,
                                 const float *A, const float *D, const float *h0, const BackwardBuffers &w,
                                 void *dx, float *ddt, float *dA, void *dB, void *dC, float *dD,
                                 cudaStream_t stream);

}  // namespace ssd
