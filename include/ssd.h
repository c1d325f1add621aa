/*
 * ssd.h -- C ABI of libssd.so, the B200 (sm_100a) Mamba-2 SSD forward scan.
 *
 * The operation (per batch b, head h; group g = h / (H / G)):
 *
 *     h_t = exp(dt_t * A_h) * h_{t-1} + dt_t * x_t B_t^T      (state, P x N)
 *     y_t = h_t C_t + D_h * x_t
 *
 * the selective SSM with a scalar-times-identity transition ("Transformers are
 * SSMs", Dao & Gu 2024; akillness.github.io "State Space Duality and Mamba-2",
 * sections "Mathematical Foundations" and "The Scalar-Identity Structural
 * Constraint"), evaluated blockwise as the chunked SSD algorithm (aifetchly
 * blog "Mamba-2 Architecture: State Space Duality Explained", section "The
 * Chunked SSD Algorithm"): the masked product (L o C B^T) X inside each chunk of
 * chunk_len tokens, and the state recurrence between chunks.  The steps are
 * ssd_chunk_cumsum, ssd_chunk_state, ssd_state_passing and ssd_chunk_scan; on
 * the tensor-core path with enough (batch, head pair) chains the last three
 * run as ONE kernel that carries each chain's state on chip from chunk to
 * chunk (see single_pass under ssd_workspace_layout).
 *
 * Conventions for every entry point:
 *  - All tensor pointers are DEVICE pointers to contiguous row-major memory,
 *    16-byte aligned.  The caller owns every buffer; the library keeps no
 *    pointer after the call returns.
 *  - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default
 *    stream) and never synchronise the host.  Argument errors are detected and
 *    returned BEFORE anything is launched; launch errors come back as
 *    SSD_ERR_CUDA.  Errors of kernels that already ran surface, as usual in
 *    CUDA, on the next synchronising call.
 *  - Shared state: a per-device cache of device properties; one device-side
 *    error word per device (set by an expired bounded wait, read and cleared by
 *    ssd_device_status); a per-device stream-ordered memory pool from which the
 *    entry points that allocate their own workspace take it (the pool keeps
 *    its reserved memory between calls, so repeated calls reuse it;
 *    ssd_workspace_trim returns the unused part); and the static scratch
 *    array of ssd_forward_static,
 *    which every call of that entry point on a device shares, so that such
 *    calls overlapping in time race (see ssd_forward_static).  The other entry
 *    points keep no state between calls and may run concurrently on
 *    different streams with separate outputs and workspaces.
 */
#ifndef SSD_H_
#define SSD_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SSD_API __attribute__((visibility("default")))
#else
#define SSD_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    SSD_OK = 0,
    SSD_ERR_NULL_ARG = 1,       /* a required pointer is NULL                    */
    SSD_ERR_INVALID_DIM = 2,    /* a size is <= 0 or H % G != 0                  */
    SSD_ERR_UNSUPPORTED = 3,    /* sizes outside the supported set (see below)   */
    SSD_ERR_MISALIGNED = 4,     /* a pointer is not 16-byte aligned              */
    SSD_ERR_CUDA = 5,           /* a CUDA runtime call or launch failed          */
    SSD_ERR_DEVICE_TIMEOUT = 6, /* a bounded device-side wait expired            */
    SSD_ERR_WORKSPACE = 7       /* workspace NULL/too small, or allocation failed */
} ssd_status_t;

/* Storage dtype of x, B, C and y.  dt, A, D and the states are always fp32. */
typedef enum { SSD_F32 = 0, SSD_BF16 = 1 } ssd_dtype_t;

typedef struct {
    int64_t batch;   /* B */
    int64_t seqlen;  /* T */
    int64_t nheads;  /* H */
    int64_t headdim; /* P */
    int64_t dstate;  /* N */
    int64_t ngroups; /* G: B and C are shared by H/G consecutive heads */
    int32_t dtype;   /* ssd_dtype_t */
    int32_t reserved; /* must be 0 */
} ssd_dims_t;

/*
 * Supported sizes (anything else returns SSD_ERR_UNSUPPORTED):
 *   chunk_len in {32, 64, 128, 256}; any seqlen >= 1 -- when seqlen is not a
 *   multiple of chunk_len the full chunks run as below and the last
 *   seqlen mod chunk_len tokens run as the recurrence itself from the state the
 *   full chunks leave (one more launch), which needs dstate in {8, 16, 32, 64}
 *   or a multiple of 64 and headdim * max(1, dstate / 64) <= 1024;
 *   1 <= headdim <= 256, 1 <= dstate <= 256; nheads % ngroups == 0;
 *   SSD_BF16 additionally: headdim % 8 == 0 and dstate % 8 == 0.
 * The tensor-core path runs for SSD_BF16 with headdim == 64,
 * dstate in {16, 32, 64, 128, 256} and chunk_len in {64, 128, 256}; other
 * supported shapes run on the CUDA-core kernels of the same library.
 */

/*
 * ssd_forward -- one forward scan.
 *
 *   x          [B, T, H, P]  dtype
 *   dt         [B, T, H]     fp32, the step sizes as used (positive; any
 *                            softplus/bias is applied by the caller)
 *   A          [H]           fp32, the per-head decay rate (negative for decay)
 *   Bm, Cm     [B, T, G, N]  dtype (input and output projections)
 *   D          [H]           fp32 skip weights, or NULL for no skip term
 *   chunk_len                tokens per chunk
 *   init_state [B, H, P, N]  fp32 initial state, or NULL for zeros
 *   y_out      [B, T, H, P]  dtype, written; must not alias any input
 *   final_state_out [B,H,P,N] fp32 final state, or NULL; it may alias
 *                            init_state (it is written after every read)
 *   stream                   cudaStream_t
 *
 * Intermediates (ssd_workspace_bytes) are allocated stream-ordered on
 * `stream` from the library's workspace pool and released to it before
 * return (cudaMallocFromPoolAsync / cudaFreeAsync).
 * Accuracy against the fp64 recurrence: max|y - y_ref| / max|y_ref| <= 1e-4
 * for SSD_F32 and <= 2e-2 for SSD_BF16 when every dt_t * A_h <= 0; the same
 * bound holds for the final state.
 */
SSD_API ssd_status_t ssd_forward(const ssd_dims_t *dims, const void *x, const float *dt,
                         const float *A, const void *Bm, const void *Cm, const float *D,
                         int chunk_len, const float *init_state, void *y_out,
                         float *final_state_out, void *stream);

/*
 * ssd_forward_ws -- ssd_forward with caller-provided workspace.
 * `workspace` is a device buffer of at least ssd_workspace_bytes(dims,
 * chunk_len) bytes, 256-byte aligned; otherwise SSD_ERR_WORKSPACE.  After the
 * call the workspace holds the intermediates described by
 * ssd_workspace_layout (valid once the stream reaches that point).
 */
SSD_API ssd_status_t ssd_forward_ws(const ssd_dims_t *dims, const void *x, const float *dt,
                            const float *A, const void *Bm, const void *Cm, const float *D,
                            int chunk_len, const float *init_state, void *y_out,
                            float *final_state_out, void *workspace, size_t workspace_bytes,
                            void *stream);

/*
 * ssd_forward_static -- ssd_forward without any allocation.  The pages have no
 * counterpart: this is a library-level convenience for callers that cannot
 * hand in a workspace and must not allocate (their device memory is held by
 * another allocator, or a cudaMalloc's device-wide synchronisation is not
 * acceptable where they run).
 *
 * Arguments, layouts, ownership and accuracy are those of ssd_forward.  The
 * intermediates live in one statically sized device array of
 * SSD_STATIC_SCRATCH_BYTES per device (64 MiB; e.g. the 8 x 2048-token,
 * 24-head, P = 64, N = 128 layer at chunk_len 256 needs 54 MiB).  A call whose
 * ssd_workspace_bytes exceeds that returns SSD_ERR_WORKSPACE before any CUDA
 * call.  The array's address is looked up once per device on the first call
 * there (set-up), so make that first call before any stream capture.  Nothing
 * in the array needs to start at zero.  All calls on a device share it: calls
 * that overlap in time (different streams, unordered host threads) race; calls
 * in order on one stream do not.
 */
#define SSD_STATIC_SCRATCH_BYTES ((size_t)64 << 20)
SSD_API ssd_status_t ssd_forward_static(const ssd_dims_t *dims, const void *x, const float *dt,
                                const float *A, const void *Bm, const void *Cm, const float *D,
                                int chunk_len, const float *init_state, void *y_out,
                                float *final_state_out, void *stream);

/*
 * ssd_forward_stage -- run ONE of the four kernels of ssd_forward_ws, with the
 * same arguments and the same launch configuration, reading the earlier
 * stages' results from `workspace` and writing its own there (or to y_out /
 * final_state_out).  Calling the stages 0, 1, 2, 3 in order on one stream is
 * equivalent to one ssd_forward_ws call; this exists to time and test each
 * kernel on its own.
 *   stage 0  ssd_chunk_cumsum   dt, A          -> l, w, alpha
 *   stage 1  ssd_chunk_state    x, B, w        -> states
 *            (fused_state layouts: x, B, w, alpha, init_state -> s_in,
 *            final_state_out)
 *   stage 2  ssd_state_passing  states, alpha, init_state -> s_in, final_state_out
 *            (fused_state layouts: nothing)
 *   stage 3  ssd_chunk_scan     x, dt, B, C, D, l, s_in   -> y_out
 *            (chunk_len 128/256 bf16 layouts: the chunk-wide scan, then the
 *            list-mode scan of the tiles it left -- the block-factored kernel,
 *            or the per-tile kernel for dstate 256 -- two launches)
 * Any other stage value returns SSD_ERR_INVALID_DIM.
 */
typedef enum {
    SSD_STAGE_CHUNK_CUMSUM = 0,
    SSD_STAGE_CHUNK_STATE = 1,
    SSD_STAGE_STATE_PASSING = 2,
    SSD_STAGE_CHUNK_SCAN = 3
} ssd_stage_t;

SSD_API ssd_status_t ssd_forward_stage(int stage, const ssd_dims_t *dims, const void *x,
                                       const float *dt, const float *A, const void *Bm,
                                       const void *Cm, const float *D, int chunk_len,
                                       const float *init_state, void *y_out,
                                       float *final_state_out, void *workspace,
                                       size_t workspace_bytes, void *stream);

/*
 * ssd_step -- one token of the recurrence for every (batch, head): the decode
 * step.  The recurrent form of the scalar-identity SSM (akillness.github.io
 * "State Space Duality and Mamba-2: Unifying Transformers and Semiseparable
 * Matrices", "Mathematical Foundations: From State Spaces to Semiseparable
 * Matrices"), with dt on the decay and the input as in ssd_forward:
 *   state <- exp(dt_t A_h) state + dt_t x_t B_t^T      (in place)
 *   y_t    = state C_t + D_h x_t                       (with the new state)
 * A generation loop calls it once per new token on the state that
 * ssd_forward's final_state_out left behind.
 *
 *   dims       seqlen must be 1 (else SSD_ERR_INVALID_DIM); batch, nheads,
 *              headdim, dstate, ngroups, dtype as for ssd_forward, with
 *              headdim, dstate <= 256 (any value, no chunk rule)
 *   x_t        [B, H, P]     dtype
 *   dt_t       [B, H]        fp32 step sizes
 *   A          [H]           fp32
 *   B_t, C_t   [B, G, N]     dtype
 *   D          [H]           fp32, or NULL for no skip term
 *   state      [B, H, P, N]  fp32, read and overwritten with the new state;
 *                            16-byte alignment and dstate in {16, 32, 64,
 *                            128, 256} take the vectorised kernel, anything
 *                            else a scalar one
 *   y_t        [B, H, P]     dtype, written; must not alias the inputs
 *   stream                   cudaStream_t
 * The caller owns every buffer (device pointers).  Asynchronous, no
 * allocation, one kernel launch; argument errors come back before the launch,
 * a failed launch as SSD_ERR_CUDA.  Accuracy against the fp64 step: the bounds
 * of ssd_forward, per call.
 */
SSD_API ssd_status_t ssd_step(const ssd_dims_t *dims, const void *x_t, const float *dt_t,
                              const float *A, const void *B_t, const void *C_t, const float *D,
                              float *state, void *y_t, void *stream);

/*
 * ssd_forward_block -- the scan together with its neighbours in the Mamba-2
 * block (aifetchly blog "Mamba-2 Architecture: State Space Duality Explained",
 * "Step 2: Full Mamba-2 Block with Gated Projections": softplus on dt before the
 * SSD call; the SSD output gated by silu of the z branch, then RMSNorm over the
 * token's d_inner = H * P values; akillness.github.io "State Space Duality and
 * Mamba-2", the block diagram: "Element-wise Gating", RMSNorm):
 *
 *   dt_eff = softplus(dt + dt_bias)        (each part only when requested)
 *   y      = the scan of ssd_forward with dt_eff
 *   g      = y * silu(z),  silu(z) = z / (1 + e^-z)            (if z != NULL)
 *   rstd_t = 1 / sqrt(mean over the token's H*P values of g^2 + norm_eps)
 *   y_out  = g * rstd_t * norm_weight  (norm_apply != 0)
 *          = g * norm_weight           (norm_apply == 0: rstd_t goes to
 *                                       rstd_out and the caller applies it; it
 *                                       is one factor per token, so it can be
 *                                       applied to the rows of the next linear
 *                                       layer's output instead)
 *          = g                         (norm_weight == NULL)
 *
 *   opts       NULL = no neighbours (then this is ssd_forward_ws);
 *              dt_bias [H] fp32 or NULL; dt_softplus nonzero for softplus;
 *              z [B, T, H, P] dtype or NULL; norm_weight [H * P] fp32 or NULL;
 *              norm_eps > 0 when norm_weight is given (else
 *              SSD_ERR_INVALID_DIM); rstd_out [B, T] fp32 (required when
 *              norm_weight is given and norm_apply == 0, else SSD_ERR_NULL_ARG;
 *              optional otherwise); reserved0 must be 0.
 *   workspace  ssd_block_workspace_bytes bytes, 256-byte aligned, or NULL:
 *              then it is allocated stream-ordered on `stream` and released
 *              before return, as in ssd_forward.
 * Every other argument is that of ssd_forward.  The final state is the scan's.
 * Accuracy: the bounds of ssd_forward, on y_out against the same chain in fp64.
 */
typedef struct {
    const float *dt_bias;
    int32_t dt_softplus;
    int32_t norm_apply;
    const void *z;
    const float *norm_weight;
    float norm_eps;
    int32_t reserved0;
    float *rstd_out;
} ssd_block_opts_t;

SSD_API size_t ssd_block_workspace_bytes(const ssd_dims_t *dims, int chunk_len,
                                         const ssd_block_opts_t *opts);
SSD_API ssd_status_t ssd_forward_block(const ssd_dims_t *dims, const void *x, const float *dt,
                                       const float *A, const void *Bm, const void *Cm,
                                       const float *D, int chunk_len, const float *init_state,
                                       void *y_out, float *final_state_out,
                                       const ssd_block_opts_t *opts, void *workspace,
                                       size_t workspace_bytes, void *stream);

/*
 * ssd_forward_varlen -- several independent sequences packed along the token
 * axis of one row (the "varlen" layout): sequence i is tokens
 * [cu_seqlens[i], cu_seqlens[i+1]) and starts from its own initial state, so
 * no state crosses a boundary (each sequence is the recurrence of
 * akillness.github.io "State Space Duality and Mamba-2", "Mathematical
 * Foundations", on its own tokens).
 *
 *   dims        batch must be 1; seqlen = total tokens; other fields as for
 *               ssd_forward (else SSD_ERR_INVALID_DIM)
 *   cu_seqlens  HOST array of nseq + 1 offsets: cu_seqlens[0] = 0,
 *               non-decreasing, cu_seqlens[nseq] = seqlen (empty sequences
 *               allowed); read during the call only
 *   x, dt, Bm, Cm, y_out   the packed tensors, layouts as for ssd_forward with
 *               B = 1; every sequence's slices must stay 16-byte aligned
 *               (SSD_ERR_MISALIGNED otherwise)
 *   A, D        [H] fp32 as for ssd_forward (D may be NULL)
 *   init_states [nseq, H, P, N] fp32, or NULL for zeros
 *   final_states_out [nseq, H, P, N] fp32, or NULL; an empty sequence's
 *               final state is its initial state
 *   workspace   ssd_varlen_workspace_bytes bytes, 256-byte aligned (may be
 *               NULL when that size is 0)
 * The sequences run one after another on `stream`, each with the plan its own
 * length selects (ragged lengths included) and all sharing the workspace.
 * Every argument is validated before the first launch.  Accuracy as for
 * ssd_forward, per sequence.
 */
SSD_API size_t ssd_varlen_workspace_bytes(const ssd_dims_t *dims, const int64_t *cu_seqlens, int64_t nseq,
                                          int chunk_len);
SSD_API ssd_status_t ssd_forward_varlen(const ssd_dims_t *dims, const int64_t *cu_seqlens, int64_t nseq,
                                        const void *x, const float *dt, const float *A, const void *Bm,
                                        const void *Cm, const float *D, int chunk_len,
                                        const float *init_states, void *y_out, float *final_states_out,
                                        void *workspace, size_t workspace_bytes, void *stream);

/*
 * ssd_backward -- the gradients of a scalar loss L through ssd_forward: given
 * dy = dL/dy and dfinal_state = dL/dfinal_state, returns dL/d(every input).
 * The reverse mode of the recurrence (akillness.github.io "State Space Duality
 * and Mamba-2", "Mathematical Foundations"): with G_t = dL/dh_t,
 *   G_t = dy_t C_t^T + exp(dt_{t+1} A_h) G_{t+1},  G_{T-1} = dy_{T-1} C_{T-1}^T + dfinal
 *   dx_t = dt_t G_t B_t + D_h dy_t,   dB_t = sum_heads dt_t G_t^T x_t,
 *   dC_t = sum_heads h_t^T dy_t,      dD_h = sum dy_t . x_t,
 *   ddt_t = x_t . (G_t B_t) + A_h exp(dt_t A_h) (G_t : h_{t-1}),
 *   dA_h = sum dt_t exp(dt_t A_h) (G_t : h_{t-1}),   dinit = exp(dt_0 A_h) G_0.
 * Computed with four scans of the library's own chunked forward (G backwards
 * in time and h forwards, in fp32 with 64-token chunks whatever chunk_len is;
 * each transposed for dB and dC, with chunk_len, on the bf16 tensor-core plans
 * when the inputs are bf16 with headdim 64 and dstate a multiple of 64, in
 * fp32 otherwise) plus element-wise and prefix-sum kernels (k_backward.cu
 * gives the identities).
 *
 *   inputs as for ssd_forward; dy [B,T,H,P] dtype; dfinal_state [B,H,P,N] fp32
 *   or NULL (zero)
 *   dx [B,T,H,P] dtype; ddt [B,T,H] fp32; dA [H] fp32; dB, dC [B,T,G,N] dtype;
 *   dD [H] fp32 or NULL (not computed); dinit_state [B,H,P,N] fp32 or NULL
 * Requires dt_t > 0 for every token (the scan of G takes a_t dy_t / dt_t as its
 * input) and nheads <= 12288 (else SSD_ERR_UNSUPPORTED).  Scratch memory
 * (about 20 fp32 copies of x's size) is allocated stream-ordered on `stream`
 * from the library's workspace pool and released to it before return.  Accuracy: the
 * gradients' max abs error over their max |value| within 1e-3 of the fp64
 * reverse mode on fp32-exact inputs.
 */
SSD_API ssd_status_t ssd_backward(const ssd_dims_t *dims, const void *x, const float *dt, const float *A,
                                  const void *Bm, const void *Cm, const float *D, int chunk_len,
                                  const float *init_state, const void *dy, const float *dfinal_state, void *dx,
                                  float *ddt, float *dA, void *dB, void *dC, float *dD, float *dinit_state,
                                  void *stream);

/* Bytes of workspace one call needs (0 if the arguments are invalid). */
SSD_API size_t ssd_workspace_bytes(const ssd_dims_t *dims, int chunk_len);

/*
 * Where each intermediate sits inside the workspace (byte offsets; nc = T/Q):
 *   l      fp32 [B, H, nc, Q]  chunk-local inclusive cumsum of dt*A
 *   w      fp32 [B, H, nc, Q]  exp(l_last - l_s) * dt_s (chunk-state weights)
 *   dtq    fp32 [B, H, nc, Q]  dt regrouped per chunk and head
 *   beta   fp32 [B, H, nc, Q]  exp(l_{32k+31} - l_s) * dt_s, k = s / 32 (source
 *                              factors of the factored in-chunk decay); dtq
 *                              and beta are written for every chunk when the
 *                              block-factored scan is the scan engine, else
 *                              only for chunks it finishes (steep tiles)
 *   alpha  fp32 [B, H, nc]     exp(l_last), the decay across a whole chunk
 *   states [B, nc, H, P, N]    per-chunk states S_c = sum_s w_s x_s B_s^T;
 *                              element type given by states_dtype
 *   s_in   [B, nc, H, P, N]    state entering each chunk; element type given
 *                              by s_in_dtype (SSD_F32 or SSD_BF16)
 * `tensor_core` is 1 when the call runs the tcgen05 kernels, 0 otherwise;
 * `launches` is the number of kernels one call launches.  `fused_state` is 1
 * when ssd_chunk_state and ssd_state_passing run as one kernel (the
 * (batch, head pair) units fill 60-100% of the GPU's SMs in one wave): the
 * per-chunk states then never
 * reach memory, the states region is empty (states_offset == s_in_offset) and
 * stage 2 of ssd_forward_stage does nothing.
 * `single_pass` is 1 when chunk state, state passing and chunk scan run as ONE
 * kernel (bf16, headdim 64, dstate 64 or 128, chunk_len 128 / 256 (64 as 128),
 * an even number of heads per group), in one of two forms:
 *  - hand-off (at least 40% as many (batch, head pair) chains as the GPU has
 *    SMs; launches == 3): each chunk's state is carried to the next through an
 *    fp32 slot per (batch, head) in the workspace, so neither the per-chunk
 *    states nor the incoming states reach memory (w, alpha and states are not
 *    written, s_in only for chunks with a tile the block-factored scan
 *    finishes).  Stage 1 of ssd_forward_stage runs that kernel, stage 2
 *    nothing, stage 3 the block-factored scan of the tiles it listed;
 *  - presolved (fewer chains, with ranges of at least 16 chunks per CTA or
 *    dstate 64; launches == 5): stage 1 computes the state entering each CTA's
 *    range (a pass over x and B in range mode, then a pass chaining those
 *    states along each chain; w and alpha are written), stage 2 nothing,
 *    stage 3 the single pass from those states and the block-factored scan.
 * `scan_engine` names the kernel
 * that computes y.  `chunk_len` is the chunk length the kernels run with: the
 * caller's, except on the tensor-core path (SSD_BF16, headdim 64), where the
 * chunk length only sets the blocking of the same recurrence: chunk_len 64
 * runs 128-token chunks (the kernels' tile height) when the single pass
 * applies; the four-kernel sequence runs 256-token chunks at chunk_len 32 /
 * 64 / 128 (half the chunk states to write and read back); dstate 256 runs
 * 128-token chunks (the chunk-wide scan holds one 128-token tile of C at that
 * dstate).  None of these is taken when it would lengthen the ragged tail
 * (seqlen mod chunk length).  The arrays above then describe the chunks the
 * kernels run (nc = T / chunk_len of this struct).
 */
typedef enum {
    SSD_ENGINE_SIMT = 0,            /* chunk scan on the CUDA cores                     */
    SSD_ENGINE_TILE = 1,            /* tensor-core scan, one 128-row tile per work item */
    SSD_ENGINE_BLOCK_FACTORED = 2,  /* tensor-core scan, block-factored decay           */
    SSD_ENGINE_CHUNK_WIDE = 3,      /* tensor-core scan, whole chunk, shared scores     */
    SSD_ENGINE_SINGLE_PASS = 4      /* chunk state + state passing + scan in one kernel */
} ssd_scan_engine_t;

typedef struct {
    size_t total_bytes;
    size_t l_offset, w_offset, dtq_offset, beta_offset, alpha_offset, states_offset, s_in_offset;
    int32_t s_in_dtype;
    int32_t tensor_core;
    int32_t launches;
    int32_t states_dtype; /* element type of states: SSD_F32 or SSD_BF16 */
    int32_t fused_state;
    int32_t single_pass;  /* 1: stages 1-3 run as one kernel (see below)   */
    int32_t scan_engine;  /* ssd_scan_engine_t of the chunk scan            */
    int32_t chunk_len;    /* chunk length the kernels use (see below)       */
} ssd_workspace_layout_t;

SSD_API ssd_status_t ssd_workspace_layout(const ssd_dims_t *dims, int chunk_len,
                                  ssd_workspace_layout_t *out);

/*
 * ssd_device_status -- synchronise `stream`, then report (and clear) the
 * device-side error word of the current device: SSD_ERR_DEVICE_TIMEOUT if a
 * bounded wait inside a tensor-core kernel expired since the last query (that
 * kernel skipped its remaining work, so its outputs are incomplete), SSD_ERR_CUDA
 * if the synchronisation reported an error, SSD_OK otherwise.  With
 * ssd_workspace_trim, the only entry points that block the host.
 */
SSD_API ssd_status_t ssd_device_status(void *stream);

/* Static description of a status code (never NULL). */
SSD_API const char *ssd_status_string(ssd_status_t status);

/*
 * ssd_workspace_trim -- synchronise the current device, then return to the
 * system the workspace memory that the library's pool on that device holds
 * but no call is using (the pool otherwise keeps it for the next call).
 * SSD_ERR_CUDA if the synchronisation or the trim failed.  Blocks the host.
 */
SSD_API ssd_status_t ssd_workspace_trim(void);

/* Library version, e.g. "ssd-b200 0.1.0 sm_100a". */
SSD_API const char *ssd_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SSD_H_ */
