/*
 * mok.h -- C ABI of the B200 (sm_100a) mixture-of-experts layer library (libmok.so).
 *
 * The layer is the one the pages centre on: a DeepSeek-V3-type MoE layer
 * ("Cursor åpner megakernelen som ga 41 prosent flere tokens i sekundet",
 * last paragraph), forward in BF16 and MXFP8 and backward in BF16
 * ("Megakernels are dead and back…", section "Números de MoK"; the MXFP8
 * backward below is this library's extension, not claimed there), computed
 * deterministically with no CPU-GPU synchronisation inside the layer
 * ("Cursor veröffentlicht MoE-Megakernel Mixture-of-Kittens als Open Source",
 * section "Kommunikation im Kernel").  All experts live on one GPU.
 *
 * Conventions shared by every entry point:
 *  - Pointers named "device" are CUDA device pointers on the current device;
 *    pointers named "host" are host memory (pinned or pageable).
 *  - All tensors are dense, row-major, contiguous, with the shapes given.
 *    bf16 tensors are passed as raw 16-bit storage.  Device pointers must be
 *    16-byte aligned.
 *  - The caller owns every buffer, including workspaces; the library never
 *    allocates device memory and never synchronises the host inside
 *    moe_fwd/moe_bwd.  Work is enqueued on `stream` (a cudaStream_t, NULL =
 *    legacy default stream).
 *  - Outputs are overwritten, never accumulated into.
 *  - Return value: MOK_OK (0) or a negative MOK_ERR_* code; argument errors are
 *    detected on the host before anything is enqueued.  Errors that arise on
 *    the device (a bounded wait that ran out) are recorded in a device status
 *    word and reported by moe_status.
 *  - Results are bit-identical across calls with the same inputs (fixed
 *    reduction orders, no floating-point atomics).
 */
#ifndef MOK_H
#define MOK_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- error codes ---------------------------------------------------------- */
#define MOK_OK 0
#define MOK_ERR_INVALID (-1)      /* bad shape, pointer, alignment or option */
#define MOK_ERR_DEVICE (-2)       /* current device is not sm_100 (B200) */
#define MOK_ERR_WORKSPACE (-3)    /* ctx or scratch buffer too small */
#define MOK_ERR_LAUNCH (-4)       /* a CUDA call failed while enqueueing */
#define MOK_ERR_UNSUPPORTED (-5)  /* valid but not implemented combination */

/* device status bits (moe_status) */
#define MOK_STATUS_TIMEOUT 1      /* a bounded wait inside a kernel ran out */
#define MOK_STATUS_BAD_INDEX 2    /* a routing index outside [0, E) reached the dispatch (it was
                                     placed as expert 0; the layer's own selection never makes one) */

/* ---- configuration -------------------------------------------------------- */
#define MOK_SCORE_SOFTMAX 0       /* softmax over all experts, top-k, renormalised */
#define MOK_SCORE_SIGMOID 1       /* sigmoid scores + selection bias, group-limited top-k */

#define MOK_DTYPE_BF16 0          /* bf16 operands, fp32 accumulation */
#define MOK_DTYPE_MXFP8 1         /* e4m3 operands with 1x32 ue8m0 block scales */

typedef struct moe_cfg {
    int32_t T;            /* tokens in the batch, >= 1 */
    int32_t H;            /* hidden size, multiple of 256 */
    int32_t E;            /* routed experts, 1..256 */
    int32_t I;            /* expert intermediate size, multiple of 128 */
    int32_t top_k;        /* experts per token, 1..min(E, 16) */
    int32_t n_shared;     /* shared experts applied to every token, 0..4 */
    int32_t I_shared;     /* shared intermediate size; must equal I when n_shared > 0 */
    int32_t score_fn;     /* MOK_SCORE_* */
    int32_t n_group;      /* expert groups for group-limited selection (1 = none); divides E */
    int32_t topk_group;   /* groups kept per token, 1..n_group */
    float routed_scale;   /* multiplies the renormalised routing weights */
    int32_t dtype;        /* MOK_DTYPE_* */
} moe_cfg;

/*
 * Layer parameters (device pointers).  Expert weights use the layouts
 *   w_gate_up [E, 2I, H]: rows 0..I-1 the gate projection, rows I..2I-1 the up projection
 *   w_down    [E, H, I]
 *   ws_*      the same for the n_shared shared experts ([S, 2I, H], [S, H, I]).
 * For MOK_DTYPE_BF16 the weights are bf16 and the s_* scale pointers are NULL.
 * For MOK_DTYPE_MXFP8 the weights are e4m3 codes (one byte each, same shapes)
 * and s_* hold one ue8m0 byte per 32 consecutive elements along the last
 * (contraction) axis, for the tensors [E*2I, H] and [E*H, I] (S in place of E
 * for the shared experts), in the packed weight-scale layout that
 * moe_quantize_mxfp8_weights writes.
 * The MXFP8 backward also reads the weights quantised along the other axis,
 * transposed, as moe_quantize_mxfp8_weights_t writes them:
 *   wt_down    [E, I, H] e4m3: W_down[e]^T quantised along H; st_down its scales
 *              (packed layout of the [E*I, H] tensor)
 *   wt_gate_up [E, H, 2I] e4m3: W_gate_up[e]^T quantised along 2I; st_gate_up its
 *              scales (packed layout of the [E*H, 2I] tensor)
 *   wst_*, sst_* the same for the shared experts.
 * They are ignored (and may be NULL) otherwise.
 */
typedef struct moe_params {
    const float *router_w;      /* [E, H] fp32 */
    const float *e_bias;        /* [E] fp32 selection bias (sigmoid scoring), or NULL */
    const float *logit_bias;    /* [E] fp32 term added to the router logits, or NULL */
    const void *w_gate_up;
    const void *w_down;
    const uint8_t *s_gate_up;
    const uint8_t *s_down;
    const void *ws_gate_up;
    const void *ws_down;
    const uint8_t *ss_gate_up;
    const uint8_t *ss_down;
    const void *wt_gate_up;
    const void *wt_down;
    const uint8_t *st_gate_up;
    const uint8_t *st_down;
    const void *wst_gate_up;
    const void *wst_down;
    const uint8_t *sst_gate_up;
    const uint8_t *sst_down;
} moe_params;

/* Routing record (device pointers; any may be NULL to skip that output). */
typedef struct moe_routing {
    int32_t *topk_idx;   /* [T, top_k] selected experts, slot order = selection order */
    float *topk_w;       /* [T, top_k] routing weights */
    int32_t *counts;     /* [E] tokens per expert */
    int32_t *offsets;    /* [E+1] exclusive prefix sum of counts */
    int32_t *perm;       /* [T*top_k] sorted row -> t*top_k + slot (expert-major, token ascending) */
    int32_t *inv_perm;   /* [T*top_k] t*top_k + slot -> sorted row */
} moe_routing;

/* Gradients (device pointers, all overwritten).  dws_* may be NULL when n_shared == 0. */
typedef struct moe_grads {
    void *dx;            /* [T, H] bf16 */
    void *dw_gate_up;    /* [E, 2I, H] bf16 */
    void *dw_down;       /* [E, H, I] bf16 */
    float *drouter_w;    /* [E, H] fp32 */
    void *dws_gate_up;   /* [S, 2I, H] bf16 */
    void *dws_down;      /* [S, H, I] bf16 */
} moe_grads;

/*
 * Sizes of the caller-allocated buffers for a configuration.
 *   ctx_bytes         saved forward state that moe_bwd reads (routing record,
 *                     gate/up pre-activations, h, weighted h, per-slot rows)
 *   fwd_scratch_bytes temporary device memory of moe_fwd
 *   bwd_scratch_bytes temporary device memory of moe_bwd
 * The forward's buffer (ctx or forward scratch) and the backward scratch also
 * hold the tile counters of that pass's grouped GEMMs.  The pass zeroes them
 * on its stream before its first launch, so nothing needs to start at zero.
 * Two passes that overlap on the GPU need separate buffers.
 * Any output pointer may be NULL.  Returns MOK_ERR_INVALID for a bad cfg.
 */
int moe_workspace_size(const moe_cfg *cfg, size_t *ctx_bytes, size_t *fwd_scratch_bytes,
                       size_t *bwd_scratch_bytes);

/*
 * Forward pass.  x: [T, H] bf16 (device); y: [T, H] bf16 (device, output).
 * routing: optional copy of the routing record (NULL = none).
 * save_for_backward != 0 stores the state moe_bwd needs in ctx, which must then
 * be at least ctx_bytes long; with save_for_backward == 0, ctx may be NULL.
 * The forward follows the steps: router logits (fp32), scoring and top-k with
 * ties to the lower expert index, deterministic counts/prefix scan/stable
 * permutation, pull-gathered gate/up grouped GEMM with a SwiGLU epilogue,
 * down grouped GEMM whose epilogue pushes each row into its (token, slot)
 * row, and a fixed-order weighted sum over slots (shared experts last,
 * weight 1).  The pull-at-dispatch / push-at-combine split follows
 * "Cursor åpner megakernelen…" (paragraph on pulling versus pushing tokens).
 * Non-finite input: a selection score that is NaN ranks below every other
 * score (as -inf), so every token still gets top_k distinct experts in
 * [0, E) (ties to the lower index); such a token's weights and outputs are
 * NaN.  Other tokens are unaffected.
 * MOK_DTYPE_MXFP8 with save_for_backward != 0 also keeps, for moe_bwd, the
 * gate/up pre-activations, the dequantised h and w * h (bf16) and the
 * dequantised x.
 */
int moe_fwd(const moe_cfg *cfg, const void *x, const moe_params *params, void *y,
            const moe_routing *routing, void *ctx, size_t ctx_bytes, int save_for_backward,
            void *scratch, size_t scratch_bytes, void *stream);

/*
 * Backward pass.  x and dy: [T, H] bf16 (device); ctx: the buffer a moe_fwd
 * call with save_for_backward != 0 filled for the same x and params.  Computes
 * dx, the expert weight gradients and the router weight gradient (the
 * selection bias gets none) with fixed reduction orders.
 * MOK_DTYPE_MXFP8: the two data-gradient GEMMs take MXFP8 operands quantised
 * along their contraction axis -- dy (1x32 blocks along H) times wt_down, and
 * dGU = d(gate, up) (1x32 blocks along 2I, quantised from fp32 in the down
 * dgrad's epilogue) times wt_gate_up; the slot gradients come from the first
 * product against the forward's quantised h; the weight gradients are BF16
 * GEMMs (dW_gate_up from the bf16 dGU and the dequantised x, dW_down from dy
 * and the saved w * h).  It needs the wt_* / st_* (and wst_* / sst_*) params
 * and I a multiple of 256 (MOK_ERR_UNSUPPORTED otherwise).  Under the
 * persistent schedule it is one launch, as the BF16 backward.
 */
int moe_bwd(const moe_cfg *cfg, const void *x, const void *dy, const moe_params *params,
            const void *ctx, size_t ctx_bytes, const moe_grads *grads, void *scratch,
            size_t scratch_bytes, void *stream);

/*
 * Host-buffer variants: x_host / y_host (and dy_host / dx_host) are host
 * memory; the call copies them through the scratch buffer (which must then be
 * at least moe_host_scratch_size bytes), runs the layer on `stream` and
 * synchronises that stream before returning.  Parameters, ctx and the other
 * gradients stay on the device.  moe_bwd_host takes x_host = NULL to reuse the
 * x that the preceding moe_fwd_host on the same stream left in the first
 * T*H*2 bytes of the same scratch buffer (nothing else may have written that
 * buffer in between): the second upload of x is then skipped.
 */
int moe_host_scratch_size(const moe_cfg *cfg, int backward, size_t *bytes);
int moe_fwd_host(const moe_cfg *cfg, const void *x_host, const moe_params *params, void *y_host,
                 void *ctx, size_t ctx_bytes, int save_for_backward, void *scratch,
                 size_t scratch_bytes, void *stream);
int moe_bwd_host(const moe_cfg *cfg, const void *x_host, const void *dy_host,
                 const moe_params *params, const void *ctx, size_t ctx_bytes, void *dx_host,
                 const moe_grads *grads, void *scratch, size_t scratch_bytes, void *stream);

/*
 * One training step through host buffers: the forward (state saved in ctx) and
 * the backward.  x_host, dy_host: [T, H] bf16 (host) in; y_host, dx_host:
 * [T, H] bf16 (host) out; the weight and router gradients go to `grads` on the
 * device (grads->dx is ignored).  The transfers overlap the passes: dy is
 * uploaded on a second stream of the library's while the forward runs, and y
 * is downloaded on it while the backward runs, so with pinned host buffers
 * only the upload of x and the download of dx add to the step.  The results
 * equal those of moe_fwd_host + moe_bwd_host byte for byte.  scratch: device
 * memory of at least moe_host_scratch_size(cfg, 2, ...) bytes (backward = 2
 * asks for this call's size).  The call waits for both streams before it
 * returns.  The second stream (one per host thread and device) is created on
 * first use and kept.
 */
int moe_step_host(const moe_cfg *cfg, const void *x_host, const void *dy_host, const moe_params *params,
                  void *y_host, void *dx_host, void *ctx, size_t ctx_bytes, const moe_grads *grads,
                  void *scratch, size_t scratch_bytes, void *stream);

/*
 * Pipelined training steps through host buffers: the same step as moe_step_host
 * (same results, byte for byte), enqueued without waiting, so that consecutive
 * calls on one stream overlap every transfer with the passes.  Each call:
 *   - takes x from the device x slot of this call when the previous call
 *     uploaded x_host there (its x_next_host), else uploads it first;
 *   - uploads dy on the library's upload stream (once the previous step's
 *     backward has read the device copy) while the forward runs;
 *   - downloads y on the library's download stream while the backward runs, and
 *     uploads x_next_host (NULL: none) into the other x slot meanwhile;
 *   - downloads dx (two device dx slots) while the next step runs.
 * Arguments as moe_step_host; scratch: at least moe_host_scratch_size(cfg, 3, ...)
 * bytes (two x slots, y, dy, two dx slots, the backward's workspace), the same
 * buffer for every call of a sequence (another buffer starts a new sequence).
 * The host buffers x_host, x_next_host, dy_host must stay unchanged, and
 * y_host, dx_host must not be read, until moe_step_host_sync returns; the
 * weight and router gradients in `grads` (device) are overwritten by every
 * call, in stream order.  On an error every stream of the sequence is drained
 * before the call returns.  The two streams (per host thread and device) are
 * created on first use and kept.
 */
int moe_step_host_async(const moe_cfg *cfg, const void *x_host, const void *x_next_host, const void *dy_host,
                        const moe_params *params, void *y_host, void *dx_host, void *ctx, size_t ctx_bytes,
                        const moe_grads *grads, void *scratch, size_t scratch_bytes, void *stream);
/* Waits until every step enqueued by moe_step_host_async on this host thread, and
 * `stream`, have completed (all of their transfers included). */
int moe_step_host_sync(void *stream);

/*
 * MXFP8 quantisation along the last axis: src [rows, K] bf16 (device) ->
 * q [rows, K] e4m3 codes and scales [rows, K/32] ue8m0 (device).  Per block of
 * 32 consecutive elements the exponent e is the smallest integer with
 * amax <= 448 * 2^e (clamped to [-127, 127]; an all-zero block takes -127),
 * the scale byte is e + 127 and each element is x / 2^e rounded to nearest
 * even e4m3 with saturation.  K must be a multiple of 32.
 */
int moe_quantize_mxfp8(const void *src, int64_t rows, int64_t K, void *q, void *scales,
                       void *stream);

/*
 * The same quantisation for expert weights, with the scales in the packed
 * weight-scale layout the MXFP8 layer reads: (K/128) x (rows/128) tiles of
 * 512 bytes, tile (kb, rb) at byte offset (kb * rows/128 + rb) * 512, holding
 * for row r = 128 rb + 32 q + i (0 <= q < 4, 0 <= i < 32) and 32-element block
 * j = 4 kb + s (0 <= s < 4) the scale byte at 16 i + 4 q + s.  This is the
 * block-scaled MMA's scale-factor layout for a 128-row block, so the layer
 * fetches one K block of a weight tile's scales as one 512-byte copy per 128
 * rows.  q is [rows, K] e4m3 as for moe_quantize_mxfp8; scales holds
 * rows * K / 32 bytes.  rows and K must be multiples of 128 (MOK_ERR_INVALID
 * otherwise).
 */
int moe_quantize_mxfp8_weights(const void *src, int64_t rows, int64_t K, void *q, void *scales,
                               void *stream);

/*
 * Transposed weight quantisation for the MXFP8 backward: src [batch, R, C]
 * bf16 (device) -> q [batch, C, R] e4m3 (row (b, c) of the [batch*C, R] matrix
 * is column c of src[b]), quantised along R in blocks of 32 with the rule of
 * moe_quantize_mxfp8, and scales in the packed weight-scale layout of that
 * [batch*C, R] matrix (as moe_quantize_mxfp8_weights).  R and batch*C must be
 * multiples of 128, C a multiple of 32 (MOK_ERR_INVALID otherwise).  W_down
 * [E, H, I] gives wt_down (R = H, C = I); W_gate_up [E, 2I, H] gives
 * wt_gate_up (R = 2I, C = H).
 */
int moe_quantize_mxfp8_weights_t(const void *src, int64_t batch, int64_t R, int64_t C, void *q,
                                 void *scales, void *stream);

/*
 * Both MXFP8 copies of a weight tensor from one read of it, for the
 * requantisation after each optimizer step of MXFP8 training: src [batch, R, C]
 * bf16 (device) -> q [batch, R, C] and scales exactly as
 * moe_quantize_mxfp8_weights(src, batch*R, C, ...) writes them, and qt
 * [batch, C, R] and scales_t exactly as moe_quantize_mxfp8_weights_t writes
 * them.  R must be a multiple of 128 and C of 256 (MOK_ERR_INVALID otherwise).
 */
int moe_quantize_mxfp8_weights_both(const void *src, int64_t batch, int64_t R, int64_t C, void *q,
                                    void *scales, void *qt, void *scales_t, void *stream);

/*
 * Phase tracing.  When events are set, every later moe_fwd (moe_bwd) records
 * fwd_events[i] (bwd_events[i]) on its stream just before launching phase i
 * and the last event after its final launch, so that elapsed times between
 * consecutive events time each phase on the launching stream.  Under the
 * persistent forward schedule the forward is one launch: fwd_events[0] is
 * recorded before it and the others after it (see moe_trace_device).  Events are
 * cudaEvent_t handles owned by the caller.  Phases:
 *   forward  (MOK_FWD_PHASES = 5, needs 6 events): router, dispatch,
 *            gate/up GEMM, down GEMM, combine
 *   backward (MOK_BWD_PHASES = 8, needs 9 events): down dgrad GEMM (its
 *            epilogue also forms the slot-gradient partial sums), slot
 *            gradient, router-gradient partial sums, router-gradient
 *            reduction, down wgrad GEMM, gate/up dgrad GEMM, gate/up wgrad
 *            GEMM, dx sum
 * Pass n = 0 to stop tracing.  The setting is per host thread.
 */
#define MOK_FWD_PHASES 5
#define MOK_BWD_PHASES 8
int moe_trace_events(void *const *fwd_events, int n_fwd, void *const *bwd_events, int n_bwd);

/*
 * Forward pass that allocates nothing and takes no workspace.
 *
 * The pages describe no such call; it exists for callers that cannot hand the
 * layer a device buffer: runtimes that plan every byte of device memory ahead
 * of time and forbid allocation once running, plug-in hosts that give a layer
 * only its inputs and outputs, and processes whose device memory is already
 * fully reserved by another allocator.
 *
 * It runs the same kernels as moe_fwd without saved state (inference; BF16 or
 * MXFP8), with its intermediate buffers placed in one static device array of
 * MOK_STATIC_SCRATCH_BYTES that the library declares at file scope.  Every GPU
 * that loads the library holds that array until the process exits.
 *   - x, y and the parameters are device pointers as for moe_fwd; the caller
 *     still owns them.
 *   - Shapes whose forward scratch (the fwd_scratch_bytes of
 *     moe_workspace_size) exceeds MOK_STATIC_SCRATCH_BYTES are rejected with
 *     MOK_ERR_WORKSPACE before anything is enqueued.
 *   - The first call on a device looks up the array's device address (a host
 *     runtime call); make that first call before any stream capture.
 *   - All calls on a device share the one array, and each call overwrites what
 *     the previous one left there (nothing in it needs to start at zero).  Two
 *     calls that overlap on the GPU, from different streams or threads, race on
 *     it: serialise them.
 * No cudaMalloc, cudaFree or allocating library routine is called.
 */
#define MOK_STATIC_SCRATCH_BYTES (32u << 20)
int moe_fwd_static(const moe_cfg *cfg, const void *x, const moe_params *params, void *y, void *stream);

/*
 * Where the forward keeps one of its intermediate tensors inside its buffer
 * (ctx when save_for_backward != 0, the forward scratch otherwise), for
 * inspection and tests: *offset = byte offset from the buffer's start, *bytes =
 * size.  The contents are valid once the forward on the stream has completed
 * and until that buffer is next written.  R = T * (top_k + n_shared) sorted
 * rows: the routed rows expert-major (the order of moe_routing.perm), then
 * n_shared blocks of T rows (shared expert s, token t at row T*top_k + s*T + t).
 *   MOK_SAVED_H          [R, I] bf16 h = silu(g) u (BF16 layer; MXFP8 with
 *                        save_for_backward: the dequantised h)
 *   MOK_SAVED_HQ         [R, I] e4m3 codes of h (MXFP8 layer)
 *   MOK_SAVED_HS         [R, I/32] ue8m0 scale bytes of h, row-major (MXFP8 layer)
 *   MOK_SAVED_GU         [R, 2I] bf16 gate and up pre-activations (save_for_backward)
 *   MOK_SAVED_HW         [R, I] bf16 routing weight times h (save_for_backward)
 *   MOK_SAVED_ROW_TOKEN  [R] int32 token of each sorted row
 *   MOK_SAVED_ROW_W      [R] fp32 routing weight of each sorted row (1 for shared rows)
 * Returns MOK_ERR_UNSUPPORTED when the configuration keeps no such tensor and
 * MOK_ERR_INVALID for an unknown `which` or a bad cfg.  The pages have no
 * counterpart; this is a window on the saved state for the library's users.
 */
#define MOK_SAVED_H 0
#define MOK_SAVED_HQ 1
#define MOK_SAVED_HS 2
#define MOK_SAVED_GU 3
#define MOK_SAVED_HW 4
#define MOK_SAVED_ROW_TOKEN 5
#define MOK_SAVED_ROW_W 6
int moe_saved_tensor(const moe_cfg *cfg, int save_for_backward, int which, size_t *offset, size_t *bytes);

/*
 * Schedule of the passes (per host thread; default PERSISTENT).
 *   MOK_SCHEDULE_PERSISTENT  each pass is one cooperative launch of one
 *       persistent kernel, one CTA per SM -- the fusion of the layer into one
 *       kernel that "Cursor åpner megakernelen…" (the quoted paragraph)
 *       describes.  Forward: router, top-k, dispatch, the two expert GEMMs and
 *       the combine are phases separated by grid barriers, except that the down
 *       GEMM starts an M tile as soon as every gate/up tile of its rows is in
 *       memory (per-tile readiness counters).  Backward: down dgrad, gate/up
 *       dgrad (started per M tile the same way), the weight gradients, the slot
 *       and router gradients and the dx sum.  No memset or other launch precedes
 *       either.
 *   MOK_SCHEDULE_SPLIT  one launch per step in stream order (router split,
 *       router GEMM, select, three dispatch kernels, [MXFP8: quantise x], gate/up,
 *       down, combine) after a memset of the tile counters; the backward the same.
 *   MOK_SCHEDULE_SPLIT_PDL  the split launches with programmatic dependent
 *       launch: each launch's CTAs are placed as soon as the previous launch's
 *       CTAs leave their SMs and wait on the device for its completion (the
 *       kernel-boundary alternative to one fused kernel that "Megakernels are
 *       dead and back…", the case against megakernels, argues for).
 * All schedules give byte-identical results.
 */
#define MOK_SCHEDULE_PERSISTENT 0
#define MOK_SCHEDULE_SPLIT 1
#define MOK_SCHEDULE_SPLIT_PDL 2
int moe_set_schedule(int schedule);
int moe_get_schedule(int *schedule);

/*
 * Device-side phase stamps of the persistent passes (per host thread).  When
 * buf (bwd_buf) -- device memory of at least MOK_TRACE_POINTS * SMs * 8 bytes --
 * is set, every later persistent forward (backward) writes, for each point p
 * and CTA b, the globaltimer value (ns) at buf[p * SMs + b].  Forward points:
 * p = 0 start, then the end of the zeroing / router-split / quantisation
 * phase, the router GEMM, the top-k, the dispatch, the gate/up GEMM, the down
 * GEMM and the combine; p = 8 repeats the end.  Backward points: p = 0 start,
 * then the end of the zeroing, of the two dgrads, of the down weight gradient,
 * of the gate/up weight gradient, of the slot gradients, of the router partial
 * sums, of dx, and of the router-gradient reduction.  NULL stops the stamps.
 */
#define MOK_TRACE_POINTS 9
int moe_trace_device(void *buf, size_t bytes, void *bwd_buf, size_t bwd_bytes);

/*
 * Number of CUDA kernels launched by the last moe_fwd / moe_bwd (or their
 * _host / _static variants) called on this host thread; 0 before the first.
 * The count depends on the configuration (dtype, whether I is a multiple of
 * 256) but not on the data.  Returns MOK_ERR_INVALID for a NULL `count`.
 */
int moe_launch_count(int *count);

/*
 * Fault-injection hook for testing the bounded waits.  While enabled (non-zero),
 * every BF16 forward launched by this host thread makes CTA 0 of the gate/up
 * GEMM and CTA 0 of the down GEMM skip the signal that hands their first
 * accumulator to the epilogue, and every backward does the same in its down
 * dgrad GEMM; each epilogue's wait then runs out after about 2 s (and, in a
 * persistent pass, so do the readiness waits of the tiles that need the missing
 * one), the kernel records MOK_STATUS_TIMEOUT and returns (no trap, no fault).
 * Results of such a call are meaningless.  Off by default.
 */
int moe_test_drop_signal(int enable);

/* Synchronise `stream`, then read and clear the device status word of the
 * current device (MOK_STATUS_* bits) into *device_status. */
int moe_status(void *stream, int32_t *device_status);

/* Static message for an error code. */
const char *moe_strerror(int code);

/* Description of the last failure of a call made by this host thread (which
 * CUDA call failed and the CUDA error string); "" if none.  Valid until the
 * thread's next failing call. */
const char *moe_last_error(void);

/* ---- expert parallelism ------------------------------------------------------
 * "Cursor åpner megakernelen…" (the pull-versus-push paragraph) and
 * "Megakernels are dead and back…" ("Números de MoK"): experts are spread over
 * `world` ranks (one GPU each); the rank that owns an expert pulls the token
 * rows routed to it from the ranks that hold them and pushes every expert
 * output row back to its token's rank, where the fixed-order k-sum runs.  The
 * backward mirrors it: the owner pulls dy rows the same way and pushes the dX
 * rows and the slot-gradient partials of each routed row back to its token's
 * rank; the weight gradients of an expert are computed whole on its owner.
 *
 * cfg describes the whole layer: E counts every routed expert and must be a
 * multiple of world (1 <= world <= MOK_EP_MAX_RANKS); T is the tokens of ONE
 * rank.  Rank r holds its own T tokens and owns the routed experts
 * [r E/world, (r+1) E/world); the router and the shared experts run on every
 * rank for its own tokens.  BF16 and MXFP8, forward and backward (an MXFP8
 * training forward or backward needs I to be a multiple of 256,
 * MOK_ERR_UNSUPPORTED otherwise).  MXFP8: each rank quantises its x in
 * moe_ep_route and the owners pull its e4m3 rows and scales (the forward's slot
 * rows are bf16); in the backward the owner pulls the bf16 dy rows and
 * quantises them itself (1x32 blocks along H depend on the row alone) and
 * decodes the pulled x codes for the gate/up weight gradient; the rank's w_*
 * are e4m3 codes with s_* scales packed for its own [E/world * 2I, H] and
 * [E/world * H, I] tensors (moe_quantize_mxfp8_weights of that slice) and, for
 * the backward, wt_* / st_* the transposed copies of the slice
 * (moe_quantize_mxfp8_weights_t).  T (top_k + n_shared) must stay below 2^24.
 *
 * Buffers (caller-allocated device memory, 16-byte aligned), from moe_ep_size:
 *   state    per rank, state_bytes: the rank's routing record and its fp32 slot
 *            rows.  Other ranks read the routing record and write slot rows.
 *   scratch  per rank, scratch_bytes: the rows the rank receives, sized for the
 *            largest possible share: the pulled token rows (x, and when training
 *            dy), one per (rank, token) with an expert here, at most world T; the
 *            expert rows (h and, when training, g/u, w h and dGU), one per
 *            (token, slot) routed here, at most world T min(top_k, E/world).
 *            A training forward's scratch is read by that rank's backward.
 *   bwd      per rank, bwd_bytes (backward only): the dX slot rows and
 *            slot-gradient partials other ranks write, and the rank's dl and
 *            router-gradient partial sums.
 *
 * A step is a sequence of phases; every rank's call of one phase must be
 * complete before any rank starts the next.  On one device (ranks emulated by
 * separate buffer sets) that is the calls in this order on one stream; on
 * several GPUs, a device-side barrier between the phases (for example a
 * one-element NCCL all-reduce on the same stream, which ends on every rank only
 * after every rank's earlier kernels).  Forward:
 *   moe_ep_route    router logits, top-k and dispatch of the rank's tokens into
 *                   its state (params: router_w, e_bias, logit_bias).
 *   moe_ep_experts  the owner's sorted rows from every rank's routing record,
 *                   the pull of those token rows into its scratch (one plain
 *                   16-byte-load copy; a token crosses the link once per owner,
 *                   whatever number of its experts that owner holds),
 *                   the gate/up GEMM with SwiGLU (training: also g/u and w h),
 *                   and the down GEMM whose epilogue stores each fp32 output row
 *                   into the slot row of the token's rank through that rank's
 *                   state pointer.  x_ranks[s] and state_ranks[s] (s < world) are
 *                   rank s's x and state as this device addresses them (its own
 *                   buffers, or peer mappings: moe_ep_ipc_*); params: w_gate_up
 *                   [E/world, 2I, H] and w_down [E/world, H, I] of the rank's
 *                   experts, ws_* of the shared experts.
 *   moe_ep_combine  y = the fixed-order sum of the rank's slot rows.
 * Backward (after a forward with training != 0 on the same buffers):
 *   moe_ep_bwd_experts  the owner pulls the dy rows of its rows from dy_ranks[s],
 *                   runs the down dgrad (SwiGLU backward) and pushes each routed
 *                   row's slot-gradient partials into bwd_ranks[s], runs the
 *                   gate/up dgrad whose epilogue stores each fp32 dX row into the
 *                   dX slot row of the token's rank, and the weight gradients:
 *                   grads->dw_gate_up [E/world, 2I, H] and dw_down [E/world, H, I]
 *                   of its experts (over every rank's rows), dws_* the shared
 *                   experts' gradient over this rank's tokens.
 *   moe_ep_bwd_combine  slot gradients, grads->drouter_w (over this rank's
 *                   tokens) and grads->dx of the rank's tokens.
 * Each rank's y and dx equal moe_fwd / moe_bwd of its T tokens with all E
 * experts, byte for byte, and so do its drouter_w and dws_* (the router and the
 * shared experts are replicated: their full gradients are the sums over ranks,
 * as for data-parallel replicas).  An owner's dw_* equal moe_bwd's rows of its
 * experts on the concatenation of every rank's tokens when that batch routes its
 * tokens the same way.  A routing record that would overflow the receive
 * buffers (impossible for one written by moe_ep_route) records
 * MOK_STATUS_BAD_INDEX and is treated as empty.  The same buffers must not be
 * used by two steps at once.
 */
#define MOK_EP_MAX_RANKS 8
#define MOK_EP_IPC_HANDLE_BYTES 64
int moe_ep_size(const moe_cfg *cfg, int32_t world, int32_t training, size_t *state_bytes, size_t *scratch_bytes,
                size_t *bwd_bytes);
int moe_ep_route(const moe_cfg *cfg, int32_t world, int32_t rank, const void *x, const moe_params *params,
                 void *state, size_t state_bytes, void *stream);
int moe_ep_experts(const moe_cfg *cfg, int32_t world, int32_t rank, int32_t training, const void *const *x_ranks,
                   void *const *state_ranks, const moe_params *params, void *scratch, size_t scratch_bytes,
                   void *stream);
int moe_ep_combine(const moe_cfg *cfg, int32_t world, int32_t rank, const void *state, void *y, void *stream);
int moe_ep_bwd_experts(const moe_cfg *cfg, int32_t world, int32_t rank, const void *const *dy_ranks,
                       void *const *bwd_ranks, const moe_params *params, const moe_grads *grads, void *scratch,
                       size_t scratch_bytes, void *stream);
int moe_ep_bwd_combine(const moe_cfg *cfg, int32_t world, int32_t rank, const void *x, const moe_params *params,
                       const void *state, void *bwd, size_t bwd_bytes, const moe_grads *grads, void *stream);

/* Peer mappings for moe_ep_experts across processes on one node.
 * moe_ep_ipc_handle writes into `handle` (MOK_EP_IPC_HANDLE_BYTES bytes) the
 * CUDA IPC handle of the device allocation that contains dev_ptr
 * (cudaIpcGetMemHandle of its base) and into *offset dev_ptr's byte offset in
 * it.  Another process maps it with moe_ep_ipc_open (cudaIpcOpenMemHandle with
 * peer access enabled lazily; *dev_ptr = mapped base + offset) and unmaps it
 * with moe_ep_ipc_close(the pointer open returned, the same offset).  A
 * process opens one allocation once: map every pointer of one allocation from
 * the first mapping.  MOK_ERR_INVALID for NULL arguments or a pointer that is
 * not device memory, MOK_ERR_LAUNCH when the CUDA call fails (moe_last_error
 * names it). */
int moe_ep_ipc_handle(const void *dev_ptr, void *handle, size_t *offset);
int moe_ep_ipc_open(const void *handle, size_t offset, void **dev_ptr);
int moe_ep_ipc_close(void *dev_ptr, size_t offset);

#ifdef __cplusplus
}
#endif
#endif /* MOK_H */
