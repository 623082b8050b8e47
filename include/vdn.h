/*
 * vdn.h -- C ABI of libvdn: the forward pass of the VDN-H3 bidirectional
 * linear-attention branch on one NVIDIA B200 (sm_100a).
 *
 * Source of the method: "VDN-Minimax-H3 bidirectional linear branch in five
 * steps" (icman.com.cn/news/81972), sections "Step 1" .. "Step 5" and "text
 * state".  The page printed its formulas with every '+' and '=' lost; the
 * restored forms used throughout are
 *     A_f = sum_s beta_s k'_s k'_s^T          B_f = sum_s beta_s v'_s k'_s^T
 *     vdn_solve    S_out = (S_in D_f + B_f)(I + A_f)^-1
 *     vdn_scaled   S_out = (S_in D_f + c B_f)(I + c^2 A_f)^-1
 *     sana_scaled  S_out = (S_in D_f)(I - c^2 A_f) + c B_f
 * with D_f = diag(alpha_f) (per key channel) and the state S a d_v x d_k map
 * read out as o = S q'.
 *
 * Conventions shared by every entry point
 *   - All tensor pointers are DEVICE pointers owned by the caller; the library
 *     never allocates device memory, so calls on different streams with
 *     different workspaces may run concurrently.  Its one piece of global state
 *     is the fixed device array behind vdn_branch_forward_static (the scratch
 *     of that entry point alone); no other entry point touches it.
 *   - Every tensor is dense and contiguous in the layout given beside it, with
 *     a 16-byte aligned base address (VDN_ERR_ALIGNMENT otherwise).
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = the legacy
 *     default stream).  Argument errors are reported before any launch; a
 *     failed launch returns VDN_ERR_CUDA.  Errors during device execution
 *     surface at the caller's next synchronisation.
 *   - Element types: q, k, v, gate and out share `shape->dtype` (fp32 or
 *     bf16); beta, alpha, rms_w, the conv taps and the text state are fp32.
 *     State and accumulation are fp32 in every configuration.
 *   - Input domains (not checked, the values live on the device): beta >= 0
 *     and alpha in (0, 1], as the sigmoids of "Step 2" and "Step 3" produce
 *     them.  The tensor-core path scales both statistics operands by
 *     sqrt(beta) (a negative beta gives NaN there) and inverts I + c^2 A by
 *     elimination without pivoting, which needs I + c^2 A symmetric positive
 *     definite; beta >= 0 guarantees that.  alpha above 1 makes the states
 *     grow and is kept in range only by the block exponents of the scans.
 */
#ifndef VDN_H
#define VDN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    VDN_OK = 0,
    VDN_ERR_INVALID_ARG = 1,   /* NULL pointer, non-positive size, bad enum, out/in overlap */
    VDN_ERR_UNSUPPORTED = 2,   /* d not in {16,128}, conv_width not in {1,3}, bf16 with d != 128 */
    VDN_ERR_ALIGNMENT = 3,     /* a tensor base not 16-byte aligned (workspace: 256-byte) */
    VDN_ERR_WORKSPACE = 4,     /* workspace smaller than vdn_branch_workspace_size() */
    VDN_ERR_CUDA = 5,          /* a CUDA runtime / driver call or a launch failed */
    VDN_ERR_TIMEOUT = 6        /* a bounded device-side wait expired (device status word) */
} vdn_status;

/* Update rule of the per-frame recurrence (page section "Step 3", rules table). */
typedef enum {
    VDN_RULE_SANA_SCALED = 0,  /* (S D)(I - c^2 A) + c B : first-order truncation          */
    VDN_RULE_VDN_SOLVE = 1,    /* (S D + B)(I + A)^-1    : exact solve, the released rule  */
    VDN_RULE_VDN_SCALED = 2,   /* (S D + c B)(I + c^2 A)^-1 : scaled exact solve           */
    VDN_RULE_ADDITIVE = 3      /* S D + B (A taken as 0) : test rule, not on the page      */
} vdn_rule;

typedef enum { VDN_DTYPE_F32 = 0, VDN_DTYPE_BF16 = 1 } vdn_dtype;

/* Implementation selector of the debug entry point.  AUTO picks the tensor-core
 * path for bf16 with d == 128 and the SIMT path otherwise. */
typedef enum { VDN_IMPL_AUTO = 0, VDN_IMPL_SIMT = 1, VDN_IMPL_TC = 2 } vdn_impl;

/* Problem sizes.  N = F * S tokens per batch element, token n = f * S + s
 * belongs to latent frame f.  d is the head dimension (d_k = d_v = d). */
typedef struct {
    int B;           /* batch                                  >= 1 */
    int H;           /* heads                                  >= 1 */
    int F;           /* latent frames                          >= 1 */
    int S;           /* tokens per latent frame                >= 1 */
    int d;           /* head dimension: 16 or 128                    */
    int conv_width;  /* taps of the k/v short conv: 1 or 3           */
    int dtype;       /* vdn_dtype of q, k, v, gate, out              */
} vdn_shape;

/* Bytes of device workspace that vdn_branch_forward needs for `shape` and
 * `rule` (0 if the arguments are invalid).  The caller allocates it (256-byte
 * aligned) and may reuse it across calls that do not overlap in time. */
size_t vdn_branch_workspace_size(const vdn_shape* shape, int rule);

/* Same, for an explicit implementation (VDN_IMPL_*), as the debug entry point needs. */
size_t vdn_branch_workspace_size_impl(const vdn_shape* shape, int rule, int impl);

/*
 * vdn_branch_forward -- the whole branch, page sections "Step 1" to "Step 5".
 *
 *   q, k, v    [B, F*S, H, d] dtype   pre-RoPE ("NoPE") features, token-major
 *   beta       [B, F*S, H]    fp32    per-token, per-head write strength (post-sigmoid, >= 0)
 *   alpha      [B, F, H, d]   fp32    per-frame, per-channel forget gate in (0, 1]
 *   gate       [B, F*S, H, d] dtype   output gate values (post-sigmoid)
 *   rms_w      [d]            fp32    RMSNorm weight (shared by the heads)
 *   conv_k_w   [H, d, conv_width] fp32  depthwise taps of the k short conv, or NULL (identity)
 *   conv_v_w   [H, d, conv_width] fp32  same for v, or NULL
 *   text_state [H, d, d]      fp32    per-head text state T (v x k, row-major), or
 *                                     NULL: both scans then start from zero.  Each
 *                                     scan starts from 0.5 * T (TEXT_STATE_SCALE).
 *   rule, c    vdn_rule and its scale c (ignored by VDN_SOLVE and ADDITIVE)
 *   chunk      softmax-window chunk in frames (>= 1); the page's value is 5
 *   radius     chunks added on each side of the query's chunk (>= 0); page: 1
 *   workspace  device scratch of at least vdn_branch_workspace_size() bytes
 *   out        [B, F*S, H, d] dtype   branch output (RMSNorm-ed and gated); must not
 *                                     overlap any input
 *
 * Step 1: k, v -> depthwise conv along each frame's token order (centred, zero
 * padding at the frame edges), SiLU on q, k, v, then L2 normalisation of q, k.
 * Step 2: per (batch, head, frame) the statistics A_f and B_f.
 * Step 3-4: the forward prefix scan P_f and backward suffix scan Q_f of the rule.
 * Step 4: query frame t with window [lo, hi] (vdn_window_bounds) reads
 *         W_t = P_{lo-1} diag(prod_{f=lo..t} alpha_f) + Q_{hi+1} diag(prod_{f=t..hi} alpha_f),
 *         where P_{-1} = Q_F = 0.5 * T (the decayed prompt at a clip edge).
 * Step 5: out = RMSNorm(W_t q') * gate, RMSNorm over d with eps 1e-6.
 */
vdn_status vdn_branch_forward(const vdn_shape* shape,
                              const void* q, const void* k, const void* v,
                              const float* beta, const float* alpha,
                              const void* gate, const float* rms_w,
                              const float* conv_k_w, const float* conv_v_w,
                              const float* text_state,
                              int rule, float c, int chunk, int radius,
                              void* workspace, size_t workspace_bytes,
                              void* out, void* stream);

/* Intermediates for per-stage checks.  Every non-NULL pointer receives an fp32
 * device array [B, H, F, d, d] (row-major d x d per frame):
 *   A, B : frame statistics of "Step 2";
 *   N    : per-frame operator of "Step 3": (I + c^2 A)^-1 (vdn rules),
 *          I - c^2 A (sana_scaled) or I (additive);
 *   P, Q : prefix state after absorbing frames 0..f and suffix state after
 *          absorbing frames f..F-1 ("Step 4");
 *   W    : gathered, bridged state of query frame f ("Step 4"). */
typedef struct {
    int impl;        /* vdn_impl */
    float* A;
    float* B;
    float* N;
    float* P;
    float* Q;
    float* W;
} vdn_debug_out;

/* vdn_branch_forward plus the intermediates requested in `dbg` (which may be
 * NULL).  Uses the workspace size of vdn_branch_workspace_size_impl(dbg->impl).
 * Not meant for timed runs: exporting intermediates adds device work. */
vdn_status vdn_branch_forward_debug(const vdn_shape* shape,
                                    const void* q, const void* k, const void* v,
                                    const float* beta, const float* alpha,
                                    const void* gate, const float* rms_w,
                                    const float* conv_k_w, const float* conv_v_w,
                                    const float* text_state,
                                    int rule, float c, int chunk, int radius,
                                    void* workspace, size_t workspace_bytes,
                                    void* out, void* stream,
                                    const vdn_debug_out* dbg);

/* Number of kernels one vdn_branch_forward call launches for `shape` with the
 * given implementation (VDN_IMPL_*): 5 on the tensor-core path (frame
 * statistics, per-frame solve, scan, gather + bridge, read-out), 6 on the SIMT
 * path (feature prep, statistics, solve, scan, gather, read-out); 0 if invalid. */
int vdn_branch_launch_count(const vdn_shape* shape, int impl);

/* vdn_branch_forward that also records caller-created CUDA events (cudaEvent_t
 * handles, timing enabled) on `stream`: events[0] before the first kernel and
 * events[i] right after kernel i, i = 1..vdn_branch_launch_count().  It adds
 * no device work; n_events must be at least launch_count + 1.  For per-kernel
 * timing by the caller (cudaEventElapsedTime between consecutive events). */
vdn_status vdn_branch_forward_timed(const vdn_shape* shape,
                                    const void* q, const void* k, const void* v,
                                    const float* beta, const float* alpha,
                                    const void* gate, const float* rms_w,
                                    const float* conv_k_w, const float* conv_v_w,
                                    const float* text_state,
                                    int rule, float c, int chunk, int radius,
                                    void* workspace, size_t workspace_bytes,
                                    void* out, void* stream,
                                    void* const* events, int n_events);

/* vdn_branch_forward without a caller workspace (the page has no counterpart:
 * this is a deployment variant).  For callers that cannot allocate device
 * memory where they run the branch -- code running while a stream is captured
 * into a CUDA graph, where cudaMalloc is refused, or runtimes whose device
 * memory belongs to a framework allocator or a fixed arena -- the scratch lives
 * in one library-owned device array of 64 MiB, which every GPU that loads the
 * library holds until the process exits.  Problems whose workspace
 * (vdn_branch_workspace_size) exceeds 64 MiB are refused with VDN_ERR_WORKSPACE
 * before any CUDA call.  Inputs, output and errors are those of
 * vdn_branch_forward.  The first call on a device looks up the array's device
 * address (cudaGetSymbolAddress, which may load the library's device code), so
 * make that first call before any stream capture.  All calls share the array
 * and it keeps the last call's contents: calls that overlap on the GPU (other
 * streams, other threads) race and must be serialised by the caller.  Calls no
 * cudaMalloc, cudaFree or allocating library routine. */
vdn_status vdn_branch_forward_static(const vdn_shape* shape,
                                     const void* q, const void* k, const void* v,
                                     const float* beta, const float* alpha,
                                     const void* gate, const float* rms_w,
                                     const float* conv_k_w, const float* conv_v_w,
                                     const float* text_state,
                                     int rule, float c, int chunk, int radius,
                                     void* out, void* stream);

/* "Step 1" alone (page: NoPE features): q' = L2(SiLU(q)), k' = L2(SiLU(conv_k(k))),
 * v' = SiLU(conv_v(v)), all [B, F*S, H, d] in shape->dtype.  Outputs must not
 * overlap the inputs.  Needs no workspace. */
vdn_status vdn_feature_prep(const vdn_shape* shape,
                            const void* q, const void* k, const void* v,
                            const float* conv_k_w, const float* conv_v_w,
                            void* q_out, void* k_out, void* v_out, void* stream);

/* Chunk-aligned softmax window of query frame t (page: "what is the far
 * field", chunk 5 / radius 1): c = t / chunk, lo = max(0, chunk (c - radius)),
 * hi = min(F - 1, chunk (c + radius + 1) - 1).  Host function, no CUDA calls. */
vdn_status vdn_window_bounds(int t, int F, int chunk, int radius, int* lo, int* hi);

/* Windowed softmax branch of the hybrid attention layer (page: the window
 * softmax sees the frames near the query, the linear branch the far field, and
 * the layer adds the two branches).  Every query token of frame t attends to
 * all tokens of frames lo..hi = vdn_window_bounds(t):
 *   o = softmax(q_rope k_rope^T * scale) v     (per batch and head, over d)
 * q_rope, k_rope: the RoPE-rotated q and k of the softmax branch (the rotation
 * is the caller's), v the shared values, all [B, F*S, H, d] in shape->dtype;
 * scale <= 0 selects 1/sqrt(d).  accumulate = 0 writes o to out, 1 adds it to
 * out (which then holds, e.g., the linear branch's output).  out must not
 * overlap the inputs.  workspace: at least vdn_window_softmax_workspace_size()
 * bytes (the device status word of the bounded waits), 256-byte aligned;
 * shape->conv_width is not used.  Asynchronous on `stream`. */
size_t vdn_window_softmax_workspace_size(const vdn_shape* shape);
vdn_status vdn_window_softmax_forward(const vdn_shape* shape,
                                      const void* q_rope, const void* k_rope, const void* v,
                                      int chunk, int radius, float scale, int accumulate,
                                      void* workspace, size_t workspace_bytes,
                                      void* out, void* stream);

/* The hybrid attention layer: out = windowed softmax branch (q_rope, k_rope,
 * v) + bidirectional linear branch (q, k, v, ... as vdn_branch_forward, whose
 * workspace this takes).  scale as above. */
vdn_status vdn_hybrid_forward(const vdn_shape* shape,
                              const void* q_rope, const void* k_rope,
                              const void* q, const void* k, const void* v,
                              const float* beta, const float* alpha,
                              const void* gate, const float* rms_w,
                              const float* conv_k_w, const float* conv_v_w,
                              const float* text_state,
                              int rule, float c, int chunk, int radius, float scale,
                              void* workspace, size_t workspace_bytes,
                              void* out, void* stream);

/* Bytes of device workspace that vdn_branch_backward needs (0 if invalid). */
size_t vdn_branch_backward_workspace_size(const vdn_shape* shape, int rule);

/*
 * vdn_branch_backward -- gradients of the branch (vdn_branch_forward, same
 * arguments) for an upstream gradient `dout` = dL/d out, [B, F*S, H, d] dtype.
 * The page trains the branch (stages A1/A2 of "VDN-Minimax-H3 bidirectional
 * linear branch in five steps") without printing a backward; this is the exact
 * gradient of the five steps and of the text-state seeds, in reverse order:
 * read-out and RMSNorm, gather and bridge, both scans (adjoint recurrences
 * through N_f), frame statistics, L2 norm, SiLU and the short conv.
 *
 * Outputs (written, not accumulated; caller-owned device memory):
 *   dq, dk, dv, dgate   [B, F*S, H, d] dtype
 *   dbeta               [B, F*S, H]    fp32
 *   dalpha              [B, F, H, d]   fp32
 *   drms_w              [d]            fp32  (summed over batch and heads)
 *   dconv_k_w, dconv_v_w [H, d, conv_width] fp32 (summed over the batch); NULL
 *                       exactly when the matching taps are NULL
 *   dtext_state         [H, d, d]      fp32 (summed over the batch); NULL exactly
 *                       when text_state is NULL
 * The forward runs first, inside the call (its per-frame statistics, operators and
 * states are kept in the workspace); then the reversed steps: on the tensor cores
 * for bf16 at d = 128 (read-out, frame statistics and the adjoint scans; fp32
 * accumulation), in fp32 SIMT kernels otherwise (fp32 inputs, d = 16).  No
 * output may overlap another output, an input or the workspace.  Rules whose
 * states leave the fp32 range (divergent sana_scaled settings) give non-finite
 * gradients.  Errors: as vdn_branch_forward, plus VDN_ERR_INVALID_ARG for a
 * missing or overlapping gradient buffer.  The device status word (first word
 * of the workspace) records an expired bounded wait of the forward recompute or
 * of a tensor-core backward kernel (vdn_workspace_status reads it).
 */
vdn_status vdn_branch_backward(const vdn_shape* shape,
                               const void* q, const void* k, const void* v,
                               const float* beta, const float* alpha,
                               const void* gate, const float* rms_w,
                               const float* conv_k_w, const float* conv_v_w,
                               const float* text_state,
                               int rule, float c, int chunk, int radius,
                               const void* dout,
                               void* workspace, size_t workspace_bytes,
                               void* dq, void* dk, void* dv,
                               float* dbeta, float* dalpha, void* dgate, float* drms_w,
                               float* dconv_k_w, float* dconv_v_w, float* dtext_state,
                               void* stream);

/* Save-for-backward (a training step: forward, then backward from the forward's state).
 * vdn_branch_forward_train is vdn_branch_forward (same output) that also keeps, in the
 * caller's `saved` buffer of vdn_branch_saved_size() bytes (256-byte aligned), the per-frame
 * state the backward reads: A_f, B_f, N_f, P_f, Q_f, W_t in fp32 and, on the tensor-core
 * path, the operand images of N_f.  vdn_branch_backward_saved is vdn_branch_backward without
 * the forward recompute: same inputs (which must be those the saved state was made from),
 * the saved buffer (read only), a workspace of vdn_branch_backward_saved_workspace_size()
 * bytes whose first word is its device status word.  Errors as vdn_branch_forward and
 * vdn_branch_backward, plus VDN_ERR_WORKSPACE for a short saved buffer and
 * VDN_ERR_INVALID_ARG when it overlaps an input, an output or the workspace. */
size_t vdn_branch_saved_size(const vdn_shape* shape);
size_t vdn_branch_backward_saved_workspace_size(const vdn_shape* shape, int rule);
vdn_status vdn_branch_forward_train(const vdn_shape* shape,
                                    const void* q, const void* k, const void* v,
                                    const float* beta, const float* alpha,
                                    const void* gate, const float* rms_w,
                                    const float* conv_k_w, const float* conv_v_w,
                                    const float* text_state,
                                    int rule, float c, int chunk, int radius,
                                    void* workspace, size_t workspace_bytes,
                                    void* out, void* saved, size_t saved_bytes, void* stream);
vdn_status vdn_branch_backward_saved(const vdn_shape* shape,
                                     const void* q, const void* k, const void* v,
                                     const float* beta, const float* alpha,
                                     const void* gate, const float* rms_w,
                                     const float* conv_k_w, const float* conv_v_w,
                                     const float* text_state,
                                     int rule, float c, int chunk, int radius,
                                     const void* dout, const void* saved, size_t saved_bytes,
                                     void* workspace, size_t workspace_bytes,
                                     void* dq, void* dk, void* dv,
                                     float* dbeta, float* dalpha, void* dgate, float* drms_w,
                                     float* dconv_k_w, float* dconv_v_w, float* dtext_state,
                                     void* stream);

/* vdn_branch_backward that also records caller-created CUDA events on `stream`:
 * events[0] before the forward recompute, events[1] after it, then events[2..7]
 * after each backward stage (read-out with its per-frame slot sums, gather and
 * bridge, adjoint scans with their per-frame gradients, frame statistics, conv,
 * reductions).  n_events must be at least 8. */
vdn_status vdn_branch_backward_timed(const vdn_shape* shape,
                                     const void* q, const void* k, const void* v,
                                     const float* beta, const float* alpha,
                                     const void* gate, const float* rms_w,
                                     const float* conv_k_w, const float* conv_v_w,
                                     const float* text_state,
                                     int rule, float c, int chunk, int radius,
                                     const void* dout,
                                     void* workspace, size_t workspace_bytes,
                                     void* dq, void* dk, void* dv,
                                     float* dbeta, float* dalpha, void* dgate, float* drms_w,
                                     float* dconv_k_w, float* dconv_v_w, float* dtext_state,
                                     void* stream, void* const* events, int n_events);

/*
 * Frame sharding -- the branch of one clip split by frames across `world` ranks
 * (one process per GPU), page sections "Step 3" and "Step 4".
 *
 * Rank r owns a contiguous run of whole chunks of the F_total-frame clip
 * (vdn_frame_range: the C = ceil(F_total / chunk) chunks split into `world`
 * runs, the first C % world ranks taking one more; world <= C).  Its inputs are
 * its own frames: q, k, v, gate [B, F*S, H, d] and beta [B, F*S, H] for those
 * F = f1 - f0 frames, `shape` describing them (shape->F = F), alpha [B, F, H, d]
 * of its frames for the first phase and of the whole clip for the second.
 *
 * Every rule's frame step is affine in the state, S_out = S_in G_f + B'_f.
 * Phase 1, vdn_frames_maps: features, statistics and solves of the rank's frames,
 * then for each of its chunks and both scan directions the chunk's composed map
 * S -> S G_c + O_c, written to `maps` (vdn_frames_map_bytes bytes):
 *     [B*H][2 directions][nch][G_c | O_c][d][d] fp32, nch = ceil(C / world),
 *     then [B*H][2 directions][nch][G_c | O_c] int32 exponents e: the map is
 *     2^e times the stored matrix (sana_scaled can grow the state past fp32
 *     range over a clip; the maps and the fold carry power-of-two exponents);
 *     slots past the rank's own chunks are unused, the size is padded to 16 bytes.
 * The caller then concatenates every rank's buffer in rank order (an all-gather)
 * into maps_all [world][vdn_frames_map_bytes / 4].
 * Phase 2, vdn_frames_finish: folds the maps from 0.5 * text_state into the
 * clip's chunk-edge states (P at chunk ends, Q at chunk starts), gathers the
 * windows of the rank's query frames and writes their read-out to out
 * [B, F*S, H, d].  The result equals vdn_branch_forward's rows of those frames
 * up to rounding.
 *
 * Supported: bf16, d = 128 (the tensor-core path), chunk <= 16; otherwise
 * VDN_ERR_UNSUPPORTED.  A partition that does not match shape->F, world > C or a
 * rank outside [0, world) is VDN_ERR_INVALID_ARG.  Both phases take one
 * workspace of vdn_frames_workspace_size bytes (256-byte aligned; it may be the
 * same buffer).  vdn_frames_maps clears the workspace's device status word and
 * vdn_frames_finish does not: given the same workspace, vdn_workspace_status
 * after phase 2 reports an expired wait of either phase; a separate phase-2
 * workspace needs its first 4 bytes zeroed by the caller.  Pointers as in
 * vdn_branch_forward: 16-byte aligned device
 * memory owned by the caller; out and maps must not overlap any other argument.
 * Work is queued on `stream`; errors are returned before any launch.
 */
vdn_status vdn_frame_range(int F_total, int world, int rank, int chunk, int* f0, int* f1);
/* the rank that owns frame `frame` (0 <= frame < F_total) under the same partition */
vdn_status vdn_frame_owner(int F_total, int world, int chunk, int frame, int* rank);
size_t vdn_frames_map_bytes(const vdn_shape* shape, int F_total, int world, int rank, int chunk);
size_t vdn_frames_workspace_size(const vdn_shape* shape, int F_total, int world, int rank, int rule, int chunk);
vdn_status vdn_frames_maps(const vdn_shape* shape, int F_total, int world, int rank,
                           const void* k, const void* v, const float* beta, const float* alpha,
                           const float* conv_k_w, const float* conv_v_w,
                           int rule, float c, int chunk,
                           void* workspace, size_t workspace_bytes,
                           float* maps, size_t maps_bytes, void* stream);
vdn_status vdn_frames_finish(const vdn_shape* shape, int F_total, int world, int rank,
                             const void* q, const float* alpha_all, const void* gate, const float* rms_w,
                             const float* text_state,
                             int rule, float c, int chunk, int radius,
                             const float* maps_all, size_t maps_all_bytes,
                             void* workspace, size_t workspace_bytes,
                             void* out, void* stream);

/* Reads the device status word that bounded waits inside the kernels set (it
 * lives in the workspace of the last call): VDN_OK or VDN_ERR_TIMEOUT.
 * Synchronises `stream`.  VDN_ERR_INVALID_ARG for a NULL workspace or one of
 * fewer than 256 bytes (checked before any CUDA call); VDN_ERR_CUDA if the
 * copy or the synchronisation fails. */
vdn_status vdn_workspace_status(const void* workspace, size_t workspace_bytes, void* stream);

/* Static description of a status code. */
const char* vdn_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* VDN_H */
