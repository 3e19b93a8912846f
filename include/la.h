/*
 * la.h -- C ABI of the B200 (sm_100a) linear-attention library (libla_b200.so).
 *
 * Three operations, forward and backward, on one GPU:
 *
 *  la_bidir_*   bidirectional (non-causal) linear attention with the feature
 *               map phi = elu + 1 and the norm term:
 *                   S = sum_s phi(k_s)^T v_s,  z = sum_s phi(k_s),
 *                   o_t = phi(q_t) S / (phi(q_t) . z + eps).
 *               Source: "Flash Bi-directional Linear Attention" README
 *               (fla-org), intro ("bi-directional linear attention for
 *               non-causal modeling") and "Benchmarks" (B8-H16-D64).
 *  la_simple_*  simple_la: the same without the norm term and with the
 *               identity feature map, o_t = q_t (sum_s k_s^T v_s).
 *               Source: same README, "Update" (2024-12-28: simple_la, a
 *               simple form of linear_attn without the norm term).
 *  la_chunk_decay_*  causal linear attention with a per-head scalar decay
 *               (retention), computed chunk by chunk:
 *                   o_t = sum_{s<=t} gamma_h^(t-s) (q_t . k_s) v_s.
 *               Source: "flash-linear-attention" README (sustcsonglin),
 *               "Benchmarks" (RetNet, B8-H32-D128) and "Different forms of
 *               linear attention" (FusedChunk / ParallelChunk).
 *
 * Common conventions
 *  - Every tensor argument is a DEVICE pointer to a contiguous [B, H, T, D]
 *    row-major array (D fastest) of `dtype`, 16-byte aligned.  Outputs have
 *    the inputs' dtype.  Accumulation is fp32 throughout.
 *  - D must be 64 or 128; B, H >= 1 with B * H <= 65535; T >= 0 (T = 0 is a
 *    no-op that still zeroes `state`).  B * H * T * D must be < 2^31.
 *  - Scaling (e.g. D^-1/2 on q) is the caller's: gradients are with respect
 *    to the tensors passed.
 *  - The caller owns all memory.  `workspace` is device scratch of at least
 *    la_workspace_size(op, B, H, T, D, dtype) bytes, 256-byte aligned; its
 *    contents on entry do not matter and are clobbered.  The library
 *    allocates no device memory.
 *  - `stream` is a cudaStream_t (NULL = legacy default stream).  Calls are
 *    asynchronous: they enqueue kernels on `stream` and return; no host
 *    synchronisation.  Results are bitwise deterministic for a given
 *    (B, H, T, D, dtype): split reductions are combined in a fixed order.
 *  - Two calls may run concurrently on different streams only with
 *    different workspaces.
 *  - Errors: arguments are validated before any CUDA call, and an invalid
 *    call enqueues nothing.  LA_ERR_CUDA means a launch or runtime call
 *    failed; la_last_error() gives the text (per calling thread).
 */
#ifndef LA_B200_H
#define LA_B200_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum { LA_F32 = 0, LA_F16 = 1, LA_BF16 = 2 } la_dtype;

typedef enum {
    LA_OK = 0,
    LA_ERR_INVALID_ARG = 1,   /* null pointer, negative size, eps < 0, decay not in (0, 1] */
    LA_ERR_UNSUPPORTED = 2,   /* D not in {64, 128}, unknown dtype, too many heads for decay */
    LA_ERR_ALIGNMENT = 3,     /* a tensor or workspace pointer is not suitably aligned */
    LA_ERR_WORKSPACE = 4,     /* workspace NULL or smaller than la_workspace_size() */
    LA_ERR_CUDA = 5,          /* a CUDA runtime call or kernel launch failed */
    LA_ERR_TIMEOUT = 6        /* a kernel gave up waiting on the GPU (see la_device_check) */
} la_status;

typedef enum {
    LA_OP_BIDIR_FWD = 0,
    LA_OP_BIDIR_BWD = 1,
    LA_OP_SIMPLE_FWD = 2,
    LA_OP_SIMPLE_BWD = 3,
    LA_OP_CHUNK_DECAY_FWD = 4,
    LA_OP_CHUNK_DECAY_BWD = 5,
    LA_OP_STATE_REDUCE = 6,
    LA_OP_STATE_APPLY = 7,
    LA_OP_STATE_BWD_Q = 8,
    LA_OP_STATE_BWD_KV = 9,
    LA_OP_CAUSAL_NORM_FWD = 10,
    LA_OP_CAUSAL_NORM_BWD = 11,
    LA_OP_GATED_FWD = 12,
    LA_OP_GATED_BWD = 13
} la_op;

/* Feature map of the state-form stages and of la_causal_norm_*: elu+1 with the
 * norm term (the la_bidir_* op), the identity without it (the la_simple_* op), or
 * the identity with the norm term (LA_FEATURE_NORM: features f(q), f(k) computed
 * by the caller, e.g. the focusing function or the polarity split of
 * la_feature_map_fwd, then attended with the norm term; dq, dk are then the
 * gradients with respect to those features).  la_causal_norm_* take
 * LA_FEATURE_ELU1 or LA_FEATURE_IDENTITY (the norm term is always on there). */
typedef enum { LA_FEATURE_IDENTITY = 0, LA_FEATURE_ELU1 = 1, LA_FEATURE_NORM = 2 } la_feature;

/* Largest H accepted by la_chunk_decay_* (the decays travel as kernel arguments). */
#define LA_MAX_DECAY_HEADS 512

/* Most segments la_chunk_decay_scan combines in one call. */
#define LA_MAX_SCAN_SEGMENTS 128

/* Bytes of device workspace the call `op` needs for this shape (0 if none).
 * Depends only on its arguments.  Returns 0 for invalid arguments too. */
size_t la_workspace_size(la_op op, int B, int H, int T, int D, la_dtype dtype);

/* Bidirectional linear attention, forward.
 *  q, k, v  in  [B,H,T,D] dtype
 *  o        out [B,H,T,D] dtype:  o_t = phi(q_t) S / (phi(q_t) . z + eps)
 *  state    out [B,H,D,D+1] fp32, or NULL: row i = (S[i][0..D-1], z[i]).
 *           Pass it to la_bidir_bwd to skip recomputing S and z.
 *  eps      >= 0, added to the denominator only.                           */
la_status la_bidir_fwd(const void *q, const void *k, const void *v, void *o, float *state,
                       int B, int H, int T, int D, la_dtype dtype, float eps,
                       void *workspace, size_t workspace_bytes, void *stream);

/* Size of the scratch array built into the library for la_bidir_fwd_static (32 MiB). */
#define LA_STATIC_SCRATCH_BYTES (32u << 20)

/* LA_STATIC_SCRATCH_BYTES as the built library has it (for bindings that do not
 * read this header). */
size_t la_static_scratch_bytes(void);

/* la_bidir_fwd without a workspace argument, for callers that cannot allocate
 * device memory: code inside a host framework that owns the CUDA allocator and
 * only hands out the tensors it manages, plugins in a serving process, or
 * runtimes that may not call cudaMalloc after start-up.  (The pages describe no
 * such entry point; it has no counterpart there.)
 *  Arguments and results are those of la_bidir_fwd.  The scratch comes from a
 *  LA_STATIC_SCRATCH_BYTES device array inside the library, which every GPU that
 *  loads the library holds until the process exits.  This call allocates
 *  nothing.
 *  - Shapes whose la_workspace_size(LA_OP_BIDIR_FWD, ...) exceeds
 *    LA_STATIC_SCRATCH_BYTES return LA_ERR_WORKSPACE (see la_last_error()).
 *  - The first call on each device looks up the array's device address on that
 *    device (the current one), and so does the first call after the current
 *    CUDA context changed (cudaDeviceReset, a re-created primary context, a
 *    driver-API context made current): the address is kept per device with the
 *    id of the context it belongs to.  Make that first call before any stream
 *    capture: during a capture it returns LA_ERR_INVALID_ARG.  Calls whose
 *    shape or dtype is invalid look nothing up (la_bidir_fwd reports them).
 *  - All calls share the array and it keeps the last call's contents; calls
 *    that overlap on the GPU (unordered streams or host threads) race on it.
 *    Nothing needs clearing between calls.                                    */
la_status la_bidir_fwd_static(const void *q, const void *k, const void *v, void *o, float *state,
                              int B, int H, int T, int D, la_dtype dtype, float eps, void *stream);

/* Bidirectional linear attention, backward.
 *  dout     in  [B,H,T,D]: gradient of the loss with respect to o
 *  state    in  [B,H,D,D+1] fp32 from la_bidir_fwd with the same q,k,v, or
 *           NULL to recompute it
 *  dq,dk,dv out [B,H,T,D] dtype: gradients with respect to q, k, v.
 * With n_t = phi(q_t).z + eps and o_t as in the forward:
 *  dS = sum_t phi(q_t)^T dout_t / n_t,   dz = -sum_t phi(q_t) (dout_t . o_t) / n_t
 *  dq_t = (dout_t S^T - (dout_t . o_t) z) / n_t * phi'(q_t)
 *  dk_s = (v_s dS^T + dz) * phi'(k_s),   dv_s = phi(k_s) dS                    */
la_status la_bidir_bwd(const void *q, const void *k, const void *v, const void *dout,
                       const float *state, void *dq, void *dk, void *dv,
                       int B, int H, int T, int D, la_dtype dtype, float eps,
                       void *workspace, size_t workspace_bytes, void *stream);

/* simple_la forward: o_t = q_t S with S = sum_s k_s^T v_s.
 *  state    out [B,H,D,D+1] fp32 or NULL (column D is written as 0).         */
la_status la_simple_fwd(const void *q, const void *k, const void *v, void *o, float *state,
                        int B, int H, int T, int D, la_dtype dtype,
                        void *workspace, size_t workspace_bytes, void *stream);

/* simple_la backward: dq_t = dout_t S^T, dS = sum_t q_t^T dout_t,
 *  dk_s = v_s dS^T, dv_s = k_s dS.   state as for la_bidir_bwd (or NULL).    */
la_status la_simple_bwd(const void *q, const void *k, const void *v, const void *dout,
                        const float *state, void *dq, void *dk, void *dv,
                        int B, int H, int T, int D, la_dtype dtype,
                        void *workspace, size_t workspace_bytes, void *stream);

/* Causal linear attention with per-head decay (retention), forward.
 *  decay    HOST pointer to H floats, gamma_h in (0, 1]; read during the call.
 *  o        out: o_t = sum_{s<=t} gamma_h^(t-s) (q_t . k_s) v_s
 * fp16 and bf16 run on the tensor cores (chunks of 64 rows, one CTA per (b, h)
 * carrying the state from chunk to chunk), D = 64 and 128; fp32 on CUDA cores.
 * With gamma_h = 1 for every head this is plain causal linear attention.      */
la_status la_chunk_decay_fwd(const void *q, const void *k, const void *v, void *o,
                             const float *decay,
                             int B, int H, int T, int D, la_dtype dtype,
                             void *workspace, size_t workspace_bytes, void *stream);

/* la_chunk_decay_fwd continuing from a state and handing its state on: with
 * S_in the state of the tokens before this call (state_in, or zero if NULL),
 *  o_t = q_t (gamma^(t+1) S_in + sum_{s<=t} gamma^(t-s) k_s^T v_s)
 * and state_out (if not NULL) <- gamma^T S_in + sum_s gamma^(T-1-s) k_s^T v_s, the
 * state after the last token (what la_chunk_decay_step continues from, or the
 * next segment of the sequence starts with).  state_in, state_out: [B,H,D,D]
 * fp32 device arrays, 16-byte aligned (row i = key index); they may alias. With
 * T = 0 state_out <- state_in.  The library's addition for chunked prefill and
 * for splitting a sequence into segments; source of the form as for
 * la_chunk_decay_fwd ("flash-linear-attention" README, FusedChunk: the
 * inter-chunk state carried from chunk to chunk).
 * o may be NULL: then only state_out is computed (q is not read and may be
 * NULL), at about half the cost of the whole op: the first pass of a sequence
 * split into segments needs only each segment's own end state. */
la_status la_chunk_decay_fwd_state(const void *q, const void *k, const void *v, void *o,
                                   const float *state_in, float *state_out, const float *decay,
                                   int B, int H, int T, int D, la_dtype dtype,
                                   void *workspace, size_t workspace_bytes, void *stream);

/* Retention backward.  With R_s = sum_{t>=s} gamma^(t-s) q_t^T dout_t and
 * S_t = sum_{s<=t} gamma^(t-s) k_s^T v_s:
 *  dq_t = dout_t S_t^T,  dk_s = v_s R_s^T,  dv_s = k_s R_s.                   */
la_status la_chunk_decay_bwd(const void *q, const void *k, const void *v, const void *dout,
                             const float *decay, void *dq, void *dk, void *dv,
                             int B, int H, int T, int D, la_dtype dtype,
                             void *workspace, size_t workspace_bytes, void *stream);

/* la_chunk_decay_bwd of one segment of a longer sequence, the backward of
 * la_chunk_decay_fwd_state.  Rows t = 0..T-1 are the segment's; S_in (state_in,
 * or zero if NULL) is the state of the tokens before it and R_in (dstate_in, or
 * zero if NULL) = sum_{u after the segment} gamma^(u-T) q_u^T dout_u comes from the
 * tokens after it (u counted from the segment's first row).  Then
 *  S_t = gamma^(t+1) S_in + sum_{s<=t} gamma^(t-s) k_s^T v_s,
 *  R_s = gamma^(T-s) R_in + sum_{s<=t<T} gamma^(t-s) q_t^T dout_t,
 *  dq_t = dout_t S_t^T,  dk_s = v_s R_s^T,  dv_s = k_s R_s,
 * and dstate_out (if not NULL) <- R_0, the dstate_in of the segment before this
 * one.  The gradient of the loss with respect to state_in is gamma R_0.  All
 * three are [B,H,D,D] fp32 device arrays, 16-byte aligned, row i = the index
 * of q (R) or k (S); dstate_out must not overlap state_in or dstate_in
 * (LA_ERR_INVALID_ARG).  dq may be NULL: then only dk and dv are computed
 * (state_in is not read).  dq, dk and dv may all be NULL: then only
 * dstate_out = R_0 is computed (k and v are not read and may be NULL), about a
 * third of the cost of the whole backward.  With T = 0, dstate_out <- dstate_in.  The library's
 * addition for splitting a sequence into segments (the reverse-time
 * recurrence is the backward of the FusedChunk form, "flash-linear-attention"
 * README). */
la_status la_chunk_decay_bwd_state(const void *q, const void *k, const void *v, const void *dout,
                                   const float *state_in, const float *dstate_in, float *dstate_out,
                                   const float *decay, void *dq, void *dk, void *dv,
                                   int B, int H, int T, int D, la_dtype dtype,
                                   void *workspace, size_t workspace_bytes, void *stream);

/* Combine of per-segment states for a sequence split into n segments:
 *   out[b,h] = sum over i < n with gaps[i] >= 0 of decay[h]^gaps[i] states[i,b,h],
 * summed in the order i = 0, 1, ... in fp32 (deterministic).  With E_i the
 * state_out of la_chunk_decay_fwd_state on segment i from a zero state, and
 * gaps[i] = the number of tokens strictly between segment i and segment r (-1
 * for i >= r), out is the state_in of segment r.  With F_i the dstate_out of
 * la_chunk_decay_bwd_state on segment i from a zero dstate_in, and gaps[i] = the
 * number of tokens strictly between segment r and segment i (-1 for i <= r),
 * out is the dstate_in of segment r.  Both follow from the recurrent form: a
 * span of L tokens maps a state S to gamma^L S + (the span's own state)
 * ("flash-linear-attention" README, FusedRecurrent).  The library's addition
 * for sequence parallelism (one segment per rank, the states all-gathered).
 *  states  in  [n,B,H,D,D] fp32 device array, 16-byte aligned
 *  gaps    HOST array of n values, read during the call
 *  decay   HOST array of H values in (0, 1]
 *  out     out [B,H,D,D] fp32 device array, 16-byte aligned; it may be one of
 *          the states (each element is read before it is written).
 * 1 <= n <= LA_MAX_SCAN_SEGMENTS (else LA_ERR_UNSUPPORTED). */
la_status la_chunk_decay_scan(const float *states, const long long *gaps, int n, const float *decay,
                              float *out, int B, int H, int D, void *stream);

/* ---- causal linear attention with the norm term ---------------------------
 * The causal counterpart of la_bidir_*: every token sees only the tokens up to
 * itself, with an optional per-head decay:
 *   S_t = gamma_h S_{t-1} + f(k_t)^T v_t,  z_t = gamma_h z_{t-1} + f(k_t)
 *   o_t = f(q_t) S_t / (f(q_t) . z_t + eps)
 * f = elu + 1 (LA_FEATURE_ELU1) or the identity (LA_FEATURE_IDENTITY; then
 * f(q_t) . z_t may come near -eps, which the caller must rule out).  decay is a
 * HOST array of H values in (0, 1], read during the call, or NULL for gamma = 1:
 * plain causal linear attention with the norm term.  Without the norm term the
 * op is la_chunk_decay_* (identity f, gamma = 1 for plain causal linear
 * attention).  Sources: "flash-linear-attention" README, "Different forms of
 * linear attention" (FusedRecurrent: the recurrent form these calls compute);
 * the norm term and f as in la_bidir_*.  All dtypes, D in {64, 128}.
 * fp16 with D = 64 runs on the tensor cores (the chunked decay kernel with a
 * column of ones next to v, which carries z, and the division in its epilogue;
 * f(q), f(k) formed first into the workspace); the rest on CUDA cores in fp32,
 * the sequence cut into chunks of 256 tokens, one CTA per (b, h, chunk) walking
 * its chunk from the state the tokens before it leave (each chunk's own state,
 * a sum of outer products, and a scan over the chunks).
 * Workspace: la_workspace_size(LA_OP_CAUSAL_NORM_FWD, ...) bytes (tensor cores:
 * f(q), f(k); CUDA cores: the chunk states, B H ceil(T / 256) D (D + 1) fp32
 * values, 0 and NULL allowed for T <= 256). */
la_status la_causal_norm_fwd(const void *q, const void *k, const void *v, void *o, const float *decay,
                             la_feature feature, float eps, int B, int H, int T, int D, la_dtype dtype,
                             void *workspace, size_t workspace_bytes, void *stream);

/* Gradients of sum(o * dout) for la_causal_norm_fwd.  With u_t = f(q_t) S_t,
 * n_t = f(q_t) . z_t + eps, o_t = u_t / n_t, du_t = dout_t / n_t and
 * dn_t = -(dout_t . o_t) / n_t:
 *   dq_t = (S_t du_t + z_t dn_t) f'(q_t)
 *   R_s = sum_{t>=s} gamma^(t-s) f(q_t)^T du_t,  r_s = sum_{t>=s} gamma^(t-s) f(q_t) dn_t
 *   dk_s = (R_s v_s + r_s) f'(k_s),  dv_s = f(k_s) R_s.
 * Workspace: la_workspace_size(LA_OP_CAUSAL_NORM_BWD, ...) bytes (tensor cores:
 * f(q), f(k), du = dout / n, dn, per-chunk sums and the fp32 dq, dk before the
 * dn terms; CUDA cores: (n_t, dn_t) of every row, 8 B per token-head, then the
 * chunk states of the forward and, reusing them, of the reverse sweep). */
la_status la_causal_norm_bwd(const void *q, const void *k, const void *v, const void *dout, const float *decay,
                             la_feature feature, float eps, void *dq, void *dk, void *dv,
                             int B, int H, int T, int D, la_dtype dtype,
                             void *workspace, size_t workspace_bytes, void *stream);

/* ---- gated linear attention ----------------------------------------------
 * Causal linear attention whose decay is data dependent, per token and per key
 * dimension (the GatedLinearAttention layer the "flash-linear-attention"
 * README lists; its gates come from the model's projections, which stay the
 * caller's):
 *   S_t = diag(exp(g_t)) S_{t-1} + k_t^T v_t,  o_t = q_t S_t,
 * g [B,H,T,D] the log gates (g <= 0 decays; dtype as q).  With g_t = log gamma_h
 * for every t and dimension this is la_chunk_decay_*.  The recurrent form
 * ("Different forms of linear attention": FusedRecurrent) on CUDA cores, fp32;
 * every dtype, D in {64, 128}.  As la_causal_norm_*, the sequence is cut into
 * chunks of 256 tokens, each walked by its own CTA from the state the chunks
 * before it leave (a chunk's own state and its gate product per key dimension,
 * then a scan over the chunks).
 * Workspace: la_workspace_size(LA_OP_GATED_FWD, ...) bytes (the chunk states and
 * gate products; 0, NULL allowed, for T <= 256). */
la_status la_gated_fwd(const void *q, const void *k, const void *v, const void *g, void *o,
                       int B, int H, int T, int D, la_dtype dtype,
                       void *workspace, size_t workspace_bytes, void *stream);

/* Gradients of sum(o * dout): dq_t = S_t dout_t, and with
 * R_t = q_t^T dout_t + diag(exp(g_{t+1})) R_{t+1}: dk_t = R_t v_t, dv_t = k_t R_t;
 * dg_t = sum_{s>=t} (q_s dq_s - k_s dk_s) (elementwise, in fp32 from the unrounded
 * dq and dk).  Workspace: la_workspace_size(LA_OP_GATED_BWD, ...) bytes (dq in
 * fp32, 4 B per element, in which the reverse sweep leaves each chunk's part of
 * dg; then the chunk states, gate products and per-chunk dg totals). */
la_status la_gated_bwd(const void *q, const void *k, const void *v, const void *g, const void *dout,
                       void *dq, void *dk, void *dv, void *dg,
                       int B, int H, int T, int D, la_dtype dtype,
                       void *workspace, size_t workspace_bytes, void *stream);

/* ---- feature maps formed by the caller ------------------------------------
 * Row-wise maps of [B,H,T,D] tensors, D in {32, 64, 128}, for the state-form
 * stages with LA_FEATURE_NORM (the bidirectional op with the norm term on the
 * features), as used by two of the models the "Flash Bi-directional Linear
 * Attention" README lists (Focused-LA, PolaFormer); the maps are those models'
 * feature maps, written from their definitions (|.| the 2-norm of a row, powers
 * elementwise):
 *  LA_FMAP_FOCUSED        y = relu(x), f = (|y| / |y^p|) y^p (0 for a row without a
 *                         positive entry): the focusing function; width D.
 *  LA_FMAP_POLARITY       f = [relu(x)^p, relu(-x)^p]; width 2 D (the query side and
 *                         the same-sign key side of the polarity split).
 *  LA_FMAP_POLARITY_SWAP  f = [relu(-x)^p, relu(x)^p]; width 2 D (the opposite-sign
 *                         key side).
 * p >= 1 (finite).  fp32 arithmetic, one warp per row; HBM bound. */
typedef enum { LA_FMAP_FOCUSED = 0, LA_FMAP_POLARITY = 1, LA_FMAP_POLARITY_SWAP = 2 } la_fmap;

/* y <- f(x): x [B,H,T,D], y [B,H,T,W] (W = D or 2 D as above), both dtype. */
la_status la_feature_map_fwd(la_fmap kind, float p, const void *x, void *y, int B, int H, int T, int D,
                             la_dtype dtype, void *stream);

/* dx <- J(x)^T dy, the gradient through f: x, dx [B,H,T,D], dy [B,H,T,W]. */
la_status la_feature_map_bwd(la_fmap kind, float p, const void *x, const void *dy, void *dx, int B, int H, int T,
                             int D, la_dtype dtype, void *stream);

/* ---- the state form in stages, for a sequence split along T -------------
 * A sequence cut into shards along T (one per rank or per call) gives each
 * shard's partial state; their sum over the shards is the state of the whole
 * sequence, so the op runs as: la_state_reduce on every shard, a sum of the
 * states over the shards (an all-reduce: the caller's collective), la_state_apply
 * on every shard.  The backward likewise: la_state_bwd_q on every shard with
 * the whole sequence's state, a sum of the shards' [dS | dz], la_state_bwd_kv
 * on every shard.  With one shard the stages compute exactly la_bidir_* /
 * la_simple_* (feature = LA_FEATURE_ELU1 / LA_FEATURE_IDENTITY); with
 * LA_FEATURE_NORM they are la_bidir_* with f the identity, on features the
 * caller formed (one shard covering the whole sequence is the single-GPU use:
 * reduce then apply, bwd_q then bwd_kv).  The library's
 * addition: the pages only motivate long sequences ("Flash Bi-directional
 * Linear Attention" README: intro), the split is the state form's own.
 * Shapes, dtypes and alignment as for la_bidir_fwd; T is the shard's length
 * (0 allowed: a reduce then writes zeros).  States are [B,H,D,D+1] fp32 device
 * arrays as in la_bidir_fwd (column D holds z, 0 for LA_FEATURE_IDENTITY).
 * f(x) below is elu(x)+1 for LA_FEATURE_ELU1 and x otherwise; the norm term
 * (z, n_t, eps) is present for LA_FEATURE_ELU1 and LA_FEATURE_NORM.
 * Workspace: la_workspace_size(LA_OP_STATE_REDUCE / LA_OP_STATE_BWD_Q, ...);
 * the apply and bwd_kv stages take none. */

/* state <- [S | z] of the shard: S = sum_s f(k_s)^T v_s, z = sum_s f(k_s). */
la_status la_state_reduce(const void *k, const void *v, float *state, int B, int H, int T, int D,
                          la_dtype dtype, la_feature feature, void *workspace, size_t workspace_bytes,
                          void *stream);

/* o <- f(q_t) S / (f(q_t) . z + eps) (elu+1 or norm), or q_t S (identity), with
 * the whole sequence's state. */
la_status la_state_apply(const void *q, const float *state, void *o, int B, int H, int T, int D,
                         la_dtype dtype, la_feature feature, float eps, void *stream);

/* dq of the shard and its [dS | dz] (dstate, out), from the whole sequence's
 * state: with n_t = f(q_t).z + eps and o_t = f(q_t) S / n_t,
 *   dq_t = ((dout_t S^T - (dout_t . o_t) z) / n_t) * f'(q_t),
 *   dS = sum_t f(q_t)^T dout_t / n_t,   dz = -sum_t f(q_t) (dout_t . o_t) / n_t
 * (identity: dq_t = dout_t S^T, dS = sum_t q_t^T dout_t, dz = 0). */
la_status la_state_bwd_q(const void *q, const void *dout, const float *state, void *dq, float *dstate,
                         int B, int H, int T, int D, la_dtype dtype, la_feature feature, float eps,
                         void *workspace, size_t workspace_bytes, void *stream);

/* dk, dv of the shard from the whole sequence's [dS | dz]:
 *   dk_s = (v_s dS^T + dz) * f'(k_s),   dv_s = f(k_s) dS. */
la_status la_state_bwd_kv(const void *k, const void *v, const float *dstate, void *dk, void *dv,
                          int B, int H, int T, int D, la_dtype dtype, la_feature feature, void *stream);

/* One recurrent step of retention (decode): for every (b, h), with the state
 * S = sum_{s<=t-1} gamma^(t-1-s) k_s^T v_s of the tokens seen so far,
 *      S <- gamma_h S + k^T v,     o = q S
 * i.e. S[i][j] <- gamma S[i][j] + k[i] v[j] and o[j] = sum_i q[i] S[i][j].
 * Source: "flash-linear-attention" README, "Different forms of linear
 * attention" (FusedRecurrent: the recurrent form, one token at a time).  The
 * library's addition for serving after a chunked prefill; T is 1.
 *  q, k, v  in  [B,H,D] device tensors of `dtype` (16-byte aligned)
 *  o        out [B,H,D] of `dtype`
 *  state    in/out [B,H,D,D] fp32 device array (16-byte aligned), updated in place
 *  decay    HOST pointer to H floats in (0, 1], read during the call
 * D must be 64 or 128.  No workspace.  Errors as for the other entry points. */
la_status la_chunk_decay_step(const void *q, const void *k, const void *v, void *o, float *state,
                              const float *decay, int B, int H, int D, la_dtype dtype, void *stream);

/* Reports, and clears, the fault word of this library's tensor-core kernels on
 * the current device.  Every wait inside those kernels is bounded (2 s); a wait
 * that runs out makes the kernel wind down early (its outputs are then invalid)
 * and sets the word.  Call it once the work of interest has completed (after a
 * stream or device synchronisation).  Returns LA_OK, LA_ERR_TIMEOUT, or
 * LA_ERR_CUDA if the word could not be read. */
la_status la_device_check(void);

/* ---- test hooks (fault injection without a GPU fault) -------------------
 * The library's own failure paths, made to run on demand by the tests.  The
 * pages describe no such hooks; they exist to test this library.              */

/* The launch that comes after `after` further kernel launches of this library
 * fails before it reaches the GPU: its entry point returns LA_ERR_CUDA and
 * la_last_error() names the kernel and "injected launch failure".  after = -1
 * disarms; only one failure is armed at a time (process wide).  Returns
 * LA_ERR_INVALID_ARG for after < -1. */
la_status la_debug_fail_launch(int after);

/* Enqueues on `stream` a one-CTA kernel whose single wait, on an mbarrier that
 * nothing arrives on, gives up after limit_us microseconds (1 .. 1000000), the
 * way every bounded wait of the tensor-core kernels does: it sets the fault
 * word that la_device_check() reports as LA_ERR_TIMEOUT and returns.  With
 * waited_out (a device int, or NULL) the kernel also writes 1 there when the
 * wait ran out.  Nothing is left in flight, so the context stays usable. */
la_status la_debug_wait_timeout(unsigned int limit_us, int *waited_out, void *stream);

/* Static text for a status code. */
const char *la_status_string(la_status status);

/* Text of the last error raised on the calling thread ("" if none). */
const char *la_last_error(void);

/* ---- instrumentation (off by default; host-side only) ------------------- */

/* Count of kernels this library has launched in this process. */
long long la_launch_count(void);

/* When enabled, every kernel launch is bracketed by two CUDA events recorded
 * on its stream.  Returns the previous setting. */
int la_prof_enable(int enabled);

/* Per-kernel totals since the last collect, for kernels launched while
 * profiling was on.  Synchronises on the recorded events.  Fills up to
 * `max_records` entries (name is a static string) and returns the number of
 * distinct kernels seen (may exceed max_records), or -1 on a CUDA error. */
typedef struct {
    const char *name;
    long long launches;
    double total_ms;
} la_prof_record;
int la_prof_collect(la_prof_record *records, int max_records);

#ifdef __cplusplus
}
#endif

#endif /* LA_B200_H */
