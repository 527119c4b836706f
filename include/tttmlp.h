/*
 * tttmlp.h -- C ABI of the TTT-MLP layer for NVIDIA B200 (sm_100a).
 *
 * The layer (One-Minute Video Generation with Test-Time Training, paper notes
 * page, sections "关键设计 / TTT-MLP 层" and "关键设计 / 门控 + 双向机制"):
 *
 *   per head h, hidden state W = (W1 [m x d], W2 [d x m]), m = 4 d,
 *   f(u; W) = W2 GELU(W1 u) with erf-GELU and no biases;
 *   per token t (in walking order), with q = theta_Q x_t, k = theta_K x_t,
 *   v = theta_V x_t:
 *       W_t = W_{t-1} - eta * grad_W || f(k; W_{t-1}) - v ||^2
 *       z_t = f(q; W_t)                      (read AFTER the update)
 *   mini-batch variant, chunk size b (b = 1 is the rule above): the gradients
 *   of a chunk are taken at the chunk-start state and token t of the chunk is
 *   read with the prefix state W^c - eta * sum_{s<=t in chunk} grad(s);
 *   gate:  out = x + tanh(alpha) * z   (alpha a vector over channels);
 *   bidirectional: X' = gate_f(X, fwd(X)), Y = gate_r(X', rev(X')), the two
 *   directions sharing theta and W_0, the reverse one walking t = T-1 .. 0
 *   with its chunks formed in that walking order.
 *
 * All functions are thread-safe, never throw, and allocate nothing: device
 * memory (inputs, outputs, workspace) is owned by the caller.  Every pointer
 * argument except the *_host ones of ttt_mlp_forward_host is a DEVICE pointer
 * on the current CUDA device.  Work is enqueued on `stream` (0 = the legacy
 * default stream) and the functions return once it is enqueued, except
 * ttt_mlp_status and ttt_mlp_forward_host, which synchronise the stream.
 * The full-width bf16 layer on the tensor-core path runs in chunk segments on
 * the library's own streams: one set per device and caller stream, created on
 * the first call with that stream (calls with the same `stream` take turns
 * while they enqueue; calls with different streams do not wait on each
 * other).  The call forks from `stream` and joins back into it with events,
 * also when it fails part-way, so `stream` orders everything it launched, and
 * the call can be captured into a CUDA graph (after one call on the capturing
 * stream outside the capture).
 * "Allocate nothing" means no device memory: those streams and their events
 * are the only resources the library creates.
 */
#ifndef TTTMLP_H_
#define TTTMLP_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define TTT_API __attribute__((visibility("default")))
#else
#define TTT_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t; declared here so the header needs no CUDA headers. */
typedef struct CUstream_st* ttt_stream_t;

typedef enum {
    TTT_OK = 0,
    TTT_ERR_INVALID_ARG = 1,   /* a pointer, size or value violates the contract below */
    TTT_ERR_UNSUPPORTED = 2,   /* valid but not implemented (e.g. a head dim other than 16/32/64) */
    TTT_ERR_CUDA = 3,          /* a CUDA runtime call failed; ttt_last_error() has its message */
    TTT_ERR_NONFINITE = 4,     /* (ttt_mlp_status) a NaN/Inf in the inputs, projections or outputs z:
                                  bad inputs or a diverged scan; outputs invalid */
    TTT_ERR_TIMEOUT = 5        /* (ttt_mlp_status) a bounded on-chip wait expired; outputs invalid */
} ttt_status;

typedef enum { TTT_FWD = 0, TTT_REV = 1, TTT_BIDIR = 2 } ttt_direction;

typedef enum { TTT_F32 = 0, TTT_BF16 = 1 } ttt_dtype;

/*
 * Shapes and layouts.
 *   T   tokens (>= 1);  H heads (>= 1);  d head dim (16, 32 or 64);  m = 4 d.
 *   D   model dim = H * d (the gate needs TTT(X) in X's own shape; the heads'
 *       outputs are concatenated, there is no output projection).
 *   per_head_input = 1:  X, Y are [H, T, d]; theta_q/k/v are [H, d, d] with
 *                        q = theta_q[h] x (row e of theta_q[h] gives q_e).
 *   per_head_input = 0:  X, Y are [T, D]; theta_q/k/v are [H*d, D] (the
 *                        nn.Linear weight layout: q_{h,e} = sum_c theta_q[h*d+e][c] x_c).
 *   x_dtype: element type of X, theta_q/k/v and Y.  The hidden state, the
 *   projections' outputs, the scan and all accumulations are fp32.
 *   All arrays are dense row-major, 16-byte aligned.
 */
typedef struct {
    int T;
    int H;
    int d;
    int m;                 /* must be 4 * d */
    int D;                 /* must be H * d */
    int per_head_input;    /* 1 or 0, see above */
    ttt_dtype x_dtype;
} ttt_mlp_desc;

/*
 * Bytes of device workspace ttt_mlp_forward needs for (desc, b, dir).
 * Returns 0 if the arguments are invalid (ttt_last_error() says why).
 */
TTT_API size_t ttt_mlp_workspace_size(const ttt_mlp_desc* desc, int b, ttt_direction dir);

/*
 * The gated TTT-MLP layer, one direction or both (see the top of this file).
 *
 *   X          input, layout/dtype per desc.
 *   theta_q/k/v  projections, layout/dtype per desc (shared by both directions).
 *   W1_0 [H, m, d], W2_0 [H, d, m]  fp32 initial hidden state (both directions).
 *   eta        gradient step, used exactly as given (finite, >= 0).
 *   b          chunk size, 1 <= b <= 256; a ragged last chunk is allowed.
 *   dir        TTT_FWD: Y = gate(X, fwd(X); alpha_f)
 *              TTT_REV: Y = gate(X, rev(X); alpha_r)
 *              TTT_BIDIR: Y = gate(X', rev(X'); alpha_r), X' = gate(X, fwd(X); alpha_f)
 *   alpha_f, alpha_r  [D] fp32 gate vectors; channel (h, e) is alpha[h*d + e].
 *              alpha_f is required for FWD and BIDIR, alpha_r for REV and BIDIR.
 *   Y          output, same layout/dtype as X.  Must not alias X.
 *   Z_out      optional (may be NULL) fp32 [n_dir, <X layout>] pre-gate outputs z_t,
 *              n_dir = 1 for FWD/REV, 2 for BIDIR (slot 0 forward, slot 1 reverse).
 *   W1_T, W2_T optional (may be NULL) fp32 [n_dir, H, m, d] and [n_dir, H, d, m]
 *              hidden state after each direction's last token.
 *   workspace  device memory of at least ttt_mlp_workspace_size(desc, b, dir)
 *              bytes, 256-byte aligned, not shared with a concurrent call.
 *
 * Returns TTT_OK once the work is enqueued; argument errors are reported
 * before anything is enqueued.  Divergence and expired waits are recorded in
 * the workspace and reported by ttt_mlp_status.
 */
TTT_API ttt_status ttt_mlp_forward(const ttt_mlp_desc* desc, const void* X,
                           const void* theta_q, const void* theta_k, const void* theta_v,
                           const float* W1_0, const float* W2_0, float eta, int b,
                           ttt_direction dir, const float* alpha_f, const float* alpha_r,
                           void* Y, float* Z_out, float* W1_T, float* W2_T,
                           void* workspace, size_t workspace_bytes, ttt_stream_t stream);

/*
 * Synchronises `stream`, reads and clears the status word a previous
 * ttt_mlp_forward left in `workspace`: TTT_OK, TTT_ERR_NONFINITE (a NaN/Inf
 * in X, theta or W_0, in the projections, or in an output, e.g. eta too large
 * for the squared-norm loss) or
 * TTT_ERR_TIMEOUT (a bounded wait inside a kernel expired; outputs invalid).
 */
TTT_API ttt_status ttt_mlp_status(void* workspace, ttt_stream_t stream);

/*
 * Bytes of device workspace ttt_mlp_forward_host needs: the workspace of
 * ttt_mlp_forward plus device staging for X and Y.  0 on invalid arguments.
 */
TTT_API size_t ttt_mlp_host_io_workspace_size(const ttt_mlp_desc* desc, int b, ttt_direction dir);

/*
 * End-to-end variant: X_host and Y_host are HOST buffers (pinned for full
 * copy speed); everything else as in ttt_mlp_forward (device pointers).
 * Copies X_host to the device, runs the layer, copies Y back to Y_host,
 * synchronises `stream` and returns the status as ttt_mlp_status would.
 * Where the layer runs in chunk segments (full-width bf16 input on the
 * tensor-core path) the copies overlap the computation: X goes over segment
 * by segment ahead of its projection, Y comes back segment by segment after
 * its last gate.
 */
TTT_API ttt_status ttt_mlp_forward_host(const ttt_mlp_desc* desc, const void* X_host,
                                const void* theta_q, const void* theta_k, const void* theta_v,
                                const float* W1_0, const float* W2_0, float eta, int b,
                                ttt_direction dir, const float* alpha_f, const float* alpha_r,
                                void* Y_host, void* workspace, size_t workspace_bytes,
                                ttt_stream_t stream);

/*
 * Backward pass of the layer (training: the paper notes page, "损失函数 /
 * 训练策略", fine-tunes the TTT layers and their gates): for a scalar loss with
 * upstream gradient dY = dLoss/dY, the gradients with respect to X, theta_Q/K/V,
 * W1_0, W2_0, alpha_f and alpha_r.  The layer's arguments are those of
 * ttt_mlp_forward (1 <= b <= 64); the forward pass is recomputed inside.
 *
 *   dY        fp32, X's layout.
 *   dX        fp32, X's layout.
 *   dtheta_q/k/v  fp32, theta's layout ([H, d, d] or [H*d, D]).
 *   dW1_0 [H, m, d], dW2_0 [H, d, m]  fp32.
 *   dalpha_f, dalpha_r  fp32 [D]; required for the directions that use them
 *             (may be NULL otherwise).
 *   workspace ttt_mlp_backward_workspace_size(desc, b, dir) bytes, 256-byte
 *             aligned; ttt_mlp_status(workspace, stream) reports non-finite
 *             values and expired waits as for ttt_mlp_forward.
 * Every gradient output is overwritten.  The scan's backward keeps its state
 * and gradients in fp32 and runs its products on tf32 tensor cores: in the
 * split form (three products, fp32-accurate) for fp32 layers, as single tf32
 * products for bf16 layers (the precision of their forward pass).  It walks
 * each head on a cluster of two CTAs while twice the head count fits on the
 * SMs (else one CTA; ttt_debug_set_backward_ctas), with the same results
 * either way.  Its forward walk keeps every chunk-start state, 2 m d fp32
 * values per chunk and head (128 KB at d = 64: about 30 GB of the workspace
 * for 48 heads and 313,344 tokens in chunks of 64).  The projections'
 * gradients run on the tensor cores for a full-width bf16 layer (fp32 dU split
 * into two bf16 halves), as fp32 GEMMs otherwise.
 * Returns TTT_ERR_UNSUPPORTED for b > 64.
 */
TTT_API size_t ttt_mlp_backward_workspace_size(const ttt_mlp_desc* desc, int b, ttt_direction dir);
TTT_API ttt_status ttt_mlp_backward(const ttt_mlp_desc* desc, const void* X, const void* theta_q,
                                    const void* theta_k, const void* theta_v, const float* W1_0, const float* W2_0,
                                    float eta, int b, ttt_direction dir, const float* alpha_f,
                                    const float* alpha_r, const float* dY, float* dX, float* dtheta_q,
                                    float* dtheta_k, float* dtheta_v, float* dW1_0, float* dW2_0, float* dalpha_f,
                                    float* dalpha_r, void* workspace, size_t workspace_bytes,
                                    ttt_stream_t stream);

/*
 * One rank's share of a head-sharded bidirectional layer (full-width input).
 *
 * Each head's chain is independent (paper notes page, "关键设计 / TTT-MLP 层":
 * every head keeps its own hidden state), and the reverse direction reads the
 * forward direction's output through theta_Q/K/V, which mix all channels
 * ("关键设计 / 门控 + 双向机制").  So a layer split over R ranks by heads runs
 * as two phases with one exchange between them:
 *
 *   TTT_PHASE_FWD  Q, K, V of heads [h0, h0 + hn) from X; the forward scan of
 *                  those heads; the gate.  Writes, in the columns of those
 *                  heads only, X' = X + tanh(alpha_f) z_f (fp32, Xp) and the
 *                  gate increment bf16(tanh(alpha_f) z_f) (bf16, delta_or_y).
 *   (exchange)     the caller sums every rank's increment array (the other
 *                  ranks' columns are zero in each), e.g. an all-reduce.
 *   TTT_PHASE_REV  Q, K, V of the same heads from theta X + theta delta_all;
 *                  the reverse scan; the gate on X'.  Writes Y (bf16,
 *                  delta_or_y) in the columns of those heads only.
 *
 * These are the computations of ttt_mlp_forward's bidirectional full-width
 * layer restricted to the heads: with the same inputs and kernels every
 * written element equals ttt_mlp_forward's.
 *
 *   desc       the WHOLE layer: T, H (all heads), d = 64, m, D = H * d,
 *              per_head_input = 0, x_dtype = TTT_BF16.
 *   h0, hn     the heads of this call: 0 <= h0, 1 <= hn, h0 + hn <= H.
 *   X          [T, D] bf16; theta_q/k/v [D, D] bf16 (all rows; rows h0*d ..
 *              (h0+hn)*d - 1 are read); W1_0 [H, m, d], W2_0 [H, d, m] fp32
 *              (heads h0 .. h0+hn-1 read); alpha [D] fp32: alpha_f for the
 *              forward phase, alpha_r for the reverse phase.
 *   delta_all  TTT_PHASE_REV: [T, D] bf16, every head's increment; NULL for
 *              TTT_PHASE_FWD.
 *   Xp         [T, D] fp32: written by TTT_PHASE_FWD, read by TTT_PHASE_REV.
 *   delta_or_y [T, D] bf16: the increment (TTT_PHASE_FWD) or Y (TTT_PHASE_REV).
 *   b          2 <= b <= 64 (the tensor-core scan).
 *   workspace  ttt_mlp_heads_workspace_size(desc, hn, b) bytes, 256-byte
 *              aligned; ttt_mlp_status(workspace, stream) reports non-finite
 *              values and expired waits as for ttt_mlp_forward.
 * Columns of other heads are neither read (Xp, in the reverse phase) nor
 * written.  Asynchronous on `stream`; no allocation.  Returns
 * TTT_ERR_UNSUPPORTED for shapes outside the tensor-core path.
 */
typedef enum { TTT_PHASE_FWD = 0, TTT_PHASE_REV = 1 } ttt_phase;

TTT_API size_t ttt_mlp_heads_workspace_size(const ttt_mlp_desc* desc, int hn, int b);
TTT_API ttt_status ttt_mlp_forward_heads(const ttt_mlp_desc* desc, int h0, int hn, ttt_phase phase,
                                         const void* X, const void* theta_q, const void* theta_k,
                                         const void* theta_v, const float* W1_0, const float* W2_0, float eta,
                                         int b, const float* alpha, const void* delta_all, float* Xp,
                                         void* delta_or_y, void* workspace, size_t workspace_bytes,
                                         ttt_stream_t stream);

/*
 * Segment-local attention, the sublayer the TTT layer follows in the pages'
 * block (paper notes page, "方法详解 / 整体框架": the backbone's self-attention
 * only spans the tokens of one 3-second segment, the TTT layer the whole
 * sequence).  For every head h and row t in [row0, row1):
 *
 *   Out[t, h*64 + j] = Xres[t, h*64 + j]
 *                    + sum_{u in seg(t)} softmax_u(q_t . k_u / sqrt(64)) v_u[j]
 *
 * where seg(t) = [s L, min((s + 1) L, T)), s = floor(t / L), and q_t, k_u, v_u
 * are the 64 columns of head h in rows t, u of Q, K, V.  The attention inside
 * a segment is full, not causal.  Arithmetic: bf16 Q, K, V; Q K^T and P V on
 * the tensor cores with fp32 accumulation; the softmax weights in fp32, then
 * rounded to bf16 for P V; the row sum in fp32; the result rounded to bf16.
 *
 *   T, H, d, L  tokens, heads (d must be 64), segment length (>= 1).
 *   Q, K, V     bf16, row t of each at Q + t * ld_qkv (ld_qkv >= H * 64, a
 *               multiple of 8): three [T, H*64] arrays, or one fused
 *               [T, 3*H*64] array passed at column offsets 0, H*64, 2*H*64.
 *   Xres        bf16 [T, ld_out] residual, or NULL for none.
 *   Out         bf16 [T, ld_out] (ld_out >= H * 64, a multiple of 8); only rows
 *               [row0, row1) are written, columns past H * 64 never.  Out may
 *               be Xres itself; it must not overlap Q, K or V.
 *   row0, row1  0 <= row0 <= row1 <= T.  Each row attends over its whole
 *               segment whatever the range.
 *   workspace   ttt_seg_attention_workspace_size() bytes, 256-byte aligned:
 *               the status word, cleared by the call; ttt_mlp_status(workspace,
 *               stream) reports non-finite outputs (TTT_ERR_NONFINITE) and
 *               expired waits (TTT_ERR_TIMEOUT).
 * All pointers are device pointers, 16-byte aligned.  Asynchronous on
 * `stream`; no allocation.  TTT_ERR_UNSUPPORTED for d != 64.
 */
TTT_API size_t ttt_seg_attention_workspace_size(void);
TTT_API ttt_status ttt_seg_attention(int T, int H, int d, int L, const void* Q, const void* K,
                                     const void* V, int ld_qkv, const void* Xres, void* Out, int ld_out,
                                     int row0, int row1, void* workspace, size_t workspace_bytes,
                                     ttt_stream_t stream);

/*
 * The block: segment-local attention, then the bidirectional TTT-MLP layer on
 * its output, in one schedule.  X = Xres + attention(Qa, Ka, Va) exactly as
 * ttt_seg_attention with segment length seg_len and ld_out = D, then
 * Y = ttt_mlp_forward(desc, X, ..., TTT_BIDIR, ...), enqueued as one schedule
 * on the layer's streams: the attention of every row as one launch on the
 * whole GPU ahead of the first projection, then the layer's segments.  (The
 * layer's scan and projections already occupy every SM, so running each
 * segment's attention beside the scan, just before that segment's projection,
 * measured slower; ttt_debug_set_block_front selects that schedule for
 * comparison.)  X and Y hold the same values as the two calls made one after
 * the other, in either schedule.
 *
 *   desc         a full-width bf16 layer (per_head_input = 0, x_dtype =
 *                TTT_BF16, D = H * d, d = 64).
 *   seg_len      the attention's segment length L.
 *   Qa, Ka, Va   bf16, row stride ld_qkv, as for ttt_seg_attention.
 *   Xres         bf16 [T, D] residual (or NULL).
 *   X            bf16 [T, D]: written (the layer's input); may be Xres.
 *   the rest     as for ttt_mlp_forward with dir = TTT_BIDIR and no optional
 *                outputs; workspace of ttt_block_workspace_size(desc, b)
 *                bytes, whose status word ttt_mlp_status reads.
 */
TTT_API size_t ttt_block_workspace_size(const ttt_mlp_desc* desc, int b);
TTT_API ttt_status ttt_block_forward(const ttt_mlp_desc* desc, int seg_len, const void* Qa, const void* Ka,
                                     const void* Va, int ld_qkv, const void* Xres, void* X,
                                     const void* theta_q, const void* theta_k, const void* theta_v,
                                     const float* W1_0, const float* W2_0, float eta, int b,
                                     const float* alpha_f, const float* alpha_r, void* Y, void* workspace,
                                     size_t workspace_bytes, ttt_stream_t stream);

/*
 * ttt_mlp_forward for callers that cannot allocate device memory.
 *
 * The paper has no counterpart: this is a deployment aid.  Code embedded in a
 * host framework that owns the allocator, plug-ins forbidden to call
 * cudaMalloc, or services that must not allocate after start-up cannot obtain
 * a workspace.  This entry point takes the same arguments as ttt_mlp_forward
 * except the workspace and runs the same kernels with the same arithmetic;
 * its scratch is a fixed 32 MiB array in the library's own device memory,
 * held by every GPU that loads the library until the process exits.
 *   - Shapes whose ttt_mlp_workspace_size exceeds 32 MiB are rejected with
 *     TTT_ERR_UNSUPPORTED and a message saying so.
 *   - It calls no cudaMalloc, cudaFree or other allocating routine, and it
 *     creates no streams or events: every kernel runs on `stream` itself
 *     (also for the full-width bf16 layer, which ttt_mlp_forward runs in
 *     chunk segments on streams of its own).  If the caller switched
 *     ttt_kernel_timing on, that hook still creates its timing events.
 *   - The first call on a device (of this function or of
 *     ttt_mlp_noalloc_status) looks up the array's device address, once per
 *     device, with that device current; make that first call before any
 *     stream capture.  The address is kept for the life of the process, so
 *     these two functions must not be used after cudaDeviceReset.
 *   - Every call shares the one array and it keeps the last call's contents;
 *     the status word is cleared at the start of each call.  Calls whose GPU
 *     work overlaps (other streams, other host threads) race on it: order them.
 *   - Divergence and expired waits are recorded in that array: read them with
 *     ttt_mlp_noalloc_status.
 */
TTT_API ttt_status ttt_mlp_forward_noalloc(const ttt_mlp_desc* desc, const void* X,
                                           const void* theta_q, const void* theta_k, const void* theta_v,
                                           const float* W1_0, const float* W2_0, float eta, int b,
                                           ttt_direction dir, const float* alpha_f, const float* alpha_r,
                                           void* Y, float* Z_out, float* W1_T, float* W2_T,
                                           ttt_stream_t stream);

/*
 * ttt_mlp_status for ttt_mlp_forward_noalloc: synchronises `stream`, then
 * reads and clears the status word in the library's fixed scratch array of
 * the current device (TTT_OK, TTT_ERR_NONFINITE or TTT_ERR_TIMEOUT, as
 * ttt_mlp_status).  The word belongs to the last no-alloc call on this device.
 */
TTT_API ttt_status ttt_mlp_noalloc_status(ttt_stream_t stream);

/*
 * Kernel selection, process-wide (for tests and comparisons): 0 = automatic
 * (the fastest kernel that takes the shape), 1 = the FP32 SIMT kernels,
 * 2 = the tensor-core kernels (a later ttt_mlp_forward returns
 * TTT_ERR_UNSUPPORTED if the shape is outside them), and for the scan only
 * 3 = the tensor-core scan with one CTA per head instead of a two-CTA
 * cluster (for b = 1: the per-token kernel with one CTA per head instead of
 * the four-CTA cluster that automatic selection uses for d = 64), 4 = the
 * two-CTA tensor-core scan whose CTAs each run the state chain and the output
 * of the chunk before on separate warp groups.
 * scan_impl selects the scan kernel, proj_impl the full-mode
 * projection kernel.
 */
TTT_API ttt_status ttt_mlp_select_kernels(int scan_impl, int proj_impl);

/*
 * TTT-Linear: the same gated layer with a linear hidden state f(u; W) = W u,
 * W [d x d] per head (paper notes page, "实验关键数据 / 消融实验").  For each
 * token W_t = W_{t-1} - eta * 2 (W k - v) k^T and z_t = W_t q; the mini-batch
 * form (gradients at the chunk-start state, prefix reading), the gate and the
 * directions are those of ttt_mlp_forward.  desc as for ttt_mlp_forward
 * (desc->m is not used by this layer and is not checked).
 *
 *   W_0   [H, d, d] fp32 initial state (both directions).
 *   W_T   optional (may be NULL) fp32 [n_dir, H, d, d]: the state after each
 *         direction's last token.
 *   Every other argument, the status (ttt_mlp_status) and the errors as in
 *   ttt_mlp_forward; workspace of ttt_linear_workspace_size bytes.  The scan
 *   takes the chunk form on the tensor cores (tf32 operands, fp32 state) for
 *   bf16 inputs with d = 64 and 2 <= b <= 64, else runs in fp32 (one CTA per
 *   16 rows of a head's state); ttt_mlp_select_kernels(1, .) forces the fp32
 *   scan.
 */
TTT_API size_t ttt_linear_workspace_size(const ttt_mlp_desc* desc, int b, ttt_direction dir);
TTT_API ttt_status ttt_linear_forward(const ttt_mlp_desc* desc, const void* X, const void* theta_q,
                              const void* theta_k, const void* theta_v, const float* W_0, float eta, int b,
                              ttt_direction dir, const float* alpha_f, const float* alpha_r, void* Y,
                              float* Z_out, float* W_T, void* workspace, size_t workspace_bytes,
                              ttt_stream_t stream);

/*
 * TTT-Linear with HOST buffers, as ttt_mlp_forward_host is for the MLP layer:
 * X_host in, Y_host out (pinned for full copy speed), everything else device
 * memory as in ttt_linear_forward; the workspace of
 * ttt_linear_host_io_workspace_size bytes adds device staging for X and Y.
 * On the segmented full-width bf16 path X crosses segment by segment ahead of
 * its projection and Y comes back segment by segment behind its gate.
 * Synchronises `stream` and returns the status as ttt_mlp_status would.
 */
TTT_API size_t ttt_linear_host_io_workspace_size(const ttt_mlp_desc* desc, int b, ttt_direction dir);
TTT_API ttt_status ttt_linear_forward_host(const ttt_mlp_desc* desc, const void* X_host,
                                           const void* theta_q, const void* theta_k, const void* theta_v,
                                           const float* W_0, float eta, int b, ttt_direction dir,
                                           const float* alpha_f, const float* alpha_r, void* Y_host,
                                           void* workspace, size_t workspace_bytes, ttt_stream_t stream);

/*
 * Fault injection for tests (process-wide).  While enabled, the two-CTA
 * tensor-core scan kernel (the default for bf16 inputs) first waits on an
 * mbarrier that nothing arrives on, with a 1 ms limit; the wait expires, the
 * kernel records TTT_ERR_TIMEOUT in the status word, lets its copies in
 * flight land, frees its tensor memory and returns (that call's outputs are
 * invalid).  It exercises the bounded-wait failure path without stalling the
 * GPU; the CUDA context stays usable.
 */
TTT_API ttt_status ttt_debug_inject_wait_timeout(int enable);

/*
 * Tests only: the chunk segments [begin, end) the pipelined full-width layer
 * uses for a walk of `nchunks` chunks, written as begin/end pairs into `out`
 * (room for `max_segments` pairs).  Returns the number of segments (which may
 * exceed max_segments: only that many are written), or -1 if nchunks < 1.
 */
TTT_API int ttt_debug_pipe_segments(int nchunks, int* out, int max_segments);

/*
 * Benchmarks only (process-wide): the schedule of ttt_block_forward.  -1 (the
 * default): the whole attention first.  0..100: the attention of each chunk
 * segment's rows just before that segment's projection, and the attention and
 * projection of the first `percent`% of the first direction's chunks on the
 * whole GPU before that direction's scan starts.  Changes timing, never results.
 */
TTT_API ttt_status ttt_debug_set_block_front(int percent);

/*
 * Tests and benchmarks only (process-wide): how many CTAs of one cluster walk
 * one head in the backward scan of ttt_mlp_backward.  0 (the default): two
 * while twice the head count fits on the GPU's SMs, else one; 1 or 2 forces
 * that number.  The products' output tiles and the elementwise passes are
 * dealt out over the cluster; every value is computed by the same operations
 * in the same order either way, so this changes timing, never results.
 * TTT_ERR_INVALID_ARG for any other value.
 */
TTT_API ttt_status ttt_debug_set_backward_ctas(int ctas);

/* Message for the last non-OK status returned on the calling thread ("" if none). */
TTT_API const char* ttt_last_error(void);

/*
 * Number of kernels the library has launched in this process (all entry
 * points, all threads).  Used to count launches inside a timed region.
 */
TTT_API uint64_t ttt_launch_count(void);

/*
 * Per-kernel timing, for benchmarks.  ttt_kernel_timing(1) clears the record
 * and starts bracketing every kernel launch of this library with two CUDA
 * events recorded on the launch's stream; ttt_kernel_timing(0) stops.
 * ttt_kernel_times waits for the recorded events and reports, per kernel
 * name (at most max_kernels), the summed device time in ms and the launch
 * count; the names go to `names` as a '\n'-separated list (truncated to
 * names_cap bytes).  Returns the number of distinct kernels, -1 on a CUDA
 * error.  total_ms and launches may be NULL.
 */
TTT_API ttt_status ttt_kernel_timing(int enable);
TTT_API int ttt_kernel_times(int max_kernels, char* names, size_t names_cap, double* total_ms,
                             uint64_t* launches);

#ifdef __cplusplus
}
#endif

#endif /* TTTMLP_H_ */
