/*
 * rat.h -- C ABI of the RAT+ dilated-inference hot path on NVIDIA B200 (sm_100a).
 *
 * The method ("RAT+: Train Dense, Infer Sparse -- Recurrence Augmented Attention for Dilated
 * Inference", abstract; "RAT+ Deep Dive" sections 2.1, 3.1 and 6) augments attention with a
 * full-sequence forget-gate recurrence over keys and values, so that at inference the
 * attention can be made dilated (every D-th key), optionally with a local window, and mixed
 * per head.  This library computes, on one GPU:
 *
 *   rat_recur_prefill        h_t = g_t h_{t-1} + (1-g_t) x_t,  g = sigmoid(gate logit), per
 *                            channel, for x = k and x = v with the same gate, over the whole
 *                            sequence (chunked associative scan); optional RoPE on k~.
 *   rat_recur_prefill_local  the same recurrence restarted every L positions (RAT's
 *                            chunk-local form).
 *   rat_recur_prefill_window the same recurrence over a fixed window of the last Lw = 64
 *                            positions (RAT+'s L*).
 *   rat_recur_backward       gradients of rat_recur_prefill's step.
 *   rat_recur_backward_local gradients of rat_recur_prefill_local's step.
 *   rat_recur_backward_window gradients of rat_recur_prefill_window's step.
 *   rat_dilated_attn_prefill causal attention of each query t over
 *                              S(t) = { t-We < j <= t }  U  { j <= t-We : j mod D = D-1 },
 *                            We = max(W, 1), D per head; optional RoPE on q.
 *   rat_dilated_attn_backward gradients of rat_dilated_attn_prefill.
 *   rat_kv_compress          the D-fold compressed cache: the chunk-end keys/values, the
 *                            ring of the W most recent ones and the recurrence state.
 *   rat_dilated_decode       one new token per sequence against that cache.
 *   rat_dilated_decode_paged the same over a paged cache, every sequence at its own position.
 *
 * Conventions shared by every call
 *   - Tensors are contiguous, row-major (B, H, T, d) with d innermost, all of one dtype
 *     (rat_dtype); every pointer must be 16-byte aligned.  d (d_head) is 64 or 128.
 *   - Device pointers are caller-owned device memory; host pointers are named "host".
 *     The library allocates no device memory: scratch lives in caller-provided workspaces.
 *   - Every call is asynchronous on `stream` (a cudaStream_t; NULL = legacy default stream).
 *     Its return value reports host-side validation and launch errors only.  Errors found
 *     on the device (a bounded wait that ran out) are recorded in the workspace and
 *     returned by rat_sync_status().
 *   - Recurrence state and all accumulation are float32; bf16 tensors are rounded to
 *     nearest-even when written.
 *   - Readings of points the pages leave open: one gate tensor shared by K and V; h_{-1} = 0
 *     unless h0 is given; the query always sees its own position (We = max(W,1)); dilated keys
 *     are the chunk ends j = D-1, 2D-1, ...; RoPE (rotate-half pairing (c, c+d/2),
 *     theta_c = base^(-2c/d)) is applied to k~ after the recurrence, at absolute position
 *     pos0 + t; softmax scale 1/sqrt(d) unless given.
 */
#ifndef RAT_H_
#define RAT_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define RAT_API __attribute__((visibility("default")))
#else
#define RAT_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Status codes (returned by every entry point, and by rat_sync_status for device errors). */
typedef enum {
    RAT_OK = 0,
    RAT_ERR_INVALID = -1,      /* bad argument: NULL pointer, bad size, misaligned pointer   */
    RAT_ERR_UNSUPPORTED = -2,  /* valid but not implemented (e.g. d not in {64, 128})       */
    RAT_ERR_CUDA = -3,         /* a CUDA runtime call or kernel launch failed               */
    RAT_ERR_TIMEOUT = -4,      /* a bounded device-side wait ran out (workspace not zeroed?) */
    RAT_ERR_WORKSPACE = -5     /* workspace missing or smaller than the *_workspace_bytes() */
} rat_status;

/* Element types. */
typedef enum { RAT_F32 = 0, RAT_BF16 = 1 } rat_dtype;

/* Human-readable name of a status code (static string, never NULL). */
RAT_API const char *rat_status_string(int status);

/* Library version string, e.g. "rat-b200 0.1 sm_100a". */
RAT_API const char *rat_version(void);

/* ------------------------------------------------------------------------------------------
 * Workspaces.
 * A workspace is caller-owned device memory that holds a 256-byte header (device error word,
 * launch epoch and CTA tickets) followed by per-call scratch.  Zero it once with
 * rat_workspace_init() before its first use; afterwards every call leaves it consistent.
 * Use one workspace per stream and per call kind (prefill recurrence or decode): calls that
 * share a workspace must not overlap on the GPU.
 * ---------------------------------------------------------------------------------------- */

/* Zero `ws_bytes` bytes of `ws` on `stream` (cudaMemsetAsync). */
RAT_API int rat_workspace_init(void *ws, size_t ws_bytes, void *stream);

/* Synchronise `stream`, then return the first device-side error recorded in workspace `ws`
 * since the last rat_sync_status() on it (RAT_OK if none) and clear it. */
RAT_API int rat_sync_status(void *ws, void *stream);

/* ------------------------------------------------------------------------------------------
 * rat_recur_prefill -- full-sequence forget-gate recurrence over keys and values.
 *   "RAT+ Deep Dive" section 2.1 (full-sequence recurrence, L = T, computed in prefill by an
 *   associative scan; forget gate g input-dependent) and section 7.3 ("parallel prefill by
 *   associative scan").
 *
 *   k, v, gate_logit : device, (B, H, T, d) of dtype          inputs x = k, x = v and a
 *   h0_k, h0_v       : device, (B, H, d) float32, or NULL     initial state (NULL = zeros)
 *   k_rec, v_rec     : device, (B, H, T, d) of dtype          outputs k~ (after RoPE, if
 *                                                            rope_base > 0) and v~
 *   hT_k, hT_v       : device, (B, H, d) float32, or NULL     final state h_{T-1} (before RoPE)
 *   pos0             : absolute position of row t = 0 (RoPE angle (pos0 + t) * theta_c)
 *   rope_base        : > 0 applies RoPE to k~ with this base; <= 0 disables it
 *   ws, ws_bytes     : workspace of at least rat_recur_workspace_bytes(B, H, T, d, dtype)
 * Computes g = 1/(1+exp(-a)), 1-g, and h_t = g h_{t-1} + (1-g) x_t in float32 for every
 * channel.  Outputs may not alias inputs.  T = 0 is a no-op.  The scan carries state between
 * chunks of the sequence with a bounded-wait decoupled look-back; if that wait runs out the
 * device error word becomes RAT_ERR_TIMEOUT (see rat_sync_status).  For bf16, d = 128 and T a
 * multiple of 16 the channels of each (b, h) scan as two independent 64-channel slices
 * (channels [32s, 32s+32) with their rotate-half partners); results are the same up to float32
 * rounding order.  Run-to-run reproducibility is to rounding, not to the bit: a chunk composes
 * whichever predecessors' records are ready when it looks back, so the float32 carries (and
 * through them a stored bf16 value) may differ in the last bit between two identical calls.
 * ---------------------------------------------------------------------------------------- */
RAT_API size_t rat_recur_workspace_bytes(int B, int H, int T, int d, int dtype);

RAT_API int rat_recur_prefill(const void *k, const void *v, const void *gate_logit,
                      const float *h0_k, const float *h0_v,
                      void *k_rec, void *v_rec, float *hT_k, float *hT_v,
                      int B, int H, int T, int d, int dtype,
                      int64_t pos0, float rope_base,
                      void *ws, size_t ws_bytes, void *stream);

/* ------------------------------------------------------------------------------------------
 * rat_recur_prefill_local -- the chunk-local recurrence of RAT: the sequence is cut into blocks
 * of L positions and the recurrence runs inside each block only.
 *   Abstract of "RAT: Bridging RNN Efficiency and Attention Accuracy via Chunk-based Sequence
 *   Modeling" (recurrence within each chunk, attention across chunks) and "RAT+ Deep Dive"
 *   section 2.1 (original RAT: blocks of size L = D, each token recurs within its own block).
 *
 *   Arguments as rat_recur_prefill, plus
 *   L : block length (>= 1).  Blocks are aligned to absolute positions: the state is set to 0
 *       before every position p = pos0 + t with p mod L = 0, i.e.
 *         h_t = (1-g_t) x_t                 if (pos0 + t) mod L = 0
 *         h_t = g_t h_{t-1} + (1-g_t) x_t   otherwise.
 *       h0_k, h0_v therefore reach only the positions before the first block start; with
 *       pos0 mod L = 0 they are ignored.  hT_k, hT_v are the state after position T-1 (the
 *       value a following call or rat_dilated_decode continues from).
 *   Returns RAT_ERR_INVALID for L < 1; everything else as rat_recur_prefill.  A block start at
 *   a chunk boundary of the scan removes that chunk's look-back wait.
 * ---------------------------------------------------------------------------------------- */
RAT_API int rat_recur_prefill_local(const void *k, const void *v, const void *gate_logit,
                            const float *h0_k, const float *h0_v,
                            void *k_rec, void *v_rec, float *hT_k, float *hT_v,
                            int B, int H, int T, int d, int dtype,
                            int64_t pos0, int64_t L, float rope_base,
                            void *ws, size_t ws_bytes, void *stream);

/* ------------------------------------------------------------------------------------------
 * rat_recur_backward -- gradients of the prefill recurrence step (rat_recur_prefill, the
 * full-sequence form), for training with dilated inference in view ("RAT+ Deep Dive" section
 * 2.2: training mixes dense and dilated samples, which needs this step's derivative).
 *   The reverse-mode derivative of h_t = g_t h_{t-1} + (1-g_t) x_t, k~ = RoPE(h^k), v~ = h^v:
 *     mu_t = e_t + g_{t+1} mu_{t+1},  mu_{T-1} = e_{T-1} + dhT,
 *     e^k_t = RoPE_t^T(dk~_t), e^v_t = dv~_t,
 *     dk_t = (1-g_t) mu^k_t,  dv_t = (1-g_t) mu^v_t,
 *     dgate_t = g_t (1-g_t) [mu^k_t (h^k_{t-1} - k_t) + mu^v_t (h^v_{t-1} - v_t)],
 *     dh0 = g_0 mu_0,   with h^k = RoPE^T(k~), h^v = v~ read from the forward outputs.
 *
 *   k, v, gate_logit : device, (B, H, T, d) of dtype          the forward inputs
 *   h0_k, h0_v       : device, (B, H, d) float32, or NULL     the forward initial state
 *   k_rec, v_rec     : device, (B, H, T, d) of dtype          the forward outputs k~, v~
 *   dk_rec, dv_rec   : device, (B, H, T, d) of dtype          upstream gradients of k~, v~
 *   dhT_k, dhT_v     : device, (B, H, d) float32, or NULL     upstream gradient of the final
 *                                                            state (NULL: zero)
 *   dk, dv, dgate_logit : device, (B, H, T, d) of dtype       outputs
 *   dh0_k, dh0_v     : device, (B, H, d) float32, or NULL     gradient of the initial state
 *   pos0, rope_base  : as given to rat_recur_prefill
 *   ws, ws_bytes     : workspace of at least rat_recur_backward_workspace_bytes(B, H, T, d)
 * float32 arithmetic; bf16 outputs rounded once.  h_{t-1} is taken from the stored (rounded)
 * forward outputs, as a memory-saving training step would.  Outputs may not alias inputs.
 * T = 0 is a no-op.  One launch: a scan from the end of the sequence whose chunks combine by a
 * decoupled look-back with bounded waits (a wait that runs out records RAT_ERR_TIMEOUT in the
 * workspace, read by rat_sync_status()).  The workspace follows the prefill rules (zeroed once
 * by rat_workspace_init, one call at a time); RAT_ERR_UNSUPPORTED when B*H*ceil(T/32) >= 2^31.
 * ---------------------------------------------------------------------------------------- */
RAT_API size_t rat_recur_backward_workspace_bytes(int B, int H, int T, int d);

RAT_API int rat_recur_backward(const void *k, const void *v, const void *gate_logit,
                       const float *h0_k, const float *h0_v, const void *k_rec,
                       const void *v_rec, const void *dk_rec, const void *dv_rec,
                       const float *dhT_k, const float *dhT_v, void *dk, void *dv,
                       void *dgate_logit, float *dh0_k, float *dh0_v, int B, int H, int T,
                       int d, int dtype, int64_t pos0, float rope_base, void *ws,
                       size_t ws_bytes, void *stream);

/* rat_recur_backward_local -- gradients of rat_recur_prefill_local's step (RAT's chunk-local
 * recurrence, restarted before every absolute position pos0 + t with (pos0 + t) mod L = 0).
 *   Arguments as rat_recur_backward, plus L >= 1 (RAT_ERR_INVALID otherwise), as given to the
 *   forward.  Both recurrences are cut at block starts:
 *     mu_t = e_t + [pos0 + t + 1 not a block start] g_{t+1} mu_{t+1},
 *     dgate_t uses h_{t-1} = 0 at a block start,
 *     dh0 = g_0 mu_0 when pos0 is not a block start, else 0 (h0 reaches only the rows before the
 *     first start). */
RAT_API int rat_recur_backward_local(const void *k, const void *v, const void *gate_logit,
                             const float *h0_k, const float *h0_v, const void *k_rec,
                             const void *v_rec, const void *dk_rec, const void *dv_rec,
                             const float *dhT_k, const float *dhT_v, void *dk, void *dv,
                             void *dgate_logit, float *dh0_k, float *dh0_v, int B, int H, int T,
                             int d, int dtype, int64_t pos0, int64_t L, float rope_base, void *ws,
                             size_t ws_bytes, void *stream);

/* ------------------------------------------------------------------------------------------
 * rat_recur_prefill_window -- the fixed-window recurrence of RAT+: each state covers only the
 * last Lw positions.
 *   "RAT+ Deep Dive" section 2.1 (a fixed recurrence window L* = 64: each token's recurrence
 *   reaches 64 positions back, and prefill computes it in parallel).  Read as: the state at t is the
 *   recurrence restarted from zero at t - Lw + 1,
 *     y_t = sum_{s = t-Lw+1}^{t} ( prod_{r = s+1}^{t} g_r ) (1 - g_s) x_s,   g = sigmoid(a),
 *   for x = k and x = v with the same gate, in float32; k~ = RoPE(y^k) when rope_base > 0.
 *
 *   k, v, gate_logit : device, (B, H, T, d) of dtype          inputs
 *   prev_k, prev_v, prev_gate_logit
 *                    : device, (B, H, Lw, d) of dtype, or all three NULL: the Lw positions just
 *                      before row 0 (oldest first), so that a sequence can be continued; NULL
 *                      clips the window at row 0
 *   k_rec, v_rec     : device, (B, H, T, d) of dtype          outputs k~, v~
 *   pos0             : absolute position of row 0 (RoPE only)
 *   Lw               : window length; 64 (the pages' L*) is the supported value
 *                      (RAT_ERR_UNSUPPORTED otherwise, RAT_ERR_INVALID below 1)
 *   ws, ws_bytes     : workspace of at least 256 bytes, 256-byte aligned (its header receives
 *                      device-side errors; see rat_sync_status)
 * There is no initial or final state: the window makes the state a function of the last Lw
 * inputs.  Outputs may not alias inputs.  T = 0 is a no-op.  No CTA waits for another (the
 * segmented form is computed block by block), so the call has no look-back.
 * ---------------------------------------------------------------------------------------- */
RAT_API int rat_recur_prefill_window(const void *k, const void *v, const void *gate_logit,
                             const void *prev_k, const void *prev_v, const void *prev_gate_logit,
                             void *k_rec, void *v_rec, int B, int H, int T, int d, int dtype,
                             int64_t pos0, int64_t Lw, float rope_base,
                             void *ws, size_t ws_bytes, void *stream);

/* ------------------------------------------------------------------------------------------
 * rat_recur_backward_window -- gradients of rat_recur_prefill_window's step (the fixed-window
 * recurrence, "RAT+ Deep Dive" section 2.1, L* = 64), for training in that form.
 *   Each output y_t is the recurrence restarted from zero at t - Lw + 1, so the gradient sums,
 *   over the Lw outputs whose windows hold a row, the reverse pass of each restarted recurrence:
 *     dL/dx_s = (1 - g_s) sum_{t=s}^{s+Lw-1} e_t prod_{r=s+1}^{t} g_r,
 *     dL/dg_s = sum_{t=s}^{s+Lw-1} e_t prod_{r=s+1}^{t} g_r (h^t_{s-1} - x_s),
 *   h^t the state restarted at t - Lw + 1 (h^t_{t-Lw} = 0), e^k_t = RoPE_t^T(dk~_t),
 *   e^v_t = dv~_t, dgate_logit = g (1 - g) (dg^k + dg^v).  Computed in blocks of Lw rows with
 *   products of one block's gates only (no division by a gate, no subtraction of older states).
 *
 *   k, v, gate_logit : device, (B, H, T, d) of dtype          the forward inputs
 *   prev_k, prev_v, prev_gate_logit
 *                    : device, (B, H, Lw, d) of dtype, or all three NULL: the forward's history
 *                      rows
 *   dk_rec, dv_rec   : device, (B, H, T, d) of dtype          upstream gradients of k~, v~
 *   dk, dv, dgate_logit : device, (B, H, T, d) of dtype       outputs
 *   dprev_k, dprev_v, dprev_gate_logit
 *                    : device, (B, H, Lw, d) of dtype, or all three NULL: gradients of the history
 *                      rows (only with them; the oldest row gets 0, no window of rows 0.. holds it)
 *   pos0, Lw, rope_base : as given to the forward (Lw = 64, RAT_ERR_UNSUPPORTED otherwise)
 * float32 arithmetic; bf16 outputs rounded once.  The forward outputs are not needed (the block
 * states are recomputed from the inputs).  Outputs may not alias inputs.  T = 0 is a no-op.  One
 * launch; no CTA waits for another, so the call needs no workspace and records no device error.
 * ---------------------------------------------------------------------------------------- */
RAT_API int rat_recur_backward_window(const void *k, const void *v, const void *gate_logit,
                              const void *prev_k, const void *prev_v,
                              const void *prev_gate_logit, const void *dk_rec,
                              const void *dv_rec, void *dk, void *dv, void *dgate_logit,
                              void *dprev_k, void *dprev_v, void *dprev_gate_logit, int B, int H,
                              int T, int d, int dtype, int64_t pos0, int64_t Lw, float rope_base,
                              void *stream);

/* ------------------------------------------------------------------------------------------
 * rat_dilated_attn_prefill -- causal dilated attention with an optional local window and a
 * per-head dilation, over the recurrence outputs.
 *   RAT+ abstract (dilation D cuts attention FLOPs and KV cache D-fold; optional local
 *   windows; hybrid head compositions); "RAT+ Deep Dive" section 3.1 table (FLOPs T/D) and
 *   section 6 "Head-Wise Hybrid" (different D per head).
 *
 *   q             : device, (B, H, T, d) of dtype   queries (RoPE applied inside if rope_base > 0)
 *   k_rec, v_rec  : device, (B, H, T, d) of dtype   recurrence outputs from rat_recur_prefill
 *   o             : device, (B, H, T, d) of dtype   output
 *   D             : dilation of every head (>= 1), used when D_per_head is NULL
 *   W             : local window (>= 0); the window is the W most recent positions, self
 *                   included; W = 0 means self only
 *   D_per_head    : host, int32[H] or NULL          per-head dilation (each >= 1)
 *   pos0          : absolute position of row 0 (RoPE only)
 *   rope_base     : > 0 rotates q with this base (k_rec is expected already rotated)
 *   scale         : softmax scale; <= 0 selects 1/sqrt(d)
 * For query t of head h:  o_t = sum_{j in S(t)} softmax_j(scale * q^_t . k~_j) v~_j with
 * S(t) = { t-We < j <= t } U { j <= t-We : j mod D_h = D_h - 1 }, We = max(W, 1).
 * bf16: QK^T and PV on tcgen05 tensor cores (bf16 operands, float32 accumulation; the
 * softmax probabilities are rounded to bf16 for PV); float32: CUDA-core FMA throughout.
 * Needs no workspace and never waits on other CTAs; its internal pipeline waits are bounded,
 * and an expired wait is recorded in a library-wide device error word that
 * rat_attn_sync_status() reads.
 * RoPE on the tensor-core path reads a per-device table of the frequency set: the first call
 * with a new rope_base (for a given d) writes it once and waits for that copy on the host
 * before returning, so calls on any number of streams may follow without host syncs.  Up to 16
 * distinct sets per device are kept for the life of the process; a 17th is refused with
 * RAT_ERR_UNSUPPORTED, and so is the first call with a new set while `stream` is being
 * captured into a CUDA graph (make one call outside the capture first).
 * ---------------------------------------------------------------------------------------- */
RAT_API int rat_dilated_attn_prefill(const void *q, const void *k_rec, const void *v_rec, void *o,
                             int B, int H, int T, int d, int dtype, int D, int W,
                             const int32_t *D_per_head, int64_t pos0, float rope_base,
                             float scale, void *stream);

/* rat_dilated_attn_prefill_sinks -- the same attention with attention sinks: the first n_sink
 * positions join every key set (StreamingLLM layers; "RAT+ Deep Dive" section 6, layer-wise
 * hybrid, where the odd layers are StreamingLLM layers).  Each key counts once (a sink already in the window or a
 * chunk end is not repeated).  A StreamingLLM layer is D larger than any position (no chunk
 * ends), W its window, n_sink its sinks; sinks also combine with dilation.
 *   Arguments as rat_dilated_attn_prefill, plus n_sink >= 0 (0: exactly
 *   rat_dilated_attn_prefill).  bf16 with d = 128, n_sink <= 64 and no chunk end among the sinks
 *   (every head has D = 1 or D > n_sink) runs the tensor-core kernel with the sinks as one more
 *   key block; other calls run the CUDA-core kernel (float32 arithmetic). */
RAT_API int rat_dilated_attn_prefill_sinks(const void *q, const void *k_rec, const void *v_rec,
                             void *o, int B, int H, int T, int d, int dtype, int D, int W,
                             const int32_t *D_per_head, int n_sink, int64_t pos0,
                             float rope_base, float scale, void *stream);

/* rat_dilated_attn_prefill_topk -- the attention with top-k chunk selection combined with the
 * dilation ("RAT+ Deep Dive" section 4: dilation reaches the whole sequence, the selected blocks
 * add dense local detail).  Read as: the blocks are the dilation's chunks [cD, cD + D - 1]; each chunk
 * wholly older than the window (cD + D - 1 <= t - We) is scored by its chunk-end key (the
 * recurrence state that sums the chunk up), s_c = scale <q^_t, k~_{cD+D-1}>; every position of
 * the top_k best chunks (ties: the earlier chunk) joins S(t) and the sinks, each key once.
 *   Arguments as rat_dilated_attn_prefill_sinks, plus top_k in [0, 16] (RAT_ERR_UNSUPPORTED
 *   above 16).  bf16 with d = 128, n_sink = 0 and T <= 65536 runs on the tensor cores: a
 *   selection pass scores the chunk ends with q^ rounded to bf16 (the MMA operand), then the
 *   key blocks holding the selected chunks join the attention with per-row masks.  Other calls
 *   run the CUDA-core kernel (float32 arithmetic, q^ in float32).  Where two chunk scores tie
 *   to within the rounding of the scoring precision, either may be taken.  Prefill only: a
 *   decode step would need the uncompressed cache. */
RAT_API int rat_dilated_attn_prefill_topk(const void *q, const void *k_rec, const void *v_rec,
                             void *o, int B, int H, int T, int d, int dtype, int D, int W,
                             const int32_t *D_per_head, int n_sink, int top_k, int64_t pos0,
                             float rope_base, float scale, void *stream);

/* Synchronise `stream`, then return (and clear) the first device-side error recorded by the
 * attention kernel since the last call (RAT_OK if none). */
RAT_API int rat_attn_sync_status(void *stream);

/* ------------------------------------------------------------------------------------------
 * rat_dilated_attn_prefill_ex -- the attention with every option of this library.
 *   Arguments as rat_dilated_attn_prefill, plus opt (NULL: no option):
 *     n_sink : attention sinks (as rat_dilated_attn_prefill_sinks)
 *     top_k  : chunks attended in full (as rat_dilated_attn_prefill_topk)
 *     lse    : device float32 [B][H][T] output, or NULL: log2 of each query's softmax
 *              denominator, log2 sum_j 2^(s_j log2 e) with s_j = scale <q^_t, k~_j> -- the
 *              value rat_dilated_attn_backward takes to rebuild the weights (4-byte aligned)
 *   Dispatch as for the other entry points (tensor cores for bf16, d = 128 when the options
 *   allow it).
 * ---------------------------------------------------------------------------------------- */
typedef struct rat_attn_options {
    int32_t n_sink;           /* attention sinks, >= 0                                     */
    int32_t top_k;            /* chunks attended in full, 0 .. 16                          */
    float *lse;               /* optional output, see above                                */
} rat_attn_options;

RAT_API int rat_dilated_attn_prefill_ex(const void *q, const void *k_rec, const void *v_rec,
                             void *o, int B, int H, int T, int d, int dtype, int D, int W,
                             const int32_t *D_per_head, int64_t pos0, float rope_base,
                             float scale, const rat_attn_options *opt, void *stream);

/* ------------------------------------------------------------------------------------------
 * rat_dilated_attn_backward -- gradients of rat_dilated_attn_prefill (training with dilated
 * samples: "RAT+ Deep Dive" section 2.2 trains half the samples with D = 1 and half with
 * D = 64, which needs this derivative for every D).
 *   With p_t the softmax weights of query t over S(t) and q^ = RoPE(q):
 *     dp_tj = <dO_t, v~_j>,  ds_tj = p_tj (dp_tj - <dO_t, o_t>),
 *     dq = RoPE^T(scale sum_j ds_tj k~_j),  dk~_j = scale sum_t ds_tj q^_t,
 *     dv~_j = sum_t p_tj dO_t.
 *   q, k_rec, v_rec, o : device (B, H, T, d) of dtype     the forward's inputs and output
 *   dO                 : device (B, H, T, d) of dtype     upstream gradient of o
 *   dq, dk_rec, dv_rec : device (B, H, T, d) of dtype     outputs (dk_rec, dv_rec are the
 *                        gradients of k~, v~: the dk_rec, dv_rec inputs of rat_recur_backward)
 *   D, W, D_per_head, n_sink, pos0, rope_base, scale : as given to the forward
 *                        (rat_dilated_attn_prefill_sinks; n_sink = 0 without sinks)
 *   lse                : device float32 [B][H][T], the forward's rat_attn_options.lse output,
 *                        or NULL (the denominators are then recomputed: one more walk over
 *                        every key set)
 *   ws, ws_bytes       : workspace of at least rat_dilated_attn_backward_workspace_bytes
 * bf16 with d = 128, n_sink = 0 and at most four distinct dilations > 1: a CUDA-core prep
 * launch (q^ rounded to bf16 as the forward's operand, <dO_t, o_t>), then dq and dk~/dv~
 * launches on the tensor cores (S, dP and S^T, dP^T products, dQ += dS K, dV += P^T dO,
 * dK += dS^T q^; P and dS rounded to bf16 as MMA operands, float32 accumulation).  Without lse
 * the forward runs once first to produce it (its output goes to dq, overwritten after).  Their
 * pipeline waits are bounded; an expired one is recorded in the workspace header
 * (rat_sync_status).  Other calls: three CUDA-core launches with float32 accumulation and no
 * device-side waits.  Outputs are rounded once. 
 * ---------------------------------------------------------------------------------------- */
RAT_API size_t rat_dilated_attn_backward_workspace_bytes(int B, int H, int T, int d, int dtype);

RAT_API int rat_dilated_attn_backward(const void *q, const void *k_rec, const void *v_rec,
                              const void *o, const void *dO, void *dq, void *dk_rec,
                              void *dv_rec, int B, int H, int T, int d, int dtype, int D, int W,
                              const int32_t *D_per_head, int n_sink, const float *lse,
                              int64_t pos0, float rope_base, float scale, void *ws,
                              size_t ws_bytes, void *stream);

/* Diagnostic: where the attention kernel's last recorded timeout happened, as
 * (wait site << 24) | (key block << 8) | phase parity; sites: 1 producer K-stage-free, 2 MMA
 * query-ready, 3 MMA K-stage-full, 4 MMA previous-PV, 5 MMA probabilities-ready, 6 softmax
 * query-loaded, 7 softmax scores-ready, 8 softmax rescale, 9 epilogue, 10 producer
 * query-rotated, 11 producer V-stage-free, 12 MMA V-stage-full; top-k selection: 13 selection
 * published, 14 MMA selection-scores-read, 15 softmax selection-scores-ready.  0 if none. */
RAT_API uint32_t rat_attn_error_site(void);

/* Diagnostic: bit s set when a wait at site s (numbering as above) was still in progress when a
 * CTA of the attention kernel aborted after a timeout. */
RAT_API uint32_t rat_attn_error_waiting(void);

/* Tuning knob of the bf16 tensor-core attention: keys per block, 64 (two CTAs per SM) or 128
 * (one CTA per SM); 0 restores the automatic choice.  Process-wide; RAT_ERR_INVALID otherwise. */
RAT_API int rat_set_attn_block_keys(int block_keys);


/* ------------------------------------------------------------------------------------------
 * Compressed KV cache (RAT+ abstract: dilation reduces the KV cache D-fold; "RAT+ Deep Dive"
 * section 3.1: "KV cache ... compressed 64x" at D = 64).
 *
 * Layout, with cap_h = floor(Tcap / D_h) and off_h = sum_{h' < h} cap_h':
 *   k_dil, v_dil : device [B][sum_h cap_h][d] of dtype; entry i of head h (row
 *                  b * sum_h cap_h + off_h + i) holds position i * D_h + D_h - 1
 *   k_win, v_win : device [B][H][W][d] of dtype; position p is in slot p mod W (NULL if W = 0)
 *   h_k, h_v     : device [B][H][d] float32 recurrence state after the last position
 *                  (before RoPE)
 *   pos          : number of positions consumed so far (the same for every sequence)
 *   k_sink, v_sink : device [B][H][n_sink][d] of dtype: positions 0 .. n_sink-1 (attention
 *                  sinks, attended by every later token as in rat_dilated_attn_prefill_sinks)
 *   reset_every  : 0 for the full-sequence recurrence of RAT+; L > 0 for the chunk-local
 *                  recurrence of RAT (state dropped before every position p with p mod L = 0,
 *                  as in rat_recur_prefill_local); read by rat_dilated_decode
 * The struct itself is host memory; the caller owns every buffer it points to.
 * ---------------------------------------------------------------------------------------- */
typedef struct rat_kv_cache {
    int32_t B, H, d, W;       /* batch, heads, head dim, local window (0 = none)           */
    int32_t Tcap;             /* maximum number of positions the cache will ever hold      */
    int32_t dtype;            /* rat_dtype of k_dil, v_dil, k_win, v_win                    */
    const int32_t *D;         /* host int32[H]: dilation of each head (>= 1)               */
    void *k_dil, *v_dil;      /* device, see layout above                                  */
    void *k_win, *v_win;      /* device ring, or NULL when W == 0                          */
    float *h_k, *h_v;         /* device float32 state                                      */
    int64_t pos;              /* positions consumed so far                                 */
    int64_t reset_every;      /* recurrence block length L, or 0 (full sequence); >= 0     */
    int32_t n_sink;           /* attention sinks kept (first positions); 0 = none          */
    void *k_sink, *v_sink;    /* device [B][H][n_sink][d] of dtype, or NULL when n_sink == 0 */
    int32_t window_rec;       /* 64: the fixed-window recurrence (L* = 64) decodes against
                                 this cache (then reset_every = 0); 0: the full-sequence or
                                 chunk-local recurrence                                    */
    void *k_raw, *v_raw, *a_raw;  /* device [B][H][window_rec][d] of dtype: raw k, v and gate
                                 logits of the last window_rec positions, position p in slot
                                 p mod window_rec (rat_kv_raw_bytes each); NULL when 0      */
} rat_kv_cache;

/* Byte sizes of the buffers a cache with these fields needs (any output may be NULL). */
RAT_API int rat_kv_cache_bytes(const rat_kv_cache *cache, size_t *dil_bytes, size_t *win_bytes,
                       size_t *state_bytes);

/* Bytes of each of the three raw rings (k_raw, v_raw, a_raw) of a cache with window_rec > 0:
 * B * H * window_rec * d * element size; 0 when window_rec is 0 or the cache is invalid. */
RAT_API size_t rat_kv_raw_bytes(const rat_kv_cache *cache);

/* rat_kv_compress -- append T positions of recurrence output to the cache.
 *   k_rec, v_rec : device (B, H, T, d) of cache->dtype: positions cache->pos .. cache->pos+T-1
 *   hT_k, hT_v   : device (B, H, d) float32 state after those positions (copied into h_k, h_v)
 * Writes every position p with p mod D_h = D_h - 1 (and p / D_h < cap_h) to its dil entry, the
 * last min(W, T) positions to their ring slots and positions below n_sink to the sink rows;
 * copies the state; then advances
 * cache->pos by T on the host.  Bit-exact copies.  Requires cache->pos + T <= Tcap.  A cache with
 * window_rec > 0 is refused (RAT_ERR_INVALID): it also needs the raw inputs, which
 * rat_kv_compress_window takes. */
RAT_API int rat_kv_compress(const void *k_rec, const void *v_rec, const float *hT_k, const float *hT_v,
                    int T, rat_kv_cache *cache, void *stream);

/* rat_kv_compress_window -- append T positions of the fixed-window recurrence (the outputs of
 * rat_recur_prefill_window) to a cache with window_rec = 64 ("RAT+ Deep Dive" section 2.1,
 * L* = 64).
 *   k_rec, v_rec     : device (B, H, T, d) of cache->dtype, positions cache->pos .. pos + T - 1
 *   k, v, gate_logit : device (B, H, T, d) of cache->dtype, the raw inputs of those positions
 * Writes the chunk ends, ring and sink rows as rat_kv_compress does (the window form has no
 * recurrence state to copy), and the raw rows of the last min(T, 64) positions to their raw
 * ring slots; then advances cache->pos by T on the host.  Bit-exact copies.  RAT_ERR_INVALID for
 * a cache without window_rec = 64 or cache->pos + T > Tcap. */
RAT_API int rat_kv_compress_window(const void *k_rec, const void *v_rec, const void *k,
                    const void *v, const void *gate_logit, int T, rat_kv_cache *cache,
                    void *stream);

/* ------------------------------------------------------------------------------------------
 * rat_dilated_decode -- one new token per sequence against the compressed cache.
 *   q, k, v, gate_logit : device (B, H, 1, d) of cache->dtype, the token at position t = pos
 *   o                   : device (B, H, 1, d) of cache->dtype
 *   rope_base, scale    : as in prefill (rope_base must match the one used for the cache)
 *   ws, ws_bytes        : workspace of at least rat_decode_workspace_bytes(cache)
 * Per (b, h): state update h = g h + (1-g) x for k and v (h taken as 0 first when
 * cache->reset_every = L > 0 and t mod L = 0; with window_rec = 64, h is instead the
 * recurrence rerun from zero over the raw rows of positions max(0, t-63) .. t-1, and the
 * token's raw k, v, gate logit go to raw slot t mod 64); k~_t = RoPE(h_k, t); append k~_t, v~_t
 * to the dil cache if t mod D_h = D_h - 1, to ring slot t mod W and to the sink rows if
 * t < n_sink; then attention of RoPE(q, t) over the dil entries with position <= t - We, the
 * ring positions t-We < j < t, the sinks older than the window that are not chunk ends, and the
 * token itself -- the same key set S(t) as in prefill.  Split over the
 * keys across CTAs, combined by log-sum-exp.  Advances cache->pos by 1 on the host.
 * Requires pos < Tcap.
 * ---------------------------------------------------------------------------------------- */
RAT_API size_t rat_decode_workspace_bytes(const rat_kv_cache *cache);

RAT_API int rat_dilated_decode(const void *q, const void *k, const void *v, const void *gate_logit,
                       rat_kv_cache *cache, void *o, float rope_base, float scale,
                       void *ws, size_t ws_bytes, void *stream);

/* ------------------------------------------------------------------------------------------
 * Paged compressed cache with per-sequence positions, for serving: sequences of different
 * lengths decode in one launch.  The content is that of rat_kv_cache (the pages' D-fold
 * compressed cache: chunk-end entries, the window ring, the recurrence state); how it is laid
 * out in memory is this library's (the pages describe no memory management).
 *
 *   k_pool, v_pool : device [n_pages][page_entries][d] of dtype
 *   page_table     : device int32 [B][H][max_pages]: dil entry i of slice (b, h) -- position
 *                    i*D_h + D_h - 1 -- is row page_table[b][h][i / page_entries] * page_entries
 *                    + (i mod page_entries) of the pool.  Every table entry that a call reaches
 *                    must name a page in [0, n_pages); one that does not is skipped and records
 *                    RAT_ERR_INVALID in the workspace header (see rat_sync_status).
 *   k_win, v_win   : device [B][H][W][d] ring, position p in slot p mod W (NULL if W = 0)
 *   h_k, h_v       : device float32 [B][H][d], each sequence's state after its last position
 *   pos            : device int64 [B], positions consumed by each sequence: set by
 *                    rat_paged_kv_compress, advanced by one on the device by every
 *                    rat_dilated_decode_paged (so a captured CUDA graph of decode steps replays
 *                    with the positions moving)
 *   page_entries   : a power of two; a slice holds at most max_pages * page_entries dil entries
 *                    (positions beyond are attended through the window only while in it, as in
 *                    rat_kv_cache with Tcap = max_pages * page_entries * D_h)
 *   reset_every    : as in rat_kv_cache
 * The struct is host memory; the caller owns every buffer and fills the page table.
 * ---------------------------------------------------------------------------------------- */
typedef struct rat_paged_kv_cache {
    int32_t B, H, d, W;       /* batch, heads, head dim, local window (0 = none)           */
    int32_t dtype;            /* rat_dtype of the pools and the ring                        */
    int32_t page_entries;     /* dil entries per page (power of two)                        */
    int32_t max_pages;        /* page-table entries per (b, h) slice                        */
    int32_t n_pages;          /* pages in each pool                                         */
    const int32_t *D;         /* host int32[H]: dilation of each head (>= 1)               */
    void *k_pool, *v_pool;    /* device pools, see above                                    */
    const int32_t *page_table;/* device int32 [B][H][max_pages]                             */
    void *k_win, *v_win;      /* device ring, or NULL when W == 0                          */
    float *h_k, *h_v;         /* device float32 state                                      */
    int64_t *pos;             /* device int64 [B]                                           */
    int64_t reset_every;      /* recurrence block length L, or 0 (full sequence)           */
} rat_paged_kv_cache;

/* rat_paged_kv_compress -- append positions pos0 .. pos0+T-1 of sequence b to a paged cache.
 *   k_rec, v_rec : device (1, H, T, d) of cache->dtype, recurrence outputs of those positions
 *   hT_k, hT_v   : device (1, H, d) float32 state after them (copied into the cache's slot b)
 *   ws, ws_bytes : workspace of at least 256 bytes, 256-byte aligned (error header)
 * Writes every position p with p mod D_h = D_h - 1 (and p / D_h below the slice capacity) to its
 * pool row, the last min(W, T) positions to their ring slots, the state, and pos[b] = pos0 + T
 * (on the device, in stream order).  Bit-exact copies.  0 <= b < B; pos0 >= 0. */
RAT_API int rat_paged_kv_compress(const void *k_rec, const void *v_rec, const float *hT_k,
                          const float *hT_v, int T, int b, int64_t pos0,
                          rat_paged_kv_cache *cache, void *ws, size_t ws_bytes, void *stream);

/* rat_dilated_decode_paged -- rat_dilated_decode for every sequence b at its own position
 * t_b = pos[b] (read on the device), over the paged cache, then pos[b] = t_b + 1.  Arguments,
 * results and numerics as rat_dilated_decode; ws of at least rat_paged_decode_workspace_bytes.
 * When t_b mod D_h = D_h - 1 the table must name a page for entry t_b / D_h below the slice
 * capacity; otherwise the entry is not stored and RAT_ERR_INVALID is recorded. */
RAT_API size_t rat_paged_decode_workspace_bytes(const rat_paged_kv_cache *cache);

RAT_API int rat_dilated_decode_paged(const void *q, const void *k, const void *v,
                             const void *gate_logit, rat_paged_kv_cache *cache, void *o,
                             float rope_base, float scale, void *ws, size_t ws_bytes,
                             void *stream);

/* Test hook for failure detection (no counterpart in the method): the next rat_recur_prefill,
 * rat_recur_prefill_local, rat_recur_backward or rat_recur_backward_local issued from the calling
 * host thread withholds the look-back publication of chunk `chunk` (chunk index >= 1 along the
 * sequence, in every (b, h) and channel slice; a prefill chunk is 128 rows of 64 channels for
 * bf16, d = 128 and T a multiple of 16, else 16 KiB of each tensor's rows; a backward chunk is
 * 64 rows for bf16 and 32 for float32) and bounds each look-back wait by wait_limit_ns
 * (1 ms .. 2 s).  The chunks that wait for it (after it for the prefill, before it for the
 * backward) run out of time, the call's results are wrong, and rat_sync_status() reports
 * RAT_ERR_TIMEOUT; nothing hangs and the context stays usable.  Returns RAT_ERR_INVALID for
 * out-of-range arguments. */
RAT_API int rat_debug_inject_lookback_fault(int64_t chunk, int64_t wait_limit_ns);

/* rat_dilated_decode_noalloc -- the same decode step, for callers that cannot allocate.
 * (The pages have no counterpart: this is a property of the library, not of the method.)
 * Some callers cannot give the library a device buffer for the decode workspace: their device
 * memory belongs to a host framework or is planned up front as a fixed arena, and they have no
 * way to ask for one more allocation.  This entry point allocates nothing; it uses a fixed
 * 8 MiB scratch array compiled into the library (each GPU that loads the library holds it until
 * the process exits) and otherwise runs exactly rat_dilated_decode.
 *   - Arguments and results are those of rat_dilated_decode, without ws / ws_bytes.
 *   - Returns RAT_ERR_WORKSPACE when rat_decode_workspace_bytes(cache) exceeds 8 MiB (for d = 128
 *     that is roughly B * H * splits above 16,000).
 *   - The first call on each device looks up the array's device address (cudaGetSymbolAddress)
 *     with that device current; make that first call before any stream capture.  The address
 *     is kept per device index for the life of the process, in the primary context: it is not
 *     looked up again after cudaDeviceReset, nor for a context the caller created itself, so
 *     such callers must not use this entry point afterwards (or in that context).
 *   - Every call shares the one array, which keeps the previous call's contents; each call
 *     clears its header and tickets on `stream` first.  Calls that overlap on the GPU (other
 *     streams, other host threads) race on the array and must be serialised by the caller.
 *   - The array is not reachable by rat_sync_status(); decode has no device-side waits. */
RAT_API int rat_dilated_decode_noalloc(const void *q, const void *k, const void *v,
                                       const void *gate_logit, rat_kv_cache *cache, void *o,
                                       float rope_base, float scale, void *stream);

/* Number of keys query t attends to: min(We, t+1) + max(0, floor((t - We + 1) / D)).
 * Host-only helper used for FLOP and byte accounting. */
RAT_API int64_t rat_attended_keys(int64_t t, int D, int W);

#ifdef __cplusplus
}
#endif

#endif /* RAT_H_ */
