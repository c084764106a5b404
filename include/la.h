/*
 * la.h -- C ABI of liblinattn: causal linear attention on NVIDIA B200 (sm_100a).
 *
 * The operations are those of the lesson page "Линейное внимание и гибриды"
 * ("Linear attention and hybrids", ai.flicky.cc, stage 5.5), cited by section:
 *   [kernel trick]  "Ядерный трюк: убираем softmax"  -- phi(x) = elu(x) + 1, S_i, z_i
 *   [three forms]   "Три формы одного вычисления"    -- recurrent and chunked forms
 *   [decay/gates]   "Память должна забывать: затухание и гейты" -- gamma, alpha_t gates
 *   [delta rule]    "Дельта-правило и Gated DeltaNet" -- delta rule, Gated DeltaNet
 *
 * Four variants ("modes"), each with a chunked prefill and a one-token decode step.
 * Per (batch, head), for t = 1..T, the state is updated first and then read:
 *
 *   LA_MODE_ELU1_NORM ([kernel trick], [three forms]):
 *       S_t = S_{t-1} + v_t phi(k_t)^T,  z_t = z_{t-1} + phi(k_t),
 *       o_t = S_t phi(q_t) / (z_t . phi(q_t)).
 *   LA_MODE_GATED ([decay/gates]; no feature map, no denominator):
 *       S_t = a_t S_{t-1} + v_t k_t^T,   o_t = S_t q_t.
 *   LA_MODE_GATED_DELTA ([delta rule], the Gated DeltaNet equation):
 *       S_t = a_t S_{t-1} (I - b_t k_t k_t^T) + b_t v_t k_t^T,   o_t = S_t q_t.
 *   LA_MODE_KDA ([delta rule], Kimi Delta Attention: the scalar a_t replaced by the
 *   diagonal matrix Diag(a_t), one decay per memory channel, the d_k columns of S):
 *       S_t = S_{t-1} Diag(a_t) (I - b_t k_t k_t^T) + b_t v_t k_t^T,   o_t = S_t q_t.
 *   LA_MODE_RETNET ([decay/gates], the constant decay gamma of RetNet / Lightning
 *   attention): S_t = g_h S_{t-1} + v_t k_t^T, o_t = S_t q_t, with one fixed gate g_h per
 *   head; `gate` is then [H] (required) and no per-token gate tensor is read.
 *
 * No 1/sqrt(d) scale is applied inside the attention; callers scale q and k.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * Pointers: every tensor argument is a DEVICE pointer (memory the current CUDA device
 *   can address: cudaMalloc, torch CUDA tensors, managed memory).  Host pointers are
 *   rejected with LA_ERR_INVALID_ARG before anything is launched.  The caller owns all
 *   buffers; the library allocates no device memory and keeps no pointer after the call
 *   returns.  Tensors are dense, row-major, and 16-byte aligned (gate and beta: 4-byte).
 * Dtypes: q, k, v, o have the I/O dtype (LA_F32 or LA_BF16).  state, z, gate and beta
 *   are always fp32; all accumulation is fp32.
 * Sizes: d_k and d_v are each 64 or 128.  B, H, N >= 1.  T >= 0.
 * Gates: gate holds the decay values a_t in [0, 1] (not their logarithms); NULL means
 *   a_t = 1.  In mode 3 it holds d_k values per token (one per channel); in mode 4 one
 *   value per head, [H].  beta holds b_t in [0, 1].  Mode 0 ignores gate and beta;
 *   modes 1 and 4 ignore beta; modes 2 and 3 require beta; mode 4 requires gate.
 * State layout: S is d_v x d_k per head, exactly the page's S ([three forms]), stored
 *   [.., d_v, d_k] row-major; z is [.., d_k].  A state written by la_prefill is the
 *   input of la_decode_step, and vice versa.
 * Streams: `stream` is a cudaStream_t (NULL = the legacy default stream).  Argument
 *   checks run on the host and finish before anything is enqueued; the work itself
 *   runs asynchronously on `stream`.  LA_OK means "enqueued"; device-side failures are
 *   reported by la_check_status().
 * Thread safety: the entry points keep no per-call state and may be called from
 *   several host threads.
 */
#ifndef LINATTN_LA_H
#define LINATTN_LA_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    LA_MODE_ELU1_NORM = 0,   /* phi = elu+1, z-normalised                 */
    LA_MODE_GATED = 1,       /* scalar gate a_t, identity feature map     */
    LA_MODE_GATED_DELTA = 2, /* Gated DeltaNet: gate a_t and delta rate b_t */
    LA_MODE_KDA = 3,         /* Kimi Delta Attention: per-channel gate a_t [d_k], rate b_t */
    LA_MODE_RETNET = 4       /* constant decay: mode 1 with one fixed gate per head, [H] */
} la_mode_t;

typedef enum {
    LA_F32 = 0,              /* q, k, v, o in fp32 */
    LA_BF16 = 1              /* q, k, v, o in bf16 (round-to-nearest-even on output) */
} la_dtype_t;

typedef enum {
    LA_OK = 0,
    LA_ERR_INVALID_ARG = 1,  /* a NULL / host / misaligned pointer, a bad size, mode or dtype */
    LA_ERR_UNSUPPORTED = 2,  /* a valid request this build has no kernel for */
    LA_ERR_CUDA = 3,         /* a CUDA runtime error at launch or while checking status */
    LA_ERR_TIMEOUT = 4       /* a kernel's bounded wait ran out; its outputs are invalid */
} la_status_t;

/* la_prefill flag: read `state` (and `z`) as the initial state S_0 (z_0).  Without it
 * S_0 = 0 and z_0 = 0, and `state` / `z` are only written. */
#define LA_FLAG_INIT_STATE 1u

/*
 * la_prefill -- the chunkwise-parallel ("chunked") form of [three forms] over a whole
 * sequence per (batch, head): inside a chunk of C tokens the masked C x C matrix, across
 * chunks the carried state; with the decay mask of [decay/gates] in mode 1 and the
 * delta-rule correction of [delta rule] in mode 2.  The result equals the recurrent
 * form above up to rounding.
 *
 *   q, k   [B, H, T, d_k]  I/O dtype
 *   v      [B, H, T, d_v]  I/O dtype
 *   gate   [B, H, T] fp32 or NULL      beta [B, H, T] fp32 (modes 2, 3) or NULL
 *          (mode 3: gate [B, H, T, d_k])
 *   state  [B, H, d_v, d_k] fp32       in (if LA_FLAG_INIT_STATE) and out: S_T
 *   z      [B, H, d_k] fp32            mode 0 only (else ignored, may be NULL): in/out z_T
 *   o      [B, H, T, d_v]  I/O dtype   out: o_1..o_T
 *   chunk  tokens per chunk; 0 picks the kernel's default.  bf16 with d_k = d_v = 128
 *          runs on the tensor cores at chunk 0 or 64; bf16 at chunk 32, fp32 and d = 64
 *          run on CUDA cores and accept 0, 32 and 64 (64 only when d_k = d_v = 64).
 *          Other values return LA_ERR_UNSUPPORTED.  In mode 3 the tensor-core kernel
 *          takes every gate as given in the state-facing terms (the read of the chunk's
 *          start state, the state's decay and update); only inside the chunk's Gram
 *          products, whose factors are split around reference tokens, is each log2 gate
 *          bounded below at -7.5 (a >= 0.0055), which moves only terms that a gate below
 *          0.0055 has already shrunk (measured <= 1 % of the outputs with gates down to
 *          1e-6).  Chunk 32 selects the CUDA-core kernel, which takes every gate as is.
 *   flags  0 or LA_FLAG_INIT_STATE.
 *   workspace, workspace_bytes
 *          optional device scratch owned by the caller (NULL / 0 allowed).  With at least
 *          la_prefill_workspace_size() bytes the tensor-core kernels take their fastest
 *          form: modes 2 and 3 with 16 to 37 head rows (B*H) first form every chunk's
 *          state-independent factors into the workspace (mode 2: 24 KB per chunk and head
 *          row; mode 3: 66 048 bytes, and the gate tensor 16-byte aligned), then carry the
 *          state through the chunks; other calls split each sequence into segments
 *          processed in parallel and chain their states exactly.  With less they take the
 *          fastest plan that fits (mode 2 with 16 to 37 head rows: its single pass; other
 *          calls: a smaller segment plan, or one pass per sequence), with the same result
 *          up to rounding.  Calls that share a workspace must not overlap on the device.
 * T = 0 is allowed: nothing is read from q, k, v, o; the state is left as given (with
 * LA_FLAG_INIT_STATE) or zeroed.  q, k, v, o may then be NULL.
 * o must not overlap q, k, v or the state.
 */
la_status_t la_prefill(la_mode_t mode, la_dtype_t dtype, int B, int H, int T, int d_k, int d_v,
                       const void *q, const void *k, const void *v,
                       const float *gate, const float *beta,
                       float *state, float *z, void *o,
                       int chunk, unsigned flags, void *workspace, size_t workspace_bytes,
                       void *stream);

/*
 * la_prefill_varlen -- la_prefill over N packed sequences of different lengths, each
 * with its own state: the batch of a serving step, or a prompt resumed from a cached
 * prefix state.  Sequence s is tokens [cu_seqlens[s], cu_seqlens[s+1]) of the packed
 * token axis; nothing crosses from one sequence into the next, exactly as if each were
 * a separate la_prefill call.  (Inside one sequence, a gate a_t = 0 forgets everything
 * before token t, the document-boundary reading of [decay/gates].)
 *
 *   cu_seqlens  [N + 1] int32, DEVICE memory: non-decreasing offsets within [0, T]
 *               (cu_seqlens[0] = 0 and cu_seqlens[N] = T in the usual case).  Entries
 *               outside [0, T] or decreasing are clamped on the device and reported as
 *               LA_ERR_INVALID_ARG by la_check_status().  Empty sequences are allowed.
 *   q, k        [H, T, d_k]  I/O dtype (the [1, H, T, d] layout of la_prefill)
 *   v, o        [H, T, d_v]  I/O dtype
 *   gate        [H, T] fp32 or NULL (mode 3: [H, T, d_k])     beta [H, T] fp32 (modes 2, 3)
 *   state       [N, H, d_v, d_k] fp32: in (with LA_FLAG_INIT_STATE: each sequence's
 *               start state, e.g. a cached prefix's final state) and out (each
 *               sequence's final state -- the snapshot to cache or to decode from)
 *   z           [N, H, d_k] fp32, mode 0 only, in/out like state
 *   chunk, flags as for la_prefill.  No workspace: one CTA per (sequence, head).
 */
la_status_t la_prefill_varlen(la_mode_t mode, la_dtype_t dtype, int N, int H, int T, int d_k,
                              int d_v, const int *cu_seqlens, const void *q, const void *k,
                              const void *v, const float *gate, const float *beta,
                              float *state, float *z, void *o, int chunk, unsigned flags,
                              void *stream);

/*
 * la_prefill_workspace_size -- bytes of workspace la_prefill can use for these sizes
 * (0 when the kernel for them needs none).  Host-only; touches no device.
 */
size_t la_prefill_workspace_size(la_mode_t mode, la_dtype_t dtype, int B, int H, int T, int d_k,
                                 int d_v, int chunk);

/*
 * la_prefill_noalloc -- la_prefill for callers that cannot allocate device memory.
 * The pages have no counterpart: this is an interface for such callers, e.g. code that
 * runs inside another framework's memory pool (a cudaMalloc there bypasses the pool)
 * or a process that reserves all device memory at start-up.  It takes the same
 * arguments as la_prefill except the workspace, which it takes from a 24 MiB array
 * that the library keeps in device memory (every GPU that loads the library holds it
 * until exit).  It allocates nothing and calls no allocating routine.
 *   - Runs the fastest segment plan whose workspace fits in 24 MiB
 *     (la_prefill_workspace_size() reports the fastest plan's need, which may be larger),
 *     or, when none fits, the single pass that needs no workspace: it accepts exactly the
 *     problems la_prefill accepts and returns the same statuses.
 *   - The first call on a device looks up the array's device address (with that device
 *     current); make that first call before any stream capture on the device.
 *   - All calls share the array and it keeps the last call's contents (no result
 *     depends on them).  Calls that overlap on the GPU race on it: serialise them.
 */
la_status_t la_prefill_noalloc(la_mode_t mode, la_dtype_t dtype, int B, int H, int T, int d_k,
                               int d_v, const void *q, const void *k, const void *v,
                               const float *gate, const float *beta, float *state, float *z,
                               void *o, int chunk, unsigned flags, void *stream);

/*
 * la_decode_step -- one token of the recurrent form ([three forms] "recurrent form",
 * [decay/gates], [delta rule]) for N independent sequences, updating the state in place:
 * the per-token cost is O(d_k d_v) and independent of how many tokens came before.
 *
 *   q, k   [N, H, d_k]  I/O dtype       v [N, H, d_v]  I/O dtype
 *   gate   [N, H] fp32 or NULL          beta [N, H] fp32 (modes 2, 3) or NULL
 *          (mode 3: gate [N, H, d_k])
 *   state  [N, H, d_v, d_k] fp32 in/out z [N, H, d_k] fp32 in/out (mode 0 only)
 *   o      [N, H, d_v] I/O dtype out
 */
la_status_t la_decode_step(la_mode_t mode, la_dtype_t dtype, int N, int H, int d_k, int d_v,
                           const void *q, const void *k, const void *v,
                           const float *gate, const float *beta,
                           float *state, float *z, void *o, void *stream);

/* Flags of la_short_conv / la_short_conv_step. */
#define LA_CONV_SILU 2u     /* y = u * sigmoid(u) after the convolution */
#define LA_CONV_L2NORM 4u   /* then every head's row y /= sqrt(sum_d y^2 + 1e-6) */

/*
 * la_short_conv -- the short causal depthwise convolution over time that Gated DeltaNet
 * and KDA layers put in front of q, k and v (section "Hybrids of 2025: Qwen3-Next and
 * Kimi Linear": kernel width 4, each token mixed with the three before it).  Per
 * channel c (C = H * d channels), with the carried window x_{-1} .. x_{-(width-1)}:
 *
 *   u_t[c] = sum_{i < width} w[c][i] x_{t-(width-1)+i}[c]      (tap width-1: token t)
 *
 * then, per flags, SiLU (LA_CONV_SILU) and the L2 norm of every head's d-row
 * (LA_CONV_L2NORM), in that order; fp32 arithmetic, one rounding to the I/O dtype.
 * The page fixes only the causal depthwise convolution and its width; the bias-free
 * taps, the activation and the norm's 1e-6 are this library's reading.
 *
 *   x           [B, T, H*d]          I/O dtype, token-major (a projection's output)
 *   w           [H*d, width]         fp32 taps
 *   window_in   [B, width-1, H*d]    I/O dtype, the inputs before x_0 (oldest first), or
 *                                    NULL for zeros
 *   window_out  [B, width-1, H*d]    I/O dtype, out: the last width-1 rows of
 *                                    [window_in; x], or NULL.  May be window_in itself
 *                                    (the window is then updated in place); any other
 *                                    overlap is LA_ERR_INVALID_ARG.
 *   y           [B, H, T, d]         I/O dtype, head-major: the q / k / v input of
 *                                    la_prefill.  Must not overlap x or the windows.
 *   d in {64, 128}; width in 1..4 (width 1 takes no window); T >= 0 (T = 0 only
 *   copies the window).  16-byte alignment for x, y and the windows, 4 for w.
 */
la_status_t la_short_conv(la_dtype_t dtype, int B, int T, int H, int d, int width,
                          const void *x, const float *w, const void *window_in,
                          void *window_out, void *y, unsigned flags, void *stream);

/*
 * la_short_conv_varlen -- la_short_conv over N packed sequences of different lengths,
 * each with its own carried window (sequence s = tokens [cu_seqlens[s],
 * cu_seqlens[s+1]) of the packed axis; nothing crosses from one sequence into the next).
 *   cu_seqlens  [N + 1] int32, DEVICE memory, as for la_prefill_varlen (entries outside
 *               [0, T] or decreasing are clamped and reported by la_check_status())
 *   x           [T, H*d]             I/O dtype, the packed projection output
 *   window_in   [N, width-1, H*d]    or NULL (zeros); window_out likewise (may be
 *                                    window_in itself)
 *   y           [H, T, d]            I/O dtype: the q / k / v input of la_prefill_varlen
 * Two launches: the convolution, then the carried windows (and the offsets check).
 */
la_status_t la_short_conv_varlen(la_dtype_t dtype, int N, int T, int H, int d, int width,
                                 const int *cu_seqlens, const void *x, const float *w,
                                 const void *window_in, void *window_out, void *y,
                                 unsigned flags, void *stream);

/*
 * la_short_conv_step -- la_short_conv for one new token of N sequences (decoding):
 *   x [N, H*d], window [N, width-1, H*d] updated in place (required when width > 1),
 *   y [N, H, d] (the q / k / v input of la_decode_step); w and flags as above.
 */
la_status_t la_short_conv_step(la_dtype_t dtype, int N, int H, int d, int width,
                               const void *x, const float *w, void *window, void *y,
                               unsigned flags, void *stream);

/*
 * la_prefill_conv -- a Gated DeltaNet layer's attention path from its projections: the
 * short convolution of section "Hybrids of 2025: Qwen3-Next and Kimi Linear" (as
 * la_short_conv) fused into the loads of the gated-delta prefill ([delta rule], mode 2, as
 * la_prefill with a workspace).  The prefill's first pass
 * reads the token-major projections with the three tokens in front of each chunk,
 * convolves them as they arrive and writes the convolved q, k, v once; the second pass
 * reads those.  The results equal three la_short_conv calls followed by la_prefill (mode
 * 2) on the same two-pass kernels, bit for bit.
 *
 *   dtype        LA_BF16 (LA_F32: LA_ERR_UNSUPPORTED)
 *   d            128 (= d_k = d_v; 64: LA_ERR_UNSUPPORTED); width 1..4
 *   xq, xk, xv   [B, T, H*d] token-major projections
 *   wq, wk, wv   [H*d, width] fp32 taps
 *   window_in    [3, B, width-1, H*d] the q, k, v windows in front of x_0, or NULL (zeros)
 *   window_out   [3, B, width-1, H*d] out, or NULL; must not overlap window_in
 *   flags_qk, flags_v   LA_CONV_SILU | LA_CONV_L2NORM for q and k, for v
 *   y            [3, B, H, T, d] out: the convolved q, k, v (the backward pass takes them)
 *   gate, beta, state, o, flags   as la_prefill in mode 2 (gate [B, H, T] or NULL)
 *   workspace    at least la_prefill_conv_workspace_size() bytes (required), 16-byte aligned
 * T >= 1.  No output may overlap an input; LA_ERR_INVALID_ARG otherwise.  Two launches.
 */
size_t la_prefill_conv_workspace_size(int B, int H, int T);
la_status_t la_prefill_conv(la_dtype_t dtype, int B, int H, int T, int d, int width, const void *xq,
                            const void *xk, const void *xv, const float *wq, const float *wk,
                            const float *wv, const void *window_in, void *window_out,
                            unsigned flags_qk, unsigned flags_v, void *y, const float *gate,
                            const float *beta, float *state, void *o, unsigned flags,
                            void *workspace, size_t workspace_bytes, void *stream);

/*
 * la_prefill_backward -- gradients of the prefill for the scalar-gate modes (1 and 4):
 * the derivatives of L = sum_t do_t . o_t + <dS_T, S_T> for the recurrence of
 * [decay/gates], S_t = a_t S_{t-1} + v_t k_t^T, o_t = S_t q_t, with respect to q, k, v, the
 * gates and the initial state.  The chunked form ([three forms]) is the one the page uses
 * for training; it gives no backward formulas, so they are the plain derivatives:
 *   dQ = diag(g) dO S_c + dP K,  dK = dP^T Q + diag(g_L/g) V G,  dV = P^T dO + diag(g_L/g) K G^T
 * per chunk (P = (Q K^T) o D, dP = (dO V^T) o D, S_c the chunk-start state, G = dL/dS at
 * the chunk's end), and d log a_t = sum_{u >= t} (q_u . dq_u - k_u . dk_u) (plus
 * <dS_T, S_T> at the last token).  Warp-level tensor-core products with fp32 accuracy
 * (computed operands split into high and low parts), fp32 accumulation.  bf16 I/O: three
 * launches (the chunk-start states and chunk-end cotangents, every chunk's gradients, the
 * gate gradient); fp32 I/O: two (forward and reverse sweeps, then dv and the gate gradient).
 *
 *   mode          LA_MODE_GATED or LA_MODE_RETNET (others: LA_ERR_UNSUPPORTED)
 *   q, k          [B, H, T, d_k] I/O dtype      v, dO [B, H, T, d_v] I/O dtype
 *   gate          as for la_prefill (mode 1: [B, H, T] or NULL; mode 4: [H], required)
 *   state0        [B, H, d_v, d_k] fp32 initial state, or NULL for zero
 *   dstate        [B, H, d_v, d_k] fp32 cotangent of the final state, or NULL for zero
 *   dq, dk, dv    out, shapes of q, k, v, I/O dtype
 *   dgate         out [B, H, T] fp32 (mode 1 with a gate), or NULL; mode 4 takes its
 *                 gates as fixed and requires NULL.  Gates must be > 0: d a = d log a / a.
 *   dstate0       out [B, H, d_v, d_k] fp32 (the gradient of state0), or NULL
 *   workspace     device scratch of at least la_backward_workspace_size() bytes
 *                 (required: every chunk-start state, and with bf16 I/O every chunk-end
 *                 cotangent, is kept there)
 * la_backward_workspace_size also sizes la_prefill_backward_delta's workspace (modes 2, 3).
 */
size_t la_backward_workspace_size(la_mode_t mode, int B, int H, int T, int d_k, int d_v);
la_status_t la_prefill_backward(la_mode_t mode, la_dtype_t dtype, int B, int H, int T, int d_k,
                                int d_v, const void *q, const void *k, const void *v,
                                const float *gate, const float *state0, const void *dO,
                                const float *dstate, void *dq, void *dk, void *dv, float *dgate,
                                float *dstate0, void *workspace, size_t workspace_bytes,
                                void *stream);

/*
 * la_prefill_backward_delta -- gradients of the prefill for the delta-rule modes (2 and 3):
 * the derivatives of L = sum_t do_t . o_t + <dS_T, S_T> for the update of [delta rule],
 * S_t = S_{t-1} A_t (I - b_t k_t k_t^T) + b_t v_t k_t^T with A_t = a_t I (Gated DeltaNet) or
 * Diag(a_t) (Kimi Delta Attention), o_t = S_t q_t, with respect to q, k, v, the gates, the
 * rates b and the initial state.  The pages give no backward formulas; these are the plain
 * derivatives, taken through the chunked form ([three forms]) with its WY factors
 * T = (I + diag(b) Kgr)^-1, W = T diag(b) Kg, U = T diag(b) V, E = U - W S^T per chunk
 * of 32 tokens; the gate gradient is d log a_t = (suffix sum within the chunk of
 * dL/dlam), da_t = d log a_t / a_t.  CUDA cores, fp32 arithmetic; d_v is split over CTAs of
 * 32 state rows each.
 *
 *   mode          LA_MODE_GATED_DELTA or LA_MODE_KDA (others: LA_ERR_UNSUPPORTED)
 *   q, k          [B, H, T, d_k] I/O dtype      v, dO [B, H, T, d_v] I/O dtype
 *   gate          [B, H, T] fp32 (mode 3: [B, H, T, d_k]) or NULL (a = 1); the gate gradient
 *                 divides by a_t, so a gate of exactly 0 gives no finite dgate there
 *   beta          [B, H, T] fp32, required
 *   state0        [B, H, d_v, d_k] fp32 or NULL (zero)
 *   dstate        [B, H, d_v, d_k] fp32 cotangent of S_T, or NULL (zero)
 *   dq, dk        out [B, H, T, d_k] I/O dtype   dv out [B, H, T, d_v] I/O dtype
 *   dgate         out, shaped like gate, or NULL (then not computed); needs gate
 *   dbeta         out [B, H, T] fp32, or NULL
 *   dstate0       out [B, H, d_v, d_k] fp32, or NULL
 *   workspace     device scratch of at least la_backward_workspace_size() bytes (every
 *                 chunk-start state and fp32 accumulators of dq, dk, db and the gate terms)
 * d_k, d_v in {64, 128} (else LA_ERR_UNSUPPORTED); T >= 1.  Every pointer is device memory
 * of the current device (16-byte aligned for the tensors of the I/O dtype and the
 * workspace).  The buffers the call writes (dq, dk, dv, dgate, dbeta, dstate0, workspace)
 * must not overlap one another or any input (LA_ERR_INVALID_ARG).  Asynchronous on
 * `stream`; the caller keeps every buffer alive until the stream has passed the call.
 */
la_status_t la_prefill_backward_delta(la_mode_t mode, la_dtype_t dtype, int B, int H, int T,
                                      int d_k, int d_v, const void *q, const void *k,
                                      const void *v, const float *gate, const float *beta,
                                      const float *state0, const void *dO, const float *dstate,
                                      void *dq, void *dk, void *dv, float *dgate, float *dbeta,
                                      float *dstate0, void *workspace, size_t workspace_bytes,
                                      void *stream);

/*
 * la_check_status -- synchronise `stream`, then report the first device-side failure
 * since the last call: LA_ERR_CUDA for a CUDA error, LA_ERR_TIMEOUT if a kernel's
 * bounded wait ran out (the kernel then returned early and its outputs are invalid),
 * LA_ERR_INVALID_ARG if a kernel met an invalid device-side argument (a cu_seqlens
 * entry out of range).
 * Clears the recorded failure.  Returns LA_OK if nothing failed.
 */
la_status_t la_check_status(void *stream);

/*
 * la_selftest_wait_timeout -- a diagnostic of the failure path: enqueues one small
 * kernel that waits, with the bounded wait every pipeline kernel uses, on a barrier
 * nothing completes.  The wait gives up after its poll limit (well under a second),
 * records the timeout and returns; the next la_check_status() reports LA_ERR_TIMEOUT
 * and the device stays usable.  Touches no caller memory.
 */
la_status_t la_selftest_wait_timeout(void *stream);

/* A static, human-readable description of a status code. */
const char *la_status_string(la_status_t status);

/* Library version, major * 10000 + minor * 100 + patch. */
int la_version(void);

/* Number of kernels this library has enqueued in this process (all devices, all
 * threads), a monotonically increasing diagnostic counter. */
unsigned long long la_kernel_launches(void);

/* Per-launch device timing, a measurement aid with no counterpart in the pages.
 * la_launch_timing(1) makes every later call of la_prefill, la_prefill_noalloc,
 * la_prefill_varlen, la_prefill_backward, la_prefill_backward_delta, la_decode_step and
 * the la_short_conv* entry
 * points bracket each
 * kernel it enqueues
 * with two CUDA events recorded on the call's stream (at most 16 launches per call are
 * timed); la_launch_timing(0) turns it off (the default).  Enabling adds two event
 * records per launch.
 *
 * la_launch_times(ms, max_n) waits for the last timed launch of the most recent call,
 * writes the device duration of each of its first max_n launches, in milliseconds and
 * launch order, to the HOST array ms, and returns how many it wrote: 0 when timing is
 * off or the call launched nothing, -1 on a null ms, a negative max_n or a CUDA error.
 * The state is process-wide: calls from several threads at once interleave. */
la_status_t la_launch_timing(int enable);
int la_launch_times(float *ms, int max_n);

#ifdef __cplusplus
}
#endif

#endif /* LINATTN_LA_H */
