/*
 * gdn.h -- C ABI of the B200 gated-delta-rule library (libgdn.so).
 *
 * The operation (source: "ATMA: Long-Context Language Modeling via Polar
 * Attention and Gated-Delta Compression Memory", Sec. 3.3, the gated-delta
 * memory equation, with the paper's gamma_t written alpha_t, M written S and
 * r written o).  For every batch row b and head h independently, with a
 * d_v x d_k float32 state S:
 *
 *     alpha_t = exp(log_alpha_t)
 *     S_t     = alpha_t S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T
 *     o_t     = S_t q_t                      (the output uses the updated state)
 *
 * No scale is applied to q, and q, k are used as given: callers that want
 * the paper's unit-norm keys and queries (its App. A.2 assumes
 * ||q_t|| = ||k_t|| = 1) normalise them before the call, or call the *_raw
 * entry points below, which normalise them (and map gate logits) in-kernel.
 *
 * Layouts (row-major, contiguous, 64-bit indexing):
 *     q, k            [B, T, H, dk]   dtype (GDN_F32 or GDN_BF16)
 *     v, out          [B, T, H, dv]   dtype
 *     log_alpha, beta [B, T, H]       float32, always
 *     S0, S_final, S  [B, H, dv, dk]  float32, always (row = value index,
 *                                     column = key index; k contiguous)
 * For gdn_decode_step the T axis is absent: q, k [B, H, dk], v, out [B, H, dv],
 * log_alpha, beta [B, H].
 *
 * Memory: every pointer may be device memory (cudaMalloc, stream-ordered or
 * managed) or host memory (pinned or pageable).  Device memory is used in
 * place.  Host buffers are staged through stream-ordered device buffers:
 * host-to-device copies are enqueued on `stream` before the kernels and
 * device-to-host copies of the results after them; with pinned host output
 * memory the results are valid after the stream has been synchronised,
 * with pageable host output memory they are valid when the call returns.
 * One exception for throughput: a gdn_forward / gdn_forward_raw whose q, k,
 * v, gates and out are all pinned host memory (64 MB or more of them) is cut
 * along T into pieces of whole chunks.  The copies of one piece in, the
 * kernels of the next and the copy of another piece out overlap on the
 * library's two copy streams and on `stream`.  The state passes between
 * pieces in float32 on the device.  `stream` still orders after every copy,
 * so results are valid once it has been synchronised.  Set the environment
 * variable GDN_HOST_PIPELINE=0 to stage the whole problem instead.
 * The library keeps no pointer after a call returns and owns no buffer.
 *
 * Streams: `stream` is a cudaStream_t passed as void* (NULL = legacy default
 * stream).  All device work of a call is enqueued on it, apart from the
 * pipelined host copies above; calls are asynchronous unless host staging
 * forces a synchronous copy.  The library's only global state is immutable
 * per-device data: device properties, the scratch pool and the two copy
 * streams.  Calls on different streams may therefore run concurrently,
 * provided their buffers do not overlap.
 *
 * Errors: every entry point returns a gdn_status.  Arguments are validated
 * on the host before anything is enqueued; a rejected call enqueues nothing
 * and writes nothing.  A failed kernel launch returns GDN_ERR_LAUNCH.  Device
 * code never traps; errors raised asynchronously by the device appear at the
 * caller's next synchronisation, as for any CUDA work.
 */
#ifndef GDN_H
#define GDN_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Element type of q, k, v and out.  Gates and states are always float32. */
typedef enum {
    GDN_F32 = 0,  /* float32: arithmetic in float32 (SIMT), for tight parity   */
    GDN_BF16 = 1  /* bfloat16: tensor-core operands, float32 accumulation/state */
} gdn_dtype;

typedef enum {
    GDN_OK = 0,
    GDN_ERR_NULL_PTR = 1,       /* a required pointer is NULL                          */
    GDN_ERR_INVALID_SIZE = 2,   /* negative size, or sizes whose product overflows     */
    GDN_ERR_UNSUPPORTED = 3,    /* dk, dv, chunk or dtype outside the supported set    */
    GDN_ERR_MISALIGNED = 4,     /* misaligned pointer (see Alignment below)            */
    GDN_ERR_ALLOC = 5,          /* stream-ordered workspace/staging allocation failed  */
    GDN_ERR_LAUNCH = 6,         /* a kernel launch or an enqueued copy failed          */
    GDN_ERR_DEVICE_TIMEOUT = 7, /* a bounded device-side wait gave up                  */
    GDN_ERR_ALIAS = 8,          /* an output overlaps an input it must not overlap     */
    GDN_ERR_DEVICE = 9,         /* no usable CUDA device / not an sm_100 device        */
    GDN_ERR_SCRATCH_LIMIT = 10  /* gdn_forward_noalloc: a forced segment count needs more
                                   scratch than GDN_NOALLOC_SCRATCH_BYTES               */
} gdn_status;

/*
 * gdn_forward -- prefill / training forward over T tokens.
 *
 * Computes o_t for t = 1..T and, if S_final != NULL, S_T, starting from S0
 * (S0 == NULL means the zero state).  Chunkwise-parallel: the sequence is cut
 * into chunks of `chunk` tokens; inside a chunk the recurrence is solved in
 * closed form (a unit-lower-triangular UT transform), and the state is passed
 * from chunk to chunk.  The result does not depend on `chunk` beyond
 * rounding.  T need not be a multiple of `chunk`.
 *
 * Arguments:
 *   q, k, v, out   see layouts above; dtype given by `dtype`
 *   log_alpha      log of the decay gate; alpha = exp(log_alpha) in [0, 1].
 *                  -inf (alpha = 0) is accepted; values below -40 act as -40
 *                  (alpha < 5e-18, below float32 resolution of the state)
 *   beta           write strength, used as given (the paper takes [0, 1])
 *   S0             initial state or NULL.  May equal S_final (in place)
 *   S_final        final state or NULL (not written)
 *   B, T, H        batch, tokens, heads.  B == 0, H == 0 or T == 0 are
 *                  valid: with T == 0, S_final receives S0 (or zeros)
 *   dk, dv         key / value head dims, each one of 16, 32, 64, 128
 *   chunk          16, 32 or 64
 *   stream         cudaStream_t
 *   dtype          gdn_dtype of q, k, v, out
 *
 * Aliasing: out must not overlap q, k, v, gates, S0 or S_final; S_final
 * must not partially overlap S0 (exact equality is allowed).
 * Alignment: q, k, v, out, S0, S_final 16-byte aligned; log_alpha and beta
 * 4-byte aligned.
 */
int gdn_forward(const void *q, const void *k, const void *v, const float *log_alpha,
                const float *beta, const float *S0, void *out, float *S_final, int64_t B,
                int64_t T, int64_t H, int64_t dk, int64_t dv, int64_t chunk, void *stream,
                int dtype);

/*
 * gdn_forward_varlen -- gdn_forward over N sequences of different lengths
 * packed along the token axis (prefill of a batch of requests).
 *
 * Same recurrence as gdn_forward (source: the Sec. 3.3 gated-delta memory
 * equation), run independently on each sequence i, which is tokens
 * cu_seqlens[i] .. cu_seqlens[i+1]-1 of the packed tensors; no state flows
 * from one sequence to the next.
 *
 * Arguments:
 *   q, k           [T_total, H, dk]    (packed; dtype given by `dtype`)
 *   v, out         [T_total, H, dv]
 *   log_alpha, beta [T_total, H] float32
 *   cu_seqlens     HOST array of N + 1 int64 offsets: cu_seqlens[0] = 0,
 *                  non-decreasing, cu_seqlens[N] = T_total.  Read during the
 *                  call only.  Empty sequences are allowed.
 *   S0, S_final    [N, H, dv, dk] float32, one state per sequence and head, or
 *                  NULL (zero initial state / not written).  S0 == S_final is
 *                  allowed.
 *   H, dk, dv, chunk, stream, dtype   as for gdn_forward
 *
 * Layout, alignment, aliasing and host-buffer staging rules are those of
 * gdn_forward with B = 1 and T = T_total.  Errors: GDN_ERR_INVALID_SIZE when
 * cu_seqlens is not a valid offset array (NULL with N > 0, cu_seqlens[0] !=
 * 0, decreasing, or cu_seqlens[N] != T_total); the rest as for gdn_forward.
 * bf16 with dk = dv = 128 and chunk = 64 runs the two-kernel tensor-core
 * forward over all sequences at once: one chain per sequence and head, except
 * that a sequence long enough to outlast the others is cut into segments
 * (transfers, a prefix from its S0, and one chain per segment), as a long
 * gdn_forward is; GDN_SEGMENTS=k cuts the longest sequence into k segments.
 * Other shapes run the CUDA-core forward once per sequence.
 */
int gdn_forward_varlen(const void *q, const void *k, const void *v, const float *log_alpha,
                       const float *beta, const int64_t *cu_seqlens, int64_t N, const float *S0,
                       void *out, float *S_final, int64_t T_total, int64_t H, int64_t dk, int64_t dv,
                       int64_t chunk, void *stream, int dtype);

/*
 * gdn_forward_plan -- what a gdn_forward call with these sizes will do on the
 * current device, without doing it: *scratch_bytes receives the device scratch
 * it takes from the library's scratch pool (the per-chunk workspace of the
 * two-kernel tensor-core forward, 32.5 KB per chunk, plus the segment
 * transfers and entry states of long sequences with few heads; excluding host
 * staging), *launches the number of kernels it launches (0 for empty
 * problems).  Either output pointer may be NULL.  Returns the status the
 * argument checks of gdn_forward would return, or GDN_ERR_DEVICE.
 */
int gdn_forward_plan(int64_t B, int64_t T, int64_t H, int64_t dk, int64_t dv, int64_t chunk, int dtype,
                     int64_t *scratch_bytes, int *launches);

/*
 * gdn_decode_step -- one token for every (b, h), state updated in place.
 *
 * Same equation as gdn_forward with T = 1 (source: the Sec. 3.3 gated-delta
 * memory equation): reads S, writes S_1 back into S and o_1 into out.  Each
 * head's state is streamed from memory once and written back once.
 *
 * Arguments: q, k [B, H, dk]; v, out [B, H, dv]; log_alpha, beta [B, H]
 * float32; S [B, H, dv, dk] float32, read and overwritten; dk, dv each one
 * of 16, 32, 64, 128; dtype of q, k, v, out.  B == 0 or H == 0 is a no-op.
 * Aliasing: out must not overlap any input or S.
 * Alignment: q, k, v, out, S 16-byte aligned; log_alpha and beta 4-byte
 * aligned (a per-step slice of a [steps, B, H] gate array is accepted).
 */
int gdn_decode_step(const void *q, const void *k, const void *v, const float *log_alpha,
                    const float *beta, float *S, void *out, int64_t B, int64_t H, int64_t dk,
                    int64_t dv, void *stream, int dtype);

/*
 * The input stage fused: gdn_forward_raw, gdn_forward_varlen_raw and
 * gdn_decode_step_raw take the memory's inputs as the layer produces them
 * and form what the recurrence reads inside the kernels.  The paper's memory
 * reads unit-norm queries and keys (App. A.2 takes ||q_t|| = ||k_t|| = 1), a
 * decay alpha_t in (0, 1) and a write strength beta_t in (0, 1); these calls
 * compute, per (token, head),
 *
 *     q_t <- q_t / sqrt(|q_t|^2 + 1e-12),   k_t <- k_t / sqrt(|k_t|^2 + 1e-12)
 *     log alpha_t = -softplus(x_alpha_t) = -log(1 + exp(x_alpha_t))
 *     beta_t      = sigmoid(x_beta_t)    = 1 / (1 + exp(-x_beta_t))
 *
 * and then run the recurrence of gdn_forward / gdn_forward_varlen /
 * gdn_decode_step on them (the 1e-12 keeps a zero vector at zero).  The
 * normalised q, k are not rounded to dtype: the norms are applied in float32
 * to the products that use q and k.
 *
 * Arguments, layouts, validation, aliasing and staging are those of the
 * matching call, with x_alpha, x_beta (float32 gate logits, the layout of
 * log_alpha, beta) in place of log_alpha, beta, and q, k in any scale.
 * bf16 with dk = dv = 128 and chunk = 64 (and every decode step) runs the
 * stage inside the kernels that already load q, k and the gates, with no pass
 * of its own; other shapes run it as one extra pass (GDN_KERNEL_INPUT) into
 * scratch before the forward.
 */
int gdn_forward_raw(const void *q, const void *k, const void *v, const float *x_alpha,
                    const float *x_beta, const float *S0, void *out, float *S_final, int64_t B,
                    int64_t T, int64_t H, int64_t dk, int64_t dv, int64_t chunk, void *stream,
                    int dtype);
int gdn_forward_varlen_raw(const void *q, const void *k, const void *v, const float *x_alpha,
                           const float *x_beta, const int64_t *cu_seqlens, int64_t N,
                           const float *S0, void *out, float *S_final, int64_t T_total, int64_t H,
                           int64_t dk, int64_t dv, int64_t chunk, void *stream, int dtype);
int gdn_decode_step_raw(const void *q, const void *k, const void *v, const float *x_alpha,
                        const float *x_beta, float *S, void *out, int64_t B, int64_t H, int64_t dk,
                        int64_t dv, void *stream, int dtype);

/*
 * gdn_backward -- reverse mode of gdn_forward (the training backward).
 *
 * For a loss L whose gradients with respect to the forward's outputs are
 * grad_out = dL/dout [B, T, H, dv] (dtype) and grad_S_final = dL/dS_final
 * [B, H, dv, dk] (float32, NULL = zero), writes dL/dq, dL/dk [B, T, H, dk]
 * and dL/dv [B, T, H, dv] in dtype, dL/dlog_alpha and dL/dbeta [B, T, H]
 * float32, and dL/dS0 [B, H, dv, dk] float32 (grad_S0 NULL = not written).
 * q, k, v, log_alpha, beta, S0 (NULL = zero), B, T, H, dk, dv, chunk,
 * stream and dtype are exactly the forward's arguments.  The recurrence is
 * the one of gdn_forward (source: the Sec. 3.3 gated-delta memory equation);
 * the gradient of log_alpha below the forward's floor of -40 is zero.
 *
 * The forward is recomputed, keeping the state entering every chunk in
 * scratch.  For bf16 with dk = dv = 128 and chunk = 64 the reverse mode then
 * runs on the tensor cores: a reverse chain over each (b, h)'s chunks (the
 * adjoint of the state in tensor memory) and a chunk-parallel pass forming
 * every chunk's gradients (scratch about 136 KB per chunk and head: the
 * recompute's workspace, bf16 checkpoints, T of every chunk, and the
 * adjoints passed between the two).  Long sequences with few heads are cut
 * into the forward's segments: the adjoint's map through each segment
 * (affine: the transpose of the segment's forward transfer plus the
 * segment's own term), a prefix over the segments from grad_S_final, then
 * every segment's reverse walk at once (3 x 64 KB more scratch per segment
 * boundary and head).  Every other shape, or
 * GDN_BWD_PATH=simt, walks the chunks backwards with the chunkwise adjoint in
 * float32 on the CUDA cores (checkpoints of dv * dk * 4 bytes per chunk and
 * head, and float32 accumulators of dq and dk for bf16).
 * Alignment and staging as for gdn_forward; no output may overlap an input
 * or another output (GDN_ERR_ALIAS).
 */
int gdn_backward(const void *q, const void *k, const void *v, const float *log_alpha,
                 const float *beta, const float *S0, const void *grad_out,
                 const float *grad_S_final, void *grad_q, void *grad_k, void *grad_v,
                 float *grad_log_alpha, float *grad_beta, float *grad_S0, int64_t B, int64_t T,
                 int64_t H, int64_t dk, int64_t dv, int64_t chunk, void *stream, int dtype);

/*
 * Grouped heads: gdn_forward_grouped and gdn_decode_step_grouped.
 *
 * Hq query heads read the memories of Hkv key-value heads, G = Hq / Hkv
 * query heads per memory.  The memory of key-value head hk is written by
 * its own k, v, log_alpha and beta with the gdn_forward recurrence (source:
 * the Sec. 3.3 gated-delta memory equation).  Query head h = hk * G + g
 * (g < G) reads it: o_t^(h) = S_t^(hk) q_t^(h).  The paper's attention
 * layers have 8 query and 2 key-value heads (Sec. 3) but it does not say how
 * the memory's heads map; this grouped-query mapping is the reading taken.
 *
 * Layouts: q, out [B, T, Hq, .]; k, v [B, T, Hkv, .]; log_alpha, beta
 * [B, T, Hkv]; S0, S_final [B, Hkv, dv, dk].  For the decode step the T
 * axis is absent and S [B, Hkv, dv, dk] is updated in place, once per memory.
 * Hq must be a multiple of Hkv (GDN_ERR_INVALID_SIZE otherwise); for decode
 * G <= 64.  G = 1 is gdn_forward / gdn_decode_step.  Validation, alignment,
 * aliasing and staging are otherwise those of the ungrouped calls.
 *
 * The decode kernel updates each memory once and forms the G outputs from
 * the updated rows.  The forward, for bf16 with dk = dv = 128 and chunk = 64,
 * runs each memory once as well: the two-kernel tensor-core forward runs the
 * memory of key-value head hk on query head hk * G's chunk items (writing
 * that head's outputs, and per chunk the bf16 state entering it and U^T, in
 * scratch; the other query heads' chunk items form only their P tiles and
 * gate records), then one chunk-parallel kernel forms the other query heads'
 * outputs from them.  Other shapes run the CUDA-core forward with
 * per-query-head work items, where each query head recomputes its memory.
 */
int gdn_forward_grouped(const void *q, const void *k, const void *v, const float *log_alpha,
                        const float *beta, const float *S0, void *out, float *S_final, int64_t B,
                        int64_t T, int64_t Hq, int64_t Hkv, int64_t dk, int64_t dv, int64_t chunk,
                        void *stream, int dtype);
int gdn_decode_step_grouped(const void *q, const void *k, const void *v, const float *log_alpha,
                            const float *beta, float *S, void *out, int64_t B, int64_t Hq,
                            int64_t Hkv, int64_t dk, int64_t dv, void *stream, int dtype);

/*
 * gdn_causal_conv -- the short depthwise causal convolution applied to q, k
 * and v before the memory (source: Sec. 3, "Canon depthwise causal
 * convolutions are applied to q, k and v"; the paper fixes neither width,
 * weights nor placement, so this is the plain reading).  Per batch row, channel
 * c (C = heads x head dim) and token t:
 *
 *     y_t[c] = sum_{j < W} weight[c][j] * x_{t-j}[c]
 *
 * x_{-1} .. x_{-(W-1)} come from state_in (NULL = zeros).  No activation is
 * applied; a residual connection is weight[c][0] + 1.
 *
 * Arguments: x, y [B, T, C] dtype; weight [C, W] float32 (W in 1..4);
 * state_in, state_out [B, W-1, C] float32, the last W - 1 inputs, oldest
 * first (NULL = zero history / not written; state_out == state_in updates in
 * place, which is how decode (T = 1) carries it).  y may not overlap any
 * input or state.  T = 0 only passes the state through.
 *
 * It is a pass of its own, bound by HBM: one read of x and one write of y.
 */
int gdn_causal_conv(const void *x, const float *weight, const float *state_in, void *y,
                    float *state_out, int64_t B, int64_t T, int64_t C, int64_t W, void *stream,
                    int dtype);

/*
 * gdn_forward_conv -- the layer's memory input in one call: the short causal
 * convolution of q, k and v (gdn_causal_conv, source: Sec. 3, "Canon"
 * depthwise causal convolutions in front of the memory), then gdn_forward_raw
 * on its outputs:
 *
 *     q' = conv(q), k' = conv(k), v' = conv(v)      (each with its own weights)
 *     out, S_final = gdn_forward_raw(q', k', v', x_alpha, x_beta, S0)
 *
 * The convolution of all three tensors runs as one launch into library
 * scratch (3 x B x T x H x d elements of the input dtype), then the raw
 * forward reads it.  The rounding is gdn_causal_conv's: the convolution in
 * float32 (w0 x_t first, then the older inputs), rounded to the input dtype;
 * the call gives the same bits as gdn_causal_conv on each tensor followed by
 * gdn_forward_raw.
 *
 * Arguments: those of gdn_forward_raw, and
 *   conv_weight     float32 [3][H*d][W]: the q block [H*dk][W], then the k
 *                   block [H*dk][W], then the v block [H*dv][W]
 *   conv_state      float32 [3][B][W-1][H*d], the last W - 1 inputs of each
 *                   tensor before this call, oldest first (blocks q, k, v as
 *                   for the weights), or NULL for a zero history
 *   conv_state_out  the same layout, or NULL (not written); may equal
 *                   conv_state (updated in place)
 *   W               1..4
 * Device memory only (GDN_ERR_UNSUPPORTED for host buffers).  With T == 0
 * S_final receives S0 and conv_state_out receives conv_state (or zeros).
 */
int gdn_forward_conv(const void *q, const void *k, const void *v, const float *x_alpha, const float *x_beta,
                     const float *conv_weight, const float *conv_state, float *conv_state_out, const float *S0,
                     void *out, float *S_final, int64_t B, int64_t T, int64_t H, int64_t dk, int64_t dv, int64_t W,
                     int64_t chunk, void *stream, int dtype);

/*
 * gdn_forward_noalloc -- gdn_forward for callers that cannot allocate device
 * memory during a call.
 *
 * The paper has no counterpart to this entry point; it exists for callers
 * whose device memory is not theirs to allocate mid-call. Examples: a framework
 * whose caching allocator already owns the device heap, a serving loop that
 * must not enter the driver's allocator on its hot path, or code without
 * permission to grow the process's device footprint.
 *
 * Arguments, layouts, results and validation are those of gdn_forward, with
 * these differences:
 *   - every pointer must be device (or managed) memory: host buffers, which
 *     gdn_forward stages through temporary device buffers, are rejected with
 *     GDN_ERR_UNSUPPORTED;
 *   - the scratch lives in one library-owned device array of
 *     GDN_NOALLOC_SCRATCH_BYTES, which every GPU that loads the library holds
 *     until the process exits.  It holds the per-chunk workspace of the
 *     two-kernel tensor-core forward when that fits (32.5 KB per chunk),
 *     else the call runs the single-kernel tensor-core forward, whose only
 *     scratch is the segment transfers and entry states of long sequences
 *     with few heads (3 x 64 KiB per head and segment boundary).  When the
 *     planned segment count needs more than the array holds, the call runs
 *     with the most segments that fit (one segment needs none), so every
 *     supported problem runs, with less chunk-level parallelism; only a
 *     segment count forced through the environment variable GDN_SEGMENTS
 *     that does not fit returns GDN_ERR_SCRATCH_LIMIT, before anything is
 *     enqueued;
 *   - no cudaMalloc, cudaMallocAsync, cudaFree or other allocating routine is
 *     called.
 * The first call on a device looks up the array's device address on that
 * device; make that first call before any stream capture. All calls share the
 * array and it keeps the last call's contents (nothing in it needs to start at
 * zero); calls whose executions overlap on the GPU race on it, so order them
 * on one stream or with events.
 */
#define GDN_NOALLOC_SCRATCH_BYTES (32 * 1024 * 1024)
int gdn_forward_noalloc(const void *q, const void *k, const void *v, const float *log_alpha,
                        const float *beta, const float *S0, void *out, float *S_final, int64_t B,
                        int64_t T, int64_t H, int64_t dk, int64_t dv, int64_t chunk, void *stream,
                        int dtype);

/*
 * gdn_scratch_release -- gdn_forward and gdn_decode_step take their device
 * scratch (the per-chunk workspace, segment transfers, copies of host
 * buffers) from a stream-ordered memory pool private to the library, one per
 * device, that keeps freed memory mapped between calls, so that repeated
 * calls do not map new memory each time.  The paper has no counterpart to
 * this housekeeping call.  It returns the pool's memory that no call is
 * using on the current device to the driver; memory of calls still executing
 * stays with them until they complete.  Returns GDN_OK, or GDN_ERR_DEVICE.
 */
int gdn_scratch_release(void);

/*
 * Per-kernel device times, for benchmarking.  The paper has no counterpart to
 * these two calls.  gdn_timing_start() turns recording on (process-wide) and
 * discards earlier records: from then on every kernel that gdn_forward,
 * gdn_forward_noalloc or gdn_decode_step launches is bracketed by a pair of
 * CUDA events recorded on the caller's stream.  gdn_timing_stop() turns it
 * off, waits for the recorded events and writes, per kernel kind, the summed
 * elapsed milliseconds into ms[kind] and the number of launches into
 * launches[kind] (arrays of GDN_KERNEL_KINDS entries; either may be NULL).
 * Recording adds host-side event records around each launch and nothing on
 * the device path.  Returns GDN_OK, or GDN_ERR_LAUNCH if an event failed.
 */
typedef enum {
    GDN_KERNEL_PREP = 0,        /* two-kernel forward: chunk-parallel prep (P, T diag(beta), W)   */
    GDN_KERNEL_CHAIN = 1,       /* two-kernel forward: state chain and outputs                     */
    GDN_KERNEL_TRANSFER = 2,    /* segment transfers of long sequences (either forward)            */
    GDN_KERNEL_PREFIX = 3,      /* entry states of segments from the transfers                     */
    GDN_KERNEL_FUSED = 4,       /* single-kernel tensor-core forward (outputs)                     */
    GDN_KERNEL_SIMT = 5,        /* float32 CUDA-core forward                                       */
    GDN_KERNEL_DECODE = 6,      /* single-token decode step                                        */
    GDN_KERNEL_INPUT = 7,       /* input stage as a pass of its own (the *_raw forwards' fallbacks) */
    GDN_KERNEL_BACKWARD = 8,    /* backward pass (its forward recompute counts as PREP and CHAIN)  */
    GDN_KERNEL_GROUP_OUT = 9,   /* grouped heads: outputs of the query heads sharing a memory       */
    GDN_KERNEL_KINDS = 10
} gdn_kernel_kind;
int gdn_timing_start(void);
int gdn_timing_stop(double *ms, int64_t *launches);

/*
 * gdn_device_status -- failure detection for waits inside the kernels.  The
 * paper has no counterpart.  Every wait inside the library's kernels is
 * bounded.  A kernel whose wait gives up aborts its other waits, frees its
 * tensor memory, sets a device error word and returns; its results are
 * wrong, but nothing hangs and the context stays usable.  This call
 * synchronises `stream`, reads and clears the words of every kernel, and
 * returns GDN_ERR_DEVICE_TIMEOUT if any was set since the last call, else
 * GDN_OK (or GDN_ERR_DEVICE / GDN_ERR_LAUNCH).
 *
 * gdn_selftest_device_timeout -- enqueues a one-thread kernel whose bounded
 * wait on an mbarrier phase that nothing completes gives up by design and
 * sets its word, so that the next gdn_device_status(stream) returns
 * GDN_ERR_DEVICE_TIMEOUT.  It exercises the reporting path without any
 * fault; it enqueues no other work.
 */
int gdn_device_status(void *stream);
int gdn_selftest_device_timeout(void *stream);

/* Static, NUL-terminated description of a gdn_status value. */
const char *gdn_status_string(int status);

/* Library ABI version: major * 10000 + minor * 100 + patch. */
int gdn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* GDN_H */
