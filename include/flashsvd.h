/*
 * flashsvd.h — C ABI of libflashsvd.so, the B200 (sm_100a) hot path of
 * SVD-compressed ("low-rank") transformer inference.
 *
 * Sources, cited by page title and section:
 *   [v1.5] "FlashSVD v1.5: Making Low-Rank Transformers Inference Actually
 *          Fast" (gist.science explainer, English), Technical Summary:
 *          Problem Statement; Methodology 1 (Unified Runtime Abstraction),
 *          2 (Dense-KV Attention, Decode Phase), 3 (Packed MLP Execution),
 *          4 (Per-Layer CUDA Graph Replay).
 *   [v1]   "FlashSVD: Memory-Efficient Inference with Streaming for
 *          Low-Rank Models" (abstract).
 *
 * Conventions for every call
 *   - Tensors are caller-owned DEVICE pointers unless stated otherwise,
 *     row-major with the last dimension contiguous, base addresses 16-byte
 *     aligned.  Matrix widths d, r, n, f, H*D must be multiples of 8 (one
 *     16-byte vector = 8 bf16).  Violations return FLASHSVD_ERR_MISALIGNED
 *     or FLASHSVD_ERR_UNSUPPORTED_SHAPE and launch nothing.
 *   - flashsvd_bf16 is the bfloat16 bit pattern.  Arithmetic is fp32
 *     (accumulation, softmax, norms); storage between kernels is bf16.
 *   - Calls are asynchronous on the given stream (a cudaStream_t; NULL is
 *     the legacy default stream).  Device-side errors surface at the
 *     caller's next synchronisation, or through
 *     flashsvd_check_device_status().
 *   - Compute calls allocate nothing, never synchronise and copy nothing
 *     between host and device, so they may be captured in a CUDA graph.
 *     They use the workspace of the calling thread's context (see
 *     flashsvd_ctx_create; by default the one made by flashsvd_init()):
 *     calls that share a workspace must be ordered on one stream
 *     (overlapping calls race).
 *   - Read-only factor pointers may alias each other (shared bases,
 *     [v1.5] Methodology 1, Basis Sharing).  Outputs must not alias inputs
 *     except where a call says "in place".
 *   - Every call returns a status (enum flashsvd_status); nothing aborts.
 */
#ifndef FLASHSVD_H
#define FLASHSVD_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define FLASHSVD_API __attribute__((visibility("default")))
#else
#define FLASHSVD_API
#endif

typedef uint16_t flashsvd_bf16;                 /* bfloat16 bit pattern */
struct CUstream_st;
typedef struct CUstream_st* flashsvd_stream;    /* same as cudaStream_t */

enum flashsvd_status {
  FLASHSVD_OK = 0,
  FLASHSVD_ERR_INVALID_ARG = 1,       /* null pointer, bad enum, size < 0 */
  FLASHSVD_ERR_MISALIGNED = 2,        /* pointer not 16-byte aligned       */
  FLASHSVD_ERR_UNSUPPORTED_SHAPE = 3, /* width not a multiple of 8, or a
                                         size beyond the workspace limits  */
  FLASHSVD_ERR_NOT_INITIALIZED = 4,   /* flashsvd_init() not called        */
  FLASHSVD_ERR_CAPTURE_UNSAFE = 5,    /* call would allocate or sync while
                                         the stream is being captured      */
  FLASHSVD_ERR_CUDA = 6,              /* a CUDA runtime call failed; see
                                         flashsvd_last_cuda_error()        */
  FLASHSVD_ERR_TIMEOUT = 7,           /* a bounded device wait expired     */
  FLASHSVD_ERR_NO_MEMORY = 8          /* workspace allocation failed       */
};

/* Text for a status code (static storage). */
FLASHSVD_API const char* flashsvd_status_string(int status);
/* The cudaError_t of the last call that returned FLASHSVD_ERR_CUDA. */
FLASHSVD_API int flashsvd_last_cuda_error(void);
/* Library version, major*10000 + minor*100 + patch. */
FLASHSVD_API int flashsvd_version(void);

/* ---------------------------------------------------------------- setup --
 * flashsvd_init: make `device` current and allocate the library workspace on
 * it: the fp32 rank-activation exchange and split-K partial sums of the
 * decode linears, the split-sequence partials of decode attention, a device
 * status word, and per-layer activation scratch for up to `max_tokens` rows
 * of width `max_hidden` and FFN width `max_ffn` (prefill and encoder
 * layers).  `max_rank` bounds every factor rank.  Calling it again with the
 * same or smaller limits is a no-op; larger limits re-allocate (not allowed
 * during stream capture: FLASHSVD_ERR_CAPTURE_UNSAFE).
 * flashsvd_shutdown frees the workspace (after a device synchronise).
 */
FLASHSVD_API int flashsvd_init(int device, int max_tokens, int max_rank, int max_hidden,
                  int max_ffn);
FLASHSVD_API int flashsvd_shutdown(void);

/* ------------------------------------------------------------ contexts --
 * A context is one workspace (the scratch listed under flashsvd_init) plus
 * its device status word, on one device.  Every compute call uses the
 * context bound to the calling host thread, or the default context of
 * flashsvd_init when none is bound.  Calls that share a context must be
 * ordered on one stream; work that should overlap (two streams, two host
 * threads, two models on one GPU, or one model per GPU from one process)
 * gives each its own context.
 * flashsvd_ctx_create: allocate a context on `device` with the limits of
 *   flashsvd_init (cudaMalloc; not during stream capture:
 *   FLASHSVD_ERR_CAPTURE_UNSAFE; FLASHSVD_ERR_NO_MEMORY).  The calling
 *   thread's current device is left as it was.
 * flashsvd_ctx_bind: bind `ctx` to the calling host thread and make its
 *   device current (NULL returns the thread to the default context).  A
 *   context may be bound by several threads, but their calls then share
 *   its workspace.  Decode plans and captured graphs hold the addresses of
 *   the workspace that was current when they were made (plans: when they
 *   run), so a context must outlive them.
 * flashsvd_ctx_destroy: synchronise the context's device and free it; the
 *   calling thread is unbound from it if it was bound.  It must not be
 *   bound by another thread or used by a graph that still runs.
 */
typedef struct flashsvd_ctx flashsvd_ctx;
FLASHSVD_API int flashsvd_ctx_create(int device, int max_tokens, int max_rank, int max_hidden,
                                     int max_ffn, flashsvd_ctx** ctx);
FLASHSVD_API int flashsvd_ctx_bind(flashsvd_ctx* ctx);
FLASHSVD_API int flashsvd_ctx_destroy(flashsvd_ctx* ctx);

/* Synchronise `stream`, then read and clear the current context's device
 * status word, written by kernels whose bounded waits expired.  Returns FLASHSVD_OK or
 * FLASHSVD_ERR_TIMEOUT (or FLASHSVD_ERR_CUDA if the stream reports an
 * error). */
FLASHSVD_API int flashsvd_check_device_status(flashsvd_stream stream);

/* Decode implementation used by flashsvd_layer_forward(DECODE): fused != 0
 * (default) runs the whole layer as one persistent kernel (one CTA per SM,
 * factor tiles streamed through a TMA ring across all nine stages, stages
 * separated by bounded grid barriers) when B <= 4; fused == 0 runs one
 * launch per stage.  Both give the same result within rounding.  The fused
 * kernel is launched cooperatively (all of its CTAs resident at once, or the
 * launch fails with FLASHSVD_ERR_CUDA), since its CTAs wait on one
 * another. */
FLASHSVD_API int flashsvd_set_decode_path(int fused);

/* Prefill attention of DECODER layers (PREFILL_CAUSAL): mode 1 forms each
 * query tile inside the attention kernel from the query's rank activation
 * (flashsvd_prefill_attn_factorized: dense q never exists); mode 0, the
 * default, runs the query's second-stage projection (dense q, RoPE in its
 * epilogue) and the plain prefill attention.  Both give the same result
 * within rounding.  Mode 0 is the faster one on B200 at every query rank
 * measured (128 to 1216, 7B-shaped layer, 2048 tokens): in mode 1 each
 * (query tile, head) item first waits for its own query tile (the operands
 * of z_q V_q through the kernel's two-stage ring, the product, then RoPE),
 * which the plain kernel loads ahead while the previous item finishes.
 * Other modes return FLASHSVD_ERR_INVALID_ARG. */
FLASHSVD_API int flashsvd_set_prefill_attention(int mode);

/* Prefill rank activations (z of the factorized linears, z1 of the streamed
 * FFN, z_q of the factorized attention) live in a workspace that stays in
 * L2 between the two kernels of a linear; on != 0 (default) the kernel that
 * reads a block of z last drops its L2 lines without write-back
 * (discard.global.L2), so z never reaches HBM.  on = 0 leaves the lines to
 * the normal write-back: a control for measuring what the discard saves.
 * Results are identical either way. */
FLASHSVD_API int flashsvd_set_l2_discard(int on);

/* Failure-detection test hook.  Arms a one-shot fault: the next launch of
 * the fused decode kernel (a DECODE-mode flashsvd_layer_forward over a
 * decode pack, or flashsvd_decode_plan_forward) takes it, and its CTA 0
 * does not arrive at the kernel's first grid barrier.  The other CTAs'
 * bounded waits then expire (after about two seconds of SM cycles); every
 * CTA abandons the step, the launch completes, and
 * flashsvd_check_device_status returns FLASHSVD_ERR_TIMEOUT.  The kernel's
 * stage counters are reset at the end of that launch, so the next launch
 * runs normally.  No GPU fault is involved.  The hook is read when the
 * launch is issued (not during stream capture: a captured launch keeps the
 * value it had). */
FLASHSVD_API int flashsvd_debug_drop_barrier_arrival(void);

/* Number of kernels this library has launched since load: eager launches
 * plus the kernel nodes of every replayed graph. */
FLASHSVD_API int64_t flashsvd_launch_count(void);

/* Profiler.  flashsvd_profile_enable(1) brackets every EAGER launch of this
 * library with CUDA events on its stream (graph replays and launches made
 * during capture are not instrumented; the events serialise the launches).
 * flashsvd_profile_report synchronises the device and writes one line per
 * operation, "name launches total_ms algorithmic_bytes flops\n", into buf
 * (NUL-terminated, truncated to buflen); reset != 0 clears the totals.  With
 * buf == NULL it returns the buffer size needed. */
FLASHSVD_API int flashsvd_profile_enable(int on);
FLASHSVD_API int flashsvd_profile_report(char* buf, int buflen, int reset);

/* ------------------------------------------------------ factorized linear --
 * y[M x n] = (x[M x d] . U[d x r]) . V[r x n] + bias[n]           (bias may be NULL)
 *
 * [v1] abstract (truncated factors applied as two chained products whose
 * rank-r intermediate is reduced on the fly, never materialised as a
 * full-size activation); [v1.5] Problem Statement (prefill and decode have
 * different bottlenecks, so each phase has its own kernel).
 *   M <= 32 (decode): split-K GEMV over U, then over V (rows in groups of
 *     8, one launch per stage); the intermediate z = x.U [M x r] stays fp32
 *     in a small L2-resident workspace.
 *   M > 32 (prefill): two tcgen05 tensor-core launches; z is rounded to
 *     bf16 into a library scratch that stays in L2 between them, and the
 *     second launch discards each 128-row block of z from L2 once every
 *     column tile has read it, so z is never written back to HBM.
 * Sizes: 1 <= M <= max_tokens; d, r, n multiples of 8 (prefill: d, r
 * multiples of 64 as well); r <= max_rank.
 */
FLASHSVD_API int flashsvd_lowrank_linear(const flashsvd_bf16* x, const flashsvd_bf16* U,
                            const flashsvd_bf16* V, const flashsvd_bf16* bias,
                            flashsvd_bf16* y, int M, int d, int r, int n,
                            flashsvd_stream stream);

/* Dense y[M x n] = x[M x d] . W[d x n] (the output head, which is not
 * factorized), fp32 result.  Same size rules as flashsvd_lowrank_linear. */
FLASHSVD_API int flashsvd_dense_linear_f32(const flashsvd_bf16* x, const flashsvd_bf16* W,
                              float* y, int M, int d, int n,
                              flashsvd_stream stream);

/* -------------------------------------------------------------- head --
 * The decode step's output head (dense, not factorized; part of the
 * per-step replay unit of [v1.5] Methodology 4) with the final RMSNorm
 * folded into the same split-K GEMV:
 *   logits[M x n] = rmsnorm(x) . W   (fp32),   W [d x n] row-major bf16.
 * x [M x d] bf16 (row stride d); g [d] bf16 RMSNorm gain, or NULL for no
 * norm (logits = x . W); eps >= 0; logits [M x n] fp32 (row stride n).
 * 1 <= M <= 32 (and <= max_tokens), d and n multiples of 8.  Each CTA sums
 * the squares of its slice of x; the CTA that completes a column tile
 * scales its sums by rstd(x) (x . g is not rounded to bf16 first, unlike a
 * separate flashsvd_rmsnorm).  Errors: FLASHSVD_ERR_INVALID_ARG (null
 * pointer, M < 0, eps < 0 with a gain), FLASHSVD_ERR_MISALIGNED,
 * FLASHSVD_ERR_UNSUPPORTED_SHAPE (M > 32, widths, workspace too small for
 * the split partials).  Allocates nothing; safe during capture.
 */
FLASHSVD_API int flashsvd_head_logits(const flashsvd_bf16* x, const flashsvd_bf16* g, float eps,
                                      const flashsvd_bf16* W, float* logits, int M, int d,
                                      int n, flashsvd_stream stream);

/* -------------------------------------------------- packed gate|up MLP --
 * [v1.5] Methodology 3 (Packed MLP Execution): the input-side gate and up
 * factors are packed offline into one tensor, U_gu[d x 2r_f] = [U_g | U_u]
 * (gate columns first); one wide projection z = x.U_gu [M x 2r_f] is taken
 * and split; V_gu[2r_f x f] holds V_g (rows 0..r_f-1) stacked on V_u.
 *   h = SiLU(z_g . V_g) * (z_u . V_u)                 [M x f]
 *   y = (h . U_dn[f x r_dn]) . V_dn[r_dn x d]         [M x d]
 * flashsvd_gateup_swiglu stops at h (the first two stages).
 */
FLASHSVD_API int flashsvd_packed_gateup_mlp(const flashsvd_bf16* x,
                               const flashsvd_bf16* U_gu,
                               const flashsvd_bf16* V_gu,
                               const flashsvd_bf16* U_dn,
                               const flashsvd_bf16* V_dn, flashsvd_bf16* y,
                               int M, int d, int r_f, int f, int r_dn,
                               flashsvd_stream stream);
FLASHSVD_API int flashsvd_gateup_swiglu(const flashsvd_bf16* x, const flashsvd_bf16* U_gu,
                           const flashsvd_bf16* V_gu, flashsvd_bf16* h, int M,
                           int d, int r_f, int f, flashsvd_stream stream);

/* ------------------------------------------------- streamed low-rank FFN --
 * [v1] abstract: the encoder FFN's intermediate activations are streamed
 * through tiles instead of being materialised.
 *   y[M x d] = GELU((x . U_up) . V_up + b_up) . U_dn . V_dn + b_dn + resid
 * x [M x d], U_up [d x r_up], V_up [r_up x f], U_dn [f x r_dn],
 * V_dn [r_dn x d]; b_up [f], b_dn [d] and resid [M x d] may be NULL; resid
 * may equal y.  GELU is the erf form.  z1 = x . U_up is one tcgen05 launch
 * into the library scratch (kept in L2 and discarded there after use); the
 * rest is ONE kernel per 128-row tile that runs f in 128-column chunks:
 * the chunk of GELU(z1 . V_up + b_up) goes from tensor memory through the
 * GELU warps into shared memory and straight into the rank-r_dn
 * accumulator of U_dn, so the [M x f] activation is never written to
 * memory.  ENCODER-layer flashsvd_layer_forward uses it for the FFN.
 * Sizes: d a multiple of 64; r_up, r_dn multiples of 64 in [64, 256]; f a
 * multiple of 8; M <= max_tokens.  Other shapes return
 * FLASHSVD_ERR_UNSUPPORTED_SHAPE (the encoder layer then runs the FFN as
 * two factorized linears with the [M x f] activation in the workspace).
 */
FLASHSVD_API int flashsvd_lowrank_ffn(const flashsvd_bf16* x, const flashsvd_bf16* U_up,
                                      const flashsvd_bf16* V_up, const flashsvd_bf16* b_up,
                                      const flashsvd_bf16* U_dn, const flashsvd_bf16* V_dn,
                                      const flashsvd_bf16* b_dn, const flashsvd_bf16* resid,
                                      flashsvd_bf16* y, int M, int d, int r_up, int f, int r_dn,
                                      flashsvd_stream stream);

/* ------------------------------------------------ dense-KV decode attention --
 * [v1.5] Methodology 2 ("reconstruct the present, read the past
 * contiguously"): the history lives in a dense contiguous KV cache laid out
 * like flash_attn_with_kvcache's, k_cache/v_cache [B, S_max, H, D] bf16, with
 * cache_seqlens a DEVICE int32[B].  If k_new and v_new (each [B x H x D]) are
 * non-NULL they are written at index cache_seqlens[b]; either way the query
 * q[B x H x D] then attends over keys 0..cache_seqlens[b] inclusive:
 *   out[b,h] = softmax(q.K^T * scale) . V               [B x H x D] bf16
 * cache_seqlens is not incremented (see flashsvd_advance_seqlens).
 * Requires cache_seqlens[b] < S_max (entries at or beyond S_max are clamped
 * to S_max-1 on the device), D in {64, 128}.
 */
FLASHSVD_API int flashsvd_dense_kv_decode_attn(const flashsvd_bf16* q,
                                  const flashsvd_bf16* k_new,
                                  const flashsvd_bf16* v_new,
                                  flashsvd_bf16* k_cache,
                                  flashsvd_bf16* v_cache,
                                  const int32_t* cache_seqlens,
                                  flashsvd_bf16* out, int B, int H, int D,
                                  int S_max, float scale,
                                  flashsvd_stream stream);

/* Full-sequence (prefill / encoder) attention, [v1.5] Methodology 2,
 * "Prefill": q and out [B, S, H, D]; keys and values are rows 0..S-1 of
 * k_cache/v_cache [B, S_max, H, D].  causal != 0 masks key j > query i.
 * D in {64, 128}. */
FLASHSVD_API int flashsvd_prefill_attn(const flashsvd_bf16* q, const flashsvd_bf16* k_cache,
                          const flashsvd_bf16* v_cache, flashsvd_bf16* out,
                          int B, int S, int H, int D, int S_max, int causal,
                          float scale, flashsvd_stream stream);

/* Factorized prefill attention, [v1.5] Methodology 2, "Prefill" (prefill
 * keeps a dedicated factorized attention kernel so that dense activations
 * are not materialised): the query of every row is formed inside the
 * kernel from the rank activation of the query projection,
 *   q[b, s, h] = rope(z_q[b*S + s] . V_q[:, h*D .. h*D + D), position s),
 *   out[b, s, h] = softmax(q . K[b, 0..S)^T * scale (causal: keys <= s)) . V
 * so dense q is neither written nor read.  z_q [B*S x r] bf16 (row stride
 * r), V_q [r x H*D], rotary tables [>= S x D/2] fp32 (flashsvd_rope_table),
 * keys and values rows 0..S-1 of k_cache / v_cache [B, S_max, H, D]; out
 * [B, S, H, D].  r a multiple of 64, D in {64, 128}.  With
 * flashsvd_set_prefill_attention(1) the DECODER layer's PREFILL_CAUSAL mode
 * uses it with the z_q of its q/k/v stage 1 (and drops that z_q from L2
 * after its last head has read it). */
FLASHSVD_API int flashsvd_prefill_attn_factorized(const flashsvd_bf16* z_q, const flashsvd_bf16* V_q,
                                                  const float* rope_cos, const float* rope_sin,
                                                  const flashsvd_bf16* k_cache,
                                                  const flashsvd_bf16* v_cache, flashsvd_bf16* out,
                                                  int B, int S, int H, int D, int S_max, int r,
                                                  int causal, float scale, flashsvd_stream stream);

/* --------------------------------------------------------------- glue ----
 * RMSNorm y = x * g / sqrt(mean(x^2) + eps); LayerNorm
 * y = (x - mean) / sqrt(var + eps) * g + b (population variance).  Rows of
 * width d, M rows; y may equal x (in place).
 * Rotary table: cos_tab/sin_tab [S_max x D/2] fp32 with
 * angle(p, i) = p * base^(-2i/D), computed in double on the device.
 * Embedding gather: x[b] = emb[tokens[b]] for b < B (tokens on the device;
 * ids outside [0, vocab) are clamped).
 * Greedy: next[m] = argmax_j logits[m, j] (ties to the lowest index).
 * advance: cache_seqlens[b] += 1 for b < B.
 */
FLASHSVD_API int flashsvd_rmsnorm(const flashsvd_bf16* x, const flashsvd_bf16* g,
                     flashsvd_bf16* y, int M, int d, float eps,
                     flashsvd_stream stream);
FLASHSVD_API int flashsvd_layernorm(const flashsvd_bf16* x, const flashsvd_bf16* g,
                       const flashsvd_bf16* b, flashsvd_bf16* y, int M, int d,
                       float eps, flashsvd_stream stream);
FLASHSVD_API int flashsvd_rope_table(float* cos_tab, float* sin_tab, int S_max, int D,
                        float base, flashsvd_stream stream);
FLASHSVD_API int flashsvd_embed(const int32_t* tokens, const flashsvd_bf16* emb,
                   flashsvd_bf16* x, int B, int d, int vocab,
                   flashsvd_stream stream);
FLASHSVD_API int flashsvd_greedy(const float* logits, int32_t* next_tokens, int M,
                    int vocab, flashsvd_stream stream);
FLASHSVD_API int flashsvd_advance_seqlens(int32_t* cache_seqlens, int B,
                             flashsvd_stream stream);

/* ------------------------------------------------ no-allocation variant --
 * No counterpart in the pages.  Same result as flashsvd_lowrank_linear,
 * y[M x n] = (x[M x d] . U[d x r]) . V[r x n] + bias[n] (bias may be NULL),
 * with the decode kernels, for callers that cannot allocate device memory:
 * flashsvd_init obtains its workspace with cudaMalloc, which a plugin inside
 * a framework whose allocator owns all device memory, or a serving process
 * that must not allocate after start-up, cannot do.  This call needs no
 * flashsvd_init and calls no cudaMalloc, cudaFree or allocating routine; its
 * scratch (rank activations, split partial sums, tile counters) is one fixed
 * array of about 2.2 MiB in device memory that every GPU which loads the
 * library holds until the process exits.
 * Limits: 1 <= M <= 8, r <= 4096, d and n <= 16384 (all multiples of 8),
 * and the split partial sums of both products must fit the array.  The call
 * accepts a shape exactly when, for (K, N) = (d, r) and (K, N) = (r, n),
 *     ceil(K / 512) * ceil(N / 64) * (64 m + 8) <= 524288,
 * with m = 1, 2, 4, 8 for M = 1, 2, 3..4, 5..8 (on GPUs of up to 336 SMs).
 * Every shape with d, n <= 8192 and r <= 2048, or with d, n, r <= 4096,
 * passes at any M <= 8.  Anything else returns
 * FLASHSVD_ERR_UNSUPPORTED_SHAPE and launches nothing.
 * The first call on each device looks up the array's device address with
 * that device current; make that first call before any stream capture.
 * All calls share the one array and each overwrites it (the tile counters
 * are cleared by a memset on `stream` at the start of every call), so calls
 * that overlap on the GPU -- on different streams or from different host
 * threads -- race: order them on one stream.
 */
FLASHSVD_API int flashsvd_lowrank_linear_noalloc(const flashsvd_bf16* x,
                                                 const flashsvd_bf16* U,
                                                 const flashsvd_bf16* V,
                                                 const flashsvd_bf16* bias,
                                                 flashsvd_bf16* y, int M, int d,
                                                 int r, int n,
                                                 flashsvd_stream stream);

/* -------------------------------------------------------------- layers ---
 * One transformer layer as caller-owned factor pointers.
 * kind = FLASHSVD_DECODER: pre-norm RMSNorm, RoPE, causal attention,
 *   packed gate|up SwiGLU MLP (U_gu, V_gu, r_f) and factorized down
 *   projection (down), no biases:
 *     h = x + o(attn(rope(q(n1)), rope(k(n1)), v(n1))),  n1 = rmsnorm(x, norm1_g)
 *     y = h + down(SiLU(gate) * up)(rmsnorm(h, norm2_g))
 * kind = FLASHSVD_ENCODER: post-LN, bidirectional attention, GELU FFN (up,
 *   down), every linear with its bias:
 *     h = LN1(x + o(attn(q(x), k(x), v(x))));  y = LN2(h + down(GELU(up(h))))
 * Heads are contiguous D-slices of the hidden width (d = H * D).
 */
typedef struct flashsvd_factor {
  const flashsvd_bf16* U;      /* [d_in x r]  */
  const flashsvd_bf16* V;      /* [r x d_out] */
  const flashsvd_bf16* bias;   /* [d_out] or NULL */
  int r;
} flashsvd_factor;

enum flashsvd_layer_kind { FLASHSVD_DECODER = 0, FLASHSVD_ENCODER = 1 };
enum flashsvd_mode {
  FLASHSVD_PREFILL_CAUSAL = 0,  /* decoder, whole prompt, fills cache [0,S) */
  FLASHSVD_DECODE = 1,          /* decoder, one token per sequence (S = 1)  */
  FLASHSVD_ENCODER_BIDIR = 2    /* encoder, whole sequence                  */
};

typedef struct flashsvd_layer {
  int kind;                     /* enum flashsvd_layer_kind */
  int d, H, D, f;               /* hidden, heads, head dim, FFN width */
  float norm_eps;
  const flashsvd_bf16* norm1_g; const flashsvd_bf16* norm1_b;  /* b: encoder */
  const flashsvd_bf16* norm2_g; const flashsvd_bf16* norm2_b;
  flashsvd_factor q, k, v, o;
  const flashsvd_bf16* U_gu;    /* decoder: [d x 2 r_f] packed gate|up */
  const flashsvd_bf16* V_gu;    /* decoder: [2 r_f x f] */
  int r_f;
  flashsvd_factor up;           /* encoder: [d -> f] */
  flashsvd_factor down;         /* [f -> d] */
  const float* rope_cos;        /* decoder: [S_max x D/2] (flashsvd_rope_table) */
  const float* rope_sin;
  const void* decode_pack;      /* decoder: flashsvd_decode_pack output, or NULL */
} flashsvd_layer;

/* ---------------------------------------------------------- decode pack ---
 * Decode is bound by reading the factors (FlashSVD v1.5 Technical Summary,
 * Problem Statement).  The fused decode-layer kernel reads a decoder layer's
 * factors from a "decode pack": a copy of q/k/v/o U and V, U_gu, V_gu and
 * down U/V re-tiled so that every 256-row x 64-output-column block the kernel
 * consumes is one contiguous run of device memory, stored in the order the
 * kernel consumes them.  It is a pure layout change: no value is altered.
 * Whole contiguous blocks stream at close to the HBM copy rate; 64- or
 * 128-byte row pieces spaced at the matrix pitch do not.
 *
 * flashsvd_decode_pack_bytes: size of L's pack (host only, no device work).
 * flashsvd_decode_pack: writes L's pack into dst (device memory, 16-byte
 *   aligned, at least the size above, owned by the caller), asynchronously
 *   on `stream`.  Then set L->decode_pack = dst: DECODE-mode
 *   flashsvd_layer_forward runs the fused single-kernel layer from it; with
 *   decode_pack NULL it runs the per-stage kernels.  The pack must outlive
 *   its use and be rebuilt whenever a factor changes.
 * Errors: INVALID_ARG (null argument, dst too small, not a decoder layer),
 *   MISALIGNED, UNSUPPORTED_SHAPE (ranks of q, k, v differ, down rank !=
 *   r_f, D not 64 or 128, d not a multiple of 64, a rank or f not a multiple
 *   of 8). */
FLASHSVD_API int flashsvd_decode_pack_bytes(const flashsvd_layer* L, size_t* bytes);
FLASHSVD_API int flashsvd_decode_pack(const flashsvd_layer* L, void* dst, size_t bytes,
                                      flashsvd_stream stream);

/* ---------------------------------------------------------- decode plan ---
 * FlashSVD v1.5 Technical Summary, Methodology 4, makes each layer's decode
 * body one replay unit.  A decode plan goes one step further: the decode
 * step of n consecutive decoder layers runs as ONE launch of the fused
 * decode kernel, which streams the next layer's factors while the current
 * layer finishes and hands each layer's output to the next on chip-wide
 * partial sums, with no launch boundary in between.
 *
 * flashsvd_decode_plan_create: layers[0..n) (each with a decode pack, equal
 *   d, H, D, f, norm_eps and RoPE tables; ranks may differ per layer), layer
 *   i's caches k_caches[i], v_caches[i] ([B, S_max, H, D] bf16, device
 *   pointers; host arrays of n pointers).  B <= 4.  Builds the kernel's
 *   per-layer descriptors in device memory it owns (synchronous; not during
 *   stream capture).  The layers' factors, packs and caches must outlive the
 *   plan.
 * flashsvd_decode_plan_forward: one decode step of all n layers in place on
 *   x_inout [B x d]; positions are cache_seqlens[b] (device int32[B]); every
 *   layer appends its new key and value there; cache_seqlens is not
 *   incremented.  Same result as n DECODE-mode flashsvd_layer_forward calls.
 *   The positions may differ freely across the rows (any mix of lengths up
 *   to S_max): the attention work, 64-key chunks of every (row, head), is
 *   split evenly over the CTAs whatever the lengths.
 *   Asynchronous, capturable, uses the context's scratch (one plan runs at a
 *   time per context).
 * Errors: INVALID_ARG, NOT_INITIALIZED, CAPTURE_UNSAFE (create during
 *   capture), UNSUPPORTED_SHAPE (a layer without a pack, B > 4, shapes the
 *   fused kernel does not cover: among them 7 * min(SMs, 14 H) < 2 B H, or
 *   B H ceil(S_max / 64) min(SMs, 14 H) >= 2^31), NO_MEMORY.  A DECODE-mode
 *   flashsvd_layer_forward on a layer the fused kernel does not cover runs
 *   the per-stage kernels instead. */
typedef struct flashsvd_decode_plan flashsvd_decode_plan;
FLASHSVD_API int flashsvd_decode_plan_create(const flashsvd_layer* layers, int n_layers,
                                             flashsvd_bf16* const* k_caches,
                                             flashsvd_bf16* const* v_caches, int B, int S_max,
                                             flashsvd_decode_plan** plan);
FLASHSVD_API int flashsvd_decode_plan_forward(const flashsvd_decode_plan* plan,
                                              flashsvd_bf16* x_inout,
                                              const int32_t* cache_seqlens, flashsvd_stream stream);
FLASHSVD_API int flashsvd_decode_plan_destroy(flashsvd_decode_plan* plan);

/* Run one layer in place on x_inout ([B*S x d] bf16, token-major).
 * PREFILL_CAUSAL: positions 0..S-1; rotated keys and values are written to
 *   cache rows [0, S) of every batch entry; cache_seqlens is not read.
 * DECODE: S must be 1; positions are cache_seqlens[b] (device); the new key
 *   and value are appended there ([v1.5] Methodology 2); cache_seqlens is not
 *   incremented.
 * ENCODER_BIDIR: k_cache/v_cache are [B, S_max >= S, H, D] scratch the
 *   caller provides; cache_seqlens may be NULL.
 * B*S <= max_tokens of flashsvd_init (DECODE: B <= 32). */
FLASHSVD_API int flashsvd_layer_forward(const flashsvd_layer* L, flashsvd_bf16* x_inout,
                           flashsvd_bf16* k_cache, flashsvd_bf16* v_cache,
                           const int32_t* cache_seqlens, int B, int S,
                           int S_max, int mode, flashsvd_stream stream);

/* -------------------------------------------------------------- graphs ---
 * [v1.5] Methodology 4 (Per-Layer CUDA Graph Replay): the stable decode body
 * of one layer is captured once and replayed every step.  Buffers, B and
 * S_max are fixed at capture; positions come from cache_seqlens in device
 * memory, so one graph serves every step.
 * flashsvd_capture_begin/end capture any sequence of library calls issued on
 * `stream` between them (e.g. embedding, output head, greedy pick and
 * advance) into a replayable graph.  A graph may also be a composition of
 * other graphs (flashsvd_graph_compose), replayed as one launch.
 */
typedef struct flashsvd_graph flashsvd_graph;

FLASHSVD_API int flashsvd_decode_graph_capture(const flashsvd_layer* L,
                                  flashsvd_bf16* x_inout,
                                  flashsvd_bf16* k_cache,
                                  flashsvd_bf16* v_cache,
                                  const int32_t* cache_seqlens, int B,
                                  int S_max, flashsvd_stream stream,
                                  flashsvd_graph** graph);
FLASHSVD_API int flashsvd_capture_begin(flashsvd_stream stream);
FLASHSVD_API int flashsvd_capture_end(flashsvd_stream stream, flashsvd_graph** graph);
FLASHSVD_API int flashsvd_graph_compose(flashsvd_graph* const* parts, int n_parts,
                           flashsvd_graph** graph);
FLASHSVD_API int flashsvd_graph_replay(flashsvd_graph* graph, flashsvd_stream stream);
/* Kernel nodes in the graph (used for launch accounting). */
FLASHSVD_API int flashsvd_graph_kernel_count(const flashsvd_graph* graph);
FLASHSVD_API int flashsvd_graph_destroy(flashsvd_graph* graph);

#ifdef __cplusplus
}
#endif
#endif /* FLASHSVD_H */
