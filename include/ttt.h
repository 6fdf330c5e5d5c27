/*
 * ttt.h — C ABI of the TTT-E2E prefill library (B200, sm_100a).
 *
 * The library runs the test-time-training prefill loop of "End-to-End
 * Test-Time Training for Long Context" (Tandon et al., arXiv:2512.23675):
 * a Transformer with sliding-window attention reads a token sequence in
 * chunks of b tokens; for every chunk it predicts each target with the
 * current fast weights W_{i-1}, records the next-token cross-entropy, takes
 * the gradient of the chunk's mean loss with respect to the fast MLPs of the
 * last n_u blocks and applies one SGD step, W_i = W_{i-1} - eta * grad A_i
 * (reading notes by Zhongzhu Zhou: eq. (9) and 算法 1 "因果预填充与内层适应").
 *
 * Conventions for every entry point:
 *  - Pointers ending in _dev are CUDA device pointers; the library never
 *    frees caller memory.  All device work is enqueued on the stream given to
 *    ttt_init and is asynchronous; ttt_sync waits and reports device-side
 *    errors.
 *  - Matrices are row-major.  Linear weights are [out_features, in_features]
 *    (y = x W^T).
 *  - Return values are TTT_OK (0) or a negative TTT_ERR_* code; after an
 *    error, ttt_last_error() gives a message.
 *  - No entry point is thread-safe on the same context.
 */
#ifndef TTT_H_
#define TTT_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- status codes ---- */
#define TTT_OK 0
#define TTT_ERR_INVALID_ARG (-1) /* bad argument or configuration */
#define TTT_ERR_STATE (-2)       /* call not allowed in the context's state */
#define TTT_ERR_OOM (-3)         /* device allocation failed */
#define TTT_ERR_CUDA (-4)        /* a CUDA runtime or driver call failed */
#define TTT_ERR_TIMEOUT (-5)     /* a kernel's bounded wait gave up (device watchdog) */
#define TTT_ERR_UNSUPPORTED (-6) /* shape or feature this build does not support */

/* ---- element types ---- */
#define TTT_F32 0  /* everything fp32 (SIMT kernels) */
#define TTT_BF16 1 /* bf16 weights and GEMM operands, fp32 accumulation, fp32 residual,
                      fp32 master fast weights with a bf16 shadow */

/*
 * Model configuration.  The backbone is a pre-norm Transformer with
 * QK-norm (the recipe in the jdon.com write-up names QK norm and the Llama3
 * tokenizer), RoPE, SwiGLU MLPs and an untied LM head.
 *   d_model == n_heads * head_dim; head_dim in {32, 64, 80, 96, 128};
 *   d_model a multiple of 8; d_ff a multiple of 64.
 *   norm_eps: RMSNorm epsilon (y = x / sqrt(mean(x^2) + eps) * g).
 *   rope_theta: RoPE base; element i is paired with i + head_dim/2.
 */
typedef struct ttt_config {
  int32_t n_layers;
  int32_t d_model;
  int32_t n_heads;
  int32_t head_dim;
  int32_t d_ff;
  int32_t vocab;
  float norm_eps;
  float rope_theta;
  int32_t dtype; /* TTT_F32 or TTT_BF16 */
} ttt_config;

/*
 * Static weights of one block.  Norm gains are fp32 [d_model] (q_norm, k_norm:
 * [head_dim]); linear weights are in the configured dtype:
 *   wq, wk, wv, wo: [d_model, d_model];  w_gate, w_up: [d_ff, d_model];
 *   w_down: [d_model, d_ff].
 */
typedef struct ttt_layer_weights {
  const float* attn_norm;
  const void* wq;
  const void* wk;
  const void* wv;
  const void* wo;
  const float* q_norm;
  const float* k_norm;
  const float* mlp_norm;
  const void* w_gate;
  const void* w_up;
  const void* w_down;
} ttt_layer_weights;

/* Initial fast weights W_init of one updated block, fp32:
 * w_gate, w_up: [d_ff, d_model];  w_down: [d_model, d_ff]. */
typedef struct ttt_fast_weights {
  const float* w_gate;
  const float* w_up;
  const float* w_down;
} ttt_fast_weights;

/*
 * All weights.  Device pointers, owned by the caller, read-only for the
 * library, and valid until ttt_free.  `layers` and `fast` are HOST arrays of
 * n_layers and n_updated_blocks entries; fast[i] belongs to block
 * n_layers - n_updated_blocks + i.
 *   embed: [vocab, d_model] (configured dtype); lm_head: [vocab, d_model]
 *   (configured dtype); final_norm: fp32 [d_model].
 */
typedef struct ttt_weights {
  const void* embed;
  const ttt_layer_weights* layers;
  const ttt_fast_weights* fast;
  const float* final_norm;
  const void* lm_head;
} ttt_weights;

typedef struct ttt_ctx ttt_ctx;

/*
 * Create a context (算法 1 inputs: W_init and phi from the outer loop, chunk
 * size b).  Copies W_init into library-owned fp32 masters (plus a bf16
 * shadow in TTT_BF16 mode) and keeps a copy for ttt_reset; the caller's
 * tensors are never written.  Allocates the per-block KV ring buffers
 * (window k plus one chunk) and all activation scratch.
 *   eta: inner SGD learning rate (finite).  k >= 1: attention window
 *   (query p sees keys p-k+1 .. p, eq. (1)).  b >= 1: chunk size.
 *   1 <= n_updated_blocks <= n_layers: the last n_updated_blocks blocks carry
 *   a fast MLP beside their static one (outputs summed).
 *   stream: a cudaStream_t (may be NULL for the legacy default stream).
 * In TTT_BF16 mode ttt_init also reads each block's QK-norm gains (q_norm,
 * k_norm) once, synchronously: max|gain| * sqrt(head_dim) bounds the norm of
 * every normalised query and key row, which lets the attention forward use a
 * fixed softmax shift (include/ttt_ops.h, ttt_op_swa_forward).  Static
 * weights are therefore fixed for the context's life, like the copies above.
 * Errors: TTT_ERR_INVALID_ARG, TTT_ERR_UNSUPPORTED, TTT_ERR_OOM, TTT_ERR_CUDA.
 * On error *out is set to NULL.
 */
int ttt_init(const ttt_config* config, const ttt_weights* weights, float eta, int32_t k, int32_t b,
             int32_t n_updated_blocks, void* stream, ttt_ctx** out);

/*
 * The prefill loop (算法 1) over tokens_dev[0 .. T-1] (int32, device).
 * For chunk c (positions [c*b, min((c+1)*b, T))) every position p is scored
 * with the fast weights of before the chunk's update: losses_dev[p] =
 * -ln softmax(z_p)[tokens[p+1]] (fp32, device, T entries; losses_dev[T-1] =
 * NaN, there is no target).  Then every full chunk takes one SGD step on the
 * mean loss of its targets (eq. (9)); a trailing partial chunk is scored only.
 * fast_out_dev: NULL, or a HOST array of 3*n_updated_blocks device pointers
 * (per updated block: w_gate [d_ff, d_model], w_up [d_ff, d_model], w_down
 * [d_model, d_ff], fp32) that receive the final fast weights.
 * Requires a fresh context (after ttt_init or ttt_reset): TTT_ERR_STATE
 * otherwise.  T >= 1.  Token ids are checked on the device; an id outside
 * [0, vocab) makes ttt_sync return TTT_ERR_INVALID_ARG (results undefined).
 */
int ttt_prefill(ttt_ctx* ctx, const int32_t* tokens_dev, int64_t T, float* losses_dev,
                float* const* fast_out_dev);

/*
 * Greedy generation with periodic fast-weight updates (算法 3 of the reading
 * notes: generate causally from the state the prefill left, collect the new
 * tokens until an inner chunk is full, update the fast weights on that
 * chunk's next-token loss, continue from the new state).
 * Each generated token is the argmax of the logits of the position before it
 * (ties: the lowest token id).  The first one comes from the logits of the
 * prompt's last position T-1, as the prefill scored it (with the fast weights
 * of before its chunk's update).  Chunks keep the prefill's grid of absolute
 * positions [c*b, (c+1)*b): when T % b != 0 the prompt's trailing partial
 * chunk (scored, not applied, by the prefill) is completed by the first
 * generated tokens.  After the forward of the last position of a chunk (its
 * argmax gives that position's target), the chunk takes one SGD step on the
 * mean loss of its b targets, exactly as in ttt_prefill, and generation
 * continues with the updated weights.
 * ttt_decode_step writes one token (int32) to next_token_dev and runs the
 * forward of its position.  Requires a ttt_prefill since the last
 * ttt_init / ttt_reset (TTT_ERR_STATE otherwise); asynchronous on the stream.
 */
int ttt_decode_step(ttt_ctx* ctx, int32_t* next_token_dev);

/*
 * n_tokens steps of ttt_decode_step in one call: tokens_dev[i] (int32,
 * device) receives the i-th generated token; losses_dev (fp32, device, may be
 * NULL) receives, for each generated token, the loss of the position before
 * it against it (log-sum-exp of that position's logits minus their maximum).
 */
int ttt_decode(ttt_ctx* ctx, int64_t n_tokens, int32_t* tokens_dev, float* losses_dev);

/* Restore W_init (a fresh copy for a new document, as 算法 2 starts each document), empty the
 * attention state and set the position to 0.  Asynchronous on the stream. */
int ttt_reset(ttt_ctx* ctx);

/* Wait for the context's stream; return the first error recorded by a kernel
 * (TTT_ERR_TIMEOUT, TTT_ERR_INVALID_ARG for a bad token) or a CUDA error. */
int ttt_sync(ttt_ctx* ctx);

/* Message of the last error on this context (or of the calling thread when
 * ctx is NULL).  Never NULL. */
const char* ttt_last_error(ttt_ctx* ctx);

/* Release everything the context owns.  NULL is ignored. */
void ttt_free(ttt_ctx* ctx);

/* Number of kernel launches issued on this context since ttt_init. */
int64_t ttt_launch_count(ttt_ctx* ctx);

/* ---- optional per-kernel-class timing ----
 * When enabled, a CUDA event is recorded on the context's stream after every
 * launch (and before the first launch of each ttt_prefill / ttt_reset call);
 * a launch's time runs from the event before it to the event after it, so
 * back-to-back launches share one event per boundary.  The launch's
 * algorithmic work is accumulated:
 *   GEMM: 2*M*N*K flops;  ATTN_FWD: 4 * d_model * (query-key pairs admitted by
 *   the window, eq. (1));  ATTN_BWD: 4 * d_model * (band pairs + causal pairs
 *   among the chunk's own positions).  OTHER: memory-bound kernels (no flops).
 * ttt_timing_read synchronises the stream and returns the totals since the
 * last ttt_timing_enable(ctx, 1). */
#define TTT_KC_GEMM 0
#define TTT_KC_ATTN_FWD 1
#define TTT_KC_ATTN_BWD 2
#define TTT_KC_OTHER 3 /* embedding, SwiGLU backward, CE finalise, targets, copies */
#define TTT_KC_NORM 4  /* RMSNorm forward and backward */
#define TTT_KC_ROPE 5  /* QK-norm + RoPE forward (with the KV-ring write) and backward */
#define TTT_KC_DECODE 6 /* generation's per-position kernels; their third total counts algorithmic
                           HBM bytes (weights and window keys/values read), not flops */
#define TTT_KC_COUNT 7
int ttt_timing_enable(ttt_ctx* ctx, int32_t enable);
int ttt_timing_read(ttt_ctx* ctx, int32_t kernel_class, double* total_ms, int64_t* launches, double* flops);

#ifdef __cplusplus
}
#endif
#endif /* TTT_H_ */
