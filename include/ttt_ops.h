/*
 * ttt_ops.h — op-level C ABI of the kernels behind ttt.h, for testing each
 * stage of the prefill loop on its own.  Every call is asynchronous on
 * `stream` (a cudaStream_t, NULL = legacy default stream); pointers are
 * device pointers owned by the caller; the return value is TTT_OK or a
 * TTT_ERR_* code from ttt.h (message: ttt_last_error(NULL)).  Kernel-side
 * failures (bounded waits that gave up) are reported by ttt_op_sync().
 */
#ifndef TTT_OPS_H_
#define TTT_OPS_H_

#include <stdint.h>

#include "ttt.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Epilogues of ttt_op_gemm (acc = the fp32 accumulator of one output element). */
#define TTT_EPI_STORE_F32 0  /* c (fp32) = acc */
#define TTT_EPI_STORE_BF16 1 /* c (bf16) = acc */
#define TTT_EPI_ADD_F32 2    /* c (fp32) = r + acc with r = c2 (fp32) if given, else c itself
                                (residual update, x_out = x_in + o W^T) */
#define TTT_EPI_SWIGLU 3     /* columns in (gate 64 | up 64) pairs: c[:, 64*pair + i] = silu(g) * u;
                                c2 (optional) = raw acc.  Output dtype = the GEMM's dtype. */
#define TTT_EPI_CE_FWD 4     /* softmax-CE partials per row and N tile (see below) */
#define TTT_EPI_CE_BWD 5     /* c = (exp(acc - row_f[m]) - [n + col_offset == row_i[m]]) * row_g[m] */
#define TTT_EPI_SGD 6        /* c (fp32) -= alpha * acc;  c2 (optional, bf16) = hi = bf16(new c);
                                c3 (optional, with c2) = lo = bf16(new c - hi) */

typedef struct ttt_epilogue_args {
  void* c;
  int64_t ldc;
  void* c2;
  int64_t ldc2;
  const float* row_f;      /* CE_BWD: log-sum-exp per row */
  const float* row_g;      /* CE_BWD: scale per row (1/n_c, or 0 for rows without a target) */
  const int32_t* row_i;    /* CE_FWD / CE_BWD: target id per row */
  float* part_max;         /* CE_FWD: [n_tiles, part_ld] running max per tile and row */
  float* part_sum;         /* CE_FWD: [n_tiles, part_ld] sum of exp(acc - max) */
  float* target_logit;     /* CE_FWD: acc at the target column (written by the tile holding it) */
  int64_t part_ld;
  float alpha;             /* SGD: learning rate */
  int64_t col_offset;      /* global column index of output column 0 (vocab chunks) */
  void* c3;                /* SGD: low bf16 half of the new master (NULL: none) */
  int64_t ldc3;
} ttt_epilogue_args;

/*
 * acc[m][n] = sum_k A(m,k) B(n,k) for m < M, n < N, then the epilogue.
 * dtype TTT_BF16 runs the tcgen05 tensor-core kernel (bf16 operands, fp32
 * accumulation); TTT_F32 the fp32 SIMT kernel (all operands fp32).
 * a_mn = 0: A stored [M, K] with row pitch lda;  a_mn = 1: stored [K, M].
 * b_mn = 0: B stored [N, K] with row pitch ldb;  b_mn = 1: stored [K, N].
 * bf16 operands: 16-byte aligned base and row pitch.  (a_mn, b_mn) = (1, 0)
 * is not supported with TTT_BF16.  bn_hint: 0 (auto), 128, 160 or 256
 * (tile width; TTT_BF16 only; 160 only with M > 128 and the STORE_F32,
 * STORE_BF16 or ADD_F32 epilogue).  A GEMM with M > 128 runs on CTA pairs
 * (clusters of two CTAs, one 256 x tile-width output tile per pair;
 * environment TTT_GEMM_PAIR=0 keeps single CTAs); the results do not depend
 * on it.  CE_FWD writes ceil(N / tile) partial tiles: query the tile count
 * with ttt_op_gemm_ce_tiles.
 */
int ttt_op_gemm(int32_t dtype, int32_t a_mn, int32_t b_mn, int64_t M, int64_t N, int64_t K, const void* A,
                int64_t lda, const void* B, int64_t ldb, int32_t epilogue, const ttt_epilogue_args* args,
                int32_t bn_hint, void* stream);

/*
 * ttt_op_gemm (TTT_BF16 only) with the K range split into ksplit parts: each
 * part's fp32 partial product goes to `workspace` (caller-owned, at least
 * ksplit * M * N floats), then one kernel sums the parts in a fixed order
 * (run-to-run identical results) and applies the epilogue.  Epilogues:
 * TTT_EPI_STORE_F32, TTT_EPI_STORE_BF16, TTT_EPI_ADD_F32.  ksplit <= 1 is the
 * plain GEMM.  Useful when the output alone has too few tiles to fill the GPU.
 */
/*
 * Two products into one accumulator (TTT_BF16 only):
 *   acc[m][n] = sum_k A(m,k) B(n,k)  +  [n >= n_ext] sum_k' A2(m,k') B2(n - n_ext, k')
 * then the epilogue.  A2 / B2 take the orientation of A / B (a_mn, b_mn) and
 * have K2 columns of reduction; B2 covers the N - n_ext outputs from n_ext
 * on, and n_ext must be a multiple of the tile width (bn_hint; 128 always
 * works).  ksplit > 1 (workspace as in ttt_op_gemm_split) needs n_ext = 0.
 * The prefill uses it for the fast MLP: a fast weight is kept as a bf16 pair
 * hi + lo of its fp32 master, and h (W_hi + W_lo)^T is h W_hi^T + h W_lo^T.
 * Not an operation of the method itself: a precision device of this library.
 */
int ttt_op_gemm_dual(int32_t a_mn, int32_t b_mn, int64_t M, int64_t N, int64_t K, const void* A, int64_t lda,
                     const void* B, int64_t ldb, int64_t K2, const void* A2, int64_t lda2, const void* B2,
                     int64_t ldb2, int64_t n_ext, int32_t epilogue, const ttt_epilogue_args* args, int32_t bn_hint,
                     int32_t ksplit, float* workspace, void* stream);

int ttt_op_gemm_split(int32_t a_mn, int32_t b_mn, int64_t M, int64_t N, int64_t K, const void* A, int64_t lda,
                      const void* B, int64_t ldb, int32_t epilogue, const ttt_epilogue_args* args, int32_t bn_hint,
                      int32_t ksplit, float* workspace, void* stream);

/* Number of N tiles a CE_FWD ttt_op_gemm of width N writes partials for. */
int64_t ttt_op_gemm_ce_tiles(int32_t dtype, int64_t M, int64_t N, int32_t bn_hint);

/*
 * The launch plan the prefill uses for a bf16 M x N x K product with this
 * epilogue: returns the split-K count (1 = none) and writes the tile width
 * to *bn_out (0 = the automatic choice of ttt_op_gemm).  Pass both to
 * ttt_op_gemm_split (workspace: split * M * N floats) to run the product as
 * the prefill does.  No device work.
 */
int64_t ttt_op_gemm_plan(int64_t M, int64_t N, int64_t K, int32_t epilogue, int32_t* bn_out);

/*
 * Sliding-window causal attention, eq. (1) of the reading notes: query at
 * absolute position p = q_pos0 + i attends to keys p-window+1 .. p.
 *   q, o: [n_q, ldq] / [n_q, ldo] rows, head h in columns h*head_dim ...
 *   k_ring, v_ring: [ring_slots, n_heads*head_dim]; the key at position j is
 *   in slot j % ring_slots, so ring_slots >= window + n_q - 1 is required
 *   when the ring holds earlier positions as well.
 *   lse: [n_heads, n_q] fp32 natural-log log-sum-exp of the scaled scores.
 * dtype TTT_F32 (all fp32, SIMT) or TTT_BF16 (bf16 tensors).  With TTT_BF16,
 * head_dim in {64, 80, 96, 128}, ring_slots a multiple of 128 and flags bit 0
 * clear, the tcgen05 tensor-core kernel runs (fp32 softmax, bf16 P); otherwise
 * the SIMT kernel (fp32 math).  Scores are scaled by 1/sqrt(head_dim).
 *
 * q_norm_max, k_norm_max (0 = unknown): upper bounds on the Euclidean norm
 * of every query row and every key row of a head, e.g. max|gain| *
 * sqrt(head_dim) after an RMSNorm with that gain (the model's QK-norm).  With
 * both given and log2(e) q_norm_max k_norm_max / sqrt(head_dim) <= 48 (about
 * 47.5 with the 1% allowance for bf16 rounding), the tensor-core path shifts
 * each query row's softmax by the Cauchy-Schwarz bound of its scores instead
 * of a running maximum (the same result: softmax is shift-invariant), which
 * lets it skip the max reduction and the rescaling of o.  The bounds are the
 * caller's promise; keys up to 3.5x longer than k_norm_max still give exact
 * results.
 * flags bits 4..7, TTT_SWA_EXP_POLY(n): on that path n of every 8 groups of
 * 8 keys (n in 0, 2, 4) take 2^x from an FMA-pipe polynomial (relative error
 * 7.5e-5) instead of the MUFU unit; 0 in these bits = library default.
 */
#define TTT_SWA_FORCE_SIMT 1
#define TTT_SWA_EXP_POLY(n) ((((n) + 1) & 15) << 4)
int ttt_op_swa_forward(int32_t dtype, int32_t n_heads, int32_t head_dim, int64_t n_q, int64_t q_pos0, int32_t window,
                       const void* q, int64_t ldq, const void* k_ring, const void* v_ring, int64_t ring_slots,
                       void* o, int64_t ldo, float* lse, float q_norm_max, float k_norm_max, int32_t flags,
                       void* stream);

/*
 * Backward of ttt_op_swa_forward given dout = dL/do: dq for every query (over
 * the full band, cached keys included) and dk, dv for the keys at positions
 * q_pos0 .. q_pos0+n_q-1 only (row i = position q_pos0 + i); keys of earlier
 * positions are treated as constants.  dq: [n_q, lddq]; dk, dv: [n_q, lddkv].
 * D_scratch: fp32 [n_heads * n_q] work space.  With TTT_BF16, head_dim in
 * {64, 80, 96, 128}, ring_slots a multiple of 128, q and dout with the same
 * row pitch, and flags bit 0 (TTT_SWA_FORCE_SIMT) clear, dq is computed on
 * the tensor cores; everything else uses the SIMT kernels.
 */
int ttt_op_swa_backward(int32_t dtype, int32_t n_heads, int32_t head_dim, int64_t n_q, int64_t q_pos0, int32_t window,
                        const void* q, int64_t ldq, const void* k_ring, const void* v_ring, int64_t ring_slots,
                        const void* o, int64_t ldo, const float* lse, const void* dout, int64_t lddo, void* dq,
                        int64_t lddq, void* dk, void* dv, int64_t lddkv, float* D_scratch, int32_t flags,
                        void* stream);

/*
 * Allocation-free variant of ttt_op_swa_backward.  The paper has no
 * counterpart: this is an addition for callers that may not allocate device
 * memory, because their memory belongs to another allocator (a framework's
 * caching pool, a fixed budget) and cudaMalloc would bypass it and
 * synchronise the whole device.
 * Same arguments and results as ttt_op_swa_backward without D_scratch: the
 * work array lives inside the library as a fixed 1 MiB array per GPU that
 * loads the library (held until the process exits), so n_heads * n_q must
 * not exceed 262144; larger calls return TTT_ERR_INVALID_ARG and change
 * nothing.  It calls no cudaMalloc or cudaFree.
 * The first call on each device looks up the array's device address
 * (cudaGetSymbolAddress) with that device current; make that first call
 * before any stream capture.
 * Every call uses the same array and leaves its last contents there (each
 * entry is rewritten before it is read, so nothing needs clearing); calls
 * whose work overlaps on the GPU (other streams, other host threads) race
 * on it and must be serialised by the caller.
 */
int ttt_op_swa_backward_noalloc(int32_t dtype, int32_t n_heads, int32_t head_dim, int64_t n_q, int64_t q_pos0,
                                int32_t window, const void* q, int64_t ldq, const void* k_ring, const void* v_ring,
                                int64_t ring_slots, const void* o, int64_t ldo, const float* lse, const void* dout,
                                int64_t lddo, void* dq, int64_t lddq, void* dk, void* dv, int64_t lddkv,
                                void* stream);

/*
 * Memory-bound kernels of the loop, one launch each (bf16 only; they exist so
 * that each can be timed and profiled on its own at the workload's shapes).
 *
 * RMSNorm (reading notes §6 block structure, pre-norm): for row i < n,
 * r = 1/sqrt(mean_j x[i,j]^2 + eps), y[i,j] = bf16(x[i,j] * r * g[j]),
 * rstd[i] = r.  x fp32 [n, ldx], g fp32 [d], y bf16 [n, ldy], rstd fp32 [n].
 */
int ttt_op_rmsnorm(int64_t n, int32_t d, const float* x, int64_t ldx, const float* g, float eps, void* y,
                   int64_t ldy, float* rstd, void* stream);

/*
 * QK-norm + RoPE of n positions p0 .. p0+n-1 with the key/value ring write:
 * qkv bf16 [n, ldqkv] holds (q | k | v) raw projections of n_heads heads of
 * head_dim; per head q and k get RMSNorm over head_dim (gains gq, gk fp32
 * [head_dim]) and the rotation of pairs (i, i + head_dim/2) by angle
 * p * theta^(-2i/head_dim); q goes to qout [n, ldq], k and v to the rings
 * [R, n_heads*head_dim] at slot p % R; rq, rk fp32 [n, n_heads] receive the
 * RMS factors.  The angles are computed in fp64 into a table (scratch `tab`,
 * fp32 pairs [n, head_dim/2], caller-owned) first.
 */
int ttt_op_qknorm_rope(int64_t n, int64_t p0, int32_t n_heads, int32_t head_dim, float eps, float theta,
                       const void* qkv, int64_t ldqkv, const float* gq, const float* gk, void* qout, int64_t ldq,
                       void* kring, void* vring, int64_t R, float* rq, float* rk, float* tab, void* stream);

/*
 * SwiGLU backward on (gate 64 | up 64) interleaved columns: for n rows and
 * nfeat features j (pair j/64, lane j%64), with g, u from gu [n, ldgu] and
 * da [n, ldda] (all bf16): dg = da * u * s(g) * (1 + g (1 - s(g))),
 * du = da * g * s(g) (s = sigmoid), written interleaved to dgu [n, lddgu].
 */
int ttt_op_swiglu_bwd(int64_t n, int64_t nfeat, const void* da, int64_t ldda, const void* gu, int64_t ldgu,
                      void* dgu, int64_t lddgu, void* stream);

/*
 * Matrix-vector product of generation (bf16 W [n, ldw], x [k]; fp32
 * accumulation): epilogue 0 stores y (bf16 [n]) to out, 1 adds y to res
 * (fp32 [n]) into out (fp32), 2 applies SwiGLU to (gate 64 | up 64) row
 * blocks (out bf16 [n/2], raw bf16 [n] or NULL), 3 greedy-picks: out (int32
 * [1]) = the row with the largest y (ties: the lowest row), lse_out (fp32 [1],
 * may be NULL) = log sum exp y; part is scratch of 3 * 1184 floats.  Rows
 * 16-byte aligned, k a multiple of 8.
 */
int ttt_op_gemv(int32_t epilogue, int64_t n, int64_t k, const void* w, int64_t ldw, const void* x, void* out,
                const float* res, void* raw, float* lse_out, float* part, void* stream);

/*
 * One query per head at absolute position p over keys p-window+1 .. p of the
 * rings (bf16 [R, n_heads*head_dim], slot = position % R, R >= window): o
 * (bf16 [n_heads*head_dim]) and lse (fp32 [n_heads], natural log, may be
 * NULL); scores scaled by 1/sqrt(head_dim).  ws: fp32 scratch of
 * n_heads * ((ceil(window / 128) + 1) * (head_dim + 2) + 1) floats whose last
 * n_heads words are zero before the first call (each call leaves them zero:
 * they count the finished splits of each head).  window <= 16384.
 */
int ttt_op_attn_decode(int32_t n_heads, int32_t head_dim, int64_t p, int32_t window, const void* q,
                       const void* kring, const void* vring, int64_t R, void* o, float* lse, float* ws,
                       void* stream);

/*
 * Outer-loop meta-gradient (End-to-End Test-Time Training for Long Context;
 * reading notes by Zhongzhu Zhou, §4, eqs. (5)-(7)) for a fast SwiGLU MLP in
 * the model's last block, the only block with fast weights.  Per chunk c of
 * b rows, with W = (w_gate, w_up, w_down):
 *   A_c(W) = mean over the chunk's rows with a target of
 *            CE(RMSNorm(r + (silu(h w_gate^T) * (h w_up^T)) w_down^T; g_final) w_head^T, target),
 * where h (the block's MLP-norm output) and r (the residual plus the static
 * MLP's output) do not depend on W, so eq. (7) is exact for this loss.
 * Inner loop W^(c+1) = W^(c) - eta grad A_c(W^(c)) from W^(0) = the given
 * weights (eq. (5)); outer loss L = (1/N) sum_c A_c(W^(c)); outputs
 * d_* = dL/dW^(0) = (1/N) sum_c J_c^T grad A_c(W^(c)), J_(c+1) = (I - eta H_c) J_c
 * (eq. (7)), evaluated from the last chunk backwards with Hessian-vector
 * products (eq. (6)).  All fp32, row-major:
 *   h, r      [n_chunks * b, d];  targets int32 [n_chunks * b], -1 = no target
 *             (another id outside [0, vocab) counts as none and makes
 *             ttt_op_sync return TTT_ERR_INVALID_ARG);
 *   w_gate, w_up, d_gate, d_up [f, d];  w_down, d_down [d, f];
 *   g_final [d];  w_head [vocab, d];  eps > 0 (RMSNorm);  eta finite;
 *   losses    (optional, [n_chunks * b]) the per-row losses along the inner
 *             loop, each scored with the W before its chunk's step (NaN
 *             without a target);
 *   work      scratch of at least ttt_op_meta_grad_work(...) floats, owned by
 *             the caller, not read before it is written.
 * The inputs are not modified.  Logits are materialised per chunk ([b, vocab]
 * three times in work).  Errors: TTT_ERR_INVALID_ARG (sizes < 1, NULL
 * pointers, work too small, eta or eps not finite or eps <= 0), TTT_ERR_CUDA.
 */
int64_t ttt_op_meta_grad_work(int64_t n_chunks, int64_t b, int32_t d, int32_t f, int64_t vocab);
int ttt_op_meta_grad(int64_t n_chunks, int64_t b, int32_t d, int32_t f, int64_t vocab, const float* h,
                     const float* r, const int32_t* targets, const float* w_gate, const float* w_up,
                     const float* w_down, const float* g_final, const float* w_head, float eps, float eta,
                     float* d_gate, float* d_up, float* d_down, float* losses, float* work, int64_t work_floats,
                     void* stream);

/* Device watchdog self-test: launches one thread that waits on an mbarrier
 * nothing ever arrives at.  The bounded wait gives up (about 2 s) and records
 * a timeout, so the following ttt_op_sync returns TTT_ERR_TIMEOUT and the
 * context stays usable. */
int ttt_op_watchdog_selftest(void* stream);

/* Wait for `stream`; return TTT_ERR_TIMEOUT if a kernel launched through this
 * header recorded a bounded-wait timeout since the last call, TTT_ERR_INVALID_ARG
 * if one met a target id outside its range (then clears the record). */
int ttt_op_sync(void* stream);

#ifdef __cplusplus
}
#endif
#endif /* TTT_OPS_H_ */
