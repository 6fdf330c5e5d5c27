// Memory-bound kernels of the prefill loop: embedding, RMSNorm, QK-norm +
// RoPE (+ KV-ring write), SwiGLU backward, cross-entropy finalisation and
// the fast-weight layout conversions.  Residual streams and gradients of the
// residual are fp32; `T` is the activation (GEMM operand) type.
#pragma once
#include "common.cuh"

namespace ttt {

// x[i, :] = E[tok[i], :] (fp32).  Bad ids read row 0 and set DEV_ERR_BAD_TOKEN.
template <typename T>
int embed_gather(const int32_t* tok, const T* E, int64_t n, int d, int V, float* x, int* err, cudaStream_t s);

// y = x * r * g, r = 1/sqrt(mean(x^2) + eps) per row; rstd[i] = r.
template <typename T>
int rmsnorm_fwd(const float* x, int64_t ldx, const float* g, float eps, int64_t n, int d, T* y, int64_t ldy,
                float* rstd, cudaStream_t s);

// dx = dres + r * (u - xh * mean(xh * u)), u = dy * g, xh = x * r (dres may be
// NULL or alias dx).  Also writes dx16 (activation copy) when non-NULL.
template <typename T>
int rmsnorm_bwd(const float* x, int64_t ldx, const float* rstd, const float* g, const float* dy, int64_t lddy,
                const float* dres, int64_t ldres, int64_t n, int d, float* dx, int64_t lddx, T* dx16, int64_t ld16,
                cudaStream_t s);

// QK-norm + RoPE of a chunk.  qkv: raw projections [n, 3*H*HD] (q | k | v).
// Writes rotated q to qout, rotated k and v into the ring (slot = (p0+i) % R),
// and the per-head RMS factors rq, rk [n, H].
template <typename T>
int qknorm_rope_fwd(const T* qkv, int64_t ldqkv, const float* gq, const float* gk, int64_t n, int64_t p0, int H,
                    int HD, float eps, const float2* tab, int64_t tab_p0, T* qout, int64_t ldq, T* kring, T* vring,
                    int64_t ldkv, int64_t R, float* rq, float* rk, cudaStream_t s);

// In place on dqkv's q and k parts: gradient w.r.t. rotated q,k -> gradient
// w.r.t. the raw projections (RoPE transpose, then per-head RMSNorm backward).
template <typename T>
int qknorm_rope_bwd(T* dqkv, int64_t ld, const T* qkv, int64_t ldqkv, const float* gq, const float* gk,
                    const float* rq, const float* rk, int64_t n, int64_t p0, int H, int HD, const float2* tab,
                    int64_t tab_p0, cudaStream_t s);

// RoPE rotation table of positions p0 .. p0+n-1 (row i = position p0 + i):
// tab[i * HD/2 + t] = (cos, sin)((p0 + i) * theta^(-2t/HD)), angles in fp64.
// qknorm_rope_fwd/bwd read the rows of their positions (tab_p0 = the table's p0).
int rope_table(float2* tab, int64_t p0, int64_t n, int HD, double theta, cudaStream_t s);

// SwiGLU backward on (gate 64 | up 64) interleaved columns: for feature j
// (pair j/64, lane j%64) with g, u from gu and da from da:
//   dg = da * u * s(g) * (1 + g * (1 - s(g))),  du = da * g * s(g).
template <typename T>
int swiglu_bwd(const T* da, int64_t ldda, const T* gu, int64_t ldgu, int64_t n, int64_t nfeat, T* dgu,
               int64_t lddgu, cudaStream_t s);

// Combine CE partials: lse = M + log(sum_t s_t exp(m_t - M)); loss = lse - z_t.
// Rows i < n_valid get loss_out[i] = loss, scale[i] = inv_nc; others NaN / 0.
int ce_finalize(const float* pmax, const float* psum, int64_t part_ld, int tiles, const float* zt, int64_t n,
                int64_t n_valid, float inv_nc, float* loss_out, float* lse, float* scale, cudaStream_t s);

// Softmax-CE gradient of n rows over logit columns col0 .. col0+ncols-1
// from stored fp32 logits z [n, ldz] (column index = vocab id):
//   dz[i, c] = (exp(z[i, col0+c] - lse[i]) - [col0+c == tgt[i]]) * scale[i]  (T, [n, lddz]).
template <typename T>
int ce_grad_from_logits(const float* z, int64_t ldz, const float* lse, const float* scale, const int32_t* tgt,
                        int64_t col0, int64_t n, int64_t ncols, T* dz, int64_t lddz, cudaStream_t s);

// Flags (DEV_ERR_BAD_TOKEN) any id outside [0, V) among tok[0 .. T-1].
int check_tokens(const int32_t* tok, int64_t T, int V, int* err, cudaStream_t s);
// targets[i] = tok[p0+i+1] when p0+i+1 < T, else -1 (no target), i < n.
int chunk_targets(const int32_t* tok, int64_t T, int64_t p0, int64_t n, int32_t* targets, cudaStream_t s);

// Gate/up rows [f, d] each <-> interleaved [2f, d] in blocks of 64 rows
// (gate 64 | up 64), converting the element type on the way.
template <typename TS, typename TD>
int interleave_gate_up(const TS* gate, const TS* up, int f, int d, TD* out, cudaStream_t s);
int deinterleave_gate_up(const float* in, int f, int d, float* gate, float* up, cudaStream_t s);

// dst = bf16(src - bf16(src)) (fp32 source): with bf16(src) it represents src to ~2^-17 relative.
int bf16_lo2d(const float* src, int64_t lds, bf16* dst, int64_t ldd, int64_t rows, int64_t cols, cudaStream_t s);
// dst[r, c] = src[r, c] for r < rows, c < cols (fp32 -> T).
template <typename T>
int copy2d_from_f32(const float* src, int64_t lds, T* dst, int64_t ldd, int64_t rows, int64_t cols, cudaStream_t s);
template <typename T>
int copy2d(const T* src, int64_t lds, T* dst, int64_t ldd, int64_t rows, int64_t cols, cudaStream_t s);

}  // namespace ttt
