// Outer-loop meta-gradient of the adapted loss with respect to the initial
// fast weights (End-to-End Test-Time Training for Long Context; reading notes
// by Zhongzhu Zhou, §4: eqs. (5)-(7)), for a fast SwiGLU MLP in the last
// block, the case in which eq. (7) is exact: the MLP reads the block's
// MLP-norm output h and adds to the residual r, then the final RMSNorm, the
// LM head and the next-token cross-entropy; h and r do not depend on W.
//
//   inner loop    W^(c+1) = W^(c) - eta grad A_c(W^(c))                (eq. (5))
//   outer loss    L = (1/N) sum_c A_c(W^(c))                          (eq. (4), by chunks)
//   meta-gradient u = grad A_(N-1) / N; u <- u - eta H_c u + grad A_c / N, c = N-2 .. 0
//                 (eq. (7) evaluated backwards; H_c u by eq. (6))
//
// H_c u is the directional derivative of the chunk gradient along u: every
// step of the forward and of the backward carries a tangent (forward mode
// over the hand-derived backward).  All arithmetic is fp32: the products are
// the fp32 SIMT GEMM, the rest are row kernels (norm, cross-entropy) and
// elementwise kernels (SwiGLU and its derivatives, the updates) below.
#include <cmath>

#include "../../include/ttt_ops.h"
#include "gemm.cuh"

namespace ttt {

int* op_err_word();

namespace {

constexpr int kRowThreads = 256;

__device__ __forceinline__ float sigm(float g) { return 1.f / (1.f + expf(-g)); }

// Sum of v over the block (kRowThreads threads); every thread gets the total.
__device__ float block_sum(float v, float* red) {
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  __syncthreads();  // red may still be read by a previous call
  if (l == 0) red[w] = v;
  __syncthreads();
  float t = 0.f;
#pragma unroll
  for (int i = 0; i < kRowThreads / 32; ++i) t += red[i];
  return t;
}

__device__ float block_max(float v, float* red) {
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  __syncthreads();
  if (l == 0) red[w] = v;
  __syncthreads();
  float t = -INFINITY;
#pragma unroll
  for (int i = 0; i < kRowThreads / 32; ++i) t = fmaxf(t, red[i]);
  return t;
}

// w = 1 / (number of rows with a target) or 0; a target outside [-1, V)
// sets the error word and counts as no target.
__global__ void count_targets_kernel(const int32_t* __restrict__ tgt, int64_t n, int64_t V, float* w, int* err) {
  __shared__ float red[kRowThreads / 32];
  float c = 0.f;
  for (int64_t i = threadIdx.x; i < n; i += kRowThreads) {
    const int32_t t = tgt[i];
    if (t >= 0 && t < V) c += 1.f;
    else if (t != -1) atomicOr(err, DEV_ERR_BAD_TOKEN);
  }
  c = block_sum(c, red);
  if (threadIdx.x == 0) *w = c > 0.f ? 1.f / c : 0.f;
}

// a = silu(G) U;  tangent at = silu'(G) Gt U + silu(G) Ut.
__global__ void swiglu_fwd_kernel(const float* __restrict__ G, const float* __restrict__ U,
                                  const float* __restrict__ Gt, const float* __restrict__ Ut, float* __restrict__ a,
                                  float* __restrict__ at, int64_t total) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x) {
    const float g = G[i], u = U[i], s = sigm(g), sl = g * s;
    if (a) a[i] = sl * u;
    if (at) {
      const float d1 = s * (1.f + g * (1.f - s));
      at[i] = d1 * Gt[i] * u + sl * Ut[i];
    }
  }
}

// dG = da U silu'(G), dU = da silu(G); with tangents (da_t, Gt, Ut given):
// dGt = da_t U s' + da Ut s' + da U s'' Gt,  dUt = da_t silu(G) + da s' Gt.
__global__ void swiglu_bwd_kernel(const float* __restrict__ G, const float* __restrict__ U,
                                  const float* __restrict__ da, float* __restrict__ dG, float* __restrict__ dU,
                                  const float* __restrict__ Gt, const float* __restrict__ Ut,
                                  const float* __restrict__ dat, float* __restrict__ dGt, float* __restrict__ dUt,
                                  int64_t total) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x) {
    const float g = G[i], u = U[i], s = sigm(g), sl = g * s;
    const float d1 = s * (1.f + g * (1.f - s));
    const float dai = da[i];
    if (dG) {
      dG[i] = dai * u * d1;
      dU[i] = dai * sl;
    }
    if (dGt) {
      const float d2 = s * (1.f - s) * (2.f + g * (1.f - 2.f * s));
      const float gt = Gt[i], ut = Ut[i], dati = dat[i];
      dGt[i] = dati * u * d1 + dai * ut * d1 + dai * u * d2 * gt;
      dUt[i] = dati * sl + dai * d1 * gt;
    }
  }
}

// One block per row: rr = 1/sqrt(mean(x^2) + eps), y = x rr g; with the
// tangent xt: rrt = -rr^3 mean(x xt), yt = g (xt rr + x rrt).
__global__ void __launch_bounds__(kRowThreads) norm_fwd_kernel(const float* __restrict__ x,
                                                               const float* __restrict__ gain, int64_t d, float eps,
                                                               float* __restrict__ y, float* __restrict__ rr,
                                                               const float* __restrict__ xt, float* __restrict__ yt,
                                                               float* __restrict__ rrt) {
  __shared__ float red[kRowThreads / 32];
  const int64_t row = blockIdx.x;
  const float* xr = x + row * d;
  float s = 0.f;
  for (int64_t j = threadIdx.x; j < d; j += kRowThreads) s += xr[j] * xr[j];
  s = block_sum(s, red);
  const float r = rsqrtf(s / (float)d + eps);
  if (y) {
    for (int64_t j = threadIdx.x; j < d; j += kRowThreads) y[row * d + j] = xr[j] * r * gain[j];
    if (threadIdx.x == 0) rr[row] = r;
  }
  if (xt) {
    const float* xtr = xt + row * d;
    float t = 0.f;
    for (int64_t j = threadIdx.x; j < d; j += kRowThreads) t += xr[j] * xtr[j];
    t = block_sum(t, red);
    const float rt = -r * r * r * t / (float)d;
    for (int64_t j = threadIdx.x; j < d; j += kRowThreads) yt[row * d + j] = gain[j] * (xtr[j] * r + xr[j] * rt);
    if (threadIdx.x == 0) rrt[row] = rt;
  }
}

// One block per row: dx = rr q - rr^3 x m with q = g dy, m = mean(x q); with
// tangents (xt, rrt, dyt): dxt = rrt q + rr qt - 3 rr^2 rrt x m - rr^3 xt m
// - rr^3 x mt, qt = g dyt, mt = mean(xt q + x qt).
__global__ void __launch_bounds__(kRowThreads) norm_bwd_kernel(const float* __restrict__ x,
                                                               const float* __restrict__ gain,
                                                               const float* __restrict__ rr, const float* __restrict__ dy,
                                                               int64_t d, float* __restrict__ dx,
                                                               const float* __restrict__ xt,
                                                               const float* __restrict__ rrt,
                                                               const float* __restrict__ dyt, float* __restrict__ dxt) {
  __shared__ float red[kRowThreads / 32];
  const int64_t row = blockIdx.x;
  const float* xr = x + row * d;
  const float* dyr = dy + row * d;
  float m = 0.f;
  for (int64_t j = threadIdx.x; j < d; j += kRowThreads) m += xr[j] * gain[j] * dyr[j];
  m = block_sum(m, red) / (float)d;
  const float r = rr[row], r3 = r * r * r;
  if (dx)
    for (int64_t j = threadIdx.x; j < d; j += kRowThreads) dx[row * d + j] = r * gain[j] * dyr[j] - r3 * xr[j] * m;
  if (dxt) {
    const float* xtr = xt + row * d;
    const float* dytr = dyt + row * d;
    float mt = 0.f;
    for (int64_t j = threadIdx.x; j < d; j += kRowThreads) mt += xtr[j] * gain[j] * dyr[j] + xr[j] * gain[j] * dytr[j];
    mt = block_sum(mt, red) / (float)d;
    const float rt = rrt[row];
    for (int64_t j = threadIdx.x; j < d; j += kRowThreads) {
      const float q = gain[j] * dyr[j], qt = gain[j] * dytr[j];
      dxt[row * d + j] = rt * q + r * qt - 3.f * r * r * rt * xr[j] * m - r3 * xtr[j] * m - r3 * xr[j] * mt;
    }
  }
}

// One block per row of the logits z [n, V]: lse, the loss (NaN without a
// target) and dz = w (softmax(z) - onehot(target)) (0 without a target).
__global__ void __launch_bounds__(kRowThreads) ce_kernel(const float* __restrict__ z, int64_t V,
                                                         const int32_t* __restrict__ tgt, const float* __restrict__ w,
                                                         float* __restrict__ lse_out, float* __restrict__ loss_out,
                                                         float* __restrict__ dz) {
  __shared__ float red[kRowThreads / 32];
  const int64_t row = blockIdx.x;
  const float* zr = z + row * V;
  float mx = -INFINITY;
  for (int64_t j = threadIdx.x; j < V; j += kRowThreads) mx = fmaxf(mx, zr[j]);
  mx = block_max(mx, red);
  float s = 0.f;
  for (int64_t j = threadIdx.x; j < V; j += kRowThreads) s += expf(zr[j] - mx);
  s = block_sum(s, red);
  const float lse = mx + logf(s);
  const int32_t t = tgt[row];
  const bool valid = t >= 0 && t < V;
  const float wr = valid ? *w : 0.f;
  if (threadIdx.x == 0) {
    lse_out[row] = lse;
    if (loss_out) loss_out[row] = valid ? lse - zr[t] : NAN;
  }
  for (int64_t j = threadIdx.x; j < V; j += kRowThreads)
    dz[row * V + j] = valid ? wr * (expf(zr[j] - lse) - (j == t ? 1.f : 0.f)) : 0.f;
}

// Tangent of dz along zt (in place): zt <- w p (zt - <p, zt>), p = softmax(z).
__global__ void __launch_bounds__(kRowThreads) ce_tangent_kernel(const float* __restrict__ z, int64_t V,
                                                                 const int32_t* __restrict__ tgt,
                                                                 const float* __restrict__ w,
                                                                 const float* __restrict__ lse, float* __restrict__ zt) {
  __shared__ float red[kRowThreads / 32];
  const int64_t row = blockIdx.x;
  const float* zr = z + row * V;
  float* ztr = zt + row * V;
  const int32_t t = tgt[row];
  if (!(t >= 0 && t < V)) {
    for (int64_t j = threadIdx.x; j < V; j += kRowThreads) ztr[j] = 0.f;
    return;
  }
  const float l = lse[row];
  float c = 0.f;
  for (int64_t j = threadIdx.x; j < V; j += kRowThreads) c += expf(zr[j] - l) * ztr[j];
  c = block_sum(c, red);
  const float wr = *w;
  for (int64_t j = threadIdx.x; j < V; j += kRowThreads) ztr[j] = wr * expf(zr[j] - l) * (ztr[j] - c);
}

// y = x + alpha a + beta b (x, a or b may be null: that term is left out).
__global__ void axpby_kernel(float* y, const float* x, float alpha,
                             const float* __restrict__ a, float beta, const float* __restrict__ b, int64_t total) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x) {
    float v = x ? x[i] : 0.f;
    if (a) v += alpha * a[i];
    if (b) v += beta * b[i];
    y[i] = v;
  }
}

unsigned ew_grid(int64_t total) { return (unsigned)imin64(ceil_div(total, 256), 148 * 16); }

// Scratch of one chunk and the persistent state, carved out of the work array.
struct MetaWork {
  int64_t n, d, f, V, P;
  float *snap;                                   // [N][P] W^(c): w_gate [f,d], w_up [f,d], w_down [d,f]
  float *g, *Hu, *u;                             // [P] each
  float *G, *U, *a, *Gt, *Ut, *at;               // [n, f]
  float *da, *dG, *dU, *dat, *dGt, *dUt;         // [n, f]
  float *x, *nrm, *dn, *dx, *xt, *nt, *dnt, *dxt;  // [n, d]
  float *rr, *rrt, *lse;                         // [n]
  float *z, *dz, *zt;                            // [n, V]
  float *w;                                      // [1] 1 / n_c
};

int64_t meta_work_floats(int64_t N, int64_t n, int64_t d, int64_t f, int64_t V) {
  const int64_t P = 3 * d * f;
  return N * P + 3 * P + 12 * n * f + 8 * n * d + 3 * n + 3 * n * V + 1;
}

MetaWork carve(float* p, int64_t N, int64_t n, int64_t d, int64_t f, int64_t V) {
  MetaWork w;
  w.n = n, w.d = d, w.f = f, w.V = V, w.P = 3 * d * f;
  auto take = [&](int64_t k) { float* q = p; p += k; return q; };
  w.snap = take(N * w.P);
  w.g = take(w.P), w.Hu = take(w.P), w.u = take(w.P);
  float** nf[] = {&w.G, &w.U, &w.a, &w.Gt, &w.Ut, &w.at, &w.da, &w.dG, &w.dU, &w.dat, &w.dGt, &w.dUt};
  for (float** q : nf) *q = take(n * f);
  float** nd[] = {&w.x, &w.nrm, &w.dn, &w.dx, &w.xt, &w.nt, &w.dnt, &w.dxt};
  for (float** q : nd) *q = take(n * d);
  w.rr = take(n), w.rrt = take(n), w.lse = take(n);
  w.z = take(n * V), w.dz = take(n * V), w.zt = take(n * V);
  w.w = take(1);
  return w;
}

// C = A B^T in the GEMM's storage conventions (gemm.cuh); add: C += (or C = R +).
int mm(cudaStream_t st, int a_mn, int b_mn, int64_t M, int64_t N, int64_t K, const float* A, int64_t lda,
       const float* B, int64_t ldb, float* C, int64_t ldc, bool add = false, const float* R = nullptr) {
  GemmShape s;
  s.a_mn = a_mn;
  s.b_mn = b_mn;
  s.a = a_mn ? MatView{A, K, M, lda} : MatView{A, M, K, lda};
  s.b = b_mn ? MatView{B, K, N, ldb} : MatView{B, N, K, ldb};
  EpiArgs e;
  e.c = C;
  e.ldc = ldc;
  if (add && R) {
    e.c2 = const_cast<float*>(R);
    e.ldc2 = ldc;
  }
  return simt_gemm(s, add ? EPI_ADD_F32 : EPI_STORE_F32, e, st);
}

#define META_TRY(expr)        \
  do {                        \
    int rc_ = (expr);         \
    if (rc_) return rc_;      \
  } while (0)

struct MetaIn {
  const float *h, *r, *gain, *head;  // h, r: this chunk's rows
  const int32_t* tgt;
  float eps;
};

// Forward and backward of one chunk at W = (wg, wu, wd): the gradient into
// w.g (and the per-row losses into loss_out when given).
int chunk_grad(const MetaWork& w, const MetaIn& in, const float* W, float* loss_out, int* err, cudaStream_t st) {
  const int64_t n = w.n, d = w.d, f = w.f, V = w.V;
  const float *wg = W, *wu = W + f * d, *wd = W + 2 * f * d;
  float *gg = w.g, *gu = w.g + f * d, *gd = w.g + 2 * f * d;
  count_targets_kernel<<<1, kRowThreads, 0, st>>>(in.tgt, n, V, w.w, err);
  TTT_CUDA_TRY(cudaGetLastError());
  META_TRY(mm(st, 0, 0, n, f, d, in.h, d, wg, d, w.G, f));
  META_TRY(mm(st, 0, 0, n, f, d, in.h, d, wu, d, w.U, f));
  swiglu_fwd_kernel<<<ew_grid(n * f), 256, 0, st>>>(w.G, w.U, nullptr, nullptr, w.a, nullptr, n * f);
  TTT_CUDA_TRY(cudaGetLastError());
  META_TRY(mm(st, 0, 0, n, d, f, w.a, f, wd, f, w.x, d, true, in.r));
  norm_fwd_kernel<<<(unsigned)n, kRowThreads, 0, st>>>(w.x, in.gain, d, in.eps, w.nrm, w.rr, nullptr, nullptr,
                                                       nullptr);
  TTT_CUDA_TRY(cudaGetLastError());
  META_TRY(mm(st, 0, 0, n, V, d, w.nrm, d, in.head, d, w.z, V));
  ce_kernel<<<(unsigned)n, kRowThreads, 0, st>>>(w.z, V, in.tgt, w.w, w.lse, loss_out, w.dz);
  TTT_CUDA_TRY(cudaGetLastError());
  // backward
  META_TRY(mm(st, 0, 1, n, d, V, w.dz, V, in.head, d, w.dn, d));
  norm_bwd_kernel<<<(unsigned)n, kRowThreads, 0, st>>>(w.x, in.gain, w.rr, w.dn, d, w.dx, nullptr, nullptr, nullptr,
                                                       nullptr);
  TTT_CUDA_TRY(cudaGetLastError());
  META_TRY(mm(st, 1, 1, d, f, n, w.dx, d, w.a, f, gd, f));
  META_TRY(mm(st, 0, 1, n, f, d, w.dx, d, wd, f, w.da, f));
  swiglu_bwd_kernel<<<ew_grid(n * f), 256, 0, st>>>(w.G, w.U, w.da, w.dG, w.dU, nullptr, nullptr, nullptr, nullptr,
                                                    nullptr, n * f);
  TTT_CUDA_TRY(cudaGetLastError());
  META_TRY(mm(st, 1, 1, f, d, n, w.dG, f, in.h, d, gg, d));
  META_TRY(mm(st, 1, 1, f, d, n, w.dU, f, in.h, d, gu, d));
  return TTT_OK;
}

// H u at the W of the last chunk_grad call (its activations and adjoints are
// still in w): the tangent of every step above along u, into w.Hu.
int chunk_hvp(const MetaWork& w, const MetaIn& in, const float* W, cudaStream_t st) {
  const int64_t n = w.n, d = w.d, f = w.f, V = w.V;
  const float *wd = W + 2 * f * d;
  const float *ug = w.u, *uu = w.u + f * d, *ud = w.u + 2 * f * d;
  float *hg = w.Hu, *hu = w.Hu + f * d, *hd = w.Hu + 2 * f * d;
  META_TRY(mm(st, 0, 0, n, f, d, in.h, d, ug, d, w.Gt, f));
  META_TRY(mm(st, 0, 0, n, f, d, in.h, d, uu, d, w.Ut, f));
  swiglu_fwd_kernel<<<ew_grid(n * f), 256, 0, st>>>(w.G, w.U, w.Gt, w.Ut, nullptr, w.at, n * f);
  TTT_CUDA_TRY(cudaGetLastError());
  META_TRY(mm(st, 0, 0, n, d, f, w.at, f, wd, f, w.xt, d));
  META_TRY(mm(st, 0, 0, n, d, f, w.a, f, ud, f, w.xt, d, true));
  norm_fwd_kernel<<<(unsigned)n, kRowThreads, 0, st>>>(w.x, in.gain, d, in.eps, nullptr, nullptr, w.xt, w.nt, w.rrt);
  TTT_CUDA_TRY(cudaGetLastError());
  META_TRY(mm(st, 0, 0, n, V, d, w.nt, d, in.head, d, w.zt, V));
  ce_tangent_kernel<<<(unsigned)n, kRowThreads, 0, st>>>(w.z, V, in.tgt, w.w, w.lse, w.zt);
  TTT_CUDA_TRY(cudaGetLastError());
  META_TRY(mm(st, 0, 1, n, d, V, w.zt, V, in.head, d, w.dnt, d));
  norm_bwd_kernel<<<(unsigned)n, kRowThreads, 0, st>>>(w.x, in.gain, w.rr, w.dn, d, nullptr, w.xt, w.rrt, w.dnt,
                                                       w.dxt);
  TTT_CUDA_TRY(cudaGetLastError());
  META_TRY(mm(st, 1, 1, d, f, n, w.dxt, d, w.a, f, hd, f));
  META_TRY(mm(st, 1, 1, d, f, n, w.dx, d, w.at, f, hd, f, true));
  META_TRY(mm(st, 0, 1, n, f, d, w.dxt, d, wd, f, w.dat, f));
  META_TRY(mm(st, 0, 1, n, f, d, w.dx, d, ud, f, w.dat, f, true));
  swiglu_bwd_kernel<<<ew_grid(n * f), 256, 0, st>>>(w.G, w.U, w.da, nullptr, nullptr, w.Gt, w.Ut, w.dat, w.dGt,
                                                    w.dUt, n * f);
  TTT_CUDA_TRY(cudaGetLastError());
  META_TRY(mm(st, 1, 1, f, d, n, w.dGt, f, in.h, d, hg, d));
  META_TRY(mm(st, 1, 1, f, d, n, w.dUt, f, in.h, d, hu, d));
  return TTT_OK;
}

}  // namespace
}  // namespace ttt

using namespace ttt;

extern "C" int64_t ttt_op_meta_grad_work(int64_t n_chunks, int64_t b, int32_t d, int32_t f, int64_t vocab) {
  if (n_chunks < 1 || b < 1 || d < 1 || f < 1 || vocab < 1) return -1;
  return meta_work_floats(n_chunks, b, d, f, vocab);
}

extern "C" int ttt_op_meta_grad(int64_t n_chunks, int64_t b, int32_t d, int32_t f, int64_t vocab, const float* h,
                                const float* r, const int32_t* targets, const float* w_gate, const float* w_up,
                                const float* w_down, const float* g_final, const float* w_head, float eps, float eta,
                                float* d_gate, float* d_up, float* d_down, float* losses, float* work,
                                int64_t work_floats, void* stream) {
  if (n_chunks < 1 || b < 1 || d < 1 || f < 1 || vocab < 1 || !h || !r || !targets || !w_gate || !w_up || !w_down ||
      !g_final || !w_head || !d_gate || !d_up || !d_down || !work || !std::isfinite(eta) || !(eps > 0.f) ||
      !std::isfinite(eps) || b > 0x7fffffff)
    return set_error(TTT_ERR_INVALID_ARG, "ttt_op_meta_grad: bad argument");
  const int64_t need = meta_work_floats(n_chunks, b, d, f, vocab);
  if (work_floats < need)
    return set_error(TTT_ERR_INVALID_ARG, "ttt_op_meta_grad: work holds " + std::to_string(work_floats) +
                                              " floats, needs " + std::to_string(need));
  int* err = op_err_word();
  if (!err) return set_error(TTT_ERR_CUDA, "ttt_op_meta_grad: no device error word");
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int64_t N = n_chunks, n = b, P = 3 * (int64_t)d * f, fd = (int64_t)f * d;
  MetaWork w = carve(work, N, n, d, f, vocab);
  auto in_of = [&](int64_t c) {
    MetaIn in;
    in.h = h + c * n * d;
    in.r = r + c * n * d;
    in.tgt = targets + c * n;
    in.gain = g_final;
    in.head = w_head;
    in.eps = eps;
    return in;
  };
  // W^(0) into the first snapshot
  TTT_CUDA_TRY(cudaMemcpyAsync(w.snap, w_gate, fd * sizeof(float), cudaMemcpyDeviceToDevice, st));
  TTT_CUDA_TRY(cudaMemcpyAsync(w.snap + fd, w_up, fd * sizeof(float), cudaMemcpyDeviceToDevice, st));
  TTT_CUDA_TRY(cudaMemcpyAsync(w.snap + 2 * fd, w_down, fd * sizeof(float), cudaMemcpyDeviceToDevice, st));
  // inner loop (eq. (5)): W^(c+1) = W^(c) - eta grad A_c(W^(c)); losses scored before each step
  for (int64_t c = 0; c < N; ++c) {
    const float* Wc = w.snap + c * P;
    META_TRY(chunk_grad(w, in_of(c), Wc, losses ? losses + c * n : nullptr, err, st));
    if (c + 1 < N) {
      axpby_kernel<<<ew_grid(P), 256, 0, st>>>(w.snap + (c + 1) * P, Wc, -eta, w.g, 0.f, nullptr, P);
      TTT_CUDA_TRY(cudaGetLastError());
    }
  }
  // eq. (7) backwards: u = grad A_(N-1) / N (still in w.g), then
  // u <- u - eta H_c u + grad A_c / N at W^(c), c = N-2 .. 0
  axpby_kernel<<<ew_grid(P), 256, 0, st>>>(w.u, nullptr, 1.f / (float)N, w.g, 0.f, nullptr, P);
  TTT_CUDA_TRY(cudaGetLastError());
  for (int64_t c = N - 2; c >= 0; --c) {
    const float* Wc = w.snap + c * P;
    const MetaIn in = in_of(c);
    META_TRY(chunk_grad(w, in, Wc, nullptr, err, st));
    META_TRY(chunk_hvp(w, in, Wc, st));
    axpby_kernel<<<ew_grid(P), 256, 0, st>>>(w.u, w.u, -eta, w.Hu, 1.f / (float)N, w.g, P);
    TTT_CUDA_TRY(cudaGetLastError());
  }
  TTT_CUDA_TRY(cudaMemcpyAsync(d_gate, w.u, fd * sizeof(float), cudaMemcpyDeviceToDevice, st));
  TTT_CUDA_TRY(cudaMemcpyAsync(d_up, w.u + fd, fd * sizeof(float), cudaMemcpyDeviceToDevice, st));
  TTT_CUDA_TRY(cudaMemcpyAsync(d_down, w.u + 2 * fd, fd * sizeof(float), cudaMemcpyDeviceToDevice, st));
  return TTT_OK;
}
