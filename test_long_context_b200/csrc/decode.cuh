// Kernels of greedy generation (one position at a time): matrix-vector
// products with the prefill's epilogues, a greedy pick fused into the
// LM-head product, and single-query attention over the window.  All are
// bound by HBM bandwidth: every generated position streams the weights and
// the window's keys and values once.
#pragma once
#include "common.cuh"

namespace ttt {

enum GemvEpi : int {
  GEMV_STORE = 0,    // out (T) [n] = y
  GEMV_ADD_F32 = 1,  // out (fp32) [n] = res[n] + y
  GEMV_SWIGLU = 2,   // rows in (gate 64 | up 64) blocks: out (T) [n/2] = silu(g) * u; raw (T) [n] = y
  GEMV_ARGMAX = 3,   // per block: (max y, lowest row with that max, sum exp(y - max)) -> part
};

// y[r] = W[r, :] . x  (+ W2[r - n_ext, :] . x2 for rows r >= n_ext), fp32
// accumulation of T products.  W rows (and W2 rows) must start on 16-byte
// boundaries, k and k2 be multiples of 16 / sizeof(T).
template <typename T>
struct GemvArgs {
  const T* w = nullptr;
  int64_t ldw = 0, n = 0, k = 0;
  const T* x = nullptr;
  const T* w2 = nullptr;
  int64_t ldw2 = 0, k2 = 0, n_ext = INT64_MAX;
  const T* x2 = nullptr;
  void* out = nullptr;
  const float* res = nullptr;
  T* raw = nullptr;
  float* part = nullptr;  // GEMV_ARGMAX: [gemv_parts(n)] x 3 floats
  // RMSNorm prologue (when xres is set, x is not read): x = T(xres * r * gain)
  // with r = 1/sqrt(mean(xres^2) + eps), computed by every block; block 0
  // also writes x to h_out and r to r_out (either may be NULL).  x2 == NULL
  // with w2 set means the second product reads the same normalised x.
  const float* xres = nullptr;
  const float* gain = nullptr;
  float eps = 0.f;
  T* h_out = nullptr;
  float* r_out = nullptr;
};

// Blocks a GEMV_ARGMAX launch writes partials for.
int64_t gemv_parts(int64_t n);
template <typename T>
int gemv(const GemvArgs<T>& a, int epi, cudaStream_t s);

// Greedy pick from the GEMV_ARGMAX partials: the largest logit (ties: the
// lowest token id).  Writes the token to tok_out and, when non-NULL, to
// tgt_row; the log-sum-exp of the row to lse_row (when non-NULL); and the
// row's loss against the picked token, lse - max, to loss_out (when non-NULL).
int argmax_finalize(const float* part, int64_t nparts, int32_t* tok_out, int32_t* tgt_row, float* lse_row,
                    float* loss_out, cudaStream_t s);

// One query per head at absolute position p over the keys p-window+1 .. p
// in the rings (slot = position % R): o (T) [H*HD], lse[h * ld_lse] (natural
// log of the scaled scores' sum of exponentials; skipped when lse is NULL).
// ws: fp32 work space of attn_decode_ws_floats(H, HD, window) floats, its
// last H words zero before the first call (every call leaves them zero);
// window <= 16 384.
int64_t attn_decode_ws_floats(int H, int HD, int64_t window);
template <typename T>
int attn_decode(const T* q, const T* kring, const T* vring, int64_t ldkv, int64_t R, int H, int HD, int64_t p,
                int64_t window, float scale, T* o, float* lse, int64_t ld_lse, float* ws, cudaStream_t s);

// dst[i] = v, i < n.
int fill_f32(float* dst, int64_t n, float v, cudaStream_t s);

}  // namespace ttt
