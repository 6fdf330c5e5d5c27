// Op-level entry points (include/ttt_ops.h): thin wrappers that validate the
// arguments and launch one kernel family each.
#include <cmath>
#include "../../include/ttt_ops.h"
#include "attention.cuh"
#include "attention_tc.cuh"
#include "decode.cuh"
#include "elementwise.cuh"
#include "gemm.cuh"
#include "ptx.cuh"

namespace ttt {

// Device error word of kernels launched through the op-level entry points.
static __device__ int g_op_err = 0;

int* op_err_word() {
  int* p = nullptr;
  if (cudaGetSymbolAddress(reinterpret_cast<void**>(&p), g_op_err) != cudaSuccess) return nullptr;
  return p;
}

static EpiArgs to_epi(const ttt_epilogue_args* a) {
  EpiArgs e;
  if (!a) return e;
  e.c = a->c;
  e.ldc = a->ldc;
  e.c2 = a->c2;
  e.ldc2 = a->ldc2;
  e.row_f = a->row_f;
  e.row_g = a->row_g;
  e.row_i = a->row_i;
  e.part_max = a->part_max;
  e.part_sum = a->part_sum;
  e.target_logit = a->target_logit;
  e.part_ld = a->part_ld;
  e.alpha = a->alpha;
  e.col_offset = a->col_offset;
  e.c3 = a->c3;
  e.ldc3 = a->ldc3;
  return e;
}

}  // namespace ttt

using namespace ttt;

extern "C" int ttt_op_gemm(int32_t dtype, int32_t a_mn, int32_t b_mn, int64_t M, int64_t N, int64_t K, const void* A,
                           int64_t lda, const void* B, int64_t ldb, int32_t epilogue, const ttt_epilogue_args* args,
                           int32_t bn_hint, void* stream) {
  if (!A || !B || !args || M < 1 || N < 1 || K < 1) return set_error(TTT_ERR_INVALID_ARG, "ttt_op_gemm: bad argument");
  GemmShape s;
  s.a_mn = a_mn ? 1 : 0;
  s.b_mn = b_mn ? 1 : 0;
  s.a = a_mn ? MatView{A, K, M, lda} : MatView{A, M, K, lda};
  s.b = b_mn ? MatView{B, K, N, ldb} : MatView{B, N, K, ldb};
  EpiArgs e = to_epi(args);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (dtype == TTT_F32) return simt_gemm(s, epilogue, e, st);
  if (dtype != TTT_BF16) return set_error(TTT_ERR_INVALID_ARG, "ttt_op_gemm: bad dtype");
  if (s.a_mn && !s.b_mn) return set_error(TTT_ERR_UNSUPPORTED, "ttt_op_gemm: (a_mn, b_mn) = (1, 0) not built");
  TcGemm g;
  int rc = tc_gemm_prepare(&g, s, epilogue, e, bn_hint);
  if (rc) return rc;
  int* err = op_err_word();
  if (!err) return set_error(TTT_ERR_CUDA, "ttt_op_gemm: no device error word");
  return tc_gemm_launch(g, st, err);
}

extern "C" int ttt_op_gemm_split(int32_t a_mn, int32_t b_mn, int64_t M, int64_t N, int64_t K, const void* A,
                                 int64_t lda, const void* B, int64_t ldb, int32_t epilogue,
                                 const ttt_epilogue_args* args, int32_t bn_hint, int32_t ksplit, float* workspace,
                                 void* stream) {
  if (!A || !B || !args || M < 1 || N < 1 || K < 1) return set_error(TTT_ERR_INVALID_ARG, "ttt_op_gemm_split: bad argument");
  if (a_mn && !b_mn) return set_error(TTT_ERR_UNSUPPORTED, "ttt_op_gemm_split: (a_mn, b_mn) = (1, 0) not built");
  GemmShape s;
  s.a_mn = a_mn ? 1 : 0;
  s.b_mn = b_mn ? 1 : 0;
  s.a = a_mn ? MatView{A, K, M, lda} : MatView{A, M, K, lda};
  s.b = b_mn ? MatView{B, K, N, ldb} : MatView{B, N, K, ldb};
  TcGemm g;
  int rc = tc_gemm_prepare(&g, s, epilogue, to_epi(args), bn_hint);
  if (rc) return rc;
  rc = tc_gemm_set_split(&g, ksplit, workspace);
  if (rc) return rc;
  int* err = op_err_word();
  if (!err) return set_error(TTT_ERR_CUDA, "ttt_op_gemm_split: no device error word");
  return tc_gemm_launch(g, reinterpret_cast<cudaStream_t>(stream), err);
}

extern "C" int ttt_op_gemm_dual(int32_t a_mn, int32_t b_mn, int64_t M, int64_t N, int64_t K, const void* A,
                                int64_t lda, const void* B, int64_t ldb, int64_t K2, const void* A2, int64_t lda2,
                                const void* B2, int64_t ldb2, int64_t n_ext, int32_t epilogue,
                                const ttt_epilogue_args* args, int32_t bn_hint, int32_t ksplit, float* workspace,
                                void* stream) {
  if (!A || !B || !A2 || !B2 || !args || M < 1 || N < 1 || K < 1 || K2 < 1 || n_ext < 0 || n_ext >= N)
    return set_error(TTT_ERR_INVALID_ARG, "ttt_op_gemm_dual: bad argument");
  if (a_mn && !b_mn) return set_error(TTT_ERR_UNSUPPORTED, "ttt_op_gemm_dual: (a_mn, b_mn) = (1, 0) not built");
  GemmShape s;
  s.a_mn = a_mn ? 1 : 0;
  s.b_mn = b_mn ? 1 : 0;
  s.a = a_mn ? MatView{A, K, M, lda} : MatView{A, M, K, lda};
  s.b = b_mn ? MatView{B, K, N, ldb} : MatView{B, N, K, ldb};
  const MatView a2 = a_mn ? MatView{A2, K2, M, lda2} : MatView{A2, M, K2, lda2};
  const MatView b2 = b_mn ? MatView{B2, K2, N - n_ext, ldb2} : MatView{B2, N - n_ext, K2, ldb2};
  TcGemm g;
  int rc = tc_gemm_prepare(&g, s, epilogue, to_epi(args), bn_hint);
  if (rc) return rc;
  rc = tc_gemm_set_ext(&g, a2, b2, n_ext);
  if (rc) return rc;
  rc = tc_gemm_set_split(&g, ksplit, workspace);
  if (rc) return rc;
  int* err = op_err_word();
  if (!err) return set_error(TTT_ERR_CUDA, "ttt_op_gemm_dual: no device error word");
  return tc_gemm_launch(g, reinterpret_cast<cudaStream_t>(stream), err);
}

extern "C" int64_t ttt_op_gemm_plan(int64_t M, int64_t N, int64_t K, int32_t epilogue, int32_t* bn_out) {
  int bn = 0;
  const int64_t S = (M < 1 || N < 1 || K < 1) ? 1 : tc_split_plan(M, N, K, epilogue, &bn);
  if (bn_out) *bn_out = bn;
  return S;
}

extern "C" int64_t ttt_op_gemm_ce_tiles(int32_t dtype, int64_t M, int64_t N, int32_t bn_hint) {
  if (dtype == TTT_F32) return (N + 127) / 128;
  return tc_ce_tiles(N, tc_pick_bn(M, N, bn_hint));
}

extern "C" int ttt_op_sync(void* stream) {
  TTT_CUDA_TRY(cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)));
  int* err = op_err_word();
  if (!err) return set_error(TTT_ERR_CUDA, "ttt_op_sync: no device error word");
  int h = 0;
  TTT_CUDA_TRY(cudaMemcpy(&h, err, sizeof(int), cudaMemcpyDeviceToHost));
  if (h) {
    int zero = 0;
    TTT_CUDA_TRY(cudaMemcpy(err, &zero, sizeof(int), cudaMemcpyHostToDevice));
    if (h & DEV_ERR_TIMEOUT) return set_error(TTT_ERR_TIMEOUT, "a kernel's bounded wait timed out");
    if (h & DEV_ERR_BAD_TOKEN) return set_error(TTT_ERR_INVALID_ARG, "a token or target id outside its range");
    return set_error(TTT_ERR_CUDA, "kernel error word " + std::to_string(h));
  }
  return TTT_OK;
}

namespace ttt {

SwaArgs op_swa_args(int32_t H, int32_t HD, int64_t n, int64_t p0, int32_t window, const void* q, int64_t ldq,
                    const void* k, const void* v, int64_t ring, void* o, int64_t ldo, const float* lse) {
  SwaArgs a;
  a.heads = H;
  a.head_dim = HD;
  a.n = n;
  a.p0 = p0;
  a.window = window;
  a.scale = 1.f / sqrtf((float)HD);
  a.q = q;
  a.ldq = ldq;
  a.k = k;
  a.v = v;
  a.ldkv = (int64_t)H * HD;
  a.ring = ring;
  a.o = o;
  a.ldo = ldo;
  a.lse = const_cast<float*>(lse);
  a.ld_lse = n;
  return a;
}

int op_swa_backward_run(const SwaArgs& a, int32_t dtype, int32_t flags, cudaStream_t st) {
  if (dtype == TTT_BF16 && !(flags & TTT_SWA_FORCE_SIMT) && swa_tc_supported(a.head_dim) && a.ring % 128 == 0 &&
      a.ldq == a.lddo) {
    SwaTcBwdPlan plan;
    int rc = swa_tc_bwd_prepare(&plan, a.heads, a.head_dim, a.q, a.dout, a.n, a.ldq, a.k, a.v, a.ring, a.ldkv);
    if (rc) return rc;
    int* err = op_err_word();
    if (!err) return set_error(TTT_ERR_CUDA, "ttt_op_swa_backward: no device error word");
    std::function<int()> dkdv;
    if (swa_tc_dkdv_supported(a) && a.lddkv == a.ldq) dkdv = [&] { return swa_tc_backward_dkdv(plan, a, st, err); };
    return swa_backward_with_dq(a, true, st, [&] { return swa_tc_backward_dq(plan, a, st, err); }, dkdv);
  }
  return swa_backward(a, dtype == TTT_BF16, st);
}

}  // namespace ttt

extern "C" int ttt_op_swa_forward(int32_t dtype, int32_t n_heads, int32_t head_dim, int64_t n_q, int64_t q_pos0,
                                  int32_t window, const void* q, int64_t ldq, const void* k_ring, const void* v_ring,
                                  int64_t ring_slots, void* o, int64_t ldo, float* lse, float q_norm_max,
                                  float k_norm_max, int32_t flags, void* stream) {
  if (!q || !k_ring || !v_ring || !o || !lse || n_q < 1 || q_pos0 < 0 || window < 1 || ring_slots < 1 ||
      n_heads < 1 || (dtype != TTT_F32 && dtype != TTT_BF16))
    return set_error(TTT_ERR_INVALID_ARG, "ttt_op_swa_forward: bad argument");
  SwaArgs a = op_swa_args(n_heads, head_dim, n_q, q_pos0, window, q, ldq, k_ring, v_ring, ring_slots, o, ldo, lse);
  a.q_norm_max = std::isfinite(q_norm_max) ? q_norm_max : 0.f;
  a.k_norm_max = std::isfinite(k_norm_max) ? k_norm_max : 0.f;
  a.exp_poly = ((flags >> 4) & 15) - 1;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (dtype == TTT_BF16 && !(flags & TTT_SWA_FORCE_SIMT) && swa_tc_supported(head_dim) && ring_slots % 128 == 0) {
    SwaTcPlan plan;
    int rc = swa_tc_prepare(&plan, n_heads, head_dim, q, n_q, ldq, k_ring, v_ring, ring_slots,
                            (int64_t)n_heads * head_dim);
    if (rc) return rc;
    int* err = op_err_word();
    if (!err) return set_error(TTT_ERR_CUDA, "ttt_op_swa_forward: no device error word");
    return swa_tc_forward(plan, a, st, err);
  }
  return swa_forward(a, dtype == TTT_BF16, st);
}

extern "C" int ttt_op_swa_backward(int32_t dtype, int32_t n_heads, int32_t head_dim, int64_t n_q, int64_t q_pos0,
                                   int32_t window, const void* q, int64_t ldq, const void* k_ring, const void* v_ring,
                                   int64_t ring_slots, const void* o, int64_t ldo, const float* lse, const void* dout,
                                   int64_t lddo, void* dq, int64_t lddq, void* dk, void* dv, int64_t lddkv,
                                   float* D_scratch, int32_t flags, void* stream) {
  if (!q || !k_ring || !v_ring || !o || !lse || !dout || !dq || !dk || !dv || !D_scratch || n_q < 1 || q_pos0 < 0 ||
      window < 1 || ring_slots < 1 || n_heads < 1 || (dtype != TTT_F32 && dtype != TTT_BF16))
    return set_error(TTT_ERR_INVALID_ARG, "ttt_op_swa_backward: bad argument");
  SwaArgs a = op_swa_args(n_heads, head_dim, n_q, q_pos0, window, q, ldq, k_ring, v_ring, ring_slots,
                          const_cast<void*>(o), ldo, lse);
  a.dout = dout;
  a.lddo = lddo;
  a.dq = dq;
  a.lddq = lddq;
  a.dk = dk;
  a.dv = dv;
  a.lddkv = lddkv;
  a.D = D_scratch;
  return op_swa_backward_run(a, dtype, flags, reinterpret_cast<cudaStream_t>(stream));
}

namespace ttt {
namespace {
__global__ void watchdog_selftest_kernel(int* err) {
  __shared__ uint64_t bar;
  ptx::mbar_init(&bar, 1);
  ptx::fence_mbar_init();
  ptx::mbar_wait(&bar, 0, err);  // nobody arrives: must give up and set the error word
}
}  // namespace
}  // namespace ttt

extern "C" int ttt_op_watchdog_selftest(void* stream) {
  int* err = op_err_word();
  if (!err) return set_error(TTT_ERR_CUDA, "ttt_op_watchdog_selftest: no device error word");
  watchdog_selftest_kernel<<<1, 1, 0, reinterpret_cast<cudaStream_t>(stream)>>>(err);
  TTT_CUDA_TRY(cudaGetLastError());
  return TTT_OK;
}

extern "C" int ttt_op_rmsnorm(int64_t n, int32_t d, const float* x, int64_t ldx, const float* g, float eps, void* y,
                              int64_t ldy, float* rstd, void* stream) {
  if (!x || !g || !y || !rstd || n < 1 || d < 1) return set_error(TTT_ERR_INVALID_ARG, "ttt_op_rmsnorm: bad argument");
  return rmsnorm_fwd<bf16>(x, ldx, g, eps, n, d, reinterpret_cast<bf16*>(y), ldy, rstd,
                           reinterpret_cast<cudaStream_t>(stream));
}

extern "C" int ttt_op_qknorm_rope(int64_t n, int64_t p0, int32_t n_heads, int32_t head_dim, float eps, float theta,
                                  const void* qkv, int64_t ldqkv, const float* gq, const float* gk, void* qout,
                                  int64_t ldq, void* kring, void* vring, int64_t R, float* rq, float* rk, float* tab,
                                  void* stream) {
  if (!qkv || !gq || !gk || !qout || !kring || !vring || !rq || !rk || !tab || n < 1 || p0 < 0 || R < 1 ||
      n_heads < 1 || head_dim < 2)
    return set_error(TTT_ERR_INVALID_ARG, "ttt_op_qknorm_rope: bad argument");
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  float2* t2 = reinterpret_cast<float2*>(tab);
  int rc = rope_table(t2, p0, n, head_dim, (double)theta, st);
  if (rc) return rc;
  return qknorm_rope_fwd<bf16>(reinterpret_cast<const bf16*>(qkv), ldqkv, gq, gk, n, p0, n_heads, head_dim, eps, t2,
                               p0, reinterpret_cast<bf16*>(qout), ldq, reinterpret_cast<bf16*>(kring),
                               reinterpret_cast<bf16*>(vring), (int64_t)n_heads * head_dim, R, rq, rk, st);
}

extern "C" int ttt_op_swiglu_bwd(int64_t n, int64_t nfeat, const void* da, int64_t ldda, const void* gu, int64_t ldgu,
                                 void* dgu, int64_t lddgu, void* stream) {
  if (!da || !gu || !dgu || n < 1 || nfeat < 1 || nfeat % 64)
    return set_error(TTT_ERR_INVALID_ARG, "ttt_op_swiglu_bwd: bad argument");
  return swiglu_bwd<bf16>(reinterpret_cast<const bf16*>(da), ldda, reinterpret_cast<const bf16*>(gu), ldgu, n, nfeat,
                          reinterpret_cast<bf16*>(dgu), lddgu, reinterpret_cast<cudaStream_t>(stream));
}

extern "C" int ttt_op_gemv(int32_t epilogue, int64_t n, int64_t k, const void* w, int64_t ldw, const void* x,
                           void* out, const float* res, void* raw, float* lse_out, float* part, void* stream) {
  if (!w || !x || !out || n < 1 || k < 1 || epilogue < 0 || epilogue > 3 || (epilogue == GEMV_ADD_F32 && !res) ||
      (epilogue == GEMV_ARGMAX && !part))
    return set_error(TTT_ERR_INVALID_ARG, "ttt_op_gemv: bad argument");
  GemvArgs<bf16> g;
  g.w = reinterpret_cast<const bf16*>(w);
  g.ldw = ldw;
  g.n = n;
  g.k = k;
  g.x = reinterpret_cast<const bf16*>(x);
  g.out = epilogue == GEMV_ARGMAX ? static_cast<void*>(part) : out;
  g.res = res;
  g.raw = reinterpret_cast<bf16*>(raw);
  g.part = part;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  int rc = gemv<bf16>(g, epilogue, st);
  if (rc || epilogue != GEMV_ARGMAX) return rc;
  return argmax_finalize(part, gemv_parts(n), reinterpret_cast<int32_t*>(out), nullptr, lse_out, nullptr, st);
}

extern "C" int ttt_op_attn_decode(int32_t n_heads, int32_t head_dim, int64_t p, int32_t window, const void* q,
                                  const void* kring, const void* vring, int64_t R, void* o, float* lse, float* ws,
                                  void* stream) {
  if (!q || !kring || !vring || !o || !ws || n_heads < 1 || p < 0 || window < 1 || R < window)
    return set_error(TTT_ERR_INVALID_ARG, "ttt_op_attn_decode: bad argument");
  return attn_decode<bf16>(reinterpret_cast<const bf16*>(q), reinterpret_cast<const bf16*>(kring),
                           reinterpret_cast<const bf16*>(vring), (int64_t)n_heads * head_dim, R, n_heads, head_dim, p,
                           window, 1.f / sqrtf((float)head_dim), reinterpret_cast<bf16*>(o), lse, 1, ws,
                           reinterpret_cast<cudaStream_t>(stream));
}
