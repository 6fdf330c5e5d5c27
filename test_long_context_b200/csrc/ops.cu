// Op-level entry points (include/ttt_ops.h): thin wrappers that validate the
// arguments and launch one kernel family each.
#include "../../include/ttt_ops.h"
#include "gemm.cuh"

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
    return set_error(TTT_ERR_CUDA, "kernel error word " + std::to_string(h));
  }
  return TTT_OK;
}
