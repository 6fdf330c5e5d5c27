// Tensor-core sliding-window attention forward (bf16): prepared tensor maps
// for one (query buffer, key ring, value ring) triple.
#pragma once
#include "attention.cuh"

namespace ttt {

struct SwaTcPlan {
  alignas(64) CUtensorMap q128;
  alignas(64) CUtensorMap qr;
  alignas(64) CUtensorMap k128;
  alignas(64) CUtensorMap kr;
  alignas(64) CUtensorMap k64;   // 64-row boxes: one CTA's half of a key tile (CTA-pair forward)
  alignas(64) CUtensorMap kr64;
  alignas(64) CUtensorMap v128;
  int head_dim = 0;
  int64_t ring = 0;
};

// Backward (dq over the band) on tensor cores: q and dout share a layout
// ([rows, heads*head_dim], pitch ld); the rings as in the forward.
struct SwaTcBwdPlan {
  alignas(64) CUtensorMap q128;
  alignas(64) CUtensorMap qr;
  alignas(64) CUtensorMap do128;
  alignas(64) CUtensorMap dor;
  alignas(64) CUtensorMap k64;
  alignas(64) CUtensorMap kr;
  alignas(64) CUtensorMap v64;
  alignas(64) CUtensorMap vr;
  alignas(64) CUtensorMap k128;  // 128-row boxes of the rings (dk/dv kernel)
  alignas(64) CUtensorMap kr128;
  alignas(64) CUtensorMap v128;
  alignas(64) CUtensorMap vr128;
  int head_dim = 0;
  int64_t ring = 0;
};

bool swa_tc_supported(int head_dim);
int swa_tc_bwd_prepare(SwaTcBwdPlan* p, int heads, int head_dim, const void* q, const void* dout, int64_t rows,
                       int64_t ld, const void* k, const void* v, int64_t ring, int64_t ldkv);
// Writes a.dq (bf16) from a.q, a.dout, the rings, a.lse and a.D (the row dot
// products dO . O, computed beforehand).
int swa_tc_backward_dq(const SwaTcBwdPlan& p, const SwaArgs& a, cudaStream_t s, int* err);
// dk, dv (bf16) for the chunk's own keys; needs a.p0 % 128 == 0 (the chunk's
// keys start a ring tile); reads a.lse and a.D.
bool swa_tc_dkdv_supported(const SwaArgs& a);
int swa_tc_backward_dkdv(const SwaTcBwdPlan& p, const SwaArgs& a, cudaStream_t s, int* err);
// q: [q_rows, heads*head_dim] (pitch ldq); k, v rings: [ring, heads*head_dim]
// (pitch ldkv); ring must be a multiple of 128.
int swa_tc_prepare(SwaTcPlan* p, int heads, int head_dim, const void* q, int64_t q_rows, int64_t ldq, const void* k,
                   const void* v, int64_t ring, int64_t ldkv);
int swa_tc_forward(const SwaTcPlan& p, const SwaArgs& a, cudaStream_t s, int* err);
// True when swa_tc_forward takes the fixed-shift kernel for these arguments.
bool swa_fixed_shift_ok(const SwaArgs& a);

// Shared by the op-level entry points (ops.cu, noalloc.cu): the forward
// arguments of one call (k/v ring pitch heads*head_dim, lse pitch n, scale
// 1/sqrt(head_dim)), and the backward dispatch - tensor cores for bf16 with a
// supported head_dim, a ring of whole 128-row tiles and q, dout sharing a
// pitch, unless flags has TTT_SWA_FORCE_SIMT; SIMT otherwise.  a.D must point
// to n*heads fp32 of work space.  Kernels report bounded-wait timeouts in the
// op-level error word (ttt_op_sync).
SwaArgs op_swa_args(int32_t H, int32_t HD, int64_t n, int64_t p0, int32_t window, const void* q, int64_t ldq,
                    const void* k, const void* v, int64_t ring, void* o, int64_t ldo, const float* lse);
int op_swa_backward_run(const SwaArgs& a, int32_t dtype, int32_t flags, cudaStream_t st);

}  // namespace ttt
