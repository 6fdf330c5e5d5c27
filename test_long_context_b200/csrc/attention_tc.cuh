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
  alignas(64) CUtensorMap v128;
  alignas(64) CUtensorMap vr;
  int head_dim = 0;
  int64_t ring = 0;
};

bool swa_tc_supported(int head_dim);
// q: [q_rows, heads*head_dim] (pitch ldq); k, v rings: [ring, heads*head_dim]
// (pitch ldkv); ring must be a multiple of 128.
int swa_tc_prepare(SwaTcPlan* p, int heads, int head_dim, const void* q, int64_t q_rows, int64_t ldq, const void* k,
                   const void* v, int64_t ring, int64_t ldkv);
int swa_tc_forward(const SwaTcPlan& p, const SwaArgs& a, cudaStream_t s, int* err);

}  // namespace ttt
