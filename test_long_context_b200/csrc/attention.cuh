// Sliding-window attention launch interface.
#pragma once
#include <functional>

#include "common.cuh"

namespace ttt {

// All row pitches in elements.  q/o/dout/dq: [n, heads*head_dim] chunk-local
// rows (row i is absolute position p0 + i).  k/v: ring [ring, heads*head_dim],
// slot = position % ring.  lse, D: [heads, ld_lse] fp32.  dk/dv: [n, ...]
// gradients of the keys/values at positions p0 .. p0+n-1 (this chunk's own).
struct SwaArgs {
  int heads = 0, head_dim = 0;
  int64_t n = 0, p0 = 0;
  int64_t window = 1;
  float scale = 1.f;
  const void* q = nullptr;
  int64_t ldq = 0;
  const void* k = nullptr;
  const void* v = nullptr;
  int64_t ldkv = 0, ring = 1;
  // Upper bounds on the Euclidean norm of every query row and key row of a
  // head (0 = unknown): with both known and scale log2(e) q_norm_max
  // k_norm_max <= 48, the tensor-core forward shifts each row's softmax by
  // the Cauchy-Schwarz bound of its scores instead of a running maximum.
  float q_norm_max = 0.f, k_norm_max = 0.f;
  // Fixed-shift forward: how many of every 8 groups of 8 keys take 2^x from
  // an FMA-pipe polynomial instead of the MUFU unit (0, 2, 4); -1 = default.
  int exp_poly = -1;
  void* o = nullptr;
  int64_t ldo = 0;
  float* lse = nullptr;
  int64_t ld_lse = 0;
  // backward
  const void* dout = nullptr;
  int64_t lddo = 0;
  void* dq = nullptr;
  int64_t lddq = 0;
  void* dk = nullptr;
  void* dv = nullptr;
  int64_t lddkv = 0;
  float* D = nullptr;
};

int swa_forward(const SwaArgs& a, bool use_bf16, cudaStream_t s);
// Needs a.o, a.lse from the forward; writes D, dq, dk, dv.
int swa_backward(const SwaArgs& a, bool use_bf16, cudaStream_t s);
// Same, with the dq part replaced by `dq` (launched after D is written) and,
// when `dkdv` is given, the dk/dv part replaced by it.
int swa_backward_with_dq(const SwaArgs& a, bool use_bf16, cudaStream_t s, const std::function<int()>& dq,
                         const std::function<int()>& dkdv = {});

}  // namespace ttt
