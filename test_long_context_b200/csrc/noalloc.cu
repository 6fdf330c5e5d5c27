// Allocation-free variant of the sliding-window attention backward.
//
// ttt_op_swa_backward needs a work array D (one fp32 per query and head,
// the row dot products dO . O) that its caller allocates.  Some callers may
// not allocate device memory at all: their device memory is owned by
// another allocator (a framework's caching pool, or a fixed budget carved
// out at start-up), and cudaMalloc would both bypass that accounting and
// synchronise the whole device, stalling every other stream.  For them,
// ttt_op_swa_backward_noalloc takes the same inputs and outputs but keeps D
// in a fixed array that lives in this library (1 MiB per GPU that loads it,
// held until the process exits).
#include <mutex>
#include <unordered_map>

#include "../../include/ttt_ops.h"
#include "attention.cuh"
#include "attention_tc.cuh"

namespace ttt {
namespace {

// Largest n_heads * n_q the built-in work array holds (1 MiB of fp32).
constexpr int64_t kNoAllocMaxRows = int64_t(1) << 18;

// The work array.  Host code must not pass this name to a kernel: on the host
// it only stands for the symbol; the device address comes from
// cudaGetSymbolAddress below.
static __device__ __align__(256) float g_swa_bwd_work[kNoAllocMaxRows];

std::mutex g_mu;
std::unordered_map<int, float*> g_work_addr;  // device ordinal -> device address of g_swa_bwd_work

// Device address of the work array on the current device, looked up once per
// device (the first call on each device does this set-up).
int work_address(float** out) {
  int dev = 0;
  TTT_CUDA_TRY(cudaGetDevice(&dev));
  std::lock_guard<std::mutex> lock(g_mu);
  auto it = g_work_addr.find(dev);
  if (it == g_work_addr.end()) {
    float* p = nullptr;
    TTT_CUDA_TRY(cudaGetSymbolAddress(reinterpret_cast<void**>(&p), g_swa_bwd_work));
    it = g_work_addr.emplace(dev, p).first;
  }
  *out = it->second;
  return TTT_OK;
}

}  // namespace
}  // namespace ttt

using namespace ttt;

extern "C" int ttt_op_swa_backward_noalloc(int32_t dtype, int32_t n_heads, int32_t head_dim, int64_t n_q,
                                           int64_t q_pos0, int32_t window, const void* q, int64_t ldq,
                                           const void* k_ring, const void* v_ring, int64_t ring_slots, const void* o,
                                           int64_t ldo, const float* lse, const void* dout, int64_t lddo, void* dq,
                                           int64_t lddq, void* dk, void* dv, int64_t lddkv, void* stream) {
  if (!q || !k_ring || !v_ring || !o || !lse || !dout || !dq || !dk || !dv || n_q < 1 || q_pos0 < 0 || window < 1 ||
      ring_slots < 1 || n_heads < 1 || (dtype != TTT_F32 && dtype != TTT_BF16))
    return set_error(TTT_ERR_INVALID_ARG, "ttt_op_swa_backward_noalloc: bad argument");
  if ((int64_t)n_heads * n_q > kNoAllocMaxRows)
    return set_error(TTT_ERR_INVALID_ARG,
                     "ttt_op_swa_backward_noalloc: n_heads * n_q = " + std::to_string((int64_t)n_heads * n_q) +
                         " exceeds the built-in work array of " + std::to_string(kNoAllocMaxRows) +
                         " rows; use ttt_op_swa_backward with caller-provided scratch");
  float* work = nullptr;
  int rc = work_address(&work);
  if (rc) return rc;
  SwaArgs a = op_swa_args(n_heads, head_dim, n_q, q_pos0, window, q, ldq, k_ring, v_ring, ring_slots,
                          const_cast<void*>(o), ldo, lse);
  a.dout = dout;
  a.lddo = lddo;
  a.dq = dq;
  a.lddq = lddq;
  a.dk = dk;
  a.dv = dv;
  a.lddkv = lddkv;
  a.D = work;  // every entry is written before it is read: no clearing needed
  // the same kernels as ttt_op_swa_backward with default flags (tensor cores where it uses them)
  return op_swa_backward_run(a, dtype, 0, reinterpret_cast<cudaStream_t>(stream));
}
