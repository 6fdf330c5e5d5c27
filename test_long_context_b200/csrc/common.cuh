// Shared helpers of the CUDA library: status handling, bf16 conversion and
// the device-side error word that bounded waits report into.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <cstdio>
#include <string>

#include "../../include/ttt.h"

namespace ttt {

using bf16 = __nv_bfloat16;

// Device error word bits (written by kernels, read by ttt_sync).
enum : int {
  DEV_ERR_TIMEOUT = 1,      // a bounded wait gave up
  DEV_ERR_BAD_TOKEN = 2,    // a token id outside [0, vocab)
};

// Bounded waits give up after this many nanoseconds of %globaltimer.
constexpr unsigned long long kWaitLimitNs = 2000000000ull;
// ... or after this many polls of the barrier (each poll may suspend briefly).
constexpr uint32_t kWaitLimitIters = 1u << 26;
// Suspend hint of one poll of a bounded mbarrier wait (the thread resumes
// earlier when the phase completes).
constexpr uint32_t kWaitSleepNs = 20000;

__device__ __forceinline__ unsigned long long globaltimer_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(bf16 x) { return __bfloat162float(x); }
template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ bf16 from_f32<bf16>(float x) { return __float2bfloat16_rn(x); }

inline int cuda_status(cudaError_t e) { return e == cudaSuccess ? TTT_OK : TTT_ERR_CUDA; }

inline unsigned ceil_div(long long a, long long b) { return (unsigned)((a + b - 1) / b); }
__host__ __device__ __forceinline__ int64_t imin64(int64_t a, int64_t b) { return a < b ? a : b; }
__host__ __device__ __forceinline__ int64_t imax64(int64_t a, int64_t b) { return a > b ? a : b; }

}  // namespace ttt

#define TTT_CUDA_TRY(expr)                                 \
  do {                                                     \
    cudaError_t e_ = (expr);                               \
    if (e_ != cudaSuccess) return ::ttt::set_cuda_error(e_, #expr, __FILE__, __LINE__); \
  } while (0)

namespace ttt {
// Records the last library-wide error message (thread-local) and returns TTT_ERR_CUDA.
int set_cuda_error(cudaError_t e, const char* what, const char* file, int line);
int set_error(int code, const std::string& msg);
const char* last_error_message();
}  // namespace ttt
