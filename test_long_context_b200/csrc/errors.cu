// Error-message bookkeeping shared by every entry point.
#include <string>

#include "common.cuh"

namespace ttt {

static thread_local std::string g_last_error = "no error";

int set_error(int code, const std::string& msg) {
  g_last_error = msg;
  return code;
}

int set_cuda_error(cudaError_t e, const char* what, const char* file, int line) {
  g_last_error = std::string(what) + ": " + cudaGetErrorString(e) + " (" + file + ":" + std::to_string(line) + ")";
  return e == cudaErrorMemoryAllocation ? TTT_ERR_OOM : TTT_ERR_CUDA;
}

const char* last_error_message() { return g_last_error.c_str(); }

}  // namespace ttt
