// placeholder, replaced below
#include "common.cuh"
extern "C" const char* ttt_last_error(ttt_ctx*) { return ttt::last_error_message(); }
