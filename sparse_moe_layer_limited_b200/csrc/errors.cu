// Last-error text for the C ABI: the launchers record which call failed and
// CUDA's message, so a MOE_ERR_CUDA status can be explained by the caller.
#include <cstdio>

#include "internal.h"

namespace moe {
namespace {
thread_local char g_last_error[256] = "";
}

cudaError_t note_cuda(cudaError_t e, const char* where) {
  if (e != cudaSuccess)
    std::snprintf(g_last_error, sizeof(g_last_error), "%s: %s (%d)", where,
                  cudaGetErrorString(e), (int)e);
  return e;
}

void note_text(const char* what) { std::snprintf(g_last_error, sizeof(g_last_error), "%s", what); }

}  // namespace moe

extern "C" const char* moe_last_error(void) { return moe::g_last_error; }
