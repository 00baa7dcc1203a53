// E4M3 expert path: not built yet; the entry points report "unsupported".
#include "internal.h"

namespace moe {

int launch_ffn_tc_e4m3(const moe_shape&, const void*, const float*, const int32_t*, const void*,
                       const void*, const void*, const float*, const float*, void*, void*, void*,
                       cudaStream_t) {
  return MOE_ERR_UNSUPPORTED;
}

cudaError_t launch_quantize_weights(const moe_shape&, const void*, const void*, void*, float*,
                                    void*, float*, cudaStream_t) {
  return cudaErrorNotSupported;
}

}  // namespace moe
