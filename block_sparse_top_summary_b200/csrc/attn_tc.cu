// Stage 2 on the tensor cores (placeholder until the tcgen05 kernel lands).
#include "kernels.h"

namespace ssa {

bool attn_tc_supported(ssa_dtype, int, int, int, int) { return false; }

cudaError_t launch_attn_tc(const void*, const void*, const void*, const int32_t*, const int32_t*,
                           int, int, int, int, int, int, float, void*, float*, cudaStream_t) {
  return cudaErrorNotSupported;
}

int read_and_reset_attn_tc_error() { return 0; }

}  // namespace ssa
