// tcgen05/TMEM tensor-core forward of the EQ-Linear layer (placeholder until the
// kernel lands: reports every shape as unsupported so dispatch uses CUDA cores).
#include "eql_kernels.h"

namespace eql {

bool fwd_tc_supported(int, DType, int64_t, int, int) { return false; }

cudaError_t launch_fwd_tc(int, const void*, int64_t, int, int, const void*, const void*, void*,
                          int*, int, cudaStream_t) {
  return cudaErrorNotSupported;
}

}  // namespace eql
