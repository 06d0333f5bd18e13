// Importance on the tensor cores (bf16): placeholder until the tcgen05 path lands.
#include "fc_common.cuh"
#include "fc_kernels.h"

namespace fc {
bool importance_tc_supported(int d) {
  (void)d;
  return false;
}
cudaError_t launch_importance_tc(const void*, const void*, int, int, int, int, float, float*,
                                 void*, cudaStream_t) {
  return cudaErrorNotSupported;
}
}  // namespace fc
