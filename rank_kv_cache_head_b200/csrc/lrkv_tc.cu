// tcgen05 split kernel (placeholder until the tensor-core path lands).
#include "lrkv_internal.h"

namespace lrkv {

bool tc_supported(const lrkv_dims&, int* smem_bytes) {
  *smem_bytes = 0;
  return false;
}

cudaError_t launch_split_tc(const SplitArgs&, const Plan&, cudaStream_t) {
  return cudaErrorNotSupported;
}

}  // namespace lrkv
