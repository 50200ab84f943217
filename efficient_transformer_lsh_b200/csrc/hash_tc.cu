// Tensor-core hashing kernel (placeholder until the tcgen05 kernel lands).
#include "internal.h"

namespace lsh {
cudaError_t launch_hash_tc(const lsh_problem&, const void*, const void*, int32_t*, int*,
                           cudaStream_t) {
  return cudaErrorNotSupported;
}
}  // namespace lsh
