// prefill.cu -- placeholder until the tensor-core prefill lands.
#include "common.cuh"
#include "internal.h"

namespace gdn {
cudaError_t launch_prefill(const PrefillArgs&, cudaStream_t) { return cudaErrorNotSupported; }
}  // namespace gdn
