// backward.cu -- placeholder until the backward pass lands.
#include "common.cuh"
#include "internal.h"

namespace gdn {
size_t backward_workspace_bytes(int B, int T, int H, int dk, int dv) {
    const size_t chunks = (size_t)(T + 63) / 64;
    return chunks * (size_t)B * H * dk * dv * sizeof(float);
}
cudaError_t launch_backward(const BackwardArgs&, cudaStream_t) { return cudaErrorNotSupported; }
}  // namespace gdn
