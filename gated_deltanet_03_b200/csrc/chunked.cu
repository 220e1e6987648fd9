// Placeholder for the tensor-core chunked prefill; the recurrent kernel serves until it lands.
#include "common.cuh"
#include "kernels.h"

namespace gdn {
cudaError_t launch_chunked(const ChunkedArgs &, cudaStream_t) { return cudaErrorNotSupported; }
}  // namespace gdn
