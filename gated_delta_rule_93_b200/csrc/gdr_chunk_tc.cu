// Tensor-core (tcgen05) chunked forward: not built yet; every shape goes to
// the CUDA-core kernel.
#include "gdr_internal.cuh"

namespace gdr {
bool chunk_tc_supports(const ChunkArgs &) { return false; }
cudaError_t launch_chunk_tc(const ChunkArgs &, cudaStream_t) { return cudaErrorNotSupported; }
}  // namespace gdr
