// gdr_chunk_tc.cu -- tensor-core (tcgen05) chunked forward. Not yet enabled.
#include "gdr_internal.cuh"

namespace gdr {

bool chunk_tc_supported(int, int, int, int, int) { return false; }
size_t chunk_tc_workspace_bytes(int, int, int, int, int, int, int) { return 0; }
cudaError_t launch_chunk_tc(const ChunkProblem&, cudaStream_t) { return cudaErrorNotSupported; }
int chunk_tc_launches(int, int, int, int, int, int, int) { return 0; }

}  // namespace gdr
