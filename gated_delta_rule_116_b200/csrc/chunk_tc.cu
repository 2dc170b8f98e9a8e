// chunk_tc.cu -- tensor-core (tcgen05/TMEM) engine of the chunked KDA prefill.
#include "kda_internal.cuh"

namespace kda {

bool chunk_tc_supported(int, int, int, int) { return false; }

size_t chunk_tc_workspace_bytes(int, int, int) { return 0; }

cudaError_t launch_chunk_tc(const ChunkArgs &, cudaStream_t) { return cudaErrorNotSupported; }

}  // namespace kda
