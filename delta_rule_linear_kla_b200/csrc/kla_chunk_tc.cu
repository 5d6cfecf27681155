// Chunkwise tensor-core prefill (placeholder until the tcgen05 kernel lands).
#include "kla_common.cuh"
#include "kla_chunk.h"

namespace kla {

size_t chunk_workspace_bytes(int, int, int, int, int, int) { return 0; }

cudaError_t launch_chunk_tc(const void*, const void*, const void*, const float*,
                            const float*, float, const float*, void*, float*, int,
                            int, int, int, int, void*, unsigned int*, cudaStream_t) {
  return cudaErrorNotSupported;
}

}  // namespace kla
