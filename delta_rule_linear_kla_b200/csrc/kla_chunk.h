// Host-side interface of the chunkwise tensor-core prefill (kla_chunk_tc.cu).
#pragma once
#include <cuda_runtime.h>
#include <stddef.h>

namespace kla {

// Device scratch the chunk kernel needs for these sizes (bytes, 0 if none).
size_t chunk_workspace_bytes(int B, int T, int H, int dk, int dv, int dtype);

// bf16 I/O chunkwise prefill.  Returns cudaErrorNotSupported for shapes the
// kernel does not handle; `err` is this device's error word.
cudaError_t launch_chunk_tc(const void* q, const void* k, const void* v,
                            const float* g, const float* eta, float eps,
                            const float* h0, void* o, float* hT, int B, int T,
                            int H, int dk, int dv, void* workspace,
                            unsigned int* err, cudaStream_t st);

}  // namespace kla
