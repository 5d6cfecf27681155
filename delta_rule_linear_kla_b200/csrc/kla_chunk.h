// Host-side interface of the chunkwise tensor-core prefill.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace kla {

// Bytes of one chunk's UT factors in the workspace: T' = T diag(beta) and
// T'' = T diag(beta e^G), two 64x64 bf16 tiles stored transposed, exactly as
// the chain kernel wants them in shared memory (128-byte swizzled rows).
constexpr size_t kUtTileBytes = 2 * 64 * 64 * 2;

// Device scratch the chunk path needs for these sizes (bytes, 0 if none):
// the UT factors of every chunk and, when the state chain is cut into
// segments, the segment states.
size_t chunk_workspace_bytes(int B, int T, int H, int dk, int dv, int dtype);
// The UT factors alone (the least a workspace must hold).
size_t chunk_ut_workspace_bytes(int B, int T, int H, int dk, int dv, int dtype);
// Bytes of a workspace of ws_bytes that the chunk path touches: all of
// chunk_workspace_bytes when it fits (segmented chain), else the UT factors.
size_t chunk_workspace_used(int B, int T, int H, int dk, int dv, int dtype, size_t ws_bytes);
// Segments the state chain runs in for a workspace of ws_bytes (1 = uncut).
int chunk_chain_segments(int B, int T, int H, int dk, int dv, size_t ws_bytes);
// Whether the bf16 prefill of this shape runs as one launch (UT lanes and
// state CTAs together) with a workspace of ws_bytes, on a B200's 148 SMs.
bool chunk_single_launch(int B, int T, int H, int dk, int dv, size_t ws_bytes);

// bf16 I/O chunkwise prefill (UT kernel, then the chain kernel).  Returns
// cudaErrorNotSupported for shapes it does not handle; `err` is this
// device's error word.
cudaError_t launch_chunk_tc(const void* q, const void* k, const void* v,
                            const float* g, const float* eta, float eps,
                            const float* h0, void* o, float* hT, int B, int T,
                            int H, int dk, int dv, void* workspace, size_t ws_bytes,
                            unsigned int* err, cudaStream_t st, float* hs = nullptr);

// The two stages of launch_chunk_tc on their own: the UT transform of every
// chunk into the workspace, then the chain kernel that reads it.
// ratio_max (device float, nullable): run the UT kernel's debug bound check
// and record the largest bound ratio there.
cudaError_t launch_chunk_ut(const void* k, const float* g, const float* eta, float eps,
                            int B, int T, int H, int dk, void* workspace, unsigned int* err,
                            cudaStream_t st, float* ratio_max = nullptr);
// The chain is cut into segments (a sequence-parallel schedule for few heads
// and long sequences) when ws_bytes also covers the segment states.
cudaError_t launch_chunk_chain(const void* q, const void* k, const void* v, const float* g,
                               const float* h0, void* o, float* hT, int B, int T, int H,
                               int dk, int dv, void* workspace, size_t ws_bytes,
                               unsigned int* err, cudaStream_t st,
                               float* hs = nullptr);

// Per-chunk factors of the per-channel-gate (KDA form) path, one tile per
// chunk in chunk-major order: byte offsets of T'^T, P, W, Q o e^G,
// K o e^{G_last - G} (64 x dk bf16 each in 64-column swizzled panels; the
// first two 64 x 64) and e^{G_last} (dk fp32), and the tile's total size.
struct KdaTileOffsets {
  uint32_t tp, p, w, q, k, d, total;
};
__host__ __device__ constexpr KdaTileOffsets kda_tile_offsets(int dk) {
  return KdaTileOffsets{0u,
                        8192u,
                        16384u,
                        16384u + (uint32_t)(dk / 64) * 8192u,
                        16384u + 2u * (uint32_t)(dk / 64) * 8192u,
                        16384u + 3u * (uint32_t)(dk / 64) * 8192u,
                        16384u + 3u * (uint32_t)(dk / 64) * 8192u + 1024u};
}

// The per-channel-gate chunk prefill: per-chunk factors (CUDA cores, fp32,
// every chunk of every head in parallel), then the chain kernel in its KDA
// mode.  g is [B][T][H][dk]; eps < 0 selects beta given (in eta).
cudaError_t launch_kda_prep(const void* q, const void* k, const float* g, const float* eta,
                            float eps, int B, int T, int H, int dk, void* ws, cudaStream_t st);
cudaError_t launch_kda_chunk(const void* q, const void* k, const void* v, const float* g,
                             const float* eta, float eps, const float* h0, void* o, float* hT,
                             int B, int T, int H, int dk, int dv, void* workspace,
                             size_t ws_bytes, unsigned int* err, cudaStream_t st);
size_t kda_chunk_workspace_bytes(int B, int T, int H, int dk, int dv, int dtype);

// UT kernel alone: T', T'' of every chunk into `ws` (chunk-major order
// ((b * H + h) * nchunks + n)).  `tm_k` maps k as [B][T][H][dk] bf16 with
// 64 x 64 boxes and 128-byte swizzle.
cudaError_t launch_ut(const CUtensorMap& tm_k, const float* g, const float* eta, float eps,
                      uint8_t* ws, int B, int T, int H, int dk, unsigned int* err,
                      cudaStream_t st, float* ratio_max = nullptr);

// The same kernel for the chunks n < n_first of every head only (chunk index
// major): the factors the first pass of a cut chain reads.
cudaError_t launch_ut_first(const CUtensorMap& tm_k, const float* g, const float* eta,
                            float eps, uint8_t* ws, int B, int T, int H, int dk, int n_first,
                            unsigned int* err, cudaStream_t st);

}  // namespace kla
