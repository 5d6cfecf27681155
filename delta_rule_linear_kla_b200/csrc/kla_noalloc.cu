// kla_chunk_fwd_noalloc: the bf16 chunkwise prefill for callers that cannot
// provide device scratch memory.
//
// kla_chunk_fwd needs a caller-owned workspace (the per-chunk UT factors).
// Some callers cannot produce one on demand: their device memory is owned by
// another allocator (an inference server's pre-reserved pool, for example),
// or their integration contract forbids allocating after start-up, where a
// cudaMalloc could stall the device or fail under memory pressure.  For them
// this entry point uses a fixed scratch array that lives in this library's
// device image instead.  Its cost: every GPU that loads the library holds
// KLA_NOALLOC_SCRATCH_BYTES (16 MiB) for the rest of the process, and one
// bf16 call handles at most KLA_NOALLOC_MAX_CHUNKS chunks of 64 tokens in
// total (B * H * ceil(T / 64)); fp32 calls use no scratch and have no limit.
// The library's uses of a workspace are covered: the per-chunk factors
// always fit, the segment states of a cut state chain only when the chunk
// count leaves room.
//
// Nothing here allocates: no cudaMalloc, cudaFree, or allocating library call.
// All calls share the single array and it keeps whatever the last call left
// there.  That is safe for sequential calls, because the UT kernel writes
// every tile of a call before the chain kernel of the same call reads it, so
// nothing has to start out zeroed.  Calls whose kernels overlap on the GPU
// (two streams, or two host threads) race on the array and must not be
// issued.
#include <cuda_runtime.h>

#include "../../include/kla.h"

namespace {

// The scratch itself.  In host code this name is only a stand-in for the
// symbol: its device address is obtained with cudaGetSymbolAddress below and
// passed on as an ordinary pointer.
static __device__ __align__(256) unsigned char g_noalloc_scratch[KLA_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
void* g_scratch_addr[kMaxDevices];

// Device address of the scratch array on the current device, looked up once
// per device (with that device current) on the first call made there.
void* scratch_address() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
      cudaGetLastError();  // leave no sticky error behind for the caller
      return nullptr;
    }
    g_scratch_addr[dev] = p;
  }
  return g_scratch_addr[dev];
}

}  // namespace

extern "C" KLA_API kla_status kla_chunk_fwd_noalloc(const void* q, const void* k, const void* v,
                                                    const float* g, const float* eta, float eps,
                                                    const float* h0, void* o, float* hT, int B,
                                                    int T, int H, int dk, int dv, int dtype,
                                                    void* stream) {
  // Size limit first, before anything touches the GPU.
  if (B < 1 || H < 1 || T < 0) return KLA_ERR_INVALID_ARG;
  // Only the bf16 chunk path uses scratch; the fp32 (token-serial) path needs
  // none, so the chunk limit does not apply to it.  64-bit arithmetic: the
  // count cannot wrap for any int-sized B, H, T.
  const long long chunks =
      (long long)B * H * (((long long)T + KLA_CHUNK - 1) / KLA_CHUNK);
  // (KLA_NOALLOC_MAX_CHUNKS tiles of UT factors fill the scratch exactly;
  // kla_chunk_fwd cuts the state chain into segments only if their states
  // fit in what is left)
  if (dtype == KLA_BF16 && chunks > KLA_NOALLOC_MAX_CHUNKS) return KLA_ERR_UNSUPPORTED;
  void* scratch = scratch_address();
  if (!scratch) return KLA_ERR_CUDA;
  return kla_chunk_fwd(q, k, v, g, eta, eps, h0, o, hT, B, T, H, dk, dv, KLA_CHUNK, dtype,
                       scratch, (size_t)KLA_NOALLOC_SCRATCH_BYTES, stream);
}
