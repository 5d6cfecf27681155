// UT transform of every chunk as a kernel of its own (kla_chunk_ut_transform,
// and the first of the two launches of the prefill where the state kernel is
// not run in the same launch): each CTA of 128 threads is one UT lane of
// kla_ut_body.cuh, persistent over pairs of chunks, several CTAs per SM.
#include "kla_ut_body.cuh"

namespace kla {
namespace {

template <int DK, bool CHECK>
__global__ void __launch_bounds__(utb::NT, utb::ctas_per_sm<DK>())
ut_kernel(const __grid_constant__ CUtensorMap tm_k, const float* __restrict__ g,
          const float* __restrict__ eta, float eps, uint8_t* __restrict__ ws, int T, int H,
          int nchunks, int BH, int total_chunks, bool nmajor, unsigned int* err,
          float* ratio_max) {
  extern __shared__ uint8_t smem_raw[];
  auto& s = *reinterpret_cast<utb::UtSmem<DK>*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  utb::ut_run<DK, CHECK>(&tm_k, g, eta, eps, ws, T, H, nchunks, BH, 0, total_chunks, nmajor,
                         err, ratio_max, nullptr, s, threadIdx.x, 1, 2, blockIdx.x, gridDim.x,
                         true);
}

template <int DK, bool CHECK>
cudaError_t launch_ut_dk(const CUtensorMap& tm_k, const float* g, const float* eta, float eps,
                         uint8_t* ws, int B, int T, int H, int n_first, unsigned int* err,
                         float* ratio_max, cudaStream_t st) {
  // n_first < 0: every chunk, head by head; else the chunks n < n_first of
  // every head, chunk index major
  const int nchunks = (T + utb::C - 1) / utb::C;
  const int total = B * H * (n_first < 0 ? nchunks : n_first);
  if (total == 0) return cudaSuccess;
  const size_t smem = sizeof(utb::UtSmem<DK>) + 1024;
  static bool attr_set[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(ut_kernel<DK, CHECK>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  // persistent grid: ctas_per_sm CTAs per SM, each taking every gridDim-th
  // pair of chunks
  static int sm_count[64] = {};
  if (!sm_count[dev]) {
    cudaError_t e = cudaDeviceGetAttribute(&sm_count[dev], cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
  }
  const int npairs = (total + 1) / 2;
  const int cap = utb::ctas_per_sm<DK>() * sm_count[dev];
  const int grid = npairs < cap ? npairs : cap;
  ut_kernel<DK, CHECK><<<grid, utb::NT, smem, st>>>(tm_k, g, eta, eps, ws, T, H, nchunks, B * H,
                                                    total, n_first >= 0, err, ratio_max);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_ut(const CUtensorMap& tm_k, const float* g, const float* eta, float eps,
                      uint8_t* ws, int B, int T, int H, int dk, unsigned int* err,
                      cudaStream_t st, float* ratio_max) {
  if (ratio_max) {
    if (dk == 128)
      return launch_ut_dk<128, true>(tm_k, g, eta, eps, ws, B, T, H, -1, err, ratio_max, st);
    if (dk == 64)
      return launch_ut_dk<64, true>(tm_k, g, eta, eps, ws, B, T, H, -1, err, ratio_max, st);
    return cudaErrorNotSupported;
  }
  if (dk == 128) return launch_ut_dk<128, false>(tm_k, g, eta, eps, ws, B, T, H, -1, err, nullptr, st);
  if (dk == 64) return launch_ut_dk<64, false>(tm_k, g, eta, eps, ws, B, T, H, -1, err, nullptr, st);
  return cudaErrorNotSupported;
}

cudaError_t launch_ut_first(const CUtensorMap& tm_k, const float* g, const float* eta,
                            float eps, uint8_t* ws, int B, int T, int H, int dk, int n_first,
                            unsigned int* err, cudaStream_t st) {
  if (n_first < 0 || n_first > (T + utb::C - 1) / utb::C) return cudaErrorInvalidValue;
  if (dk == 128)
    return launch_ut_dk<128, false>(tm_k, g, eta, eps, ws, B, T, H, n_first, err, nullptr, st);
  if (dk == 64)
    return launch_ut_dk<64, false>(tm_k, g, eta, eps, ws, B, T, H, n_first, err, nullptr, st);
  return cudaErrorNotSupported;
}

}  // namespace kla
