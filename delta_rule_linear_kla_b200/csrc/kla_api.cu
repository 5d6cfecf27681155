// C ABI entry points of libkla.so: argument validation on the host, then a
// launch on the caller's stream.  No entry point allocates device memory or
// synchronises, except kla_check_device_error which is documented to.
#include <string.h>

#include "kla_common.cuh"
#include "kla_chunk.h"
#include "kla_sync.cuh"

namespace kla {

// Device error word (see kla_common.cuh); read back by kla_check_device_error.
__device__ unsigned int g_device_error = 0;

static const int kMaxDevices = 64;
static unsigned int* g_err_ptr[kMaxDevices];

// Address of this device's error word (looked up once per device).
unsigned int* device_error_ptr() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  if (!g_err_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_device_error) != cudaSuccess) return nullptr;
    g_err_ptr[dev] = (unsigned int*)p;
  }
  return g_err_ptr[dev];
}

static bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

struct Range {
  uintptr_t lo, hi;
};
static Range rng(const void* p, size_t bytes) {
  return Range{(uintptr_t)p, (uintptr_t)p + bytes};
}
static bool overlap(Range a, Range b) {
  return a.lo < b.hi && b.lo < a.hi && a.lo != a.hi && b.lo != b.hi;
}

static bool head_dims_ok(int dk, int dv) {
  return (dk == 64 && dv == 64) || (dk == 128 && dv == 128);
}

// Shared validation of the prefill entry points; gdim = log-gates per token
// (1, or dk for the per-channel gate).
static kla_status check_prefill(const void* q, const void* k, const void* v,
                                const float* g, const float* eta, float eps,
                                const float* h0, const void* o, const float* hT,
                                int B, int T, int H, int dk, int dv, int dtype,
                                int gdim = 1, bool o_optional = false) {
  if (B < 1 || H < 1 || T < 0 || dk < 1 || dv < 1) return KLA_ERR_INVALID_ARG;
  if (dtype != KLA_BF16 && dtype != KLA_FP32) return KLA_ERR_INVALID_ARG;
  if (!(eps >= 0.0f) || eps != eps) return KLA_ERR_INVALID_ARG;
  if ((long long)B * T * H * (dk > dv ? dk : dv) >= (1LL << 40)) return KLA_ERR_INVALID_ARG;
  if (T > 0 && (!q || !k || !v || !g || !eta || (!o && !o_optional))) return KLA_ERR_INVALID_ARG;
  if (T == 0 && hT == nullptr) return KLA_OK;
  const void* ptrs[] = {q, k, v, g, eta, h0, o, hT};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return KLA_ERR_INVALID_ARG;
  if (!head_dims_ok(dk, dv)) return KLA_ERR_UNSUPPORTED;
  const size_t es = dtype == KLA_BF16 ? 2 : 4;
  const size_t ntok = (size_t)B * T * H, sb = (size_t)B * H * dk * dv * 4;
  if (T > 0) {
    // o and hT are written: neither may overlap an input (hT may alias h0
    // exactly) or the other
    Range ins[] = {rng(q, ntok * dk * es), rng(k, ntok * dk * es), rng(v, ntok * dv * es),
                   rng(g, ntok * gdim * 4), rng(eta, ntok * 4)};
    Range ro = rng(o, ntok * dv * es), rh = rng(hT, hT ? sb : 0);
    for (Range r : ins)
      if (overlap(ro, r) || overlap(rh, r)) return KLA_ERR_INVALID_ARG;
    if (overlap(ro, rng(h0, h0 ? sb : 0)) || overlap(ro, rh)) return KLA_ERR_INVALID_ARG;
  }
  if (hT && h0 && hT != h0) {
    if (overlap(rng(hT, sb), rng(h0, sb))) return KLA_ERR_INVALID_ARG;
  }
  return KLA_OK;
}

// True when [ws, ws + used) overlaps any argument of a prefill call.
static bool workspace_overlaps(const void* ws, size_t used, const void* q, const void* k,
                               const void* v, const float* g, const float* eta,
                               const float* h0, const void* o, const float* hT, int B, int T,
                               int H, int dk, int dv, int dtype) {
  const size_t es = dtype == KLA_BF16 ? 2 : 4;
  const size_t ntok = (size_t)B * T * H, sb = (size_t)B * H * dk * dv * 4;
  const Range rw = rng(ws, used);
  const Range args[] = {rng(q, ntok * dk * es), rng(k, ntok * dk * es), rng(v, ntok * dv * es),
                        rng(g, ntok * 4),       rng(eta, eta ? ntok * 4 : 0),
                        rng(h0, h0 ? sb : 0),   rng(o, ntok * dv * es),
                        rng(hT, hT ? sb : 0)};
  for (Range r : args)
    if (overlap(rw, r)) return true;
  return false;
}

// T == 0: the final state is the initial state.
static kla_status empty_prefill(const float* h0, float* hT, int B, int H, int dk,
                                int dv, cudaStream_t st) {
  if (!hT) return KLA_OK;
  const size_t sb = (size_t)B * H * dk * dv * sizeof(float);
  cudaError_t e = h0 ? (hT == h0 ? cudaSuccess
                                 : cudaMemcpyAsync(hT, h0, sb, cudaMemcpyDeviceToDevice, st))
                     : cudaMemsetAsync(hT, 0, sb, st);
  return e == cudaSuccess ? KLA_OK : KLA_ERR_CUDA;
}

}  // namespace kla

using namespace kla;

extern "C" {

size_t kla_chunk_fwd_workspace_size(int B, int T, int H, int dk, int dv, int dtype) {
  return chunk_workspace_bytes(B, T, H, dk, dv, dtype);
}

int kla_chunk_fwd_segments(int B, int T, int H, int dk, int dv, int dtype, size_t ws_bytes) {
  if (!head_dims_ok(dk, dv) || chunk_ut_workspace_bytes(B, T, H, dk, dv, dtype) == 0) return 0;
  return chunk_chain_segments(B, T, H, dk, dv, ws_bytes);
}

int kla_chunk_fwd_single_launch(int B, int T, int H, int dk, int dv, int dtype,
                                size_t ws_bytes) {
  if (!head_dims_ok(dk, dv) || chunk_ut_workspace_bytes(B, T, H, dk, dv, dtype) == 0) return 0;
  return chunk_single_launch(B, T, H, dk, dv, ws_bytes) ? 1 : 0;
}

}  // extern "C"

// Prefill with the KLA step size, or (eps == kBetaGiven) with beta given.
static kla_status chunk_fwd_impl(const void* q, const void* k, const void* v,
                                 const float* g, const float* eta, float eps,
                                 const float* h0, void* o, float* hT, int B, int T, int H,
                                 int dk, int dv, int chunk, int dtype, void* workspace,
                                 size_t ws_bytes, void* stream) {
  kla_status s = check_prefill(q, k, v, g, eta, eps < 0.f ? 0.f : eps, h0, o, hT, B, T, H,
                               dk, dv, dtype);
  if (s != KLA_OK) return s;
  if (chunk != KLA_CHUNK) return KLA_ERR_UNSUPPORTED;
  cudaStream_t st = (cudaStream_t)stream;
  if (T == 0) return empty_prefill(h0, hT, B, H, dk, dv, st);
  // the UT factors are required; the segment states (the rest of
  // kla_chunk_fwd_workspace_size) only enable the segmented chain
  const size_t need = chunk_ut_workspace_bytes(B, T, H, dk, dv, dtype);
  if (ws_bytes < need || (need > 0 && workspace == nullptr)) return KLA_ERR_INVALID_ARG;
  if (workspace && !aligned16(workspace)) return KLA_ERR_INVALID_ARG;
  if (need > 0 && workspace_overlaps(workspace, chunk_workspace_used(B, T, H, dk, dv, dtype,
                                                                     ws_bytes),
                                     q, k, v, g, eta, h0, o, hT, B, T, H, dk, dv, dtype))
    return KLA_ERR_INVALID_ARG;
  cudaError_t e;
  if (dtype == KLA_FP32) {
    e = launch_recurrent(q, k, v, g, false, eta, eps, h0, o, hT, B, T, H, dk, dv, dtype, st);
  } else {
    unsigned int* err = device_error_ptr();
    if (!err) return KLA_ERR_CUDA;
    e = launch_chunk_tc(q, k, v, g, eta, eps, h0, o, hT, B, T, H, dk, dv, workspace, ws_bytes,
                        err, st);
    if (e == cudaErrorNotSupported) return KLA_ERR_UNSUPPORTED;
  }
  return e == cudaSuccess ? KLA_OK : KLA_ERR_CUDA;
}

extern "C" {

kla_status kla_chunk_fwd_states(const void* q, const void* k, const void* v, const float* g,
                                const float* eta, float eps, const float* h0, void* o,
                                float* hT, float* hs, int B, int T, int H, int dk, int dv,
                                int dtype, void* workspace, size_t ws_bytes, void* stream) {
  if (!(eps >= 0.0f)) return KLA_ERR_INVALID_ARG;
  kla_status s = check_prefill(q, k, v, g, eta, eps, h0, o, hT, B, T, H, dk, dv, dtype, 1, true);
  if (s != KLA_OK) return s;
  if (dtype != KLA_BF16) return KLA_ERR_UNSUPPORTED;
  if (T < 1 || !hs || !aligned16(hs)) return KLA_ERR_INVALID_ARG;
  const size_t need = chunk_ut_workspace_bytes(B, T, H, dk, dv, dtype);
  if (ws_bytes < need || !workspace || !aligned16(workspace)) return KLA_ERR_INVALID_ARG;
  const size_t used = chunk_workspace_used(B, T, H, dk, dv, dtype, ws_bytes);
  if (workspace_overlaps(workspace, used, q, k, v, g, eta, h0, o, hT, B, T, H, dk, dv, dtype))
    return KLA_ERR_INVALID_ARG;
  // hs is written: disjoint from every other argument
  const size_t ntok = (size_t)B * T * H, sb = (size_t)B * H * dk * dv * 4;
  const Range rs = rng(hs, (size_t)B * H * ((T + KLA_CHUNK - 1) / KLA_CHUNK) * dk * dv * 4);
  const Range others[] = {rng(q, ntok * dk * 2), rng(k, ntok * dk * 2), rng(v, ntok * dv * 2),
                          rng(g, ntok * 4),      rng(eta, ntok * 4),    rng(h0, h0 ? sb : 0),
                          rng(o, o ? ntok * dv * 2 : 0), rng(hT, hT ? sb : 0),
                          rng(workspace, used)};
  for (const Range& r : others)
    if (overlap(rs, r)) return KLA_ERR_INVALID_ARG;
  unsigned int* err = device_error_ptr();
  if (!err) return KLA_ERR_CUDA;
  cudaError_t e = launch_chunk_tc(q, k, v, g, eta, eps, h0, o, hT, B, T, H, dk, dv, workspace,
                                  ws_bytes, err, (cudaStream_t)stream, hs);
  if (e == cudaErrorNotSupported) return KLA_ERR_UNSUPPORTED;
  return e == cudaSuccess ? KLA_OK : KLA_ERR_CUDA;
}

kla_status kla_chunk_fwd(const void* q, const void* k, const void* v,
                         const float* g, const float* eta, float eps,
                         const float* h0, void* o, float* hT, int B, int T, int H,
                         int dk, int dv, int chunk, int dtype, void* workspace,
                         size_t ws_bytes, void* stream) {
  if (!(eps >= 0.0f)) return KLA_ERR_INVALID_ARG;
  return chunk_fwd_impl(q, k, v, g, eta, eps, h0, o, hT, B, T, H, dk, dv, chunk, dtype,
                        workspace, ws_bytes, stream);
}

kla_status kla_gdn_chunk_fwd(const void* q, const void* k, const void* v,
                             const float* g, const float* beta, const float* h0, void* o,
                             float* hT, int B, int T, int H, int dk, int dv, int chunk,
                             int dtype, void* workspace, size_t ws_bytes, void* stream) {
  return chunk_fwd_impl(q, k, v, g, beta, kBetaGiven, h0, o, hT, B, T, H, dk, dv, chunk, dtype,
                        workspace, ws_bytes, stream);
}

// Shared checks of the two prefill stages (bf16 chunk path only).
static kla_status check_stage(int T, int dtype, void* workspace, size_t ws_bytes, int B, int H,
                              int dk, int dv) {
  if (dtype != KLA_BF16) return dtype == KLA_FP32 ? KLA_ERR_UNSUPPORTED : KLA_ERR_INVALID_ARG;
  if (T < 1) return KLA_ERR_INVALID_ARG;
  const size_t need = chunk_ut_workspace_bytes(B, T, H, dk, dv, dtype);
  if (need == 0 || ws_bytes < need || workspace == nullptr || !aligned16(workspace))
    return KLA_ERR_INVALID_ARG;
  return KLA_OK;
}

kla_status kla_chunk_ut_transform(const void* k, const float* g, const float* eta, float eps,
                                  int B, int T, int H, int dk, int dtype, void* workspace,
                                  size_t ws_bytes, void* stream) {
  if (B < 1 || H < 1 || T < 1 || !k || !g || !eta) return KLA_ERR_INVALID_ARG;
  if (!(eps >= 0.0f)) return KLA_ERR_INVALID_ARG;
  if ((long long)B * T * H * dk >= (1LL << 40)) return KLA_ERR_INVALID_ARG;
  const void* ptrs[] = {k, g, eta};
  for (const void* p : ptrs)
    if (!aligned16(p)) return KLA_ERR_INVALID_ARG;
  if (!head_dims_ok(dk, dk)) return KLA_ERR_UNSUPPORTED;
  kla_status s = check_stage(T, dtype, workspace, ws_bytes, B, H, dk, dk);
  if (s != KLA_OK) return s;
  const size_t ntok = (size_t)B * T * H;
  Range rw = rng(workspace, chunk_ut_workspace_bytes(B, T, H, dk, dk, dtype));
  if (overlap(rw, rng(k, ntok * dk * 2)) || overlap(rw, rng(g, ntok * 4)) ||
      overlap(rw, rng(eta, ntok * 4)))
    return KLA_ERR_INVALID_ARG;
  unsigned int* err = device_error_ptr();
  if (!err) return KLA_ERR_CUDA;
  cudaError_t e = launch_chunk_ut(k, g, eta, eps, B, T, H, dk, workspace, err,
                                  (cudaStream_t)stream);
  if (e == cudaErrorNotSupported) return KLA_ERR_UNSUPPORTED;
  return e == cudaSuccess ? KLA_OK : KLA_ERR_CUDA;
}

kla_status kla_chunk_ut_bound_check(const void* k, const float* g, const float* eta, float eps,
                                    int B, int T, int H, int dk, int dtype, void* workspace,
                                    size_t ws_bytes, float* ratio_max, void* stream) {
  if (!ratio_max || !aligned16(ratio_max)) return KLA_ERR_INVALID_ARG;
  if (B < 1 || H < 1 || T < 1 || !k || !g || !eta) return KLA_ERR_INVALID_ARG;
  if (!(eps >= 0.0f)) return KLA_ERR_INVALID_ARG;
  if ((long long)B * T * H * dk >= (1LL << 40)) return KLA_ERR_INVALID_ARG;
  const void* ptrs[] = {k, g, eta};
  for (const void* p : ptrs)
    if (!aligned16(p)) return KLA_ERR_INVALID_ARG;
  if (!head_dims_ok(dk, dk)) return KLA_ERR_UNSUPPORTED;
  kla_status s = check_stage(T, dtype, workspace, ws_bytes, B, H, dk, dk);
  if (s != KLA_OK) return s;
  const size_t ntok = (size_t)B * T * H;
  Range rw = rng(workspace, chunk_ut_workspace_bytes(B, T, H, dk, dk, dtype));
  const Range rr = rng(ratio_max, sizeof(float));
  if (overlap(rw, rng(k, ntok * dk * 2)) || overlap(rw, rng(g, ntok * 4)) ||
      overlap(rw, rng(eta, ntok * 4)) || overlap(rr, rw) || overlap(rr, rng(k, ntok * dk * 2)) ||
      overlap(rr, rng(g, ntok * 4)) || overlap(rr, rng(eta, ntok * 4)))
    return KLA_ERR_INVALID_ARG;
  unsigned int* err = device_error_ptr();
  if (!err) return KLA_ERR_CUDA;
  if (cudaMemsetAsync(ratio_max, 0, sizeof(float), (cudaStream_t)stream) != cudaSuccess)
    return KLA_ERR_CUDA;
  cudaError_t e = launch_chunk_ut(k, g, eta, eps, B, T, H, dk, workspace, err,
                                  (cudaStream_t)stream, ratio_max);
  if (e == cudaErrorNotSupported) return KLA_ERR_UNSUPPORTED;
  return e == cudaSuccess ? KLA_OK : KLA_ERR_CUDA;
}

kla_status kla_chunk_state_fwd(const void* q, const void* k, const void* v, const float* g,
                               const float* h0, void* o, float* hT, int B, int T, int H,
                               int dk, int dv, int dtype, void* workspace,
                               size_t ws_bytes, void* stream) {
  // eta only enters through the workspace; validate with a stand-in pointer
  kla_status s = check_prefill(q, k, v, g, g, 0.f, h0, o, hT, B, T, H, dk, dv, dtype);
  if (s != KLA_OK) return s;
  s = check_stage(T, dtype, workspace, ws_bytes, B, H, dk, dv);
  if (s != KLA_OK) return s;
  if (workspace_overlaps(workspace, chunk_workspace_used(B, T, H, dk, dv, dtype, ws_bytes), q,
                         k, v, g, nullptr, h0, o, hT, B, T, H, dk, dv, dtype))
    return KLA_ERR_INVALID_ARG;
  unsigned int* err = device_error_ptr();
  if (!err) return KLA_ERR_CUDA;
  cudaError_t e = launch_chunk_chain(q, k, v, g, h0, o, hT, B, T, H, dk, dv, workspace,
                                     ws_bytes, err, (cudaStream_t)stream);
  if (e == cudaErrorNotSupported) return KLA_ERR_UNSUPPORTED;
  return e == cudaSuccess ? KLA_OK : KLA_ERR_CUDA;
}

kla_status kla_recurrent_fwd(const void* q, const void* k, const void* v,
                             const float* g, const float* eta, float eps,
                             const float* h0, void* o, float* hT, int B, int T,
                             int H, int dk, int dv, int dtype, void* stream) {
  kla_status s = check_prefill(q, k, v, g, eta, eps, h0, o, hT, B, T, H, dk, dv, dtype);
  if (s != KLA_OK) return s;
  cudaStream_t st = (cudaStream_t)stream;
  if (T == 0) return empty_prefill(h0, hT, B, H, dk, dv, st);
  cudaError_t e = launch_recurrent(q, k, v, g, false, eta, eps, h0, o, hT, B, T, H, dk, dv,
                                   dtype, st);
  return e == cudaSuccess ? KLA_OK : KLA_ERR_CUDA;
}

}  // extern "C"

// Prefill with the per-channel gate as chunks: bf16 runs the per-chunk
// factor kernel and the chain kernel's KDA mode, fp32 the token-serial
// kernel; KLA step size or (eps == kBetaGiven) beta given.
static kla_status kda_chunk_impl(const void* q, const void* k, const void* v, const float* g,
                                 const float* eta, float eps, const float* h0, void* o,
                                 float* hT, int B, int T, int H, int dk, int dv, int chunk,
                                 int dtype, void* workspace, size_t ws_bytes, void* stream) {
  kla_status s = check_prefill(q, k, v, g, eta, eps < 0.f ? 0.f : eps, h0, o, hT, B, T, H,
                               dk, dv, dtype, dk);
  if (s != KLA_OK) return s;
  if (chunk != KLA_CHUNK) return KLA_ERR_UNSUPPORTED;
  cudaStream_t st = (cudaStream_t)stream;
  if (T == 0) return empty_prefill(h0, hT, B, H, dk, dv, st);
  if (dtype == KLA_FP32) {
    cudaError_t e = launch_recurrent(q, k, v, g, true, eta, eps, h0, o, hT, B, T, H, dk, dv,
                                     dtype, st);
    return e == cudaSuccess ? KLA_OK : KLA_ERR_CUDA;
  }
  // the per-chunk factors are required; the segment states after them only
  // enable the cut state chain
  const size_t full = kda_chunk_workspace_bytes(B, T, H, dk, dv, dtype);
  const size_t tiles = (size_t)B * H * ((T + KLA_CHUNK - 1) / KLA_CHUNK) *
                       kda_tile_offsets(dk).total;
  if (!workspace || ws_bytes < tiles || !aligned16(workspace)) return KLA_ERR_INVALID_ARG;
  if (workspace_overlaps(workspace, ws_bytes >= full ? full : tiles, q, k, v, g, eta, h0, o, hT,
                         B, T, H, dk, dv, dtype))
    return KLA_ERR_INVALID_ARG;
  // The chunk kernels of this form (kda_prep_kernel, then the chain kernel
  // in its per-channel mode) raised intermittent illegal-instruction faults
  // whose cause has not been found; until it is, the bf16 call runs the
  // token-serial per-channel kernel (exact fp32 evaluation, slower) and
  // leaves the workspace untouched.
  cudaError_t e = launch_recurrent(q, k, v, g, true, eta, eps, h0, o, hT, B, T, H, dk, dv,
                                   dtype, st);
  return e == cudaSuccess ? KLA_OK : KLA_ERR_CUDA;
}

// Prefill with the per-channel gate (token-serial kernel), KLA step size or
// (eps == kBetaGiven) beta given.
static kla_status kda_fwd_impl(const void* q, const void* k, const void* v, const float* g,
                               const float* eta, float eps, const float* h0, void* o,
                               float* hT, int B, int T, int H, int dk, int dv, int dtype,
                               void* stream) {
  kla_status s = check_prefill(q, k, v, g, eta, eps < 0.f ? 0.f : eps, h0, o, hT, B, T, H,
                               dk, dv, dtype, dk);
  if (s != KLA_OK) return s;
  cudaStream_t st = (cudaStream_t)stream;
  if (T == 0) return empty_prefill(h0, hT, B, H, dk, dv, st);
  cudaError_t e = launch_recurrent(q, k, v, g, true, eta, eps, h0, o, hT, B, T, H, dk, dv,
                                   dtype, st);
  return e == cudaSuccess ? KLA_OK : KLA_ERR_CUDA;
}

extern "C" {

kla_status kla_kda_fwd(const void* q, const void* k, const void* v, const float* g,
                       const float* eta, float eps, const float* h0, void* o, float* hT,
                       int B, int T, int H, int dk, int dv, int dtype, void* stream) {
  if (!(eps >= 0.0f)) return KLA_ERR_INVALID_ARG;
  return kda_fwd_impl(q, k, v, g, eta, eps, h0, o, hT, B, T, H, dk, dv, dtype, stream);
}

size_t kla_kda_chunk_fwd_workspace_size(int B, int T, int H, int dk, int dv, int dtype) {
  return kda_chunk_workspace_bytes(B, T, H, dk, dv, dtype);
}

kla_status kla_kda_chunk_fwd(const void* q, const void* k, const void* v, const float* g,
                             const float* eta, float eps, const float* h0, void* o, float* hT,
                             int B, int T, int H, int dk, int dv, int chunk, int dtype,
                             void* workspace, size_t ws_bytes, void* stream) {
  if (!(eps >= 0.0f)) return KLA_ERR_INVALID_ARG;
  return kda_chunk_impl(q, k, v, g, eta, eps, h0, o, hT, B, T, H, dk, dv, chunk, dtype,
                        workspace, ws_bytes, stream);
}

kla_status kla_kda_chunk_fwd_beta(const void* q, const void* k, const void* v, const float* g,
                                  const float* beta, const float* h0, void* o, float* hT, int B,
                                  int T, int H, int dk, int dv, int chunk, int dtype,
                                  void* workspace, size_t ws_bytes, void* stream) {
  return kda_chunk_impl(q, k, v, g, beta, kBetaGiven, h0, o, hT, B, T, H, dk, dv, chunk, dtype,
                        workspace, ws_bytes, stream);
}

kla_status kla_kda_fwd_beta(const void* q, const void* k, const void* v, const float* g,
                            const float* beta, const float* h0, void* o, float* hT, int B,
                            int T, int H, int dk, int dv, int dtype, void* stream) {
  return kda_fwd_impl(q, k, v, g, beta, kBetaGiven, h0, o, hT, B, T, H, dk, dv, dtype,
                      stream);
}

}  // extern "C"

// Gradients of the prefill (token-serial backward), KLA step size or
// (eps == kBetaGiven) beta given; per-channel gate (g, grad_g [B][T][H][dk])
// when vector_gate.
static kla_status bwd_impl(const void* q, const void* k, const void* v, const float* g,
                           const float* eta, float eps, const float* h0, const void* grad_o,
                           const float* grad_hT, float* grad_q, float* grad_k, float* grad_v,
                           float* grad_g, float* grad_eta, float* grad_h0, int B, int T, int H,
                           int dk, int dv, int dtype, void* workspace, size_t ws_bytes,
                           void* stream, bool vector_gate = false, bool chunked = false) {
  if (B < 1 || H < 1 || T < 0) return KLA_ERR_INVALID_ARG;
  if (dtype != KLA_BF16 && dtype != KLA_FP32) return KLA_ERR_INVALID_ARG;
  if (!(eps >= 0.0f) && eps != kBetaGiven) return KLA_ERR_INVALID_ARG;
  if ((long long)B * T * H * (dk > dv ? dk : dv) >= (1LL << 40)) return KLA_ERR_INVALID_ARG;
  if (T > 0 && (!q || !k || !v || !g || !eta || !grad_o || !grad_q || !grad_k || !grad_v ||
                !grad_g || !grad_eta))
    return KLA_ERR_INVALID_ARG;
  const void* ptrs[] = {q,      k,      v,      g,      eta,      h0,      grad_o, grad_hT,
                        grad_q, grad_k, grad_v, grad_g, grad_eta, grad_h0, workspace};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return KLA_ERR_INVALID_ARG;
  if (!head_dims_ok(dk, dv)) return KLA_ERR_UNSUPPORTED;
  const size_t es = dtype == KLA_BF16 ? 2 : 4;
  const size_t ntok = (size_t)B * T * H, sb = (size_t)B * H * dk * dv * 4;
  const size_t gdim = vector_gate ? dk : 1;
  // the chunkwise kernels cover bf16 with d = 128 and the scalar gate; the
  // rest runs the token-serial kernels
  const bool use_chunks = chunked && !vector_gate && dtype == KLA_BF16 && dk == dv;
  const size_t need = use_chunks ? chunk_bwd_workspace_bytes(B, T, H, dk, dv)
                                 : recurrent_bwd_workspace_bytes(B, T, H, dk, dv, vector_gate);
  if (T > 0 && (!workspace || ws_bytes < need)) return KLA_ERR_INVALID_ARG;
  // every written range (gradients, workspace) is disjoint from every input
  // and from the other written ranges
  const Range ins[] = {rng(q, ntok * dk * es),         rng(k, ntok * dk * es),
                       rng(v, ntok * dv * es),         rng(g, ntok * gdim * 4),
                       rng(eta, ntok * 4),             rng(h0, h0 ? sb : 0),
                       rng(grad_o, ntok * dv * es),    rng(grad_hT, grad_hT ? sb : 0)};
  const Range outs[] = {rng(grad_q, ntok * dk * 4), rng(grad_k, ntok * dk * 4),
                        rng(grad_v, ntok * dv * 4), rng(grad_g, ntok * gdim * 4),
                        rng(grad_eta, ntok * 4),    rng(grad_h0, grad_h0 ? sb : 0),
                        rng(workspace, T > 0 ? need : 0)};
  for (size_t a = 0; a < sizeof(outs) / sizeof(outs[0]); ++a) {
    for (const Range& r : ins)
      if (overlap(outs[a], r)) return KLA_ERR_INVALID_ARG;
    for (size_t b2 = a + 1; b2 < sizeof(outs) / sizeof(outs[0]); ++b2)
      if (overlap(outs[a], outs[b2])) return KLA_ERR_INVALID_ARG;
  }
  cudaStream_t st = (cudaStream_t)stream;
  if (T == 0) {  // no tokens: dL/dh0 = dL/dh_T
    if (!grad_h0) return KLA_OK;
    cudaError_t e = grad_hT ? cudaMemcpyAsync(grad_h0, grad_hT, sb, cudaMemcpyDeviceToDevice, st)
                            : cudaMemsetAsync(grad_h0, 0, sb, st);
    return e == cudaSuccess ? KLA_OK : KLA_ERR_CUDA;
  }
  unsigned int* err = use_chunks ? device_error_ptr() : nullptr;
  if (use_chunks && !err) return KLA_ERR_CUDA;
  cudaError_t e =
      use_chunks
          ? launch_chunk_bwd(q, k, v, g, eta, eps, h0, grad_o, grad_hT, grad_q, grad_k, grad_v,
                             grad_g, grad_eta, grad_h0, B, T, H, dk, dv, workspace, err, st)
          : launch_recurrent_bwd(q, k, v, g, vector_gate, eta, eps, h0, grad_o, grad_hT, grad_q,
                                 grad_k, grad_v, grad_g, grad_eta, grad_h0, B, T, H, dk, dv,
                                 dtype, workspace, st);
  return e == cudaSuccess ? KLA_OK : KLA_ERR_CUDA;
}

extern "C" {

size_t kla_recurrent_bwd_workspace_size(int B, int T, int H, int dk, int dv) {
  if (!head_dims_ok(dk, dv)) return 0;
  return recurrent_bwd_workspace_bytes(B, T, H, dk, dv, false);
}

size_t kla_chunk_bwd_workspace_size(int B, int T, int H, int dk, int dv, int dtype) {
  if (!head_dims_ok(dk, dv)) return 0;
  if (dtype == KLA_BF16 && dk == dv) return chunk_bwd_workspace_bytes(B, T, H, dk, dv);
  return recurrent_bwd_workspace_bytes(B, T, H, dk, dv, false);
}

kla_status kla_chunk_bwd(const void* q, const void* k, const void* v, const float* g,
                         const float* eta, float eps, const float* h0, const void* grad_o,
                         const float* grad_hT, float* grad_q, float* grad_k, float* grad_v,
                         float* grad_g, float* grad_eta, float* grad_h0, int B, int T, int H,
                         int dk, int dv, int dtype, void* workspace, size_t ws_bytes,
                         void* stream) {
  if (!(eps >= 0.0f)) return KLA_ERR_INVALID_ARG;
  return bwd_impl(q, k, v, g, eta, eps, h0, grad_o, grad_hT, grad_q, grad_k, grad_v, grad_g,
                  grad_eta, grad_h0, B, T, H, dk, dv, dtype, workspace, ws_bytes, stream, false,
                  true);
}

kla_status kla_gdn_chunk_bwd(const void* q, const void* k, const void* v, const float* g,
                             const float* beta, const float* h0, const void* grad_o,
                             const float* grad_hT, float* grad_q, float* grad_k, float* grad_v,
                             float* grad_g, float* grad_beta, float* grad_h0, int B, int T,
                             int H, int dk, int dv, int dtype, void* workspace, size_t ws_bytes,
                             void* stream) {
  return bwd_impl(q, k, v, g, beta, kBetaGiven, h0, grad_o, grad_hT, grad_q, grad_k, grad_v,
                  grad_g, grad_beta, grad_h0, B, T, H, dk, dv, dtype, workspace, ws_bytes,
                  stream, false, true);
}

size_t kla_kda_recurrent_bwd_workspace_size(int B, int T, int H, int dk, int dv) {
  if (!head_dims_ok(dk, dv)) return 0;
  return recurrent_bwd_workspace_bytes(B, T, H, dk, dv, true);
}

kla_status kla_kda_recurrent_bwd(const void* q, const void* k, const void* v, const float* g,
                                 const float* eta, float eps, const float* h0,
                                 const void* grad_o, const float* grad_hT, float* grad_q,
                                 float* grad_k, float* grad_v, float* grad_g, float* grad_eta,
                                 float* grad_h0, int B, int T, int H, int dk, int dv, int dtype,
                                 void* workspace, size_t ws_bytes, void* stream) {
  if (!(eps >= 0.0f)) return KLA_ERR_INVALID_ARG;
  return bwd_impl(q, k, v, g, eta, eps, h0, grad_o, grad_hT, grad_q, grad_k, grad_v, grad_g,
                  grad_eta, grad_h0, B, T, H, dk, dv, dtype, workspace, ws_bytes, stream, true);
}

kla_status kla_kda_recurrent_bwd_beta(const void* q, const void* k, const void* v,
                                      const float* g, const float* beta, const float* h0,
                                      const void* grad_o, const float* grad_hT, float* grad_q,
                                      float* grad_k, float* grad_v, float* grad_g,
                                      float* grad_beta, float* grad_h0, int B, int T, int H,
                                      int dk, int dv, int dtype, void* workspace,
                                      size_t ws_bytes, void* stream) {
  return bwd_impl(q, k, v, g, beta, kBetaGiven, h0, grad_o, grad_hT, grad_q, grad_k, grad_v,
                  grad_g, grad_beta, grad_h0, B, T, H, dk, dv, dtype, workspace, ws_bytes,
                  stream, true);
}

kla_status kla_recurrent_bwd(const void* q, const void* k, const void* v, const float* g,
                             const float* eta, float eps, const float* h0, const void* grad_o,
                             const float* grad_hT, float* grad_q, float* grad_k, float* grad_v,
                             float* grad_g, float* grad_eta, float* grad_h0, int B, int T,
                             int H, int dk, int dv, int dtype, void* workspace, size_t ws_bytes,
                             void* stream) {
  if (!(eps >= 0.0f)) return KLA_ERR_INVALID_ARG;
  return bwd_impl(q, k, v, g, eta, eps, h0, grad_o, grad_hT, grad_q, grad_k, grad_v, grad_g,
                  grad_eta, grad_h0, B, T, H, dk, dv, dtype, workspace, ws_bytes, stream);
}

kla_status kla_gdn_recurrent_bwd(const void* q, const void* k, const void* v, const float* g,
                                 const float* beta, const float* h0, const void* grad_o,
                                 const float* grad_hT, float* grad_q, float* grad_k,
                                 float* grad_v, float* grad_g, float* grad_beta, float* grad_h0,
                                 int B, int T, int H, int dk, int dv, int dtype, void* workspace,
                                 size_t ws_bytes, void* stream) {
  return bwd_impl(q, k, v, g, beta, kBetaGiven, h0, grad_o, grad_hT, grad_q, grad_k, grad_v,
                  grad_g, grad_beta, grad_h0, B, T, H, dk, dv, dtype, workspace, ws_bytes,
                  stream);
}

}  // extern "C"

// One decode step with the KLA step size, or (eps == kBetaGiven) beta given;
// a per-channel gate when vector_gate (g [B][H][dk]).
static kla_status decode_impl(const void* q, const void* k, const void* v,
                              const float* g, const float* eta, float eps, float* S,
                              void* o, int B, int H, int dk, int dv, int dtype,
                              void* stream, bool vector_gate = false) {
  if (B < 1 || H < 1) return KLA_ERR_INVALID_ARG;
  if (dtype != KLA_BF16 && dtype != KLA_FP32) return KLA_ERR_INVALID_ARG;
  const void* ptrs[] = {q, k, v, g, eta, S, o};
  for (const void* p : ptrs)
    if (!p || !aligned16(p)) return KLA_ERR_INVALID_ARG;
  if (!head_dims_ok(dk, dv)) return KLA_ERR_UNSUPPORTED;
  const size_t es = dtype == KLA_BF16 ? 2 : 4;
  const size_t nh = (size_t)B * H;
  Range ro = rng(o, nh * dv * es);
  Range rs = rng(S, nh * dk * dv * 4);
  Range ins[] = {rng(q, nh * dk * es), rng(k, nh * dk * es), rng(v, nh * dv * es),
                 rng(g, nh * (vector_gate ? dk : 1) * 4), rng(eta, nh * 4)};
  if (overlap(ro, rs)) return KLA_ERR_INVALID_ARG;
  for (Range r : ins)
    if (overlap(ro, r) || overlap(rs, r)) return KLA_ERR_INVALID_ARG;
  cudaError_t e = launch_decode(q, k, v, g, vector_gate, eta, eps, S, o, B, H, dk, dv, dtype,
                                (cudaStream_t)stream);
  return e == cudaSuccess ? KLA_OK : KLA_ERR_CUDA;
}

extern "C" {

kla_status kla_decode_step(const void* q, const void* k, const void* v,
                           const float* g, const float* eta, float eps, float* S,
                           void* o, int B, int H, int dk, int dv, int dtype,
                           void* stream) {
  if (!(eps >= 0.0f)) return KLA_ERR_INVALID_ARG;
  return decode_impl(q, k, v, g, eta, eps, S, o, B, H, dk, dv, dtype, stream);
}

kla_status kla_gdn_decode_step(const void* q, const void* k, const void* v,
                               const float* g, const float* beta, float* S, void* o, int B,
                               int H, int dk, int dv, int dtype, void* stream) {
  return decode_impl(q, k, v, g, beta, kBetaGiven, S, o, B, H, dk, dv, dtype, stream);
}

kla_status kla_kda_decode_step(const void* q, const void* k, const void* v, const float* g,
                               const float* eta, float eps, float* S, void* o, int B, int H,
                               int dk, int dv, int dtype, void* stream) {
  if (!(eps >= 0.0f)) return KLA_ERR_INVALID_ARG;
  return decode_impl(q, k, v, g, eta, eps, S, o, B, H, dk, dv, dtype, stream, true);
}

kla_status kla_kda_decode_step_beta(const void* q, const void* k, const void* v,
                                    const float* g, const float* beta, float* S, void* o,
                                    int B, int H, int dk, int dv, int dtype, void* stream) {
  return decode_impl(q, k, v, g, beta, kBetaGiven, S, o, B, H, dk, dv, dtype, stream, true);
}

}  // extern "C"

namespace kla {
// One thread waits, with the kernels' bounded wait, on an mbarrier phase
// that nothing completes (no thread arrives); when the limit runs out it
// reports a timeout through the device error word, exactly as a stuck
// tensor-core kernel would, and returns.
__global__ void selftest_wait_kernel(uint64_t limit_ns, unsigned int* err) {
  __shared__ uint64_t bar;
  ptx::mbar_init(&bar, 1);
  ptx::mbar_init_fence();
  if (!wait_bounded_ns(&bar, 0, limit_ns)) report_timeout(err);
}
}  // namespace kla

extern "C" {

kla_status kla_selftest_wait_timeout(unsigned int limit_ms, void* stream) {
  if (limit_ms < 1 || limit_ms > 10000) return KLA_ERR_INVALID_ARG;
  unsigned int* err = device_error_ptr();
  if (!err) return KLA_ERR_CUDA;
  selftest_wait_kernel<<<1, 1, 0, (cudaStream_t)stream>>>((uint64_t)limit_ms * 1000000ull, err);
  return cudaGetLastError() == cudaSuccess ? KLA_OK : KLA_ERR_CUDA;
}

kla_status kla_check_device_error(void* stream) {
  if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return KLA_ERR_CUDA;
  unsigned int v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, g_device_error, sizeof(v)) != cudaSuccess) return KLA_ERR_CUDA;
  if (v && cudaMemcpyToSymbol(g_device_error, &zero, sizeof(zero)) != cudaSuccess)
    return KLA_ERR_CUDA;
  if (v & KLA_DEVERR_TIMEOUT) return KLA_ERR_TIMEOUT;
  return v ? KLA_ERR_BOUND : KLA_OK;
}

const char* kla_status_string(int status) {
  switch (status) {
    case KLA_OK: return "ok";
    case KLA_ERR_INVALID_ARG: return "invalid argument";
    case KLA_ERR_UNSUPPORTED: return "unsupported configuration";
    case KLA_ERR_CUDA: return "CUDA error";
    case KLA_ERR_TIMEOUT: return "device-side wait timed out";
    case KLA_ERR_BOUND: return "a debug bound check found a value above its bound";
    default: return "unknown status";
  }
}

int kla_version(void) { return 100; }

}  // extern "C"
