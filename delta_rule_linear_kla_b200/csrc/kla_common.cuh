// Shared helpers of the KLA CUDA library: element loads/stores for the two
// I/O types, warp reductions and the device error word.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/kla.h"

namespace kla {

// Device error word: one per device, owned by kla_api.cu, passed to kernels
// as a pointer.  Bounded waits that give up set a bit instead of hanging.
// KLA_DEVERR_BOUND: a debug bound check of the UT factors found an entry
// above its bound (kla_chunk_ut_bound_check).
enum : unsigned int { KLA_DEVERR_TIMEOUT = 1u, KLA_DEVERR_BOUND = 2u };

__device__ __forceinline__ void report_timeout(unsigned int* err) {
  atomicOr(err, KLA_DEVERR_TIMEOUT);
}

// eps value that selects the gated-delta form inside the kernels: beta_t is
// then the per-token input itself (the `eta` argument) instead of
// eta_t / (||k_t||^2 + eps).  The C ABI never passes a negative eps otherwise.
constexpr float kBetaGiven = -1.0f;

__device__ __forceinline__ float step_size(float eta, float knorm2, float eps) {
  return eps < 0.f ? eta : eta / (knorm2 + eps);
}

// Launchers (one per kernel family), all queue work on `st` only.
// vector_gate: g holds one log-gate per key channel (KDA form) instead of one
// per token / head.
cudaError_t launch_decode(const void* q, const void* k, const void* v,
                          const float* g, bool vector_gate, const float* eta, float eps,
                          float* S, void* o, int B, int H, int dk, int dv, int dtype,
                          cudaStream_t st);
cudaError_t launch_recurrent(const void* q, const void* k, const void* v,
                             const float* g, bool vector_gate, const float* eta, float eps,
                             const float* h0, void* o, float* hT, int B, int T,
                             int H, int dk, int dv, int dtype, cudaStream_t st);

// Token-serial backward (kla_backward.cu): gradients of q, k, v (fp32), of
// the log-gate(s), of eta (or of beta when eps == kBetaGiven) and of h0.
size_t recurrent_bwd_workspace_bytes(int B, int T, int H, int dk, int dv, bool vector_gate);
cudaError_t launch_recurrent_bwd(const void* q, const void* k, const void* v, const float* g,
                                 bool vector_gate, const float* eta, float eps,
                                 const float* h0, const void* dout, const float* dhT,
                                 float* dq, float* dk, float* dv, float* dg, float* deta,
                                 float* dh0, int B, int T, int H, int dkd, int dvd, int dtype,
                                 void* ws, cudaStream_t st);

// Chunkwise backward (kla_chunk_bwd.cu; bf16, d_k = d_v in {64, 128}, scalar gate).
size_t chunk_bwd_workspace_bytes(int B, int T, int H, int dk, int dv);
cudaError_t launch_chunk_bwd(const void* q, const void* k, const void* v, const float* g,
                             const float* eta, float eps, const float* h0, const void* dout,
                             const float* dhT, float* dq, float* dk, float* dv, float* dg,
                             float* deta, float* dh0, int B, int T, int H, int dkd, int dvd,
                             void* ws, unsigned int* err, cudaStream_t st);

template <typename T> struct IO;

template <> struct IO<float> {
  static __device__ __forceinline__ float ld(const float* p) { return *p; }
  static __device__ __forceinline__ void st(float* p, float x) { *p = x; }
  // 4 consecutive elements
  static __device__ __forceinline__ float4 ld4(const float* p) {
    return *reinterpret_cast<const float4*>(p);
  }
  static __device__ __forceinline__ void st4(float* p, float4 x) {
    *reinterpret_cast<float4*>(p) = x;
  }
};

template <> struct IO<__nv_bfloat16> {
  static __device__ __forceinline__ float ld(const __nv_bfloat16* p) {
    return __bfloat162float(*p);
  }
  static __device__ __forceinline__ void st(__nv_bfloat16* p, float x) {
    *p = __float2bfloat16_rn(x);
  }
  static __device__ __forceinline__ float4 ld4(const __nv_bfloat16* p) {
    uint2 u = *reinterpret_cast<const uint2*>(p);
    __nv_bfloat162 a = *reinterpret_cast<__nv_bfloat162*>(&u.x);
    __nv_bfloat162 b = *reinterpret_cast<__nv_bfloat162*>(&u.y);
    float2 fa = __bfloat1622float2(a), fb = __bfloat1622float2(b);
    return make_float4(fa.x, fa.y, fb.x, fb.y);
  }
  static __device__ __forceinline__ void st4(__nv_bfloat16* p, float4 x) {
    __nv_bfloat162 a = __floats2bfloat162_rn(x.x, x.y);
    __nv_bfloat162 b = __floats2bfloat162_rn(x.z, x.w);
    uint2 u;
    u.x = *reinterpret_cast<uint32_t*>(&a);
    u.y = *reinterpret_cast<uint32_t*>(&b);
    *reinterpret_cast<uint2*>(p) = u;
  }
};

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

}  // namespace kla
