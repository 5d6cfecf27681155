// Token-serial KLA prefill on CUDA cores (fp32 arithmetic).
//
// Evaluates the recurrence one token at a time, exactly as stated:
//   beta_t = eta_t / (||k_t||^2 + eps)       ("Kaczmarz Linear Attention",
//                                              Abstract)
//   r = h^T k_t;  u = beta_t (v_t - alpha_t r);  h <- alpha_t h + k_t u^T;
//   o_t = h^T q_t                             ("Deep Dive into KDA", 2.2)
// With a per-channel gate (KDA form, "Deep Dive into KDA", section 2.3:
// S_t = (I - beta_t k_t k_t^T) Diag(a_t) S_{t-1} + beta_t v_t k_t^T) the rows
// of h are first scaled by a_i = exp(g_{t,i}) and the erase reads that
// decayed state:  h <- Diag(a) h;  r = h^T k_t;  u = beta_t (v_t - r);
// h <- h + k_t u^T.  (For a scalar gate this is the line above.)
// Columns of h are independent: a lane owns one column j and DK/4 of its
// rows; the four lanes sharing a column (lane bits 3..4) combine their
// partial dot products with two shuffles.  A warp covers 8 columns and a
// CTA of 4 warps a 32-column slab of one head.  The next token's operands
// are loaded while the current token is processed.
#include "kla_common.cuh"

namespace kla {

// VG: g is per key channel ([B][T][H][DK]) instead of per token.
template <typename T, int DK, int DV, bool VG>
__global__ void __launch_bounds__(128)
recurrent_kernel(const T* __restrict__ q, const T* __restrict__ k,
                 const T* __restrict__ v, const float* __restrict__ g,
                 const float* __restrict__ eta, float eps,
                 const float* __restrict__ h0, T* __restrict__ o,
                 float* __restrict__ hT, int Tlen, int H) {
  constexpr int R = DK / 4;  // rows per lane
  static_assert(R % 4 == 0, "rows");
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int rg = lane >> 3, c = lane & 7;
  const int j = blockIdx.x * 32 + warp * 8 + c;
  const int hh = blockIdx.y, b = blockIdx.z;
  const size_t head = (size_t)b * H + hh;

  float hs[R];
#pragma unroll
  for (int m = 0; m < R; ++m)
    hs[m] = h0 ? h0[(head * DK + rg * R + m) * DV + j] : 0.f;

  constexpr int RG = VG ? R : 1;  // gate values a lane needs per token
  float kk[R], qq[R], gk[RG];
  float vj = 0.f, et = 0.f;
  auto load_tok = [&](int t, float* kd, float* qd, float* gd, float& vv, float& ee) {
    const size_t tok = ((size_t)b * Tlen + t) * H + hh;
    const T* kt = k + tok * DK + rg * R;
    const T* qt = q + tok * DK + rg * R;
#pragma unroll
    for (int m = 0; m < R; m += 4) {
      float4 a = IO<T>::ld4(kt + m), bq = IO<T>::ld4(qt + m);
      kd[m] = a.x; kd[m + 1] = a.y; kd[m + 2] = a.z; kd[m + 3] = a.w;
      qd[m] = bq.x; qd[m + 1] = bq.y; qd[m + 2] = bq.z; qd[m + 3] = bq.w;
    }
    if constexpr (VG) {
#pragma unroll
      for (int m = 0; m < R; m += 4) {
        const float4 x = *reinterpret_cast<const float4*>(g + tok * DK + rg * R + m);
        gd[m] = x.x; gd[m + 1] = x.y; gd[m + 2] = x.z; gd[m + 3] = x.w;
      }
    } else {
      gd[0] = g[tok];
    }
    vv = IO<T>::ld(v + tok * DV + j);
    ee = eta[tok];
  };
  if (Tlen > 0) load_tok(0, kk, qq, gk, vj, et);

  for (int t = 0; t < Tlen; ++t) {
    float kn[R], qn[R], gn[RG], vn = 0.f, en = 0.f;
    if (t + 1 < Tlen) load_tok(t + 1, kn, qn, gn, vn, en);

    float alpha = 1.f;
    if constexpr (VG) {  // Diag(a) h first; the erase reads the decayed rows
#pragma unroll
      for (int m = 0; m < R; ++m) hs[m] *= expf(gk[m]);
    } else {
      alpha = expf(gk[0]);
    }
    float n2 = 0.f, r = 0.f;
#pragma unroll
    for (int m = 0; m < R; ++m) {
      n2 = fmaf(kk[m], kk[m], n2);
      r = fmaf(hs[m], kk[m], r);
    }
    n2 += __shfl_xor_sync(0xffffffffu, n2, 8);
    n2 += __shfl_xor_sync(0xffffffffu, n2, 16);
    r += __shfl_xor_sync(0xffffffffu, r, 8);
    r += __shfl_xor_sync(0xffffffffu, r, 16);
    const float beta = step_size(et, n2, eps);
    const float u = beta * (vj - alpha * r);
    float s = 0.f;
#pragma unroll
    for (int m = 0; m < R; ++m) {
      hs[m] = fmaf(kk[m], u, alpha * hs[m]);
      s = fmaf(hs[m], qq[m], s);
    }
    s += __shfl_xor_sync(0xffffffffu, s, 8);
    s += __shfl_xor_sync(0xffffffffu, s, 16);
    if (rg == 0) IO<T>::st(o + (((size_t)b * Tlen + t) * H + hh) * DV + j, s);

#pragma unroll
    for (int m = 0; m < R; ++m) {
      kk[m] = kn[m];
      qq[m] = qn[m];
    }
#pragma unroll
    for (int m = 0; m < RG; ++m) gk[m] = gn[m];
    vj = vn;
    et = en;
  }
  if (hT) {
#pragma unroll
    for (int m = 0; m < R; ++m) hT[(head * DK + rg * R + m) * DV + j] = hs[m];
  }
}

template <typename T, int DK, int DV>
static cudaError_t launch_rec_t(const void* q, const void* k, const void* v,
                                const float* g, bool vector_gate, const float* eta,
                                float eps, const float* h0, void* o, float* hT, int B,
                                int Tlen, int H, cudaStream_t st) {
  dim3 grid(DV / 32, H, B);
  if (vector_gate)
    recurrent_kernel<T, DK, DV, true><<<grid, 128, 0, st>>>(
        (const T*)q, (const T*)k, (const T*)v, g, eta, eps, h0, (T*)o, hT, Tlen, H);
  else
    recurrent_kernel<T, DK, DV, false><<<grid, 128, 0, st>>>(
        (const T*)q, (const T*)k, (const T*)v, g, eta, eps, h0, (T*)o, hT, Tlen, H);
  return cudaGetLastError();
}

cudaError_t launch_recurrent(const void* q, const void* k, const void* v,
                             const float* g, bool vector_gate, const float* eta, float eps,
                             const float* h0, void* o, float* hT, int B, int T,
                             int H, int dk, int dv, int dtype, cudaStream_t st) {
  const bool vg = vector_gate;
  if (dtype == KLA_BF16) {
    if (dk == 128 && dv == 128)
      return launch_rec_t<__nv_bfloat16, 128, 128>(q, k, v, g, vg, eta, eps, h0, o, hT, B,
                                                   T, H, st);
    if (dk == 64 && dv == 64)
      return launch_rec_t<__nv_bfloat16, 64, 64>(q, k, v, g, vg, eta, eps, h0, o, hT, B, T,
                                                 H, st);
  } else {
    if (dk == 128 && dv == 128)
      return launch_rec_t<float, 128, 128>(q, k, v, g, vg, eta, eps, h0, o, hT, B, T, H, st);
    if (dk == 64 && dv == 64)
      return launch_rec_t<float, 64, 64>(q, k, v, g, vg, eta, eps, h0, o, hT, B, T, H, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace kla
