// Single-token decode step of Kaczmarz Linear Attention, in place on the state.
//
// Per head (h = S^T, [DK][DV] fp32) and new token (q, k, v, g, eta):
//   beta = eta / (||k||^2 + eps)      ("Kaczmarz Linear Attention", Abstract)
//   alpha = exp(g)
//   r = h^T k,  s = h^T q             (one read of the state)
//   u = beta (v - alpha r)
//   h <- alpha h + k u^T              (one write of the state)
//   o = h_new^T q = alpha s + u (k . q)
// which is one step of the gated delta rule ("Deep Dive into KDA",
// section 2.2) with o read from the updated state.  With a per-channel gate
// (KDA form, same page, section 2.3) the rows of h are scaled by
// a_i = exp(g_i) as they are loaded and the step above runs on the decayed
// state with alpha = 1.  Columns of h are independent, so a CTA owns one head
// and a slab of CW columns.
//
// The state is the only large operand (DK*DV*4 bytes per head, read once and
// written once with 128-bit accesses); the kernel is a pure HBM stream, so
// everything is arranged for coalescing and bytes in flight: each thread
// keeps RT rows x 4 columns of h in registers between the reduction and the
// update, so h is never re-read.  The grid is persistent (4 CTAs per SM,
// each walking (head, slab) tiles grid-stride), so every SM stays loaded to
// the end instead of a last, partly filled wave of CTAs.
#include "kla_common.cuh"

namespace kla {

// VG: g is per key channel ([B][H][DK]) instead of per head.
template <typename T, int DK, int DV, int CW, int NT, bool VG>
__global__ void __launch_bounds__(NT, 65536 / (NT * 64))  // <= 64 registers: 4 CTAs/SM
decode_kernel(const T* __restrict__ q, const T* __restrict__ k,
              const T* __restrict__ v, const float* __restrict__ g,
              const float* __restrict__ eta, float eps, float* __restrict__ S,
              T* __restrict__ o, int H, int ntiles) {
  constexpr int LPR = CW / 4;        // threads per state row (float4 each)
  constexpr int RPP = NT / LPR;      // rows covered per pass
  constexpr int RT = DK / RPP;       // rows held per thread
  static_assert(NT % LPR == 0 && DK % RPP == 0, "tile");
  constexpr int NSLAB = DV / CW;

  __shared__ float red_r[RPP][CW];
  __shared__ float red_s[RPP][CW];
  __shared__ float u_sh[CW];
  __shared__ float kq_sh[3];  // n2, k.q

  const int tid = threadIdx.x;
#pragma unroll 1
  for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
  const int slab = tile % NSLAB;
  const int head = tile / NSLAB;  // = b * H + h
  const int c4 = tid % LPR;
  const int row0 = tid / LPR;
  const int col = slab * CW + 4 * c4;

  float* Sh = S + (size_t)head * DK * DV;
  const T* kp = k + (size_t)head * DK;
  const T* qp = q + (size_t)head * DK;

  // State tile: issue every load first (bytes in flight), then compute.
  float4 hv[RT];
#pragma unroll
  for (int m = 0; m < RT; ++m)
    hv[m] = *reinterpret_cast<const float4*>(Sh + (size_t)(row0 + m * RPP) * DV + col);

  float kr[RT], qr[RT];
#pragma unroll
  for (int m = 0; m < RT; ++m) {
    kr[m] = IO<T>::ld(kp + row0 + m * RPP);
    qr[m] = IO<T>::ld(qp + row0 + m * RPP);
  }
  if constexpr (VG) {  // Diag(a) h: row i of the state times exp(g_i)
#pragma unroll
    for (int m = 0; m < RT; ++m) {
      const float a = expf(g[(size_t)head * DK + row0 + m * RPP]);
      hv[m].x *= a; hv[m].y *= a; hv[m].z *= a; hv[m].w *= a;
    }
  }

  // ||k||^2 and k.q over the full key dimension (warp 0).
  if (tid < 32) {
    float n2 = 0.f, kq = 0.f;
    for (int i = tid; i < DK; i += 32) {
      float a = IO<T>::ld(kp + i), b = IO<T>::ld(qp + i);
      n2 = fmaf(a, a, n2);
      kq = fmaf(a, b, kq);
    }
    n2 = warp_sum(n2);
    kq = warp_sum(kq);
    if (tid == 0) {
      kq_sh[0] = n2;
      kq_sh[1] = kq;
    }
  }

  // Partial column reductions over this thread's rows.
  float4 pr = make_float4(0.f, 0.f, 0.f, 0.f), ps = pr;
#pragma unroll
  for (int m = 0; m < RT; ++m) {
    pr.x = fmaf(hv[m].x, kr[m], pr.x); pr.y = fmaf(hv[m].y, kr[m], pr.y);
    pr.z = fmaf(hv[m].z, kr[m], pr.z); pr.w = fmaf(hv[m].w, kr[m], pr.w);
    ps.x = fmaf(hv[m].x, qr[m], ps.x); ps.y = fmaf(hv[m].y, qr[m], ps.y);
    ps.z = fmaf(hv[m].z, qr[m], ps.z); ps.w = fmaf(hv[m].w, qr[m], ps.w);
  }
  *reinterpret_cast<float4*>(&red_r[row0][4 * c4]) = pr;
  *reinterpret_cast<float4*>(&red_s[row0][4 * c4]) = ps;
  __syncthreads();

  const float alpha = VG ? 1.f : expf(g[head]);
  const float beta = step_size(eta[head], kq_sh[0], eps);
  if (tid < CW) {
    float r = 0.f, s = 0.f;
#pragma unroll
    for (int p = 0; p < RPP; ++p) {
      r += red_r[p][tid];
      s += red_s[p][tid];
    }
    const int j = slab * CW + tid;
    const float u = beta * (IO<T>::ld(v + (size_t)head * DV + j) - alpha * r);
    u_sh[tid] = u;
    IO<T>::st(o + (size_t)head * DV + j, fmaf(u, kq_sh[1], alpha * s));
  }
  __syncthreads();

  const float4 u4 = *reinterpret_cast<const float4*>(&u_sh[4 * c4]);
#pragma unroll
  for (int m = 0; m < RT; ++m) {
    float4 x = hv[m];
    const float kk = kr[m];
    x.x = fmaf(kk, u4.x, alpha * x.x); x.y = fmaf(kk, u4.y, alpha * x.y);
    x.z = fmaf(kk, u4.z, alpha * x.z); x.w = fmaf(kk, u4.w, alpha * x.w);
    *reinterpret_cast<float4*>(Sh + (size_t)(row0 + m * RPP) * DV + col) = x;
  }
  // no barrier here: every read of red_r, red_s and kq_sh for this tile came
  // before the barrier above, and the next tile writes u_sh only after its
  // first barrier, which every thread reaches after this update
  }
}

template <typename T, int DK, int DV>
static cudaError_t launch_decode_t(const void* q, const void* k, const void* v,
                                   const float* g, bool vector_gate, const float* eta,
                                   float eps, float* S, void* o, int B, int H,
                                   cudaStream_t st) {
  constexpr int CW = (DV >= 128) ? 64 : DV;
  constexpr int NT = 256;
  const int ntiles = B * H * (DV / CW);
  if (ntiles == 0) return cudaSuccess;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  static int sms[64] = {};
  if (!sms[dev]) {
    cudaError_t e = cudaDeviceGetAttribute(&sms[dev], cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
  }
  const int cap = 4 * sms[dev];  // resident CTAs (<= 64 registers, 256 threads)
  const int grid = ntiles < cap ? ntiles : cap;
  if (vector_gate)
    decode_kernel<T, DK, DV, CW, NT, true><<<grid, NT, 0, st>>>(
        (const T*)q, (const T*)k, (const T*)v, g, eta, eps, S, (T*)o, H, ntiles);
  else
    decode_kernel<T, DK, DV, CW, NT, false><<<grid, NT, 0, st>>>(
        (const T*)q, (const T*)k, (const T*)v, g, eta, eps, S, (T*)o, H, ntiles);
  return cudaGetLastError();
}

cudaError_t launch_decode(const void* q, const void* k, const void* v,
                          const float* g, bool vector_gate, const float* eta, float eps,
                          float* S, void* o, int B, int H, int dk, int dv, int dtype,
                          cudaStream_t st) {
  const bool vg = vector_gate;
  if (dtype == KLA_BF16) {
    if (dk == 128 && dv == 128)
      return launch_decode_t<__nv_bfloat16, 128, 128>(q, k, v, g, vg, eta, eps, S, o, B, H,
                                                      st);
    if (dk == 64 && dv == 64)
      return launch_decode_t<__nv_bfloat16, 64, 64>(q, k, v, g, vg, eta, eps, S, o, B, H, st);
  } else {
    if (dk == 128 && dv == 128)
      return launch_decode_t<float, 128, 128>(q, k, v, g, vg, eta, eps, S, o, B, H, st);
    if (dk == 64 && dv == 64)
      return launch_decode_t<float, 64, 64>(q, k, v, g, vg, eta, eps, S, o, B, H, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace kla
