// Chunkwise backward of the KLA / gated delta rule prefill (bf16 I/O,
// scalar gate, d_k = d_v = 64 or 128): the gradients of a loss L given dL/do and dL/dh_T, from the
// chunk form of the forward ("Deep Dive into KDA", section 3, with the KLA
// step size of "Kaczmarz Linear Attention", Abstract).  Per chunk n of C = 64
// tokens with start state h_n (G = in-chunk cumsum of g, gamma = e^G,
// gamma_C = e^{G_last}, Gamma_rs = e^{G_r - G_s}):
//   A = strict_lower(diag(beta) K K^T (*) Gamma),  T = (I + A)^{-1}
//   W = T diag(beta gamma) K,  U = T diag(beta) V,  V' = U - W h_n
//   P = lower_incl(Q K^T (*) Gamma),  O = diag(gamma) Q h_n + P V'
//   h_{n+1} = gamma_C h_n + Kt^T V',  Kt = diag(gamma_C / gamma) K.
// The pages print no backward.  Its adjoint, derived here, splits into one
// reverse chain over the chunks and independent per-chunk work:
//   dV'_n = P^T dO + Kt dH_{n+1}
//   dH_n  = gamma_C dH_{n+1} + (diag(gamma) Q)^T dO - W^T dV'_n      (chain)
//   dP = dO V'^T (*) incl;  dQ = diag(gamma) dO h_n^T + (dP (*) Gamma) K
//   dW = -dV' h_n^T;  dT = dW (diag(beta gamma) K)^T + dV' (diag(beta) V)^T
//   dA = -strict_lower(T^T dT T^T);  E = dA (*) Gamma
//   dV = diag(beta) T^T dV'
//   dK = (dP (*) Gamma)^T Q + diag(gamma_C / gamma) V' dH_{n+1}^T
//        + diag(beta gamma) T^T dW + diag(beta) E K + (diag(beta) E)^T K
//   dbeta = gamma (*) rowdot(T^T dW, K) + rowdot(T^T dV', V) + rowsum(E (*) K K^T)
//   dG = rowsum(F) - colsum(F) for F = dA (*) A and F = dP (*) P,
//        + rowdot(dO, diag(gamma) Q h_n) + beta gamma rowdot(T^T dW, K)
//        - rowdot(dKt, Kt);  dG_last += sum rowdot(dKt, Kt) + gamma_C <dH_{n+1}, h_n>
//   dg = reverse in-chunk cumsum of dG;  KLA: deta = dbeta / (||k||^2 + eps),
//   dk += -2 dbeta eta k / (||k||^2 + eps)^2.
//
// Kernels (after the forward chunk prefill of kla_ut.cu / kla_chunk_tc.cu run
// with its outputs off and its chain writing every h_n, fp32):
//   cbwd_prep_kernel     per chunk (two CTAs per SM): T, V', W and the two
//                        dH-independent terms of the chain, X = P^T dO and
//                        Y = (diag(gamma) Q)^T dO, into the workspace (fp32)
//   cbwd_adjoint_kernel  per head and 32-column slab, chunks in reverse:
//                        dV' = X + Kt dH, dH <- gamma_C dH + Y - W^T dV' (two
//                        products per chunk), dH in registers; the chunk
//                        operands arrive by asynchronous copies (double
//                        buffered, or single buffered at two CTAs per SM);
//                        writes dV'_n and dH_{n+1}
//   cbwd_grad_kernel     per chunk (16 warps): every gradient of the chunk's
//                        tokens, in three phases around one shared-memory plan
// Products are warp-level tensor-core MMAs (mma.sync m16n8k8, tf32 operands,
// fp32 sums); operands are read from shared memory through small accessors,
// so transposed or row-scaled operands need no extra copies.  Ragged tails
// are zero rows with g = 0 and beta = 0 (identity steps).
#include "kla_chunk.h"
#include "kla_common.cuh"

namespace kla {
namespace cbwd {

constexpr int C = 64;
constexpr int NT = 256;
constexpr int BVA = 32;  // state columns per adjoint-chain CTA

// An fp32 value rounded to a tf32 operand (to nearest; the tensor core would
// otherwise truncate, which measured three times the gradient error).
__device__ __forceinline__ uint32_t tf32(float x) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
  return r;
}

// d[nt] (16 x 8 tiles at rows m0.., columns n0 + 8 nt ..) += A (16 x K) B (K x 8):
// A(m, k) and B(k, n) are callables returning fp32.  Fragment element e of a
// tile: row m0 + g + 8 (e >> 1), column n0 + 8 nt + 2 t + (e & 1), with
// g = lane / 4, t = lane % 4.
template <int NTL, class FA, class FB>
__device__ __forceinline__ void mma_rows(float (&d)[NTL][4], const FA& A, const FB& B, int m0,
                                         int n0, int K, int lane) {
  const int g = lane >> 2, t = lane & 3;
#pragma unroll 4
  for (int k0 = 0; k0 < K; k0 += 8) {
    const uint32_t a0 = tf32(A(m0 + g, k0 + t)), a1 = tf32(A(m0 + g + 8, k0 + t));
    const uint32_t a2 = tf32(A(m0 + g, k0 + t + 4)), a3 = tf32(A(m0 + g + 8, k0 + t + 4));
#pragma unroll
    for (int nt = 0; nt < NTL; ++nt) {
      const uint32_t b0 = tf32(B(k0 + t, n0 + 8 * nt + g));
      const uint32_t b1 = tf32(B(k0 + t + 4, n0 + 8 * nt + g));
      asm volatile(
          "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0, %1, %2, %3}, "
          "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
          : "+f"(d[nt][0]), "+f"(d[nt][1]), "+f"(d[nt][2]), "+f"(d[nt][3])
          : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
    }
  }
}

template <int NTL>
__device__ __forceinline__ void zero(float (&d)[NTL][4]) {
#pragma unroll
  for (int i = 0; i < NTL; ++i) d[i][0] = d[i][1] = d[i][2] = d[i][3] = 0.f;
}

// Row / column of fragment element e.
__device__ __forceinline__ int frow(int m0, int lane, int e) { return m0 + (lane >> 2) + 8 * (e >> 1); }
__device__ __forceinline__ int fcol(int n0, int nt, int lane, int e) {
  return n0 + 8 * nt + 2 * (lane & 3) + (e & 1);
}

__device__ __forceinline__ float bf(const __nv_bfloat16& x) { return __bfloat162float(x); }

// Strides (elements) of the shared-memory tiles: fp32 rows padded by 4, bf16
// rows by 8, against bank conflicts of the fragment reads.
template <int D> constexpr int LF() { return D + 4; }
template <int D> constexpr int LB() { return D + 8; }

__device__ __forceinline__ void cp_async16(void* dst, const void* src, bool valid) {
  const uint32_t d = (uint32_t)__cvta_generic_to_shared(dst);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(d), "l"(src),
               "r"(valid ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async4(void* dst, const void* src, bool valid) {
  const uint32_t d = (uint32_t)__cvta_generic_to_shared(dst);
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(d), "l"(src),
               "r"(valid ? 4 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.wait_group 0;" ::: "memory");
}

// Asynchronous copy of n rows of a [rows][D] bf16 matrix with row stride rs
// (elements) into a padded tile (rows >= n zero-filled up to C); complete
// after cp_async_commit + cp_async_wait_all.
template <int D, int NTH = NT>
__device__ __forceinline__ void load_rows_bf16(__nv_bfloat16* dst, const __nv_bfloat16* src,
                                               size_t rs, int n) {
  constexpr int PR = D / 8;  // 16-byte pieces per row
  for (int p = threadIdx.x; p < C * PR; p += NTH) {
    const int r = p / PR, ch = p % PR;
    const bool ok = r < n;
    cp_async16(dst + r * LB<D>() + ch * 8, ok ? src + r * rs + ch * 8 : src, ok);
  }
}

// Asynchronous copy of a [R][D] fp32 block (row stride rs) into a padded tile.
template <int R, int D, int NTH = NT>
__device__ __forceinline__ void load_f32(float* dst, const float* src, size_t rs) {
  constexpr int PR = D / 4;
  for (int p = threadIdx.x; p < R * PR; p += NTH) {
    const int r = p / PR, ch = p % PR;
    cp_async16(dst + r * LF<D>() + ch * 4, src + r * rs + ch * 4, true);
  }
}

// Wait for this thread's copies, then for the whole CTA's.
__device__ __forceinline__ void copies_landed() {
  cp_async_commit();
  cp_async_wait_all();
  __syncthreads();
}

// Per-chunk scalars: G (in-chunk cumsum of g), gamma = e^G, beta, ||k||^2,
// from the staged keys (rows >= n: g = 0, beta = 0).  Decay ratios are only
// ever formed as e^{difference} (gamma_C / gamma_r as e^{G_last - G_r}): with
// strong gates e^G itself underflows to 0 inside a chunk.
template <int DK, int NTH = NT>
__device__ __forceinline__ void chunk_scalars(float* G, float* gam, float* beta, float* n2,
                                              const __nv_bfloat16* kb, const float* g,
                                              const float* eta, float eps, size_t tok0,
                                              size_t tstride, int n) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int r = warp; r < C; r += NTH / 32) {
    float a = 0.f;
    for (int i = lane; i < DK; i += 32) {
      const float x = bf(kb[r * LB<DK>() + i]);
      a = fmaf(x, x, a);
    }
    a = warp_sum(a);
    if (lane == 0) {
      n2[r] = a;
      beta[r] = r < n ? step_size(eta[tok0 + r * tstride], a, eps) : 0.f;
    }
  }
  if (warp == 0) {  // inclusive cumsum of the 64 gates: two per lane
    float x0 = 2 * lane < n ? g[tok0 + (2 * lane) * tstride] : 0.f;
    float x1 = 2 * lane + 1 < n ? g[tok0 + (2 * lane + 1) * tstride] : 0.f;
    float s = x0 + x1;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const float y = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += y;
    }
    const float base = s - (x0 + x1);
    G[2 * lane] = base + x0;
    G[2 * lane + 1] = s;
    gam[2 * lane] = __expf(base + x0);
    gam[2 * lane + 1] = __expf(s);
  }
}

// T = (I + A)^{-1} for the strictly lower A (fp32 [C][LF<C>]) by forward
// substitution, four threads per column (column tid / 4); writes Tm.
__device__ __forceinline__ void unit_lower_inverse(float* Tm, const float* A) {
  const int c = threadIdx.x >> 2, l = threadIdx.x & 3;
  float tc[C / 4];  // T[4 j + l][c]
#pragma unroll
  for (int j = 0; j < C / 4; ++j) tc[j] = 0.f;
#pragma unroll
  for (int r = 0; r < C; ++r) {
    float p = 0.f;
#pragma unroll
    for (int j = 0; j < C / 4; ++j) p = fmaf(A[r * LF<C>() + 4 * j + l], tc[j], p);
    p += __shfl_xor_sync(0xffffffffu, p, 1);
    p += __shfl_xor_sync(0xffffffffu, p, 2);
    const float val = r < c ? 0.f : (r == c ? 1.f : -p);
    if (l == (r & 3)) tc[r >> 2] = val;
  }
#pragma unroll
  for (int j = 0; j < C / 4; ++j) Tm[(4 * j + l) * LF<C>() + c] = tc[j];
}

}  // namespace cbwd

using namespace cbwd;

// ---------------------------------------------------------------- prep
// Two CTAs per SM: the shared-memory plan follows the lifetimes.  The start
// state h_n passes through in 64-row pieces, only to form K h_n (kept in
// registers), so V' = T (diag(beta) V - diag(beta gamma) K h_n) needs neither
// W nor h_n as a tile (W = T diag(beta gamma) K, so W h_n is the same
// product reassociated); the right operand Z of that last product takes the
// place of the queries and dL/do once X and Y are formed.
constexpr int HR = 64;  // rows of h_n staged at a time

template <int DK, int DV>
struct PrepSmem {
  __nv_bfloat16 kb[C][LB<DK>()];
  __nv_bfloat16 vb[C][LB<DV>()];
  union {
    struct {
      __nv_bfloat16 qb[C][LB<DK>()];
      __nv_bfloat16 ob[C][LB<DV>()];
    } in;
    float Z[C][LF<DV>()];  // diag(beta) V - diag(beta gamma) K h_n
  } qo;
  union {
    float h[HR][LF<DV>()];  // rows of h_n
    struct {
      float A[C][LF<C>()];  // A, then P
      float Tm[C][LF<C>()];
    } at;
  } u;
  float G[C], gam[C], beta[C], n2[C];
};

// Per chunk: T, V' = T diag(beta) V - W h_n, W, X = P^T dO and
// Y = (diag(gamma) Q)^T dO into the workspace.
template <int DK, int DV>
__global__ void __launch_bounds__(NT, 2)
cbwd_prep_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
                 const __nv_bfloat16* __restrict__ v, const __nv_bfloat16* __restrict__ dout,
                 const float* __restrict__ g, const float* __restrict__ eta, float eps,
                 const float* __restrict__ ck, float* __restrict__ Tws, float* __restrict__ Vws,
                 float* __restrict__ Wws, float* __restrict__ Xws, float* __restrict__ Yws,
                 int Tlen, int H, int nblk) {
  using Smem = PrepSmem<DK, DV>;
  static_assert(sizeof(Smem::qo.Z) <= sizeof(Smem::qo.in), "Z over the queries and dL/do");
  static_assert(sizeof(Smem::u.h) <= sizeof(Smem::u.at), "h_n rows over A and T");
  extern __shared__ __align__(16) unsigned char smem_raw[];
  auto& s = *reinterpret_cast<Smem*>(smem_raw);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int n = blockIdx.x, hh = blockIdx.y, b = blockIdx.z;
  const size_t head = (size_t)b * H + hh, chunk = head * nblk + n;
  const int t0 = n * C, len = min(C, Tlen - t0);
  const size_t tok0 = ((size_t)b * Tlen + t0) * H + hh;
  const float* hsrc = ck + chunk * DK * DV;

  load_rows_bf16<DK>(&s.kb[0][0], k + tok0 * DK, (size_t)H * DK, len);
  load_rows_bf16<DV>(&s.vb[0][0], v + tok0 * DV, (size_t)H * DV, len);
  load_rows_bf16<DK>(&s.qo.in.qb[0][0], q + tok0 * DK, (size_t)H * DK, len);
  load_rows_bf16<DV>(&s.qo.in.ob[0][0], dout + tok0 * DV, (size_t)H * DV, len);
  load_f32<HR, DV>(&s.u.h[0][0], hsrc, DV);
  copies_landed();
  chunk_scalars<DK>(s.G, s.gam, s.beta, s.n2, &s.kb[0][0], g, eta, eps, tok0, H, len);

  const int mt = warp & 3, nh = warp >> 2;  // m-tile of 16 rows; column half
  // K h_n: rows 16 mt.., columns (DV / 2) nh.. of this warp, by HR-row pieces
  float kh[DV / 16][4];
  zero(kh);
#pragma unroll 1
  for (int i0 = 0; i0 < DK; i0 += HR) {
    if (i0 > 0) {
      __syncthreads();  // every warp is done with the previous piece
      load_f32<HR, DV>(&s.u.h[0][0], hsrc + (size_t)i0 * DV, DV);
      copies_landed();
    }
    auto Ka = [&](int r, int i) { return bf(s.kb[r][i0 + i]); };
    auto Hb = [&](int i, int j) { return s.u.h[i][j]; };
    mma_rows<DV / 16>(kh, Ka, Hb, 16 * mt, (DV / 2) * nh, HR, lane);
  }
  __syncthreads();  // h_n read (A and T take its place); the scalars are in

  {  // A = beta_r (k_r . k_s) Gamma_rs, s < r
    float d[4][4];
    zero(d);
    auto Ka = [&](int r, int i) { return bf(s.kb[r][i]); };
    auto Kb = [&](int i, int c) { return bf(s.kb[c][i]); };
    mma_rows<4>(d, Ka, Kb, 16 * mt, 32 * nh, DK, lane);
#pragma unroll
    for (int nt = 0; nt < 4; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int r = frow(16 * mt, lane, e), c = fcol(32 * nh, nt, lane, e);
        s.u.at.A[r][c] = c < r ? s.beta[r] * d[nt][e] * __expf(s.G[r] - s.G[c]) : 0.f;
      }
  }
  __syncthreads();
  unit_lower_inverse(&s.u.at.Tm[0][0], &s.u.at.A[0][0]);
  __syncthreads();
  {  // W = T diag(beta gamma) K (to the workspace only)
    float d[DK / 16][4];
    zero(d);
    auto Ta = [&](int r, int c) { return s.u.at.Tm[r][c]; };
    auto Kb = [&](int c, int i) { return s.beta[c] * s.gam[c] * bf(s.kb[c][i]); };
    mma_rows<DK / 16>(d, Ta, Kb, 16 * mt, (DK / 2) * nh, C, lane);
    float* wdst = Wws + chunk * C * DK;
#pragma unroll
    for (int nt = 0; nt < DK / 16; ++nt)
#pragma unroll
      for (int e = 0; e < 4; e += 2) {
        const int r = frow(16 * mt, lane, e), i = fcol((DK / 2) * nh, nt, lane, e);
        *reinterpret_cast<float2*>(wdst + r * DK + i) = make_float2(d[nt][e], d[nt][e + 1]);
      }
  }
  {  // P = lower_incl(Q K^T (*) Gamma) over A (no longer read after the inverse)
    float p[4][4];
    zero(p);
    auto Qa = [&](int r, int i) { return bf(s.qo.in.qb[r][i]); };
    auto Kb = [&](int i, int c) { return bf(s.kb[c][i]); };
    mma_rows<4>(p, Qa, Kb, 16 * mt, 32 * nh, DK, lane);
#pragma unroll
    for (int nt = 0; nt < 4; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int r = frow(16 * mt, lane, e), c = fcol(32 * nh, nt, lane, e);
        s.u.at.A[r][c] = c <= r ? p[nt][e] * __expf(s.G[r] - s.G[c]) : 0.f;
      }
  }
  __syncthreads();
  {  // Y = (diag(gamma) Q)^T dO  [DK x DV]: DK / 16 row tiles; with 8 row tiles
     // warp w takes row tile w and both column halves, with 4 it takes row
     // tile w % 4 and column half w / 4
    constexpr int RT = DK / 16;
    auto QTa = [&](int i, int c) { return s.gam[c] * bf(s.qo.in.qb[c][i]); };
    auto Ob = [&](int c, int j) { return bf(s.qo.in.ob[c][j]); };
    float* ydst = Yws + chunk * DK * DV;
    const int ym = warp % RT;
    for (int half = RT == 8 ? 0 : warp / RT; half < 2; half += RT == 8 ? 1 : 2) {
      float d[DV / 16][4];
      zero(d);
      mma_rows<DV / 16>(d, QTa, Ob, 16 * ym, half * (DV / 2), C, lane);
#pragma unroll
      for (int nt = 0; nt < DV / 16; ++nt)
#pragma unroll
        for (int e = 0; e < 4; e += 2) {
          const int i = frow(16 * ym, lane, e), j = fcol(half * (DV / 2), nt, lane, e);
          *reinterpret_cast<float2*>(ydst + i * DV + j) = make_float2(d[nt][e], d[nt][e + 1]);
        }
    }
  }
  {  // X = P^T dO  [C x DV]
    float d[DV / 16][4];
    zero(d);
    auto PTa = [&](int r, int c) { return s.u.at.A[c][r]; };
    auto Ob = [&](int c, int j) { return bf(s.qo.in.ob[c][j]); };
    mma_rows<DV / 16>(d, PTa, Ob, 16 * mt, (DV / 2) * nh, C, lane);
    float* xdst = Xws + chunk * C * DV;
#pragma unroll
    for (int nt = 0; nt < DV / 16; ++nt)
#pragma unroll
      for (int e = 0; e < 4; e += 2) {
        const int r = frow(16 * mt, lane, e), j = fcol((DV / 2) * nh, nt, lane, e);
        *reinterpret_cast<float2*>(xdst + r * DV + j) = make_float2(d[nt][e], d[nt][e + 1]);
      }
  }
  __syncthreads();  // the queries and dL/do are read: Z takes their place
#pragma unroll
  for (int nt = 0; nt < DV / 16; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int r = frow(16 * mt, lane, e), j = fcol((DV / 2) * nh, nt, lane, e);
      s.qo.Z[r][j] = s.beta[r] * (bf(s.vb[r][j]) - s.gam[r] * kh[nt][e]);
    }
  __syncthreads();
  {  // V' = T Z
    float d[DV / 16][4];
    zero(d);
    auto Ta = [&](int r, int c) { return s.u.at.Tm[r][c]; };
    auto Zb = [&](int c, int j) { return s.qo.Z[c][j]; };
    mma_rows<DV / 16>(d, Ta, Zb, 16 * mt, (DV / 2) * nh, C, lane);
    float* dst = Vws + chunk * C * DV;
#pragma unroll
    for (int nt = 0; nt < DV / 16; ++nt)
#pragma unroll
      for (int e = 0; e < 4; e += 2) {
        const int r = frow(16 * mt, lane, e), j = fcol((DV / 2) * nh, nt, lane, e);
        *reinterpret_cast<float2*>(dst + r * DV + j) = make_float2(d[nt][e], d[nt][e + 1]);
      }
  }
  {
    float* dst = Tws + chunk * C * C;
    for (int p = tid; p < C * C; p += NT) dst[p] = s.u.at.Tm[p / C][p % C];
  }
}

// ---------------------------------------------------------------- adjoint chain
// One chunk's operands of the adjoint chain (the CTA's 32 columns of X, Y).
template <int DK>
struct AdjBuf {
  __nv_bfloat16 kb[C][LB<DK>()];
  float W[C][LF<DK>()];
  float X[C][LF<BVA>()];
  float Y[DK][LF<BVA>()];
  float g[C];
};

template <int DK, int NBUF>
struct AdjSmem {
  AdjBuf<DK> buf[NBUF];
  float dH[DK][LF<BVA>()];
  float dV[C][LF<BVA>()];
  float kts[C];
  float gC;
};

// Copies of chunk n's operands into a buffer (zero rows past the sequence).
template <int DK, int DV>
__device__ __forceinline__ void adj_fetch(AdjBuf<DK>& d, const __nv_bfloat16* k,
                                          const float* g, const float* Wws, const float* Xws,
                                          const float* Yws, size_t head, int n, int nblk,
                                          int j0, int b, int hh, int Tlen, int H) {
  const size_t chunk = head * nblk + n;
  const int t0 = n * C, len = min(C, Tlen - t0);
  const size_t tok0 = ((size_t)b * Tlen + t0) * H + hh;
  for (int p = threadIdx.x; p < C * (DK / 8); p += NT) {  // keys, bf16
    const int r = p / (DK / 8), ch = p % (DK / 8);
    const bool ok = r < len;
    cp_async16(&d.kb[r][ch * 8], k + (ok ? (tok0 + (size_t)r * H) * DK + ch * 8 : 0), ok);
  }
  for (int p = threadIdx.x; p < C * (DK / 4); p += NT) {  // W
    const int r = p / (DK / 4), ch = p % (DK / 4);
    cp_async16(&d.W[r][ch * 4], Wws + (chunk * C + r) * DK + ch * 4, true);
  }
  for (int p = threadIdx.x; p < C * (BVA / 4); p += NT) {  // X columns j0 ..
    const int r = p / (BVA / 4), ch = p % (BVA / 4);
    cp_async16(&d.X[r][ch * 4], Xws + (chunk * C + r) * DV + j0 + ch * 4, true);
  }
  for (int p = threadIdx.x; p < DK * (BVA / 4); p += NT) {  // Y columns j0 ..
    const int r = p / (BVA / 4), ch = p % (BVA / 4);
    cp_async16(&d.Y[r][ch * 4], Yws + (chunk * DK + r) * DV + j0 + ch * 4, true);
  }
  if (threadIdx.x < C) {
    const bool ok = (int)threadIdx.x < len;
    cp_async4(&d.g[threadIdx.x], g + (ok ? tok0 + (size_t)threadIdx.x * H : 0), ok);
  }
  cp_async_commit();
}

// One CTA per (head, 32-column slab); chunks in reverse.  dH (the adjoint of
// h_{n+1}) lives in registers.  NBUF = 2: the next chunk's operands are
// copied in while the current one is worked on (for few CTAs, one per SM);
// NBUF = 1: one buffer, small enough for two CTAs per SM, whose work hides
// each other's copies (for many CTAs).
template <int DK, int DV, int NBUF>
__global__ void __launch_bounds__(NT)
cbwd_adjoint_kernel(const __nv_bfloat16* __restrict__ k, const float* __restrict__ g,
                    const float* __restrict__ dhT, const float* __restrict__ Wws,
                    const float* __restrict__ Xws, const float* __restrict__ Yws,
                    float* __restrict__ dVws, float* __restrict__ dHws, float* __restrict__ dh0,
                    int Tlen, int H, int nblk) {
  // the dH slab [DK x 32] in 16-row tiles: DK / 16 of them, NT / 32 / (DK / 16)
  // warps per tile splitting its columns
  constexpr int RT = DK / 16, WPT = (NT / 32) / RT, NTH = (BVA / 8) / WPT;
  static_assert(RT * WPT == NT / 32 && NTH >= 1, "state tiling");
  extern __shared__ __align__(16) unsigned char smem_raw[];
  auto& s = *reinterpret_cast<AdjSmem<DK, NBUF>*>(smem_raw);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int slab = blockIdx.x, hh = blockIdx.y, b = blockIdx.z;
  const int j0 = slab * BVA;
  const size_t head = (size_t)b * H + hh;
  const int hm0 = 16 * (warp % RT), hn0 = (BVA / WPT) * (warp / RT);  // this warp's dH tile

  float acc[NTH][4];  // dH rows hm0 .., columns j0 + hn0 ..
#pragma unroll
  for (int nt = 0; nt < NTH; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e)
      acc[nt][e] = dhT ? dhT[(head * DK + frow(hm0, lane, e)) * DV + j0 +
                             fcol(hn0, nt, lane, e)]
                       : 0.f;
  if constexpr (NBUF == 2)
    adj_fetch<DK, DV>(s.buf[(nblk - 1) & 1], k, g, Wws, Xws, Yws, head, nblk - 1, nblk, j0, b,
                      hh, Tlen, H);

  for (int n = nblk - 1; n >= 0; --n) {
    const size_t chunk = head * nblk + n;
    AdjBuf<DK>& cur = s.buf[NBUF == 2 ? (n & 1) : 0];
    if constexpr (NBUF == 1) {
      __syncthreads();  // the previous chunk is done with the buffer
      adj_fetch<DK, DV>(cur, k, g, Wws, Xws, Yws, head, n, nblk, j0, b, hh, Tlen, H);
    }
    cp_async_wait_all();
    __syncthreads();  // chunk n's operands are in; the previous chunk is done
    if constexpr (NBUF == 2)
      if (n > 0)
        adj_fetch<DK, DV>(s.buf[(n - 1) & 1], k, g, Wws, Xws, Yws, head, n - 1, nblk, j0, b,
                          hh, Tlen, H);
    // dH_{n+1}: to shared memory (operand) and to the workspace
#pragma unroll
    for (int nt = 0; nt < NTH; ++nt)
#pragma unroll
      for (int e = 0; e < 4; e += 2) {
        const int r = frow(hm0, lane, e), c = fcol(hn0, nt, lane, e);
        s.dH[r][c] = acc[nt][e];
        s.dH[r][c + 1] = acc[nt][e + 1];
        *reinterpret_cast<float2*>(dHws + (chunk * DK + r) * DV + j0 + c) =
            make_float2(acc[nt][e], acc[nt][e + 1]);
      }
    if (warp == 0) {  // G (in-chunk cumsum) -> e^{G_last - G_r}, e^{G_last}
      const float x0 = cur.g[2 * lane], x1 = cur.g[2 * lane + 1];
      float sum = x0 + x1;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const float y = __shfl_up_sync(0xffffffffu, sum, o);
        if (lane >= o) sum += y;
      }
      const float last = __shfl_sync(0xffffffffu, sum, 31);
      s.kts[2 * lane] = __expf(last - (sum - x1));
      s.kts[2 * lane + 1] = __expf(last - sum);
      if (lane == 0) s.gC = __expf(last);
    }
    __syncthreads();
    const int mt = warp & 3, nq = warp >> 2;
    {  // dV' = X + Kt dH_{n+1}   [C x 32]: warp (mt, nq) has 2 column tiles
      float d[2][4];
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e)
          d[nt][e] = cur.X[frow(16 * mt, lane, e)][fcol(16 * nq, nt, lane, e)];
      auto Kta = [&](int r, int i) { return s.kts[r] * bf(cur.kb[r][i]); };
      auto Hb = [&](int i, int j) { return s.dH[i][j]; };
      mma_rows<2>(d, Kta, Hb, 16 * mt, 16 * nq, DK, lane);
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 4; e += 2) {
          const int r = frow(16 * mt, lane, e), c = fcol(16 * nq, nt, lane, e);
          s.dV[r][c] = d[nt][e];
          s.dV[r][c + 1] = d[nt][e + 1];
          *reinterpret_cast<float2*>(dVws + (chunk * C + r) * DV + j0 + c) =
              make_float2(d[nt][e], d[nt][e + 1]);
        }
    }
    __syncthreads();
    {  // dH_n = gamma_C dH_{n+1} + Y - W^T dV'
      const float gC = s.gC;
#pragma unroll
      for (int nt = 0; nt < NTH; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e)
          acc[nt][e] = fmaf(gC, acc[nt][e], cur.Y[frow(hm0, lane, e)][fcol(hn0, nt, lane, e)]);
      auto WTa = [&](int i, int c) { return -cur.W[c][i]; };
      auto dVb = [&](int c, int j) { return s.dV[c][j]; };
      mma_rows<NTH>(acc, WTa, dVb, hm0, hn0, C, lane);
    }
  }
  if (dh0) {
#pragma unroll
    for (int nt = 0; nt < NTH; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e)
        dh0[(head * DK + frow(hm0, lane, e)) * DV + j0 + fcol(hn0, nt, lane, e)] = acc[nt][e];
  }
}

// ---------------------------------------------------------------- gradients
template <int DK, int DV>
struct GradSmem {
  __nv_bfloat16 qb[C][LB<DK>()];
  __nv_bfloat16 kb[C][LB<DK>()];
  __nv_bfloat16 vb[C][LB<DV>()];
  __nv_bfloat16 ob[C][LB<DV>()];
  float Tm[C][LF<C>()];
  float Vp[C][LF<DV>()];   // V'
  float dVp[C][LF<DV>()];  // dV'
  // a column half of h_n or dH ([DK][LF<DV/2>]), or dW ([C][LF<DK>])
  float big[(DK * LF<DV / 2>() > C * LF<DK>()) ? DK * LF<DV / 2>() : C * LF<DK>()];
  float X1[C][LF<C>()];
  float X2[C][LF<C>()];
  float G[C], gam[C], beta[C], n2[C], kts[C];
  float dG[C], dB[C];
  float part[4][C];  // per-row partial sums of the four warps sharing a row tile
  float red[16];
};

// Sum a per-row value over the 4 lanes holding one fragment row (t), then the
// two warps (nh) sharing the row tile, into dst[row] in a fixed order.
__device__ __forceinline__ float quad_sum(float x) {
  x += __shfl_xor_sync(0xffffffffu, x, 1);
  x += __shfl_xor_sync(0xffffffffu, x, 2);
  return x;
}

constexpr int GT = 512;  // threads of the gradient kernel: 16 warps, 4 per row tile

template <int DK, int DV>
__global__ void __launch_bounds__(GT)
cbwd_grad_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
                 const __nv_bfloat16* __restrict__ v, const __nv_bfloat16* __restrict__ dout,
                 const float* __restrict__ g, const float* __restrict__ eta, float eps,
                 const float* __restrict__ ck, const float* __restrict__ Tws,
                 const float* __restrict__ Vws, const float* __restrict__ dVws,
                 const float* __restrict__ dHws, float* __restrict__ dq, float* __restrict__ dk,
                 float* __restrict__ dv, float* __restrict__ dg, float* __restrict__ deta,
                 int Tlen, int H, int nblk) {
  static_assert(DK == DV, "square heads");
  extern __shared__ __align__(16) unsigned char smem_raw[];
  auto& s = *reinterpret_cast<GradSmem<DK, DV>*>(smem_raw);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int n = blockIdx.x, hh = blockIdx.y, b = blockIdx.z;
  const size_t head = (size_t)b * H + hh, chunk = head * nblk + n;
  const int t0 = n * C, len = min(C, Tlen - t0);
  const size_t tok0 = ((size_t)b * Tlen + t0) * H + hh;
  const int mt = warp & 3, nq = warp >> 2;  // row tile; column quarter
  constexpr int HALF = DV / 2;
  const float* hn = ck + chunk * DK * DV;
  const float* dHn = dHws + chunk * DK * DV;

  load_rows_bf16<DK, GT>(&s.qb[0][0], q + tok0 * DK, (size_t)H * DK, len);
  load_rows_bf16<DK, GT>(&s.kb[0][0], k + tok0 * DK, (size_t)H * DK, len);
  load_rows_bf16<DV, GT>(&s.vb[0][0], v + tok0 * DV, (size_t)H * DV, len);
  load_rows_bf16<DV, GT>(&s.ob[0][0], dout + tok0 * DV, (size_t)H * DV, len);
  load_f32<C, C, GT>(&s.Tm[0][0], Tws + chunk * C * C, C);
  load_f32<C, DV, GT>(&s.Vp[0][0], Vws + chunk * C * DV, DV);
  load_f32<C, DV, GT>(&s.dVp[0][0], dVws + chunk * C * DV, DV);
  if (tid < C) s.dG[tid] = s.dB[tid] = 0.f;
  copies_landed();
  chunk_scalars<DK, GT>(s.G, s.gam, s.beta, s.n2, &s.kb[0][0], g, eta, eps, tok0, H, len);
  __syncthreads();
  if (tid < C) s.kts[tid] = __expf(s.G[C - 1] - s.G[tid]);
  const float gC = s.gam[C - 1];

  // ---- phase 1: products with h_n, one 64-column half of it at a time
  float accQ[DK / 32][4], accW[DK / 32][4];  // rows 16 mt .., columns (DK/4) nq ..
  zero(accQ);
  zero(accW);
  float rowO[2] = {0.f, 0.f};  // rowdot(dO, diag(gamma) Q h_n) for rows g, g + 8
  for (int half = 0; half < 2; ++half) {
    __syncthreads();
    load_f32<DK, HALF, GT>(s.big, hn + half * HALF, DV);
    copies_landed();
    // dO h_n^T and -dV' h_n^T over this half of the dv index
    auto Oa = [&](int r, int j) { return bf(s.ob[r][half * HALF + j]); };
    auto dVa = [&](int r, int j) { return -s.dVp[r][half * HALF + j]; };
    auto HTb = [&](int j, int i) { return s.big[i * LF<HALF>() + j]; };
    mma_rows<DK / 32>(accQ, Oa, HTb, 16 * mt, (DK / 4) * nq, HALF, lane);
    mma_rows<DK / 32>(accW, dVa, HTb, 16 * mt, (DK / 4) * nq, HALF, lane);
    // diag(gamma) Q h_n on this half's columns: [C x HALF], a quarter per warp
    constexpr int OQ = HALF / 4, NTO = OQ / 8;
    float o[NTO][4];
    zero(o);
    auto Qa = [&](int r, int i) { return s.gam[r] * bf(s.qb[r][i]); };
    auto Hb = [&](int i, int j) { return s.big[i * LF<HALF>() + j]; };
    mma_rows<NTO>(o, Qa, Hb, 16 * mt, OQ * nq, DK, lane);
#pragma unroll
    for (int nt = 0; nt < NTO; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e)
        rowO[e >> 1] += o[nt][e] * bf(s.ob[frow(16 * mt, lane, e)]
                                          [half * HALF + fcol(OQ * nq, nt, lane, e)]);
  }
  // <dH_{n+1}, h_n> (block sum, fixed order; every load issued up front)
  float hd = 0.f;
  {
    constexpr int NV = DK * DV / 4 / GT;  // float4 pieces per thread
    float4 a[NV], c[NV];
#pragma unroll
    for (int u = 0; u < NV; ++u) {
      a[u] = reinterpret_cast<const float4*>(hn)[tid + u * GT];
      c[u] = reinterpret_cast<const float4*>(dHn)[tid + u * GT];
    }
#pragma unroll
    for (int u = 0; u < NV; ++u)
      hd = fmaf(a[u].x, c[u].x, fmaf(a[u].y, c[u].y, fmaf(a[u].z, c[u].z, fmaf(a[u].w, c[u].w, hd))));
  }
  hd = warp_sum(hd);
  if (lane == 0) s.red[warp] = hd;
  // rowO -> dG (four warps per row tile, warp quarter nq writes part[nq])
#pragma unroll
  for (int hr = 0; hr < 2; ++hr) {
    const float x = quad_sum(rowO[hr]);
    if ((lane & 3) == 0) s.part[nq][16 * mt + (lane >> 2) + 8 * hr] = x;
  }
  __syncthreads();
  if (tid < C) s.dG[tid] += s.part[0][tid] + s.part[1][tid] + s.part[2][tid] + s.part[3][tid];
  // dq (first part) stays in accQ; dW -> big as [C][DK]
  float* dW = s.big;  // [C][LF<DK>]
#pragma unroll
  for (int nt = 0; nt < DK / 32; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e)
      dW[frow(16 * mt, lane, e) * LF<DK>() + fcol((DK / 4) * nq, nt, lane, e)] = accW[nt][e];

  // ---- phase 2: the C x C quantities
  {  // dP = dO V'^T (*) incl -> X1;  Q K^T -> X2
    float d[2][4], p[2][4];
    zero(d);
    zero(p);
    auto Oa = [&](int r, int j) { return bf(s.ob[r][j]); };
    auto VTb = [&](int j, int c) { return s.Vp[c][j]; };
    mma_rows<2>(d, Oa, VTb, 16 * mt, 16 * nq, DV, lane);
    auto Qa = [&](int r, int i) { return bf(s.qb[r][i]); };
    auto KTb = [&](int i, int c) { return bf(s.kb[c][i]); };
    mma_rows<2>(p, Qa, KTb, 16 * mt, 16 * nq, DK, lane);
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int r = frow(16 * mt, lane, e), c = fcol(16 * nq, nt, lane, e);
        const bool in = c <= r;
        s.X1[r][c] = in ? d[nt][e] : 0.f;
        s.X2[r][c] = in ? p[nt][e] * __expf(s.G[r] - s.G[c]) : 0.f;  // P
      }
  }
  __syncthreads();
  // F = dP (*) P: dG_r += rowsum, dG_s -= colsum (four threads per row);
  // X1 <- dP (*) Gamma
  if (tid < 4 * C) {
    const int r = tid >> 2, c0 = 16 * (tid & 3);
    float rs = 0.f, cs = 0.f;
#pragma unroll 4
    for (int c = c0; c < c0 + 16; ++c) {
      rs = fmaf(s.X1[r][c], s.X2[r][c], rs);
      cs = fmaf(s.X1[c][r], s.X2[c][r], cs);
    }
    rs = quad_sum(rs);
    cs = quad_sum(cs);
    if ((tid & 3) == 0) s.dG[r] += rs - cs;
  }
  __syncthreads();
  for (int p = tid; p < C * C; p += GT) {
    const int r = p / C, c = p % C;
    if (c <= r) s.X1[r][c] *= __expf(s.G[r] - s.G[c]);
  }
  __syncthreads();
  float accK[DK / 32][4];
  zero(accK);
  {  // dQ += (dP (*) Gamma) K -> dq;  dK = (dP (*) Gamma)^T Q
    auto Xa = [&](int r, int c) { return s.X1[r][c]; };
    auto Kb = [&](int c, int i) { return bf(s.kb[c][i]); };
#pragma unroll
    for (int nt = 0; nt < DK / 32; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) accQ[nt][e] *= s.gam[frow(16 * mt, lane, e)];
    mma_rows<DK / 32>(accQ, Xa, Kb, 16 * mt, (DK / 4) * nq, C, lane);
    auto XTa = [&](int r, int c) { return s.X1[c][r]; };
    auto Qb = [&](int c, int i) { return bf(s.qb[c][i]); };
    mma_rows<DK / 32>(accK, XTa, Qb, 16 * mt, (DK / 4) * nq, C, lane);
#pragma unroll
    for (int nt = 0; nt < DK / 32; ++nt)
#pragma unroll
      for (int e = 0; e < 4; e += 2) {
        const int r = frow(16 * mt, lane, e), i = fcol((DK / 4) * nq, nt, lane, e);
        if (r < len)
          *reinterpret_cast<float2*>(dq + (tok0 + (size_t)r * H) * DK + i) =
              make_float2(accQ[nt][e], accQ[nt][e + 1]);
      }
  }
  {  // T^T dW: dK += diag(beta gamma) T^T dW;  dbeta, dG += rowdot(T^T dW, K) terms
    float d[DK / 32][4];
    zero(d);
    auto TTa = [&](int r, int c) { return s.Tm[c][r]; };
    auto dWb = [&](int c, int i) { return dW[c * LF<DK>() + i]; };
    mma_rows<DK / 32>(d, TTa, dWb, 16 * mt, (DK / 4) * nq, C, lane);
    float rk[2] = {0.f, 0.f};
#pragma unroll
    for (int nt = 0; nt < DK / 32; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int r = frow(16 * mt, lane, e), i = fcol((DK / 4) * nq, nt, lane, e);
        accK[nt][e] = fmaf(s.beta[r] * s.gam[r], d[nt][e], accK[nt][e]);
        rk[e >> 1] = fmaf(d[nt][e], bf(s.kb[r][i]), rk[e >> 1]);
      }
#pragma unroll
    for (int hr = 0; hr < 2; ++hr) {
      const float x = quad_sum(rk[hr]);
      if ((lane & 3) == 0) s.part[nq][16 * mt + (lane >> 2) + 8 * hr] = x;
    }
  }
  __syncthreads();
  if (tid < C) {
    const float x = s.part[0][tid] + s.part[1][tid] + s.part[2][tid] + s.part[3][tid];
    s.dB[tid] += s.gam[tid] * x;
    s.dG[tid] += s.beta[tid] * s.gam[tid] * x;
  }
  __syncthreads();
  {  // T^T dV': dv = diag(beta) T^T dV';  dbeta += rowdot(T^T dV', V)
    float d[DV / 32][4];
    zero(d);
    auto TTa = [&](int r, int c) { return s.Tm[c][r]; };
    auto dVb = [&](int c, int j) { return s.dVp[c][j]; };
    mma_rows<DV / 32>(d, TTa, dVb, 16 * mt, (DV / 4) * nq, C, lane);
    float rv[2] = {0.f, 0.f};
#pragma unroll
    for (int nt = 0; nt < DV / 32; ++nt)
#pragma unroll
      for (int e = 0; e < 4; e += 2) {
        const int r = frow(16 * mt, lane, e), j = fcol((DV / 4) * nq, nt, lane, e);
        rv[e >> 1] = fmaf(d[nt][e], bf(s.vb[r][j]), rv[e >> 1]);
        rv[e >> 1] = fmaf(d[nt][e + 1], bf(s.vb[r][j + 1]), rv[e >> 1]);
        if (r < len)
          *reinterpret_cast<float2*>(dv + (tok0 + (size_t)r * H) * DV + j) =
              make_float2(s.beta[r] * d[nt][e], s.beta[r] * d[nt][e + 1]);
      }
#pragma unroll
    for (int hr = 0; hr < 2; ++hr) {
      const float x = quad_sum(rv[hr]);
      if ((lane & 3) == 0) s.part[nq][16 * mt + (lane >> 2) + 8 * hr] = x;
    }
  }
  __syncthreads();
  if (tid < C) s.dB[tid] += s.part[0][tid] + s.part[1][tid] + s.part[2][tid] + s.part[3][tid];
  {  // dT = dW (diag(beta gamma) K)^T + dV' (diag(beta) V)^T -> X2 (P is done)
    float d[2][4];
    zero(d);
    auto dWa = [&](int r, int i) { return dW[r * LF<DK>() + i]; };
    auto KTb = [&](int i, int c) { return s.beta[c] * s.gam[c] * bf(s.kb[c][i]); };
    mma_rows<2>(d, dWa, KTb, 16 * mt, 16 * nq, DK, lane);
    auto dVa = [&](int r, int j) { return s.dVp[r][j]; };
    auto VTb = [&](int j, int c) { return s.beta[c] * bf(s.vb[c][j]); };
    mma_rows<2>(d, dVa, VTb, 16 * mt, 16 * nq, DV, lane);
    __syncthreads();  // every warp is done reading X2 (P) and X1 (dP Gamma)
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) s.X2[frow(16 * mt, lane, e)][fcol(16 * nq, nt, lane, e)] = d[nt][e];
  }
  __syncthreads();
  {  // Y = T^T dT -> X1
    float d[2][4];
    zero(d);
    auto TTa = [&](int r, int c) { return s.Tm[c][r]; };
    auto Xb = [&](int c, int j) { return s.X2[c][j]; };
    mma_rows<2>(d, TTa, Xb, 16 * mt, 16 * nq, C, lane);
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) s.X1[frow(16 * mt, lane, e)][fcol(16 * nq, nt, lane, e)] = d[nt][e];
  }
  __syncthreads();
  {  // dA = -strict_lower(Y T^T) -> X2;  K K^T kept in registers
    float d[2][4], kk[2][4];
    zero(d);
    zero(kk);
    auto Ya = [&](int r, int c) { return s.X1[r][c]; };
    auto TTb = [&](int c, int j) { return s.Tm[j][c]; };
    mma_rows<2>(d, Ya, TTb, 16 * mt, 16 * nq, C, lane);
    auto Ka = [&](int r, int i) { return bf(s.kb[r][i]); };
    auto KTb = [&](int i, int c) { return bf(s.kb[c][i]); };
    mma_rows<2>(kk, Ka, KTb, 16 * mt, 16 * nq, DK, lane);
    __syncthreads();  // X2 (dT) fully read
    // E = dA (*) Gamma -> X2;  F = dA (*) A -> X1 (A = beta_r KK Gamma);
    // dbeta_r += sum_s E_rs KK_rs
    float rb[2] = {0.f, 0.f};
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int r = frow(16 * mt, lane, e), c = fcol(16 * nq, nt, lane, e);
        const float E = c < r ? -d[nt][e] * __expf(s.G[r] - s.G[c]) : 0.f;  // dA (*) Gamma
        s.X2[r][c] = E;
        s.X1[r][c] = E * s.beta[r] * kk[nt][e];  // dA (*) A
        rb[e >> 1] = fmaf(E, kk[nt][e], rb[e >> 1]);
      }
#pragma unroll
    for (int hr = 0; hr < 2; ++hr) {
      const float x = quad_sum(rb[hr]);
      if ((lane & 3) == 0) s.part[nq][16 * mt + (lane >> 2) + 8 * hr] = x;
    }
  }
  __syncthreads();
  if (tid < 4 * C) {  // F = dA (*) A: row and column sums, four threads per row
    const int r = tid >> 2, c0 = 16 * (tid & 3);
    float rs = 0.f, cs = 0.f;
#pragma unroll 4
    for (int c = c0; c < c0 + 16; ++c) {
      rs += s.X1[r][c];
      cs += s.X1[c][r];
    }
    rs = quad_sum(rs);
    cs = quad_sum(cs);
    if ((tid & 3) == 0)
      s.dG[r] += rs - cs;
  }
  if (tid < C) s.dB[tid] += s.part[0][tid] + s.part[1][tid] + s.part[2][tid] + s.part[3][tid];
  {  // dK += diag(beta) E K + (diag(beta) E)^T K
    auto Ea = [&](int r, int c) { return s.beta[r] * s.X2[r][c]; };
    auto ETa = [&](int r, int c) { return s.beta[c] * s.X2[c][r]; };
    auto Kb = [&](int c, int i) { return bf(s.kb[c][i]); };
    mma_rows<DK / 32>(accK, Ea, Kb, 16 * mt, (DK / 4) * nq, C, lane);
    mma_rows<DK / 32>(accK, ETa, Kb, 16 * mt, (DK / 4) * nq, C, lane);
  }

  // ---- phase 3: dKt = V' dH_{n+1}^T, a 64-column half of dH at a time
  float dKt[DK / 32][4];
  zero(dKt);
  for (int half = 0; half < 2; ++half) {
    __syncthreads();  // big (dW, or the other half of dH) is no longer read
    load_f32<DK, HALF, GT>(s.big, dHn + half * HALF, DV);
    copies_landed();
    auto Va = [&](int r, int j) { return s.Vp[r][half * HALF + j]; };
    auto HTb = [&](int j, int i) { return s.big[i * LF<HALF>() + j]; };
    mma_rows<DK / 32>(dKt, Va, HTb, 16 * mt, (DK / 4) * nq, HALF, lane);
  }
  float rt[2] = {0.f, 0.f};
#pragma unroll
  for (int nt = 0; nt < DK / 32; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int r = frow(16 * mt, lane, e), i = fcol((DK / 4) * nq, nt, lane, e);
      const float sc = s.kts[r];
      accK[nt][e] = fmaf(sc, dKt[nt][e], accK[nt][e]);
      rt[e >> 1] = fmaf(dKt[nt][e], sc * bf(s.kb[r][i]), rt[e >> 1]);
    }
#pragma unroll
  for (int hr = 0; hr < 2; ++hr) {
    const float x = quad_sum(rt[hr]);
    if ((lane & 3) == 0) s.part[nq][16 * mt + (lane >> 2) + 8 * hr] = x;
  }
  __syncthreads();
  if (tid < C) s.dG[tid] -= s.part[0][tid] + s.part[1][tid] + s.part[2][tid] + s.part[3][tid];
  __syncthreads();
  if (warp == 0) {
    float tot = 0.f;
    for (int r = lane; r < C; r += 32)
      tot += s.part[0][r] + s.part[1][r] + s.part[2][r] + s.part[3][r];
    tot = warp_sum(tot);
    const float hdt = warp_sum(lane < GT / 32 ? s.red[lane] : 0.f);
    if (lane == 0) s.dG[C - 1] += tot + gC * hdt;
    __syncwarp();
    // dg = reverse in-chunk cumsum of dG (rows >= len carry no gradient):
    // lane l holds rows 2l, 2l + 1; suffix sums of the pairs across lanes
    const float a0 = s.dG[2 * lane], a1 = s.dG[2 * lane + 1];
    float suf = a0 + a1;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const float y = __shfl_down_sync(0xffffffffu, suf, o);
      if (lane + o < 32) suf += y;
    }
    s.dG[2 * lane] = suf;
    s.dG[2 * lane + 1] = suf - a0;
  }
  __syncthreads();
  // step size: KLA beta = eta / (||k||^2 + eps)
  if (tid < len) {
    const size_t tok = tok0 + (size_t)tid * H;
    dg[tok] = s.dG[tid];
    if (eps >= 0.f) {
      const float den = s.n2[tid] + eps;
      deta[tok] = s.dB[tid] / den;
      s.part[0][tid] = -2.f * s.dB[tid] * eta[tok] / (den * den);
    } else {
      deta[tok] = s.dB[tid];
      s.part[0][tid] = 0.f;
    }
  }
  __syncthreads();
#pragma unroll
  for (int nt = 0; nt < DK / 32; ++nt)
#pragma unroll
    for (int e = 0; e < 4; e += 2) {
      const int r = frow(16 * mt, lane, e), i = fcol((DK / 4) * nq, nt, lane, e);
      if (r < len) {
        const float cf = s.part[0][r];
        *reinterpret_cast<float2*>(dk + (tok0 + (size_t)r * H) * DK + i) =
            make_float2(fmaf(cf, bf(s.kb[r][i]), accK[nt][e]),
                        fmaf(cf, bf(s.kb[r][i + 1]), accK[nt][e + 1]));
      }
    }
}

// ---------------------------------------------------------------- launch

static size_t al256(size_t x) { return (x + 255) & ~(size_t)255; }

struct CbwdWs {
  size_t ck, Tm, Vp, dVp, dH, W, X, Y, fwd, fwd_bytes, total;
};

// h_n, T, V', dV', dH_{n+1}, W, X, Y per chunk (fp32), then the forward
// prefill's own workspace (UT factors and, where the chain is cut, segment
// states).
static CbwdWs cbwd_layout(int B, int T, int H, int dk, int dv) {
  const size_t nblk = ((size_t)T + C - 1) / C, chunks = (size_t)B * H * nblk;
  CbwdWs w;
  w.ck = 0;
  w.Tm = w.ck + al256(chunks * dk * dv * 4);
  w.Vp = w.Tm + al256(chunks * C * C * 4);
  w.dVp = w.Vp + al256(chunks * C * dv * 4);
  w.dH = w.dVp + al256(chunks * C * dv * 4);
  w.W = w.dH + al256(chunks * dk * dv * 4);
  w.X = w.W + al256(chunks * C * dk * 4);
  w.Y = w.X + al256(chunks * C * dv * 4);
  w.fwd = w.Y + al256(chunks * dk * dv * 4);
  w.fwd_bytes = chunk_workspace_bytes(B, T, H, dk, dv, KLA_BF16);
  w.total = w.fwd + al256(w.fwd_bytes);
  return w;
}

size_t chunk_bwd_workspace_bytes(int B, int T, int H, int dk, int dv) {
  if (B < 1 || H < 1 || T < 1 || dk != dv || (dk != 64 && dk != 128)) return 0;
  return cbwd_layout(B, T, H, dk, dv).total;
}

template <int D>
static cudaError_t launch_chunk_bwd_d(const void* q, const void* k, const void* v,
                                      const float* g, const float* eta, float eps,
                                      const float* h0, const void* dout, const float* dhT,
                                      float* dq, float* dk, float* dv, float* dg, float* deta,
                                      float* dh0, int B, int Tlen, int H, void* ws,
                                      unsigned int* err, cudaStream_t st) {
  constexpr int DK = D, DV = D;
  const CbwdWs w = cbwd_layout(B, Tlen, H, DK, DV);
  char* base = (char*)ws;
  float* ck = (float*)(base + w.ck);
  float* Tws = (float*)(base + w.Tm);
  float* Vws = (float*)(base + w.Vp);
  float* dVws = (float*)(base + w.dVp);
  float* dHws = (float*)(base + w.dH);
  float* Wws = (float*)(base + w.W);
  float* Xws = (float*)(base + w.X);
  float* Yws = (float*)(base + w.Y);
  const int nblk = (Tlen + C - 1) / C;
  // the forward chunk prefill, outputs off, leaves every h_n in ck
  cudaError_t e = launch_chunk_tc(q, k, v, g, eta, eps, h0, nullptr, nullptr, B, Tlen, H, DK,
                                  DV, base + w.fwd, w.fwd_bytes, err, st, ck);
  if (e != cudaSuccess) return e;
  const auto* qb = (const __nv_bfloat16*)q;
  const auto* kb = (const __nv_bfloat16*)k;
  const auto* vb = (const __nv_bfloat16*)v;
  const auto* ob = (const __nv_bfloat16*)dout;
  constexpr size_t sp = sizeof(PrepSmem<DK, DV>), sa = sizeof(AdjSmem<DK, 2>),
                   sa1 = sizeof(AdjSmem<DK, 1>), sg = sizeof(GradSmem<DK, DV>);
  static_assert(sp <= 227 * 1024 && sa <= 227 * 1024 && sg <= 227 * 1024, "shared memory");
  static_assert(2 * (sa1 + 1024) <= 228 * 1024, "two single-buffered adjoint CTAs per SM");
  static bool attr_set[64] = {};  // the kernels' shared-memory limits, once per device
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!attr_set[dev]) {
    if ((e = cudaFuncSetAttribute(cbwd_prep_kernel<DK, DV>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sp)) ||
        (e = cudaFuncSetAttribute(cbwd_adjoint_kernel<DK, DV, 2>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sa)) ||
        (e = cudaFuncSetAttribute(cbwd_adjoint_kernel<DK, DV, 1>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sa1)) ||
        (e = cudaFuncSetAttribute(cbwd_grad_kernel<DK, DV>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sg)))
      return e;
    attr_set[dev] = true;
  }
  cbwd_prep_kernel<DK, DV><<<dim3(nblk, H, B), NT, sp, st>>>(
      qb, kb, vb, ob, g, eta, eps, ck, Tws, Vws, Wws, Xws, Yws, Tlen, H, nblk);
  // one buffer and two CTAs per SM where that turns two waves into one
  // (149 .. 296 CTAs); otherwise double buffering (measured: 4K layer 0.54 ->
  // 0.46 ms single-buffered; 512 CTAs 0.55 double- against 0.58 single-)
  const dim3 agrid(DV / BVA, H, B);
  const long actas = (long)B * H * (DV / BVA);
  if (actas > 148 && actas <= 2 * 148)
    cbwd_adjoint_kernel<DK, DV, 1><<<agrid, NT, sa1, st>>>(kb, g, dhT, Wws, Xws, Yws, dVws,
                                                           dHws, dh0, Tlen, H, nblk);
  else
    cbwd_adjoint_kernel<DK, DV, 2><<<agrid, NT, sa, st>>>(kb, g, dhT, Wws, Xws, Yws, dVws,
                                                          dHws, dh0, Tlen, H, nblk);
  cbwd_grad_kernel<DK, DV><<<dim3(nblk, H, B), GT, sg, st>>>(
      qb, kb, vb, ob, g, eta, eps, ck, Tws, Vws, dVws, dHws, dq, dk, dv, dg, deta, Tlen, H,
      nblk);
  return cudaGetLastError();
}

cudaError_t launch_chunk_bwd(const void* q, const void* k, const void* v, const float* g,
                             const float* eta, float eps, const float* h0, const void* dout,
                             const float* dhT, float* dq, float* dk, float* dv, float* dg,
                             float* deta, float* dh0, int B, int Tlen, int H, int dkd, int dvd,
                             void* ws, unsigned int* err, cudaStream_t st) {
  if (dkd == 128 && dvd == 128)
    return launch_chunk_bwd_d<128>(q, k, v, g, eta, eps, h0, dout, dhT, dq, dk, dv, dg, deta,
                                   dh0, B, Tlen, H, ws, err, st);
  if (dkd == 64 && dvd == 64)
    return launch_chunk_bwd_d<64>(q, k, v, g, eta, eps, h0, dout, dhT, dq, dk, dv, dg, deta,
                                  dh0, B, Tlen, H, ws, err, st);
  return cudaErrorInvalidValue;
}

}  // namespace kla
