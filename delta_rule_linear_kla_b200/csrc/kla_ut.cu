// UT transform of every chunk, in parallel over all chunks of all heads.
//
// For one chunk of C = 64 tokens ("Deep Dive into KDA", section 3; the
// intermediates U and W named there are T diag(beta) V and T diag(beta e^G) K
// in the reading this library takes, with the key-norm step size of
// "Kaczmarz Linear Attention", Abstract):
//
//   beta_r = eta_r / (||k_r||^2 + eps),   G_r = sum_{j <= r} g_j (in chunk)
//   A_rs   = beta_r (k_r . k_s) e^{G_r - G_s}   for s < r, else 0
//   T      = (I + A)^{-1}                       (unit lower triangular)
//   out:   T' = T diag(beta),  T'' = T diag(beta e^G)   (bf16)
//
// A CTA of 128 threads takes two chunks: their keys are stacked into one
// 128-row operand so a single tcgen05.mma (M = N = 128) yields both Gram
// matrices (the two diagonal 64x64 blocks of the product); the squared key
// norms are their diagonals.  Thread t owns
// row (t mod 64) of chunk (t / 64) for the A matrix, then column
// (t mod 64) for the solve, which runs by forward substitution on CUDA cores
// in fp32 with the column held in registers and the rows of A broadcast from
// shared memory.  The factors are written to global memory already in the
// 128-byte swizzled row layout the chain kernel's MMAs read, so it can fetch
// them with one bulk copy.
#include "kla_chunk.h"
#include "kla_common.cuh"
#include "kla_sync.cuh"
#include "ptx_sm100.cuh"
#include "tile_sw128.cuh"

namespace kla {
namespace {

constexpr int C = 64;
constexpr int NT = 128;
constexpr int AST = 68;  // row stride (floats) of A / T in shared memory

template <int DK>
struct alignas(1024) UtSmem {
  static constexpr int NP = DK / 64;
  uint8_t kk[NP][16384];  // per 64-column panel: chunk 0 rows, then chunk 1 rows
  float Af[2][C][AST];    // A, then T (row-major) after the solve
  float G[2][C];
  float beta[2][C];
  float eg[2][C];         // e^{G}
  float eb[2][4][C];      // e^{G_{16 I} - G_s} for s < 16 I (row block I)
  uint64_t bar_tma, bar_mma;
  uint32_t tmem_base;
};

// Forward substitution for column c of T = (I + A)^{-1}; columns >= START
// only (x_s = 0 for s < START <= c).  Fully unrolled: x stays in registers.
template <int START>
__device__ __forceinline__ void solve_column(const float (*A)[AST], int c, float* x) {
#pragma unroll
  for (int r = START; r < C; ++r) {
    float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
    for (int s = START; s < r; s += 4) {
      if (s + 4 <= r) {
        const float4 av = *reinterpret_cast<const float4*>(&A[r][s]);
        a0 = fmaf(av.x, x[s], a0);
        a1 = fmaf(av.y, x[s + 1], a1);
        a2 = fmaf(av.z, x[s + 2], a2);
        a3 = fmaf(av.w, x[s + 3], a3);
      } else {
        a0 = fmaf(A[r][s], x[s], a0);
        if (s + 1 < r) a1 = fmaf(A[r][s + 1], x[s + 1], a1);
        if (s + 2 < r) a2 = fmaf(A[r][s + 2], x[s + 2], a2);
      }
    }
    const float acc = (a0 + a1) + (a2 + a3);
    x[r] = (r == c) ? 1.f : (r < c ? 0.f : -acc);
  }
}

template <int DK>
__global__ void __launch_bounds__(NT)
ut_kernel(const __grid_constant__ CUtensorMap tm_k, const float* __restrict__ g,
          const float* __restrict__ eta, float eps, uint8_t* __restrict__ ws, int T, int H,
          int nchunks, int total_chunks, unsigned int* err) {
  using Smem = UtSmem<DK>;
  constexpr int NP = Smem::NP;
  extern __shared__ uint8_t smem_raw[];
  Smem& s = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                     ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5;
  const int j = tid >> 6, r = tid & 63;  // chunk slot, row / column
  const int ci0 = 2 * blockIdx.x;
  const int nvalid = min(2, total_chunks - ci0);

  if (warp == 0) {
    ptx::tmem_alloc(&s.tmem_base, 128);
    ptx::tmem_relinquish();
  }
  if (tid == 0) {
    ptx::mbar_init(&s.bar_tma, 1);
    ptx::mbar_init(&s.bar_mma, 1);
    ptx::mbar_init_fence();
    ptx::mbar_arrive_expect_tx(&s.bar_tma, (uint32_t)(nvalid * NP * 8192));
    for (int jj = 0; jj < nvalid; ++jj) {
      const int ci = ci0 + jj, head = ci / nchunks, n = ci % nchunks;
      const int b = head / H, h = head % H;
#pragma unroll
      for (int p = 0; p < NP; ++p)
        ptx::tma_load_4d(s.kk[p] + jj * 8192, &tm_k, &s.bar_tma, p * 64, h, n * C, b);
    }
  }
  // gate and relaxation of my token (zero beyond the sequence end)
  const int ci = ci0 + j;
  const bool valid = j < nvalid;
  const int head = valid ? ci / nchunks : 0, n = valid ? ci % nchunks : 0;
  const int t = n * C + r;
  float gr = 0.f, er = 0.f;
  if (valid && t < T) {
    const int b = head / H, h = head % H;
    const size_t tok = ((size_t)b * T + t) * H + h;
    gr = g[tok];
    er = eta[tok];
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tb = s.tmem_base;
  bool ok = wait_bounded(&s.bar_tma, 0);

  // ---- chunk-local inclusive cumsum of g
  float gs = gr;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const float y = __shfl_up_sync(0xffffffffu, gs, off);
    if ((tid & 31) >= off) gs += y;
  }
  s.G[j][r] = gs;
  __syncthreads();
  if (r >= 32) s.G[j][r] = gs + s.G[j][31];
  __syncthreads();
  const float Gr = s.G[j][r];
  s.eg[j][r] = __expf(Gr);
  // decay from block starts: eb[j][I][s] = e^{G_{16I} - G_s}, s < 16 I
#pragma unroll
  for (int I = 1; I < 4; ++I)
    if (r < 16 * I) s.eb[j][I][r] = __expf(s.G[j][16 * I] - s.G[j][r]);

  // ---- Gram matrices of both chunks in one MMA
  if (tid == 0 && ok) {
    ptx::tc_fence_after();
    constexpr uint32_t id = ptx::idesc_bf16(128, 128, 0, 0);
#pragma unroll
    for (int kk = 0; kk < DK / 16; ++kk) {
      const uint32_t a = ptx::smem_u32(s.kk[kk >> 2]) + (kk & 3) * 32;
      ptx::mma_bf16(tb, ptx::sdesc_sw128(a, 16, 1024), ptx::sdesc_sw128(a, 16, 1024), id, kk > 0);
    }
    ptx::mma_commit(&s.bar_mma);
  }
  __syncthreads();
  if (ok) ok = wait_bounded(&s.bar_mma, 0);
  ptx::tc_fence_after();

  // ---- A row r of chunk j.  beta_r = eta_r / (||k_r||^2 + eps) takes the
  // squared norm from the Gram diagonal.  Decays: within r's own 16-row block
  // e^{G_r - G_s} directly; for earlier blocks e^{G_r - G_b} e^{G_b - G_s}
  // with b = 16 * (r / 16) (both factors <= 1, never overflowing).
  if (ok) {
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    const int I = r >> 4, b0 = 16 * I;
    float srow[64];
    ptx::tmem_ld32(tb + lane_base + j * 64, srow);
    ptx::tmem_ld32(tb + lane_base + j * 64 + 32, srow + 32);
    float diag = 0.f;
#pragma unroll
    for (int c = 0; c < 64; ++c) diag = (c == r) ? srow[c] : diag;
    const float br = er / (diag + eps);
    s.beta[j][r] = br;
    const float cr = br * __expf(Gr - s.G[j][b0]);
#pragma unroll
    for (int c4 = 0; c4 < 64; c4 += 4) {
      float a[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int sc = c4 + e;
        float v;
        if (sc < b0) v = cr * srow[sc] * s.eb[j][I][sc];
        else if (sc < r) v = br * srow[sc] * __expf(Gr - s.G[j][sc]);
        else v = 0.f;
        a[e] = v;
      }
      *reinterpret_cast<float4*>(&s.Af[j][r][c4]) = make_float4(a[0], a[1], a[2], a[3]);
    }
  }
  ptx::tc_fence_before();
  __syncthreads();

  // ---- T = (I + A)^{-1}, column r of chunk j (warp-uniform start column)
  float x[64];
  if ((warp & 1) == 0) {
    solve_column<0>(s.Af[j], r, x);
  } else {
#pragma unroll
    for (int i = 0; i < 32; ++i) x[i] = 0.f;
    solve_column<32>(s.Af[j], r, x);
  }
  __syncthreads();  // everyone is done reading A
#pragma unroll
  for (int i = 0; i < C; ++i) s.Af[j][i][r] = x[i];
  __syncthreads();

  // ---- T' and T'' rows -> workspace (swizzled bf16 rows, 128 B each)
  if (ok && valid) {
    float row[64];
#pragma unroll
    for (int c4 = 0; c4 < C; c4 += 4) {
      const float4 tv = *reinterpret_cast<const float4*>(&s.Af[j][r][c4]);
      row[c4] = tv.x * s.beta[j][c4];
      row[c4 + 1] = tv.y * s.beta[j][c4 + 1];
      row[c4 + 2] = tv.z * s.beta[j][c4 + 2];
      row[c4 + 3] = tv.w * s.beta[j][c4 + 3];
    }
    uint8_t* dst = ws + (size_t)ci * kUtTileBytes;
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      uint4 u;
      u.x = pack_bf16x2(row[8 * c + 0], row[8 * c + 1]);
      u.y = pack_bf16x2(row[8 * c + 2], row[8 * c + 3]);
      u.z = pack_bf16x2(row[8 * c + 4], row[8 * c + 5]);
      u.w = pack_bf16x2(row[8 * c + 6], row[8 * c + 7]);
      *reinterpret_cast<uint4*>(dst + sw128_chunk_off(r, c)) = u;
    }
#pragma unroll
    for (int c = 0; c < 64; ++c) row[c] *= s.eg[j][c];
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      uint4 u;
      u.x = pack_bf16x2(row[8 * c + 0], row[8 * c + 1]);
      u.y = pack_bf16x2(row[8 * c + 2], row[8 * c + 3]);
      u.z = pack_bf16x2(row[8 * c + 4], row[8 * c + 5]);
      u.w = pack_bf16x2(row[8 * c + 6], row[8 * c + 7]);
      *reinterpret_cast<uint4*>(dst + 8192 + sw128_chunk_off(r, c)) = u;
    }
  }
  if (!ok && tid == 0) report_timeout(err);
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tb, 128);
  }
}

template <int DK>
cudaError_t launch_ut_dk(const CUtensorMap& tm_k, const float* g, const float* eta, float eps,
                         uint8_t* ws, int B, int T, int H, unsigned int* err, cudaStream_t st) {
  const int nchunks = (T + C - 1) / C;
  const int total = B * H * nchunks;
  if (total == 0) return cudaSuccess;
  const size_t smem = sizeof(UtSmem<DK>) + 1024;
  static bool attr_set[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(ut_kernel<DK>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  const int grid = (total + 1) / 2;
  ut_kernel<DK><<<grid, NT, smem, st>>>(tm_k, g, eta, eps, ws, T, H, nchunks, total, err);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_ut(const CUtensorMap& tm_k, const float* g, const float* eta, float eps,
                      uint8_t* ws, int B, int T, int H, int dk, unsigned int* err,
                      cudaStream_t st) {
  if (dk == 128) return launch_ut_dk<128>(tm_k, g, eta, eps, ws, B, T, H, err, st);
  if (dk == 64) return launch_ut_dk<64>(tm_k, g, eta, eps, ws, B, T, H, err, st);
  return cudaErrorNotSupported;
}

}  // namespace kla
