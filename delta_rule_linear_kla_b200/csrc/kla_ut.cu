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
// The inverse is taken by blocks of 16 on the tensor cores.  With A_D the
// four 16x16 diagonal blocks of A, A_O the rest (strictly block-lower) and
// D = (I + A_D)^{-1}, one has I + A = (I + A_D)(I + D A_O), and N = D A_O is
// strictly block-lower with N^4 = 0, so
//
//   T = (I + N)^{-1} D = (I - N + N^2 - N^3) D = D - N (D - N (D - N D)).
//
// D (sixteen-row forward substitutions) is computed on CUDA cores in fp32;
// N = D A_O and the three Horner products are tcgen05.mma kind::tf32 products
// with fp32 accumulation.
//
// A CTA of 128 threads takes two chunks: every operand tile stacks them along
// its 128 rows, so each product is one M = N = 128 MMA whose two diagonal
// 64x64 blocks are the two chunks' results (thread t then owns row t).  The
// squared key norms are the diagonals of the Gram matrices of the first
// (bf16) MMA.  tf32 operands are K-major on both sides, so a B operand X is
// stored as X^T (row c holds column c of X).  The decays e^{G_r - G_s} are
// running products of alpha_j = e^{g_j} over s < j <= r (every factor <= 1).
//
// The factors are written to global memory already in the 128-byte swizzled
// bf16 row layout the chain kernel's MMAs read, so it fetches them with one
// bulk copy per chunk.
#include "kla_chunk.h"
#include "kla_common.cuh"
#include "kla_sync.cuh"
#include "ptx_sm100.cuh"
#include "tile_sw128.cuh"

namespace kla {
namespace {

constexpr int C = 64;
constexpr int NT = 128;
constexpr uint32_t TILE = 128 * 64 * 4;  // one fp32 operand tile: 128 rows x 64 (32 KB)

// fp32 operand tile, K-major with 128-byte swizzle: two panels of 32 columns,
// each panel 128 rows x 128 B.  Byte offset of element (row, k).
__device__ __forceinline__ uint32_t f32_off(int row, int k) {
  const int p = k >> 5, b = (k & 31) * 4;
  return (uint32_t)p * 16384u + (uint32_t)row * 128u + ((((b >> 4) ^ (row & 7)) & 7) << 4) +
         (b & 15);
}

template <int DK>
struct alignas(1024) UtSmem {
  static constexpr int NP = DK / 64;
  // region 0: keys (bf16, per panel: chunk 0 rows then chunk 1 rows); after
  //           the Gram MMA: D^T (fp32 B operand), later V2^T
  uint8_t r0[TILE > NP * 16384 ? TILE : NP * 16384];
  uint8_t r1[TILE];           // A_O^T (B operand), later V1^T
  uint8_t r2[TILE];           // D (A operand), later N (A operand)
  float adiag[2][4][16][17];  // diagonal 16x16 blocks of A
  float G[2][C];
  float beta[2][C];
  float alpha[2][C];
  uint64_t bar_tma, bar_mma;
  uint32_t tmem_base;
};

__device__ __forceinline__ void mma_tf32(uint32_t d, uint64_t a, uint64_t b, uint32_t id,
                                         uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
      "l"(a), "l"(b), "r"(id), "r"(acc)
      : "memory");
}

// idesc of kind::tf32: D f32, A and B tf32 (format 2), both K-major.
constexpr uint32_t idesc_tf32(int M, int N) {
  return (1u << 4) | (2u << 7) | (2u << 10) | ((uint32_t)(N >> 3) << 17) |
         ((uint32_t)(M >> 4) << 24);
}

// D_out(128x128, TMEM) = Atile(128x64) . Btile^T, both tiles K-major fp32.
__device__ __forceinline__ void issue_tf32_product(uint32_t d, const uint8_t* at,
                                                   const uint8_t* bt) {
  constexpr uint32_t id = idesc_tf32(128, 128);
#pragma unroll
  for (int kk = 0; kk < 8; ++kk) {  // K = 8 per instruction
    const uint32_t off = (uint32_t)(kk >> 2) * 16384u + (uint32_t)(kk & 3) * 32u;
    mma_tf32(d, ptx::sdesc_sw128(ptx::smem_u32(at) + off, 16, 1024),
             ptx::sdesc_sw128(ptx::smem_u32(bt) + off, 16, 1024), id, kk > 0);
  }
}

__device__ __forceinline__ void st_f32(uint8_t* tile, int row, int k, float v) {
  *reinterpret_cast<float*>(tile + f32_off(row, k)) = v;
}

// Column k of rows base_row + c (c = 0..63, base_row a multiple of 8): the
// swizzle phase is c & 7, so the eight addresses per phase are precomputed
// and every store is one STS with an immediate row offset.
struct ColWriter {
  uint8_t* p[8];
  __device__ __forceinline__ ColWriter(uint8_t* tile, int base_row, int k) {
    const int pan = k >> 5, b = (k & 31) * 4;
    uint8_t* base = tile + pan * 16384 + base_row * 128 + (b & 15);
#pragma unroll
    for (int e = 0; e < 8; ++e) p[e] = base + ((((b >> 4) ^ e) & 7) << 4);
  }
  __device__ __forceinline__ void put(int c, float v) const {  // c compile-time
    *reinterpret_cast<float*>(p[c & 7] + c * 128) = v;
  }
};

// Row `row` (64 values) stored with 16-byte vector stores.
__device__ __forceinline__ void st_row64(uint8_t* tile, int row, const float* v) {
#pragma unroll
  for (int q = 0; q < 16; ++q) {  // 16-byte chunk q: columns 4q .. 4q+3
    const int pan = q >> 3, ch = q & 7;
    *reinterpret_cast<float4*>(tile + pan * 16384 + row * 128 + (((ch ^ (row & 7)) & 7) << 4)) =
        make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
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
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int j = tid >> 6, r = tid & 63;  // chunk slot and its row
  const int ci0 = 2 * blockIdx.x;
  const int nvalid = min(2, total_chunks - ci0);
  const uint32_t lane_base = (uint32_t)(warp * 32) << 16;

  if (warp == 0) {
    ptx::tmem_alloc(&s.tmem_base, 256);
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
        ptx::tma_load_4d(s.r0 + p * 16384 + jj * 8192, &tm_k, &s.bar_tma, p * 64, h, n * C, b);
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
  // chunk-local inclusive cumsum of g (warps 2j, 2j+1 hold chunk j)
  float gs = gr;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const float y = __shfl_up_sync(0xffffffffu, gs, off);
    if (lane >= off) gs += y;
  }
  s.G[j][r] = gs;
  s.alpha[j][r] = __expf(gr);
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  if (r >= 32) s.G[j][r] = gs + s.G[j][31];
  const uint32_t tb = s.tmem_base;
  const uint32_t t_gram = tb, t_prod = tb + 128;
  bool ok = wait_bounded(&s.bar_tma, 0);
  __syncthreads();

  uint32_t mma_phase = 0;
  auto mma_done = [&]() {
    __syncwarp();
    if (ok) ok = wait_bounded(&s.bar_mma, mma_phase);
    mma_phase ^= 1u;
    ptx::tc_fence_after();
  };

  // ---- Gram matrices of both chunks: [K0; K1] [K0; K1]^T (bf16, fp32 acc)
  if (tid == 0 && ok) {
    ptx::tc_fence_after();
    constexpr uint32_t id = ptx::idesc_bf16(128, 128, 0, 0);
#pragma unroll
    for (int kk = 0; kk < DK / 16; ++kk) {
      const uint32_t a = ptx::smem_u32(s.r0 + (kk >> 2) * 16384) + (kk & 3) * 32;
      ptx::mma_bf16(t_gram, ptx::sdesc_sw128(a, 16, 1024), ptx::sdesc_sw128(a, 16, 1024), id,
                    kk > 0);
    }
    ptx::mma_commit(&s.bar_mma);
  }
  mma_done();

  // ---- A row r of chunk j.  beta_r from the Gram diagonal; e^{G_r - G_s} for
  // s < r as running products of alpha.  A_O^T -> r1 (row 64 j + c, column r);
  // the diagonal block -> adiag.
  const int bb = r >> 4;  // my 16-row block
  {
    float srow[64];
    ptx::tmem_ld32(t_gram + lane_base + j * 64, srow);
    ptx::tmem_ld32(t_gram + lane_base + j * 64 + 32, srow + 32);
    float diag = 0.f;
#pragma unroll
    for (int c = 0; c < 64; ++c) diag = (c == r) ? srow[c] : diag;
    const float br = er / (diag + eps);
    s.beta[j][r] = br;
    float d = br;  // beta_r e^{G_r - G_c}, built from c = r leftwards
#pragma unroll
    for (int c = 63; c >= 0; --c) {
      d = (c < r) ? d * s.alpha[j][c + 1] : d;
      srow[c] = (c < r) ? srow[c] * d : 0.f;
    }
    const ColWriter col(s.r1, 64 * j, r);
#pragma unroll
    for (int c = 0; c < 64; ++c) col.put(c, ((c >> 4) == bb) ? 0.f : srow[c]);
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      float v = 0.f;
#pragma unroll
      for (int blk = 0; blk < 4; ++blk) v = (blk == bb) ? srow[16 * blk + i] : v;
      s.adiag[j][bb][r & 15][i] = v;
    }
  }
  ptx::tc_fence_before();
  __syncthreads();

  // ---- D: thread r solves column (r & 15) of (I + A_bb)^{-1}, bb = r >> 4.
  // Written as D^T (B operand, r0: the keys are dead) and D (A operand, r2).
  {
    const int cq = r & 15;
    float x[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      float acc = 0.f;
#pragma unroll
      for (int m = 0; m < i; ++m) acc = fmaf(s.adiag[j][bb][i][m], x[m], acc);
      x[i] = (i == cq) ? 1.f : (i < cq ? 0.f : -acc);
    }
    // D^T row 64 j + r is column r of D_j: x in block bb, zero elsewhere
    {
      float v[64];
#pragma unroll
      for (int blk = 0; blk < 4; ++blk)
#pragma unroll
        for (int i = 0; i < 16; ++i) v[16 * blk + i] = (blk == bb) ? x[i] : 0.f;
      st_row64(s.r0, 64 * j + r, v);
    }
    // D: element (16 bb + i, r) = x[i]; row r of D is zeroed outside its block
    {
      const ColWriter col(s.r2, 64 * j + 16 * bb, r);
#pragma unroll
      for (int i = 0; i < 16; ++i) col.put(i, x[i]);
    }
#pragma unroll
    for (int blk = 0; blk < 4; ++blk)
      if (blk != bb)
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int ch = 4 * blk + q, pan = ch >> 3;
          const int row = 64 * j + r;
          *reinterpret_cast<float4*>(s.r2 + pan * 16384 + row * 128 +
                                     ((((ch & 7) ^ (row & 7)) & 7) << 4)) =
              make_float4(0.f, 0.f, 0.f, 0.f);
        }
  }
  ptx::fence_proxy_async_smem();
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  // my row of D (its 16 non-zeros sit in block bb)
  float drow[16];
#pragma unroll
  for (int i = 0; i < 16; ++i)
    drow[i] = *reinterpret_cast<const float*>(s.r2 + f32_off(64 * j + r, 16 * bb + i));

  // ---- N = D A_O  ->  r2 (A operand rows); D is dead afterwards
  if (tid == 0 && ok) {
    issue_tf32_product(t_prod, s.r2, s.r1);
    ptx::mma_commit(&s.bar_mma);
  }
  mma_done();
  {
    float v[64];
    ptx::tmem_ld32(t_prod + lane_base + j * 64, v);
    ptx::tmem_ld32(t_prod + lane_base + j * 64 + 32, v + 32);
    ptx::tc_fence_before();
    __syncthreads();  // everyone has read its row of D
    st_row64(s.r2, 64 * j + r, v);
  }
  ptx::fence_proxy_async_smem();
  ptx::tc_fence_before();
  __syncthreads();

  // ---- Horner: V1 = D - N D (-> r1 as V1^T), V2 = D - N V1 (-> r0 as V2^T),
  // T = D - N V2
  float trow[64];
#pragma unroll 1
  for (int step = 0; step < 3; ++step) {
    const uint8_t* bsrc = (step == 1) ? s.r1 : s.r0;
    if (tid == 0 && ok) {
      ptx::tc_fence_after();
      issue_tf32_product(t_prod, s.r2, bsrc);
      ptx::mma_commit(&s.bar_mma);
    }
    mma_done();
    ptx::tmem_ld32(t_prod + lane_base + j * 64, trow);
    ptx::tmem_ld32(t_prod + lane_base + j * 64 + 32, trow + 32);
#pragma unroll
    for (int c = 0; c < 64; ++c) trow[c] = (((c >> 4) == bb) ? drow[c & 15] : 0.f) - trow[c];
    if (step < 2) {
      uint8_t* bdst = (step == 0) ? s.r1 : s.r0;
      ptx::tc_fence_before();
      __syncthreads();  // the product that read the destination has finished
      const ColWriter col(bdst, 64 * j, r);
#pragma unroll
      for (int c = 0; c < 64; ++c) col.put(c, trow[c]);
      ptx::fence_proxy_async_smem();
      ptx::tc_fence_before();
      __syncthreads();
    }
  }

  // ---- T' and T'' rows -> workspace (swizzled bf16 rows, 128 B each)
  if (ok && valid) {
    float row[64];
#pragma unroll
    for (int c = 0; c < 64; ++c) row[c] = trow[c] * s.beta[j][c];
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
    // e^{G_c} as a running product of alpha from the chunk start
    float e = 1.f;
#pragma unroll
    for (int c = 0; c < 64; ++c) {
      e *= s.alpha[j][c];
      row[c] *= e;
    }
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
    ptx::tmem_dealloc(tb, 256);
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
