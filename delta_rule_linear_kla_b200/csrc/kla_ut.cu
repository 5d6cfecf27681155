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
//   out:   T' = T diag(beta),  T'' = T diag(beta e^G), stored transposed
//          (row c of each tile is column c of the factor), bf16
//
// The inverse is taken by blocks of 16 on the tensor cores.  With A_D the
// four 16x16 diagonal blocks of A, A_O the rest (strictly block-lower) and
// D = (I + A_D)^{-1}, one has I + A = (I + A_D)(I + D A_O), and N = D A_O is
// strictly block-lower with N^4 = 0, so
//
//   T = (I + N)^{-1} D = (I - N + N^2 - N^3) D = D - N (D - N (D - N D)),
//
// evaluated on the transposes: X_0 = D, X_{i+1}^T = D^T - X_i^T N^T, T = X_3.
// D (sixteen-row forward substitutions) and every combination are fp32 on
// CUDA cores; N = D A_O and the three Horner products are tcgen05.mma
// products of bf16 operands with fp32 accumulation.  Rounding those operands
// to bf16 moves the final outputs far less than the bf16 rounding of T' and
// T'' themselves, which the state kernel consumes as bf16 anyway.
//
// A CTA of 128 threads takes two chunks: every operand tile stacks them along
// its 128 rows, so each product is one M = N = 128 MMA whose two diagonal
// 64x64 blocks are the two chunks' results (thread t owns row t).  The
// squared key norms are the diagonals of the Gram matrices of the first MMA.
// Operands are K-major on both sides, so a B operand X is stored as X^T (row
// c holds column c of X).  The orientation of every product is chosen so
// that the row a thread holds is a row of the next operand: every
// shared-memory write is a whole swizzled row.  The decays e^{G_s - G_r} are
// running products of alpha_j = e^{g_j} over r < j <= s (every factor <= 1).
// The key tile and one 16 KB operand tile are all the shared memory a CTA
// needs, so four CTAs share an SM; each is persistent over pairs of chunks
// and fetches the next pair's keys and gates while it works.
//
// The factors are written to global memory already in the 128-byte swizzled
// bf16 layout the chain kernel's MMAs read (as MN-major A operands), so it
// fetches them with one bulk copy per chunk.
#include "kla_chunk.h"
#include "kla_common.cuh"
#include "kla_sync.cuh"
#include "ptx_sm100.cuh"
#include "tile_sw128.cuh"

namespace kla {
namespace {

constexpr int C = 64;
constexpr int NT = 128;
constexpr int CTAS_PER_SM = 4;
constexpr uint32_t TILE = 128 * 64 * 2;  // one bf16 operand tile: 128 rows x 64 (16 KB)

// Diagonal 16x16 blocks of A ([row][column], padded), later the same blocks
// of D; kept in the second tile of r0, which is idle from the Gram MMA until
// the next pair's keys arrive.
typedef float DiagBlocks[2][4][16][17];
static_assert(sizeof(DiagBlocks) <= TILE, "diagonal blocks fit one tile");

template <int DK>
struct alignas(1024) UtSmem {
  static constexpr int NP = DK / 64;
  static constexpr int R0_TILES = NP < 2 ? 2 : NP;
  // keys (per 64-column panel: chunk 0 rows then chunk 1 rows); after the
  // Gram MMA its first tile holds A_O^T, then N (B operands), its second
  // tile the diagonal blocks
  uint8_t r0[R0_TILES * TILE];
  uint8_t r1[TILE];  // D (A operand of N), then X_i^T (Horner A operands)
  float G[2][C];
  float beta[2][C];
  float alpha[2][C];
  uint64_t bar_tma, bar_mma;
  uint32_t tmem_base;
};

// D (TMEM, 128 x 128 fp32) = Atile (128 x 64) . Btile^T, both bf16 K-major.
__device__ __forceinline__ void issue_product(uint32_t d, const uint8_t* at, const uint8_t* bt) {
  constexpr uint32_t id = ptx::idesc_bf16(128, 128, 0, 0);
#pragma unroll
  for (int kk = 0; kk < C / 16; ++kk)  // K = 16 per instruction
    ptx::mma_bf16(d, ptx::sdesc_sw128(ptx::smem_u32(at) + kk * 32, 16, 1024),
                  ptx::sdesc_sw128(ptx::smem_u32(bt) + kk * 32, 16, 1024), id, kk > 0);
}

// Column half hf (32 values) of a 64-wide row that is zero outside the 16
// values x of block bb.
__device__ __forceinline__ void block_half(float* v, const float* x, int bb, int hf) {
  const bool lo = (bb >> 1) == hf && !(bb & 1), hi = (bb >> 1) == hf && (bb & 1);
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    v[i] = lo ? x[i] : 0.f;
    v[16 + i] = hi ? x[i] : 0.f;
  }
}

template <int DK>
__global__ void __launch_bounds__(NT, CTAS_PER_SM)
ut_kernel(const __grid_constant__ CUtensorMap tm_k, const float* __restrict__ g,
          const float* __restrict__ eta, float eps, uint8_t* __restrict__ ws, int T, int H,
          int nchunks, int total_chunks, unsigned int* err) {
  using Smem = UtSmem<DK>;
  constexpr int NP = Smem::NP;
  extern __shared__ uint8_t smem_raw[];
  Smem& s = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                     ~uintptr_t(1023));
  DiagBlocks& adiag = *reinterpret_cast<DiagBlocks*>(s.r0 + TILE);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int j = tid >> 6, r = tid & 63;  // chunk slot and its row
  const int npairs = (total_chunks + 1) / 2;
  const uint32_t lane_base = (uint32_t)(warp * 32) << 16;

  // keys of pair `pr` (two chunks stacked) -> r0, on bar_tma
  auto load_keys = [&](int pr) {
    const int c0 = 2 * pr, nv = min(2, total_chunks - c0);
    ptx::mbar_arrive_expect_tx(&s.bar_tma, (uint32_t)(nv * NP * 8192));
    for (int jj = 0; jj < nv; ++jj) {
      const int cj = c0 + jj, hd = cj / nchunks, nn = cj % nchunks;
#pragma unroll
      for (int p = 0; p < NP; ++p)
        ptx::tma_load_4d(s.r0 + p * TILE + jj * 8192, &tm_k, &s.bar_tma, p * 64, hd % H,
                         nn * C, hd / H);
    }
  };
  // gate and relaxation of my token in pair `pr` (zero beyond the sequence)
  auto load_gates = [&](int pr, float& gv, float& ev) {
    gv = 0.f;
    ev = 0.f;
    const int cj = 2 * pr + j;
    if (pr < npairs && cj < total_chunks) {
      const int hd = cj / nchunks, tt = (cj % nchunks) * C + r;
      if (tt < T) {
        const size_t tok = ((size_t)(hd / H) * T + tt) * H + hd % H;
        gv = g[tok];
        ev = eta[tok];
      }
    }
  };

  if (warp == 0) {
    ptx::tmem_alloc(&s.tmem_base, 128);
    ptx::tmem_relinquish();
  }
  if (tid == 0) {
    ptx::prefetch_tensormap(&tm_k);
    ptx::mbar_init(&s.bar_tma, 1);
    ptx::mbar_init(&s.bar_mma, 1);
    ptx::mbar_init_fence();
    if ((int)blockIdx.x < npairs) load_keys(blockIdx.x);
  }
  float gr, er;
  load_gates(blockIdx.x, gr, er);
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  // one 128-column accumulator: the Gram matrices, then every product
  const uint32_t tacc = s.tmem_base;
  bool ok = true;

  uint32_t mma_phase = 0;
  auto mma_done = [&]() {
    __syncwarp();
    if (ok) ok = wait_bounded(&s.bar_mma, mma_phase);
    mma_phase ^= 1u;
    ptx::tc_fence_after();
  };
  // column half hf of row t of the accumulator's diagonal block (my chunk)
  auto ld_half = [&](int hf, float* v) {
    ptx::tmem_ld32(tacc + lane_base + j * 64 + 32 * hf, v);
  };

  uint32_t tma_phase = 0;
  bool keys_in_flight = tid == 0 && (int)blockIdx.x < npairs;
  // persistent: pairs blockIdx.x, blockIdx.x + gridDim.x, ...  Every thread
  // takes the same number of trips (the exit test is block-uniform).
#pragma unroll 1
  for (int pair = blockIdx.x; pair < npairs; pair += gridDim.x) {
    if (!__syncthreads_and(ok)) break;
    const int ci = 2 * pair + j;
    const bool valid = ci < total_chunks;
    float gn, en;  // next pair's gate and relaxation
    load_gates(pair + gridDim.x, gn, en);
    // chunk-local inclusive cumsum of g (warps 2j, 2j+1 hold chunk j)
    float gs = gr;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const float y = __shfl_up_sync(0xffffffffu, gs, off);
      if (lane >= off) gs += y;
    }
    __syncthreads();  // the previous pair's readers of G, alpha, beta are done
    s.G[j][r] = gs;
    s.alpha[j][r] = __expf(gr);
    __syncthreads();
    const float G31 = s.G[j][31];
    if (r >= 32) s.G[j][r] = gs + G31;
    ok = wait_bounded(&s.bar_tma, tma_phase);
    if (ok) {
      tma_phase ^= 1u;
      keys_in_flight = false;
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();

    // ---- Gram matrices of both chunks: [K0; K1] [K0; K1]^T
    if (tid == 0 && ok) {
      constexpr uint32_t id = ptx::idesc_bf16(128, 128, 0, 0);
#pragma unroll
      for (int kk = 0; kk < DK / 16; ++kk) {
        const uint32_t a = ptx::smem_u32(s.r0 + (kk >> 2) * TILE) + (kk & 3) * 32;
        ptx::mma_bf16(tacc, ptx::sdesc_sw128(a, 16, 1024), ptx::sdesc_sw128(a, 16, 1024), id,
                      kk > 0);
      }
      ptx::mma_commit(&s.bar_mma);
    }
    mma_done();

    // ---- beta_r from the Gram diagonal, then column r of A (A_sr for s > r):
    // A_sr = beta_s (k_s . k_r) e^{G_s - G_r}, the decay a running product of
    // alpha_s from s = r + 1 on (every factor <= 1).  The Gram matrix is
    // symmetric, so row r of it is also column r.  Column r of A_O is row r
    // of A_O^T (B operand of N = D A_O, -> first tile of r0: the keys are
    // dead); the entries inside my diagonal block go to adiag.
    const int bb = r >> 4;  // my 16-row block
    const int cq = r & 15;  // my position inside it
    {
      float v[32];
      ld_half(r >> 5, v);
      float diag = 0.f;
#pragma unroll
      for (int c = 0; c < 32; ++c) diag = (c == (r & 31)) ? v[c] : diag;
      s.beta[j][r] = step_size(er, diag, eps);
      __syncthreads();  // beta complete
      float d = 1.f;
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        ld_half(hf, v);
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          const int sc = 32 * hf + c;
          d = (sc > r) ? d * s.alpha[j][sc] : d;
          v[c] = (sc > r) ? s.beta[j][sc] * v[c] * d : 0.f;
        }
        if ((bb >> 1) == hf) {
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            adiag[j][bb][i][cq] = (bb & 1) ? v[16 + i] : v[i];  // A_bb[i][cq]
            if (bb & 1) v[16 + i] = 0.f; else v[i] = 0.f;
          }
        }
        sw128_store_row32(s.r0, tid, hf, v);
      }
    }
    ptx::tc_fence_before();
    __syncthreads();  // every thread has read the Gram row; A_O^T, A_D complete

    // ---- D = (I + A_D)^{-1}: thread r solves column cq of (I + A_bb)^{-1}
    // by forward substitution and keeps it (it is row r of D^T); rows of D
    // (A operand of N, -> r1) are read back through the padded adiag, which
    // then holds D's blocks.
    float x[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      float acc = 0.f;
#pragma unroll
      for (int m = 0; m < i; ++m) acc = fmaf(adiag[j][bb][i][m], x[m], acc);
      x[i] = (i == cq) ? 1.f : (i < cq ? 0.f : -acc);
    }
    __syncthreads();  // every solve has read A_D
#pragma unroll
    for (int i = 0; i < 16; ++i) adiag[j][bb][i][cq] = x[i];
    __syncthreads();
    {
      float y[16], v[32];
#pragma unroll
      for (int i = 0; i < 16; ++i) y[i] = adiag[j][bb][cq][i];
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        block_half(v, y, bb, hf);
        sw128_store_row32(s.r1, tid, hf, v);
      }
    }
    ptx::fence_proxy_async_smem();
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();

    // ---- N = D A_O (lane t = row r of N) -> r0 as the Horner B operand (a
    // K-major B operand X^T stored by rows is X = N, row-major); D^T -> r1
    // as the first Horner A operand
    if (tid == 0 && ok) {
      issue_product(tacc, s.r1, s.r0);
      ptx::mma_commit(&s.bar_mma);
    }
    mma_done();
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      float v[32];
      ld_half(hf, v);
      sw128_store_row32(s.r0, tid, hf, v);
      block_half(v, x, bb, hf);
      sw128_store_row32(s.r1, tid, hf, v);
    }
    ptx::fence_proxy_async_smem();
    ptx::tc_fence_before();
    __syncthreads();

    // ---- Horner on the transposes: X_0 = D, X_{i+1}^T = D^T - X_i^T N^T, so
    // lane t of each product is row r of X_{i+1}^T, the next A operand row as
    // is (written in place: the product that read r1 has finished).  The
    // last one, row r of T^T = column r of T, goes straight to the outputs.
#pragma unroll 1
    for (int step = 0; step < 3; ++step) {
      if (tid == 0 && ok) {
        ptx::tc_fence_after();
        issue_product(tacc, s.r1, s.r0);
        ptx::mma_commit(&s.bar_mma);
      }
      mma_done();
      if (step < 2) {
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          float v[32], dc[32];
          ld_half(hf, v);
          block_half(dc, x, bb, hf);
#pragma unroll
          for (int c = 0; c < 32; ++c) v[c] = dc[c] - v[c];
          sw128_store_row32(s.r1, tid, hf, v);
        }
        ptx::fence_proxy_async_smem();
        ptx::tc_fence_before();
        __syncthreads();
      }
    }
    // the last product has read r0: the next pair's keys may land there
    if (tid == 0 && ok && pair + (int)gridDim.x < npairs) {
      load_keys(pair + gridDim.x);
      keys_in_flight = true;
    }

    // ---- outputs: row r of T'^T = beta_r (column r of T) and row r of
    // T''^T = beta_r e^{G_r} (column r of T), swizzled bf16 rows of 128 B
    if (ok && valid) {
      const float b1 = s.beta[j][r], b2 = b1 * __expf(s.G[j][r]);
      uint8_t* dst = ws + (size_t)ci * kUtTileBytes;
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        float v[32], dc[32];
        ld_half(hf, v);
        block_half(dc, x, bb, hf);
#pragma unroll
        for (int c = 0; c < 32; ++c) v[c] = dc[c] - v[c];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint4 u;
          u.x = pack_bf16x2(b1 * v[8 * c + 0], b1 * v[8 * c + 1]);
          u.y = pack_bf16x2(b1 * v[8 * c + 2], b1 * v[8 * c + 3]);
          u.z = pack_bf16x2(b1 * v[8 * c + 4], b1 * v[8 * c + 5]);
          u.w = pack_bf16x2(b1 * v[8 * c + 6], b1 * v[8 * c + 7]);
          *reinterpret_cast<uint4*>(dst + sw128_chunk_off(r, 4 * hf + c)) = u;
          u.x = pack_bf16x2(b2 * v[8 * c + 0], b2 * v[8 * c + 1]);
          u.y = pack_bf16x2(b2 * v[8 * c + 2], b2 * v[8 * c + 3]);
          u.z = pack_bf16x2(b2 * v[8 * c + 4], b2 * v[8 * c + 5]);
          u.w = pack_bf16x2(b2 * v[8 * c + 6], b2 * v[8 * c + 7]);
          *reinterpret_cast<uint4*>(dst + 8192 + sw128_chunk_off(r, 4 * hf + c)) = u;
        }
      }
    }
    gr = gn;
    er = en;
  }  // pair loop
  if (!ok) report_timeout(err);
  // a wait gave up: let this CTA's own key copy land before it exits
  if (keys_in_flight) wait_bounded(&s.bar_tma, tma_phase);
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tacc, 128);
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
  // persistent grid: CTAS_PER_SM CTAs per SM, each taking every gridDim-th
  // pair of chunks
  static int sm_count[64] = {};
  if (!sm_count[dev]) {
    cudaError_t e = cudaDeviceGetAttribute(&sm_count[dev], cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
  }
  const int npairs = (total + 1) / 2;
  const int grid = npairs < CTAS_PER_SM * sm_count[dev] ? npairs : CTAS_PER_SM * sm_count[dev];
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
