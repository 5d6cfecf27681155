// UT transform of every chunk (the device code, shared by the stand-alone UT
// kernel and the single-launch prefill), in parallel over all chunks.
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
// The inverse is taken by blocks of 16.  With A_bj the 16 x 16 blocks of A
// and D_b = (I + A_bb)^{-1}, block forward substitution gives T_bb = D_b and
// T_bc = -D_b sum_{c <= j < b} A_bj T_jc (b > c).  It is evaluated on the
// transposes, Y = T^T:
//
//   Y_cc = D_c^T,   Y_cb = -(sum_{c <= j < b} Y_cj A_bj^T) D_b^T   (b > c),
//
// so every block just formed is the left operand of the next product.
//
// A CTA of 128 threads takes two chunks (a "pair"):
//   1. the Gram matrices of both chunks as one tcgen05 MMA, [K0; K1][K0; K1]^T
//      (M = N = 128, bf16, fp32 in TMEM; the two 64 x 64 diagonal blocks are
//      the chunks' Gram matrices); their diagonals give ||k||^2 and beta;
//   2. thread t holds row t: it forms row r of A and stores the blocks left
//      of its diagonal block (bf16) and its part of the diagonal block (fp32,
//      transposed).  The decay e^{G_r - G_s} (s < r, so <= 1) is one
//      exponential per entry inside the row's own 16-column diagonal block;
//      in a block q wholly left of row r it is the product of
//      e^{G_r - G_{16q+15}} and E_s = e^{G_{16q+15} - G_s}, both <= 1, with
//      E tabulated once per chunk.  A warp holds 32 rows of one chunk, so the
//      half-row test is uniform over it: rows 0..31 touch columns 0..31 only;
//   3. thread (chunk, b, c) solves column c of D_b by forward substitution
//      (fp32, reading the transposed diagonal block four entries at a time);
//      the outputs' diagonal blocks and the zeros left of them are then
//      written row by row, eight threads to a 128-byte row (scattered
//      16-byte stores of one row per thread had cost a third of the
//      kernel's time);
//   4. warp (chunk, half) forms the off-diagonal row blocks Y_cb with
//      warp-level bf16 products (mma.sync m16n8k16, fp32 sums): the fp32
//      accumulators of one product are, packed to bf16, the left operand of
//      the next one, so a row block never leaves its warp's registers.
// Rounding the products' operands to bf16 moves the outputs no more than the
// bf16 rounding of T' and T'' themselves (a CPU simulation of this exact
// scheme on the stress and 0.4B-layer distributions gives the same error as
// rounding the exact factors).  Once the Gram MMA has read the keys, their
// shared memory holds A and its diagonal blocks (steps 2 to 4); the next
// pair's keys are loaded when step 4 is done.  That keeps a lane at ~42 KB
// of shared memory and 128 registers, so four lanes share an SM: the phases
// are short dependent chains separated by barriers, and more lanes per SM
// hide more of their latency.
//
// The factors are written to global memory (16- and 4-byte stores) already
// in the 128-byte swizzled bf16 layout the chain kernel's MMAs read (as
// MN-major A operands), so it fetches them with one bulk copy per chunk.
//
// Debug bound check (CHECK): for eta in [0, 2] every factor
// (I - beta_j k_j k_j^T) of the chunk's transition has norm <= 1, and then
// |T_rs| ||k_r|| / ||k_s|| <= eta'_r e^{G_r - G_s} for r > s, with
// eta'_r = beta_r ||k_r||^2.  The checked variant measures the largest ratio
// of the two sides over every entry it forms (entries below 1e-30 skipped),
// records it (atomicMax on the float's bits) and sets the device error word
// when it exceeds kBoundSlack.
#pragma once

#include "kla_chunk.h"
#include "kla_common.cuh"
#include "kla_sync.cuh"
#include "ptx_sm100.cuh"
#include "tile_sw128.cuh"

namespace kla {
namespace utb {

constexpr int C = 64;
constexpr int NT = 128;
constexpr uint32_t TILE = 128 * 64 * 2;  // one key panel of a pair: 128 rows x 64 bf16
constexpr int AROW = 72;                 // bf16 per row of the A tile (64 + 8: 144 B rows)
constexpr int DROW = 24;                 // bf16 per row of a D_b^T block (16 + 8: 48 B rows)
constexpr float kBoundSlack = 1.25f;     // allowance for the factors' own rounding

template <int DK>
constexpr int ctas_per_sm() {
  return 4;
}

template <int DK>
struct alignas(1024) UtSmem {
  static constexpr int NP = DK / 64;
  // A of both chunks, in the keys' bytes once the Gram MMA has read them
  struct Work {
    __nv_bfloat16 a[2][C][AROW];  // A left of the diagonal blocks, bf16, row-major
    // diagonal blocks of A, fp32, transposed: entry (row i, column m) of
    // block b at [b][16 m + i]; 272-float block pitch (16 banks apart)
    alignas(16) float adt[2][4][272];
  };
  union {
    uint8_t keys[NP * TILE];  // [K0; K1] per 64-column panel (TMA, 128-byte swizzle)
    Work w;
  };
  __nv_bfloat16 dt[2][4][16][DROW];  // D_b^T (row c = column c of D_b), bf16
  float G[2][C], E[2][C], eta[2][C], n2[2][C];  // E_s = e^{G_{s | 15} - G_s}
  float b1[2][C], b2[2][C];          // beta, beta e^G
  uint64_t bar_tma, bar_mma;
  uint32_t tmem_base;
};

// ---------------------------------------------------------------- warp MMA
__device__ __forceinline__ void ldsm_x4(uint32_t* r, const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(ptx::smem_u32(p)));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t* r, const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(ptx::smem_u32(p)));
}
// d (16 x 8, fp32) += a (16 x 16, bf16, row-major fragment) . b (16 x 8)
__device__ __forceinline__ void mma16816(float* d, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
      "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Byte offset of element (row m, column n) in a 64 x 64 bf16 tile of 128-B
// swizzled rows.
__device__ __forceinline__ uint32_t tile_off(int m, int n) {
  return (uint32_t)(m * 128 + ((((n >> 3) ^ (m & 7)) & 7) << 4) + (n & 7) * 2);
}

__device__ __forceinline__ void atomic_max_nonneg(float* p, float x) {
  atomicMax(reinterpret_cast<unsigned int*>(p), __float_as_uint(x));
}

// Ratio of the P-UT bound for entry T_rs (r > s) of one chunk.
template <int DK>
__device__ __forceinline__ float bound_ratio(const UtSmem<DK>& s, int j, int r, int sc,
                                             float t_rs) {
  const float a = fabsf(t_rs);
  if (!(a > 1e-30f)) return 0.f;
  const float etap = s.b1[j][r] * s.n2[j][r];
  const float den = etap * __expf(s.G[j][r] - s.G[j][sc]) * sqrtf(s.n2[j][sc]);
  const float num = a * sqrtf(s.n2[j][r]);
  if (!(den > 1e-30f)) return num > 1e-30f ? 3.0e38f : 0.f;
  return num / den;
}


// Named barrier of one 128-thread lane, of the 64 threads (two warps) of
// one chunk slot, and the lane barrier's AND-reduction form.
__device__ __forceinline__ void nbar_sync(int id) {
  asm volatile("bar.sync %0, 128;" ::"r"(id) : "memory");
}
__device__ __forceinline__ void nbar_sync64(int id) {
  asm volatile("bar.sync %0, 64;" ::"r"(id) : "memory");
}
__device__ __forceinline__ bool nbar_and(int id, bool v) {
  uint32_t out;
  asm volatile(
      "{\n\t.reg .pred pi, po;\n\t"
      "setp.ne.u32 pi, %1, 0;\n\t"
      "bar.red.and.pred po, %2, 128, pi;\n\t"
      "selp.u32 %0, 1, 0, po;\n\t}"
      : "=r"(out)
      : "r"((uint32_t)v), "r"(id)
      : "memory");
  return out != 0;
}

// One UT "lane": 128 threads (tid 0..127, TMEM lanes 0..127 of their own
// 128-column allocation) that own the shared memory `s` and synchronise on
// named barrier `bar_id`; between the Gram product and the end of a pair the
// two warps of chunk slot j (threads 64 j .. 64 j + 63, which alone read and
// write that chunk's rows, blocks and outputs) synchronise on their own
// barrier chunk_bar + j, so one chunk's phases do not wait for the other's.  It takes pairs first_pair, first_pair +
// pair_stride, ... of the `count` chunks p0, p0 + 1, ... of a chunk order
// over the BH heads: chunk-major within each head, or (nmajor) chunk index n
// major over all heads (n = 0 of every head first).  With `flags` it raises
// flags[head * nchunks + n] = 1 once a chunk's factors are in memory (for
// state CTAs of the same launch that wait on them; needs nmajor).
// `standalone`: the lane is the whole CTA (it may relinquish the TMEM
// allocation permit).
template <int DK, bool CHECK>
__device__ __forceinline__ void ut_run(const CUtensorMap* tm_k, const float* __restrict__ g,
                                       const float* __restrict__ eta, float eps,
                                       uint8_t* __restrict__ ws, int T, int H, int nchunks,
                                       int BH, int p0, int total_chunks, bool nmajor,
                                       unsigned int* err, float* ratio_max,
                                       unsigned int* flags, UtSmem<DK>& s, const int tid,
                                       const int bar_id, const int chunk_bar,
                                       const int first_pair,
                                       const int pair_stride, const bool standalone) {
  constexpr int NP = UtSmem<DK>::NP;
  const int warp = tid >> 5, lane = tid & 31;
  const int j = tid >> 6, r = tid & 63;  // chunk slot and its row
  const int npairs = (total_chunks + 1) / 2;
  const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
  // processing index (0 .. total_chunks - 1) -> (head, chunk)
  auto chunk_of = [&](int p, int& hd, int& nn) {
    p += p0;
    if (nmajor) {
      nn = p / BH;
      hd = p - nn * BH;
    } else {
      hd = p / nchunks;
      nn = p - hd * nchunks;
    }
  };

  // keys of pair `pr` (two chunks stacked) -> s.keys, on bar_tma
  auto load_keys = [&](int pr) {
    const int c0 = 2 * pr, nv = min(2, total_chunks - c0);
    ptx::mbar_arrive_expect_tx(&s.bar_tma, (uint32_t)(nv * NP * 8192));
    for (int jj = 0; jj < nv; ++jj) {
      int hd, nn;
      chunk_of(c0 + jj, hd, nn);
#pragma unroll
      for (int p = 0; p < NP; ++p)
        ptx::tma_load_4d(s.keys + p * TILE + jj * 8192, tm_k, &s.bar_tma, p * 64, hd % H,
                         nn * C, hd / H);
    }
  };
  // gate and relaxation of my token in pair `pr` (zero beyond the sequence:
  // an identity step)
  auto load_gates = [&](int pr, float& gv, float& ev) {
    gv = 0.f;
    ev = 0.f;
    const int cj = 2 * pr + j;
    if (pr < npairs && cj < total_chunks) {
      int hd, nn;
      chunk_of(cj, hd, nn);
      const int tt = nn * C + r;
      if (tt < T) {
        const size_t tok = ((size_t)(hd / H) * T + tt) * H + hd % H;
        gv = g[tok];
        ev = eta[tok];
      }
    }
  };

  if (warp == 0) {
    ptx::tmem_alloc(&s.tmem_base, 128);
    if (standalone) ptx::tmem_relinquish();
  }
  if (tid == 0) {
    ptx::prefetch_tensormap(tm_k);
    ptx::mbar_init(&s.bar_tma, 1);
    ptx::mbar_init(&s.bar_mma, 1);
    ptx::mbar_init_fence();
    if (first_pair < npairs) load_keys(first_pair);
  }
  float gr, er;
  load_gates(first_pair, gr, er);
  ptx::tc_fence_before();
  nbar_sync(bar_id);
  ptx::tc_fence_after();
  const uint32_t tacc = s.tmem_base;  // the two Gram matrices (128 x 128 fp32)
  bool ok = true;
  uint32_t mma_phase = 0, tma_phase = 0;
  bool keys_in_flight = tid == 0 && first_pair < npairs;
  // raise the ready flags of both chunks of pair `pr` (after every thread's
  // stores of its factors and a fence)
  auto publish = [&](int pr) {
    for (int jj = 0; jj < 2; ++jj) {
      if (2 * pr + jj < total_chunks) {
        int hd, nn;
        chunk_of(2 * pr + jj, hd, nn);
        atomicExch(flags + (size_t)hd * nchunks + nn, 1u);
      }
    }
  };
  float worst = 0.f;  // CHECK: largest bound ratio this thread saw

  // persistent: pairs first_pair, first_pair + pair_stride, ...  Every
  // thread of the lane takes the same number of trips (the exit test is
  // uniform over the lane).
#pragma unroll 1
  for (int pair = first_pair; pair < npairs; pair += pair_stride) {
    if (!nbar_and(bar_id, ok)) break;  // also: the previous pair's readers are done
    const bool valid = 2 * pair + j < total_chunks;
    // chunk-local inclusive cumsum of g (warps 2j, 2j+1 hold chunk j)
    float gs = gr;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const float y = __shfl_up_sync(0xffffffffu, gs, off);
      if (lane >= off) gs += y;
    }
    s.G[j][r] = gs;
    // s and s | 15 lie in the same warp: the difference of the warp's
    // partial sums is G_{s | 15} - G_s (<= 0)
    s.E[j][r] = __expf(__shfl_sync(0xffffffffu, gs, lane | 15) - gs);
    s.eta[j][r] = er;
    nbar_sync64(chunk_bar + j);
    const float G31 = s.G[j][31];  // row 31 is not rewritten below
    if (r >= 32) s.G[j][r] = gs + G31;
    float gn, en;  // next pair's gate and relaxation
    load_gates(pair + pair_stride, gn, en);

    // ---- Gram matrices of both chunks: [K0; K1] [K0; K1]^T
    if (tid == 0) {
      ok = wait_bounded(&s.bar_tma, tma_phase);
      tma_phase ^= 1u;
      keys_in_flight = !ok;
      if (ok) {
        ptx::tc_fence_after();
        constexpr uint32_t id = ptx::idesc_bf16(128, 128, 0, 0);
#pragma unroll
        for (int kk = 0; kk < DK / 16; ++kk) {
          const uint32_t a = ptx::smem_u32(s.keys + (kk >> 2) * TILE) + (kk & 3) * 32;
          ptx::mma_bf16(tacc, ptx::sdesc_sw128(a, 16, 1024), ptx::sdesc_sw128(a, 16, 1024),
                        id, kk > 0);
        }
        ptx::mma_commit(&s.bar_mma);
        ok = wait_bounded(&s.bar_mma, mma_phase);
      }
    }
    mma_phase ^= 1u;
    __syncwarp();
    if (!nbar_and(bar_id, ok)) break;
    ptx::tc_fence_after();

    // ---- row r of the chunk's Gram matrix (its diagonal block), beta_r and
    // row r of A
    const int bb = r >> 4;  // my 16-row block
    {
      // hd: the 32-column half that holds the diagonal (warp-uniform)
      const int hd = warp & 1;
      float v[32], vl[32];  // the half that holds the diagonal; (hd = 1) the left half
      if (hd == 1)
        ptx::tmem_ld32x2(tacc + lane_base + 64 * j + 32, tacc + lane_base + 64 * j, v, vl);
      else
        ptx::tmem_ld32(tacc + lane_base + 64 * j, v);
      float nn2 = 0.f;
#pragma unroll
      for (int c = 0; c < 32; ++c) nn2 = (c == (r & 31)) ? v[c] : nn2;
      const float beta = step_size(er, nn2, eps);
      const float Gr = s.G[j][r];
      __nv_bfloat16* arow = &s.w.a[j][r][0];
      // A_rs = beta_r (k_r . k_s) e^{G_r - G_s} for s < r: the diagonal half,
      // blocks 2 hd (v[0..15]) and 2 hd + 1 (v[16..31]); lanes 0..15 of the
      // warp have their diagonal block first, lanes 16..31 second.  The
      // decays inside my own block, one exponential per entry (argument
      // <= 0; zero for s >= r); a first block left of my own one takes
      // e^{G_r - G_{32 hd + 15}} E_s (both <= 1); a second block right of
      // my own one is zero.  Every lane runs the same instructions: the
      // two roles are selects.
      const bool second = (bb & 1) != 0;
      float ev[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int c = 16 * bb + i;
        ev[i] = c < r ? __expf(Gr - s.G[j][c]) : 0.f;
      }
      // meaningful in the second block only (the select below discards it
      // in the first, where the argument is >= 0)
      const float fl = beta * __expf(Gr - s.G[j][32 * hd + 15]);
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const float own0 = beta * v[i] * ev[i], left = v[i] * (fl * s.E[j][32 * hd + i]);
        const float own1 = beta * v[16 + i] * ev[i];
        v[i] = second ? left : own0;
        v[16 + i] = second ? own1 : 0.f;
        // my row of the diagonal block, as a column of adt
        s.w.adt[j][bb][16 * i + (r & 15)] = second ? own1 : own0;
      }
      auto store_bf16 = [&](int h) {  // the blocks of half h left of block bb
#pragma unroll
        for (int q8 = 0; q8 < 4; ++q8) {
          if (4 * h + q8 < 2 * bb) {
            uint4 u;
            u.x = pack_bf16x2(v[8 * q8 + 0], v[8 * q8 + 1]);
            u.y = pack_bf16x2(v[8 * q8 + 2], v[8 * q8 + 3]);
            u.z = pack_bf16x2(v[8 * q8 + 4], v[8 * q8 + 5]);
            u.w = pack_bf16x2(v[8 * q8 + 6], v[8 * q8 + 7]);
            *reinterpret_cast<uint4*>(arow + 8 * (4 * h + q8)) = u;
          }
        }
      };
      store_bf16(hd);
      if (hd == 1) {
        // columns 0..31 lie wholly left of rows 32..63:
        // e^{G_r - G_s} = e^{G_r - G_{16q+15}} E_s, both factors <= 1
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          const float f = beta * __expf(Gr - s.G[j][16 * q + 15]);
#pragma unroll
          for (int i = 0; i < 16; ++i) v[16 * q + i] = vl[16 * q + i] * (f * s.E[j][16 * q + i]);
        }
        store_bf16(0);
      }
      s.b1[j][r] = beta;
      s.b2[j][r] = beta * __expf(s.G[j][r]);
      s.n2[j][r] = nn2;
    }
    ptx::tc_fence_before();
    nbar_sync64(chunk_bar + j);

    // this chunk's factor tile in the workspace: T'^T, then T''^T
    uint8_t* dst = ws;
    if (valid) {
      int hd, nn;
      chunk_of(2 * pair + j, hd, nn);
      dst = ws + ((size_t)hd * nchunks + nn) * kUtTileBytes;
    }
    // ---- D_b = (I + A_bb)^{-1}: thread (j, b, c) solves column c; it is row
    // m = 16 b + c of Y's diagonal block (kept for the products below as
    // D_b^T, and for the outputs)
    {
      const int b = (tid >> 4) & 3, c = tid & 15, m = 16 * b + c;
      // right-looking: once x_m is final, it is subtracted from every later
      // row at once (16 dependent steps of independent updates)
      float x[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) x[i] = (i == c) ? 1.f : 0.f;
#pragma unroll
      for (int mm = 0; mm < 15; ++mm) {
        const float* col = &s.w.adt[j][b][16 * mm];  // column mm of A_bb
#pragma unroll
        for (int i4 = (mm + 1) / 4; i4 < 4; ++i4) {
          const float4 a4 = *reinterpret_cast<const float4*>(col + 4 * i4);
          const float ae[4] = {a4.x, a4.y, a4.z, a4.w};
#pragma unroll
          for (int e = 0; e < 4; ++e)
            if (4 * i4 + e > mm) x[4 * i4 + e] = fmaf(-ae[e], x[mm], x[4 * i4 + e]);
        }
      }
      uint4 lo, hi;
      lo.x = pack_bf16x2(x[0], x[1]);   lo.y = pack_bf16x2(x[2], x[3]);
      lo.z = pack_bf16x2(x[4], x[5]);   lo.w = pack_bf16x2(x[6], x[7]);
      hi.x = pack_bf16x2(x[8], x[9]);   hi.y = pack_bf16x2(x[10], x[11]);
      hi.z = pack_bf16x2(x[12], x[13]); hi.w = pack_bf16x2(x[14], x[15]);
      *reinterpret_cast<uint4*>(&s.dt[j][b][c][0]) = lo;
      *reinterpret_cast<uint4*>(&s.dt[j][b][c][8]) = hi;
      // row m of both outputs' diagonal block (16 columns each), bf16
      const float f1 = s.b1[j][m], f2 = s.b2[j][m];
      uint4 u1[2], u2[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const float* xh = x + 8 * h;
        u1[h].x = pack_bf16x2(f1 * xh[0], f1 * xh[1]); u1[h].y = pack_bf16x2(f1 * xh[2], f1 * xh[3]);
        u1[h].z = pack_bf16x2(f1 * xh[4], f1 * xh[5]); u1[h].w = pack_bf16x2(f1 * xh[6], f1 * xh[7]);
        u2[h].x = pack_bf16x2(f2 * xh[0], f2 * xh[1]); u2[h].y = pack_bf16x2(f2 * xh[2], f2 * xh[3]);
        u2[h].z = pack_bf16x2(f2 * xh[4], f2 * xh[5]); u2[h].w = pack_bf16x2(f2 * xh[6], f2 * xh[7]);
      }
      if constexpr (CHECK) {
        if (valid) {
#pragma unroll
          for (int i = 0; i < 16; ++i)
            if (i > c) worst = fmaxf(worst, bound_ratio(s, j, 16 * b + i, m, x[i]));
        }
      }
      // staged over the chunk's diagonal blocks of A once every thread of
      // the chunk is done reading them: [output][row m][half]
      uint4* stg = reinterpret_cast<uint4*>(&s.w.adt[j][0][0]);
      nbar_sync64(chunk_bar + j);
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        stg[m * 2 + h] = u1[h];
        stg[(64 + m) * 2 + h] = u2[h];
      }
    }
    nbar_sync64(chunk_bar + j);
    // The 16-byte chunks of both output tiles that are known now (in row m
    // of block b: the 2 b zero chunks left of the diagonal block and its 2
    // chunks), written row by row: eight threads per 128-byte row, so a
    // warp's store covers four whole rows (the off-diagonal chunks follow
    // from the products below).
    if (valid) {
      const uint4* stg = reinterpret_cast<const uint4*>(&s.w.adt[j][0][0]);
      const int u = tid & 63, p = u & 7;
#pragma unroll
      for (int t = 0; t < 2; ++t) {
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const int m = 8 * k + (u >> 3), q = p ^ (m & 7), bq = m >> 4;
          if (q < 2 * bq + 2) {
            const uint4 val = q < 2 * bq ? make_uint4(0, 0, 0, 0)
                                         : stg[(64 * t + m) * 2 + (q - 2 * bq)];
            *reinterpret_cast<uint4*>(dst + t * 8192 + m * 128 + p * 16) = val;
          }
        }
      }
    }

    // ---- off-diagonal row blocks of Y = T^T: warp 2j takes row block 0,
    // warp 2j + 1 row blocks 1 and 2 (row block 3 is D_3^T alone)
    {
      const int half = warp & 1;
      const int g8 = lane >> 3, l8 = lane & 7;  // ldmatrix: matrix and row
      const int fr = lane >> 2, fc = 2 * (lane & 3);  // fragment row / column pair
      // c is a compile-time index in every unrolled copy (the register
      // fragments y[] are indexed by it); the warp-uniform test picks the
      // row blocks this warp owns
#pragma unroll
      for (int c = 0; c < 3; ++c) {
        if (half ? c == 0 : c != 0) continue;
        uint32_t y[4][4];  // A fragments of Y_cb, b = c .. 3 (bf16)
        ldsm_x4(y[c], &s.dt[j][c][(g8 & 1) * 8 + l8][(g8 >> 1) * 8]);
#pragma unroll
        for (int b = 1; b < 4; ++b) {
          if (b <= c) continue;
          float acc[2][4] = {};
#pragma unroll
          for (int jj = 0; jj < 3; ++jj) {
            if (jj < c || jj >= b) continue;
            // A_{b,jj}^T as the B operand: rows 16 b + 8 h + (0..7) of A,
            // columns 16 jj + (0..15)
            uint32_t bf[4];
            ldsm_x4(bf, &s.w.a[j][16 * b + (g8 >> 1) * 8 + l8][16 * jj + (g8 & 1) * 8]);
            mma16816(acc[0], y[jj], bf[0], bf[1]);
            mma16816(acc[1], y[jj], bf[2], bf[3]);
          }
          uint32_t sa[4] = {pack_bf16x2(acc[0][0], acc[0][1]), pack_bf16x2(acc[0][2], acc[0][3]),
                            pack_bf16x2(acc[1][0], acc[1][1]), pack_bf16x2(acc[1][2], acc[1][3])};
          // times D_b^T (stored row-major as D_b^T: transposed loads give the
          // B fragments)
          uint32_t db[4];
          ldsm_x4_t(db, &s.dt[j][b][(g8 & 1) * 8 + l8][(g8 >> 1) * 8]);
          float yb[2][4] = {};
          mma16816(yb[0], sa, db[0], db[1]);
          mma16816(yb[1], sa, db[2], db[3]);
#pragma unroll
          for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int e = 0; e < 4; ++e) yb[h][e] = -yb[h][e];
          y[b][0] = pack_bf16x2(yb[0][0], yb[0][1]);
          y[b][1] = pack_bf16x2(yb[0][2], yb[0][3]);
          y[b][2] = pack_bf16x2(yb[1][0], yb[1][1]);
          y[b][3] = pack_bf16x2(yb[1][2], yb[1][3]);
          if (valid) {
#pragma unroll
            for (int rr = 0; rr < 2; ++rr) {
              const int m = 16 * c + fr + 8 * rr;
              const float f1 = s.b1[j][m], f2 = s.b2[j][m];
#pragma unroll
              for (int h = 0; h < 2; ++h) {
                const int n = 16 * b + 8 * h + fc;
                const float e0 = yb[h][2 * rr], e1 = yb[h][2 * rr + 1];
                const uint32_t off = tile_off(m, n);
                *reinterpret_cast<uint32_t*>(dst + off) = pack_bf16x2(f1 * e0, f1 * e1);
                *reinterpret_cast<uint32_t*>(dst + 8192 + off) = pack_bf16x2(f2 * e0, f2 * e1);
                if constexpr (CHECK) {
                  worst = fmaxf(worst, bound_ratio(s, j, n, m, e0));
                  worst = fmaxf(worst, bound_ratio(s, j, n + 1, m, e1));
                }
              }
            }
          }
        }
      }
    }
    // every thread's factor stores are visible GPU-wide before the flags go
    // up; A and its blocks have been read, so the next pair's keys may land
    // in their place
    if (flags) __threadfence();
    ptx::fence_proxy_async_smem();
    nbar_sync(bar_id);
    if (tid == 0) {
      if (flags && ok) {
        __threadfence();
        publish(pair);
      }
      if (pair + pair_stride < npairs) {
        load_keys(pair + pair_stride);
        keys_in_flight = true;
      }
    }
    gr = gn;
    er = en;
  }  // pair loop
  if (!ok) report_timeout(err);
  if constexpr (CHECK) {
    if (worst > 0.f) atomic_max_nonneg(ratio_max, worst);
    if (worst > kBoundSlack) atomicOr(err, KLA_DEVERR_BOUND);
  }
  // a wait gave up: let this CTA's own key copy land before it exits
  if (keys_in_flight) wait_bounded(&s.bar_tma, tma_phase);
  ptx::tc_fence_before();
  nbar_sync(bar_id);
  if (warp == 0) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tacc, 128);
  }
}


}  // namespace utb
}  // namespace kla
