// Per-chunk factors of the chunkwise prefill with a per-channel gate (KDA
// form, "Deep Dive into KDA", section 2.3), in parallel over all chunks of
// all heads, fp32 on CUDA cores.
//
// With G_s the in-chunk inclusive cumsum of the gate, one value per key
// channel i, and the decay before the erase, unrolling the recurrence over a
// chunk from its start state h gives (s, r token positions in the chunk):
//
//   A_rs = beta_r sum_i k_ri k_si e^{G_ri - G_si}      (s < r)
//   T    = (I + A)^{-1},   T' = T diag(beta)
//   U    = T' V,   W = T' (K o e^{G}),   V' = U - W h
//   o_r  = (q_r o e^{G_r})^T h + sum_{s <= r} P_rs V'_s,
//   P_rs = sum_i q_ri k_si e^{G_ri - G_si}             (s <= r)
//   h   <- Diag(e^{G_last}) h + (K o e^{G_last - G})^T V'
//
// The state kernel of the scalar-gate path runs the last three lines
// unchanged once it is handed W, P, the decayed keys and queries and the
// chunk decay; what the per-channel gate changes is A and P, whose decay no
// longer factors into one scalar mask.  They are summed here channel by
// channel with one exponential of a difference e^{G_ri - G_si} per term:
// every factor is at most 1 (G does not increase along the chunk), so no
// gate, however strong, overflows anything.  Every other decay used is also
// of that form (e^{G_r}, e^{G_last - G_s}).
//
// Output per chunk, in the byte layout the state kernel's shared-memory
// stage wants (128-byte swizzled bf16 rows, fetched with bulk copies):
//   [T'^T][P][W panels][Q o e^G panels][K o e^{G_last - G} panels][e^{G_last}]
// (see kda_tile_offsets in kla_chunk.h).
//
// A and P inside each 16-token sub-block are summed with one exponential per
// (pair, channel) in fp32; between sub-blocks the decay factors through the
// sub-block's first row (both factors <= 1) and those entries, like W, are
// bf16 warp-level tensor-core products with fp32 sums -- the same operand
// rounding the scalar-gate path applies to its Gram matrix and W.
#include "kla_chunk.h"
#include "kla_common.cuh"
#include "tile_sw128.cuh"

namespace kla {
namespace {

constexpr int C = 64;
constexpr int NT = 256;
constexpr int SB = 16;  // sub-block of rows sharing one decay reference

// Shared memory, two CTAs per SM.  Rows are padded so that the threads of a
// warp reading different rows at one channel (or the fragment loads of a
// tensor-core product) hit distinct banks: the token-major bf16 rows by 2
// elements (an odd number of words), the gate rows by 2 words (an even
// stride, so that two channels load as one 8-byte word: 16 rows then cover
// the 32 banks once), the bf16 operand rows by 8 elements.  The union follows the
// lifetimes: q, the sub-block operands and A live until T is formed; T and
// the operands of W after that (T's rows overlap only q and the sub-block
// operands, never A, which other warps may still be reading while T is
// written).
template <int DK>
struct KdaPrepHead {  // the operands that live before A in the first phase
  __nv_bfloat16 q[C][DK + 2];
  __nv_bfloat16 x[2 * SB][DK + 8];
  __nv_bfloat16 y[3 * SB][DK + 8];
};
constexpr size_t kInvBytes = 3 * C * (C + 8) * 2;  // the inverse's first operands

template <int DK>
struct KdaPrepSmem {
  __nv_bfloat16 k[C][DK + 2];  // keys, token-major (the bf16 inputs, exact)
  float g[C][DK + 2];          // G, the in-chunk cumsum of the gate, token-major
  union {
    struct {
      __nv_bfloat16 q[C][DK + 2];       // queries, token-major
      __nv_bfloat16 x[2 * SB][DK + 8];  // rows of one sub-block: k_ri e^{G_ri - G_ref,i},
                                        // then q_ri e^{G_ri - G_ref,i}
      __nv_bfloat16 y[3 * SB][DK + 8];  // k_si e^{G_ref,i - G_si}, s before the sub-block
      // A comes after the inverse's first operands, which are formed from it
      uint8_t pad[sizeof(KdaPrepHead<DK>) >= kInvBytes
                      ? 16
                      : kInvBytes - sizeof(KdaPrepHead<DK>) + 16];
      float a[C][C + 1];  // A, row r column s
    } p1;
    struct {  // the inverse: N = D A_O, X_{i+1} = D - N X_i (bf16 operands)
      __nv_bfloat16 d[C][C + 8];   // D = block-diagonal (I + A_D)^{-1}, row-major; then X_1^T
      __nv_bfloat16 xt[C][C + 8];  // X_0^T = D^T, then X_2^T
      __nv_bfloat16 aot[C][C + 8];  // A_O^T (A outside the diagonal blocks, transposed)
    } p3;
    struct {
      float t[C][C + 1];            // T = (I + A)^{-1}, then T' = T diag(beta)
      __nv_bfloat16 tb[C][C + 8];   // T', bf16
      __nv_bfloat16 kc[DK][C + 8];  // k_si e^{G_si}, channel-major
    } p2;
  } u;
  float beta[C];
};

// One warp-level tensor-core product D (16 x 8, fp32) += A (16 x 16) B (16 x 8),
// bf16 operands.  A is taken from a row-major tile (rows m0 .. m0 + 15,
// columns k0 .. k0 + 15), B from a tile holding B^T row-major (rows = the 8
// columns n0 .. n0 + 7 of B, columns k0 .. k0 + 15); `lda`, `ldb` elements
// per row.  Fragment ownership (PTX ISA, mma.m16n8k16): lane
// (g = lane / 4, t = lane % 4) holds A rows g and g + 8 at columns 2t, 2t + 1
// and 2t + 8, 2t + 9, B column n = g at rows 2t, 2t + 1 and 2t + 8, 2t + 9,
// and D rows g, g + 8 at columns 2t, 2t + 1.  The sub-block products here are
// 16 to 64 wide: too small for the CTA-level tcgen05 products and their
// tensor-memory round trip, a natural fit for warp-level products.
__device__ __forceinline__ void mma_16x8x16(float* d, const __nv_bfloat16* a, int lda, int m0,
                                            const __nv_bfloat16* bt, int ldb, int n0, int k0,
                                            int lane) {
  const int g = lane >> 2, t = lane & 3;
  auto w32 = [](const __nv_bfloat16* p) { return *reinterpret_cast<const uint32_t*>(p); };
  const uint32_t a0 = w32(a + (m0 + g) * lda + k0 + 2 * t);
  const uint32_t a1 = w32(a + (m0 + g + 8) * lda + k0 + 2 * t);
  const uint32_t a2 = w32(a + (m0 + g) * lda + k0 + 2 * t + 8);
  const uint32_t a3 = w32(a + (m0 + g + 8) * lda + k0 + 2 * t + 8);
  const uint32_t b0 = w32(bt + (n0 + g) * ldb + k0 + 2 * t);
  const uint32_t b1 = w32(bt + (n0 + g) * ldb + k0 + 2 * t + 8);
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
      "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Two consecutive bf16 values (4-byte aligned) as floats.
__device__ __forceinline__ float2 bf16x2_at(const __nv_bfloat16* p) {
  return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(p));
}

__device__ __forceinline__ void store_bf16_at(uint8_t* tile, int row, int col, float x) {
  reinterpret_cast<__nv_bfloat16*>(tile)[(sw128_chunk_off(row, col >> 3) >> 1) + (col & 7)] =
      __float2bfloat16_rn(x);
}

// Columns col, col + 1 (col even: one 4-byte word of an 8-column chunk).
__device__ __forceinline__ void store_bf16x2_at(uint8_t* tile, int row, int col, float x0,
                                                float x1) {
  *reinterpret_cast<uint32_t*>(tile + sw128_chunk_off(row, col >> 3) + 2 * (col & 7)) =
      pack_bf16x2(x0, x1);
}

__device__ __forceinline__ uint4 pack8(const float* x) {
  uint4 u;
  u.x = pack_bf16x2(x[0], x[1]);
  u.y = pack_bf16x2(x[2], x[3]);
  u.z = pack_bf16x2(x[4], x[5]);
  u.w = pack_bf16x2(x[6], x[7]);
  return u;
}

template <int DK>
__global__ void __launch_bounds__(NT, 2)
kda_prep_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
                const float* __restrict__ g, const float* __restrict__ eta, float eps,
                uint8_t* __restrict__ ws, int T, int H, int nchunks) {
  using Smem = KdaPrepSmem<DK>;
  extern __shared__ __align__(16) uint8_t smem_raw[];
  Smem& s = *reinterpret_cast<Smem*>(smem_raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int cidx = blockIdx.x;  // chunk (b * H + h) * nchunks + n
  const int head = cidx / nchunks, n = cidx % nchunks;
  const int b = head / H, hh = head % H;
  const int t0 = n * C;
  const KdaTileOffsets off = kda_tile_offsets(DK);
  uint8_t* out = ws + (size_t)cidx * off.total;
  uint8_t* outP = out + off.p;

  // ---- load (threads over channels; tokens past T are zero: an identity
  // step with g = 0, eta = 0)
  for (int p = tid; p < C * DK / 4; p += NT) {
    const int tok = p / (DK / 4), i0 = (p % (DK / 4)) * 4, t = t0 + tok;
    const size_t base = (((size_t)b * T + t) * H + hh) * DK + i0;
    float4 gv = make_float4(0.f, 0.f, 0.f, 0.f);
    uint2 kv = make_uint2(0, 0), qv = make_uint2(0, 0);
    if (t < T) {
      gv = *reinterpret_cast<const float4*>(g + base);
      kv = *reinterpret_cast<const uint2*>(k + base);
      qv = *reinterpret_cast<const uint2*>(q + base);
    }
    *reinterpret_cast<float2*>(&s.g[tok][i0]) = make_float2(gv.x, gv.y);
    *reinterpret_cast<float2*>(&s.g[tok][i0 + 2]) = make_float2(gv.z, gv.w);
    *reinterpret_cast<uint32_t*>(&s.k[tok][i0]) = kv.x;
    *reinterpret_cast<uint32_t*>(&s.k[tok][i0 + 2]) = kv.y;
    *reinterpret_cast<uint32_t*>(&s.u.p1.q[tok][i0]) = qv.x;
    *reinterpret_cast<uint32_t*>(&s.u.p1.q[tok][i0 + 2]) = qv.y;
  }
  __syncthreads();

  // ---- G: inclusive cumsum over the chunk per channel; beta per token
  if (tid < DK) {
    float acc = 0.f;
    for (int tok = 0; tok < C; ++tok) {
      acc += s.g[tok][tid];
      s.g[tok][tid] = acc;
    }
  } else if (tid >= 128 && tid < 128 + C) {
    const int tok = tid - 128, t = t0 + tok;
    float n2 = 0.f;
    for (int i = 0; i < DK; ++i) {
      const float x = __bfloat162float(s.k[tok][i]);
      n2 = fmaf(x, x, n2);
    }
    const size_t tk = ((size_t)b * T + t) * H + hh;
    s.beta[tok] = t < T ? step_size(eta[tk], n2, eps) : 0.f;
  }
  __syncthreads();

  // ---- Q o e^{G} (token rows in 64-column panels), written while the
  // queries are still in shared memory
  for (int p = tid; p < C * (DK / 8); p += NT) {
    const int tok = p / (DK / 8), i0 = (p % (DK / 8)) * 8;
    float x[8];
#pragma unroll
    for (int jj = 0; jj < 8; jj += 2) {
      const float2 gg = *reinterpret_cast<const float2*>(&s.g[tok][i0 + jj]);
      const float2 qq = bf16x2_at(&s.u.p1.q[tok][i0 + jj]);
      x[jj] = qq.x * __expf(gg.x);
      x[jj + 1] = qq.y * __expf(gg.y);
    }
    *reinterpret_cast<uint4*>(out + off.q + (i0 / 64) * 8192 +
                              sw128_chunk_off(tok, (i0 % 64) / 8)) = pack8(x);
  }

  // ---- diagonal sub-blocks of A (s < r) and P (s <= r), both tokens in one
  // sub-block: one thread per row and pair of columns (row rl of a sub-block
  // has rl / 2 + 1 pairs; a second column past the diagonal is computed as a
  // copy of the first and dropped: the zero fill below owns it), two
  // channels per step (the row's key, query and gate loads serve both
  // columns), one exponential per (pair, channel)
  constexpr int TPB = (SB / 2) * (SB / 2 + 1);  // tasks per sub-block
  for (int ti = tid; ti < (C / SB) * TPB; ti += NT) {
    const int blk = ti / TPB;
    int rem = ti % TPB, rl = 0;
    while (rem > rl / 2) {  // task index -> (row, column pair) inside the sub-block
      rem -= rl / 2 + 1;
      ++rl;
    }
    const int r = blk * SB + rl, s0 = blk * SB + 2 * rem;
    const bool two = s0 + 1 <= r;
    const int s1 = two ? s0 + 1 : s0;
    float a0 = 0.f, a1 = 0.f, p0 = 0.f, p1 = 0.f;
#pragma unroll 4
    for (int i = 0; i < DK; i += 2) {
      const float2 gr = *reinterpret_cast<const float2*>(&s.g[r][i]);
      const float2 g0 = *reinterpret_cast<const float2*>(&s.g[s0][i]);
      const float2 g1 = *reinterpret_cast<const float2*>(&s.g[s1][i]);
      const float2 kr = bf16x2_at(&s.k[r][i]), qr = bf16x2_at(&s.u.p1.q[r][i]);
      const float2 k0 = bf16x2_at(&s.k[s0][i]), k1 = bf16x2_at(&s.k[s1][i]);
      const float x00 = k0.x * __expf(gr.x - g0.x), x01 = k0.y * __expf(gr.y - g0.y);
      const float x10 = k1.x * __expf(gr.x - g1.x), x11 = k1.y * __expf(gr.y - g1.y);
      a0 = fmaf(kr.y, x01, fmaf(kr.x, x00, a0));
      p0 = fmaf(qr.y, x01, fmaf(qr.x, x00, p0));
      a1 = fmaf(kr.y, x11, fmaf(kr.x, x10, a1));
      p1 = fmaf(qr.y, x11, fmaf(qr.x, x10, p1));
    }
    s.u.p1.a[r][s0] = s0 < r ? s.beta[r] * a0 : 0.f;
    if (two) {
      s.u.p1.a[r][s1] = s1 < r ? s.beta[r] * a1 : 0.f;
      store_bf16x2_at(outP, r, s0, p0, p1);  // s0 even
    } else {
      store_bf16_at(outP, r, s0, p0);
    }
  }
  // zeros of P above the diagonal (s > r), by 16-byte chunks of 8 columns
  // where the whole chunk is above it (A above its diagonal is never read:
  // the inverse takes only its strictly lower part)
  for (int p = tid; p < C * (C / 8); p += NT) {
    const int r = p / (C / 8), c8 = p % (C / 8);
    if (8 * c8 > r)
      *reinterpret_cast<uint4*>(outP + sw128_chunk_off(r, c8)) = make_uint4(0u, 0u, 0u, 0u);
    else
      for (int sc = r + 1; sc < 8 * c8 + 8; ++sc) store_bf16_at(outP, r, sc, 0.f);
  }
  // ---- off-diagonal sub-blocks: for row sub-block R and s < 16 R the decay
  // factors through the reference G_ref = G at the sub-block's first row:
  // e^{G_ri - G_si} = e^{G_ri - G_ref,i} e^{G_ref,i - G_si}, both <= 1, so
  // these entries are dot products of pre-scaled rows (bf16, fp32 sums)
  for (int R = 1; R < C / SB; ++R) {
    const int r0 = R * SB, ns = r0;
    __syncthreads();  // the previous sub-block's products have read x, y
    for (int p = tid; p < SB * DK / 2; p += NT) {  // two channels per item
      const int rl = p / (DK / 2), i = 2 * (p % (DK / 2));
      const float2 gt = *reinterpret_cast<const float2*>(&s.g[r0 + rl][i]);
      const float2 gf = *reinterpret_cast<const float2*>(&s.g[r0][i]);
      const float2 kk = bf16x2_at(&s.k[r0 + rl][i]), qq = bf16x2_at(&s.u.p1.q[r0 + rl][i]);
      const float e0 = __expf(gt.x - gf.x), e1 = __expf(gt.y - gf.y);
      *reinterpret_cast<__nv_bfloat162*>(&s.u.p1.x[rl][i]) =
          __floats2bfloat162_rn(kk.x * e0, kk.y * e1);
      *reinterpret_cast<__nv_bfloat162*>(&s.u.p1.x[SB + rl][i]) =
          __floats2bfloat162_rn(qq.x * e0, qq.y * e1);
    }
    for (int p = tid; p < ns * DK / 2; p += NT) {
      const int sc = p / (DK / 2), i = 2 * (p % (DK / 2));
      const float2 gf = *reinterpret_cast<const float2*>(&s.g[r0][i]);
      const float2 gs = *reinterpret_cast<const float2*>(&s.g[sc][i]);
      const float2 kk = bf16x2_at(&s.k[sc][i]);
      *reinterpret_cast<__nv_bfloat162*>(&s.u.p1.y[sc][i]) =
          __floats2bfloat162_rn(kk.x * __expf(gf.x - gs.x), kk.y * __expf(gf.y - gs.y));
    }
    __syncthreads();
    // [A rows; P rows] (32 x ns) = x (32 x DK) y^T, in 16 x 8 tiles
    const int ntile = ns / 8;
    for (int task = warp; task < 2 * ntile; task += NT / 32) {
      const int mt = task / ntile, nt = task % ntile;
      float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int k0 = 0; k0 < DK; k0 += 16)
        mma_16x8x16(d, &s.u.p1.x[0][0], DK + 8, 16 * mt, &s.u.p1.y[0][0], DK + 8, 8 * nt, k0,
                    lane);
      const int gq = lane >> 2, tq = lane & 3;
#pragma unroll
      for (int h = 0; h < 2; ++h) {  // rows gq, gq + 8; columns 2 tq, 2 tq + 1
        const int r = r0 + gq + 8 * h, sc = 8 * nt + 2 * tq;
        if (mt == 0) {
          s.u.p1.a[r][sc] = s.beta[r] * d[2 * h];
          s.u.p1.a[r][sc + 1] = s.beta[r] * d[2 * h + 1];
        } else {
          store_bf16x2_at(outP, r, sc, d[2 * h], d[2 * h + 1]);
        }
      }
    }
  }
  __syncthreads();

  // ---- T = (I + A)^{-1} by 16-blocks: with A_D the diagonal 16 x 16
  // blocks of A, A_O the rest and D = (I + A_D)^{-1}, I + A = (I + A_D)(I + N)
  // with N = D A_O strictly block-lower (N^4 = 0), so
  // T = (I - N + N^2 - N^3) D:  X_0 = D, X_{i+1} = D - N X_i, T = X_3.
  // The blocks of D by forward substitution (fp32), N and the three Horner
  // products as bf16 warp-level tensor-core products with fp32 sums.
  static_assert(offsetof(Smem, u.p1.a) - offsetof(Smem, u) >= kInvBytes, "A after D, D^T, A_O^T");
  __nv_bfloat16 (*nbuf)[C + 8] = reinterpret_cast<__nv_bfloat16 (*)[C + 8]>(&s.u.p1.a[0][0]);
  if (tid < C) {  // thread (block R, column c): column c of (I + A_RR)^{-1}
    const int R = tid / SB, c = tid % SB, o0 = R * SB;
    float xcol[SB];
#pragma unroll
    for (int i = 0; i < SB; ++i) {
      float acc = 0.f;
#pragma unroll
      for (int m = 0; m < i; ++m) acc = fmaf(s.u.p1.a[o0 + i][o0 + m], xcol[m], acc);
      xcol[i] = i == c ? 1.f : (i < c ? 0.f : -acc);
    }
#pragma unroll
    for (int i = 0; i < SB; ++i) {
      s.u.p3.d[o0 + i][o0 + c] = __float2bfloat16_rn(xcol[i]);   // D, row-major
      s.u.p3.xt[o0 + c][o0 + i] = __float2bfloat16_rn(xcol[i]);  // D^T
    }
  }
  for (int p = tid; p < C * C; p += NT) {
    const int r = p / C, c = p % C;
    if (r / SB != c / SB) {  // zeros of D and D^T outside the diagonal blocks
      s.u.p3.d[r][c] = __float2bfloat16_rn(0.f);
      s.u.p3.xt[r][c] = __float2bfloat16_rn(0.f);
    }
    // A_O^T (threads on consecutive c read row r of A)
    s.u.p3.aot[c][r] = __float2bfloat16_rn(r / SB > c / SB ? s.u.p1.a[r][c] : 0.f);
  }
  __syncthreads();  // A is consumed: N may take its place
  // warp w: output rows 16 (w % 4), column tiles 2 (w / 4) .. + 1 of 8
  const int mt = warp & 3, nt0 = (warp >> 2) * 4;
  const int gq = lane >> 2, tq = lane & 3;
  {  // N = D A_O
    float dn[4][4] = {};
#pragma unroll
    for (int k0 = 0; k0 < C; k0 += 16)
#pragma unroll
      for (int q2 = 0; q2 < 4; ++q2)
        mma_16x8x16(dn[q2], &s.u.p3.d[0][0], C + 8, 16 * mt, &s.u.p3.aot[0][0], C + 8,
                    8 * (nt0 + q2), k0, lane);
#pragma unroll
    for (int q2 = 0; q2 < 4; ++q2)
#pragma unroll
      for (int e = 0; e < 4; ++e)
        nbuf[16 * mt + gq + 8 * (e >> 1)][8 * (nt0 + q2) + 2 * tq + (e & 1)] =
            __float2bfloat16_rn(dn[q2][e]);
  }
  // D at this thread's output positions, for the Horner combination
  float dloc[4][4];
#pragma unroll
  for (int q2 = 0; q2 < 4; ++q2)
#pragma unroll
    for (int e = 0; e < 4; ++e)
      dloc[q2][e] = __bfloat162float(
          s.u.p3.xt[8 * (nt0 + q2) + 2 * tq + (e & 1)][16 * mt + gq + 8 * (e >> 1)]);
  __syncthreads();  // N complete; D (row-major) is free for X_1^T
  float xr[4][4];
#pragma unroll
  for (int step = 0; step < 3; ++step) {
    // X_{step+1} = D - N X_step; X_step^T in xt (step 0, 2) or d (step 1)
    const __nv_bfloat16* xin = step == 1 ? &s.u.p3.d[0][0] : &s.u.p3.xt[0][0];
    __nv_bfloat16(*xout)[C + 8] = step == 0 ? s.u.p3.d : s.u.p3.xt;
#pragma unroll
    for (int q2 = 0; q2 < 4; ++q2)
#pragma unroll
      for (int e = 0; e < 4; ++e) xr[q2][e] = 0.f;
#pragma unroll
    for (int k0 = 0; k0 < C; k0 += 16)
#pragma unroll
      for (int q2 = 0; q2 < 4; ++q2)
        mma_16x8x16(xr[q2], &nbuf[0][0], C + 8, 16 * mt, xin, C + 8, 8 * (nt0 + q2), k0, lane);
#pragma unroll
    for (int q2 = 0; q2 < 4; ++q2)
#pragma unroll
      for (int e = 0; e < 4; ++e) xr[q2][e] = dloc[q2][e] - xr[q2][e];
    __syncthreads();  // every warp has read X_step
    if (step < 2) {
#pragma unroll
      for (int q2 = 0; q2 < 4; ++q2)
#pragma unroll
        for (int e = 0; e < 4; ++e)
          xout[8 * (nt0 + q2) + 2 * tq + (e & 1)][16 * mt + gq + 8 * (e >> 1)] =
              __float2bfloat16_rn(xr[q2][e]);
      __syncthreads();
    }
  }
  // T' = T diag(beta) in fp32 (T = X_3, still in registers)
#pragma unroll
  for (int q2 = 0; q2 < 4; ++q2)
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int r = 16 * mt + gq + 8 * (e >> 1), c = 8 * (nt0 + q2) + 2 * tq + (e & 1);
      s.u.p2.t[r][c] = xr[q2][e] * s.beta[c];
    }
  __syncthreads();

  // ---- T'^T rows (row c = column c of T'), K o e^{G_last - G}, e^{G_last},
  // and the bf16 operands of W
  if (tid < C) {
    float col[C];
#pragma unroll
    for (int r = 0; r < C; ++r) col[r] = s.u.p2.t[r][tid];
    sw128_store_row(out + off.tp, tid, col);
  }
  for (int p = tid; p < C * (DK / 8); p += NT) {
    const int tok = p / (DK / 8), i0 = (p % (DK / 8)) * 8;
    float x[8];
#pragma unroll
    for (int jj = 0; jj < 8; jj += 2) {
      const float2 gl = *reinterpret_cast<const float2*>(&s.g[C - 1][i0 + jj]);
      const float2 gt = *reinterpret_cast<const float2*>(&s.g[tok][i0 + jj]);
      const float2 kk = bf16x2_at(&s.k[tok][i0 + jj]);
      x[jj] = kk.x * __expf(gl.x - gt.x);
      x[jj + 1] = kk.y * __expf(gl.y - gt.y);
    }
    *reinterpret_cast<uint4*>(out + off.k + (i0 / 64) * 8192 +
                              sw128_chunk_off(tok, (i0 % 64) / 8)) = pack8(x);
  }
  if (tid < DK) reinterpret_cast<float*>(out + off.d)[tid] = __expf(s.g[C - 1][tid]);
  for (int p = tid; p < C * C; p += NT)
    s.u.p2.tb[p / C][p % C] = __float2bfloat16_rn(s.u.p2.t[p / C][p % C]);
  for (int p = tid; p < C * DK; p += NT) {  // threads on consecutive tokens
    const int tok = p % C, i = p / C;
    s.u.p2.kc[i][tok] = __float2bfloat16_rn(__bfloat162float(s.k[tok][i]) * __expf(s.g[tok][i]));
  }
  __syncthreads();

  // ---- W = T' (K o e^{G}) (64 x DK): warp w takes the 16 rows 16 (w % 4)
  // and NTW column tiles of 8 from 8 NTW (w / 4)
  {
    constexpr int NTW = DK / 16;
    const int mt = warp & 3, nt0 = (warp >> 2) * NTW;
    float d[NTW][4];
#pragma unroll
    for (int q2 = 0; q2 < NTW; ++q2)
#pragma unroll
      for (int e = 0; e < 4; ++e) d[q2][e] = 0.f;
#pragma unroll
    for (int k0 = 0; k0 < C; k0 += 16)
#pragma unroll
      for (int q2 = 0; q2 < NTW; ++q2)
        mma_16x8x16(d[q2], &s.u.p2.tb[0][0], C + 8, 16 * mt, &s.u.p2.kc[0][0], C + 8,
                    8 * (nt0 + q2), k0, lane);
    const int gq = lane >> 2, tq = lane & 3;
#pragma unroll
    for (int q2 = 0; q2 < NTW; ++q2)
#pragma unroll
      for (int h = 0; h < 2; ++h) {  // rows gq, gq + 8; channels 2 tq, 2 tq + 1
        const int r = 16 * mt + gq + 8 * h, i = 8 * (nt0 + q2) + 2 * tq;
        store_bf16x2_at(out + off.w + (i / 64) * 8192, r, i % 64, d[q2][2 * h],
                        d[q2][2 * h + 1]);
      }
  }
}

}  // namespace

cudaError_t launch_kda_prep(const void* q, const void* k, const float* g, const float* eta,
                            float eps, int B, int T, int H, int dk, void* ws,
                            cudaStream_t st) {
  const int nchunks = (T + C - 1) / C;
  const int total = B * H * nchunks;
  if (total == 0) return cudaSuccess;
  auto go = [&](auto kernel, size_t smem) -> cudaError_t {
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    kernel<<<total, NT, smem, st>>>((const __nv_bfloat16*)q, (const __nv_bfloat16*)k, g, eta,
                                    eps, (uint8_t*)ws, T, H, nchunks);
    return cudaGetLastError();
  };
  if (dk == 128) return go(kda_prep_kernel<128>, sizeof(KdaPrepSmem<128>));
  if (dk == 64) return go(kda_prep_kernel<64>, sizeof(KdaPrepSmem<64>));
  return cudaErrorNotSupported;
}

}  // namespace kla
