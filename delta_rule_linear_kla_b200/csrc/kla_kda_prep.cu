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
#include "kla_chunk.h"
#include "kla_common.cuh"
#include "tile_sw128.cuh"

namespace kla {
namespace {

constexpr int C = 64;
constexpr int NT = 512;
constexpr int SB = 16;  // sub-block of rows sharing one decay reference

// fp32 rows are padded to an odd number of words so that threads reading
// different rows at the same channel hit different banks.
template <int DK>
struct KdaPrepSmem {
  float k[C][DK + 1];          // keys, token-major
  float g[C][DK + 1];          // G (in-chunk cumsum of the gate), token-major
  __nv_bfloat16 q[C][DK + 2];  // queries, token-major
  union {
    struct {
      float xk[SB][DK + 1];   // k_ri e^{G_ri - G_ref,i}, rows of one sub-block
      float xq[SB][DK + 1];   // q_ri e^{G_ri - G_ref,i}
      float y[DK][3 * SB + 1];  // k_si e^{G_ref,i - G_si}, s before the sub-block
    } ap;
    float khat[C][DK + 1];  // k_si e^{G_si} (W)
  } u;
  float a[C][C + 1];  // A, row r column s
  float t[C][C + 1];  // T = (I + A)^{-1}, then T' = T diag(beta)
  float beta[C];
};

__device__ __forceinline__ void store_bf16_at(uint8_t* tile, int row, int col, float x) {
  reinterpret_cast<__nv_bfloat16*>(tile)[(sw128_chunk_off(row, col >> 3) >> 1) + (col & 7)] =
      __float2bfloat16_rn(x);
}

template <int DK>
__global__ void __launch_bounds__(NT, 1)
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
    float kx[4] = {0.f, 0.f, 0.f, 0.f};
    uint2 qv = make_uint2(0, 0);
    if (t < T) {
      gv = *reinterpret_cast<const float4*>(g + base);
      const uint2 kv = *reinterpret_cast<const uint2*>(k + base);
      const __nv_bfloat16* kb = reinterpret_cast<const __nv_bfloat16*>(&kv);
#pragma unroll
      for (int j = 0; j < 4; ++j) kx[j] = __bfloat162float(kb[j]);
      qv = *reinterpret_cast<const uint2*>(q + base);
    }
    s.g[tok][i0] = gv.x; s.g[tok][i0 + 1] = gv.y; s.g[tok][i0 + 2] = gv.z; s.g[tok][i0 + 3] = gv.w;
#pragma unroll
    for (int j = 0; j < 4; ++j) s.k[tok][i0 + j] = kx[j];
    const __nv_bfloat16* qb = reinterpret_cast<const __nv_bfloat16*>(&qv);
#pragma unroll
    for (int j = 0; j < 4; ++j) s.q[tok][i0 + j] = qb[j];
  }
  __syncthreads();

  // ---- G: inclusive cumsum over the chunk per channel; beta per token
  if (tid < DK) {
    float acc = 0.f;
    for (int tok = 0; tok < C; ++tok) {
      acc += s.g[tok][tid];
      s.g[tok][tid] = acc;
    }
  } else if (tid >= 256 && tid < 256 + C) {
    const int tok = tid - 256, t = t0 + tok;
    float n2 = 0.f;
    for (int i = 0; i < DK; ++i) n2 = fmaf(s.k[tok][i], s.k[tok][i], n2);
    const size_t tk = ((size_t)b * T + t) * H + hh;
    s.beta[tok] = t < T ? step_size(eta[tk], n2, eps) : 0.f;
  }
  __syncthreads();

  // ---- diagonal sub-blocks of A (s < r) and P (s <= r), both tokens in one
  // sub-block: one thread per pair, one exponential per channel
  constexpr int NPAIR = SB * (SB + 1) / 2;  // pairs per sub-block, s <= r
  for (int pi = tid; pi < (C / SB) * NPAIR; pi += NT) {
    const int blk = pi / NPAIR;
    int rem = pi % NPAIR, rl = 0;
    while (rem > rl) {  // pair index -> (row, column) inside the sub-block
      rem -= rl + 1;
      ++rl;
    }
    const int r = blk * SB + rl, sc = blk * SB + rem;
    float aa = 0.f, pp = 0.f;
#pragma unroll 4
    for (int i = 0; i < DK; ++i) {
      const float x = s.k[sc][i] * __expf(s.g[r][i] - s.g[sc][i]);
      aa = fmaf(s.k[r][i], x, aa);
      pp = fmaf(__bfloat162float(s.q[r][i]), x, pp);
    }
    s.a[r][sc] = sc < r ? s.beta[r] * aa : 0.f;
    store_bf16_at(outP, r, sc, pp);
  }
  // zeros of A and P above the diagonal (s > r)
  for (int p = tid; p < C * C; p += NT) {
    const int r = p / C, sc = p % C;
    if (sc > r) {
      s.a[r][sc] = 0.f;
      store_bf16_at(outP, r, sc, 0.f);
    }
  }
  // ---- off-diagonal sub-blocks: for row sub-block R and s < 16 R the decay
  // factors through the reference G_ref = G at the sub-block's first row:
  // e^{G_ri - G_si} = e^{G_ri - G_ref,i} e^{G_ref,i - G_si}, both <= 1.
  for (int R = 1; R < C / SB; ++R) {
    const int r0 = R * SB, ns = r0;
    __syncthreads();  // the previous sub-block's products have read xk, xq, y
    for (int p = tid; p < SB * DK; p += NT) {
      const int rl = p / DK, i = p % DK;
      const float e = __expf(s.g[r0 + rl][i] - s.g[r0][i]);
      s.u.ap.xk[rl][i] = s.k[r0 + rl][i] * e;
      s.u.ap.xq[rl][i] = __bfloat162float(s.q[r0 + rl][i]) * e;
    }
    for (int p = tid; p < ns * DK; p += NT) {
      const int sc = p / DK, i = p % DK;
      s.u.ap.y[i][sc] = s.k[sc][i] * __expf(s.g[r0][i] - s.g[sc][i]);
    }
    __syncthreads();
    // warp w: row r0 + w; lanes: columns lane, lane + 32 (< ns)
    {
      const int rl = warp, r = r0 + rl;
      const int s0 = lane, s1 = lane + 32;
      const bool on0 = s0 < ns, on1 = s1 < ns;
      float a0 = 0.f, a1 = 0.f, p0 = 0.f, p1 = 0.f;
#pragma unroll 4
      for (int i = 0; i < DK; ++i) {
        const float xk = s.u.ap.xk[rl][i], xq = s.u.ap.xq[rl][i];
        const float y0 = on0 ? s.u.ap.y[i][s0] : 0.f;
        const float y1 = on1 ? s.u.ap.y[i][s1] : 0.f;
        a0 = fmaf(xk, y0, a0);
        p0 = fmaf(xq, y0, p0);
        a1 = fmaf(xk, y1, a1);
        p1 = fmaf(xq, y1, p1);
      }
      const float br = s.beta[r];
      if (on0) {
        s.a[r][s0] = br * a0;
        store_bf16_at(outP, r, s0, p0);
      }
      if (on1) {
        s.a[r][s1] = br * a1;
        store_bf16_at(outP, r, s1, p1);
      }
    }
  }
  __syncthreads();

  // ---- T = (I + A)^{-1} by forward substitution, eight threads per column
  // c (they split the sum over m and combine it with three shuffles)
  {
    const int c = tid >> 3, j = tid & 7;
    for (int r = 0; r < C; ++r) {
      float part = 0.f;
      if (r > c)
        for (int m = c + j; m < r; m += 8) part = fmaf(s.a[r][m], s.t[m][c], part);
      part += __shfl_xor_sync(0xffffffffu, part, 1);
      part += __shfl_xor_sync(0xffffffffu, part, 2);
      part += __shfl_xor_sync(0xffffffffu, part, 4);
      if (j == 0) s.t[r][c] = r < c ? 0.f : (r == c ? 1.f : -part);
      __syncwarp();
    }
  }
  __syncthreads();
  // T' = T diag(beta), in place
  for (int p = tid; p < C * C; p += NT) s.t[p / C][p % C] *= s.beta[p % C];
  __syncthreads();

  // ---- T'^T rows (row c = column c of T'), K o e^{G_last - G},
  // e^{G_last}, Q o e^{G}, and K o e^{G} for W
  if (tid < C) {
    float col[C];
#pragma unroll
    for (int r = 0; r < C; ++r) col[r] = s.t[r][tid];
    sw128_store_row(out + off.tp, tid, col);
  }
  for (int p = tid; p < C * (DK / 8); p += NT) {
    const int tok = p / (DK / 8), i0 = (p % (DK / 8)) * 8;
    float xk[8], xq[8];
#pragma unroll
    for (int jj = 0; jj < 8; ++jj) {
      const int i = i0 + jj;
      xk[jj] = s.k[tok][i] * __expf(s.g[C - 1][i] - s.g[tok][i]);
      xq[jj] = __bfloat162float(s.q[tok][i]) * __expf(s.g[tok][i]);
    }
    uint4 uk, uq;
    uk.x = pack_bf16x2(xk[0], xk[1]); uk.y = pack_bf16x2(xk[2], xk[3]);
    uk.z = pack_bf16x2(xk[4], xk[5]); uk.w = pack_bf16x2(xk[6], xk[7]);
    uq.x = pack_bf16x2(xq[0], xq[1]); uq.y = pack_bf16x2(xq[2], xq[3]);
    uq.z = pack_bf16x2(xq[4], xq[5]); uq.w = pack_bf16x2(xq[6], xq[7]);
    const uint32_t o16 = (i0 / 64) * 8192 + sw128_chunk_off(tok, (i0 % 64) / 8);
    *reinterpret_cast<uint4*>(out + off.k + o16) = uk;
    *reinterpret_cast<uint4*>(out + off.q + o16) = uq;
  }
  if (tid < DK) reinterpret_cast<float*>(out + off.d)[tid] = __expf(s.g[C - 1][tid]);
  for (int p = tid; p < C * DK; p += NT) {
    const int tok = p / DK, i = p % DK;
    s.u.khat[tok][i] = s.k[tok][i] * __expf(s.g[tok][i]);
  }
  __syncthreads();

  // ---- W = T' (K o e^{G}): thread on channel i and four rows at a time
  {
    constexpr int RG = NT / DK;  // row groups
    const int i = tid % DK, rg = tid / DK;
    uint8_t* outW = out + off.w + (i / 64) * 8192;
    const int ic = i % 64;
    for (int r0 = 4 * rg; r0 < C; r0 += 4 * RG) {
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
      for (int sc = 0; sc <= r0 + 3; ++sc) {
        const float kh = s.u.khat[sc][i];
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) acc[jj] = fmaf(s.t[r0 + jj][sc], kh, acc[jj]);
      }
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) store_bf16_at(outW, r0 + jj, ic, acc[jj]);
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
