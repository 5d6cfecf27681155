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
constexpr int NT = 256;

template <int DK>
struct KdaPrepSmem {
  __nv_bfloat16 kt[DK][C];  // keys, channel-major: kt[i][s] = k_si
  float gt[DK][C];          // G, channel-major; later e^{G}
  union {
    struct {
      __nv_bfloat16 qs[C][DK];  // queries, token-major
      float a[C][C + 1];        // A
    } p1;
    float khat[C][DK];  // K o e^{G}, token-major (after A and Q o e^G are done)
  } u;
  float t[C][C + 1];  // T = (I + A)^{-1}
  float beta[C];
};

template <int DK>
__global__ void __launch_bounds__(NT, 2)
kda_prep_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
                const float* __restrict__ g, const float* __restrict__ eta, float eps,
                uint8_t* __restrict__ ws, int T, int H, int nchunks) {
  constexpr int NP = DK / 64;
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

  // ---- load: keys and gates transposed (lanes on consecutive tokens),
  // queries as they are; tokens past T are zero (an identity step)
  for (int p = tid; p < C * (DK / 8); p += NT) {
    const int tok = p % C, i0 = (p / C) * 8, t = t0 + tok;
    uint4 kv = make_uint4(0, 0, 0, 0);
    if (t < T) kv = *reinterpret_cast<const uint4*>(k + (((size_t)b * T + t) * H + hh) * DK + i0);
    const __nv_bfloat16* kb = reinterpret_cast<const __nv_bfloat16*>(&kv);
#pragma unroll
    for (int j = 0; j < 8; ++j) s.kt[i0 + j][tok] = kb[j];
  }
  for (int p = tid; p < C * (DK / 4); p += NT) {
    const int tok = p % C, i0 = (p / C) * 4, t = t0 + tok;
    float4 gv = make_float4(0.f, 0.f, 0.f, 0.f);
    if (t < T) gv = *reinterpret_cast<const float4*>(g + (((size_t)b * T + t) * H + hh) * DK + i0);
    s.gt[i0][tok] = gv.x;
    s.gt[i0 + 1][tok] = gv.y;
    s.gt[i0 + 2][tok] = gv.z;
    s.gt[i0 + 3][tok] = gv.w;
  }
  for (int p = tid; p < C * (DK / 8); p += NT) {
    const int tok = p / (DK / 8), i0 = (p % (DK / 8)) * 8, t = t0 + tok;
    uint4 qv = make_uint4(0, 0, 0, 0);
    if (t < T) qv = *reinterpret_cast<const uint4*>(q + (((size_t)b * T + t) * H + hh) * DK + i0);
    *reinterpret_cast<uint4*>(&s.u.p1.qs[tok][i0]) = qv;
  }
  __syncthreads();

  // ---- G: inclusive cumsum over the chunk, per channel; beta per token
  if (tid < DK) {
    float acc = 0.f;
    for (int tok = 0; tok < C; ++tok) {
      acc += s.gt[tid][tok];
      s.gt[tid][tok] = acc;
    }
  } else if (tid >= 128 && tid < 128 + C) {
    const int tok = tid - 128, t = t0 + tok;
    float n2 = 0.f;
    for (int i = 0; i < DK; ++i) {
      const float x = __bfloat162float(s.kt[i][tok]);
      n2 = fmaf(x, x, n2);
    }
    const size_t tk = ((size_t)b * T + t) * H + hh;
    s.beta[tok] = t < T ? step_size(eta[tk], n2, eps) : 0.f;
  }
  __syncthreads();

  // ---- A (s < r) and P (s <= r): warp w takes rows w, w + 8, ...; lane
  // takes columns lane and lane + 32
  uint8_t* outP = out + off.p;
  for (int r = warp; r < C; r += NT / 32) {
    float a0 = 0.f, a1 = 0.f, p0 = 0.f, p1 = 0.f;
    const int s0 = lane, s1 = lane + 32;
    const bool on0 = s0 <= r, on1 = s1 <= r;
#pragma unroll 4
    for (int i = 0; i < DK; ++i) {
      const float kr = __bfloat162float(s.kt[i][r]);
      const float qr = __bfloat162float(s.u.p1.qs[r][i]);
      const float gr = s.gt[i][r];
      if (on0) {
        const float x = __bfloat162float(s.kt[i][s0]) * __expf(gr - s.gt[i][s0]);
        a0 = fmaf(kr, x, a0);
        p0 = fmaf(qr, x, p0);
      }
      if (on1) {
        const float x = __bfloat162float(s.kt[i][s1]) * __expf(gr - s.gt[i][s1]);
        a1 = fmaf(kr, x, a1);
        p1 = fmaf(qr, x, p1);
      }
    }
    const float br = s.beta[r];
    s.u.p1.a[r][s0] = s0 < r ? br * a0 : 0.f;
    s.u.p1.a[r][s1] = s1 < r ? br * a1 : 0.f;
    // P row r, bf16, swizzled (column s: 16-byte chunk s / 8, element s % 8)
    __nv_bfloat16* prow = reinterpret_cast<__nv_bfloat16*>(outP);
    prow[(sw128_chunk_off(r, s0 >> 3) >> 1) + (s0 & 7)] = __float2bfloat16_rn(on0 ? p0 : 0.f);
    prow[(sw128_chunk_off(r, s1 >> 3) >> 1) + (s1 & 7)] = __float2bfloat16_rn(on1 ? p1 : 0.f);
  }
  __syncthreads();

  // ---- T = (I + A)^{-1} by forward substitution, four threads per column
  // c (they split the sum over m and combine it with two shuffles)
  {
    const int c = tid >> 2, j = tid & 3;
    for (int r = 0; r < C; ++r) {
      float part = 0.f;
      if (r > c)
        for (int m = c + j; m < r; m += 4) part = fmaf(s.u.p1.a[r][m], s.t[m][c], part);
      part += __shfl_xor_sync(0xffffffffu, part, 1);
      part += __shfl_xor_sync(0xffffffffu, part, 2);
      if (j == 0) s.t[r][c] = r < c ? 0.f : (r == c ? 1.f : -part);
      __syncwarp();
    }
  }
  __syncthreads();

  // ---- T'^T rows: row c = beta_c (column c of T)
  if (tid < C) {
    const int c = tid;
    const float bc = s.beta[c];
    float col[C];
#pragma unroll
    for (int r = 0; r < C; ++r) col[r] = bc * s.t[r][c];
    sw128_store_row(out + off.tp, c, col);
  }
  // ---- K o e^{G_last - G}, token rows in 64-column panels, and e^{G_last}
  for (int p = tid; p < C * (DK / 8); p += NT) {
    const int tok = p % C, i0 = (p / C) * 8;
    float x[8];
#pragma unroll
    for (int jj = 0; jj < 8; ++jj) {
      const int i = i0 + jj;
      x[jj] = __bfloat162float(s.kt[i][tok]) * __expf(s.gt[i][C - 1] - s.gt[i][tok]);
    }
    uint4 u4;
    u4.x = pack_bf16x2(x[0], x[1]);
    u4.y = pack_bf16x2(x[2], x[3]);
    u4.z = pack_bf16x2(x[4], x[5]);
    u4.w = pack_bf16x2(x[6], x[7]);
    *reinterpret_cast<uint4*>(out + off.k + (i0 / 64) * 8192 +
                              sw128_chunk_off(tok, (i0 % 64) / 8)) = u4;
  }
  if (tid < DK) reinterpret_cast<float*>(out + off.d)[tid] = __expf(s.gt[tid][C - 1]);
  __syncthreads();

  // ---- e^{G} in place, then Q o e^{G}
  for (int p = tid; p < DK * C; p += NT) s.gt[p / C][p % C] = __expf(s.gt[p / C][p % C]);
  __syncthreads();
  for (int p = tid; p < C * (DK / 8); p += NT) {
    const int tok = p % C, i0 = (p / C) * 8;
    float x[8];
#pragma unroll
    for (int jj = 0; jj < 8; ++jj)
      x[jj] = __bfloat162float(s.u.p1.qs[tok][i0 + jj]) * s.gt[i0 + jj][tok];
    uint4 u4;
    u4.x = pack_bf16x2(x[0], x[1]);
    u4.y = pack_bf16x2(x[2], x[3]);
    u4.z = pack_bf16x2(x[4], x[5]);
    u4.w = pack_bf16x2(x[6], x[7]);
    *reinterpret_cast<uint4*>(out + off.q + (i0 / 64) * 8192 +
                              sw128_chunk_off(tok, (i0 % 64) / 8)) = u4;
  }
  __syncthreads();  // Q and A are dead: their space becomes K o e^{G}
  for (int p = tid; p < C * DK; p += NT) {
    const int tok = p % C, i = p / C;
    s.u.khat[tok][i] = __bfloat162float(s.kt[i][tok]) * s.gt[i][tok];
  }
  __syncthreads();

  // ---- W = T' (K o e^{G}): thread on channel i, rows r = row0, row0 + RS, ...
  {
    constexpr int RS = NT / DK;  // row groups
    const int i = tid % DK, row0 = tid / DK;
    uint8_t* outW = out + off.w + (i / 64) * 8192;
    const int ic = i % 64;
    for (int r = row0; r < C; r += RS) {
      float acc = 0.f;
      for (int sc = 0; sc <= r; ++sc) acc = fmaf(s.t[r][sc] * s.beta[sc], s.u.khat[sc][i], acc);
      reinterpret_cast<__nv_bfloat16*>(outW)[(sw128_chunk_off(r, ic >> 3) >> 1) + (ic & 7)] =
          __float2bfloat16_rn(acc);
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
