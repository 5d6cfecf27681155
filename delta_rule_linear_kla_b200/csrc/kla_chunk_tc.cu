// Chunkwise KLA prefill on sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// Two kernels.  The UT kernel (kla_ut.cu) runs first, in parallel over every
// chunk, and leaves T' = T diag(beta) and T'' = T diag(beta e^G) of each chunk
// in the workspace, where T = (I + A)^{-1} and
// A = strict_lower(diag(beta) K K^T (*) e^{G_r - G_s}).  The chain kernel here
// has one CTA per head (b, h) and 64-column slab of the state h = S^T
// ([DK][DV] fp32) and walks the sequence chunk by chunk (C = 64 tokens),
// keeping its fp32 state slab in registers.  Per chunk ("Deep Dive into
// KDA", section 3, specialised to a scalar gate, with the KLA step size of
// "Kaczmarz Linear Attention", Abstract):
//
//   G_r = sum_{j<=r} g_j  (in chunk)
//   P  = lower_incl(Q K^T (*) e^{G_r - G_s})                          [MMA 1]
//   W  = T'' K,  U = T' V                                             [MMA 2,3]
//   X  = [W; Q] h          (rows 0..63: W h, rows 64..127: Q h)       [MMA 4]
//   V' = U - W h
//   h <- e^{G_63} h + K^T diag(e^{G_63 - G_s}) V'                      [MMA 5]
//   O  = diag(e^G) Q h + P V'                                         [MMA 6]
//
// The decay ratios are only formed as masked differences of G (never
// K / Gamma), so strong gates cannot overflow.  A ragged tail is zero-filled
// by TMA and given g = 0 (and eta = 0 in the UT kernel): an identity step.
//
// All contractions are single-CTA tcgen05.mma with M = 128, bf16 operands in
// 128-byte swizzled shared-memory panels and fp32 accumulators in TMEM (lane
// = row; 64-row products are stacked or padded to 128 lanes):
//   MMA 1  D_S [128x64]  = [W_stale; Q] . K^T   A, B K-major  (lanes 64..127)
//   MMA 2  D_W [128xDK]  = [T''; P] . K          B MN-major    (lanes 0..63)
//   MMA 3  D_U [128x64]  = [T'; T''] . V         B MN-major    (lanes 0..63)
//   MMA 4  D_X [128x64]  = [W; Q] . h            B MN-major
//   MMA 5  D_H [128x64]  = K^T . (decay V')      A, B MN-major (lanes < DK)
//   MMA 6  D_PV[128x64]  = [T''; P] . V'         B MN-major    (lanes 64..127)
//
// Warp roles (320 threads), synchronised only through mbarriers:
//   warp 0      TMA producer: K, Q, V slab and the UT tiles of chunk n into
//               stage n % 2 (double buffered).
//   warp 1      MMA issuer (one thread).  Per iteration n it issues the chain
//               MMAs of chunk n (4, then 5 and 6) interleaved with the
//               state-independent MMAs of chunk n + 1 (1, then 2 and 3), so
//               the tensor pipe works on chunk n + 1 while the chain warps
//               run chunk n's epilogues.
//   warps 2..5  "next-chunk" epilogues: the gate cumsum G, P (lanes 64..127)
//               and W (lanes 0..63), written into the stage's P and W slots.
//   warps 6..9  "chain" epilogues: V' (lanes 0..63), the state update (lanes
//               < DK) and the output rows (lanes 64..127).
// Every wait is bounded (about 2 s); on timeout the kernel raises the device
// error word, stops all roles, drains its own TMA loads and frees TMEM.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "kla_chunk.h"
#include "kla_common.cuh"
#include "kla_sync.cuh"
#include "ptx_sm100.cuh"
#include "tile_sw128.cuh"

namespace kla {
namespace {

constexpr int C = 64;       // chunk length
constexpr int BV = 64;      // state columns per CTA
constexpr int NTHREADS = 320;
constexpr uint32_t TMEM_COLS = 512;
// TMEM column offsets of the accumulators
constexpr uint32_t COL_S = 0, COL_W = 64, COL_U = 192 /* 2 buffers */, COL_X = 320,
                   COL_H = 384, COL_PV = 448;

// One pipeline stage.  Per 64-column key panel: [W rows | Q rows | K rows]
// (8 KB each), so [W; Q] is one 128-row K-major operand.  Then the V slab and
// [T' | T'' | P]: MMA A operands take 128 rows starting at T' or T''.
template <int DK>
struct alignas(1024) Stage {
  static constexpr int NP = DK / 64;
  uint8_t panel[NP][3][8192];
  uint8_t v[8192];
  uint8_t tp[3][8192];
};

template <int DK>
struct alignas(1024) ChainSmem {
  Stage<DK> st[2];
  uint8_t hm[DK * 128];  // bf16 state slab (MMA 4 operand), row i = key index
  uint8_t vp[8192];      // V'
  uint8_t vpd[8192];     // V' scaled by e^{G_63 - G_s}
  float G[3][C];         // gate cumsum of chunk n in slot n % 3
  uint64_t full[2], empty[2];
  uint64_t bS, bWU, bX, bHP;             // MMA completions
  uint64_t p_done, w_done, vp_ready;     // epilogue -> MMA
  uint64_t u_free[2], x_free, h_done, pv_free;
  uint64_t g_ready[3];
  uint64_t mma_drain;
  uint32_t tmem_base;
  int abort_flag;
};

enum Slot { SW = 0, SQ = 1, SK = 2 };

// Bounded wait that also gives up as soon as another role has aborted.
__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity,
                                              volatile int* abort_flag) {
  if (ptx::mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 64; ++i)
      if (ptx::mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (globaltimer() - t0 > kWaitLimitNs) {
      *abort_flag = 1;
      return false;
    }
  }
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(ptx::smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void named_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

template <int DK>
__global__ void __launch_bounds__(NTHREADS, 1)
chain_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
             const __grid_constant__ CUtensorMap tm_v, const float* __restrict__ g,
             const float* __restrict__ h0, __nv_bfloat16* __restrict__ o,
             float* __restrict__ hT, int T, int H, int DV, const uint8_t* __restrict__ ws,
             unsigned int* err) {
  using Smem = ChainSmem<DK>;
  constexpr int NP = Stage<DK>::NP;
  constexpr uint32_t PANEL = 3 * 8192;  // byte stride between key panels
  extern __shared__ uint8_t smem_raw[];
  Smem& s = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                     ~uintptr_t(1023));
  volatile int* abort_flag = &s.abort_flag;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int slab = blockIdx.x, hh = blockIdx.y, b = blockIdx.z;
  const int nchunks = (T + C - 1) / C;
  const size_t head = (size_t)b * H + hh;
  // TMEM lane group this warp may access, and the row it stands for
  const int row = 32 * (warp & 3) + lane;
  const uint32_t lane_base = (uint32_t)(32 * (warp & 3)) << 16;

  if (warp == 0) {
    ptx::tmem_alloc(&s.tmem_base, TMEM_COLS);
    ptx::tmem_relinquish();
  }
  if (tid == 32) {
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(&s.full[i], 1);
      ptx::mbar_init(&s.empty[i], 1);
      ptx::mbar_init(&s.u_free[i], 2);
    }
    ptx::mbar_init(&s.bS, 1);
    ptx::mbar_init(&s.bWU, 1);
    ptx::mbar_init(&s.bX, 1);
    ptx::mbar_init(&s.bHP, 1);
    ptx::mbar_init(&s.p_done, 2);
    ptx::mbar_init(&s.w_done, 2);
    ptx::mbar_init(&s.vp_ready, 2);
    ptx::mbar_init(&s.x_free, 4);
    ptx::mbar_init(&s.h_done, 4);
    ptx::mbar_init(&s.pv_free, 2);
    for (int i = 0; i < 3; ++i) ptx::mbar_init(&s.g_ready[i], 2);
    ptx::mbar_init(&s.mma_drain, 1);
    ptx::mbar_init_fence();
    s.abort_flag = 0;
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tb = s.tmem_base;

  if (warp == 0) {
    // =========================== TMA producer ===========================
    if (lane == 0) {
      ptx::prefetch_tensormap(&tm_q);
      ptx::prefetch_tensormap(&tm_k);
      ptx::prefetch_tensormap(&tm_v);
      constexpr uint32_t BYTES = (uint32_t)(2 * NP * 8192 + 8192 + kUtTileBytes);
      const uint8_t* ws_head = ws + head * (size_t)nchunks * kUtTileBytes;
      int issued = 0, drained = 0;
      for (int n = 0; n < nchunks; ++n) {
        const int st = n & 1;
        if (n >= 2) {
          if (!wait_or_abort(&s.empty[st], (uint32_t)(((n - 2) >> 1) & 1), abort_flag)) break;
          drained = n - 1;  // chunks up to n-2 fully consumed
        }
        Stage<DK>& S = s.st[st];
        ptx::mbar_arrive_expect_tx(&s.full[st], BYTES);
        ptx::bulk_load(S.tp[0], ws_head + (size_t)n * kUtTileBytes, (uint32_t)kUtTileBytes,
                       &s.full[st]);
#pragma unroll
        for (int p = 0; p < NP; ++p) {
          ptx::tma_load_4d(S.panel[p][SK], &tm_k, &s.full[st], p * 64, hh, n * C, b);
          ptx::tma_load_4d(S.panel[p][SQ], &tm_q, &s.full[st], p * 64, hh, n * C, b);
        }
        ptx::tma_load_4d(S.v, &tm_v, &s.full[st], slab * BV, hh, n * C, b);
        issued = n + 1;
      }
      if (*abort_flag) {
        // let this CTA's own copies land before the CTA goes away
        for (int n = drained; n < issued; ++n)
          if (!wait_bounded(&s.full[n & 1], (uint32_t)((n >> 1) & 1))) break;
      }
    }
  } else if (warp == 1) {
    // ============================ MMA issuer ============================
    if (lane == 0) {
      constexpr uint32_t id_s = ptx::idesc_bf16(128, 64, 0, 0);
      constexpr uint32_t id_w = ptx::idesc_bf16(128, DK, 0, 1);
      constexpr uint32_t id_64 = ptx::idesc_bf16(128, 64, 0, 1);
      constexpr uint32_t id_h = ptx::idesc_bf16(128, 64, 1, 1);
      auto mma1 = [&](int n) {  // D_S = [W_stale; Q] K^T
        Stage<DK>& S = s.st[n & 1];
#pragma unroll
        for (int kk = 0; kk < DK / 16; ++kk) {
          const uint32_t a = ptx::smem_u32(S.panel[kk >> 2][SW]) + (kk & 3) * 32;
          const uint32_t bk = ptx::smem_u32(S.panel[kk >> 2][SK]) + (kk & 3) * 32;
          ptx::mma_bf16(tb + COL_S, ptx::sdesc_sw128(a, 16, 1024), ptx::sdesc_sw128(bk, 16, 1024),
                        id_s, kk > 0);
        }
        ptx::mma_commit(&s.bS);
      };
      auto mma23 = [&](int n) {  // D_W = [T''; P] K ;  D_U[n%2] = [T'; T''] V
        Stage<DK>& S = s.st[n & 1];
#pragma unroll
        for (int kk = 0; kk < C / 16; ++kk) {
          const uint32_t a = ptx::smem_u32(S.tp[1]) + kk * 32;
          const uint32_t bk = ptx::smem_u32(S.panel[0][SK]) + kk * 2048;
          ptx::mma_bf16(tb + COL_W, ptx::sdesc_sw128(a, 16, 1024),
                        ptx::sdesc_sw128(bk, PANEL, 1024), id_w, kk > 0);
        }
#pragma unroll
        for (int kk = 0; kk < C / 16; ++kk) {
          const uint32_t a = ptx::smem_u32(S.tp[0]) + kk * 32;
          const uint32_t bv = ptx::smem_u32(S.v) + kk * 2048;
          ptx::mma_bf16(tb + COL_U + 64 * (n & 1), ptx::sdesc_sw128(a, 16, 1024),
                        ptx::sdesc_sw128(bv, 1024, 1024), id_64, kk > 0);
        }
        ptx::mma_commit(&s.bWU);
      };
      bool ok = nchunks > 0;
      if (ok) ok = wait_or_abort(&s.full[0], 0, abort_flag);
      if (ok) {
        ptx::tc_fence_after();
        mma1(0);
        mma23(0);
      }
      for (int n = 0; n < nchunks && ok; ++n) {
        Stage<DK>& S = s.st[n & 1];
        const uint32_t par = (uint32_t)(n & 1);
        // ---- MMA 4 (chunk n): needs W(n), h_n, and D_X free
        if (!wait_or_abort(&s.w_done, par, abort_flag)) break;
        if (!wait_or_abort(&s.h_done, par, abort_flag)) break;
        if (n > 0 && !wait_or_abort(&s.x_free, par ^ 1u, abort_flag)) break;
        ptx::tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < DK / 16; ++kk) {
          const uint32_t a = ptx::smem_u32(S.panel[kk >> 2][SW]) + (kk & 3) * 32;
          const uint32_t bh = ptx::smem_u32(s.hm) + kk * 2048;
          ptx::mma_bf16(tb + COL_X, ptx::sdesc_sw128(a, 16, 1024),
                        ptx::sdesc_sw128(bh, 1024, 1024), id_64, kk > 0);
        }
        ptx::mma_commit(&s.bX);
        // ---- MMA 1 (chunk n+1): needs its data and D_S free (P(n) read)
        if (!wait_or_abort(&s.p_done, par, abort_flag)) break;
        if (n + 1 < nchunks) {
          if (!wait_or_abort(&s.full[(n + 1) & 1], (uint32_t)(((n + 1) >> 1) & 1), abort_flag))
            break;
          ptx::tc_fence_after();
          mma1(n + 1);
        }
        // ---- MMA 5, 6 (chunk n): need V'(n), P(n), D_PV free
        if (!wait_or_abort(&s.vp_ready, par, abort_flag)) break;
        if (n > 0 && !wait_or_abort(&s.pv_free, par ^ 1u, abort_flag)) break;
        ptx::tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < C / 16; ++kk) {
          const uint32_t a = ptx::smem_u32(S.panel[0][SK]) + kk * 2048;
          const uint32_t bv = ptx::smem_u32(s.vpd) + kk * 2048;
          ptx::mma_bf16(tb + COL_H, ptx::sdesc_sw128(a, PANEL, 1024),
                        ptx::sdesc_sw128(bv, 1024, 1024), id_h, kk > 0);
        }
#pragma unroll
        for (int kk = 0; kk < C / 16; ++kk) {
          const uint32_t a = ptx::smem_u32(S.tp[1]) + kk * 32;
          const uint32_t bv = ptx::smem_u32(s.vp) + kk * 2048;
          ptx::mma_bf16(tb + COL_PV, ptx::sdesc_sw128(a, 16, 1024),
                        ptx::sdesc_sw128(bv, 1024, 1024), id_64, kk > 0);
        }
        ptx::mma_commit(&s.bHP);
        ptx::mma_commit(&s.empty[n & 1]);
        // ---- MMA 2, 3 (chunk n+1): need D_W free (w_done(n) seen above) and
        //      D_U[(n+1)%2] free (V'(n-1) done)
        if (n + 1 < nchunks) {
          if (n >= 1 &&
              !wait_or_abort(&s.u_free[(n + 1) & 1], (uint32_t)(((n - 1) >> 1) & 1), abort_flag))
            break;
          ptx::tc_fence_after();
          mma23(n + 1);
        }
      }
      // every MMA this thread issued has finished before TMEM is released
      ptx::mma_commit(&s.mma_drain);
      wait_bounded(&s.mma_drain, 0);
    }
  } else if (warp < 6) {
    // ===================== next-chunk epilogues (P, W) ===================
    const bool p_rows = row >= 64;  // warps 2, 3
    for (int n = 0; n < nchunks; ++n) {
      Stage<DK>& S = s.st[n & 1];
      float* Gn = s.G[n % 3];
      const uint32_t par = (uint32_t)(n & 1);
      if (p_rows) {
        // gate cumsum of chunk n (warps 2, 3: token r = row - 64)
        const int r = row - 64, t = n * C + r;
        float x = (t < T) ? g[((size_t)b * T + t) * H + hh] : 0.f;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
          const float y = __shfl_up_sync(0xffffffffu, x, off);
          if (lane >= off) x += y;
        }
        Gn[r] = x;
        named_sync(1, 64);
        if (r >= 32) Gn[r] = x + Gn[31];
        named_sync(1, 64);
        __syncwarp();
        if (lane == 0) mbar_arrive(&s.g_ready[n % 3]);
        // P row r
        if (!wait_or_abort(&s.bS, par, abort_flag)) break;
        ptx::tc_fence_after();
        const float Gr = Gn[r];
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          float srow[32];
          ptx::tmem_ld32(tb + lane_base + COL_S + 32 * hf, srow);
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            const int cc = 32 * hf + c;
            srow[c] = (cc <= r) ? srow[c] * __expf(Gr - Gn[cc]) : 0.f;
          }
          sw128_store_row32(S.tp[2], r, hf, srow);
        }
        ptx::fence_proxy_async_smem();
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&s.p_done);
      } else {
        // W row `row` (0..63)
        if (!wait_or_abort(&s.bWU, par, abort_flag)) break;
        ptx::tc_fence_after();
#pragma unroll
        for (int p = 0; p < NP; ++p) {
#pragma unroll
          for (int hf = 0; hf < 2; ++hf) {
            float w[32];
            ptx::tmem_ld32(tb + lane_base + COL_W + p * 64 + 32 * hf, w);
            sw128_store_row32(S.panel[p][SW], row, hf, w);
          }
        }
        ptx::fence_proxy_async_smem();
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&s.w_done);
      }
    }
  } else {
    // ========================= chain epilogues ==========================
    const bool has_h = row < DK;
    float hreg[BV];
    if (has_h) {
      if (h0) {
        const float4* src =
            reinterpret_cast<const float4*>(h0 + (head * DK + row) * DV + slab * BV);
#pragma unroll
        for (int j = 0; j < BV / 4; ++j) {
          const float4 x = src[j];
          hreg[4 * j] = x.x; hreg[4 * j + 1] = x.y; hreg[4 * j + 2] = x.z; hreg[4 * j + 3] = x.w;
        }
      } else {
#pragma unroll
        for (int j = 0; j < BV; ++j) hreg[j] = 0.f;
      }
      sw128_store_row(s.hm, row, hreg);
      ptx::fence_proxy_async_smem();
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&s.h_done);  // h_0 is in place
    const bool v_rows = row < 64;           // warps 8, 9
    bool ok = true;
    for (int n = 0; n < nchunks && ok; ++n) {
      const float* Gn = s.G[n % 3];
      const uint32_t par = (uint32_t)(n & 1);
      if (!wait_or_abort(&s.g_ready[n % 3], (uint32_t)((n / 3) & 1), abort_flag)) { ok = false; break; }
      const float gC = Gn[C - 1];
      if (!wait_or_abort(&s.bX, par, abort_flag)) { ok = false; break; }
      ptx::tc_fence_after();
      if (v_rows) {
        // V'_r = U_r - (W h)_r, and its copy decayed to the chunk end
        const float dec = __expf(gC - Gn[row]);
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          float u[32], x[32];
          ptx::tmem_ld32(tb + lane_base + COL_U + 64 * (n & 1) + 32 * hf, u);
          ptx::tmem_ld32(tb + lane_base + COL_X + 32 * hf, x);
#pragma unroll
          for (int j = 0; j < 32; ++j) u[j] -= x[j];
          sw128_store_row32(s.vp, row, hf, u);
#pragma unroll
          for (int j = 0; j < 32; ++j) u[j] *= dec;
          sw128_store_row32(s.vpd, row, hf, u);
        }
        ptx::tc_fence_before();
        ptx::fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&s.u_free[n & 1]);
          mbar_arrive(&s.x_free);
          mbar_arrive(&s.vp_ready);
        }
      }
      if (!wait_or_abort(&s.bHP, par, abort_flag)) { ok = false; break; }
      ptx::tc_fence_after();
      if (has_h) {
        const float a = __expf(gC);
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          float dh[32];
          ptx::tmem_ld32(tb + lane_base + COL_H + 32 * hf, dh);
#pragma unroll
          for (int j = 0; j < 32; ++j) hreg[32 * hf + j] = fmaf(a, hreg[32 * hf + j], dh[j]);
        }
        sw128_store_row(s.hm, row, hreg);
        ptx::fence_proxy_async_smem();
      }
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s.h_done);  // h_{n+1} in place, D_H read
      if (!v_rows) {
        // output row r = row - 64: o_r = e^{G_r} (Q h)_r + (P V')_r
        const int r = row - 64, t = n * C + r;
        const float e = __expf(Gn[r]);
        uint4* dst = reinterpret_cast<uint4*>(o + (((size_t)b * T + t) * H + hh) * DV + slab * BV);
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          float x[32], pv[32];
          ptx::tmem_ld32(tb + lane_base + COL_X + 32 * hf, x);
          ptx::tmem_ld32(tb + lane_base + COL_PV + 32 * hf, pv);
          if (t < T) {
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              uint4 u4;
              u4.x = pack_bf16x2(fmaf(e, x[8 * c + 0], pv[8 * c + 0]), fmaf(e, x[8 * c + 1], pv[8 * c + 1]));
              u4.y = pack_bf16x2(fmaf(e, x[8 * c + 2], pv[8 * c + 2]), fmaf(e, x[8 * c + 3], pv[8 * c + 3]));
              u4.z = pack_bf16x2(fmaf(e, x[8 * c + 4], pv[8 * c + 4]), fmaf(e, x[8 * c + 5], pv[8 * c + 5]));
              u4.w = pack_bf16x2(fmaf(e, x[8 * c + 6], pv[8 * c + 6]), fmaf(e, x[8 * c + 7], pv[8 * c + 7]));
              dst[4 * hf + c] = u4;
            }
          }
        }
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&s.x_free);
          mbar_arrive(&s.pv_free);
        }
      }
    }
    if (ok && has_h && hT) {
      float4* dst = reinterpret_cast<float4*>(hT + (head * DK + row) * DV + slab * BV);
#pragma unroll
      for (int j = 0; j < BV / 4; ++j)
        dst[j] = make_float4(hreg[4 * j], hreg[4 * j + 1], hreg[4 * j + 2], hreg[4 * j + 3]);
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (tid == 0 && s.abort_flag) report_timeout(err);
  if (warp == 0) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tb, TMEM_COLS);
  }
}

// ------------------------------------------------------------------ host
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = (PFN_cuTensorMapEncodeTiled_v12000)p;
  }
  return fn;
}

// [B][T][H][d] bf16 tensor, boxes of 64 (d) x 64 (t) for one (b, h).
bool make_map(CUtensorMap* m, const void* base, int d, int H, int T, int B) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
  cuuint64_t strides[3] = {(cuuint64_t)d * 2, (cuuint64_t)H * d * 2, (cuuint64_t)T * H * d * 2};
  cuuint32_t box[4] = {64, 1, (cuuint32_t)C, 1};
  cuuint32_t es[4] = {1, 1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box,
            es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int DK>
cudaError_t launch_dk(const void* q, const void* k, const void* v, const float* g,
                      const float* eta, float eps, const float* h0, void* o, float* hT, int B,
                      int T, int H, int DV, uint8_t* ws, unsigned int* err, cudaStream_t st) {
  CUtensorMap mq, mk, mv;
  if (!make_map(&mq, q, DK, H, T, B) || !make_map(&mk, k, DK, H, T, B) ||
      !make_map(&mv, v, DV, H, T, B))
    return cudaErrorInvalidValue;
  cudaError_t eu = launch_ut(mk, g, eta, eps, ws, B, T, H, DK, err, st);
  if (eu != cudaSuccess) return eu;
  const size_t smem = sizeof(ChainSmem<DK>) + 1024;
  static bool attr_set[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(chain_kernel<DK>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  dim3 grid(DV / BV, H, B);
  chain_kernel<DK><<<grid, NTHREADS, smem, st>>>(mq, mk, mv, g, h0, (__nv_bfloat16*)o, hT, T,
                                                 H, DV, ws, err);
  return cudaGetLastError();
}

}  // namespace

size_t chunk_workspace_bytes(int B, int T, int H, int dk, int dv, int dtype) {
  if (dtype != KLA_BF16 || B < 1 || H < 1 || T < 1 || dk != dv) return 0;
  return (size_t)B * H * ((T + C - 1) / C) * kUtTileBytes;
}

cudaError_t launch_chunk_tc(const void* q, const void* k, const void* v, const float* g,
                            const float* eta, float eps, const float* h0, void* o, float* hT,
                            int B, int T, int H, int dk, int dv, void* workspace,
                            unsigned int* err, cudaStream_t st) {
  if (dk != dv) return cudaErrorNotSupported;
  uint8_t* ws = (uint8_t*)workspace;
  if (dk == 128) return launch_dk<128>(q, k, v, g, eta, eps, h0, o, hT, B, T, H, dv, ws, err, st);
  if (dk == 64) return launch_dk<64>(q, k, v, g, eta, eps, h0, o, hT, B, T, H, dv, ws, err, st);
  return cudaErrorNotSupported;
}

}  // namespace kla
