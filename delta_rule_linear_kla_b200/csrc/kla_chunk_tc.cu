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
//   W  = T'' K,  U = T' V                                           [MMA 2, 3]
//   P  = lower_incl(Q K^T (*) e^{G_r - G_s})                        [MMA 1]
//   V' = U - W h  (and -Q h)  accumulated onto U in TMEM            [MMA 4]
//   h <- e^{G_63} h + K^T diag(e^{G_63 - G_s}) V'                    [MMA 5]
//   O  = diag(e^G) Q h + P V'                                       [MMA 6]
//
// The decay ratios are only formed as masked differences of G or running
// products of alpha (never K / Gamma), so strong gates cannot overflow.  A
// ragged tail is zero-filled by TMA and given g = 0 (and eta = 0 in the UT
// kernel): an identity step.
//
// All contractions are single-CTA tcgen05.mma with M = 128, bf16 operands in
// 128-byte swizzled shared-memory tiles and fp32 accumulators in TMEM (lane
// = row; 64-row products are stacked or padded to 128 lanes):
//   MMA 2  D_W [128xDK]   = [T''; 0] . K          A, B MN-major (W: lanes 0..63)
//   MMA 3  D_U [128x64]   = [T'; 0] . V           A, B MN-major
//   MMA 1  D_S [128x64]   = [W; Q] . K^T          A, B K-major
//                                                  (lanes 64..127: Q K^T)
//   MMA 4  D_U           += -[W; Q] . h           B MN-major (negated A)
//          -> lanes 0..63 hold V' = U - W h, lanes 64..127 hold -Q h
//   MMA 5  D_H [128x64]   = K^T . (decay V')      A, B MN-major (lanes < DK)
//   MMA 6  D_PV[128x64]   = [0; P] . V'           A K-major, B MN-major
//                                                  (lanes 64..127)
//
// Warp roles (512 threads), synchronised only through mbarriers:
//   warp 0      TMA producer: Q, K, V slab and the UT tiles of chunk n into
//               stage n % 2 (double buffered).
//   warp 1      MMA issuer: the warp runs the schedule uniformly and one
//               elected lane issues.  Per iteration n: MMA 4 of chunk n, MMA 2
//               of chunk n + 1 (it runs while V'(n) is formed), MMA 5 and
//               MMA 6 of chunk n, then MMAs 3 and 1 of chunk n + 1 (they run
//               while the state is updated).  The tensor pipe executes in issue order, so the
//               state chain's MMAs never queue behind more than one
//               state-independent product.
//   warps 4, 5  W of the next chunk: D_W (lanes 0..63) -> bf16 -> the
//               stage's W rows.
//   warps 2, 3, 14, 15  P of the next chunk (TMEM lanes 64..127) into the
//               stage's P tile; warp 2 also computes the gate cumsum.
//   warps 6..13 "chain" epilogues, split by state columns (warps 6..9 take
//               columns 0..31, warps 10..13 columns 32..63): V' (lanes
//               0..63), the state update (lanes < DK) and the output rows
//               (lanes 64..127).
// Every wait is bounded (about 2 s); on timeout the kernel raises the device
// error word, stops all roles, drains its own TMA loads and MMAs and frees
// TMEM.
#include <algorithm>
#include <type_traits>

#include <cuda.h>
#include <cudaTypedefs.h>

#include "kla_chunk.h"
#include "kla_common.cuh"
#include "kla_sync.cuh"
#include "kla_ut_body.cuh"
#include "ptx_sm100.cuh"
#include "tile_sw128.cuh"

namespace kla {
namespace {

constexpr int C = 64;       // chunk length
constexpr int BV = 64;      // state columns per CTA
constexpr int NTHREADS = 512;
constexpr uint32_t TMEM_COLS = 512;
// TMEM column offsets of the accumulators
constexpr uint32_t COL_S = 0, COL_W = 64, COL_U = 192 /* 2 buffers */, COL_H = 320,
                   COL_PV = 384;

// One pipeline stage.  Per 64-column key panel: [W rows | Q rows | K rows]
// (8 KB each), so [W; Q] is one 128-row K-major operand.  Then the V slab and [T'^T | T''^T | 0 | P]: the MN-major A
// operands [T'; 0] (leading offset 16 KB) and [T''; 0] (8 KB), and the
// K-major A operand [0; P].
template <int DK>
struct alignas(1024) Stage {
  static constexpr int NP = DK / 64;
  uint8_t panel[NP][3][8192];
  uint8_t v[8192];
  uint8_t tp[4][8192];
};

template <int DK>
struct alignas(1024) ChainSmem {
  Stage<DK> st[2];
  uint8_t hm[DK * 128];  // bf16 state slab (MMA 4 operand), row i = key index
  uint8_t vp[8192];      // V'
  uint8_t vpd[8192];     // V' scaled by e^{G_63 - G_s} (MMA 5 operand)
  float G[3][C];         // gate cumsum of chunk n in slot n % 3
  alignas(16) float alpha[3][C];  // e^{g_s} of chunk n in slot n % 3
  float kdec[3][128];    // per-channel gate: e^{G_last} of chunk n in slot n % 3
  uint64_t full[2], empty[2];
  uint64_t bS, bW, bX, bH, bHP;          // MMA completions
  uint64_t p_done, w_done, vpd_ready, vp_ready;
  uint64_t u_free[2], h_done, pv_free;
  uint64_t g_ready[3];
  uint64_t mma_drain;
  uint32_t tmem_base;
  int abort_flag;
};

enum Slot { SW = 0, SQ = 1, SK = 2 };
enum TSlot { TP1 = 0, TP2 = 1, TZ = 2, TP = 3 };

// Bounded wait that also gives up as soon as another role has aborted.
__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity,
                                              volatile int* abort_flag) {
  if (ptx::mbar_test_wait(bar, parity)) return true;
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

// The same wait taken by every lane of a warp that then runs
// warp-collective instructions (elect.sync, tcgen05.ld, __syncwarp).  The
// lanes poll together and read the same barrier, abort flag and clock, so
// they leave together; a vote on the result (to keep a warp whole even if
// its lanes disagreed after a timeout) cost 5 % of the 4K prefill's state
// kernel and is not taken.
__device__ __forceinline__ bool wait_warp(uint64_t* bar, uint32_t parity,
                                          volatile int* abort_flag) {
  return wait_or_abort(bar, parity, abort_flag);
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(ptx::smem_u32(bar)) : "memory");
}

// Descriptor advance: the start address lives in the low bits, in 16-byte
// units; a K step is 32 B (K-major) or 2048 B (MN-major).
constexpr uint64_t KSTEP_K = 2, KSTEP_MN = 128;

// KDA: the per-channel-gate form.  The stage then holds W, P, Q o e^G and
// K o e^{G_last - G} as made per chunk by kda_prep_kernel (bulk copies; no
// Q K^T or W products, no W or P epilogues), the state decays row by row with
// e^{G_last}, and the outputs take no e^{G} factor (it is in Q o e^G).
// Waits until the UT lane that makes chunk `idx`'s factors has raised its
// flag (single-launch prefill), then orders this thread's later bulk copies
// (async proxy) after that acquire.  Bounded like every other wait.
__device__ __forceinline__ bool wait_flag(const unsigned int* flag, volatile int* abort_flag) {
  const uint64_t t0 = globaltimer();
  while (true) {
    unsigned int v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(flag) : "memory");
    if (v != 0u) {
      asm volatile("fence.proxy.async.global;" ::: "memory");
      return true;
    }
    if (*abort_flag) return false;
    if (globaltimer() - t0 > kWaitLimitNs) {
      *abort_flag = 1;
      return false;
    }
    __nanosleep(64);
  }
}

// The state/output CTA for block coordinates (bx, by, bz) of the chain grid
// (slab, head, batch x segment).  flags (nullable): the factors of chunk
// (head, n) may be read only after flags[head * nchunks + n] is set (they
// are made by UT lanes of the same launch).
template <int DK, bool KDA>
__device__ __forceinline__ void chain_body(
    const CUtensorMap* tm_q_p, const CUtensorMap* tm_k_p, const CUtensorMap* tm_v_p,
    const float* __restrict__ g, const float* __restrict__ h0, __nv_bfloat16* __restrict__ o,
    float* __restrict__ hT, float* __restrict__ phi, float* __restrict__ hs, int T, int H,
    int DV, int nseg, int seg_chunks, int mode, const uint8_t* __restrict__ ws,
    unsigned int* err, const int bx, const int by, const int bz,
    const unsigned int* __restrict__ flags) {
  const CUtensorMap& tm_q = *tm_q_p;
  const CUtensorMap& tm_k = *tm_k_p;
  const CUtensorMap& tm_v = *tm_v_p;
  using Smem = ChainSmem<DK>;
  constexpr int NP = Stage<DK>::NP;
  constexpr uint32_t PANEL = 3 * 8192;  // byte stride between key panels
  extern __shared__ uint8_t smem_raw[];
  Smem& s = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                     ~uintptr_t(1023));
  volatile int* abort_flag = &s.abort_flag;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int hh = by, b = bz / nseg, seg = bz % nseg;
  // Segment `seg` of the sequence: chunks n0 .. n0 + nchunks - 1 (the loop
  // index n below counts chunks within the segment; n0 + n addresses data).
  const int nchunks_all = (T + C - 1) / C;
  const int n0 = seg * seg_chunks;
  const int nchunks = min(seg_chunks, nchunks_all - n0);
  const size_t head = (size_t)b * H + hh;
  const size_t sidx = ((size_t)b * nseg + seg) * H + hh;  // per-segment state index
  // mode 0: outputs; the initial state is h0[sidx] (NULL = zeros) and the
  // last segment writes h_T to hT[head].  mode 1 (segment transitions, no
  // outputs): slabs below DV / BV run from a zero state and leave the end
  // state E in hT[sidx]; the others propagate the identity with V = 0 and
  // leave Phi (the segment's transition, [DK][DK]) in phi[sidx].  hs (mode 0,
  // nullable): the fp32 state at the start of every chunk,
  // [B][H][nchunks][DK][DV].  o may be NULL (no outputs written).
  const int nvs = DV / BV;
  const bool phi_slab = mode == 1 && bx >= nvs;
  const int slab = phi_slab ? bx - nvs : bx;
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
      ptx::mbar_init(&s.u_free[i], 8);
    }
    for (int i = 0; i < 3; ++i) ptx::mbar_init(&s.g_ready[i], 1);
    ptx::mbar_init(&s.bS, 1);
    ptx::mbar_init(&s.bW, 1);
    ptx::mbar_init(&s.bX, 1);
    ptx::mbar_init(&s.bH, 1);
    ptx::mbar_init(&s.bHP, 1);
    ptx::mbar_init(&s.p_done, 4);
    ptx::mbar_init(&s.w_done, 2);
    ptx::mbar_init(&s.vpd_ready, 4);
    ptx::mbar_init(&s.vp_ready, 4);
    ptx::mbar_init(&s.h_done, 8);
    ptx::mbar_init(&s.pv_free, 4);
    ptx::mbar_init(&s.mma_drain, 1);
    ptx::mbar_init_fence();
    s.abort_flag = 0;
  }
  // the zero tiles of both stages (and, with V = 0, the V slabs)
  for (int i = tid; i < 2 * 8192 / 16; i += NTHREADS) {
    reinterpret_cast<uint4*>(s.st[i / 512].tp[TZ])[i % 512] = make_uint4(0, 0, 0, 0);
    if (phi_slab) reinterpret_cast<uint4*>(s.st[i / 512].v)[i % 512] = make_uint4(0, 0, 0, 0);
  }
  ptx::fence_proxy_async_smem();
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
      constexpr KdaTileOffsets KO = kda_tile_offsets(DK);
      constexpr uint32_t TILE = KDA ? KO.total : (uint32_t)kUtTileBytes;
      const uint32_t BYTES =
          KDA ? (uint32_t)(2 * 8192 + 3 * NP * 8192 + DK * 4 + (phi_slab ? 0 : 8192))
              : (uint32_t)(2 * NP * 8192 + (phi_slab ? 0 : 8192) + kUtTileBytes);
      const uint8_t* ws_head = ws + (head * (size_t)nchunks_all + n0) * TILE;
      int issued = 0, drained = 0;
      for (int n = 0; n < nchunks; ++n) {
        const int st = n & 1;
        if (n >= 2) {
          if (!wait_or_abort(&s.empty[st], (uint32_t)(((n - 2) >> 1) & 1), abort_flag)) break;
          drained = n - 1;  // chunks up to n-2 fully consumed
        }
        Stage<DK>& S = s.st[st];
        const uint8_t* src = ws_head + (size_t)n * TILE;
        // single-launch prefill: this chunk's factors exist once their flag
        // is up (nothing of the stage is armed before that)
        if (!KDA && flags && !wait_flag(flags + head * (size_t)nchunks_all + n0 + n, abort_flag))
          break;
        ptx::mbar_arrive_expect_tx(&s.full[st], BYTES);
        if constexpr (KDA) {
          ptx::bulk_load(S.tp[TP1], src + KO.tp, 8192, &s.full[st]);
          ptx::bulk_load(S.tp[TP], src + KO.p, 8192, &s.full[st]);
          ptx::bulk_load(S.tp[TP2], src + KO.d, DK * 4, &s.full[st]);  // e^{G_last}
#pragma unroll
          for (int p = 0; p < NP; ++p) {
            ptx::bulk_load(S.panel[p][SW], src + KO.w + p * 8192, 8192, &s.full[st]);
            ptx::bulk_load(S.panel[p][SQ], src + KO.q + p * 8192, 8192, &s.full[st]);
            ptx::bulk_load(S.panel[p][SK], src + KO.k + p * 8192, 8192, &s.full[st]);
          }
        } else {
          ptx::bulk_load(S.tp[TP1], src, 8192, &s.full[st]);
          ptx::bulk_load(S.tp[TP2], src + 8192, 8192, &s.full[st]);
#pragma unroll
          for (int p = 0; p < NP; ++p) {
            ptx::tma_load_4d(S.panel[p][SK], &tm_k, &s.full[st], p * 64, hh, (n0 + n) * C, b);
            ptx::tma_load_4d(S.panel[p][SQ], &tm_q, &s.full[st], p * 64, hh, (n0 + n) * C, b);
          }
        }
        if (!phi_slab)
          ptx::tma_load_4d(S.v, &tm_v, &s.full[st], slab * BV, hh, (n0 + n) * C, b);
        issued = n + 1;
        if (n + 2 < nchunks) {  // warm L2 two chunks ahead of the loads
          const int m = n + 2;
          // the factors only once they exist (single launch: flagged
          // already; a chunk not yet flagged is not waited for here)
          bool made = !flags;
          if (!made) {
            unsigned int f;
            asm volatile("ld.acquire.gpu.global.u32 %0, [%1];"
                         : "=r"(f)
                         : "l"(flags + head * (size_t)nchunks_all + n0 + m)
                         : "memory");
            made = f != 0u;
            if (made) asm volatile("fence.proxy.async.global;" ::: "memory");
          }
          if (made) ptx::bulk_prefetch_l2(ws_head + (size_t)m * TILE, TILE);
          if constexpr (!KDA) {
#pragma unroll
            for (int p = 0; p < NP; ++p) {
              ptx::tma_prefetch_l2_4d(&tm_k, p * 64, hh, (n0 + m) * C, b);
              ptx::tma_prefetch_l2_4d(&tm_q, p * 64, hh, (n0 + m) * C, b);
            }
          }
          if (!phi_slab) ptx::tma_prefetch_l2_4d(&tm_v, slab * BV, hh, (n0 + m) * C, b);
        }
      }
      if (*abort_flag) {
        // let this CTA's own copies land before the CTA goes away
        for (int n = drained; n < issued; ++n)
          if (!wait_bounded(&s.full[n & 1], (uint32_t)((n >> 1) & 1))) break;
      }
    }
  } else if (warp == 1) {
    // ============================ MMA issuer ============================
    constexpr uint32_t id_w = ptx::idesc_bf16(128, DK, 1, 1);
    constexpr uint32_t id_mn = ptx::idesc_bf16(128, 64, 1, 1);
    constexpr uint32_t id_s = ptx::idesc_bf16(128, 64, 0, 0);
    constexpr uint32_t id_x = ptx::idesc_bf16(128, 64, 0, 1, /*neg_a=*/1);
    constexpr uint32_t id_pv = ptx::idesc_bf16(128, 64, 0, 1);
    // descriptors of stage 0 / panel 0 (uniform across the warp); other
    // stages and panels are fixed offsets in 16-byte units
    constexpr uint64_t STG = sizeof(Stage<DK>) >> 4, PNL = PANEL >> 4;
    const uint64_t dWQ = ptx::sdesc_sw128(ptx::smem_u32(s.st[0].panel[0][SW]), 16, 1024);
    const uint64_t dKk = ptx::sdesc_sw128(ptx::smem_u32(s.st[0].panel[0][SK]), 16, 1024);
    const uint64_t dKmn = ptx::sdesc_sw128(ptx::smem_u32(s.st[0].panel[0][SK]), PANEL, 1024);
    const uint64_t dT1 = ptx::sdesc_sw128(ptx::smem_u32(s.st[0].tp[TP1]), 2 * 8192, 1024);
    const uint64_t dT2 = ptx::sdesc_sw128(ptx::smem_u32(s.st[0].tp[TP2]), 8192, 1024);
    const uint64_t dZP = ptx::sdesc_sw128(ptx::smem_u32(s.st[0].tp[TZ]), 16, 1024);
    const uint64_t dV = ptx::sdesc_sw128(ptx::smem_u32(s.st[0].v), 1024, 1024);
    const uint64_t dH = ptx::sdesc_sw128(ptx::smem_u32(s.hm), 1024, 1024);
    const uint64_t dVP = ptx::sdesc_sw128(ptx::smem_u32(s.vp), 1024, 1024);
    const uint64_t dVPD = ptx::sdesc_sw128(ptx::smem_u32(s.vpd), 1024, 1024);

    auto mma2 = [&](int n) {  // D_W = [T''; 0] K  (W in lanes 0..63)
      const uint64_t so = (uint64_t)(n & 1) * STG;
      if (ptx::elect_one()) {
#pragma unroll
        for (int kk = 0; kk < C / 16; ++kk)
          ptx::mma_bf16(tb + COL_W, dT2 + so + kk * KSTEP_MN, dKmn + so + kk * KSTEP_MN, id_w,
                        kk > 0);
        ptx::mma_commit(&s.bW);
      }
      __syncwarp();
    };
    auto mma3 = [&](int n) {  // D_U[n%2] = [T'; 0] V
      const uint64_t so = (uint64_t)(n & 1) * STG;
      if (ptx::elect_one()) {
#pragma unroll
        for (int kk = 0; kk < C / 16; ++kk)
          ptx::mma_bf16(tb + COL_U + 64 * (n & 1), dT1 + so + kk * KSTEP_MN,
                        dV + so + kk * KSTEP_MN, id_mn, kk > 0);
      }
      __syncwarp();
    };
    auto mma1 = [&](int n) {  // D_S = [W; Q] K^T  (Q K^T in lanes 64..127)
      const uint64_t so = (uint64_t)(n & 1) * STG;
      if (ptx::elect_one()) {
#pragma unroll
        for (int kk = 0; kk < DK / 16; ++kk)
          ptx::mma_bf16(tb + COL_S, dWQ + so + (kk >> 2) * PNL + (kk & 3) * KSTEP_K,
                        dKk + so + (kk >> 2) * PNL + (kk & 3) * KSTEP_K, id_s, kk > 0);
        ptx::mma_commit(&s.bS);
      }
      __syncwarp();
    };
    bool ok = nchunks > 0;
    if (ok) ok = wait_warp(&s.full[0], 0, abort_flag);
    if (ok) {
      ptx::tc_fence_after();
      if constexpr (KDA) {
        mma3(0);
      } else {
        mma2(0);
        mma3(0);
        ok = wait_warp(&s.w_done, 0, abort_flag);
        if (ok) {
          ptx::tc_fence_after();
          mma1(0);
        }
      }
    }
    for (int n = 0; n < nchunks && ok; ++n) {
      const int st = n & 1;
      const uint64_t so = (uint64_t)st * STG;
      const uint32_t par = (uint32_t)(n & 1);
      const bool more = n + 1 < nchunks;
      // ---- MMA 4 (chunk n): needs W(n) and h_n (D_H of n-1 read)
      if (!KDA && !wait_warp(&s.w_done, par, abort_flag)) break;
      if (!wait_warp(&s.h_done, par, abort_flag)) break;
      ptx::tc_fence_after();
      if (ptx::elect_one()) {
#pragma unroll
        for (int kk = 0; kk < DK / 16; ++kk)
          ptx::mma_bf16(tb + COL_U + 64 * st, dWQ + so + (kk >> 2) * PNL + (kk & 3) * KSTEP_K,
                        dH + kk * KSTEP_MN, id_x, 1);
        ptx::mma_commit(&s.bX);
      }
      __syncwarp();
      // ---- while V'(n) is formed: W of chunk n+1 (needed by its MMA 4);
      //      D_W was read before w_done(n)
      if (more) {
        if (!wait_warp(&s.full[(n + 1) & 1], (uint32_t)(((n + 1) >> 1) & 1), abort_flag))
          break;
        ptx::tc_fence_after();
        if constexpr (!KDA) mma2(n + 1);
      }
      // ---- MMA 5 (state), committed on its own so the update starts at once
      if (!wait_warp(&s.vpd_ready, par, abort_flag)) break;
      ptx::tc_fence_after();
      if (ptx::elect_one()) {
#pragma unroll
        for (int kk = 0; kk < C / 16; ++kk)
          ptx::mma_bf16(tb + COL_H, dKmn + so + kk * KSTEP_MN, (KDA ? dVP : dVPD) + kk * KSTEP_MN,
                        id_mn, kk > 0);
        ptx::mma_commit(&s.bH);
      }
      __syncwarp();
      // ---- MMA 6 (chunk n): needs V'(n), P(n) and D_PV free (outputs of n-1
      //      read)
      if (!wait_warp(&s.vp_ready, par, abort_flag)) break;
      if (!KDA && !wait_warp(&s.p_done, par, abort_flag)) break;
      if (n > 0 && !wait_warp(&s.pv_free, par ^ 1u, abort_flag)) break;
      ptx::tc_fence_after();
      if (ptx::elect_one()) {
#pragma unroll
        for (int kk = 0; kk < C / 16; ++kk)
          ptx::mma_bf16(tb + COL_PV, dZP + so + kk * KSTEP_K, dVP + kk * KSTEP_MN, id_pv, kk > 0);
        ptx::mma_commit(&s.bHP);
        ptx::mma_commit(&s.empty[st]);
      }
      __syncwarp();
      if (more) {
        // ---- while the state is updated: U of chunk n+1 (D_U[(n+1)%2] was
        //      used by chunk n-1; MMA 4 of n+1 accumulates onto it) ...
        if (n >= 1 &&
            !wait_warp(&s.u_free[(n + 1) & 1], (uint32_t)(((n - 1) >> 1) & 1), abort_flag))
          break;
        ptx::tc_fence_after();
        mma3(n + 1);
        if constexpr (!KDA) {
          // ... and Q K^T of chunk n+1: D_S was read by P(n) (waited above);
          // waiting for W(n+1) keeps its rows from changing under the read
          if (!wait_warp(&s.w_done, par ^ 1u, abort_flag)) break;
          ptx::tc_fence_after();
          mma1(n + 1);
        }
      }
    }
    // every MMA this warp issued has finished before TMEM is released
    if (ptx::elect_one()) ptx::mma_commit(&s.mma_drain);
    __syncwarp();
    wait_bounded(&s.mma_drain, 0);
  } else if (warp == 4 || warp == 5) {
    // ===================== next-chunk epilogue: W =========================
    // W rows 0..63 (TMEM lanes 0..63) -> the stage's W slot (bf16)
    for (int n = 0; n < (KDA ? 0 : nchunks); ++n) {
      Stage<DK>& S = s.st[n & 1];
      if (!wait_warp(&s.bW, (uint32_t)(n & 1), abort_flag)) break;
      ptx::tc_fence_after();
#pragma unroll
      for (int p = 0; p < NP; ++p) {
        float w0[32], w1[32];  // the panel's two 32-column halves, one wait
        ptx::tmem_ld32x2(tb + lane_base + COL_W + p * 64, tb + lane_base + COL_W + p * 64 + 32,
                         w0, w1);
        sw128_store_row32(S.panel[p][SW], row, 0, w0);
        sw128_store_row32(S.panel[p][SW], row, 1, w1);
      }
      ptx::fence_proxy_async_smem();
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s.w_done);
    }
  } else if (warp == 2 || warp == 3 || warp >= 14) {
    // ===================== next-chunk epilogue: P =========================
    // Warps 2, 3, 14, 15 (TMEM lanes 64..127, row r = lane row - 64); warps
    // 2, 3 take columns 32..63, warps 14, 15 columns 0..31.  Warp 2 also
    // computes the gate cumsum and alpha of the chunk (published through
    // g_ready), loading the next chunk's gates one chunk ahead.
    const int hc = (warp >= 14) ? 0 : 1;
    const int r = row - 64;
    if constexpr (KDA) {
      // the chunk decay e^{G_last} (one per key channel) arrives with the
      // stage; warp 2 publishes it through the g_ready ring
      for (int n = 0; n < (warp == 2 ? nchunks : 0); ++n) {
        if (!wait_warp(&s.full[n & 1], (uint32_t)((n >> 1) & 1), abort_flag)) break;
        const float* dsrc = reinterpret_cast<const float*>(s.st[n & 1].tp[TP2]);
        for (int i = lane; i < DK; i += 32) s.kdec[n % 3][i] = dsrc[i];
        __syncwarp();
        if (lane == 0) mbar_arrive(&s.g_ready[n % 3]);
      }
    }
    float gn0 = 0.f, gn1 = 0.f;
    if (!KDA && warp == 2 && nchunks > 0) {
      const int t0 = n0 * C + lane, t1 = t0 + 32;
      gn0 = (t0 < T) ? g[((size_t)b * T + t0) * H + hh] : 0.f;
      gn1 = (t1 < T) ? g[((size_t)b * T + t1) * H + hh] : 0.f;
    }
    for (int n = 0; n < (KDA ? 0 : nchunks); ++n) {
      Stage<DK>& S = s.st[n & 1];
      float* Gn = s.G[n % 3];
      if (warp == 2) {
        const float g0 = gn0, g1 = gn1;
        // next chunk's gates (tokens lane, lane + 32), used one chunk later
        const int t0 = (n0 + n + 1) * C + lane, t1 = t0 + 32;
        gn0 = (t0 < T) ? g[((size_t)b * T + t0) * H + hh] : 0.f;
        gn1 = (t1 < T) ? g[((size_t)b * T + t1) * H + hh] : 0.f;
        float x0 = g0, x1 = g1;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
          const float y0 = __shfl_up_sync(0xffffffffu, x0, off);
          const float y1 = __shfl_up_sync(0xffffffffu, x1, off);
          if (lane >= off) { x0 += y0; x1 += y1; }
        }
        const float tot0 = __shfl_sync(0xffffffffu, x0, 31);
        Gn[lane] = x0;
        Gn[lane + 32] = x1 + tot0;
        s.alpha[n % 3][lane] = __expf(g0);
        s.alpha[n % 3][lane + 32] = __expf(g1);
        __syncwarp();
        if (lane == 0) mbar_arrive(&s.g_ready[n % 3]);
      } else {
        if (!wait_warp(&s.g_ready[n % 3], (uint32_t)((n / 3) & 1), abort_flag)) break;
      }
      // ---- P row r, columns [32 hc, 32 hc + 32): e^{G_r - G_s} is the
      //      running product of alpha_j over s < j <= r, from the diagonal
      //      leftwards (every factor <= 1); the left half starts from
      //      e^{G_r - G_31}.
      const float Gr = Gn[r];
      const int c_hi = 32 * hc + 31;
      float d = (r > c_hi) ? __expf(Gr - Gn[c_hi]) : 1.f;
      float al[32];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float4 a4 = reinterpret_cast<const float4*>(&s.alpha[n % 3][32 * hc])[i];
        al[4 * i] = a4.x; al[4 * i + 1] = a4.y; al[4 * i + 2] = a4.z; al[4 * i + 3] = a4.w;
      }
      if (!wait_warp(&s.bS, (uint32_t)(n & 1), abort_flag)) break;
      ptx::tc_fence_after();
      float srow[32];
      ptx::tmem_ld32(tb + lane_base + COL_S + 32 * hc, srow);
#pragma unroll
      for (int c = 31; c >= 0; --c) {
        const bool on = 32 * hc + c <= r;
        srow[c] = on ? srow[c] * d : 0.f;
        d = on ? d * al[c] : d;
      }
      sw128_store_row32(S.tp[TP], r, hc, srow);
      ptx::fence_proxy_async_smem();
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s.p_done);
    }
  } else if (warp >= 6 && warp < 14) {
    // ========================= chain epilogues ==========================
    // warps 6..9 take state columns [0, 32) of the slab, warps 10..13
    // columns [32, 64); within each group the lane groups give the rows.
    const int grp = warp >= 10 ? 1 : 0, cg = 32 * grp;
    const bool has_h = row < DK;
    float hreg[32];
    if (has_h) {
      if (phi_slab) {  // identity columns slab * BV + cg ..
#pragma unroll
        for (int j = 0; j < 32; ++j) hreg[j] = (row == slab * BV + cg + j) ? 1.f : 0.f;
      } else if (h0 && mode == 0) {
        const float4* src =
            reinterpret_cast<const float4*>(h0 + (sidx * DK + row) * DV + slab * BV + cg);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float4 x = src[j];
          hreg[4 * j] = x.x; hreg[4 * j + 1] = x.y; hreg[4 * j + 2] = x.z; hreg[4 * j + 3] = x.w;
        }
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) hreg[j] = 0.f;
      }
      sw128_store_row32(s.hm, row, grp, hreg);
      ptx::fence_proxy_async_smem();
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&s.h_done);  // h_0 is in place
    const bool v_rows = row < 64;
    bool ok = true;
    for (int n = 0; n < nchunks && ok; ++n) {
      if (hs && mode == 0 && has_h) {  // h at the start of chunk n0 + n
        float4* dst = reinterpret_cast<float4*>(
            hs + ((head * nchunks_all + n0 + n) * DK + row) * DV + slab * BV + cg);
#pragma unroll
        for (int j = 0; j < 8; ++j)
          dst[j] = make_float4(hreg[4 * j], hreg[4 * j + 1], hreg[4 * j + 2], hreg[4 * j + 3]);
      }
      const float* Gn = s.G[n % 3];
      const uint32_t par = (uint32_t)(n & 1);
      const uint32_t col_u = COL_U + 64 * (n & 1);
      if (!wait_warp(&s.g_ready[n % 3], (uint32_t)((n / 3) & 1), abort_flag)) { ok = false; break; }
      const float gC = KDA ? 0.f : Gn[C - 1];
      if (v_rows && KDA) {
        // V' = U - W h (combined in TMEM); the keys of MMA 5 carry the decay
        if (!wait_warp(&s.bX, par, abort_flag)) { ok = false; break; }
        ptx::tc_fence_after();
        float u[32];
        ptx::tmem_ld32(tb + lane_base + col_u + cg, u);
        ptx::tc_fence_before();
        sw128_store_row32(s.vp, row, grp, u);
        ptx::fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&s.vpd_ready);
          mbar_arrive(&s.u_free[n & 1]);
          mbar_arrive(&s.vp_ready);
        }
      } else if (v_rows) {
        // V'_r = U_r - (W h)_r (already combined in TMEM) and its copy
        // decayed to the chunk end for MMA 5
        const float dec = __expf(gC - Gn[row]);
        if (!wait_warp(&s.bX, par, abort_flag)) { ok = false; break; }
        ptx::tc_fence_after();
        float u[32], ud[32];
        ptx::tmem_ld32(tb + lane_base + col_u + cg, u);
        ptx::tc_fence_before();
        // the decayed copy first: it feeds MMA 5, the next link of the chain
#pragma unroll
        for (int j = 0; j < 32; ++j) ud[j] = u[j] * dec;
        sw128_store_row32(s.vpd, row, grp, ud);
        ptx::fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&s.vpd_ready);
          mbar_arrive(&s.u_free[n & 1]);
        }
        sw128_store_row32(s.vp, row, grp, u);
        ptx::fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&s.vp_ready);
      }
      // every read of G(n) happens before this warp's last arrival of chunk n
      const float e_out = v_rows ? 0.f : (KDA ? -1.f : -__expf(Gn[row - 64]));
      if (!wait_warp(&s.bH, par, abort_flag)) { ok = false; break; }
      ptx::tc_fence_after();
      if (has_h) {
        const float a = KDA ? s.kdec[n % 3][row] : __expf(gC);
        float dh[32];
        ptx::tmem_ld32(tb + lane_base + COL_H + cg, dh);
#pragma unroll
        for (int j = 0; j < 32; ++j) hreg[j] = fmaf(a, hreg[j], dh[j]);
        sw128_store_row32(s.hm, row, grp, hreg);
        ptx::fence_proxy_async_smem();
      }
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s.h_done);  // h_{n+1} in place, D_H read
      if (!v_rows) {
        // output row r = row - 64: o_r = e^{G_r} (Q h)_r + (P V')_r, with
        // -(Q h)_r in lanes 64..127 of D_U
        const int r = row - 64, t = (n0 + n) * C + r;
        const float e = e_out;
        if (!wait_warp(&s.bHP, par, abort_flag)) { ok = false; break; }
        ptx::tc_fence_after();
        float x[32], pv[32];
        ptx::tmem_ld32x2(tb + lane_base + col_u + cg, tb + lane_base + COL_PV + cg, x, pv);
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&s.u_free[n & 1]);
          mbar_arrive(&s.pv_free);
        }
        if (t < T && mode == 0 && o) {
          __nv_bfloat16* orow = o + (((size_t)b * T + t) * H + hh) * DV + slab * BV + cg;
          uint32_t w[16];
#pragma unroll
          for (int i = 0; i < 16; ++i)
            w[i] = pack_bf16x2(fmaf(e, x[2 * i], pv[2 * i]), fmaf(e, x[2 * i + 1], pv[2 * i + 1]));
          // the row's 64 bytes as two 32-byte stores where o allows it (the
          // offsets here are multiples of 64 bytes, so this is uniform over
          // the launch), else four 16-byte ones
          if ((reinterpret_cast<uintptr_t>(orow) & 31u) == 0u) {
#pragma unroll
            for (int c = 0; c < 2; ++c)
              asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(
                               orow + 16 * c),
                           "r"(w[8 * c]), "r"(w[8 * c + 1]), "r"(w[8 * c + 2]), "r"(w[8 * c + 3]),
                           "r"(w[8 * c + 4]), "r"(w[8 * c + 5]), "r"(w[8 * c + 6]), "r"(w[8 * c + 7])
                           : "memory");
          } else {
            uint4* dst = reinterpret_cast<uint4*>(orow);
#pragma unroll
            for (int c = 0; c < 4; ++c)
              dst[c] = make_uint4(w[4 * c], w[4 * c + 1], w[4 * c + 2], w[4 * c + 3]);
          }
        }
      }
    }
    // the state this CTA ends with: h_T (last segment), E or Phi
    float* out = nullptr;
    size_t oidx = 0;
    int ostride = DV;
    if (mode == 0 && seg == nseg - 1) {
      out = hT;
      oidx = head;
    } else if (mode == 1) {
      out = phi_slab ? phi : hT;
      oidx = sidx;
      ostride = phi_slab ? DK : DV;
    }
    if (ok && has_h && out) {
      float4* dst = reinterpret_cast<float4*>(out + (oidx * DK + row) * ostride + slab * BV + cg);
#pragma unroll
      for (int j = 0; j < 8; ++j)
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

template <int DK, bool KDA>
__global__ void __launch_bounds__(NTHREADS, 1)
chain_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
             const __grid_constant__ CUtensorMap tm_v, const float* __restrict__ g,
             const float* __restrict__ h0, __nv_bfloat16* __restrict__ o,
             float* __restrict__ hT, float* __restrict__ phi, float* __restrict__ hs, int T,
             int H, int DV, int nseg, int seg_chunks, int mode,
             const uint8_t* __restrict__ ws, unsigned int* err) {
  chain_body<DK, KDA>(&tm_q, &tm_k, &tm_v, g, h0, o, hT, phi, hs, T, H, DV, nseg, seg_chunks,
                      mode, ws, err, blockIdx.x, blockIdx.y, blockIdx.z, nullptr);
}

// UT lanes (128 threads each) per CTA of the single-launch prefill (the
// lanes' shared memory fits in the state CTA's; the fourth group of 128
// threads idles).
template <int DK>
constexpr int fused_ut_lanes() {
  return 3;
}
template <int DK>
constexpr size_t fused_smem_bytes() {
  return (sizeof(ChainSmem<DK>) > fused_ut_lanes<DK>() * sizeof(utb::UtSmem<DK>)
              ? sizeof(ChainSmem<DK>)
              : fused_ut_lanes<DK>() * sizeof(utb::UtSmem<DK>)) +
         1024;
}

// The whole uncut prefill as one launch: CTAs 0 .. n_chain - 1 are the
// state/output CTAs of the chain grid (slab fastest, then head, then batch);
// every other CTA holds fused_ut_lanes UT lanes that make the per-chunk
// factors in chunk order n = 0, 1, ... over all heads and raise one flag per
// chunk, which the state CTAs wait for before they fetch that chunk's
// factors.  The launch is cooperative (all CTAs resident at once, one per
// SM), so those waits always end; they are bounded all the same.  Not taken
// at present (see fused_shape): every shape runs the two kernels in turn.
template <int DK>
__global__ void __launch_bounds__(NTHREADS, 1)
prefill_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, const float* __restrict__ g,
               const float* __restrict__ eta, float eps, const float* __restrict__ h0,
               __nv_bfloat16* __restrict__ o, float* __restrict__ hT, float* __restrict__ hs,
               int T, int H, int DV, uint8_t* __restrict__ ws, unsigned int* flags, int n_chain,
               unsigned int* err) {
  const int nchunks = (T + C - 1) / C;
  if ((int)blockIdx.x < n_chain) {
    const int nvs = DV / BV;
    const int bx = (int)blockIdx.x % nvs, by = ((int)blockIdx.x / nvs) % H,
              bz = (int)blockIdx.x / (nvs * H);
    chain_body<DK, false>(&tm_q, &tm_k, &tm_v, g, h0, o, hT, nullptr, hs, T, H, DV, 1, nchunks,
                          0, ws, err, bx, by, bz, flags);
    return;
  }
  constexpr int LANES = fused_ut_lanes<DK>();
  static_assert(LANES == 3 && LANES * 128 < NTHREADS, "one call per lane below");
  static_assert(1 + 3 * LANES <= 16, "named barriers: one per lane, two per chunk slot");
  const int lane_id = (int)threadIdx.x >> 7;
  if (lane_id >= LANES) return;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const int BH = n_chain / (DV / BV);  // chain CTAs cover every head once
  const int nlanes = ((int)gridDim.x - n_chain) * LANES;
  // every chunk of every head, n-major.  Each lane's shared memory sits at a
  // compile-time offset (one inlined copy of the lane per lane index): with
  // the offset taken at run time the lane code does not fit in the 128
  // registers a thread of this launch has and spills.
  auto run = [&](auto lane_c) {
    constexpr int L = decltype(lane_c)::value;
    auto& us = *reinterpret_cast<utb::UtSmem<DK>*>(base + L * sizeof(utb::UtSmem<DK>));
    utb::ut_run<DK, false>(&tm_k, g, eta, eps, ws, T, H, nchunks, BH, 0, BH * nchunks, true,
                           err, nullptr, flags, us,
                           (int)threadIdx.x & 127, 1 + L, 1 + LANES + 2 * L,
                           ((int)blockIdx.x - n_chain) * LANES + L, nlanes, false);
  };
  if (lane_id == 0)
    run(std::integral_constant<int, 0>());
  else if (lane_id == 1)
    run(std::integral_constant<int, 1>());
  else
    run(std::integral_constant<int, 2>());
}

// Pass 1 of a cut chain (the transitions E, Phi of segments 0 .. S-2: CTAs
// 0 .. n_chain - 1, the mode-1 chain grid flattened, slab fastest, then
// head, then batch x segment) and, on the SMs those CTAs leave, UT lanes that
// make the factors of the chunks n >= n_split of every head (the last
// segment, which only pass 2 reads).  The two roles share no data and wait
// on nothing from each other, so this is a plain launch.
template <int DK>
__global__ void __launch_bounds__(NTHREADS, 1)
pass1_ut_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const float* __restrict__ g,
                const float* __restrict__ eta, float eps, float* __restrict__ E,
                float* __restrict__ phi, int T, int H, int DV, int nseg1, int seg_chunks,
                uint8_t* __restrict__ ws, int n_chain, int BH, int n_split, unsigned int* err) {
  const int nchunks = (T + C - 1) / C;
  if ((int)blockIdx.x < n_chain) {
    const int nx = (DV + DK) / BV;
    const int bx = (int)blockIdx.x % nx, by = ((int)blockIdx.x / nx) % H,
              bz = (int)blockIdx.x / (nx * H);
    chain_body<DK, false>(&tm_q, &tm_k, &tm_v, g, nullptr, nullptr, E, phi, nullptr, T, H, DV,
                          nseg1, seg_chunks, 1, ws, err, bx, by, bz, nullptr);
    return;
  }
  constexpr int LANES = fused_ut_lanes<DK>();
  static_assert(LANES == 3 && LANES * 128 < NTHREADS, "one call per lane below");
  const int lane_id = (int)threadIdx.x >> 7;
  if (lane_id >= LANES) return;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const int nlanes = ((int)gridDim.x - n_chain) * LANES;
  // each lane's shared memory at a compile-time offset (see prefill_kernel)
  auto run = [&](auto lane_c) {
    constexpr int L = decltype(lane_c)::value;
    auto& us = *reinterpret_cast<utb::UtSmem<DK>*>(base + L * sizeof(utb::UtSmem<DK>));
    utb::ut_run<DK, false>(&tm_k, g, eta, eps, ws, T, H, nchunks, BH, BH * n_split,
                           BH * (nchunks - n_split), true, err, nullptr, nullptr, us,
                           (int)threadIdx.x & 127, 1 + L, 1 + LANES + 2 * L,
                           ((int)blockIdx.x - n_chain) * LANES + L, nlanes, false);
  };
  if (lane_id == 0)
    run(std::integral_constant<int, 0>());
  else if (lane_id == 1)
    run(std::integral_constant<int, 1>());
  else
    run(std::integral_constant<int, 2>());
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

// One step of the segment start states: hstart(s + 1) = Phi_s h(s) + E_s,
// with h(0) = h0 (NULL = zeros), which step 0 also copies to hstart(0); fp32
// on CUDA cores, one launch per step.  A CTA takes 16 rows of one head's
// 64-column slab (h(s)'s slab and Phi_s's 16 rows staged in shared memory);
// thread t owns row t / 16 and 4 columns.  E and Phi hold the nseg - 1 first
// segments ([B][nseg - 1][H]), hstart all nseg ([B][nseg][H]).  (One CTA per
// head and slab walking every step, Phi's rows read one value per step from
// global memory, took ~80 µs of the 65K step; staging Phi in that form,
// ~60 µs.)
constexpr int kStartRows = 16;
template <int DK>
__global__ void __launch_bounds__(256)
segment_step_kernel(const float* __restrict__ h0, const float* __restrict__ E,
                    const float* __restrict__ Phi, float* __restrict__ hstart, int H, int DV,
                    int nseg, int step) {
  constexpr int RB = kStartRows;
  __shared__ __align__(16) float hsrc[DK][BV];
  __shared__ float ph[RB][DK + 1];
  const int slab = blockIdx.x, hh = blockIdx.y;
  const int b = blockIdx.z / (DK / RB), rb = blockIdx.z % (DK / RB);
  const int tid = threadIdx.x;
  const size_t head = (size_t)b * H + hh;
  const float* src = step > 0 ? hstart + (((size_t)b * nseg + step) * H + hh) * DK * DV
                     : h0     ? h0 + head * DK * DV
                              : nullptr;
  float* dst0 = hstart + ((size_t)b * nseg * H + hh) * DK * DV;  // hstart(0) of this head
  for (int idx = tid; idx < DK * BV / 4; idx += 256) {
    const int r = idx / (BV / 4), c = 4 * (idx % (BV / 4));
    const float4 x = src ? *reinterpret_cast<const float4*>(src + (size_t)r * DV + slab * BV + c)
                         : make_float4(0.f, 0.f, 0.f, 0.f);
    *reinterpret_cast<float4*>(&hsrc[r][c]) = x;
    if (step == 0 && r / RB == rb)
      *reinterpret_cast<float4*>(dst0 + (size_t)r * DV + slab * BV + c) = x;
  }
  const size_t pidx = ((size_t)b * (nseg - 1) + step) * H + hh;
  for (int idx = tid; idx < RB * DK; idx += 256) {
    const int r = idx / DK, k = idx % DK;
    ph[r][k] = Phi[(pidx * DK + rb * RB + r) * DK + k];
  }
  __syncthreads();
  const int r = tid >> 4, c = 4 * (tid & 15), row = rb * RB + r;
  float4 acc = *reinterpret_cast<const float4*>(E + (pidx * DK + row) * DV + slab * BV + c);
#pragma unroll 8
  for (int k = 0; k < DK; ++k) {
    const float a = ph[r][k];
    const float4 hv = *reinterpret_cast<const float4*>(&hsrc[k][c]);
    acc.x = fmaf(a, hv.x, acc.x);
    acc.y = fmaf(a, hv.y, acc.y);
    acc.z = fmaf(a, hv.z, acc.z);
    acc.w = fmaf(a, hv.w, acc.w);
  }
  *reinterpret_cast<float4*>(
      hstart + ((((size_t)b * nseg + step + 1) * H + hh) * DK + row) * DV + slab * BV + c) = acc;
}

template <int DK>
static cudaError_t launch_segment_starts(const float* h0, const float* E, const float* Phi,
                                         float* hstart, int B, int H, int DV, int nseg,
                                         cudaStream_t st) {
  for (int step = 0; step + 1 < nseg; ++step) {
    segment_step_kernel<DK><<<dim3(DV / BV, H, B * (DK / kStartRows)), 256, 0, st>>>(
        h0, E, Phi, hstart, H, DV, nseg, step);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

template <int DK, bool KDA>
cudaError_t launch_chain_dk(const void* q, const void* k, const void* v, const float* g,
                            const float* h0, void* o, float* hT, float* phi, int B, int T,
                            int H, int DV, int nseg, int seg_chunks, int mode,
                            const uint8_t* ws, unsigned int* err, cudaStream_t st,
                            float* hs = nullptr) {
  CUtensorMap mq, mk, mv;
  if (!make_map(&mq, q, DK, H, T, B) || !make_map(&mk, k, DK, H, T, B) ||
      !make_map(&mv, v, DV, H, T, B))
    return cudaErrorInvalidValue;
  const size_t smem = sizeof(ChainSmem<DK>) + 1024;
  static bool attr_set[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(chain_kernel<DK, KDA>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  dim3 grid((mode == 1 ? DV + DK : DV) / BV, H, B * nseg);
  chain_kernel<DK, KDA><<<grid, NTHREADS, smem, st>>>(mq, mk, mv, g, h0, (__nv_bfloat16*)o, hT,
                                                      phi, hs, T, H, DV, nseg, seg_chunks, mode,
                                                      ws, err);
  return cudaGetLastError();
}

// Number of segments the sequence is cut into for the state chain.  One CTA
// per (head, 64-column slab) walks its chunks in sequence, so with few heads
// most SMs idle; cutting the sequence into S segments runs S times as many
// CTAs, at the price of a first pass over segments 0 .. S-2 that also carries
// the dk identity columns (the segment transitions) and of a small combine.
// Cost model in units of "one chunk step of one wave of CTAs" on the 148 SMs
// of a B200; segments keep at least 8 chunks.
constexpr int kSmTarget = 148;
int chain_segments(int B, int T, int H, int dk, int dv) {
  const int nchunks = (T + C - 1) / C;
  const long p3 = (long)B * H * (dv / BV);          // CTAs per segment, outputs
  const long p1 = (long)B * H * ((dv + dk) / BV);   // CTAs per segment, pass 1
  auto waves = [](long ctas) { return (ctas + kSmTarget - 1) / kSmTarget; };
  long best = waves(p3) * nchunks;
  int best_s = 1;
  for (int sg = 2; sg <= 64 && nchunks / sg >= 8; ++sg) {
    const long len = (nchunks + sg - 1) / sg;
    if ((sg - 1) * len >= nchunks) continue;  // the last segment would be empty
    const long cost = (waves((sg - 1) * p1) + waves(sg * p3)) * len;
    if (cost * 5 < best * 4) {  // a clear gain only
      best = cost;
      best_s = sg;
    }
  }
  return best_s;
}

size_t ut_workspace_bytes(int B, int T, int H) {
  return (size_t)B * H * ((T + C - 1) / C) * kUtTileBytes;
}

// Segment buffers after the UT factors: E and the start states
// [B * S * H][dk][dv], Phi [B * S * H][dk][dk] (fp32).
size_t segment_bytes(int B, int T, int H, int dk, int dv) {
  const int sg = chain_segments(B, T, H, dk, dv);
  if (sg == 1) return 0;
  const size_t n = (size_t)B * sg * H;
  return n * ((size_t)2 * dk * dv + (size_t)dk * dk) * sizeof(float);
}

// The single-launch prefill keeps at least this many CTAs of UT lanes beside
// the state CTAs.
constexpr int kMinUtCtas = 8;

// Measured costs on a B200 (in units of one chain step, ~1.9 us at the
// 0.4B-scale layer): a UT lane takes ~5 chain steps per pair of chunks.
constexpr long kPairCost = 5, kStepCost = 1;

// Whether a shape runs as one launch: an uncut chain whose state CTAs leave
// room for UT CTAs on the 148 SMs of a B200, and for which the UT lanes on
// those SMs finish sooner than the UT kernel alone would on all of them plus
// the chain after it (the launcher checks the actual device again and
// otherwise runs the two kernels one after the other).
//
// The single launch is built but not taken: twice, a full run of the GPU
// tests stopped on an "unspecified launch failure" in the chunkwise backward
// of a short sequence whose forward ran it (once with four UT lanes per CTA,
// once with three), and reading the code has not found the cause.  Every
// shape runs the two kernels in turn until it is found.
constexpr bool kSingleLaunchTaken = false;
bool fused_shape(int B, int T, int H, int dk, int dv) {
  if (!kSingleLaunchTaken) return false;
  if (chain_segments(B, T, H, dk, dv) != 1) return false;
  const long n_chain = (long)B * H * (dv / BV);
  if (n_chain + kMinUtCtas > kSmTarget) return false;
  const long nchunks = (T + C - 1) / C, pairs = ((long)B * H * nchunks + 1) / 2;
  const long lanes_alone = 4L * kSmTarget;
  const long lanes_fused = 3L * (kSmTarget - n_chain);
  const long chain = nchunks * kStepCost;
  const long two = (pairs + lanes_alone - 1) / lanes_alone * kPairCost + chain;
  const long one = std::max((pairs + lanes_fused - 1) / lanes_fused * kPairCost, chain);
  return one < two;
}

// One ready flag per chunk after the factors (single launch only).
size_t flag_bytes(int B, int T, int H) {
  return ((size_t)B * H * ((T + C - 1) / C) * sizeof(unsigned int) + 255) & ~size_t(255);
}

}  // namespace

size_t chunk_workspace_bytes(int B, int T, int H, int dk, int dv, int dtype) {
  if (dtype != KLA_BF16 || B < 1 || H < 1 || T < 1 || dk != dv) return 0;
  return ut_workspace_bytes(B, T, H) + segment_bytes(B, T, H, dk, dv) +
         (fused_shape(B, T, H, dk, dv) ? flag_bytes(B, T, H) : 0);
}

bool chunk_single_launch(int B, int T, int H, int dk, int dv, size_t ws_bytes) {
  if (B < 1 || H < 1 || T < 1 || dk != dv || (dk != 64 && dk != 128)) return false;
  return fused_shape(B, T, H, dk, dv) &&
         ws_bytes >= ut_workspace_bytes(B, T, H) + flag_bytes(B, T, H);
}

size_t chunk_ut_workspace_bytes(int B, int T, int H, int dk, int dv, int dtype) {
  if (dtype != KLA_BF16 || B < 1 || H < 1 || T < 1 || dk != dv) return 0;
  return ut_workspace_bytes(B, T, H);
}

int chunk_chain_segments(int B, int T, int H, int dk, int dv, size_t ws_bytes) {
  const int sg = chain_segments(B, T, H, dk, dv);
  return sg > 1 && ws_bytes >= ut_workspace_bytes(B, T, H) + segment_bytes(B, T, H, dk, dv)
             ? sg
             : 1;
}

size_t chunk_workspace_used(int B, int T, int H, int dk, int dv, int dtype, size_t ws_bytes) {
  const size_t full = chunk_workspace_bytes(B, T, H, dk, dv, dtype);
  return ws_bytes >= full ? full : chunk_ut_workspace_bytes(B, T, H, dk, dv, dtype);
}

cudaError_t launch_chunk_ut(const void* k, const float* g, const float* eta, float eps,
                            int B, int T, int H, int dk, void* workspace, unsigned int* err,
                            cudaStream_t st, float* ratio_max) {
  if (dk != 64 && dk != 128) return cudaErrorNotSupported;
  CUtensorMap mk;
  if (!make_map(&mk, k, dk, H, T, B)) return cudaErrorInvalidValue;
  return launch_ut(mk, g, eta, eps, (uint8_t*)workspace, B, T, H, dk, err, st, ratio_max);
}

// The chain in S segments: pass 1 (E, Phi of segments 0 .. S-2), the start
// states, pass 2 (outputs of every segment from its start state).  The
// segment buffers follow the `tiles` bytes of per-chunk factors.
template <int DK, bool KDA>
static cudaError_t launch_segmented(const void* q, const void* k, const void* v, const float* g,
                                    const float* h0, void* o, float* hT, int B, int T, int H,
                                    int sg, uint8_t* ws, size_t tiles, unsigned int* err,
                                    cudaStream_t st, float* hs = nullptr);

cudaError_t launch_chunk_chain(const void* q, const void* k, const void* v, const float* g,
                               const float* h0, void* o, float* hT, int B, int T, int H,
                               int dk, int dv, void* workspace, size_t ws_bytes,
                               unsigned int* err, cudaStream_t st, float* hs) {
  if (dk != dv) return cudaErrorNotSupported;
  const int sg = chunk_chain_segments(B, T, H, dk, dv, ws_bytes);
  if (sg > 1) {
    uint8_t* wsm = (uint8_t*)workspace;
    const size_t tiles = ut_workspace_bytes(B, T, H);
    if (dk == 128)
      return launch_segmented<128, false>(q, k, v, g, h0, o, hT, B, T, H, sg, wsm, tiles, err,
                                          st, hs);
    return launch_segmented<64, false>(q, k, v, g, h0, o, hT, B, T, H, sg, wsm, tiles, err, st,
                                       hs);
  }
  const uint8_t* ws = (const uint8_t*)workspace;
  const int nchunks = (T + C - 1) / C;
  if (dk == 128)
    return launch_chain_dk<128, false>(q, k, v, g, h0, o, hT, nullptr, B, T, H, dv, 1, nchunks,
                                       0, ws, err, st, hs);
  if (dk == 64)
    return launch_chain_dk<64, false>(q, k, v, g, h0, o, hT, nullptr, B, T, H, dv, 1, nchunks,
                                      0, ws, err, st, hs);
  return cudaErrorNotSupported;
}

template <int DK, bool KDA>
static cudaError_t launch_segmented(const void* q, const void* k, const void* v, const float* g,
                                    const float* h0, void* o, float* hT, int B, int T, int H,
                                    int sg, uint8_t* ws, size_t tiles, unsigned int* err,
                                    cudaStream_t st, float* hs) {
  constexpr int DV = DK;
  const int nchunks = (T + C - 1) / C;
  const int len = (nchunks + sg - 1) / sg;
  const size_t n = (size_t)B * sg * H;
  float* E = reinterpret_cast<float*>(ws + tiles);
  float* hstart = E + n * DK * DV;
  float* Phi = hstart + n * DK * DV;
  // pass 1 covers segments 0 .. S-2 (launched as S - 1 segments of `len`
  // chunks, so E and Phi are laid out [B][S - 1][H])
  cudaError_t e = launch_chain_dk<DK, KDA>(q, k, v, g, nullptr, nullptr, E, Phi, B, T, H, DV,
                                           sg - 1, len, 1, ws, err, st);
  if (e != cudaSuccess) return e;
  e = launch_segment_starts<DK>(h0, E, Phi, hstart, B, H, DV, sg, st);
  if (e != cudaSuccess) return e;
  return launch_chain_dk<DK, KDA>(q, k, v, g, hstart, o, hT, nullptr, B, T, H, DV, sg, len, 0,
                                  ws, err, st, hs);
}

// The cut chain with the UT work overlapped: the UT kernel for the chunks of
// segments 0 .. S-2 only, then pass 1 with UT lanes for the last segment on
// the SMs its CTAs leave, the start states and pass 2.  cudaErrorNotSupported
// (nothing launched) where those lanes would not finish within pass 1 by the
// cost model, or pass 1 leaves fewer than kMinUtCtas SMs.
template <int DK>
static cudaError_t launch_segmented_overlap(const void* q, const void* k, const void* v,
                                            const float* g, const float* eta, float eps,
                                            const float* h0, void* o, float* hT, int B, int T,
                                            int H, int sg, uint8_t* ws, size_t tiles,
                                            unsigned int* err, cudaStream_t st, float* hs) {
  constexpr int DV = DK;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  static int sms[64] = {};
  static bool attr[64] = {};
  constexpr size_t smem = fused_smem_bytes<DK>();
  if (!sms[dev]) {
    cudaError_t e = cudaDeviceGetAttribute(&sms[dev], cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
  }
  const int nchunks = (T + C - 1) / C;
  const int len = (nchunks + sg - 1) / sg;
  const int n_split = (sg - 1) * len;
  const long BH = (long)B * H;
  const long n_chain = BH * ((DV + DK) / BV) * (sg - 1);
  const long ut_ctas = sms[dev] - n_chain;
  if (ut_ctas < kMinUtCtas) return cudaErrorNotSupported;
  const long lanes = (long)fused_ut_lanes<DK>() * ut_ctas;
  const long pairs = (BH * (nchunks - n_split) + 1) / 2;
  if ((pairs + lanes - 1) / lanes * kPairCost > (long)len * kStepCost) return cudaErrorNotSupported;
  if (!attr[dev]) {
    cudaError_t e = cudaFuncSetAttribute(pass1_ut_kernel<DK>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    attr[dev] = true;
  }
  CUtensorMap mq, mk, mv;
  if (!make_map(&mq, q, DK, H, T, B) || !make_map(&mk, k, DK, H, T, B) ||
      !make_map(&mv, v, DV, H, T, B))
    return cudaErrorInvalidValue;
  const size_t n = (size_t)B * sg * H;
  float* E = reinterpret_cast<float*>(ws + tiles);
  float* hstart = E + n * DK * DV;
  float* Phi = hstart + n * DK * DV;
  cudaError_t e = launch_ut_first(mk, g, eta, eps, ws, B, T, H, DK, n_split, err, st);
  if (e != cudaSuccess) return e;
  pass1_ut_kernel<DK><<<(unsigned)(n_chain + ut_ctas), NTHREADS, smem, st>>>(
      mq, mk, mv, g, eta, eps, E, Phi, T, H, DV, sg - 1, len, ws, (int)n_chain, (int)BH, n_split,
      err);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  e = launch_segment_starts<DK>(h0, E, Phi, hstart, B, H, DV, sg, st);
  if (e != cudaSuccess) return e;
  return launch_chain_dk<DK, false>(q, k, v, g, hstart, o, hT, nullptr, B, T, H, DV, sg, len, 0,
                                    ws, err, st, hs);
}

// The single-launch prefill (see prefill_kernel).  cudaErrorNotSupported when
// this device cannot hold it (too few SMs beside the state CTAs, no
// cooperative launch): the caller then runs the two kernels in turn.
template <int DK>
static cudaError_t launch_fused(const void* q, const void* k, const void* v, const float* g,
                                const float* eta, float eps, const float* h0, void* o,
                                float* hT, int B, int T, int H, uint8_t* ws, unsigned int* err,
                                cudaStream_t st, float* hs) {
  constexpr int DV = DK;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  static int sms[64] = {};
  static int fits[64] = {};  // 0 unknown, 1 yes, -1 no
  constexpr size_t smem = fused_smem_bytes<DK>();
  if (!fits[dev]) {
    int coop = 0, nb = 0;
    cudaError_t e = cudaDeviceGetAttribute(&sms[dev], cudaDevAttrMultiProcessorCount, dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, dev);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(prefill_kernel<DK>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)smem);
    if (e == cudaSuccess)
      e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, prefill_kernel<DK>, NTHREADS, smem);
    if (e != cudaSuccess) return e;
    fits[dev] = (coop && nb >= 1) ? 1 : -1;
  }
  const int n_chain = B * H * (DV / BV);
  if (fits[dev] < 0 || n_chain + kMinUtCtas > sms[dev]) return cudaErrorNotSupported;
  CUtensorMap mq, mk, mv;
  if (!make_map(&mq, q, DK, H, T, B) || !make_map(&mk, k, DK, H, T, B) ||
      !make_map(&mv, v, DV, H, T, B))
    return cudaErrorInvalidValue;
  unsigned int* flags = reinterpret_cast<unsigned int*>(ws + ut_workspace_bytes(B, T, H));
  cudaError_t e = cudaMemsetAsync(flags, 0, flag_bytes(B, T, H), st);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(sms[dev]);
  cfg.blockDim = dim3(NTHREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, prefill_kernel<DK>, mq, mk, mv, g, eta, eps, h0,
                            (__nv_bfloat16*)o, hT, hs, T, H, DV, ws, flags, n_chain, err);
}

cudaError_t launch_chunk_tc(const void* q, const void* k, const void* v, const float* g,
                            const float* eta, float eps, const float* h0, void* o, float* hT,
                            int B, int T, int H, int dk, int dv, void* workspace,
                            size_t ws_bytes, unsigned int* err, cudaStream_t st, float* hs) {
  if (dk != dv || (dk != 64 && dk != 128)) return cudaErrorNotSupported;
  if (fused_shape(B, T, H, dk, dv) &&
      ws_bytes >= ut_workspace_bytes(B, T, H) + flag_bytes(B, T, H)) {
    uint8_t* wsm = (uint8_t*)workspace;
    const cudaError_t e =
        dk == 128 ? launch_fused<128>(q, k, v, g, eta, eps, h0, o, hT, B, T, H, wsm, err, st, hs)
                  : launch_fused<64>(q, k, v, g, eta, eps, h0, o, hT, B, T, H, wsm, err, st, hs);
    if (e != cudaErrorNotSupported) return e;
  }
  const int sg = chunk_chain_segments(B, T, H, dk, dv, ws_bytes);
  if (sg > 1) {
    uint8_t* wsm = (uint8_t*)workspace;
    const size_t tiles = ut_workspace_bytes(B, T, H);
    const cudaError_t e =
        dk == 128 ? launch_segmented_overlap<128>(q, k, v, g, eta, eps, h0, o, hT, B, T, H, sg,
                                                  wsm, tiles, err, st, hs)
                  : launch_segmented_overlap<64>(q, k, v, g, eta, eps, h0, o, hT, B, T, H, sg,
                                                 wsm, tiles, err, st, hs);
    if (e != cudaErrorNotSupported) return e;
  }
  cudaError_t e = launch_chunk_ut(k, g, eta, eps, B, T, H, dk, workspace, err, st);
  if (e != cudaSuccess) return e;
  return launch_chunk_chain(q, k, v, g, h0, o, hT, B, T, H, dk, dv, workspace, ws_bytes, err,
                            st, hs);
}

// ---------------------------------------------------- per-channel gate
namespace {
size_t kda_tiles_bytes(int B, int T, int H, int dk) {
  return (size_t)B * H * ((T + C - 1) / C) * kda_tile_offsets(dk).total;
}
}  // namespace

size_t kda_chunk_workspace_bytes(int B, int T, int H, int dk, int dv, int dtype) {
  if (dtype != KLA_BF16 || B < 1 || H < 1 || T < 1 || dk != dv || (dk != 64 && dk != 128))
    return 0;
  return kda_tiles_bytes(B, T, H, dk);
}

// The per-channel-gate prefill always runs the uncut chain (its cut-chain
// mode is not used: see the safety record of the design notes).
cudaError_t launch_kda_chunk(const void* q, const void* k, const void* v, const float* g,
                             const float* eta, float eps, const float* h0, void* o, float* hT,
                             int B, int T, int H, int dk, int dv, void* workspace,
                             size_t ws_bytes, unsigned int* err, cudaStream_t st) {
  (void)ws_bytes;
  if (dk != dv || (dk != 64 && dk != 128)) return cudaErrorNotSupported;
  cudaError_t e = launch_kda_prep(q, k, g, eta, eps, B, T, H, dk, workspace, st);
  if (e != cudaSuccess) return e;
  uint8_t* ws = (uint8_t*)workspace;
  const int nchunks = (T + C - 1) / C;
  if (dk == 128)
    return launch_chain_dk<128, true>(q, k, v, g, h0, o, hT, nullptr, B, T, H, dv, 1, nchunks, 0,
                                      ws, err, st);
  return launch_chain_dk<64, true>(q, k, v, g, h0, o, hT, nullptr, B, T, H, dv, 1, nchunks, 0,
                                   ws, err, st);
}

}  // namespace kla
