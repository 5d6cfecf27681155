// Token-serial backward of the KLA / gated delta rule prefill on CUDA cores
// (fp32 arithmetic): the gradients of a loss L given dL/do and dL/dh_T.  Also
// the per-channel-gate (KDA) form, see the end of this comment.
//
// Forward per token, h = S^T [dk x dv] ("Kaczmarz Linear Attention",
// Abstract; "Deep Dive into KDA", section 2.2):
//   beta = eta / (||k||^2 + eps) (KLA) or given (gated delta form);
//   alpha = e^g;  r = h^T k;  u = beta (v - alpha r);  h <- alpha h + k u^T;
//   o = h^T q.
// The pages print no backward; this is the adjoint of those lines taken in
// reverse token order (dH = dL/dh_t):
//   dH += q do^T;  dq = h_t do;  du = dH^T k;  dr = -alpha beta du;
//   dk = dH u + h_{t-1} dr;  dv = beta du;  dbeta = du . (v - alpha r);
//   dalpha = <dH, h_{t-1}> - beta du . r;  dH <- alpha dH + k dr^T;
//   dg = alpha dalpha;  KLA: deta = dbeta / (||k||^2 + eps),
//   dk += -2 dbeta eta k / (||k||^2 + eps)^2.
//
// The reverse sweep needs h_{t-1} at every token.  The step is not inverted
// (with beta ||k||^2 = 1 it is singular); states are recomputed instead:
//  * bwd_checkpoint_kernel runs the forward and stores h at the start of every
//    64-token block, fp32 [B][H][nblk][dk][dv], and every token's beta and
//    alpha;
//  * bwd_kernel walks the blocks in reverse; per block it reruns the forward
//    from the checkpoint keeping the state at every 4th token (thread-private
//    scratch in global memory, 256 KB per CTA, so it stays in L2), then for
//    each 4-token sub-block in reverse reruns those tokens keeping their
//    states in shared memory and takes the reverse steps.
// Both kernels first copy a block's operands (k, q, the CTA's columns of v and
// dL/do, beta, alpha) into shared memory, so no token step waits on a global
// load.  Every rerun uses the same step function on the same beta and alpha,
// so the recomputed states are bitwise those of the first forward.
//
// Layout: a CTA of 256 threads owns a 32-column slab of one head's state and
// of its adjoint.  Warp w has columns 4w .. 4w+3; lane 4 rg + c owns column
// 4w + c and rows rg R .. rg R + R - 1 (R = dk / 8).  Sums over rows (r, du,
// ||k||^2) take three shuffles.  Row vectors summed over columns (dq, dk) are
// reduced over the 4 column lanes of a warp by two halving exchanges, over the
// 8 warps in shared memory once per sub-block, and over the dv / 32 slabs by
// bwd_finish_kernel, which also applies the step size's chain rule.
//
// Per-channel gate ("Deep Dive into KDA", section 2.3; template flag VG):
// forward  hd = Diag(a) h_{t-1} (a = e^{g_t}, one per key channel);
// r = hd^T k;  u = beta (v - r);  h_t = hd + k u^T.  Reverse:
//   dH += q do^T;  dq = h_t do;  du = dH^T k;  dr = -beta du;  dv = beta du;
//   dbeta = du . (v - r);  dk = dH u + hd dr;  Hd = dH + k dr^T;
//   dg_i = sum_j Hd_ij hd_ij;  dH <- Diag(a) Hd.
// dg is a third row vector summed over the columns.  The block stage then
// also holds a = e^g per token and channel, so the sub-blocks are 2 tokens
// to stay within shared memory.
#include "kla_common.cuh"

namespace kla {

namespace bwd {

constexpr int NT = 256;    // threads per CTA
constexpr int BV = 32;     // state columns per CTA
constexpr int BLK = 64;    // tokens per checkpoint (and per operand stage)
constexpr unsigned FULL = 0xffffffffu;

// Tokens per sub-block (their states kept in shared memory) and the number of
// row vectors summed over the columns per token (dq, dk; dg with VG).
template <bool VG> constexpr int sub_tokens() { return VG ? 2 : 4; }
template <bool VG> constexpr int n_rowvec() { return VG ? 3 : 2; }

// Sum over the 8 row groups of one column (lane bits 2..4).
__device__ __forceinline__ float rows_sum(float x) {
  x += __shfl_xor_sync(FULL, x, 4);
  x += __shfl_xor_sync(FULL, x, 8);
  x += __shfl_xor_sync(FULL, x, 16);
  return x;
}

// Key and query rows in shared memory get 4 floats of padding after every 32:
// a lane reads 4-float pieces of its row group's R rows, and without the pad
// the row groups 2 apart (64 or 32 bytes) fall on the same banks.
__host__ __device__ constexpr int kpad(int i) { return i + ((i >> 5) << 2); }

// One 64-token block's operands, staged in shared memory widened to fp32: the
// full key and query rows, the CTA's 32 columns of v and dL/do, per token the
// step size beta and the decay alpha = e^g, and with a per-channel gate the
// decays a = e^g per token and key channel.
template <int DK, bool VG>
struct alignas(16) Ops {
  float k[BLK][kpad(DK)];
  float q[BLK][kpad(DK)];
  float a[VG ? BLK : 1][VG ? kpad(DK) : 4];
  float v[BLK][BV];
  float d[BLK][BV];
  float beta[BLK];
  float alpha[BLK];
};

// Elements row0 .. row0 + R - 1 of a padded shared-memory row.
template <int R>
__device__ __forceinline__ void row_ld(const float* row, int row0, float (&x)[R]) {
#pragma unroll
  for (int m = 0; m < R; m += 4) {
    const float4 a = *reinterpret_cast<const float4*>(row + kpad(row0 + m));
    x[m] = a.x; x[m + 1] = a.y; x[m + 2] = a.z; x[m + 3] = a.w;
  }
}

// A thread's R state values to / from a [R/4][NT][4] scratch slot: 4-float
// pieces interleaved by thread, so one vector access of a warp is 512
// contiguous bytes (p = slot + 4 * tid).
template <int R>
__device__ __forceinline__ void vec_st(float* p, const float (&x)[R]) {
#pragma unroll
  for (int m = 0; m < R; m += 4)
    *reinterpret_cast<float4*>(p + m * NT) = make_float4(x[m], x[m + 1], x[m + 2], x[m + 3]);
}
template <int R>
__device__ __forceinline__ void vec_ld(const float* p, float (&x)[R]) {
#pragma unroll
  for (int m = 0; m < R; m += 4) {
    const float4 a = *reinterpret_cast<const float4*>(p + m * NT);
    x[m] = a.x; x[m + 1] = a.y; x[m + 2] = a.z; x[m + 3] = a.w;
  }
}

// 4 consecutive elements from global memory -> 4 floats in shared memory.
template <typename T>
__device__ __forceinline__ void copy4(float* dst, const T* src) {
  *reinterpret_cast<float4*>(dst) = IO<T>::ld4(src);
}

// Cooperative copy of tokens t0 .. t0 + n - 1 into the stage, widened; with
// VG also a = e^g of every key channel.
template <typename T, int DK, int DV, bool VG, bool WITH_QD>
__device__ __forceinline__ void stage_block(Ops<DK, VG>& s, const T* __restrict__ q,
                                            const T* __restrict__ k, const T* __restrict__ v,
                                            const T* __restrict__ dout,
                                            const float* __restrict__ g, int b, int hh,
                                            int Tlen, int H, int t0, int n, int j0) {
  constexpr int RK = DK / 4, RV = BV / 4;  // 4-element pieces per row
  for (int p = threadIdx.x; p < n * RK; p += NT) {
    const int t = p / RK, ch = p % RK;
    const size_t tok = ((size_t)b * Tlen + t0 + t) * H + hh;
    copy4(&s.k[t][kpad(ch * 4)], k + tok * DK + ch * 4);
    if constexpr (WITH_QD) copy4(&s.q[t][kpad(ch * 4)], q + tok * DK + ch * 4);
    if constexpr (VG) {
      const float4 x = *reinterpret_cast<const float4*>(g + tok * DK + ch * 4);
      *reinterpret_cast<float4*>(&s.a[t][kpad(ch * 4)]) =
          make_float4(expf(x.x), expf(x.y), expf(x.z), expf(x.w));
    }
  }
  for (int p = threadIdx.x; p < n * RV; p += NT) {
    const int t = p / RV, ch = p % RV;
    const size_t tok = ((size_t)b * Tlen + t0 + t) * H + hh;
    copy4(&s.v[t][ch * 4], v + tok * DV + j0 + ch * 4);
    if constexpr (WITH_QD) copy4(&s.d[t][ch * 4], dout + tok * DV + j0 + ch * 4);
  }
}

// One forward token step of the lane's part of the state, operands from the
// stage (token t of the block).
template <int DK, bool VG>
__device__ __forceinline__ void fwd_step(float (&hs)[DK / 8], const Ops<DK, VG>& s, int t,
                                         int row0, int col) {
  constexpr int R = DK / 8;
  float kk[R];
  row_ld<R>(s.k[t], row0, kk);
  float alpha = 1.f;
  if constexpr (VG) {  // Diag(a) h first; the erase reads the decayed rows
    float aa[R];
    row_ld<R>(s.a[t], row0, aa);
#pragma unroll
    for (int m = 0; m < R; ++m) hs[m] *= aa[m];
  } else {
    alpha = s.alpha[t];
  }
  float r0 = 0.f, r1 = 0.f;
#pragma unroll
  for (int m = 0; m < R; m += 2) {
    r0 = fmaf(hs[m], kk[m], r0);
    r1 = fmaf(hs[m + 1], kk[m + 1], r1);
  }
  const float r = rows_sum(r0 + r1);
  const float u = s.beta[t] * (s.v[t][col] - alpha * r);
#pragma unroll
  for (int m = 0; m < R; ++m) hs[m] = fmaf(kk[m], u, alpha * hs[m]);
}

// Sum the lane's R row values over the 4 column lanes of its row group; the
// lane stores R/4 of the sums, rows base .. base + R/4 - 1 of the group, at
// dst[base ..].
template <int R>
__device__ __forceinline__ void cols_sum_store(const float (&x)[R], float* dst, int c) {
  constexpr int H1 = R / 2, H2 = R / 4;
  const bool b1 = (c >> 1) & 1, b0 = c & 1;
  float y[H1];
#pragma unroll
  for (int i = 0; i < H1; ++i) {
    const float keep = b1 ? x[i + H1] : x[i], send = b1 ? x[i] : x[i + H1];
    y[i] = keep + __shfl_xor_sync(FULL, send, 2);
  }
  float z[H2];
#pragma unroll
  for (int i = 0; i < H2; ++i) {
    const float keep = b0 ? y[i + H2] : y[i], send = b0 ? y[i] : y[i + H2];
    z[i] = keep + __shfl_xor_sync(FULL, send, 1);
  }
  const int base = (b1 ? H1 : 0) + (b0 ? H2 : 0);
#pragma unroll
  for (int i = 0; i < H2; i += 2)
    *reinterpret_cast<float2*>(dst + base + i) = make_float2(z[i], z[i + 1]);
}

template <int DK, bool VG>
constexpr size_t smem_bytes() {
  constexpr size_t SUB = sub_tokens<VG>(), NQ = n_rowvec<VG>();
  return sizeof(Ops<DK, VG>) +
         sizeof(float) * (SUB * (DK / 8) * NT + SUB * NQ * 8 * DK + SUB * 2 * NT);
}

}  // namespace bwd

// Forward with a checkpoint of h at the start of each 64-token block; also
// writes every token's beta and alpha = e^g (CTAs of slab 0).
template <typename T, int DK, int DV, bool VG>
__global__ void __launch_bounds__(bwd::NT)
bwd_checkpoint_kernel(const T* __restrict__ k, const T* __restrict__ v,
                      const float* __restrict__ g, const float* __restrict__ eta, float eps,
                      const float* __restrict__ h0, float* __restrict__ ck,
                      float* __restrict__ beta_out, float* __restrict__ alpha_out, int Tlen,
                      int H, int nblk) {
  using namespace bwd;
  constexpr int R = DK / 8;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  Ops<DK, VG>& s = *reinterpret_cast<Ops<DK, VG>*>(smem_raw);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int rg = lane >> 2, c = lane & 3;
  const int col = warp * 4 + c, j = blockIdx.x * BV + col, row0 = rg * R;
  const int hh = blockIdx.y, b = blockIdx.z;
  const size_t head = (size_t)b * H + hh;

  float hs[R];
#pragma unroll
  for (int m = 0; m < R; ++m) hs[m] = h0 ? h0[(head * DK + row0 + m) * DV + j] : 0.f;

  for (int blk = 0; blk < nblk; ++blk) {
    const int t0 = blk * BLK, n = min(BLK, Tlen - t0);
    {
      float* dst = ck + ((head * nblk + blk) * DK + row0) * DV + j;
#pragma unroll
      for (int m = 0; m < R; ++m) dst[(size_t)m * DV] = hs[m];
    }
    __syncthreads();  // the previous block's stage is no longer read
    stage_block<T, DK, DV, VG, false>(s, nullptr, k, v, nullptr, g, b, hh, Tlen, H, t0, n,
                                      blockIdx.x * BV);
    for (int t = threadIdx.x; t < n; t += NT) {  // eta and g, replaced below
      const size_t tok = ((size_t)b * Tlen + t0 + t) * H + hh;
      s.beta[t] = eta[tok];
      s.alpha[t] = VG ? 0.f : g[tok];
    }
    __syncthreads();
    for (int t = warp; t < n; t += NT / 32) {  // ||k||^2 -> beta, and alpha
      float a = 0.f;
      for (int i = lane; i < DK; i += 32) a = fmaf(s.k[t][kpad(i)], s.k[t][kpad(i)], a);
      a = warp_sum(a);
      if (lane == 0) {
        const size_t tok = ((size_t)b * Tlen + t0 + t) * H + hh;
        const float be = step_size(s.beta[t], a, eps), al = expf(s.alpha[t]);
        s.beta[t] = be;
        s.alpha[t] = al;
        if (blockIdx.x == 0) {
          beta_out[tok] = be;
          alpha_out[tok] = al;
        }
      }
    }
    __syncthreads();
    if (blk + 1 < nblk)
      for (int t = 0; t < n; ++t) fwd_step<DK, VG>(hs, s, t, row0, col);
  }
}

template <typename T, int DK, int DV, bool VG>
__global__ void __launch_bounds__(bwd::NT)
bwd_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
           const float* __restrict__ g, const T* __restrict__ dout,
           const float* __restrict__ dhT, const float* __restrict__ beta_in,
           const float* __restrict__ alpha_in, const float* __restrict__ ck,
           float* __restrict__ sub, float* __restrict__ part, float* __restrict__ ps,
           float* __restrict__ dv_out, float* __restrict__ dh0, int Tlen, int H, int nblk) {
  using namespace bwd;
  constexpr int R = DK / 8;
  constexpr int NSLAB = DV / BV;
  constexpr int SUB = sub_tokens<VG>(), NSUB = BLK / SUB, NQ = n_rowvec<VG>();
  extern __shared__ __align__(16) unsigned char smem_raw[];
  Ops<DK, VG>& s = *reinterpret_cast<Ops<DK, VG>*>(smem_raw);
  float* st = reinterpret_cast<float*>(smem_raw + sizeof(Ops<DK, VG>));  // [SUB][R/4][NT][4]
  float* red = st + SUB * R * NT;         // [SUB][NQ][8 warps][DK]
  float* reds = red + SUB * NQ * 8 * DK;  // [SUB][2][NT]: dalpha, dbeta per thread

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int rg = lane >> 2, c = lane & 3;
  const int slab = blockIdx.x, hh = blockIdx.y, b = blockIdx.z;
  const int col = warp * 4 + c, j = slab * BV + col, row0 = rg * R;
  const size_t head = (size_t)b * H + hh;
  const size_t ntok = (size_t)gridDim.z * Tlen * H;
  float* my_sub = sub + (head * NSLAB + slab) * (size_t)(NSUB * R * NT);
  auto tok_of = [&](int t) { return ((size_t)b * Tlen + t) * H + hh; };

  float dH[R];
#pragma unroll
  for (int m = 0; m < R; ++m) dH[m] = dhT ? dhT[(head * DK + row0 + m) * DV + j] : 0.f;

  for (int blk = nblk - 1; blk >= 0; --blk) {
    const int t0 = blk * BLK, n = min(BLK, Tlen - t0);
    stage_block<T, DK, DV, VG, true>(s, q, k, v, dout, g, b, hh, Tlen, H, t0, n, slab * BV);
    for (int t = tid; t < n; t += NT) {
      s.beta[t] = beta_in[tok_of(t0 + t)];
      s.alpha[t] = alpha_in[tok_of(t0 + t)];
    }
    float hs[R];
    {
      const float* src = ck + ((head * nblk + blk) * DK + row0) * DV + j;
#pragma unroll
      for (int m = 0; m < R; ++m) hs[m] = src[(size_t)m * DV];
    }
    __syncthreads();
    // the state at every SUB-th token of the block (thread-private scratch)
    for (int t = 0; t < n; ++t) {
      if (t % SUB == 0) vec_st<R>(my_sub + (size_t)(t / SUB) * R * NT + 4 * tid, hs);
      if (t + 1 < n) fwd_step<DK, VG>(hs, s, t, row0, col);
    }
    const int nsb = (n + SUB - 1) / SUB;
    float hn[R];  // the next sub-block's start state, loaded one sub-block ahead
    vec_ld<R>(my_sub + (size_t)(nsb - 1) * R * NT + 4 * tid, hn);
    for (int sb = nsb - 1; sb >= 0; --sb) {
      const int s0 = sb * SUB, s1 = min(s0 + SUB, n);  // block-local tokens
#pragma unroll
      for (int m = 0; m < R; ++m) hs[m] = hn[m];
      if (sb > 0) vec_ld<R>(my_sub + (size_t)(sb - 1) * R * NT + 4 * tid, hn);
      // states before each token of the sub-block
      for (int t = s0; t < s1; ++t) {
        vec_st<R>(st + (size_t)(t - s0) * R * NT + 4 * tid, hs);
        if (t + 1 < s1) fwd_step<DK, VG>(hs, s, t, row0, col);
      }
      // reverse steps
      for (int t = s1 - 1; t >= s0; --t) {
        const int si = t - s0;
        float hp[R], kk[R], aa[R];
        vec_ld<R>(st + (size_t)si * R * NT + 4 * tid, hp);
        row_ld<R>(s.k[t], row0, kk);
        float alpha = 1.f;
        if constexpr (VG) {  // hp <- the decayed state Diag(a) h_{t-1}
          row_ld<R>(s.a[t], row0, aa);
#pragma unroll
          for (int m = 0; m < R; ++m) hp[m] *= aa[m];
        } else {
          alpha = s.alpha[t];
        }
        float r0 = 0.f, r1 = 0.f;
#pragma unroll
        for (int m = 0; m < R; m += 2) {
          r0 = fmaf(hp[m], kk[m], r0);
          r1 = fmaf(hp[m + 1], kk[m + 1], r1);
        }
        const float r = rows_sum(r0 + r1);
        const float beta = s.beta[t];
        const float vj = s.v[t][col], dj = s.d[t][col];
        const float u = beta * (vj - alpha * r);
        float x[R];
        {
          float qq[R];
          row_ld<R>(s.q[t], row0, qq);
          float du0 = 0.f, du1 = 0.f;
#pragma unroll
          for (int m = 0; m < R; ++m) {
            x[m] = fmaf(kk[m], u, alpha * hp[m]) * dj;  // h_t[i][j] do_j
            dH[m] = fmaf(qq[m], dj, dH[m]);
            if (m & 1)
              du1 = fmaf(dH[m], kk[m], du1);
            else
              du0 = fmaf(dH[m], kk[m], du0);
          }
          cols_sum_store(x, red + ((size_t)(si * NQ + 0) * 8 + warp) * DK + row0, c);
          const float du = rows_sum(du0 + du1);
          const float dr = -alpha * beta * du;
          float da0 = 0.f, da1 = 0.f, db = 0.f;
          if constexpr (VG) {
            float xg[R];
#pragma unroll
            for (int m = 0; m < R; ++m) {
              x[m] = fmaf(dH[m], u, hp[m] * dr);
              const float hd = fmaf(kk[m], dr, dH[m]);  // dL/d(decayed state)
              xg[m] = hd * hp[m];
              dH[m] = aa[m] * hd;
            }
            cols_sum_store(xg, red + ((size_t)(si * NQ + 2) * 8 + warp) * DK + row0, c);
          } else {
#pragma unroll
            for (int m = 0; m < R; ++m) {
              x[m] = fmaf(dH[m], u, hp[m] * dr);
              if (m & 1)
                da1 = fmaf(dH[m], hp[m], da1);
              else
                da0 = fmaf(dH[m], hp[m], da0);
              dH[m] = fmaf(kk[m], dr, alpha * dH[m]);
            }
          }
          float da = da0 + da1;
          if (rg == 0) {  // per-column terms, once per column
            da -= beta * du * r;
            db = du * (vj - alpha * r);
            dv_out[tok_of(t0 + t) * DV + j] = beta * du;
          }
          cols_sum_store(x, red + ((size_t)(si * NQ + 1) * 8 + warp) * DK + row0, c);
          // per-thread terms, summed over the CTA after the sub-block
          reds[(si * 2 + 0) * NT + tid] = VG ? 0.f : da;
          reds[(si * 2 + 1) * NT + tid] = db;
        }
      }
      __syncthreads();
      // sums over the 8 warps -> this slab's partials (row vector qi of the
      // token in part[qi][slab][tok][DK])
      const int ns = s1 - s0;
      for (int p = tid; p < ns * NQ * DK; p += NT) {
        const int si = p / (NQ * DK), qi = (p / DK) % NQ, i = p % DK;
        const float* src = red + ((size_t)(si * NQ + qi) * 8) * DK + i;
        float a = 0.f;
#pragma unroll
        for (int w = 0; w < 8; ++w) a += src[w * DK];
        part[(((size_t)qi * NSLAB + slab) * ntok + tok_of(t0 + s0 + si)) * DK + i] = a;
      }
      if (warp < ns * 2) {  // warp (si, qi) sums its token's NT terms
        const int si = warp >> 1, qi = warp & 1;
        const float* src = reds + (si * 2 + qi) * NT;
        float a = 0.f;
#pragma unroll
        for (int w = 0; w < NT / 32; ++w) a += src[w * 32 + lane];
        a = warp_sum(a);
        if (lane == 0) ps[((size_t)slab * ntok + tok_of(t0 + s0 + si)) * 2 + qi] = a;
      }
      __syncthreads();
    }
  }
  if (dh0) {
#pragma unroll
    for (int m = 0; m < R; ++m) dh0[(head * DK + row0 + m) * DV + j] = dH[m];
  }
}

// Per token (one warp): dq, dk (and with VG dg) summed over the slabs; for a
// per-token gate dg = alpha dalpha; the step size's chain rule into deta and
// dk (KLA), or dbeta as is (eps < 0).
template <typename T, int DK, bool VG>
__global__ void __launch_bounds__(256)
bwd_finish_kernel(const T* __restrict__ k, const float* __restrict__ eta,
                  const float* __restrict__ alpha_in, float eps, const float* __restrict__ part,
                  const float* __restrict__ ps, int nslab, size_t ntok, float* __restrict__ dq,
                  float* __restrict__ dk, float* __restrict__ dg, float* __restrict__ deta) {
  constexpr int E = DK / 32;  // elements per lane
  const int lane = threadIdx.x & 31;
  const size_t tok = (size_t)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
  if (tok >= ntok) return;
  const size_t qstride = (size_t)nslab * ntok * DK;  // between row vectors
  float kk[E], sq[E], sk[E], sg[E];
  float n2 = 0.f;
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const int i = lane * E + e;
    kk[e] = IO<T>::ld(k + tok * DK + i);
    n2 = fmaf(kk[e], kk[e], n2);
    sq[e] = 0.f;
    sk[e] = 0.f;
    sg[e] = 0.f;
  }
  n2 = warp_sum(n2);
  float sa = 0.f, sb = 0.f;
  for (int sl = 0; sl < nslab; ++sl) {
    const size_t base = (size_t)sl * ntok + tok;
#pragma unroll
    for (int e = 0; e < E; ++e) {
      sq[e] += part[base * DK + lane * E + e];
      sk[e] += part[qstride + base * DK + lane * E + e];
      if constexpr (VG) sg[e] += part[2 * qstride + base * DK + lane * E + e];
    }
    sa += ps[base * 2 + 0];
    sb += ps[base * 2 + 1];
  }
  float coef = 0.f;
  if (eps >= 0.f) {  // beta = eta / (||k||^2 + eps)
    const float den = n2 + eps;
    coef = -2.f * sb * eta[tok] / (den * den);
    if (lane == 0) deta[tok] = sb / den;
  } else if (lane == 0) {
    deta[tok] = sb;  // dbeta
  }
  if constexpr (!VG) {
    if (lane == 0) dg[tok] = alpha_in[tok] * sa;
  }
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const int i = lane * E + e;
    dq[tok * DK + i] = sq[e];
    dk[tok * DK + i] = fmaf(coef, kk[e], sk[e]);
    if constexpr (VG) dg[tok * DK + i] = sg[e];
  }
}

// ---- workspace and launch

static size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

struct BwdWs {
  size_t ck, sub, part, ps, beta, alpha, total;
};

static BwdWs bwd_layout(int B, int T, int H, int dk, int dv, bool vg) {
  const size_t nblk = ((size_t)T + bwd::BLK - 1) / bwd::BLK;
  const size_t heads = (size_t)B * H, nslab = dv / bwd::BV, ntok = (size_t)B * T * H;
  const size_t nsub = bwd::BLK / (vg ? bwd::sub_tokens<true>() : bwd::sub_tokens<false>());
  const size_t nq = vg ? bwd::n_rowvec<true>() : bwd::n_rowvec<false>();
  BwdWs w;
  w.ck = 0;
  w.sub = w.ck + align256(heads * nblk * dk * dv * 4);
  w.part = w.sub + align256(heads * nslab * nsub * (dk / 8) * bwd::NT * 4);
  w.ps = w.part + align256(nq * nslab * ntok * dk * 4);
  w.beta = w.ps + align256(nslab * ntok * 2 * 4);
  w.alpha = w.beta + align256(ntok * 4);
  w.total = w.alpha + align256(ntok * 4);
  return w;
}

size_t recurrent_bwd_workspace_bytes(int B, int T, int H, int dk, int dv, bool vector_gate) {
  if (B < 1 || H < 1 || T < 1) return 0;
  return bwd_layout(B, T, H, dk, dv, vector_gate).total;
}

template <typename T, int DK, int DV, bool VG>
static cudaError_t launch_bwd_t(const void* q, const void* k, const void* v, const float* g,
                                const float* eta, float eps, const float* h0,
                                const void* dout, const float* dhT, float* dq, float* dk,
                                float* dv, float* dg, float* deta, float* dh0, int B, int Tlen,
                                int H, void* ws, cudaStream_t st) {
  const BwdWs w = bwd_layout(B, Tlen, H, DK, DV, VG);
  char* base = (char*)ws;
  float* ck = (float*)(base + w.ck);
  float* sub = (float*)(base + w.sub);
  float* part = (float*)(base + w.part);
  float* ps = (float*)(base + w.ps);
  float* wbeta = (float*)(base + w.beta);
  float* walpha = (float*)(base + w.alpha);
  const int nblk = (Tlen + bwd::BLK - 1) / bwd::BLK;
  const dim3 grid(DV / bwd::BV, H, B);
  constexpr size_t smem_ck = sizeof(bwd::Ops<DK, VG>);
  constexpr size_t smem = bwd::smem_bytes<DK, VG>();
  static_assert(smem <= 227 * 1024, "shared memory");
  static bool attr_set[64] = {};  // the kernels' shared-memory limits, once per device
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  cudaError_t e = cudaSuccess;
  if (!attr_set[dev]) {
    if ((e = cudaFuncSetAttribute(bwd_checkpoint_kernel<T, DK, DV, VG>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_ck)) ||
        (e = cudaFuncSetAttribute(bwd_kernel<T, DK, DV, VG>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)))
      return e;
    attr_set[dev] = true;
  }
  bwd_checkpoint_kernel<T, DK, DV, VG><<<grid, bwd::NT, smem_ck, st>>>(
      (const T*)k, (const T*)v, g, eta, eps, h0, ck, wbeta, walpha, Tlen, H, nblk);
  bwd_kernel<T, DK, DV, VG><<<grid, bwd::NT, smem, st>>>(
      (const T*)q, (const T*)k, (const T*)v, g, (const T*)dout, dhT, wbeta, walpha, ck, sub,
      part, ps, dv, dh0, Tlen, H, nblk);
  const size_t ntok = (size_t)B * Tlen * H;
  const unsigned nb = (unsigned)((ntok + 7) / 8);
  bwd_finish_kernel<T, DK, VG><<<nb, 256, 0, st>>>((const T*)k, eta, walpha, eps, part, ps,
                                                  DV / bwd::BV, ntok, dq, dk, dg, deta);
  return cudaGetLastError();
}

template <bool VG>
static cudaError_t launch_bwd_vg(const void* q, const void* k, const void* v, const float* g,
                                 const float* eta, float eps, const float* h0,
                                 const void* dout, const float* dhT, float* dq, float* dk,
                                 float* dv, float* dg, float* deta, float* dh0, int B, int T,
                                 int H, int dkd, int dvd, int dtype, void* ws,
                                 cudaStream_t st) {
#define KLA_BWD(TY, D)                                                                     \
  launch_bwd_t<TY, D, D, VG>(q, k, v, g, eta, eps, h0, dout, dhT, dq, dk, dv, dg, deta, dh0, \
                             B, T, H, ws, st)
  if (dtype == KLA_BF16) {
    if (dkd == 128 && dvd == 128) return KLA_BWD(__nv_bfloat16, 128);
    if (dkd == 64 && dvd == 64) return KLA_BWD(__nv_bfloat16, 64);
  } else {
    if (dkd == 128 && dvd == 128) return KLA_BWD(float, 128);
    if (dkd == 64 && dvd == 64) return KLA_BWD(float, 64);
  }
#undef KLA_BWD
  return cudaErrorInvalidValue;
}

cudaError_t launch_recurrent_bwd(const void* q, const void* k, const void* v, const float* g,
                                 bool vector_gate, const float* eta, float eps,
                                 const float* h0, const void* dout, const float* dhT,
                                 float* dq, float* dk, float* dv, float* dg, float* deta,
                                 float* dh0, int B, int T, int H, int dkd, int dvd, int dtype,
                                 void* ws, cudaStream_t st) {
  if (vector_gate)
    return launch_bwd_vg<true>(q, k, v, g, eta, eps, h0, dout, dhT, dq, dk, dv, dg, deta, dh0,
                               B, T, H, dkd, dvd, dtype, ws, st);
  return launch_bwd_vg<false>(q, k, v, g, eta, eps, h0, dout, dhT, dq, dk, dv, dg, deta, dh0,
                              B, T, H, dkd, dvd, dtype, ws, st);
}

}  // namespace kla
