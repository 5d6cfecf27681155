// Token-serial backward of the KLA / gated delta rule prefill on CUDA cores
// (fp32 arithmetic): the gradients of a loss L given dL/do and dL/dh_T.
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
//    64-token block, fp32 [B][H][nblk][dk][dv];
//  * bwd_kernel walks the blocks in reverse; per block it reruns the forward
//    from the checkpoint keeping the state at every 8th token (thread-private
//    scratch in global memory, a few MB in all, so it stays in L2), then for
//    each 8-token sub-block in reverse reruns those 8 tokens keeping their
//    states in shared memory and takes the 8 reverse steps.
// Every rerun uses the same step function, so the recomputed states are
// bitwise those of the first forward.
//
// Layout: a CTA of 256 threads owns a 32-column slab of one head's state and
// of its adjoint.  Warp w has columns 4w .. 4w+3; lane 4 rg + c owns column
// 4w + c and rows rg R .. rg R + R - 1 (R = dk / 8).  Sums over rows (r, du,
// ||k||^2) take three shuffles.  Row vectors summed over columns (dq, dk) are
// reduced over the 4 column lanes of a warp by two halving exchanges, over the
// 8 warps in shared memory once per sub-block, and over the dv / 32 slabs by
// bwd_finish_kernel, which also applies the step size's chain rule.
#include "kla_common.cuh"

namespace kla {

namespace bwd {

constexpr int NT = 256;    // threads per CTA
constexpr int BV = 32;     // state columns per CTA
constexpr int BLK = 64;    // tokens per checkpoint
constexpr int SUB = 8;     // tokens per sub-block (states kept in shared memory)
constexpr int NSUB = BLK / SUB;
constexpr unsigned FULL = 0xffffffffu;

// Sum over the 8 row groups of one column (lane bits 2..4).
__device__ __forceinline__ float rows_sum(float x) {
  x += __shfl_xor_sync(FULL, x, 4);
  x += __shfl_xor_sync(FULL, x, 8);
  x += __shfl_xor_sync(FULL, x, 16);
  return x;
}

// Operands of one token as one lane needs them.
template <int R>
struct Tok {
  float k[R], q[R];
  float v, d, g, e;  // v_j, do_j, log-gate, eta (or beta)
};

template <typename T, int DK, int DV, bool WITH_Q>
__device__ __forceinline__ void load_tok(Tok<DK / 8>& x, const T* __restrict__ q,
                                         const T* __restrict__ k, const T* __restrict__ v,
                                         const T* __restrict__ dout, const float* __restrict__ g,
                                         const float* __restrict__ eta, size_t tok, int row0,
                                         int j) {
  constexpr int R = DK / 8;
  const T* kt = k + tok * DK + row0;
#pragma unroll
  for (int m = 0; m < R; m += 4) {
    const float4 a = IO<T>::ld4(kt + m);
    x.k[m] = a.x; x.k[m + 1] = a.y; x.k[m + 2] = a.z; x.k[m + 3] = a.w;
  }
  if constexpr (WITH_Q) {
    const T* qt = q + tok * DK + row0;
#pragma unroll
    for (int m = 0; m < R; m += 4) {
      const float4 a = IO<T>::ld4(qt + m);
      x.q[m] = a.x; x.q[m + 1] = a.y; x.q[m + 2] = a.z; x.q[m + 3] = a.w;
    }
    x.d = IO<T>::ld(dout + tok * DV + j);
  }
  x.v = IO<T>::ld(v + tok * DV + j);
  x.g = g[tok];
  x.e = eta[tok];
}

// One forward token step of the lane's part of the state.
template <int R>
__device__ __forceinline__ void fwd_step(float (&hs)[R], const Tok<R>& x, float eps) {
  float n2 = 0.f, r = 0.f;
#pragma unroll
  for (int m = 0; m < R; ++m) {
    n2 = fmaf(x.k[m], x.k[m], n2);
    r = fmaf(hs[m], x.k[m], r);
  }
  n2 = rows_sum(n2);
  r = rows_sum(r);
  const float beta = step_size(x.e, n2, eps), alpha = expf(x.g);
  const float u = beta * (x.v - alpha * r);
#pragma unroll
  for (int m = 0; m < R; ++m) hs[m] = fmaf(x.k[m], u, alpha * hs[m]);
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
  for (int i = 0; i < H2; ++i) dst[base + i] = z[i];
}

template <int DK>
constexpr size_t smem_bytes() {
  return sizeof(float) * ((size_t)SUB * (DK / 8) * NT + (size_t)SUB * 2 * 8 * DK + SUB * 2 * 8);
}

}  // namespace bwd

// Forward with a checkpoint of h at the start of each 64-token block.
template <typename T, int DK, int DV>
__global__ void __launch_bounds__(bwd::NT)
bwd_checkpoint_kernel(const T* __restrict__ k, const T* __restrict__ v,
                      const float* __restrict__ g, const float* __restrict__ eta, float eps,
                      const float* __restrict__ h0, float* __restrict__ ck, int Tlen, int H,
                      int nblk) {
  using namespace bwd;
  constexpr int R = DK / 8;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int rg = lane >> 2, c = lane & 3;
  const int j = blockIdx.x * BV + warp * 4 + c, row0 = rg * R;
  const int hh = blockIdx.y, b = blockIdx.z;
  const size_t head = (size_t)b * H + hh;

  float hs[R];
#pragma unroll
  for (int m = 0; m < R; ++m) hs[m] = h0 ? h0[(head * DK + row0 + m) * DV + j] : 0.f;

  Tok<R> cur, nxt;
  auto tok_of = [&](int t) { return ((size_t)b * Tlen + t) * H + hh; };
  const int tlast = (nblk - 1) * BLK;  // tokens before the last checkpoint
  if (tlast > 0) load_tok<T, DK, DV, false>(cur, nullptr, k, v, nullptr, g, eta, tok_of(0), row0, j);
  for (int t = 0; t <= tlast; ++t) {
    if (t % BLK == 0) {
      float* dst = ck + ((head * nblk + t / BLK) * DK + row0) * DV + j;
#pragma unroll
      for (int m = 0; m < R; ++m) dst[(size_t)m * DV] = hs[m];
    }
    if (t == tlast) break;
    if (t + 1 < tlast)
      load_tok<T, DK, DV, false>(nxt, nullptr, k, v, nullptr, g, eta, tok_of(t + 1), row0, j);
    fwd_step(hs, cur, eps);
    cur = nxt;
  }
}

template <typename T, int DK, int DV>
__global__ void __launch_bounds__(bwd::NT)
bwd_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
           const float* __restrict__ g, const float* __restrict__ eta, float eps,
           const T* __restrict__ dout, const float* __restrict__ dhT,
           const float* __restrict__ ck, float* __restrict__ sub, float* __restrict__ pq,
           float* __restrict__ pk, float* __restrict__ ps, float* __restrict__ dv_out,
           float* __restrict__ dh0, int Tlen, int H, int nblk) {
  using namespace bwd;
  constexpr int R = DK / 8;
  constexpr int NSLAB = DV / BV;
  extern __shared__ float smem[];
  float* st = smem;                           // [SUB][R][NT] thread-private states
  float* red = st + SUB * R * NT;             // [SUB][2][8 warps][DK]
  float* reds = red + SUB * 2 * 8 * DK;       // [SUB][2][8 warps]

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int rg = lane >> 2, c = lane & 3;
  const int slab = blockIdx.x, hh = blockIdx.y, b = blockIdx.z;
  const int j = slab * BV + warp * 4 + c, row0 = rg * R;
  const size_t head = (size_t)b * H + hh;
  const size_t ntok = (size_t)gridDim.z * Tlen * H;
  float* my_sub = sub + (head * NSLAB + slab) * (size_t)(NSUB * R * NT);
  auto tok_of = [&](int t) { return ((size_t)b * Tlen + t) * H + hh; };

  float dH[R];
#pragma unroll
  for (int m = 0; m < R; ++m) dH[m] = dhT ? dhT[(head * DK + row0 + m) * DV + j] : 0.f;

  Tok<R> cur, nxt;
  for (int blk = nblk - 1; blk >= 0; --blk) {
    const int t0 = blk * BLK, t1 = min(t0 + BLK, Tlen);
    float hs[R];
    {
      const float* src = ck + ((head * nblk + blk) * DK + row0) * DV + j;
#pragma unroll
      for (int m = 0; m < R; ++m) hs[m] = src[(size_t)m * DV];
    }
    // the state at every SUB-th token of the block
    load_tok<T, DK, DV, false>(cur, q, k, v, dout, g, eta, tok_of(t0), row0, j);
    for (int t = t0; t < t1; ++t) {
      if ((t - t0) % SUB == 0) {
        float* dst = my_sub + (size_t)((t - t0) / SUB) * R * NT + tid;
#pragma unroll
        for (int m = 0; m < R; ++m) dst[m * NT] = hs[m];
      }
      if (t + 1 == t1) break;
      load_tok<T, DK, DV, false>(nxt, q, k, v, dout, g, eta, tok_of(t + 1), row0, j);
      fwd_step(hs, cur, eps);
      cur = nxt;
    }
    const int nsb = (t1 - t0 + SUB - 1) / SUB;
    for (int sb = nsb - 1; sb >= 0; --sb) {
      const int s0 = t0 + sb * SUB, s1 = min(s0 + SUB, t1);
      {
        const float* src = my_sub + (size_t)sb * R * NT + tid;
#pragma unroll
        for (int m = 0; m < R; ++m) hs[m] = src[m * NT];
      }
      // states before each token of the sub-block
      load_tok<T, DK, DV, false>(cur, q, k, v, dout, g, eta, tok_of(s0), row0, j);
      for (int t = s0; t < s1; ++t) {
        float* dst = st + (size_t)(t - s0) * R * NT + tid;
#pragma unroll
        for (int m = 0; m < R; ++m) dst[m * NT] = hs[m];
        if (t + 1 == s1) break;
        load_tok<T, DK, DV, false>(nxt, q, k, v, dout, g, eta, tok_of(t + 1), row0, j);
        fwd_step(hs, cur, eps);
        cur = nxt;
      }
      // reverse steps
      load_tok<T, DK, DV, true>(cur, q, k, v, dout, g, eta, tok_of(s1 - 1), row0, j);
      for (int t = s1 - 1; t >= s0; --t) {
        const int s = t - s0;
        if (t > s0) load_tok<T, DK, DV, true>(nxt, q, k, v, dout, g, eta, tok_of(t - 1), row0, j);
        float hp[R];
        {
          const float* src = st + (size_t)s * R * NT + tid;
#pragma unroll
          for (int m = 0; m < R; ++m) hp[m] = src[m * NT];
        }
        float n2 = 0.f, r = 0.f;
#pragma unroll
        for (int m = 0; m < R; ++m) {
          n2 = fmaf(cur.k[m], cur.k[m], n2);
          r = fmaf(hp[m], cur.k[m], r);
        }
        n2 = rows_sum(n2);
        r = rows_sum(r);
        const float beta = step_size(cur.e, n2, eps), alpha = expf(cur.g);
        const float u = beta * (cur.v - alpha * r);
        float xq[R], xk[R];
        float du = 0.f;
#pragma unroll
        for (int m = 0; m < R; ++m) {
          xq[m] = fmaf(cur.k[m], u, alpha * hp[m]) * cur.d;  // h_t[i][j] do_j
          dH[m] = fmaf(cur.q[m], cur.d, dH[m]);
          du = fmaf(dH[m], cur.k[m], du);
        }
        du = rows_sum(du);
        const float dr = -alpha * beta * du;
        float da = 0.f, db = 0.f;
#pragma unroll
        for (int m = 0; m < R; ++m) {
          xk[m] = fmaf(dH[m], u, hp[m] * dr);
          da = fmaf(dH[m], hp[m], da);
          dH[m] = fmaf(cur.k[m], dr, alpha * dH[m]);
        }
        if (rg == 0) {  // per-column terms, once per column
          da -= beta * du * r;
          db = du * (cur.v - alpha * r);
          dv_out[tok_of(t) * DV + j] = beta * du;
        }
        cols_sum_store(xq, red + ((size_t)(s * 2 + 0) * 8 + warp) * DK + row0, c);
        cols_sum_store(xk, red + ((size_t)(s * 2 + 1) * 8 + warp) * DK + row0, c);
        da = warp_sum(da);
        db = warp_sum(db);
        if (lane == 0) {
          reds[(s * 2 + 0) * 8 + warp] = da;
          reds[(s * 2 + 1) * 8 + warp] = db;
        }
        cur = nxt;
      }
      __syncthreads();
      // sums over the 8 warps -> this slab's partials
      const int n = s1 - s0;
      for (int p = tid; p < n * 2 * DK; p += NT) {
        const int s = p / (2 * DK), qi = (p / DK) & 1, i = p % DK;
        const float* src = red + ((size_t)(s * 2 + qi) * 8) * DK + i;
        float a = 0.f;
#pragma unroll
        for (int w = 0; w < 8; ++w) a += src[w * DK];
        float* dst = qi == 0 ? pq : pk;
        dst[((size_t)slab * ntok + tok_of(s0 + s)) * DK + i] = a;
      }
      if (tid < n * 2) {
        const int s = tid >> 1, qi = tid & 1;
        float a = 0.f;
#pragma unroll
        for (int w = 0; w < 8; ++w) a += reds[(s * 2 + qi) * 8 + w];
        ps[((size_t)slab * ntok + tok_of(s0 + s)) * 2 + qi] = a;
      }
      __syncthreads();
    }
  }
  if (dh0) {
#pragma unroll
    for (int m = 0; m < R; ++m) dh0[(head * DK + row0 + m) * DV + j] = dH[m];
  }
}

// Per token (one warp): dq, dk summed over the slabs; dg = alpha dalpha; the
// step size's chain rule into deta and dk (KLA), or dbeta as is (eps < 0).
template <typename T, int DK>
__global__ void __launch_bounds__(256)
bwd_finish_kernel(const T* __restrict__ k, const float* __restrict__ g,
                  const float* __restrict__ eta, float eps, const float* __restrict__ pq,
                  const float* __restrict__ pk, const float* __restrict__ ps, int nslab,
                  size_t ntok, float* __restrict__ dq, float* __restrict__ dk,
                  float* __restrict__ dg, float* __restrict__ deta) {
  constexpr int E = DK / 32;  // elements per lane
  const int lane = threadIdx.x & 31;
  const size_t tok = (size_t)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
  if (tok >= ntok) return;
  float kk[E], sq[E], sk[E];
  float n2 = 0.f;
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const int i = lane * E + e;
    kk[e] = IO<T>::ld(k + tok * DK + i);
    n2 = fmaf(kk[e], kk[e], n2);
    sq[e] = 0.f;
    sk[e] = 0.f;
  }
  n2 = warp_sum(n2);
  float sa = 0.f, sb = 0.f;
  for (int sl = 0; sl < nslab; ++sl) {
    const size_t base = (size_t)sl * ntok + tok;
#pragma unroll
    for (int e = 0; e < E; ++e) {
      sq[e] += pq[base * DK + lane * E + e];
      sk[e] += pk[base * DK + lane * E + e];
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
  if (lane == 0) dg[tok] = expf(g[tok]) * sa;
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const int i = lane * E + e;
    dq[tok * DK + i] = sq[e];
    dk[tok * DK + i] = fmaf(coef, kk[e], sk[e]);
  }
}

// ---- workspace and launch

static size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

struct BwdWs {
  size_t ck, sub, pq, pk, ps, total;
};

static BwdWs bwd_layout(int B, int T, int H, int dk, int dv) {
  const size_t nblk = ((size_t)T + bwd::BLK - 1) / bwd::BLK;
  const size_t heads = (size_t)B * H, nslab = dv / bwd::BV, ntok = (size_t)B * T * H;
  BwdWs w;
  w.ck = 0;
  w.sub = w.ck + align256(heads * nblk * dk * dv * 4);
  w.pq = w.sub + align256(heads * nslab * (size_t)bwd::NSUB * (dk / 8) * bwd::NT * 4);
  w.pk = w.pq + align256(nslab * ntok * dk * 4);
  w.ps = w.pk + align256(nslab * ntok * dk * 4);
  w.total = w.ps + align256(nslab * ntok * 2 * 4);
  return w;
}

size_t recurrent_bwd_workspace_bytes(int B, int T, int H, int dk, int dv) {
  if (B < 1 || H < 1 || T < 1) return 0;
  return bwd_layout(B, T, H, dk, dv).total;
}

template <typename T, int DK, int DV>
static cudaError_t launch_bwd_t(const void* q, const void* k, const void* v, const float* g,
                                const float* eta, float eps, const float* h0,
                                const void* dout, const float* dhT, float* dq, float* dk,
                                float* dv, float* dg, float* deta, float* dh0, int B, int Tlen,
                                int H, void* ws, cudaStream_t st) {
  const BwdWs w = bwd_layout(B, Tlen, H, DK, DV);
  char* base = (char*)ws;
  float* ck = (float*)(base + w.ck);
  float* sub = (float*)(base + w.sub);
  float* pq = (float*)(base + w.pq);
  float* pk = (float*)(base + w.pk);
  float* ps = (float*)(base + w.ps);
  const int nblk = (Tlen + bwd::BLK - 1) / bwd::BLK;
  const dim3 grid(DV / bwd::BV, H, B);
  bwd_checkpoint_kernel<T, DK, DV><<<grid, bwd::NT, 0, st>>>(
      (const T*)k, (const T*)v, g, eta, eps, h0, ck, Tlen, H, nblk);
  constexpr size_t smem = bwd::smem_bytes<DK>();
  cudaError_t e = cudaFuncSetAttribute(bwd_kernel<T, DK, DV>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  bwd_kernel<T, DK, DV><<<grid, bwd::NT, smem, st>>>(
      (const T*)q, (const T*)k, (const T*)v, g, eta, eps, (const T*)dout, dhT, ck, sub, pq, pk,
      ps, dv, dh0, Tlen, H, nblk);
  const size_t ntok = (size_t)B * Tlen * H;
  const unsigned nb = (unsigned)((ntok + 7) / 8);
  bwd_finish_kernel<T, DK><<<nb, 256, 0, st>>>((const T*)k, g, eta, eps, pq, pk, ps,
                                              DV / bwd::BV, ntok, dq, dk, dg, deta);
  return cudaGetLastError();
}

cudaError_t launch_recurrent_bwd(const void* q, const void* k, const void* v, const float* g,
                                 const float* eta, float eps, const float* h0,
                                 const void* dout, const float* dhT, float* dq, float* dk,
                                 float* dv, float* dg, float* deta, float* dh0, int B, int T,
                                 int H, int dkd, int dvd, int dtype, void* ws,
                                 cudaStream_t st) {
#define KLA_BWD(TY, D) \
  launch_bwd_t<TY, D, D>(q, k, v, g, eta, eps, h0, dout, dhT, dq, dk, dv, dg, deta, dh0, B, T, H, ws, st)
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

}  // namespace kla
