// Single-token decode step of Kaczmarz Linear Attention, in place on the state.
//
// Per head (h = S^T, [DK][DV] fp32) and new token (q, k, v, g, eta):
//   beta = eta / (||k||^2 + eps)      ("Kaczmarz Linear Attention", Abstract)
//   alpha = exp(g)
//   r = h^T k,  s = h^T q             (one read of the state)
//   u = beta (v - alpha r)
//   h <- alpha h + k u^T              (one write of the state)
//   o = h_new^T q = alpha s + u (k . q)
// which is one step of the gated delta rule ("Deep Dive into KDA",
// section 2.2) with o read from the updated state.  With a per-channel gate
// (KDA form, same page, section 2.3) the rows of h are scaled by
// a_i = exp(g_i) as they are loaded and the step above runs on the decayed
// state with alpha = 1.
//
// The state is the only large operand (DK*DV*4 bytes per head, read once and
// written once); the kernel is an HBM stream.  Persistent CTAs, one per SM,
// walk the heads: a head's whole state (contiguous, 64 KB at d = 128) comes
// in with one bulk copy into a ring of NST shared-memory stages, issued NST-1
// heads ahead, so HBM keeps streaming while the head in hand is reduced and
// updated; the updated state goes back to its stage and out with one bulk
// store.  Each thread keeps its rows x 4 columns in registers between the
// reduction and the update, so shared memory is read once and written once
// per head.  Every wait is bounded (an error bit instead of a hang).
#include "kla_common.cuh"
#include "kla_sync.cuh"
#include "ptx_sm100.cuh"

namespace kla {
namespace {

constexpr int DEC_NT = 512;  // threads per CTA
constexpr int DEC_NST = 3;   // shared-memory stages (heads in flight)

template <int DK, int DV>
struct alignas(128) DecSmem {
  float st[DEC_NST][DK * DV];                   // head states, row-major
  float red[2][DEC_NT / (DV / 4)][DV];          // column partial sums: r, s
  float u[DV];
  float kq[2];                                  // ||k||^2, k . q
  uint64_t full[DEC_NST];
};

// Bulk store shared -> global (one per head), tracked in this thread's bulk
// async-group.
__device__ __forceinline__ void bulk_store(void* dst, const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(
                   reinterpret_cast<uint64_t>(dst)),
               "r"(ptx::smem_u32(src)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// Waits until at most N of this thread's committed bulk groups are still
// reading their shared-memory source.
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void bulk_wait_all() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

// VG: g is per key channel ([B][H][DK]) instead of per head.
template <typename T, int DK, int DV, bool VG>
__global__ void __launch_bounds__(DEC_NT, 1)
decode_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
              const float* __restrict__ g, const float* __restrict__ eta, float eps,
              float* __restrict__ S, T* __restrict__ o, int nheads, unsigned int* err) {
  using Smem = DecSmem<DK, DV>;
  constexpr int LPR = DV / 4;           // threads per state row (one float4 each)
  constexpr int RPP = DEC_NT / LPR;     // rows per pass
  constexpr int RT = DK / RPP;          // rows held per thread
  static_assert(DEC_NT % LPR == 0 && DK % RPP == 0, "tile");
  constexpr uint32_t HEAD_BYTES = DK * DV * 4;
  extern __shared__ uint8_t smem_raw[];
  Smem& s = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) &
                                     ~uintptr_t(127));
  const int tid = threadIdx.x;
  const int c4 = tid % LPR, row0 = tid / LPR;

  if (tid == 0) {
    for (int i = 0; i < DEC_NST; ++i) ptx::mbar_init(&s.full[i], 1);
    ptx::mbar_init_fence();
  }
  __syncthreads();
  // the first NST - 1 heads of this CTA
  if (tid == 0) {
    for (int i = 0; i < DEC_NST - 1; ++i) {
      const int hd = blockIdx.x + i * gridDim.x;
      if (hd < nheads) {
        ptx::mbar_arrive_expect_tx(&s.full[i], HEAD_BYTES);
        ptx::bulk_load(s.st[i], S + (size_t)hd * DK * DV, HEAD_BYTES, &s.full[i]);
      }
    }
  }
  bool ok = true;
  int it = 0;
#pragma unroll 1
  for (int hd = blockIdx.x; hd < nheads; hd += gridDim.x, ++it) {
    const int stg = it % DEC_NST;
    // one head ahead of the loads already issued: its stage last held the
    // head stored NST - 1 iterations ago, whose store must have read it
    if (tid == 0) {
      const int nxt = hd + (DEC_NST - 1) * gridDim.x;
      if (nxt < nheads) {
        const int ns = (it + DEC_NST - 1) % DEC_NST;
        bulk_wait_read<0>();
        ptx::mbar_arrive_expect_tx(&s.full[ns], HEAD_BYTES);
        ptx::bulk_load(s.st[ns], S + (size_t)nxt * DK * DV, HEAD_BYTES, &s.full[ns]);
      }
    }
    const T* kp = k + (size_t)hd * DK;
    const T* qp = q + (size_t)hd * DK;
    float kr[RT], qr[RT];
#pragma unroll
    for (int m = 0; m < RT; ++m) {
      kr[m] = IO<T>::ld(kp + row0 + m * RPP);
      qr[m] = IO<T>::ld(qp + row0 + m * RPP);
    }
    float gr[RT];
    if constexpr (VG) {
#pragma unroll
      for (int m = 0; m < RT; ++m) gr[m] = expf(g[(size_t)hd * DK + row0 + m * RPP]);
    }
    // ||k||^2 and k.q over the full key dimension (warp 0)
    if (tid < 32) {
      float n2 = 0.f, kq = 0.f;
      for (int i = tid; i < DK; i += 32) {
        const float a = IO<T>::ld(kp + i), b = IO<T>::ld(qp + i);
        n2 = fmaf(a, a, n2);
        kq = fmaf(a, b, kq);
      }
      n2 = warp_sum(n2);
      kq = warp_sum(kq);
      if (tid == 0) {
        s.kq[0] = n2;
        s.kq[1] = kq;
      }
    }
    // a wait that gives up ends this CTA's walk (no update or store of a
    // state that did not arrive)
    ok = wait_bounded(&s.full[stg], (uint32_t)((it / DEC_NST) & 1));
    if (!__syncthreads_and(ok)) break;
    float* st = s.st[stg];
    float4 hv[RT];
#pragma unroll
    for (int m = 0; m < RT; ++m) {
      hv[m] = *reinterpret_cast<const float4*>(st + (row0 + m * RPP) * DV + 4 * c4);
      if constexpr (VG) {
        hv[m].x *= gr[m]; hv[m].y *= gr[m]; hv[m].z *= gr[m]; hv[m].w *= gr[m];
      }
    }
    float4 pr = make_float4(0.f, 0.f, 0.f, 0.f), ps = pr;
#pragma unroll
    for (int m = 0; m < RT; ++m) {
      pr.x = fmaf(hv[m].x, kr[m], pr.x); pr.y = fmaf(hv[m].y, kr[m], pr.y);
      pr.z = fmaf(hv[m].z, kr[m], pr.z); pr.w = fmaf(hv[m].w, kr[m], pr.w);
      ps.x = fmaf(hv[m].x, qr[m], ps.x); ps.y = fmaf(hv[m].y, qr[m], ps.y);
      ps.z = fmaf(hv[m].z, qr[m], ps.z); ps.w = fmaf(hv[m].w, qr[m], ps.w);
    }
    *reinterpret_cast<float4*>(&s.red[0][row0][4 * c4]) = pr;
    *reinterpret_cast<float4*>(&s.red[1][row0][4 * c4]) = ps;
    __syncthreads();
    const float alpha = VG ? 1.f : expf(g[hd]);
    if (tid < DV) {
      const float beta = step_size(eta[hd], s.kq[0], eps);
      float r = 0.f, sq = 0.f;
#pragma unroll
      for (int p = 0; p < RPP; ++p) {
        r += s.red[0][p][tid];
        sq += s.red[1][p][tid];
      }
      const float u = beta * (IO<T>::ld(v + (size_t)hd * DV + tid) - alpha * r);
      s.u[tid] = u;
      IO<T>::st(o + (size_t)hd * DV + tid, fmaf(u, s.kq[1], alpha * sq));
    }
    __syncthreads();
    const float4 u4 = *reinterpret_cast<const float4*>(&s.u[4 * c4]);
#pragma unroll
    for (int m = 0; m < RT; ++m) {
      float4 x = hv[m];
      const float kk = kr[m];
      x.x = fmaf(kk, u4.x, alpha * x.x); x.y = fmaf(kk, u4.y, alpha * x.y);
      x.z = fmaf(kk, u4.z, alpha * x.z); x.w = fmaf(kk, u4.w, alpha * x.w);
      *reinterpret_cast<float4*>(st + (row0 + m * RPP) * DV + 4 * c4) = x;
    }
    ptx::fence_proxy_async_smem();  // the updated state is visible to the bulk store
    __syncthreads();                 // ... from every thread; red and u are free again
    if (tid == 0) {
      bulk_store(S + (size_t)hd * DK * DV, st, HEAD_BYTES);
      bulk_commit();
    }
  }
  if (tid == 0) {
    bulk_wait_all();  // every store has landed before the CTA ends
    if (!ok) report_timeout(err);
  }
}

template <typename T, int DK, int DV>
cudaError_t launch_decode_t(const void* q, const void* k, const void* v, const float* g,
                            bool vector_gate, const float* eta, float eps, float* S, void* o,
                            int B, int H, unsigned int* err, cudaStream_t st) {
  const int nheads = B * H;
  if (nheads == 0) return cudaSuccess;
  constexpr size_t smem = sizeof(DecSmem<DK, DV>) + 128;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  static int sms[64] = {};
  static bool attr_set[2][64] = {};
  if (!sms[dev]) {
    cudaError_t e = cudaDeviceGetAttribute(&sms[dev], cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
  }
  const int vg = vector_gate ? 1 : 0;
  if (!attr_set[vg][dev]) {
    cudaError_t e = vector_gate
                        ? cudaFuncSetAttribute(decode_kernel<T, DK, DV, true>,
                                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               (int)smem)
                        : cudaFuncSetAttribute(decode_kernel<T, DK, DV, false>,
                                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               (int)smem);
    if (e != cudaSuccess) return e;
    attr_set[vg][dev] = true;
  }
  const int grid = nheads < sms[dev] ? nheads : sms[dev];
  if (vector_gate)
    decode_kernel<T, DK, DV, true><<<grid, DEC_NT, smem, st>>>(
        (const T*)q, (const T*)k, (const T*)v, g, eta, eps, S, (T*)o, nheads, err);
  else
    decode_kernel<T, DK, DV, false><<<grid, DEC_NT, smem, st>>>(
        (const T*)q, (const T*)k, (const T*)v, g, eta, eps, S, (T*)o, nheads, err);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode(const void* q, const void* k, const void* v,
                          const float* g, bool vector_gate, const float* eta, float eps,
                          float* S, void* o, int B, int H, int dk, int dv, int dtype,
                          unsigned int* err, cudaStream_t st) {
  const bool vg = vector_gate;
  if (dtype == KLA_BF16) {
    if (dk == 128 && dv == 128)
      return launch_decode_t<__nv_bfloat16, 128, 128>(q, k, v, g, vg, eta, eps, S, o, B, H,
                                                      err, st);
    if (dk == 64 && dv == 64)
      return launch_decode_t<__nv_bfloat16, 64, 64>(q, k, v, g, vg, eta, eps, S, o, B, H, err,
                                                    st);
  } else {
    if (dk == 128 && dv == 128)
      return launch_decode_t<float, 128, 128>(q, k, v, g, vg, eta, eps, S, o, B, H, err, st);
    if (dk == 64 && dv == 64)
      return launch_decode_t<float, 64, 64>(q, k, v, g, vg, eta, eps, S, o, B, H, err, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace kla
