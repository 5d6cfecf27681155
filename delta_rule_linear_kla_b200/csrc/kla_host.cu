// kla_chunk_fwd_host: the prefill from host buffers, with the host<->device
// copies pipelined against the kernels.
//
// The batch is cut into pieces of whole sequences (contiguous slices of every
// [B, ...] tensor).  Each piece goes through a staging slot in caller-owned
// device memory: its inputs are copied in on one internal stream, the prefill
// (kla_chunk_fwd on the slot) runs on the caller's stream, and its outputs are
// copied out on a second internal stream.  With three slots the copy-in of
// piece i+1, the kernels of piece i and the copy-out of piece i-1 run at the
// same time, so a step costs about the larger of the two copy directions
// instead of their sum plus the kernels.  Events join everything back into
// the caller's stream: when that stream reaches the end of the call, every
// output is in host memory.
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "../../include/kla.h"

namespace {

constexpr int kMaxSlots = 3;
constexpr int kMaxPieces = 8;
constexpr int kMaxDevices = 64;
constexpr size_t kAlign = 256;

size_t up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

// Per-device copy streams and events, created on first use and kept for the
// life of the process.  Enqueueing a call holds the device's mutex, so two
// host threads never interleave their records and waits on these events.
struct DeviceResources {
  bool ready = false;
  cudaStream_t h2d = nullptr, d2h = nullptr;
  cudaEvent_t start = nullptr, done = nullptr;
  cudaEvent_t in[kMaxSlots] = {}, out[kMaxSlots] = {}, free_[kMaxSlots] = {};
  std::mutex mu;
};
DeviceResources g_res[kMaxDevices];

bool init_resources(DeviceResources& r) {
  if (r.ready) return true;
  const unsigned ef = cudaEventDisableTiming;
  if (cudaStreamCreateWithFlags(&r.h2d, cudaStreamNonBlocking) != cudaSuccess) return false;
  if (cudaStreamCreateWithFlags(&r.d2h, cudaStreamNonBlocking) != cudaSuccess) return false;
  if (cudaEventCreateWithFlags(&r.start, ef) != cudaSuccess) return false;
  if (cudaEventCreateWithFlags(&r.done, ef) != cudaSuccess) return false;
  for (int s = 0; s < kMaxSlots; ++s) {
    if (cudaEventCreateWithFlags(&r.in[s], ef) != cudaSuccess) return false;
    if (cudaEventCreateWithFlags(&r.out[s], ef) != cudaSuccess) return false;
    if (cudaEventCreateWithFlags(&r.free_[s], ef) != cudaSuccess) return false;
  }
  r.ready = true;
  return true;
}

// How the batch is cut: `bp` sequences per piece, `npieces` pieces, `nslots`
// staging slots.  Every piece costs a fixed overhead (its kernels run on a
// smaller batch, its copies start and end on their own), so pieces carry at
// least ~64 MiB of inputs: measured on the 4K-token layer (203 MB of inputs,
// B = 8), 3 pieces take 4.40 ms, 4 pieces 4.51, 2 pieces 4.64, 8 pieces 4.83.
constexpr double kPieceBytes = 64.0 * 1024 * 1024;
struct Plan {
  int bp, npieces, nslots;
};
Plan plan(int B, int T, int H, int dk, int dv, int dtype) {
  const double es = dtype == KLA_BF16 ? 2.0 : 4.0;
  const double in_bytes = (double)B * T * H * ((2.0 * dk + dv) * es + 8.0);
  int np = (int)(in_bytes / kPieceBytes + 0.5);
  np = np < 1 ? 1 : (np > kMaxPieces ? kMaxPieces : np);
  np = np > B ? B : np;
  const int bp = (B + np - 1) / np;
  const int npieces = (B + bp - 1) / bp;
  return Plan{bp, npieces, npieces < kMaxSlots ? npieces : kMaxSlots};
}

// Byte offsets of one slot's buffers (a piece of nb <= bp sequences).
struct Slot {
  size_t q, k, v, g, eta, h0, o, hT, ws, ws_bytes, total;
};
Slot slot_layout(int bp, int T, int H, int dk, int dv, int dtype) {
  const size_t es = dtype == KLA_BF16 ? 2 : 4;
  const size_t ntok = (size_t)bp * T * H, st = (size_t)bp * H * dk * dv * 4;
  Slot s;
  size_t at = 0;
  s.q = at; at += up(ntok * dk * es);
  s.k = at; at += up(ntok * dk * es);
  s.v = at; at += up(ntok * dv * es);
  s.g = at; at += up(ntok * 4);
  s.eta = at; at += up(ntok * 4);
  s.h0 = at; at += up(st);
  s.o = at; at += up(ntok * dv * es);
  s.hT = at; at += up(st);
  s.ws_bytes = kla_chunk_fwd_workspace_size(bp, T, H, dk, dv, dtype);
  s.ws = at; at += up(s.ws_bytes);
  s.total = at;
  return s;
}

bool shape_ok(int B, int T, int H, int dk, int dv, int dtype) {
  if (B < 1 || H < 1 || T < 1) return false;
  if (dtype != KLA_BF16 && dtype != KLA_FP32) return false;
  return (long long)B * T * H * (dk > dv ? dk : dv) < (1LL << 40);
}

}  // namespace

extern "C" {

size_t kla_chunk_fwd_host_staging_size(int B, int T, int H, int dk, int dv, int dtype) {
  if (!shape_ok(B, T, H, dk, dv, dtype)) return 0;
  const Plan p = plan(B, T, H, dk, dv, dtype);
  return (size_t)p.nslots * slot_layout(p.bp, T, H, dk, dv, dtype).total;
}

kla_status kla_chunk_fwd_host(const void* q, const void* k, const void* v, const float* g,
                              const float* eta, float eps, const float* h0, void* o, float* hT,
                              int B, int T, int H, int dk, int dv, int dtype, void* staging,
                              size_t staging_bytes, void* stream) {
  if (!shape_ok(B, T, H, dk, dv, dtype)) return KLA_ERR_INVALID_ARG;
  if (!q || !k || !v || !g || !eta || !o || !staging) return KLA_ERR_INVALID_ARG;
  if (!(eps >= 0.0f)) return KLA_ERR_INVALID_ARG;
  if (((uintptr_t)staging & (kAlign - 1)) != 0) return KLA_ERR_INVALID_ARG;
  if (!((dk == 64 && dv == 64) || (dk == 128 && dv == 128))) return KLA_ERR_UNSUPPORTED;
  const Plan p = plan(B, T, H, dk, dv, dtype);
  const Slot L = slot_layout(p.bp, T, H, dk, dv, dtype);
  if (staging_bytes < (size_t)p.nslots * L.total) return KLA_ERR_INVALID_ARG;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return KLA_ERR_CUDA;
  DeviceResources& R = g_res[dev];
  std::lock_guard<std::mutex> lock(R.mu);
  if (!init_resources(R)) return KLA_ERR_CUDA;

  cudaStream_t st = (cudaStream_t)stream;
  const size_t es = dtype == KLA_BF16 ? 2 : 4;
  const size_t tok_per_seq = (size_t)T * H, state_per_seq = (size_t)H * dk * dv * 4;
  uint8_t* base = (uint8_t*)staging;
  auto ok = [](cudaError_t e) { return e == cudaSuccess; };
  const cudaMemcpyKind H2D = cudaMemcpyHostToDevice, D2H = cudaMemcpyDeviceToHost;

  // nothing of this call starts before the caller's earlier work on `st`
  if (!ok(cudaEventRecord(R.start, st))) return KLA_ERR_CUDA;
  for (int i = 0; i < p.npieces; ++i) {
    const int s = i % p.nslots;
    const int b0 = i * p.bp, nb = (B - b0) < p.bp ? (B - b0) : p.bp;
    uint8_t* sb = base + (size_t)s * L.total;
    const size_t t0 = (size_t)b0 * tok_per_seq, nt = (size_t)nb * tok_per_seq;
    const size_t s0 = (size_t)b0 * state_per_seq, ns = (size_t)nb * state_per_seq;
    // copy-in, once the slot's previous piece has been copied out
    if (!ok(cudaStreamWaitEvent(R.h2d, i < p.nslots ? R.start : R.free_[s], 0)))
      return KLA_ERR_CUDA;
    struct {
      size_t dst;
      const void* src;
      size_t off, bytes;
    } in[] = {{L.q, q, t0 * dk * es, nt * dk * es},
              {L.k, k, t0 * dk * es, nt * dk * es},
              {L.v, v, t0 * dv * es, nt * dv * es},
              {L.g, g, t0 * 4, nt * 4},
              {L.eta, eta, t0 * 4, nt * 4},
              {L.h0, h0, s0, h0 ? ns : 0}};
    for (auto& c : in)
      if (c.bytes && !ok(cudaMemcpyAsync(sb + c.dst, (const uint8_t*)c.src + c.off, c.bytes, H2D,
                                          R.h2d)))
        return KLA_ERR_CUDA;
    if (!ok(cudaEventRecord(R.in[s], R.h2d))) return KLA_ERR_CUDA;
    // the kernels, on the caller's stream
    if (!ok(cudaStreamWaitEvent(st, R.in[s], 0))) return KLA_ERR_CUDA;
    // a short last piece may want a different (cut-chain) workspace; the
    // slot's always holds its UT factors, and kla_chunk_fwd runs uncut when
    // the segment states do not fit
    size_t wsb = kla_chunk_fwd_workspace_size(nb, T, H, dk, dv, dtype);
    if (wsb > L.ws_bytes) wsb = L.ws_bytes;
    kla_status ks = kla_chunk_fwd(sb + L.q, sb + L.k, sb + L.v, (const float*)(sb + L.g),
                                  (const float*)(sb + L.eta), eps,
                                  h0 ? (const float*)(sb + L.h0) : nullptr, sb + L.o,
                                  hT ? (float*)(sb + L.hT) : nullptr, nb, T, H, dk, dv,
                                  KLA_CHUNK, dtype, wsb ? sb + L.ws : nullptr, wsb, st);
    if (ks != KLA_OK) return ks;
    if (!ok(cudaEventRecord(R.out[s], st))) return KLA_ERR_CUDA;
    // copy-out
    if (!ok(cudaStreamWaitEvent(R.d2h, R.out[s], 0))) return KLA_ERR_CUDA;
    if (!ok(cudaMemcpyAsync((uint8_t*)o + t0 * dv * es, sb + L.o, nt * dv * es, D2H, R.d2h)))
      return KLA_ERR_CUDA;
    if (hT && !ok(cudaMemcpyAsync((uint8_t*)hT + s0, sb + L.hT, ns, D2H, R.d2h)))
      return KLA_ERR_CUDA;
    if (!ok(cudaEventRecord(R.free_[s], R.d2h))) return KLA_ERR_CUDA;
  }
  // the caller's stream passes the end of the call only after the last copy
  if (!ok(cudaEventRecord(R.done, R.d2h))) return KLA_ERR_CUDA;
  if (!ok(cudaStreamWaitEvent(st, R.done, 0))) return KLA_ERR_CUDA;
  return KLA_OK;
}

}  // extern "C"
