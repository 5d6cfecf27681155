// 128-byte-swizzled shared-memory tiles (the layout TMA writes with
// CU_TENSOR_MAP_SWIZZLE_128B and tcgen05 reads with layout type SWIZZLE_128B).
//
// A "panel" is 64 bf16 columns wide: every row is 128 bytes; the 16-byte
// chunk c of row r sits at chunk position c ^ (r & 7).  Panels start on
// 1024-byte boundaries so the swizzle phase equals the row index mod 8.
// Wider tiles are several panels placed one after another.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

namespace kla {

__device__ __forceinline__ uint32_t sw128_chunk_off(int row, int chunk) {
  return (uint32_t)(row * 128 + (((chunk ^ (row & 7)) & 7) << 4));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

// Writes 64 floats as one bf16 row (128 B) of a swizzled panel.
__device__ __forceinline__ void sw128_store_row(uint8_t* panel, int row, const float* x) {
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    uint4 u;
    u.x = pack_bf16x2(x[8 * c + 0], x[8 * c + 1]);
    u.y = pack_bf16x2(x[8 * c + 2], x[8 * c + 3]);
    u.z = pack_bf16x2(x[8 * c + 4], x[8 * c + 5]);
    u.w = pack_bf16x2(x[8 * c + 6], x[8 * c + 7]);
    *reinterpret_cast<uint4*>(panel + sw128_chunk_off(row, c)) = u;
  }
}

// Writes 32 floats (columns [32*half32, 32*half32 + 32)) of a bf16 row.
__device__ __forceinline__ void sw128_store_row32(uint8_t* panel, int row, int half32,
                                                  const float* x) {
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    uint4 u;
    u.x = pack_bf16x2(x[8 * c + 0], x[8 * c + 1]);
    u.y = pack_bf16x2(x[8 * c + 2], x[8 * c + 3]);
    u.z = pack_bf16x2(x[8 * c + 4], x[8 * c + 5]);
    u.w = pack_bf16x2(x[8 * c + 6], x[8 * c + 7]);
    *reinterpret_cast<uint4*>(panel + sw128_chunk_off(row, 4 * half32 + c)) = u;
  }
}

__device__ __forceinline__ void unpack_bf16x8(uint4 u, float* x) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    __nv_bfloat162 h = *reinterpret_cast<const __nv_bfloat162*>(&w[i]);
    float2 f = __bfloat1622float2(h);
    x[2 * i] = f.x;
    x[2 * i + 1] = f.y;
  }
}

// Reads one bf16 row (64 values) of a swizzled panel as floats.
__device__ __forceinline__ void sw128_load_row(const uint8_t* panel, int row, float* x) {
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    uint4 u = *reinterpret_cast<const uint4*>(panel + sw128_chunk_off(row, c));
    unpack_bf16x8(u, x + 8 * c);
  }
}

}  // namespace kla
