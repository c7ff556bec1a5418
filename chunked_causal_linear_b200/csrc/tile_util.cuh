// Small helpers shared by the warp-specialised tcgen05 kernels: 1024-byte alignment of the
// dynamic shared memory, bf16 packing, the hi / lo split of float32 values into two bf16
// operands, and shared-memory descriptors advanced by a byte offset.
#pragma once

#include <cuda_bf16.h>

#include <cstdint>

#include "ptx.cuh"

namespace la {

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  const uint32_t a = smem_u32(p);
  return p + ((1024u - (a & 1023u)) & 1023u);
}

__device__ __forceinline__ void unpack8(uint4 raw, float (&x)[8]) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float2 f = __bfloat1622float2(h[e]);
    x[2 * e] = f.x;
    x[2 * e + 1] = f.y;
  }
}

__device__ __forceinline__ uint4 pack8(const float (&x)[8]) {
  uint4 raw;
  __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&raw);
#pragma unroll
  for (int e = 0; e < 4; ++e) h[e] = __floats2bfloat162_rn(x[2 * e], x[2 * e + 1]);
  return raw;
}

// x = hi + lo with hi = bf16(x) and lo = bf16(x - hi): about 16 significant bits in two
// bf16 operands.
__device__ __forceinline__ void split8(const float (&x)[8], uint4& hi, uint4& lo) {
  hi = pack8(x);
  float h[8], r[8];
  unpack8(hi, h);
#pragma unroll
  for (int e = 0; e < 8; ++e) r[e] = x[e] - h[e];
  lo = pack8(r);
}

__device__ __forceinline__ uint32_t pack2(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

// A shared-memory descriptor advanced by a byte offset: the start address field holds
// address >> 4 in its low 14 bits and every operand of these kernels lies below 256 KB, so
// the addition never carries out of the field.
__device__ __forceinline__ uint64_t desc_at(uint64_t d, uint32_t bytes) { return d + (bytes >> 4); }

}  // namespace la
