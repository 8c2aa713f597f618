// Helpers shared by the tensor-core kernels (step_tc.cu, prefill_tc.cu).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <stdint.h>

namespace onela {

// Copies n parent indices (int32, global) to shared memory as 16-bit
// indices, by the 32 lanes of one warp: 16-byte loads when the source allows
// it, single ints otherwise.  dst is 8-byte aligned; parents are below 2^16
// (anything else is out of range and is clamped where it is used).
__device__ __forceinline__ void copy_parents16_warp(uint16_t *dst, const int32_t *src, int n, int lane) {
  int done = 0;
  if ((reinterpret_cast<uintptr_t>(src) & 15u) == 0) {
    done = n & ~3;
#pragma unroll 2
    for (int e = lane * 4; e < done; e += 128) {
      const int4 v = __ldg(reinterpret_cast<const int4 *>(src + e));
      *reinterpret_cast<uint2 *>(dst + e) = make_uint2(((uint32_t)v.x & 0xffffu) | ((uint32_t)v.y << 16),
                                                      ((uint32_t)v.z & 0xffffu) | ((uint32_t)v.w << 16));
    }
  }
  for (int e = done + lane; e < n; e += 32) dst[e] = (uint16_t)__ldg(src + e);
}

// Four consecutive bf16 elements (packed in u, or at p, 8-byte aligned) as floats.
__device__ __forceinline__ float4 bf16x4(uint2 u) {
  const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.x));
  const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.y));
  return make_float4(a.x, a.y, b.x, b.y);
}
__device__ __forceinline__ float4 bf16x4(const uint8_t *p) { return bf16x4(*reinterpret_cast<const uint2 *>(p)); }

// 4-D tensor map over a [R][W][H][d] bf16 tensor: {d, H, W, R}, box
// {64, 1, box_rows, 1} (one 128-byte K atom of box_rows beam rows), 128-byte
// swizzle (the K-major operand layout), zeros outside the tensor.  False when
// the driver's encoder is unavailable or rejects the tensor.
bool encode_rows(CUtensorMap *m, const void *base, int d, int H, int W, int R, int box_rows = 32);

}  // namespace onela
