// Epilogue helpers shared by the bf16 expert GEMM kernels.
#pragma once
#include <cuda_bf16.h>
#include <cstdint>

namespace moe {

// silu(v) = v / (1 + e^-v) with the hardware exponential and an approximate
// divide (relative error ~1e-6, far below bf16 and E4M3 rounding): the
// tensor-core epilogues evaluate it for every hidden feature on the path
// between the MMA and the next tile.  For v below about -87, 1 + e^-v
// overflows or passes 2^126 and the quotient is 0, where the exact value is
// under 1e-36 in magnitude.
__device__ __forceinline__ float silu_fast(float v) { return __fdividef(v, 1.f + __expf(-v)); }

// SwiGLU backward for one hidden feature: with dh the gradient of
// h = silu(g) * u, dg = dh * u * silu'(g) (silu'(g) = s (1 + g (1 - s)),
// s = sigmoid(g)) and du = dh * silu(g).
__device__ __forceinline__ void swiglu_bwd(float dh, float g, float u, float& dg, float& du) {
  const float sg = 1.f / (1.f + expf(-g));
  dg = dh * u * (sg * (1.f + g * (1.f - sg)));
  du = dh * (g * sg);
}

// 32 fp32 values -> 32 bf16 (round to nearest even), four 16-byte stores.
__device__ __forceinline__ void store_row32(__nv_bfloat16* dst, const float* v) {
  uint4 w[4];
  __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(w);
#pragma unroll
  for (int i = 0; i < 16; ++i) h[i] = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
  uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int i = 0; i < 4; ++i) d4[i] = w[i];
}

// Two fp32 -> bf16x2 bits (round to nearest even), `lo` in the low half.
__device__ __forceinline__ uint32_t bf16x2_bits(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// 8 bf16 packed in 16 bytes -> 8 fp32.
__device__ __forceinline__ void bf16x8_unpack(const uint4& w, float* v) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&w);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __bfloat1622float2(h[i]);
    v[2 * i] = f.x;
    v[2 * i + 1] = f.y;
  }
}

// 8 bf16 (one 16-byte load) -> 8 fp32.
__device__ __forceinline__ void bf16x8_load(const __nv_bfloat16* src, float* v) {
  const uint4 w = *reinterpret_cast<const uint4*>(src);
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&w);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __bfloat1622float2(h[i]);
    v[2 * i] = f.x;
    v[2 * i + 1] = f.y;
  }
}

}  // namespace moe
