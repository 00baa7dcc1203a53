// E4M3 helpers shared by the dispatch gather and the FP8 GEMM file:
// 1x128 tile quantisation (scale = amax/448 and inverse 448/amax in fp32,
// code = E4M3 round-to-nearest-even with saturation of v * inverse; an
// all-zero tile gets scale 1 and zero codes), following the fine-grained
// online scaling of the mhpq.cn article §4.1.
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include <cstdint>

namespace moe {

constexpr int QB = 128;  // quantisation tile / K slice

// A half-warp (16 lanes) holds one 128-wide tile, 8 consecutive elements per
// lane.  Returns the tile scale; writes this lane's 8 codes.  kE5M2: the
// gradient format of the backward pass (largest finite 57344) instead of
// E4M3 (448), with the same scaling rule.
template <bool kE5M2 = false>
static __device__ __forceinline__ float quant_tile_16lanes(const float (&v)[8], uint2& codes) {
  constexpr float kMax = kE5M2 ? 57344.f : 448.f;
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(v[i]));
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if (amax == 0.f) {
    codes = make_uint2(0u, 0u);
    return 1.f;
  }
  const float scale = __fdiv_rn(amax, kMax);
  const float inv = __fdiv_rn(kMax, amax);
  uint32_t w[2];
#pragma unroll
  for (int p = 0; p < 2; ++p) {
    uint32_t word = 0;
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      const int i = 4 * p + 2 * q;
      const __nv_fp8x2_storage_t c2 = __nv_cvt_float2_to_fp8x2(
          make_float2(__fmul_rn(v[i], inv), __fmul_rn(v[i + 1], inv)), __NV_SATFINITE,
          kE5M2 ? __NV_E5M2 : __NV_E4M3);
      word |= (uint32_t)c2 << (16 * q);
    }
    w[p] = word;
  }
  codes = make_uint2(w[0], w[1]);
  return scale;
}

static __device__ __forceinline__ void bf16x8_to_f32(const uint4& u, float (&f)[8]) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 t = __bfloat1622float2(h[i]);
    f[2 * i] = t.x;
    f[2 * i + 1] = t.y;
  }
}

}  // namespace moe
