// Combine, bias update and weight packing.
//
// Combine is the COMBINE step (mhpq.cn article §2.2): y_t = y_shared_t +
// sum_k gate[t,k] * y_perm[slot[t,k]], fp32 accumulation in k order, one
// rounding to the output dtype; one CTA per token row, 16-byte vectors.
//
// Bias update: the auxiliary-loss-free rule (kaiyunto.com walk-through,
// DeepSeekMoE paragraphs; mhpq.cn article §1.2): b_i -= gamma when expert i
// took more than its share T*K/N of the rows, += gamma when it took fewer.
#include <cuda_bf16.h>

#include "internal.h"
#include "ptx.cuh"
#include "tile_transpose.cuh"

namespace moe {
namespace {

__device__ __forceinline__ void to_f32x8(const uint4& v, float (&o)[8]) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __bfloat1622float2(h[i]);
    o[2 * i] = f.x;
    o[2 * i + 1] = f.y;
  }
}

// KM > 0 (K <= KM): a thread loads its piece of all K rows before the first
// multiply-add, so K loads are in flight; KM = 0 takes the rows one by one.
// Either way the sums run in k order from y_shared.
template <int KM>
__global__ void __launch_bounds__(128) combine_bf16_kernel(const __nv_bfloat16* __restrict__ y_perm,
                                                           const __nv_bfloat16* __restrict__ y_sh,
                                                           const int32_t* __restrict__ slot,
                                                           const float* __restrict__ gate, int T,
                                                           int d, int K,
                                                           __nv_bfloat16* __restrict__ y) {
  __shared__ int ss[kMaxK];
  __shared__ float sg[kMaxK];
  const int t = blockIdx.x;
  if (threadIdx.x < K) {
    const int r = slot[(size_t)t * K + threadIdx.x];
    const bool ok = r >= 0 && r < T * K;  // a slot outside the rows is skipped
    ss[threadIdx.x] = ok ? r : 0;
    sg[threadIdx.x] = ok ? gate[(size_t)t * K + threadIdx.x] : 0.f;
  }
  __syncthreads();
  const int nvec = d / 8;
  for (int v = threadIdx.x; v < nvec; v += blockDim.x) {
    float acc[8];
    if constexpr (KM > 0) {
      uint4 raw[KM];
#pragma unroll
      for (int k = 0; k < KM; ++k)
        if (k < K) raw[k] = __ldg(reinterpret_cast<const uint4*>(y_perm + (size_t)ss[k] * d) + v);
      to_f32x8(__ldg(reinterpret_cast<const uint4*>(y_sh + (size_t)t * d) + v), acc);
#pragma unroll
      for (int k = 0; k < KM; ++k) {
        if (k >= K) break;
        float r[8];
        to_f32x8(raw[k], r);
        const float g = sg[k];
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = fmaf(g, r[i], acc[i]);
      }
    } else {
      to_f32x8(__ldg(reinterpret_cast<const uint4*>(y_sh + (size_t)t * d) + v), acc);
      for (int k = 0; k < K; ++k) {
        float r[8];
        to_f32x8(__ldg(reinterpret_cast<const uint4*>(y_perm + (size_t)ss[k] * d) + v), r);
        const float g = sg[k];
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = fmaf(g, r[i], acc[i]);
      }
    }
    uint4 out;
    __nv_bfloat162* o = reinterpret_cast<__nv_bfloat162*>(&out);
#pragma unroll
    for (int i = 0; i < 4; ++i) o[i] = __floats2bfloat162_rn(acc[2 * i], acc[2 * i + 1]);
    reinterpret_cast<uint4*>(y + (size_t)t * d)[v] = out;
  }
}

__global__ void __launch_bounds__(128) combine_f32_kernel(const float* __restrict__ y_perm,
                                                          const float* __restrict__ y_sh,
                                                          const int32_t* __restrict__ slot,
                                                          const float* __restrict__ gate, int T,
                                                          int d, int K, float* __restrict__ y) {
  __shared__ int ss[kMaxK];
  __shared__ float sg[kMaxK];
  const int t = blockIdx.x;
  if (threadIdx.x < K) {
    const int r = slot[(size_t)t * K + threadIdx.x];
    const bool ok = r >= 0 && r < T * K;
    ss[threadIdx.x] = ok ? r : 0;
    sg[threadIdx.x] = ok ? gate[(size_t)t * K + threadIdx.x] : 0.f;
  }
  __syncthreads();
  const int nvec = d / 4;
  for (int v = threadIdx.x; v < nvec; v += blockDim.x) {
    float4 acc = __ldg(reinterpret_cast<const float4*>(y_sh + (size_t)t * d) + v);
    for (int k = 0; k < K; ++k) {
      const float4 r = __ldg(reinterpret_cast<const float4*>(y_perm + (size_t)ss[k] * d) + v);
      const float g = sg[k];
      acc.x = fmaf(g, r.x, acc.x);
      acc.y = fmaf(g, r.y, acc.y);
      acc.z = fmaf(g, r.z, acc.z);
      acc.w = fmaf(g, r.w, acc.w);
    }
    reinterpret_cast<float4*>(y + (size_t)t * d)[v] = acc;
  }
}

__global__ void bias_update_kernel(const int32_t* __restrict__ counts, float* __restrict__ bias,
                                   int N, long long TK, float gamma) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= N) return;
  const long long load = (long long)counts[i] * N;
  const float b = bias[i];
  if (load > TK)
    bias[i] = __fsub_rn(b, gamma);
  else if (load < TK)
    bias[i] = __fadd_rn(b, gamma);
}

// w13[e][P*2j + r] = w1[e][P*j + r], w13[e][P*(2j+1) + r] = w3[e][P*j + r]
// for P = pack_block(f); rows of d elements copied as 16-byte vectors.
__global__ void pack_w13_kernel(const uint4* __restrict__ w1, const uint4* __restrict__ w3,
                                uint4* __restrict__ w13, int E, int f, int P,
                                int vec_per_row) {
  const long long total = (long long)E * 2 * f * vec_per_row;
  for (long long q = (long long)blockIdx.x * blockDim.x + threadIdx.x; q < total;
       q += (long long)gridDim.x * blockDim.x) {
    const long long row = q / vec_per_row;  // row in w13
    const int v = (int)(q - row * vec_per_row);
    const int e = (int)(row / (2 * f));
    const int r = (int)(row - (long long)e * 2 * f);
    const int blk = r / (2 * P), within = r % (2 * P);
    const bool is_w3 = within >= P;
    const int src_row = blk * P + (is_w3 ? within - P : within);
    const uint4* src = is_w3 ? w3 : w1;
    w13[q] = src[((long long)e * f + src_row) * vec_per_row + v];
  }
}

}  // namespace

cudaError_t launch_combine(const moe_shape& s, const void* y_perm, const void* y_shared,
                           const int32_t* slot, const float* gate, void* y, cudaStream_t st) {
  if (s.dtype == MOE_DTYPE_FP32)
    combine_f32_kernel<<<s.T, 128, 0, st>>>(static_cast<const float*>(y_perm),
                                            static_cast<const float*>(y_shared), slot, gate,
                                            s.T, s.d, s.K, static_cast<float*>(y));
  else if (s.K <= 8)
    combine_bf16_kernel<8><<<s.T, 128, 0, st>>>(static_cast<const __nv_bfloat16*>(y_perm),
                                                static_cast<const __nv_bfloat16*>(y_shared), slot,
                                                gate, s.T, s.d, s.K,
                                                static_cast<__nv_bfloat16*>(y));
  else
    combine_bf16_kernel<0><<<s.T, 128, 0, st>>>(static_cast<const __nv_bfloat16*>(y_perm),
                                                static_cast<const __nv_bfloat16*>(y_shared), slot,
                                                gate, s.T, s.d, s.K,
                                                static_cast<__nv_bfloat16*>(y));
  return cudaGetLastError();
}

cudaError_t launch_bias_update(const moe_shape& s, const int32_t* counts, float* bias,
                               float gamma, cudaStream_t st) {
  bias_update_kernel<<<(s.N + 255) / 256, 256, 0, st>>>(counts, bias, s.N,
                                                        (long long)s.T * s.K, gamma);
  return cudaGetLastError();
}

cudaError_t launch_pack_w13(const moe_shape& s, const void* w1, const void* w3, void* w13,
                            cudaStream_t st) {
  const size_t eb = (s.dtype == MOE_DTYPE_FP32) ? 4 : 2;  // E4M3 packs the bf16 weights
  const int vec_per_row = (int)(s.d * eb / 16);
  const long long total = (long long)(s.N + 1) * 2 * s.f * vec_per_row;
  long long blocks = (total + 255) / 256;
  if (blocks > 148 * 16) blocks = 148 * 16;
  pack_w13_kernel<<<(int)blocks, 256, 0, st>>>(static_cast<const uint4*>(w1),
                                               static_cast<const uint4*>(w3),
                                               static_cast<uint4*>(w13), s.N + 1, s.f,
                                               pack_block(s.f), vec_per_row);
  return cudaGetLastError();
}

// [B, R, C] bf16 -> [B, C, R] in 64 x 64 tiles (tile_transpose.cuh); R and
// C are multiples of 64 (the bf16 shape rules make d, f and 2f so).  A CTA
// moves kRowTiles tiles of the same 64 rows and consecutive columns, with all
// its 16-byte loads issued before any shared-memory write (2 * kRowTiles
// loads in flight per thread).
namespace {
constexpr int kRowTiles = 4;
constexpr int kTItems = kTile * 8 / kTileThreads;  // 16-byte items per thread per tile

__global__ void __launch_bounds__(kTileThreads) transpose_tiles_kernel(
    const __nv_bfloat16* __restrict__ src, __nv_bfloat16* __restrict__ dst, int R, int C) {
  __shared__ alignas(16) uint8_t sm[kRowTiles][kTileBytes];
  const size_t b = blockIdx.z;
  const int r0 = blockIdx.y * kTile, cb = blockIdx.x * kRowTiles * kTile;
  uint4 v[kRowTiles][kTItems];
#pragma unroll
  for (int t = 0; t < kRowTiles; ++t) {
    const int c0 = cb + t * kTile;
#pragma unroll
    for (int j = 0; j < kTItems; ++j) {
      const int it = threadIdx.x + j * kTileThreads;
      const int i = it >> 3, p = it & 7;
      v[t][j] = make_uint4(0u, 0u, 0u, 0u);
      if (r0 + i < R && c0 + p * 8 + 8 <= C)
        v[t][j] = __ldg(reinterpret_cast<const uint4*>(src + (b * R + r0 + i) * C + c0 + p * 8));
    }
  }
#pragma unroll
  for (int t = 0; t < kRowTiles; ++t)
#pragma unroll
    for (int j = 0; j < kTItems; ++j) {
      const int it = threadIdx.x + j * kTileThreads;
      tile_put(sm[t], it >> 3, it & 7, v[t][j]);
    }
  __syncthreads();
#pragma unroll
  for (int t = 0; t < kRowTiles; ++t) {
    const int c0 = cb + t * kTile;
    for (int it = threadIdx.x; it < kTile * 8; it += kTileThreads) {
      const int c = it >> 3, q = it & 7;
      if (c0 + c < C && r0 + q * 8 + 8 <= R)
        *reinterpret_cast<uint4*>(dst + (b * C + c0 + c) * R + r0 + q * 8) = tile_get(sm[t], c, q);
    }
  }
}
}  // namespace

cudaError_t launch_transpose_weights(const moe_shape& s, const void* w13, const void* w2,
                                     void* w13t, void* w2t, cudaStream_t st) {
  if (s.d % kTile != 0 || (2 * s.f) % kTile != 0 || s.f % kTile != 0)
    return cudaErrorInvalidValue;
  const unsigned E = (unsigned)(s.N + 1);
  const auto blocks = [](int C) { return (unsigned)((C / kTile + kRowTiles - 1) / kRowTiles); };
  transpose_tiles_kernel<<<dim3(blocks(s.d), 2 * s.f / kTile, E), kTileThreads, 0, st>>>(
      static_cast<const __nv_bfloat16*>(w13), static_cast<__nv_bfloat16*>(w13t), 2 * s.f, s.d);
  transpose_tiles_kernel<<<dim3(blocks(s.f), s.d / kTile, E), kTileThreads, 0, st>>>(
      static_cast<const __nv_bfloat16*>(w2), static_cast<__nv_bfloat16*>(w2t), s.d, s.f);
  return cudaGetLastError();
}

}  // namespace moe
