// Routing: fp32 affinity scores, biased group-limited top-K, gates, counts.
//
// DeepSeek-V3 pages: sigmoid affinity and gate = normalisation over the
// selected affinities (kaiyunto.com walk-through, DeepSeekMoE paragraphs); the
// bias is added to the affinity for expert selection only (gkm0120.cn notes
// Q3; mhpq.cn article §1.2); each token reaches at most topG expert groups
// (mhpq.cn article §3.1, "at most 4 nodes").  Group score = sum of the two
// largest biased scores in the group (the reading this library takes).
//
// One CTA handles 32 tokens against all N (<= 256) experts.  Phase 1 is a
// SIMT fp32 GEMM tile: x and the router are staged through shared memory in
// 32-wide slices of d; warp w accumulates tokens 4w..4w+3 and lane l holds
// experts l, l+32, ..., so after the K loop a warp owns every score of its
// four tokens in registers.  Phase 2 (per token, inside the warp, no shared
// memory): group top-2 sums by butterfly shuffles, top-topG groups and top-K
// experts by warp arg-max rounds (ties to the lower index), ascending-id
// ordering of the K winners, fp32 gates, and a shared-memory histogram that
// is added to counts[] with integer atomics (order-independent).
#include <cuda_bf16.h>

#include "internal.h"
#include "ptx.cuh"

namespace moe {
namespace {

constexpr int kBT = kRouteTokens;  // 32 tokens / CTA
constexpr int kKC = 32;            // d slice
constexpr int kEPL = kRouteMaxN / 32;  // experts per lane

__device__ __forceinline__ float load_f(const float* p) { return *p; }
__device__ __forceinline__ float load_f(const __nv_bfloat16* p) { return __bfloat162float(*p); }

// (v, i) beats (w, j) if v > w, or v == w and i < j.
__device__ __forceinline__ bool better(float v, int i, float w, int j) {
  return v > w || (v == w && i < j);
}

__device__ __forceinline__ void warp_argmax(float& v, int& i) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    float w = __shfl_xor_sync(0xffffffffu, v, o);
    int j = __shfl_xor_sync(0xffffffffu, i, o);
    if (better(w, j, v, i)) { v = w; i = j; }
  }
}

// Merge two (largest, second largest) pairs.
__device__ __forceinline__ void top2_merge(float& a1, float& a2, float b1, float b2) {
  if (b1 > a1) {
    a2 = fmaxf(a1, b2);
    a1 = b1;
  } else {
    a2 = fmaxf(a2, b1);
  }
}

template <typename XT>
__global__ void __launch_bounds__(256) route_kernel(const XT* __restrict__ x,
                                                    const float* __restrict__ router,
                                                    const float* __restrict__ bias, int T, int d,
                                                    int N, int K, int G, int topG,
                                                    int32_t* __restrict__ topk_idx,
                                                    float* __restrict__ topk_gate,
                                                    int32_t* __restrict__ counts,
                                                    uint32_t* __restrict__ status) {
  __shared__ float xs[kBT][kKC + 1];
  __shared__ float rs[kRouteMaxN][kKC + 1];
  __shared__ int hist[kRouteMaxN];

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int t0 = blockIdx.x * kBT;

  for (int e = tid; e < kRouteMaxN; e += blockDim.x) hist[e] = 0;

  float acc[4][kEPL];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < kEPL; ++j) acc[i][j] = 0.f;

  // ---- phase 1: scores z[t, e] = x_t . e_e in fp32 ----
  for (int k0 = 0; k0 < d; k0 += kKC) {
    for (int q = tid; q < kBT * kKC; q += blockDim.x) {
      const int r = q / kKC, c = q % kKC;
      const int t = t0 + r;
      xs[r][c] = (t < T) ? load_f(x + (size_t)t * d + k0 + c) : 0.f;
    }
    for (int q = tid; q < N * kKC; q += blockDim.x) {
      const int r = q / kKC, c = q % kKC;
      rs[r][c] = router[(size_t)r * d + k0 + c];
    }
    __syncthreads();
#pragma unroll 4
    for (int c = 0; c < kKC; ++c) {
      float xv[4], rv[kEPL];
#pragma unroll
      for (int i = 0; i < 4; ++i) xv[i] = xs[warp * 4 + i][c];
#pragma unroll
      for (int j = 0; j < kEPL; ++j) rv[j] = (lane + 32 * j < N) ? rs[lane + 32 * j][c] : 0.f;
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < kEPL; ++j) acc[i][j] = fmaf(xv[i], rv[j], acc[i][j]);
    }
    __syncthreads();
  }

  // ---- phase 2: selection, one token at a time per warp ----
  const int gs = N / G;
  float bj[kEPL];
#pragma unroll
  for (int j = 0; j < kEPL; ++j) {
    const int e = lane + 32 * j;
    bj[j] = (e < N) ? bias[e] : 0.f;
  }

#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int t = t0 + warp * 4 + i;
    if (t >= T) break;  // warp-uniform
    float s[kEPL], sb[kEPL];
#pragma unroll
    for (int j = 0; j < kEPL; ++j) {
      const int e = lane + 32 * j;
      s[j] = 1.f / (1.f + expf(-acc[i][j]));
      sb[j] = (e < N) ? s[j] + bj[j] : -INFINITY;
    }
    // group scores: lane g ends up holding group g's score
    float my_gscore = -INFINITY;
    for (int g = 0; g < G; ++g) {
      float m1 = -INFINITY, m2 = -INFINITY;
#pragma unroll
      for (int j = 0; j < kEPL; ++j) {
        const int e = lane + 32 * j;
        if (e < N && e / gs == g) top2_merge(m1, m2, sb[j], -INFINITY);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const float b1 = __shfl_xor_sync(0xffffffffu, m1, o);
        const float b2 = __shfl_xor_sync(0xffffffffu, m2, o);
        top2_merge(m1, m2, b1, b2);
      }
      const float score = (gs >= 2) ? m1 + m2 : m1;
      if (lane == g) my_gscore = score;
    }
    // keep the topG best groups
    uint32_t kept = 0;
    for (int r = 0; r < topG; ++r) {
      float v = ((kept >> lane) & 1u) ? -INFINITY : my_gscore;
      int gi = (lane < G && !((kept >> lane) & 1u)) ? lane : 0x7fffffff;
      if (lane >= G) v = -INFINITY;
      warp_argmax(v, gi);
      kept |= 1u << gi;
    }
    // top-K among experts of kept groups
    uint32_t taken = 0;  // bit j: this lane's expert lane+32j already chosen
    int my_e = 0x7fffffff;
    float my_s = 0.f;
    for (int r = 0; r < K; ++r) {
      float v = -INFINITY;
      int ei = 0x7fffffff;
#pragma unroll
      for (int j = 0; j < kEPL; ++j) {
        const int e = lane + 32 * j;
        if (e < N && ((kept >> (e / gs)) & 1u) && !((taken >> j) & 1u) &&
            better(sb[j], e, v, ei)) {
          v = sb[j];
          ei = e;
        }
      }
      warp_argmax(v, ei);
      // the owner marks it and broadcasts its un-biased score
      float sv = 0.f;
#pragma unroll
      for (int j = 0; j < kEPL; ++j) {
        if (lane + 32 * j == ei) {
          taken |= 1u << j;
          sv = s[j];
        }
      }
      const int owner = ei & 31;
      sv = __shfl_sync(0xffffffffu, sv, owner);
      if (lane == r) {
        my_e = ei;
        my_s = sv;
      }
    }
    // ascending expert order and gates
    int rank = 0;
    for (int q = 0; q < K; ++q) {
      const int eq = __shfl_sync(0xffffffffu, my_e, q);
      rank += (eq < my_e) ? 1 : 0;
    }
    float sum = (lane < K) ? my_s : 0.f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    if (lane < K) {
      if (my_e < 0 || my_e >= N) {
        atomicOr(status, kErrBadIndex);
      } else {
        topk_idx[(size_t)t * K + rank] = my_e;
        topk_gate[(size_t)t * K + rank] = my_s / sum;
        atomicAdd(&hist[my_e], 1);
      }
    }
  }
  __syncthreads();
  for (int e = tid; e < N; e += blockDim.x)
    if (hist[e]) atomicAdd(&counts[e], hist[e]);
}

}  // namespace

cudaError_t launch_route(const moe_shape& s, const void* x, const float* router,
                         const float* bias, int32_t* idx, float* gate, int32_t* counts,
                         uint32_t* status, cudaStream_t st) {
  cudaError_t e = cudaMemsetAsync(counts, 0, sizeof(int32_t) * s.N, st);
  if (e != cudaSuccess) return e;
  const int grid = (s.T + kBT - 1) / kBT;
  if (s.dtype == MOE_DTYPE_FP32)
    route_kernel<float><<<grid, 256, 0, st>>>(static_cast<const float*>(x), router, bias, s.T,
                                              s.d, s.N, s.K, s.G, s.topG, idx, gate, counts,
                                              status);
  else
    route_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(
        static_cast<const __nv_bfloat16*>(x), router, bias, s.T, s.d, s.N, s.K, s.G, s.topG,
        idx, gate, counts, status);
  return cudaGetLastError();
}

}  // namespace moe
