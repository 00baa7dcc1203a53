// Routing: fp32 affinity scores, biased group-limited top-K, gates, counts.
//
// DeepSeek-V3 pages: sigmoid affinity and gate = normalisation over the
// selected affinities (kaiyunto.com walk-through, DeepSeekMoE paragraphs); the
// bias is added to the affinity for expert selection only (gkm0120.cn notes
// Q3; mhpq.cn article §1.2); each token reaches at most topG expert groups
// (mhpq.cn article §3.1, "at most 4 nodes").  Group score = sum of the two
// largest biased scores in the group (the reading this library takes).
//
// bf16 inputs: the logits come from the tensor cores (an exact three-part
// bf16 split of the fp32 router, see gemm_tc.cu) as fp32 K-split partials,
// and select_kernel sums them, applies the sigmoid and selects (below).
//
// fp32 inputs: one CTA handles 32 tokens against all N (<= 256) experts.
// Phase 1 is a SIMT fp32 GEMM tile: x and the router are staged through shared memory in
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

// (v, i) beats (w, j) if v > w, or v == w and i < j.
__device__ __forceinline__ bool better(float v, int i, float w, int j) {
  return v > w || (v == w && i < j);
}

// Unsigned keys in the order of the floats (NaN never occurs here); -0 is
// taken as +0 first, so equal floats have equal keys.
__device__ __forceinline__ uint32_t order_key(float v) {
  const uint32_t u = __float_as_uint(v == 0.f ? 0.f : v);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key_float(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

// The warp's best (v, i) under `better` (largest v, then smallest i), on
// every lane: two warp-wide reductions (max of the value keys, then min of
// the indices holding that value).  i >= 0.
__device__ __forceinline__ void warp_argmax(float& v, int& i) {
  const uint32_t k = order_key(v);
  const uint32_t kmax = __reduce_max_sync(0xffffffffu, k);
  i = (int)__reduce_min_sync(0xffffffffu, k == kmax ? (uint32_t)i : 0xffffffffu);
  v = key_float(kmax);
}

// The two largest of the 32 lanes' (largest, second largest) pairs, on every
// lane: the largest first value, then the largest of the other lanes' first
// values and that lane's second value.
__device__ __forceinline__ void warp_top2(float& m1, float& m2, int lane) {
  const uint32_t k1 = order_key(m1);
  const uint32_t kmax = __reduce_max_sync(0xffffffffu, k1);
  const uint32_t owner = __reduce_min_sync(0xffffffffu, k1 == kmax ? (uint32_t)lane : 32u);
  const uint32_t k2 = __reduce_max_sync(0xffffffffu, (uint32_t)lane == owner ? order_key(m2) : k1);
  m1 = key_float(kmax);
  m2 = key_float(k2);
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

// Selection for one token by one warp.  Lane l holds experts l + 32 j in
// s[j] (un-biased sigmoid scores) and bj[j] (their biases).  Writes the K
// chosen experts in ascending id order with their gates, and counts them in
// the shared-memory histogram.
// Group of each expert a lane holds (expert lane + 32 j; -1 past N).
__device__ __forceinline__ void lane_groups(int lane, int N, int G, int (&grp)[kEPL]) {
  const int gs = N / G;
#pragma unroll
  for (int j = 0; j < kEPL; ++j) grp[j] = (lane + 32 * j < N) ? (lane + 32 * j) / gs : -1;
}

__device__ __forceinline__ void select_token(const float (&s)[kEPL], const float (&bj)[kEPL],
                                             const int (&grp)[kEPL], int lane, int t, int N,
                                             int K, int G, int topG,
                                             int32_t* __restrict__ topk_idx,
                                             float* __restrict__ topk_gate, int* hist,
                                             uint32_t* status) {
  const int gs = N / G;
  float sb[kEPL];
#pragma unroll
  for (int j = 0; j < kEPL; ++j) sb[j] = (grp[j] >= 0) ? s[j] + bj[j] : -INFINITY;
  // group scores: lane g ends up holding group g's score
  float my_gscore = -INFINITY;
  for (int g = 0; g < G; ++g) {
    float m1 = -INFINITY, m2 = -INFINITY;
#pragma unroll
    for (int j = 0; j < kEPL; ++j)
      if (grp[j] == g) top2_merge(m1, m2, sb[j], -INFINITY);
    warp_top2(m1, m2, lane);
    const float score = (gs >= 2) ? m1 + m2 : m1;
    if (lane == g) my_gscore = score;
  }
  // keep the topG best groups
  uint32_t kept = 0;
  for (int r = 0; r < topG; ++r) {
    float v = (lane < G && !((kept >> lane) & 1u)) ? my_gscore : -INFINITY;
    int gi = (lane < G && !((kept >> lane) & 1u)) ? lane : 0x7fffffff;
    warp_argmax(v, gi);
    kept |= 1u << (gi & 31);
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
      if (grp[j] >= 0 && ((kept >> grp[j]) & 1u) && !((taken >> j) & 1u) &&
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
    sv = __shfl_sync(0xffffffffu, sv, ei & 31);
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

// fp32 inputs: SIMT score tile + selection (see the top of this file).
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
  float bj[kEPL];
  int grp[kEPL];
  lane_groups(lane, N, G, grp);
#pragma unroll
  for (int j = 0; j < kEPL; ++j) bj[j] = (lane + 32 * j < N) ? bias[lane + 32 * j] : 0.f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int t = t0 + warp * 4 + i;
    if (t >= T) break;  // warp-uniform
    float s[kEPL];
#pragma unroll
    for (int j = 0; j < kEPL; ++j) s[j] = 1.f / (1.f + expf(-acc[i][j]));
    select_token(s, bj, grp, lane, t, N, K, G, topG, topk_idx, topk_gate, hist, status);
  }
  __syncthreads();
  for (int e = tid; e < N; e += blockDim.x)
    if (hist[e]) atomicAdd(&counts[e], hist[e]);
}

// Selection from the tensor-core logits Z [splits, T, N]: z is the sum of
// the split partials in split order, s = sigmoid(z); one warp per token,
// 8 tokens per CTA.
//
// kSoftmax: the conventional softmax gate kept as a baseline (the DeepSeek-V3
// walk-through's gating paragraph: a softmax on top of a classifier, balanced
// by an auxiliary penalty).  The selection score is e = exp(z - max_i z)
// (monotone in z) with no bias and one group, so the same top-K picks the K
// largest logits and the gate normalisation gives e_k / sum over the selected,
// the softmax over the selected logits.  The CTA also writes, per expert, the
// sum over its tokens (in warp order) of p = e / sum_i e, for the balance
// statistic.
constexpr int kSelTokens = 8;

template <bool kSoftmax>
__global__ void __launch_bounds__(256) select_kernel(const float* __restrict__ Z, int splits,
                                                     const float* __restrict__ bias, int T, int N,
                                                     int K, int G, int topG,
                                                     int32_t* __restrict__ topk_idx,
                                                     float* __restrict__ topk_gate,
                                                     int32_t* __restrict__ counts,
                                                     float* __restrict__ prob_part,
                                                     uint32_t* __restrict__ status) {
  __shared__ int hist[kRouteMaxN];
  __shared__ float pbuf[kSoftmax ? kSelTokens : 1][kSoftmax ? kRouteMaxN : 1];
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  for (int e = tid; e < N; e += blockDim.x) hist[e] = 0;
  __syncthreads();
  const int t = blockIdx.x * kSelTokens + warp;
  if (t < T) {
    float bj[kEPL], s[kEPL];
    int grp[kEPL];
    lane_groups(lane, N, G, grp);
    float zmax = -INFINITY;
#pragma unroll
    for (int j = 0; j < kEPL; ++j) {
      float z = 0.f;
      bj[j] = 0.f;
      if (grp[j] >= 0) {
        if (!kSoftmax) bj[j] = __ldg(bias + lane + 32 * j);
        z = __ldg(Z + (size_t)t * N + lane + 32 * j);
        for (int p = 1; p < splits; ++p)
          z = __fadd_rn(z, __ldg(Z + ((size_t)p * T + t) * N + lane + 32 * j));
        zmax = fmaxf(zmax, z);
      }
      s[j] = kSoftmax ? z : 1.f / (1.f + expf(-z));
    }
    if constexpr (kSoftmax) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) zmax = fmaxf(zmax, __shfl_xor_sync(0xffffffffu, zmax, o));
      float esum = 0.f;
#pragma unroll
      for (int j = 0; j < kEPL; ++j) {
        s[j] = grp[j] >= 0 ? expf(s[j] - zmax) : 0.f;
        esum += s[j];
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) esum += __shfl_xor_sync(0xffffffffu, esum, o);
#pragma unroll
      for (int j = 0; j < kEPL; ++j)
        if (grp[j] >= 0) pbuf[warp][lane + 32 * j] = __fdiv_rn(s[j], esum);
    }
    select_token(s, bj, grp, lane, t, N, K, G, topG, topk_idx, topk_gate, hist, status);
  }
  __syncthreads();
  if constexpr (kSoftmax) {  // this CTA's per-expert probability sums, tokens in order
    const int nt = min(kSelTokens, T - (int)blockIdx.x * kSelTokens);
    for (int e = tid; e < N; e += blockDim.x) {
      float a = 0.f;
      for (int w = 0; w < nt; ++w) a += pbuf[w][e];
      prob_part[(size_t)blockIdx.x * N + e] = a;
    }
  }
  for (int e = tid; e < N; e += blockDim.x)
    if (hist[e]) atomicAdd(&counts[e], hist[e]);
}

// prob_sum[e]: the selection CTAs' partials summed in a fixed order (eight
// running sums over the CTAs b = j mod 8, then added j = 0..7), so the result
// does not depend on scheduling.  Block: 32 experts (lanes) x the eight sums
// (warps); each sum takes its CTAs in increasing order, eight loads ahead.
__global__ void __launch_bounds__(256) prob_sum_kernel(const float* __restrict__ part,
                                                       int nblocks, int N,
                                                       float* __restrict__ prob_sum) {
  __shared__ float run[8][32];
  const int lane = threadIdx.x & 31, j = threadIdx.x >> 5;
  const int e = blockIdx.x * 32 + lane;
  float a = 0.f;
  if (e < N) {
    for (int b = j; b < nblocks; b += 64) {
      float v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u)
        v[u] = (b + 8 * u < nblocks) ? part[(size_t)(b + 8 * u) * N + e] : 0.f;
#pragma unroll
      for (int u = 0; u < 8; ++u)
        if (b + 8 * u < nblocks) a += v[u];
    }
  }
  run[j][lane] = a;
  __syncthreads();
  if (j == 0 && e < N) {
    float sum = 0.f;
#pragma unroll
    for (int q = 0; q < 8; ++q) sum += run[q][lane];
    prob_sum[e] = sum;
  }
}

}  // namespace

int launch_route(const moe_shape& s, const void* x, const float* router, const float* bias,
                 int32_t* idx, float* gate, int32_t* counts, void* ws, cudaStream_t st) {
  const WsLayout L = ws_layout(s);
  uint8_t* w = static_cast<uint8_t*>(ws);
  uint32_t* status = reinterpret_cast<uint32_t*>(w + L.status);
  if (cudaMemsetAsync(counts, 0, sizeof(int32_t) * s.N, st) != cudaSuccess) return MOE_ERR_CUDA;
  const int grid = (s.T + kBT - 1) / kBT;
  if (s.dtype == MOE_DTYPE_FP32) {
    route_kernel<float><<<grid, 256, 0, st>>>(static_cast<const float*>(x), router, bias, s.T,
                                              s.d, s.N, s.K, s.G, s.topG, idx, gate, counts,
                                              status);
  } else {
    float* Z = reinterpret_cast<float*>(w + L.scores);
    const int splits = router_k_splits(s);
    const int rc = launch_router_scores_tc(s, x, router, Z, splits, ws, st);
    if (rc != MOE_OK) return rc;
    select_kernel<false><<<(s.T + kSelTokens - 1) / kSelTokens, 256, 0, st>>>(
        Z, splits, bias, s.T, s.N, s.K, s.G, s.topG, idx, gate, counts, nullptr, status);
  }
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

int launch_route_softmax(const moe_shape& s, const void* x, const float* router, int32_t* idx,
                         float* gate, int32_t* counts, float* prob_sum, void* ws,
                         cudaStream_t st) {
  const WsLayout L = ws_layout(s);
  uint8_t* w = static_cast<uint8_t*>(ws);
  uint32_t* status = reinterpret_cast<uint32_t*>(w + L.status);
  if (cudaMemsetAsync(counts, 0, sizeof(int32_t) * s.N, st) != cudaSuccess) return MOE_ERR_CUDA;
  float* Z = reinterpret_cast<float*>(w + L.scores);
  float* part = reinterpret_cast<float*>(w + L.prob_part);
  const int splits = router_k_splits(s);
  const int rc = launch_router_scores_tc(s, x, router, Z, splits, ws, st);
  if (rc != MOE_OK) return rc;
  const int nb = (s.T + kSelTokens - 1) / kSelTokens;
  // one group kept of one: plain top-K over all experts
  select_kernel<true><<<nb, 256, 0, st>>>(Z, splits, nullptr, s.T, s.N, s.K, 1, 1, idx, gate,
                                          counts, part, status);
  if (prob_sum != nullptr)
    prob_sum_kernel<<<(s.N + 31) / 32, 256, 0, st>>>(part, nb, s.N, prob_sum);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

}  // namespace moe
