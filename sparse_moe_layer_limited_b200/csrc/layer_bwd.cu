// Backward of COMBINE, of the gates and of DISPATCH: the steps around the
// expert backward (gemm_tc.cu, gemm_wgrad.cu) in the backward order
// COMBINE -> MLP_B -> MLP_W -> DISPATCH of the mhpq.cn article §2.2.
//
//   combine:   dy_perm[slot[t,k]] = gate[t,k] * dy_t,  dgate[t,k] = dy_t . y_perm[slot[t,k]]
//   gates:     with s = sigmoid(x e_i) (kaiyunto.com walk-through, DeepSeekMoE
//              paragraphs) and gate_k = s_k / S over the K selected experts,
//              dz_k = s_k (1 - s_k) (dgate_k - sum_j gate_j dgate_j) / S;
//              dx_route_t = sum_k dz_k e_{idx_k},  de_i = sum of dz x_t over
//              expert i's dispatched rows (the bias gets no gradient: it only
//              selects, gkm0120.cn reading notes Q3)
//   dispatch:  dx_t = dx_shared_t + sum_k dx_perm[slot[t,k]] (+ dx_route_t)
//
// Every sum runs in fp32 in a fixed order (k order, row order, a fixed
// shuffle tree), so the results are deterministic; no atomics.
#include <cuda_bf16.h>

#include "internal.h"

namespace moe {
namespace {

// V consecutive activations as fp32: bf16 moves 8 per 16-byte vector, fp32 4.
template <typename T>
struct Act;
template <>
struct Act<__nv_bfloat16> {
  static constexpr int V = 8;
  // one 16-byte vector as loaded, and its V values as fp32
  __device__ static uint4 raw(const __nv_bfloat16* p) {
    return __ldg(reinterpret_cast<const uint4*>(p));
  }
  __device__ static void cvt(const uint4& w, float* o) {
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&w);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = __bfloat1622float2(h[i]);
      o[2 * i] = f.x;
      o[2 * i + 1] = f.y;
    }
  }
  __device__ static void load(const __nv_bfloat16* p, float* o) {
    const uint4 w = __ldg(reinterpret_cast<const uint4*>(p));
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&w);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = __bfloat1622float2(h[i]);
      o[2 * i] = f.x;
      o[2 * i + 1] = f.y;
    }
  }
  __device__ static void store(__nv_bfloat16* p, const float* v) {
    uint4 w;
    __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&w);
#pragma unroll
    for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
    *reinterpret_cast<uint4*>(p) = w;
  }
  // 4 activations (8 bytes)
  __device__ static void load4(const __nv_bfloat16* p, float* o) {
    const uint2 w = __ldg(reinterpret_cast<const uint2*>(p));
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&w);
    const float2 a = __bfloat1622float2(h[0]), b = __bfloat1622float2(h[1]);
    o[0] = a.x;
    o[1] = a.y;
    o[2] = b.x;
    o[3] = b.y;
  }
};
template <>
struct Act<float> {
  static constexpr int V = 4;
  __device__ static uint4 raw(const float* p) { return __ldg(reinterpret_cast<const uint4*>(p)); }
  __device__ static void cvt(const uint4& w, float* o) {
    o[0] = __uint_as_float(w.x);
    o[1] = __uint_as_float(w.y);
    o[2] = __uint_as_float(w.z);
    o[3] = __uint_as_float(w.w);
  }
  __device__ static void load(const float* p, float* o) {
    const float4 w = __ldg(reinterpret_cast<const float4*>(p));
    o[0] = w.x;
    o[1] = w.y;
    o[2] = w.z;
    o[3] = w.w;
  }
  __device__ static void store(float* p, const float* v) {
    *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
  }
  __device__ static void load4(const float* p, float* o) { load(p, o); }
};

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// ---- COMBINE backward: one CTA of 128 threads per token -----------------------------
// KM > 0 (K <= KM): one pass over d; each thread loads its piece of dy_t once
// and of all K rows of y_perm before the multiply-adds (K loads in flight),
// and keeps the K partial dots.  KM = 0: one pass per k.  Each dgate_k is the
// same fixed reduction either way: this thread's multiply-adds in v order,
// then the warp's shuffle tree, then the four warps' sums in a fixed pairing.
template <typename T, int KM>
__global__ void __launch_bounds__(128) combine_bwd_kernel(
    const T* __restrict__ dy, const T* __restrict__ y_perm, const int32_t* __restrict__ slot,
    const float* __restrict__ gate, int ntok, int d, int K, T* __restrict__ dy_perm,
    float* __restrict__ dgate) {
  constexpr int V = Act<T>::V;
  __shared__ int ss[kMaxK];
  __shared__ float sg[kMaxK];
  __shared__ float red[4][KM > 0 ? KM : 1];
  const int t = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x < K) {
    const int r = slot[(size_t)t * K + threadIdx.x];
    const bool ok = r >= 0 && r < ntok * K;  // a slot outside the rows is skipped
    ss[threadIdx.x] = ok ? r : -1;
    sg[threadIdx.x] = ok ? gate[(size_t)t * K + threadIdx.x] : 0.f;
  }
  __syncthreads();
  const int nvec = d / V;
  const T* dyt = dy + (size_t)t * d;
  if constexpr (KM > 0) {
    int rk[KM];
    float part[KM];
#pragma unroll
    for (int k = 0; k < KM; ++k) {
      rk[k] = k < K ? ss[k] : -1;
      part[k] = 0.f;
    }
    for (int v = threadIdx.x; v < nvec; v += blockDim.x) {
      float a[V];
      uint4 braw[KM];
      Act<T>::load(dyt + v * V, a);
#pragma unroll
      for (int k = 0; k < KM; ++k)
        if (rk[k] >= 0) braw[k] = Act<T>::raw(y_perm + (size_t)rk[k] * d + v * V);
#pragma unroll
      for (int k = 0; k < KM; ++k) {
        if (rk[k] < 0) continue;
        const float g = sg[k];
        float b[V], o[V];
        Act<T>::cvt(braw[k], b);
#pragma unroll
        for (int i = 0; i < V; ++i) {
          part[k] = fmaf(a[i], b[i], part[k]);
          o[i] = g * a[i];
        }
        Act<T>::store(dy_perm + (size_t)rk[k] * d + v * V, o);
      }
    }
#pragma unroll
    for (int k = 0; k < KM; ++k) {
      const float w = warp_sum(part[k]);
      if (lane == 0) red[warp][k] = w;
    }
    __syncthreads();
    if (threadIdx.x < K) {
      const int k = threadIdx.x;
      dgate[(size_t)t * K + k] =
          ss[k] >= 0 ? (red[0][k] + red[1][k]) + (red[2][k] + red[3][k]) : 0.f;
    }
  } else {
    for (int k = 0; k < K; ++k) {
      const int r = ss[k];
      const float g = sg[k];
      float part = 0.f;
      if (r >= 0) {
        const T* yr = y_perm + (size_t)r * d;
        T* out = dy_perm + (size_t)r * d;
        for (int v = threadIdx.x; v < nvec; v += blockDim.x) {
          float a[V], b[V], o[V];
          Act<T>::load(dyt + v * V, a);
          Act<T>::load(yr + v * V, b);
#pragma unroll
          for (int i = 0; i < V; ++i) {
            part = fmaf(a[i], b[i], part);
            o[i] = g * a[i];
          }
          Act<T>::store(out + v * V, o);
        }
      }
      part = warp_sum(part);
      if (lane == 0) red[warp][0] = part;
      __syncthreads();
      if (threadIdx.x == 0)
        dgate[(size_t)t * K + k] =
            r >= 0 ? (red[0][0] + red[1][0]) + (red[2][0] + red[3][0]) : 0.f;
      __syncthreads();
    }
  }
}

// ---- gate backward per token: one warp per token ------------------------------------
// Lane k (k < K) holds the selected expert idx[t,k], its recomputed logit and
// affinity; the K dot products x_t . e_i and the output row run over d in
// 4-wide pieces, lanes interleaved (coalesced).  For K <= 8 the output row
// takes the K experts and their dz from lists built once, and each lane loads
// its pieces of all K router rows before the first multiply-add (the same
// k-order sums).
template <typename T>
__global__ void __launch_bounds__(256) route_bwd_token_kernel(
    const T* __restrict__ x, const float* __restrict__ R, const int32_t* __restrict__ idx,
    const float* __restrict__ dgate, int ntok, int d, int N, int K, float* __restrict__ dz_out,
    float* __restrict__ dx_route) {
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (t >= ntok) return;
  const T* xt = x + (size_t)t * d;
  int my_e = -1;
  float my_z = 0.f;
  for (int k = 0; k < K; ++k) {
    const int e = idx[(size_t)t * K + k];
    const bool ok = e >= 0 && e < N;  // warp-uniform
    float part = 0.f;
    if (ok) {
      const float* re = R + (size_t)e * d;
      for (int j = lane * 4; j < d; j += 128) {
        float xv[4];
        Act<T>::load4(xt + j, xv);
        const float4 rv = __ldg(reinterpret_cast<const float4*>(re + j));
        part = fmaf(xv[0], rv.x, part);
        part = fmaf(xv[1], rv.y, part);
        part = fmaf(xv[2], rv.z, part);
        part = fmaf(xv[3], rv.w, part);
      }
    }
    part = warp_sum(part);
    if (lane == k) {
      my_e = ok ? e : -1;
      my_z = part;
    }
  }
  const bool mine = lane < K && my_e >= 0;
  const float s = mine ? 1.f / (1.f + expf(-my_z)) : 0.f;
  const float S = fmaxf(warp_sum(s), 1e-30f);  // every affinity underflowed: dz = 0
  const float dg = mine ? dgate[(size_t)t * K + lane] : 0.f;
  const float gt = mine ? s / S : 0.f;
  const float m = warp_sum(gt * dg);
  const float dz = mine ? s * (1.f - s) * (dg - m) / S : 0.f;
  if (lane < K) dz_out[(size_t)t * K + lane] = dz;
  float* out = dx_route + (size_t)t * d;
  if (K <= 8) {
    int ek[8];
    float wk[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      ek[k] = __shfl_sync(0xffffffffu, my_e, k);
      wk[k] = __shfl_sync(0xffffffffu, dz, k);
      if (k >= K) ek[k] = -1;
    }
    for (int j = lane * 4; j < d; j += 128) {
      float4 rv[8];
#pragma unroll
      for (int k = 0; k < 8; ++k)
        if (ek[k] >= 0) rv[k] = __ldg(reinterpret_cast<const float4*>(R + (size_t)ek[k] * d + j));
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        if (ek[k] < 0) continue;
        acc.x = fmaf(wk[k], rv[k].x, acc.x);
        acc.y = fmaf(wk[k], rv[k].y, acc.y);
        acc.z = fmaf(wk[k], rv[k].z, acc.z);
        acc.w = fmaf(wk[k], rv[k].w, acc.w);
      }
      *reinterpret_cast<float4*>(out + j) = acc;
    }
    return;
  }
  for (int j0 = 0; j0 < d; j0 += 128) {  // the same trip count in every lane (shuffles)
    const int j = j0 + lane * 4;
    const bool in = j < d;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int k = 0; k < K; ++k) {
      const int e = __shfl_sync(0xffffffffu, my_e, k);
      const float w = __shfl_sync(0xffffffffu, dz, k);
      if (e < 0 || !in) continue;
      const float4 rv = __ldg(reinterpret_cast<const float4*>(R + (size_t)e * d + j));
      acc.x = fmaf(w, rv.x, acc.x);
      acc.y = fmaf(w, rv.y, acc.y);
      acc.z = fmaf(w, rv.z, acc.z);
      acc.w = fmaf(w, rv.w, acc.w);
    }
    if (in) *reinterpret_cast<float4*>(out + j) = acc;
  }
}

// ---- router-weight gradient: one CTA per (expert, 1024 columns) -----------------------
// The expert's dispatched rows are taken in row order, 128 at a time: each
// thread finds its row's token and that token's dz for this expert (the k with
// slot[t,k] = row), then every thread adds dz * x_t over its 8 columns.
constexpr int kRouterCols = 1024;

template <typename T>
__global__ void __launch_bounds__(128) route_bwd_router_kernel(
    const T* __restrict__ x, const int32_t* __restrict__ offsets,
    const int32_t* __restrict__ perm_tok, const int32_t* __restrict__ slot,
    const float* __restrict__ dz, int ntok, int d, int K, float* __restrict__ drouter) {
  __shared__ float sdz[128];
  __shared__ int stok[128];
  const int e = blockIdx.x;
  const int c0 = blockIdx.y * kRouterCols + threadIdx.x * 8;
  const int rows = ntok * K;
  const int r0 = min(max(offsets[e], 0), rows), r1 = min(max(offsets[e + 1], r0), rows);
  float acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = 0.f;
  for (int base = r0; base < r1; base += 128) {
    const int r = base + threadIdx.x;
    float w = 0.f;
    int tok = -1;
    if (r < r1) {
      const int t = perm_tok[r];
      if (t >= 0 && t < ntok) {
        for (int k = 0; k < K; ++k)
          if (slot[(size_t)t * K + k] == r) {
            w = dz[(size_t)t * K + k];
            tok = t;
          }
      }
    }
    sdz[threadIdx.x] = w;
    stok[threadIdx.x] = tok;
    __syncthreads();
    const int n = min(128, r1 - base);
    if (c0 < d) {
      for (int i = 0; i < n; ++i) {
        const int t = stok[i];
        if (t < 0) continue;
        const float a = sdz[i];
        float xv[8];
        Act<T>::load(x + (size_t)t * d + c0, xv);
        if constexpr (Act<T>::V == 4) Act<T>::load(x + (size_t)t * d + c0 + 4, xv + 4);
#pragma unroll
        for (int q = 0; q < 8; ++q) acc[q] = fmaf(a, xv[q], acc[q]);
      }
    }
    __syncthreads();
  }
  if (c0 < d) {
    float4* o = reinterpret_cast<float4*>(drouter + (size_t)e * d + c0);
    o[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
    o[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
  }
}

// ---- DISPATCH backward: one CTA of 128 threads per token ----------------------------
template <typename T>
__global__ void __launch_bounds__(128) dispatch_bwd_kernel(
    const T* __restrict__ dx_perm, const T* __restrict__ dx_sh, const int32_t* __restrict__ slot,
    const float* __restrict__ dx_route, int ntok, int d, int K, T* __restrict__ dx) {
  constexpr int V = Act<T>::V;
  __shared__ int ss[kMaxK];
  const int t = blockIdx.x;
  if (threadIdx.x < K) {
    const int r = slot[(size_t)t * K + threadIdx.x];
    ss[threadIdx.x] = (r >= 0 && r < ntok * K) ? r : -1;
  }
  __syncthreads();
  const int nvec = d / V;
  for (int v = threadIdx.x; v < nvec; v += blockDim.x) {
    float acc[V];
    Act<T>::load(dx_sh + (size_t)t * d + v * V, acc);
    for (int k = 0; k < K; ++k) {
      if (ss[k] < 0) continue;
      float r[V];
      Act<T>::load(dx_perm + (size_t)ss[k] * d + v * V, r);
#pragma unroll
      for (int i = 0; i < V; ++i) acc[i] += r[i];
    }
    if (dx_route != nullptr) {
      const float4* q = reinterpret_cast<const float4*>(dx_route + (size_t)t * d + v * V);
#pragma unroll
      for (int i = 0; i < V / 4; ++i) {
        const float4 w = __ldg(q + i);
        acc[4 * i] += w.x;
        acc[4 * i + 1] += w.y;
        acc[4 * i + 2] += w.z;
        acc[4 * i + 3] += w.w;
      }
    }
    Act<T>::store(dx + (size_t)t * d + v * V, acc);
  }
}

template <typename T>
cudaError_t combine_bwd(const moe_shape& s, const void* dy, const void* y_perm,
                        const int32_t* slot, const float* gate, void* dy_perm, float* dgate,
                        cudaStream_t st) {
  if (s.K <= 8)
    combine_bwd_kernel<T, 8><<<s.T, 128, 0, st>>>(static_cast<const T*>(dy),
                                                  static_cast<const T*>(y_perm), slot, gate, s.T,
                                                  s.d, s.K, static_cast<T*>(dy_perm), dgate);
  else
    combine_bwd_kernel<T, 0><<<s.T, 128, 0, st>>>(static_cast<const T*>(dy),
                                                  static_cast<const T*>(y_perm), slot, gate, s.T,
                                                  s.d, s.K, static_cast<T*>(dy_perm), dgate);
  return cudaGetLastError();
}

template <typename T>
cudaError_t route_bwd(const moe_shape& s, const void* x, const float* R, const int32_t* idx,
                      const float* dgate, const int32_t* offsets, const int32_t* perm_tok,
                      const int32_t* slot, float* dz, float* dx_route, float* drouter,
                      cudaStream_t st) {
  route_bwd_token_kernel<T><<<(s.T + 7) / 8, 256, 0, st>>>(static_cast<const T*>(x), R, idx,
                                                           dgate, s.T, s.d, s.N, s.K, dz,
                                                           dx_route);
  const dim3 grid((unsigned)s.N, (unsigned)((s.d + kRouterCols - 1) / kRouterCols));
  route_bwd_router_kernel<T><<<grid, 128, 0, st>>>(static_cast<const T*>(x), offsets, perm_tok,
                                                   slot, dz, s.T, s.d, s.K, drouter);
  return cudaGetLastError();
}

template <typename T>
cudaError_t dispatch_bwd(const moe_shape& s, const void* dx_perm, const void* dx_shared,
                         const int32_t* slot, const float* dx_route, void* dx, cudaStream_t st) {
  dispatch_bwd_kernel<T><<<s.T, 128, 0, st>>>(static_cast<const T*>(dx_perm),
                                              static_cast<const T*>(dx_shared), slot, dx_route,
                                              s.T, s.d, s.K, static_cast<T*>(dx));
  return cudaGetLastError();
}

}  // namespace

// Activations are fp32 in FP32 mode and bf16 otherwise (E4M3 mode keeps its
// layer input and outputs in bf16).
cudaError_t launch_combine_backward(const moe_shape& s, const void* dy, const void* y_perm,
                                    const int32_t* slot, const float* gate, void* dy_perm,
                                    float* dgate, cudaStream_t st) {
  return s.dtype == MOE_DTYPE_FP32
             ? combine_bwd<float>(s, dy, y_perm, slot, gate, dy_perm, dgate, st)
             : combine_bwd<__nv_bfloat16>(s, dy, y_perm, slot, gate, dy_perm, dgate, st);
}

cudaError_t launch_route_backward(const moe_shape& s, const void* x, const float* router_w,
                                  const int32_t* idx, const float* dgate, const int32_t* offsets,
                                  const int32_t* perm_tok, const int32_t* slot, float* dlogit,
                                  float* dx_route, float* drouter, cudaStream_t st) {
  return s.dtype == MOE_DTYPE_FP32
             ? route_bwd<float>(s, x, router_w, idx, dgate, offsets, perm_tok, slot, dlogit,
                                dx_route, drouter, st)
             : route_bwd<__nv_bfloat16>(s, x, router_w, idx, dgate, offsets, perm_tok, slot,
                                        dlogit, dx_route, drouter, st);
}

cudaError_t launch_dispatch_backward(const moe_shape& s, const void* dx_perm,
                                     const void* dx_shared, const int32_t* slot,
                                     const float* dx_route, void* dx, cudaStream_t st) {
  return s.dtype == MOE_DTYPE_FP32
             ? dispatch_bwd<float>(s, dx_perm, dx_shared, slot, dx_route, dx, st)
             : dispatch_bwd<__nv_bfloat16>(s, dx_perm, dx_shared, slot, dx_route, dx, st);
}

}  // namespace moe
