// fp32 SwiGLU experts on CUDA cores (the fp32 layer: tensor-core tf32 would
// not meet an fp32 tolerance).  Same grouping as the tensor-core path: rows
// 0..T*K-1 are the dispatched rows of the routed experts (expert found from
// offsets[]), rows T*K..T*K+T-1 are the shared expert (index N) on x.
//   kernel 1: H[r, j] = silu(a_r . W1[e][j]) * (a_r . W3[e][j])
//   kernel 2: Y[r, c] = H[r, :] . W2[e][c, :]
// One thread per output element, fp32 accumulation in index order.
#include "internal.h"

namespace moe {
namespace {

__device__ __forceinline__ int expert_of_row(const int32_t* offsets, int N, int r) {
  int lo = 0, hi = N;  // largest e with offsets[e] <= r
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (offsets[mid] <= r) lo = mid; else hi = mid;
  }
  return lo;
}

__global__ void gemm1_swiglu_f32(const float* __restrict__ x_perm,
                                 const int32_t* __restrict__ offsets,
                                 const float* __restrict__ x, const float* __restrict__ w13,
                                 int T, int d, int N, int K, int f, int P,
                                 float* __restrict__ H) {
  const long long TK = (long long)T * K;
  const long long total = (TK + T) * f;
  for (long long q = (long long)blockIdx.x * blockDim.x + threadIdx.x; q < total;
       q += (long long)gridDim.x * blockDim.x) {
    const long long r = q / f;
    const int j = (int)(q - r * f);
    int e;
    const float* a;
    if (r < TK) {
      e = expert_of_row(offsets, N, (int)r);
      a = x_perm + r * d;
    } else {
      e = N;
      a = x + (r - TK) * d;
    }
    const int blk = j / P, within = j % P;
    const float* w1 = w13 + ((size_t)e * 2 * f + (size_t)blk * 2 * P + within) * d;
    const float* w3 = w1 + (size_t)P * d;
    float g = 0.f, u = 0.f;
    for (int c = 0; c < d; ++c) {
      g = fmaf(a[c], w1[c], g);
      u = fmaf(a[c], w3[c], u);
    }
    H[q] = g / (1.f + expf(-g)) * u;
  }
}

__global__ void gemm2_f32(const float* __restrict__ H, const int32_t* __restrict__ offsets,
                          const float* __restrict__ w2, int T, int d, int N, int K, int f,
                          float* __restrict__ y_perm, float* __restrict__ y_shared) {
  const long long TK = (long long)T * K;
  const long long total = (TK + T) * d;
  for (long long q = (long long)blockIdx.x * blockDim.x + threadIdx.x; q < total;
       q += (long long)gridDim.x * blockDim.x) {
    const long long r = q / d;
    const int c = (int)(q - r * d);
    const int e = (r < TK) ? expert_of_row(offsets, N, (int)r) : N;
    const float* h = H + r * f;
    const float* w = w2 + ((size_t)e * d + c) * f;
    float acc = 0.f;
    for (int j = 0; j < f; ++j) acc = fmaf(h[j], w[j], acc);
    if (r < TK)
      y_perm[r * d + c] = acc;
    else
      y_shared[(r - TK) * d + c] = acc;
  }
}

}  // namespace

cudaError_t launch_ffn_simt(const moe_shape& s, const float* x_perm, const int32_t* offsets,
                            const float* x, const float* w13, const float* w2, float* y_perm,
                            float* y_shared, void* ws, cudaStream_t st) {
  const WsLayout L = ws_layout(s);
  float* H = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + L.h);
  const long long rows = (long long)s.T * s.K + s.T;
  long long b1 = (rows * s.f + 255) / 256, b2 = (rows * s.d + 255) / 256;
  if (b1 > 148 * 32) b1 = 148 * 32;
  if (b2 > 148 * 32) b2 = 148 * 32;
  gemm1_swiglu_f32<<<(int)b1, 256, 0, st>>>(x_perm, offsets, x, w13, s.T, s.d, s.N, s.K, s.f,
                                            pack_block(s.f), H);
  gemm2_f32<<<(int)b2, 256, 0, st>>>(H, offsets, w2, s.T, s.d, s.N, s.K, s.f, y_perm, y_shared);
  return cudaGetLastError();
}

}  // namespace moe
