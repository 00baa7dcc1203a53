// Dispatch: deterministic grouping of the (token, expert) pairs by expert
// and the gather of x rows into expert order (the DISPATCH step of the
// forward order ATTN -> DISPATCH -> MLP -> COMBINE, mhpq.cn article §2.2; on
// one GPU it is a permutation, not an all-to-all).
//
// Row of (t, e) = offsets[e] + #{t' < t : t' chose e}.  Computed without
// atomics in three launches:
//   1. per 32-token chunk, a histogram of the chosen experts;
//   2. per expert (one CTA each), the exclusive prefix over experts of
//      counts[] and over chunks of that expert's histogram column;
//   3. per chunk, each pair's rank among the chunk's earlier tokens, the slot
//      and perm_tok writes, then the row gather: one warp per token reads x
//      once with 16-byte loads and writes it to its K destination rows
//      (E4M3 mode: quantised per 1x128 tile on the way, mhpq.cn §4.1).
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include <cstdlib>
#include <cstring>
#include <mutex>

#include "fp8_util.cuh"
#include "internal.h"
#include "ptx.cuh"

namespace moe {
namespace {

__global__ void __launch_bounds__(256) chunk_hist_kernel(const int32_t* __restrict__ idx, int T,
                                                         int K, int N,
                                                         int32_t* __restrict__ chunk_hist,
                                                         uint32_t* __restrict__ status) {
  __shared__ int h[kRouteMaxN];
  const int c = blockIdx.x;
  for (int e = threadIdx.x; e < N; e += blockDim.x) h[e] = 0;
  __syncthreads();
  const int t0 = c * kChunkTokens;
  const int nt = min(kChunkTokens, T - t0);
  for (int p = threadIdx.x; p < nt * K; p += blockDim.x) {
    const int e = idx[(size_t)t0 * K + p];
    if (e < 0 || e >= N)
      atomicOr(status, kErrBadIndex);
    else
      atomicAdd(&h[e], 1);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < N; e += blockDim.x) chunk_hist[(size_t)c * N + e] = h[e];
}

__device__ __forceinline__ int block_sum_256(int v, int* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  __syncthreads();
  if (l == 0) red[w] = v;
  __syncthreads();
  int s = 0;
  for (int i = 0; i < 8; ++i) s += red[i];
  return s;
}

// Exclusive scan of one int per thread over a 256-thread block.
__device__ __forceinline__ int block_exclusive_scan_256(int v, int* red) {
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  int inc = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int n = __shfl_up_sync(0xffffffffu, inc, o);
    if (l >= o) inc += n;
  }
  __syncthreads();
  if (l == 31) red[w] = inc;
  __syncthreads();
  int base = 0;
  for (int i = 0; i < w; ++i) base += red[i];
  return base + inc - v;
}

__global__ void __launch_bounds__(256) expert_scan_kernel(const int32_t* __restrict__ counts,
                                                          const int32_t* __restrict__ chunk_hist,
                                                          int nchunks, int N,
                                                          int32_t* __restrict__ offsets,
                                                          int32_t* __restrict__ chunk_base,
                                                          uint32_t* __restrict__ status) {
  __shared__ int red[8];
  const int e = blockIdx.x;
  int part = 0;
  for (int i = threadIdx.x; i < e; i += blockDim.x) part += counts[i];
  const int off_e = block_sum_256(part, red);

  const int per = (nchunks + blockDim.x - 1) / blockDim.x;
  const int c0 = threadIdx.x * per;
  const int c1 = min(nchunks, c0 + per);
  int mine = 0;
  for (int c = c0; c < c1; ++c) mine += chunk_hist[(size_t)c * N + e];
  int run = off_e + block_exclusive_scan_256(mine, red);
  for (int c = c0; c < c1; ++c) {
    chunk_base[(size_t)c * N + e] = run;
    run += chunk_hist[(size_t)c * N + e];
  }
  const int total = block_sum_256(mine, red);
  if (threadIdx.x == 0) {
    const int ce = counts[e];
    if (total != ce) atomicOr(status, kErrCountMismatch);
    offsets[e] = off_e;
    if (e == N - 1) offsets[N] = off_e + ce;
  }
}

// Rows of this chunk's (token, expert) pairs: rank among the chunk's earlier
// tokens that chose the same expert, plus the chunk's base row for that
// expert.  Writes slot[] and perm_tok[] and leaves the rows in sslot (-1 for
// a pair that cannot be placed, which only happens when counts[] disagree
// with idx; that is flagged by the histogram and scan kernels).
__device__ __forceinline__ void chunk_slots(const int32_t* __restrict__ idx,
                                            const int32_t* __restrict__ chunk_base, int c,
                                            int t0, int nt, int T, int K, int N,
                                            int32_t* __restrict__ perm_tok,
                                            int32_t* __restrict__ slot, int* sidx, int* sslot) {
  for (int p = threadIdx.x; p < nt * K; p += blockDim.x) sidx[p] = idx[(size_t)t0 * K + p];
  __syncthreads();
  for (int p = threadIdx.x; p < nt * K; p += blockDim.x) {
    const int tl = p / K;
    const int e = sidx[p];
    if (e < 0 || e >= N) {
      sslot[p] = -1;
      continue;
    }
    int rank = 0;
    for (int q = 0; q < tl * K; ++q) rank += (sidx[q] == e) ? 1 : 0;
    const int r = chunk_base[(size_t)c * N + e] + rank;
    if (r < 0 || r >= T * K) {
      sslot[p] = -1;
      continue;
    }
    sslot[p] = r;
    slot[(size_t)t0 * K + p] = r;
    perm_tok[r] = t0 + tl;
  }
  __syncthreads();
}

// Slots for one chunk, then the row gather (bf16 / fp32 rows copied verbatim;
// skipped when x_perm is null).
template <typename XT>
__global__ void __launch_bounds__(256) scatter_gather_kernel(
    const XT* __restrict__ x, const int32_t* __restrict__ idx,
    const int32_t* __restrict__ chunk_base, int T, int d, int K, int N,
    int32_t* __restrict__ perm_tok, int32_t* __restrict__ slot, XT* __restrict__ x_perm) {
  __shared__ int sidx[kChunkTokens * kMaxK];
  __shared__ int sslot[kChunkTokens * kMaxK];
  const int c = blockIdx.x;
  const int t0 = c * kChunkTokens;
  const int nt = min(kChunkTokens, T - t0);
  chunk_slots(idx, chunk_base, c, t0, nt, T, K, N, perm_tok, slot, sidx, sslot);
  if (x_perm == nullptr) return;  // slots only: the expert GEMM gathers the rows itself
  // gather: warp per token, 16-byte vectors, four loads in flight per lane
  constexpr int kElems = 16 / sizeof(XT);
  constexpr int kUnroll = 4;
  const int nvec = d / kElems;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int tl = warp; tl < nt; tl += 8) {
    const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)(t0 + tl) * d);
    for (int v0 = lane; v0 < nvec; v0 += 32 * kUnroll) {
      uint4 val[kUnroll];
#pragma unroll
      for (int j = 0; j < kUnroll; ++j) {
        const int v = v0 + 32 * j;
        if (v < nvec) val[j] = __ldg(src + v);
      }
      for (int k = 0; k < K; ++k) {
        const int r = sslot[tl * K + k];
        if (r < 0) continue;
        uint4* dst = reinterpret_cast<uint4*>(x_perm + (size_t)r * d);
#pragma unroll
        for (int j = 0; j < kUnroll; ++j) {
          const int v = v0 + 32 * j;
          if (v < nvec) dst[v] = val[j];
        }
      }
    }
  }
}

// E4M3 layer: slots as above, then each x row is quantised once per 1x128
// tile (a half-warp per tile) and its codes and scales are written to the
// token's K destination rows.  Scales: kStaged writes each destination row's
// scales contiguously into sc_rows ([T*K][sc_stride], eight tiles per pass as
// two 16-byte stores) for scale_rows_to_blocks_kernel to lay out block-major;
// otherwise they go straight to the block-major [d/128][sc_ld] array, one
// 4-byte store per tile and destination row.
template <bool kStaged>
__global__ void __launch_bounds__(256) scatter_gather_fp8_kernel(
    const __nv_bfloat16* __restrict__ x, const int32_t* __restrict__ idx,
    const int32_t* __restrict__ chunk_base, int T, int d, int K, int N,
    int32_t* __restrict__ perm_tok, int32_t* __restrict__ slot, uint8_t* __restrict__ x_perm,
    float* __restrict__ x_perm_scales, long long sc_ld, float* __restrict__ sc_rows,
    int sc_stride) {
  __shared__ int sidx[kChunkTokens * kMaxK];
  __shared__ int sslot[kChunkTokens * kMaxK];
  const int c = blockIdx.x;
  const int t0 = c * kChunkTokens;
  const int nt = min(kChunkTokens, T - t0);
  chunk_slots(idx, chunk_base, c, t0, nt, T, K, N, perm_tok, slot, sidx, sslot);
  const int tiles = d / QB;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int half = lane >> 4, l16 = lane & 15;
  constexpr int kUnroll = 4;  // tiles per half-warp per pass, their loads in flight together
  for (int tl = warp; tl < nt; tl += 8) {
    const __nv_bfloat16* src = x + (size_t)(t0 + tl) * d;
    for (int tc0 = 0; tc0 < tiles; tc0 += 2 * kUnroll) {  // eight tiles per warp pass
      float v[kUnroll][8];
#pragma unroll
      for (int j = 0; j < kUnroll; ++j) {
        const int tc = tc0 + 2 * j + half;
#pragma unroll
        for (int i = 0; i < 8; ++i) v[j][i] = 0.f;
        if (tc < tiles)
          bf16x8_to_f32(__ldg(reinterpret_cast<const uint4*>(src + tc * QB) + l16), v[j]);
      }
      float scs[kUnroll];  // this half-warp's tile scales (every lane of the half holds them)
#pragma unroll
      for (int j = 0; j < kUnroll; ++j) {
        const int tc = tc0 + 2 * j + half;
        uint2 codes;
        scs[j] = quant_tile_16lanes(v[j], codes);  // both halves take part
        if (tc >= tiles) continue;
        for (int k = 0; k < K; ++k) {
          const int r = sslot[tl * K + k];
          if (r < 0) continue;
          *reinterpret_cast<uint2*>(x_perm + (size_t)r * d + tc * QB + 8 * l16) = codes;
          if (!kStaged && l16 == 0) x_perm_scales[(size_t)tc * sc_ld + r] = scs[j];
        }
      }
      if constexpr (kStaged) {
        // lane 0 writes the pass's eight scales (tiles tc0..tc0+7, half 0 holding
        // the even ones, half 1 the odd ones) of every destination row; entries
        // past the last tile land in the row's padding
        float odd[kUnroll];
#pragma unroll
        for (int j = 0; j < kUnroll; ++j) odd[j] = __shfl_sync(0xffffffffu, scs[j], 16);
        if (lane == 0) {
          for (int k = 0; k < K; ++k) {
            const int r = sslot[tl * K + k];
            if (r < 0) continue;
            float4* dst = reinterpret_cast<float4*>(sc_rows + (size_t)r * sc_stride + tc0);
            dst[0] = make_float4(scs[0], odd[0], scs[1], odd[1]);
            dst[1] = make_float4(scs[2], odd[2], scs[3], odd[3]);
          }
        }
      }
    }
  }
}

// sc_rows [rows][stride] -> out [tiles][ld] (block-major), 32 x 32 tiles
// through shared memory.
__global__ void __launch_bounds__(256) scale_rows_to_blocks_kernel(
    const float* __restrict__ rows, int stride, long long nrows, int tiles,
    float* __restrict__ out, long long ld) {
  __shared__ float t[32][33];
  const long long r0 = (long long)blockIdx.x * 32;
  const int c0 = blockIdx.y * 32;
  for (int i = threadIdx.y; i < 32; i += 8) {
    const long long r = r0 + i;
    const int c = c0 + threadIdx.x;
    t[i][threadIdx.x] = (r < nrows && c < tiles) ? rows[r * stride + c] : 0.f;
  }
  __syncthreads();
  for (int i = threadIdx.y; i < 32; i += 8) {
    const int c = c0 + i;
    const long long r = r0 + threadIdx.x;
    if (c < tiles && r < nrows) out[(long long)c * ld + r] = t[threadIdx.x][i];
  }
}

// MOE_FP8_SCALES=direct writes the dispatch's E4M3 scales straight to the
// block-major array (read once per process); the default stages them per row
bool fp8_scales_direct() {
  static int v = -1;
  if (v < 0) {
    const char* e = std::getenv("MOE_FP8_SCALES");
    v = (e != nullptr && std::strcmp(e, "direct") == 0) ? 1 : 0;
  }
  return v == 1;
}

}  // namespace

cudaError_t launch_dispatch(const moe_shape& s, const void* x, const int32_t* idx,
                            const int32_t* counts, int32_t* offsets, int32_t* perm_tok,
                            int32_t* slot, void* x_perm, float* x_perm_scales, void* ws,
                            cudaStream_t st) {
  const WsLayout L = ws_layout(s);
  uint8_t* w = static_cast<uint8_t*>(ws);
  uint32_t* status = reinterpret_cast<uint32_t*>(w + L.status);
  int32_t* chunk_hist = reinterpret_cast<int32_t*>(w + L.chunk_hist);
  int32_t* chunk_base = reinterpret_cast<int32_t*>(w + L.chunk_base);
  const int nch = chunks_of(s.T);
  chunk_hist_kernel<<<nch, 256, 0, st>>>(idx, s.T, s.K, s.N, chunk_hist, status);
  expert_scan_kernel<<<s.N, 256, 0, st>>>(counts, chunk_hist, nch, s.N, offsets, chunk_base,
                                          status);
  if (s.dtype == MOE_DTYPE_FP32)
    scatter_gather_kernel<float><<<nch, 256, 0, st>>>(
        static_cast<const float*>(x), idx, chunk_base, s.T, s.d, s.K, s.N, perm_tok, slot,
        static_cast<float*>(x_perm));
  else if (s.dtype == MOE_DTYPE_BF16)
    scatter_gather_kernel<__nv_bfloat16><<<nch, 256, 0, st>>>(
        static_cast<const __nv_bfloat16*>(x), idx, chunk_base, s.T, s.d, s.K, s.N, perm_tok,
        slot, static_cast<__nv_bfloat16*>(x_perm));
  else {
    const long long TK = (long long)s.T * s.K;
    const int tiles = s.d / QB;
    const int stride = (tiles + 7) / 8 * 8;
    float* sc_rows = reinterpret_cast<float*>(w + L.sc_rows);
    if (fp8_scales_direct()) {
      scatter_gather_fp8_kernel<false><<<nch, 256, 0, st>>>(
          static_cast<const __nv_bfloat16*>(x), idx, chunk_base, s.T, s.d, s.K, s.N, perm_tok,
          slot, static_cast<uint8_t*>(x_perm), x_perm_scales, scale_ld(TK), nullptr, stride);
    } else {
      scatter_gather_fp8_kernel<true><<<nch, 256, 0, st>>>(
          static_cast<const __nv_bfloat16*>(x), idx, chunk_base, s.T, s.d, s.K, s.N, perm_tok,
          slot, static_cast<uint8_t*>(x_perm), x_perm_scales, scale_ld(TK), sc_rows, stride);
      scale_rows_to_blocks_kernel<<<dim3((unsigned)((TK + 31) / 32), (unsigned)((tiles + 31) / 32)),
                                    dim3(32, 8), 0, st>>>(sc_rows, stride, TK, tiles,
                                                          x_perm_scales, scale_ld(TK));
    }
  }
  return cudaGetLastError();
}

}  // namespace moe

// ---------------------------------------------------------------------------
// Dispatch without a caller-provided workspace.
//
// For callers that cannot allocate device memory at call time (code running
// inside a framework's allocator-free region, or a plugin host that hands
// over only its input and output buffers), moe_dispatch_noalloc keeps the
// three scratch regions of the dispatch (status word, per-chunk histograms,
// per-chunk bases) in one fixed static device array of this file instead of
// the caller's workspace.  The array is kNoAllocScratchBytes long (1 MiB of
// tables plus the 256-byte status word, so T = 16384 fits at N = 256) and
// lives on every GPU that loads the library until the process exits; shapes
// that need more are rejected.  Host code cannot pass the array's name to a
// kernel (on the host it is only a stand-in symbol), so its device address
// is looked up with cudaGetSymbolAddress once per device, with that device
// current, on the first call there.
namespace moe {
namespace {

constexpr size_t kNoAllocStatusBytes = 256;
constexpr size_t kNoAllocScratchBytes = ((size_t)1 << 20) + kNoAllocStatusBytes;
constexpr int kNoAllocMaxDevices = 64;

static __device__ __align__(256) uint8_t g_dispatch_scratch[kNoAllocScratchBytes];

std::mutex g_scratch_mu;
void* g_scratch_ptr[kNoAllocMaxDevices] = {};

// Device address of g_dispatch_scratch on the current device (nullptr on error).
void* scratch_on_current_device() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kNoAllocMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_dispatch_scratch) != cudaSuccess) return nullptr;
    g_scratch_ptr[dev] = p;
  }
  return g_scratch_ptr[dev];
}

size_t noalloc_scratch_need(const moe_shape& s) {
  const size_t table = (size_t)chunks_of(s.T) * s.N * sizeof(int32_t);
  return kNoAllocStatusBytes + 2 * ((table + 255) & ~size_t(255));
}

}  // namespace
}  // namespace moe

extern "C" int moe_dispatch_noalloc(const moe_shape* shape, const void* x,
                                    const int32_t* topk_idx, const int32_t* counts,
                                    int32_t* offsets, int32_t* perm_tok, int32_t* slot,
                                    void* x_perm, float* x_perm_scales, void* stream) {
  using namespace moe;
  const int rc = moe_check_shape(shape);
  if (rc != MOE_OK) return rc;
  const moe_shape& s = *shape;
  auto ok16 = [](const void* p) {
    return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 15u) == 0;
  };
  if (!ok16(x) || !ok16(topk_idx) || !ok16(counts) || !ok16(offsets) || !ok16(perm_tok) ||
      !ok16(slot))
    return MOE_ERR_ARG;
  // as in moe_dispatch, x_perm may be NULL: offsets, perm_tok and slot only
  if (x_perm != nullptr && !ok16(x_perm)) return MOE_ERR_ARG;
  if (s.dtype == MOE_DTYPE_E4M3) return MOE_ERR_UNSUPPORTED;
  if (noalloc_scratch_need(s) > kNoAllocScratchBytes) return MOE_ERR_WORKSPACE;
  (void)x_perm_scales;

  uint8_t* base = static_cast<uint8_t*>(scratch_on_current_device());
  if (!base) return MOE_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t table = ((size_t)chunks_of(s.T) * s.N * sizeof(int32_t) + 255) & ~size_t(255);
  uint32_t* status = reinterpret_cast<uint32_t*>(base);
  int32_t* chunk_hist = reinterpret_cast<int32_t*>(base + kNoAllocStatusBytes);
  int32_t* chunk_base = reinterpret_cast<int32_t*>(base + kNoAllocStatusBytes + table);
  // the status word accumulates bits: start each call from zero (the tables are
  // fully rewritten by the kernels below)
  if (cudaMemsetAsync(status, 0, sizeof(uint32_t), st) != cudaSuccess) return MOE_ERR_CUDA;
  const int nch = chunks_of(s.T);
  chunk_hist_kernel<<<nch, 256, 0, st>>>(topk_idx, s.T, s.K, s.N, chunk_hist, status);
  expert_scan_kernel<<<s.N, 256, 0, st>>>(counts, chunk_hist, nch, s.N, offsets, chunk_base,
                                          status);
  if (s.dtype == MOE_DTYPE_FP32)
    scatter_gather_kernel<float><<<nch, 256, 0, st>>>(
        static_cast<const float*>(x), topk_idx, chunk_base, s.T, s.d, s.K, s.N, perm_tok, slot,
        static_cast<float*>(x_perm));
  else
    scatter_gather_kernel<__nv_bfloat16><<<nch, 256, 0, st>>>(
        static_cast<const __nv_bfloat16*>(x), topk_idx, chunk_base, s.T, s.d, s.K, s.N,
        perm_tok, slot, static_cast<__nv_bfloat16*>(x_perm));
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
