// Grouped bf16 GEMMs on the 5th-generation tensor cores: the SwiGLU expert
// GEMMs and the router score GEMM.
//
// The experts are FFNs (mhpq.cn article §1.1; wenxiaobai §二(一)4) in the
// SwiGLU form y = (silu(a W1^T) * (a W3^T)) W2^T; the routed experts run on
// their dispatched rows and the shared expert on every token, all in one
// persistent launch per GEMM:
//   GEMM1  H[rows_g, f] = SwiGLU of [rows_g, d] x [d, 2f]   (bf16 out)
//   GEMM2  Y[rows_g, d] = [rows_g, f] x [f, d]             (bf16 out)
// Group g < N is routed expert g (rows offsets[g]..offsets[g+1]); group N is
// the shared expert (T rows).
//
// Orientation: the weights are the MMA's M side and the tokens its N side
// (D^T = W . A^T).  A tile is 256 weight rows (two tcgen05.mma M=128 halves
// into two TMEM column ranges) by up to 128 token rows; the token count of a
// tile is rounded up to a multiple of 16 only, so the ragged last tile of an
// expert costs MMA work in proportion to its rows (a 128-row M tile over the
// tokens would waste about a quarter of the routed work at ~256 rows per
// expert).  In GEMM1 the packed weight rows hold, per 128-row block j, W1
// rows then W3 rows, so TMEM lane i of the two halves holds the gate and the
// up projection of the same hidden feature: SwiGLU needs no data exchange.
//
// Work units are ordered group-major, then weight tile, then token tile, so
// CTAs running side by side read the same weight tile (one HBM read, the
// rest from L2).  Each CTA (one per SM) walks units blockIdx.x, +gridDim.x,
// ... with three roles:
//   warp 0    one thread issues TMA loads (128-byte swizzle) of 64-wide K
//             slices: 256 weight rows + 128 token rows per stage, 4 stages;
//   warp 1    allocates 512 TMEM columns (two 256-column accumulators) and
//             one thread issues the MMAs (K=16 each), committing each ring
//             slot back to the producer and each accumulator to the epilogue;
//   warps 2-5 drain an accumulator with tcgen05.ld (thread = weight row,
//             32 token columns per load) while the next unit accumulates in
//             the other buffer, apply the epilogue and store: consecutive
//             lanes write consecutive output features of one token row.
// The producer also prefetches each weight K block into L2 a few blocks
// ahead of its shared-memory load, so the first CTA on a weight tile does not
// stall on HBM latency with only four stages in flight.
// Every mbarrier wait is bounded (~2 s); a wait that gives up sets the
// device status word and the CTA unwinds, frees its TMEM and returns.
//
// The same kernel computes the router scores z = x . e_i (one group of T
// token rows; the "weights" are the experts): the fp32 router matrix is
// split exactly into three bf16 parts R = R0 + R1 + R2 (R0 = bf16(R),
// R1 = bf16(R - R0), R2 = bf16(R - R0 - R1), residual below 2^-27 |R|),
// stored as one [N, 3d] operand whose 64-column blocks run (R0, R1, R2) per
// 64 columns of d; each token tile of x serves three consecutive K blocks
// (x_rep = 3), so the fp32 accumulator receives x.R0 + x.R1 + x.R2 = x.R.
// The sigmoid epilogue writes s = sigmoid(z) as fp32 [T, N].
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>

#include <mutex>

#include "internal.h"
#include "ptx.cuh"

namespace moe {
namespace {

constexpr int BW = 256;   // weight rows per unit (two M=128 MMAs)
constexpr int BT = 128;   // token rows per unit (MMA N <= 128)
constexpr int BK = 64;    // bf16 K slice: 128 bytes = one swizzle row
constexpr int kStages = 4;
constexpr int kWBytes = BW * BK * 2;         // 32 KB
constexpr int kXBytes = BT * BK * 2;         // 16 KB
constexpr int kStageBytes = kWBytes + kXBytes;
constexpr int kAccCols = 256;                // per accumulator: 2 halves x 128 token columns
constexpr int kTmemCols = 2 * kAccCols;
constexpr int kThreads = 192;
constexpr int kPrefetchAhead = 8;  // weight K blocks brought into L2 ahead of their load
constexpr uint64_t kTimeoutNs = 2000000000ull;

enum Epi { kEpiSwiGLU = 0, kEpiStore = 1, kEpiSigmoid = 2 };

struct alignas(64) GemmArgs {
  CUtensorMap tmW;          // weights [(groups) * n_feat rows, k_dim], box {64, 256}
  CUtensorMap tmX_routed;   // token rows of routed groups, box {64, 128}
  CUtensorMap tmX_shared;   // token rows of the shared group
  const int32_t* offsets;
  __nv_bfloat16* out_routed;  // row (offsets[g] + r)
  __nv_bfloat16* out_shared;  // row r
  float* out_f32;             // sigmoid epilogue: [T, n_valid]
  uint32_t* status;
  int N, T;
  int rows_routed;    // T*K
  int x_shared_row0;  // first token row of the shared group in tmX_shared
  int n_feat;         // weight rows per group (2f for GEMM1, d for GEMM2)
  int k_dim;          // contraction length of the weight operand
  int x_rep;          // K blocks served by one token tile (3 for the split router)
  int out_ld;         // output row stride (elements)
  int n_valid;        // sigmoid epilogue: experts to store
};

constexpr size_t smem_bytes_for(int groups) {
  return 1024 + (size_t)kStages * kStageBytes + 256 + (size_t)(groups + 1) * 4;
}

__device__ __forceinline__ float silu_f(float v) { return v / (1.f + expf(-v)); }

template <int kEpi>
__global__ void __launch_bounds__(kThreads, 1) grouped_gemm_bf16_kernel(
    const __grid_constant__ GemmArgs args) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + (size_t)kStages * kStageBytes);
  uint64_t* full = bars;                 // [kStages]
  uint64_t* empty = bars + kStages;      // [kStages]
  uint64_t* tfull = bars + 2 * kStages;  // [2]
  uint64_t* tempty = tfull + 2;          // [2]
  uint64_t* drain = tempty + 2;          // [1]
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
  int* unit_start = reinterpret_cast<int*>(base + (size_t)kStages * kStageBytes + 256);

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int G1 = args.N + 1;
  const int NF = args.n_feat / BW;   // weight tiles per group (router: 1)
  const int KB = args.k_dim / BK;

  // ---- set-up: barriers, TMEM, unit schedule --------------------------------
  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 4);
    }
    mbar_init(drain, 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, kTmemCols);
    tmem_relinquish();
  }
  for (int g = tid; g < G1; g += kThreads) {
    const int rows = (g < args.N) ? args.offsets[g + 1] - args.offsets[g] : args.T;
    unit_start[g] = rows > 0 ? (rows + BT - 1) / BT : 0;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) {  // exclusive scan of token tiles per group, times NF
    const int per = (G1 + 31) / 32;
    const int g0 = min(G1, lane * per), g1 = min(G1, g0 + per);
    int sum = 0;
    for (int g = g0; g < g1; ++g) sum += unit_start[g];
    int inc = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, inc, o);
      if (lane >= o) inc += v;
    }
    int run = inc - sum;
    for (int g = g0; g < g1; ++g) {
      const int mt = unit_start[g];
      unit_start[g] = run * NF;
      run += mt;
    }
    if (lane == 31) unit_start[G1] = inc * NF;
  }
  __syncthreads();
  const uint32_t tmem_base = *tmem_holder;
  const int total = unit_start[G1];

  // unit -> (group g, weight tile nf, token tile mt, token tiles of g)
  auto decode = [&](int u, int& g, int& nf, int& mt) {
    int lo = 0, hi = G1;
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (unit_start[mid] <= u) lo = mid; else hi = mid;
    }
    g = lo;
    const int tiles = (unit_start[g + 1] - unit_start[g]) / NF;
    const int local = u - unit_start[g];
    nf = local / tiles;
    mt = local - nf * tiles;
  };
  auto group_rows = [&](int g) {
    return (g < args.N) ? args.offsets[g + 1] - args.offsets[g] : args.T;
  };

  if (warp == 0) {
    // ---- TMA producer ---------------------------------------------------------
    if (lane == 0) {
      tma_prefetch_desc(&args.tmW);
      tma_prefetch_desc(&args.tmX_routed);
      tma_prefetch_desc(&args.tmX_shared);
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued = 0, issued_parity = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < total && ok; u += gridDim.x) {
        int g, nf, mt;
        decode(u, g, nf, mt);
        const CUtensorMap* xm = (g < args.N) ? &args.tmX_routed : &args.tmX_shared;
        const int xrow = ((g < args.N) ? args.offsets[g] : args.x_shared_row0) + mt * BT;
        const int wrow = g * args.n_feat + nf * BW;
        // the first CTA to reach a weight tile misses L2 on every K block; an
        // L2 prefetch a few blocks ahead turns those misses into hits
        for (int kb = 0; kb < min(kPrefetchAhead, KB); ++kb)
          tma_prefetch_l2_2d(&args.tmW, kb * BK, wrow);
        for (int kb = 0; kb < KB; ++kb) {
          if (kb + kPrefetchAhead < KB)
            tma_prefetch_l2_2d(&args.tmW, (kb + kPrefetchAhead) * BK, wrow);
          if (!mbar_wait_bounded(&empty[stage], phase ^ 1u, args.status, kTimeoutNs)) {
            ok = false;
            break;
          }
          uint8_t* sw = base + (size_t)stage * kStageBytes;
          mbar_arrive_expect_tx(&full[stage], kStageBytes);
          tma_load_2d(sw, &args.tmW, kb * BK, wrow, &full[stage]);
          tma_load_2d(sw + kWBytes, xm, (kb / args.x_rep) * BK, xrow, &full[stage]);
          issued |= 1u << stage;
          issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {  // let the copies already issued land before the CTA exits
        for (int s = 0; s < kStages; ++s)
          if ((issued >> s) & 1u)
            mbar_wait_bounded(&full[s], (issued_parity >> s) & 1u, args.status, kTimeoutNs / 8);
      }
    }
  } else if (warp == 1) {
    // ---- MMA issuer -----------------------------------------------------------
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int local = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < total && ok; u += gridDim.x, ++local) {
        int g, nf, mt;
        decode(u, g, nf, mt);
        const int ntok = min(BT, group_rows(g) - mt * BT);
        const int n_mma = (ntok + 15) & ~15;
        const uint32_t idesc = idesc_bf16_f32(128, n_mma);
        const int acc = local & 1;
        const uint32_t aphase = (local >> 1) & 1;
        if (!mbar_wait_bounded(&tempty[acc], aphase ^ 1u, args.status, kTimeoutNs)) break;
        tc_fence_after();
        const uint32_t d0 = tmem_base + acc * kAccCols;
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait_bounded(&full[stage], phase, args.status, kTimeoutNs)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t w0 = smem_u32(base + (size_t)stage * kStageBytes);
          const uint32_t x0 = w0 + kWBytes;
#pragma unroll
          for (int k = 0; k < BK / 16; ++k) {
            const uint64_t xd = smem_desc_sw128(x0 + k * 32);
            mma_bf16(d0, smem_desc_sw128(w0 + k * 32), xd, idesc, (kb | k) != 0);
            mma_bf16(d0 + 128, smem_desc_sw128(w0 + kWBytes / 2 + k * 32), xd, idesc,
                     (kb | k) != 0);
          }
          mma_commit(&empty[stage]);
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (ok) mma_commit(&tfull[acc]);
      }
      mma_commit(drain);
      mbar_wait_bounded(drain, 0, args.status, kTimeoutNs / 8);
    }
  } else {
    // ---- epilogue: warps 2..5 --------------------------------------------------
    const int q = warp & 3;      // TMEM lane quadrant this warp may access
    const int j = q * 32 + lane; // weight row within each 128-row half
    int local = 0;
    for (int u = blockIdx.x; u < total; u += gridDim.x, ++local) {
      int g, nf, mt;
      decode(u, g, nf, mt);
      const int acc = local & 1;
      const uint32_t aphase = (local >> 1) & 1;
      if (!mbar_wait_bounded(&tfull[acc], aphase, args.status, kTimeoutNs)) break;
      tc_fence_after();
      const int ntok = min(BT, group_rows(g) - mt * BT);
      // output row of the unit's first token
      const long long row0 =
          (g < args.N) ? (long long)args.offsets[g] + mt * BT : (long long)mt * BT;
      const bool in_range =
          (g == args.N) || (args.offsets[g] >= 0 && row0 + ntok <= args.rows_routed);
      const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + acc * kAccCols;
#pragma unroll 1
      for (int c = 0; c < ntok; c += 32) {
        uint32_t v0[32], v1[32];
        tmem_ld32(taddr + c, v0);
        tmem_ld32(taddr + 128 + c, v1);
        tmem_wait_ld();
        if (!in_range) continue;
        if constexpr (kEpi == kEpiSwiGLU) {
          __nv_bfloat16* o = ((g < args.N) ? args.out_routed : args.out_shared) +
                             (row0 + c) * args.out_ld + nf * 128 + j;
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (c + i < ntok)
              o[(long long)i * args.out_ld] = __float2bfloat16_rn(
                  silu_f(__uint_as_float(v0[i])) * __uint_as_float(v1[i]));
        } else if constexpr (kEpi == kEpiStore) {
          __nv_bfloat16* o = ((g < args.N) ? args.out_routed : args.out_shared) +
                             (row0 + c) * args.out_ld + nf * BW + j;
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (c + i < ntok) {
              o[(long long)i * args.out_ld] = __float2bfloat16_rn(__uint_as_float(v0[i]));
              o[(long long)i * args.out_ld + 128] = __float2bfloat16_rn(__uint_as_float(v1[i]));
            }
        } else {  // sigmoid scores, fp32, experts < n_valid
          float* o = args.out_f32 + (row0 + c) * args.n_valid;
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (c + i < ntok) {
              if (j < args.n_valid)
                o[(long long)i * args.n_valid + j] =
                    1.f / (1.f + expf(-__uint_as_float(v0[i])));
              if (128 + j < args.n_valid)
                o[(long long)i * args.n_valid + 128 + j] =
                    1.f / (1.f + expf(-__uint_as_float(v1[i])));
            }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[acc]);
    }
  }

  // ---- teardown ------------------------------------------------------------------
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

// ---- host side -----------------------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 2-D row-major tensor [rows, inner] with a (box_inner x box_rows) box and
// the 128-byte swizzle; out-of-range rows read as zero.
bool make_map(CUtensorMap* map, const void* ptr, CUtensorMapDataType dt, size_t elem_bytes,
              uint64_t inner, uint64_t rows, uint32_t box_inner, uint32_t box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {inner * elem_bytes};
  cuuint32_t box[2] = {box_inner, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, dt, 2, const_cast<void*>(ptr), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

int num_sms() {
  static int n = 0;
  if (n == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

template <int kEpi>
cudaError_t launch_gemm(const GemmArgs& a, cudaStream_t st) {
  const size_t smem = smem_bytes_for(a.N + 1);
  cudaError_t e = cudaFuncSetAttribute(grouped_gemm_bf16_kernel<kEpi>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  grouped_gemm_bf16_kernel<kEpi><<<num_sms(), kThreads, smem, st>>>(a);
  return cudaGetLastError();
}

// R fp32 [N, d] -> three exact bf16 parts laid out [N, 3d] as described at
// the top of this file.
__global__ void router_split_kernel(const float* __restrict__ R, int N, int d,
                                    __nv_bfloat16* __restrict__ Rs) {
  const long long total = (long long)N * d;
  for (long long q = (long long)blockIdx.x * blockDim.x + threadIdx.x; q < total;
       q += (long long)gridDim.x * blockDim.x) {
    const long long n = q / d;
    const int c = (int)(q - n * d);
    const float v = R[q];
    const __nv_bfloat16 p0 = __float2bfloat16_rn(v);
    const float r1 = __fsub_rn(v, __bfloat162float(p0));
    const __nv_bfloat16 p1 = __float2bfloat16_rn(r1);
    const float r2 = __fsub_rn(r1, __bfloat162float(p1));
    const __nv_bfloat16 p2 = __float2bfloat16_rn(r2);
    const int cb = c / BK, i = c % BK;
    __nv_bfloat16* row = Rs + n * 3LL * d + (long long)(3 * cb) * BK + i;
    row[0] = p0;
    row[BK] = p1;
    row[2 * BK] = p2;
  }
}

}  // namespace

int launch_ffn_tc_bf16(const moe_shape& s, const void* x_perm, const int32_t* offsets,
                       const void* x, const void* w13, const void* w2, void* y_perm,
                       void* y_shared, void* ws, cudaStream_t st) {
  const WsLayout L = ws_layout(s);
  uint8_t* w = static_cast<uint8_t*>(ws);
  __nv_bfloat16* H = reinterpret_cast<__nv_bfloat16*>(w + L.h);
  const uint64_t TK = (uint64_t)s.T * s.K;
  const auto BF = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  uint32_t* status = reinterpret_cast<uint32_t*>(w + L.status);

  // GEMM1: weights W13 [(N+1)*2f, d], tokens x_perm (routed) / x (shared)
  GemmArgs g1{};
  bool ok = make_map(&g1.tmW, w13, BF, 2, s.d, (uint64_t)(s.N + 1) * 2 * s.f, BK, BW) &&
            make_map(&g1.tmX_routed, x_perm, BF, 2, s.d, TK, BK, BT) &&
            make_map(&g1.tmX_shared, x, BF, 2, s.d, s.T, BK, BT);
  if (!ok) return MOE_ERR_CUDA;
  g1.offsets = offsets;
  g1.out_routed = H;
  g1.out_shared = H + TK * s.f;
  g1.status = status;
  g1.N = s.N;
  g1.T = s.T;
  g1.rows_routed = (int)TK;
  g1.x_shared_row0 = 0;
  g1.n_feat = 2 * s.f;
  g1.k_dim = s.d;
  g1.x_rep = 1;
  g1.out_ld = s.f;
  if (launch_gemm<kEpiSwiGLU>(g1, st) != cudaSuccess) return MOE_ERR_CUDA;

  // GEMM2: weights W2 [(N+1)*d, f], tokens H (routed rows, then the shared rows)
  GemmArgs g2{};
  ok = make_map(&g2.tmW, w2, BF, 2, s.f, (uint64_t)(s.N + 1) * s.d, BK, BW) &&
       make_map(&g2.tmX_routed, H, BF, 2, s.f, TK + s.T, BK, BT) &&
       make_map(&g2.tmX_shared, H, BF, 2, s.f, TK + s.T, BK, BT);
  if (!ok) return MOE_ERR_CUDA;
  g2.offsets = offsets;
  g2.out_routed = static_cast<__nv_bfloat16*>(y_perm);
  g2.out_shared = static_cast<__nv_bfloat16*>(y_shared);
  g2.status = status;
  g2.N = s.N;
  g2.T = s.T;
  g2.rows_routed = (int)TK;
  g2.x_shared_row0 = (int)TK;
  g2.n_feat = s.d;
  g2.k_dim = s.f;
  g2.x_rep = 1;
  g2.out_ld = s.d;
  if (launch_gemm<kEpiStore>(g2, st) != cudaSuccess) return MOE_ERR_CUDA;
  return MOE_OK;
}

int launch_router_scores_tc(const moe_shape& s, const void* x, const float* router, float* S,
                            void* ws, cudaStream_t st) {
  const WsLayout L = ws_layout(s);
  uint8_t* w = static_cast<uint8_t*>(ws);
  __nv_bfloat16* Rs = reinterpret_cast<__nv_bfloat16*>(w + L.router_split);
  const long long total = (long long)s.N * s.d;
  long long blocks = (total + 255) / 256;
  if (blocks > 148 * 8) blocks = 148 * 8;
  router_split_kernel<<<(int)blocks, 256, 0, st>>>(router, s.N, s.d, Rs);
  if (cudaGetLastError() != cudaSuccess) return MOE_ERR_CUDA;

  GemmArgs a{};
  const auto BF = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  bool ok = make_map(&a.tmW, Rs, BF, 2, 3ull * s.d, s.N, BK, BW) &&
            make_map(&a.tmX_routed, x, BF, 2, s.d, s.T, BK, BT) &&
            make_map(&a.tmX_shared, x, BF, 2, s.d, s.T, BK, BT);
  if (!ok) return MOE_ERR_CUDA;
  a.offsets = nullptr;
  a.out_f32 = S;
  a.status = reinterpret_cast<uint32_t*>(w + L.status);
  a.N = 0;  // a single group: all T token rows of x
  a.T = s.T;
  a.rows_routed = 0;
  a.x_shared_row0 = 0;
  a.n_feat = BW;  // one weight tile: experts 0..255 (rows >= N read as zero)
  a.k_dim = 3 * s.d;
  a.x_rep = 3;
  a.out_ld = s.N;
  a.n_valid = s.N;
  return launch_gemm<kEpiSigmoid>(a, st) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

}  // namespace moe
