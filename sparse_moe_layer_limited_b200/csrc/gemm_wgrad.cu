// Backward of the expert FFNs, weight gradients (MLP_W of the mhpq.cn
// article §2.2 backward order COMBINE -> MLP_B -> MLP_W -> DISPATCH), bf16.
//
// Per expert e (group N = the shared expert, on all T rows of x):
//   dW2_e  = dY_e^T H_e           [d, f],   H = silu(g) * u
//   dW13_e = [dg du]_e^T A_e      [2f, d],  packed like W13
// Each contracts over the expert's rows, a different count per expert.  The
// activations are first laid out transposed, expert by expert: each group
// takes a block of columns padded with zeros to a multiple of 64 (the MMA's
// K step), so both operands of every product are K-major:
//   AT [d, R] (x_perm / x),  dYT [d, R],  HT [f, R] (from the stored g, u),
//   dGUT [2f, R] (the input-gradient pass's dg, du)
// Then one persistent tensor-core kernel runs all products: a unit is one
// 128 x 256 output tile of one expert, its K loop the expert's column block
// (tcgen05.mma cta_group::1, M=128, N=256, K=16, fp32 accumulate in TMEM,
// two accumulators in turn); eight epilogue warps round the tile to bf16 and
// store it into the gradient laid out like the weight.  An expert without rows gets zeros.
// Every mbarrier wait is bounded (~2 s) and sets the device status word.
#include <cuda.h>
#include <cuda_bf16.h>

#include "epilogue.cuh"
#include "internal.h"
#include "ptx.cuh"

namespace moe {
namespace {

constexpr int WBM = 128, WBN = 256, WBK = 64;
constexpr int WStages = 4;
constexpr int WABytes = WBM * WBK * 2;
constexpr int WBBytes = WBN * WBK * 2;
constexpr int WStageBytes = WABytes + WBBytes;
constexpr int WThreads = 320;  // warp 0 TMA, warp 1 MMA, warps 2-9 epilogue (2 per quadrant)
constexpr uint64_t WTimeoutNs = 2000000000ull;

// ---- layout: column blocks per group --------------------------------------------

// colbase[g] = sum over g' < g of round_up(rows_g', 64); colbase[N+1] = R.
__global__ void colbase_kernel(const int32_t* __restrict__ offsets, int N, int T,
                               int32_t* __restrict__ colbase) {
  const int lane = threadIdx.x;
  const int G1 = N + 1;
  const int per = (G1 + 31) / 32;
  const int g0 = min(G1, lane * per), g1 = min(G1, g0 + per);
  auto padded = [&](int g) {
    const int rows = (g < N) ? offsets[g + 1] - offsets[g] : T;
    return (max(rows, 0) + WBK - 1) / WBK * WBK;
  };
  int sum = 0;
  for (int g = g0; g < g1; ++g) sum += padded(g);
  int inc = sum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += v;
  }
  int run = inc - sum;
  for (int g = g0; g < g1; ++g) {
    colbase[g] = run;
    run += padded(g);
  }
  if (lane == 31) colbase[G1] = inc;
}

// col_of_row[r]: the column of dispatched row r (r < T*K) or of shared row
// r - T*K in the transposed layouts.
__global__ void col_of_row_kernel(const int32_t* __restrict__ offsets,
                                  const int32_t* __restrict__ colbase, int N, int T, int TK,
                                  int32_t* __restrict__ col_of_row) {
  const int r = blockIdx.x * blockDim.x + threadIdx.x;
  if (r >= TK + T) return;
  if (r >= TK) {
    col_of_row[r] = colbase[N] + (r - TK);
    return;
  }
  int lo = 0, hi = N;  // the group g with offsets[g] <= r < offsets[g+1]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (offsets[mid] <= r) lo = mid; else hi = mid;
  }
  col_of_row[r] = colbase[lo] + (r - offsets[lo]);
}

// Zero the padding columns of each group in a [C, R] layout.
__global__ void zero_padding_kernel(const int32_t* __restrict__ offsets,
                                    const int32_t* __restrict__ colbase, int N, int T, int C,
                                    long long ld, __nv_bfloat16* __restrict__ dst) {
  const int g = blockIdx.y;
  const int rows = (g < N) ? offsets[g + 1] - offsets[g] : T;
  // columns stay inside the layout even if offsets[] is inconsistent
  const int c0 = (int)min((long long)colbase[g] + max(rows, 0), ld);
  const int c1 = (int)min((long long)colbase[g + 1], ld);
  const int npad = c1 - c0;
  if (npad <= 0) return;
  const __nv_bfloat16 z = __float2bfloat16_rn(0.f);
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < (long long)C * npad;
       i += (long long)gridDim.x * blockDim.x) {
    const long long c = i / npad;
    dst[c * ld + c0 + (i - c * npad)] = z;
  }
}

// Rows [rows, C] (dispatched rows from `routed`, then the shared expert's
// from `shared`) -> dst [C, R] at the rows' columns.  kSwiGLUH: the source
// holds the packed gate/up products [rows, 2f] and the value moved is
// h = silu(g) * u for feature c (C = f).
template <bool kSwiGLUH>
__global__ void transpose_rows_kernel(const __nv_bfloat16* __restrict__ routed,
                                      const __nv_bfloat16* __restrict__ shared, int TK, int T,
                                      int C, int src_ld, const int32_t* __restrict__ col_of_row,
                                      long long ld, __nv_bfloat16* __restrict__ dst) {
  __shared__ float tile[32][33];
  const int r0 = blockIdx.y * 32, c0 = blockIdx.x * 32;
  const int rows = TK + T;
  for (int i = threadIdx.y; i < 32; i += 8) {
    const int r = r0 + i, c = c0 + threadIdx.x;
    float v = 0.f;
    if (r < rows && c < C) {
      const __nv_bfloat16* row =
          r < TK ? routed + (size_t)r * src_ld : shared + (size_t)(r - TK) * src_ld;
      if constexpr (kSwiGLUH) {
        const int col = (c / 128) * 256 + (c % 128);
        const float gt = __bfloat162float(row[col]), up = __bfloat162float(row[col + 128]);
        v = silu_f(gt) * up;
      } else {
        v = __bfloat162float(row[c]);
      }
    }
    tile[i][threadIdx.x] = v;
  }
  __syncthreads();
  for (int i = threadIdx.y; i < 32; i += 8) {
    const int c = c0 + i, r = r0 + threadIdx.x;
    if (c < C && r < rows) {
      const int col = col_of_row[r];
      if (col >= 0 && col < ld) dst[(size_t)c * ld + col] = __float2bfloat16_rn(tile[threadIdx.x][i]);
    }
  }
}

// ---- the weight-gradient products ---------------------------------------------------
struct alignas(64) WgradArgs {
  CUtensorMap tmL;  // left operand [M_total, R] (rows of the gradient), box {64, 128}
  CUtensorMap tmR;  // right operand [N_total, R] (its columns), box {64, 256}
  const int32_t* colbase;  // [G1 + 1] column block of each group
  __nv_bfloat16* out;      // [G1, M_total, N_total]
  uint32_t* status;
  int G1, M_total, N_total;
};

__global__ void __launch_bounds__(WThreads, 1) wgrad_gemm_kernel(
    const __grid_constant__ WgradArgs args) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + (size_t)WStages * WStageBytes);
  uint64_t* full = bars;
  uint64_t* empty = full + WStages;
  uint64_t* tfull = empty + WStages;   // [2]
  uint64_t* tempty = tfull + 2;        // [2]
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int MT = args.M_total / WBM, NT = args.N_total / WBN;
  const int per_group = MT * NT;
  const int total = args.G1 * per_group;

  if (tid == 0) {
    for (int s = 0; s < WStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 8);
    }
    mbar_init(drain, 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, 2 * WBN);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  // unit -> group g, right tile n, left tile m (m fastest: neighbours share the
  // 256-row right tile); K blocks of the group's column block
  auto decode = [&](int u, int& g, int& n, int& m, int& kb0, int& kcnt) {
    g = u / per_group;
    const int local = u - g * per_group;
    n = local / MT;
    m = local - n * MT;
    kb0 = args.colbase[g] / WBK;
    kcnt = (args.colbase[g + 1] - args.colbase[g]) / WBK;
  };

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&args.tmL);
      tma_prefetch_desc(&args.tmR);
      int stage = 0;
      uint32_t phase = 0, issued = 0, issued_parity = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < total && ok; u += gridDim.x) {
        int g, n, m, kb0, kcnt;
        decode(u, g, n, m, kb0, kcnt);
        for (int kb = 0; kb < kcnt; ++kb) {
          if (!mbar_wait_bounded(&empty[stage], phase ^ 1u, args.status, WTimeoutNs)) {
            ok = false;
            break;
          }
          uint8_t* sa = base + (size_t)stage * WStageBytes;
          mbar_arrive_expect_tx(&full[stage], WStageBytes);
          tma_load_2d(sa, &args.tmL, (kb0 + kb) * WBK, m * WBM, &full[stage]);
          tma_load_2d(sa + WABytes, &args.tmR, (kb0 + kb) * WBK, n * WBN, &full[stage]);
          issued |= 1u << stage;
          issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == WStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {
        for (int s = 0; s < WStages; ++s)
          if ((issued >> s) & 1u)
            mbar_wait_bounded(&full[s], (issued_parity >> s) & 1u, args.status, WTimeoutNs / 8);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(WBM, WBN);
      int stage = 0;
      uint32_t phase = 0;
      int local = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < total && ok; u += gridDim.x, ++local) {
        int g, n, m, kb0, kcnt;
        decode(u, g, n, m, kb0, kcnt);
        const int acc = local & 1;
        if (!mbar_wait_bounded(&tempty[acc], ((local >> 1) & 1) ^ 1u, args.status, WTimeoutNs))
          break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * WBN;
        for (int kb = 0; kb < kcnt; ++kb) {
          if (!mbar_wait_bounded(&full[stage], phase, args.status, WTimeoutNs)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(base + (size_t)stage * WStageBytes);
          const uint32_t b0 = a0 + WABytes;
#pragma unroll
          for (int k = 0; k < WBK / 16; ++k)
            mma_bf16(d_tmem, smem_desc_sw128(a0 + k * 32), smem_desc_sw128(b0 + k * 32), idesc,
                     (kb | k) != 0);
          mma_commit(&empty[stage]);
          if (++stage == WStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (ok) mma_commit(&tfull[acc]);  // with no K blocks: arrives at once
      }
      mma_commit(drain);
      mbar_wait_bounded(drain, 0, args.status, WTimeoutNs / 8);
    }
  } else {
    // units are short (a few K blocks) and each stores a 64 KB tile, so two
    // warps per TMEM lane quadrant drain it, 128 columns each
    const int q = warp & 3;
    const int half = (warp - 2) >> 2;
    const int row = q * 32 + lane;
    int local = 0;
    for (int u = blockIdx.x; u < total; u += gridDim.x, ++local) {
      int g, n, m, kb0, kcnt;
      decode(u, g, n, m, kb0, kcnt);
      const int acc = local & 1;
      if (!mbar_wait_bounded(&tfull[acc], (local >> 1) & 1, args.status, WTimeoutNs)) break;
      tc_fence_after();
      __nv_bfloat16* orow = args.out + ((size_t)g * args.M_total + (size_t)m * WBM + row) *
                                           args.N_total + (size_t)n * WBN;
      const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + acc * WBN;
#pragma unroll 1
      for (int c = half * (WBN / 2); c < (half + 1) * (WBN / 2); c += 32) {
        float y[32];
        if (kcnt > 0) {  // a group without rows has a zero gradient
          uint32_t v[32];
          tmem_ld32(taddr + c, v);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) y[i] = __uint_as_float(v[i]);
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) y[i] = 0.f;
        }
        store_row32(orow + c, y);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[acc]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 2 * WBN);
  }
}

cudaError_t launch_wgrad(const WgradArgs& a, cudaStream_t st) {
  const size_t smem = 1024 + (size_t)WStages * WStageBytes + 256;
  cudaError_t e = note_cuda(cudaFuncSetAttribute(wgrad_gemm_kernel,
                                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 (int)smem),
                            "weight-gradient GEMM: set shared-memory size");
  if (e != cudaSuccess) return e;
  wgrad_gemm_kernel<<<num_sms(), WThreads, smem, st>>>(a);
  return note_cuda(cudaGetLastError(), "weight-gradient GEMM launch");
}

}  // namespace

// Columns of the transposed layouts: all rows plus up to 63 of padding per group.
long long wgrad_cols(const moe_shape& s) {
  const long long rows = (long long)s.T * s.K + s.T;
  return (rows + (long long)(s.N + 1) * (WBK - 1) + WBK - 1) / WBK * WBK;
}

int launch_ffn_bwd_dw_bf16(const moe_shape& s, const void* x_perm, const int32_t* offsets,
                           const void* x, const void* dy_perm, const void* dy_shared,
                           void* dw13, void* dw2, void* ws_bwd, cudaStream_t st) {
  const BwdLayout B = bwd_layout(s);
  uint8_t* w = static_cast<uint8_t*>(ws_bwd);
  uint32_t* status = reinterpret_cast<uint32_t*>(w);
  const __nv_bfloat16* GU = reinterpret_cast<const __nv_bfloat16*>(w + B.gu);
  const __nv_bfloat16* dGU = reinterpret_cast<const __nv_bfloat16*>(w + B.dgu);
  int32_t* colbase = reinterpret_cast<int32_t*>(w + B.colbase);
  int32_t* col_of_row = reinterpret_cast<int32_t*>(w + B.col_of_row);
  __nv_bfloat16* AT = reinterpret_cast<__nv_bfloat16*>(w + B.at);
  __nv_bfloat16* dYT = reinterpret_cast<__nv_bfloat16*>(w + B.dyt);
  __nv_bfloat16* HT = reinterpret_cast<__nv_bfloat16*>(w + B.ht);
  __nv_bfloat16* dGUT = reinterpret_cast<__nv_bfloat16*>(w + B.dgut);
  const int TK = s.T * s.K, rows = TK + s.T;
  const long long R = wgrad_cols(s);
  const int twof = 2 * s.f;
  const auto bf = [](const void* p) { return static_cast<const __nv_bfloat16*>(p); };

  colbase_kernel<<<1, 32, 0, st>>>(offsets, s.N, s.T, colbase);
  col_of_row_kernel<<<(rows + 255) / 256, 256, 0, st>>>(offsets, colbase, s.N, s.T, TK,
                                                         col_of_row);
  const dim3 blk(32, 8);
  auto zero_pad = [&](int C, __nv_bfloat16* dst) {
    zero_padding_kernel<<<dim3(64, s.N + 1), 256, 0, st>>>(offsets, colbase, s.N, s.T, C, R, dst);
  };
  // AT = [x_perm; x]^T, dYT = [dy_perm; dy_shared]^T, HT from GU, dGUT = dGU^T
  transpose_rows_kernel<false><<<dim3((s.d + 31) / 32, (rows + 31) / 32), blk, 0, st>>>(
      bf(x_perm), bf(x), TK, s.T, s.d, s.d, col_of_row, R, AT);
  zero_pad(s.d, AT);
  transpose_rows_kernel<false><<<dim3((s.d + 31) / 32, (rows + 31) / 32), blk, 0, st>>>(
      bf(dy_perm), bf(dy_shared), TK, s.T, s.d, s.d, col_of_row, R, dYT);
  zero_pad(s.d, dYT);
  transpose_rows_kernel<true><<<dim3((s.f + 31) / 32, (rows + 31) / 32), blk, 0, st>>>(
      GU, GU + (size_t)TK * twof, TK, s.T, s.f, twof, col_of_row, R, HT);
  zero_pad(s.f, HT);
  transpose_rows_kernel<false><<<dim3((twof + 31) / 32, (rows + 31) / 32), blk, 0, st>>>(
      dGU, dGU + (size_t)TK * twof, TK, s.T, twof, twof, col_of_row, R, dGUT);
  zero_pad(twof, dGUT);
  if (note_cuda(cudaGetLastError(), "weight-gradient layout kernels") != cudaSuccess)
    return MOE_ERR_CUDA;

  const auto BF = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  // dW2_e [d, f] = dYT_e HT_e^T
  WgradArgs a2{};
  bool ok = make_map(&a2.tmL, dYT, BF, 2, R, s.d, WBK, WBM) &&
            make_map(&a2.tmR, HT, BF, 2, R, s.f, WBK, WBN);
  // dW13_e [2f, d] = dGUT_e AT_e^T (rows in the packed W13 order)
  WgradArgs a13{};
  ok = ok && make_map(&a13.tmL, dGUT, BF, 2, R, twof, WBK, WBM) &&
       make_map(&a13.tmR, AT, BF, 2, R, s.d, WBK, WBN);
  if (!ok) {
    note_text("weight-gradient GEMM: tensor-map encoding failed");
    return MOE_ERR_CUDA;
  }
  a2.colbase = a13.colbase = colbase;
  a2.status = a13.status = status;
  a2.G1 = a13.G1 = s.N + 1;
  a2.out = static_cast<__nv_bfloat16*>(dw2);
  a2.M_total = s.d;
  a2.N_total = s.f;
  a13.out = static_cast<__nv_bfloat16*>(dw13);
  a13.M_total = twof;
  a13.N_total = s.d;
  if (launch_wgrad(a2, st) != cudaSuccess || launch_wgrad(a13, st) != cudaSuccess)
    return MOE_ERR_CUDA;
  return MOE_OK;
}

}  // namespace moe
