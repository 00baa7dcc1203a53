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
// write it with TMA tensor stores into the gradient laid out like the weight.
// An expert without rows gets zeros.
// Every mbarrier wait is bounded (~2 s) and sets the device status word.
#include <cuda.h>
#include <cuda_bf16.h>

#include <cstdlib>
#include <cstring>

#include "epilogue.cuh"
#include "internal.h"
#include "ptx.cuh"
#include "tile_transpose.cuh"

namespace moe {
namespace {

constexpr int WBM = 128, WBN = 256, WBK = 64;
constexpr int WStages = 4;
constexpr int WABytes = WBM * WBK * 2;
constexpr int WBBytes = WBN * WBK * 2;
constexpr int WStageBytes = WABytes + WBBytes;
constexpr int WThreads = 320;  // warp 0 TMA, warp 1 MMA, warps 2-9 epilogue (2 per quadrant)
constexpr int WStgBytes = 32 * 128;  // per epilogue warp: 32 rows x 64 bf16, 128B-swizzled
constexpr int WSmemBytes = 1024 + WStages * WStageBytes + 8 * WStgBytes + 256;
static_assert(WSmemBytes <= 232448, "weight-gradient kernel exceeds the shared-memory opt-in");
constexpr uint64_t WTimeoutNs = 2000000000ull;

// ---- layout: column blocks per group --------------------------------------------

// colbase[g] = sum over g' < g of round_up(rows_g', pad); colbase[N+1] = R.
__global__ void colbase_kernel(const int32_t* __restrict__ offsets, int N, int T, int pad,
                               int32_t* __restrict__ colbase) {
  const int lane = threadIdx.x;
  const int G1 = N + 1;
  const int per = (G1 + 31) / 32;
  const int g0 = min(G1, lane * per), g1 = min(G1, g0 + per);
  auto padded = [&](int g) {
    const int rows = (g < N) ? offsets[g + 1] - offsets[g] : T;
    return (max(rows, 0) + pad - 1) / pad * pad;
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

// Rows [rows, C] (dispatched rows from `routed`, then the shared expert's
// from `shared`; with `perm_tok`, dispatched row r is row perm_tok[r] of
// `routed`) -> dst [C, R]: group g's rows go, in order, to its columns
// colbase[g] .. colbase[g] + rows_g - 1, and its padding columns up to
// colbase[g + 1] get zeros.  A CTA moves kGroupTiles 64 x 64 tiles
// (tile_transpose.cuh) of the same 64 columns and consecutive features: all
// their 16-byte loads are issued before any shared-memory write, so each
// thread keeps 2 * kGroupTiles loads in flight.  The colbase values are
// multiples of 64 (the padding is 64 or 128), so a column tile lies in one
// group.
// kSwiGLUH: the source holds the packed gate/up products [rows, 2f] and the
// value moved is h = silu(g) * u of feature c (C = f), rounded to bf16.
constexpr int kGroupTiles = 4;
constexpr int kItems = kTile * 8 / kTileThreads;  // 16-byte items per thread per tile

template <bool kSwiGLUH>
__global__ void __launch_bounds__(kTileThreads) transpose_groups_kernel(
    const __nv_bfloat16* __restrict__ routed, const __nv_bfloat16* __restrict__ shared, int TK,
    int T, int N, int C, int src_ld, const int32_t* __restrict__ offsets,
    const int32_t* __restrict__ perm_tok, const int32_t* __restrict__ colbase, long long ld,
    __nv_bfloat16* __restrict__ dst) {
  __shared__ alignas(16) uint8_t sm[kGroupTiles][kTileBytes];
  __shared__ int s_group;
  const long long col0 = (long long)blockIdx.y * kTile;
  const int fb = blockIdx.x * kGroupTiles * kTile;
  const int G1 = N + 1;
  if (col0 >= colbase[G1]) return;  // past the last group's block
  if (threadIdx.x == 0) {
    int lo = 0, hi = G1;  // colbase[lo] <= col0 < colbase[hi]
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (colbase[mid] <= col0) lo = mid; else hi = mid;
    }
    s_group = lo;
  }
  __syncthreads();
  const int g = s_group;
  const long long first = g < N ? offsets[g] : TK;
  const long long count = g < N ? (long long)offsets[g + 1] - offsets[g] : T;
  const long long limit = g < N ? TK : (long long)TK + T;  // a group's rows stay below
  const long long local0 = col0 - colbase[g];
  // this thread's source rows (the same in every tile of the CTA)
  const __nv_bfloat16* rowp[kItems];
#pragma unroll
  for (int j = 0; j < kItems; ++j) {
    const int i = (threadIdx.x + j * kTileThreads) >> 3;
    const long long r = first + local0 + i;
    const long long src = (perm_tok != nullptr && r >= 0 && r < TK) ? perm_tok[r] : r;
    const bool src_ok = perm_tok == nullptr || r >= TK || (src >= 0 && src < T);
    rowp[j] = (local0 + i < count && r >= 0 && r < limit && src_ok)
                  ? (r < TK ? routed + (size_t)src * src_ld : shared + (size_t)(r - TK) * src_ld)
                  : nullptr;
  }
  uint4 v[kGroupTiles][kItems];
#pragma unroll
  for (int t = 0; t < kGroupTiles; ++t) {
    const int f0 = fb + t * kTile;
#pragma unroll
    for (int j = 0; j < kItems; ++j) {
      const int p = (threadIdx.x + j * kTileThreads) & 7;
      v[t][j] = make_uint4(0u, 0u, 0u, 0u);
      if (rowp[j] != nullptr && f0 + p * 8 + 8 <= C) {
        if constexpr (kSwiGLUH) {
          const int col = (f0 / 128) * 256 + (f0 % 128) + p * 8;
          float gt[8], up[8];
          bf16x8_load(rowp[j] + col, gt);
          bf16x8_load(rowp[j] + col + 128, up);
          __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&v[t][j]);
#pragma unroll
          for (int e = 0; e < 4; ++e)
            h[e] = __floats2bfloat162_rn(silu_fast(gt[2 * e]) * up[2 * e],
                                         silu_fast(gt[2 * e + 1]) * up[2 * e + 1]);
        } else {
          v[t][j] = __ldg(reinterpret_cast<const uint4*>(rowp[j] + f0 + p * 8));
        }
      }
    }
  }
#pragma unroll
  for (int t = 0; t < kGroupTiles; ++t)
#pragma unroll
    for (int j = 0; j < kItems; ++j) {
      const int it = threadIdx.x + j * kTileThreads;
      tile_put(sm[t], it >> 3, it & 7, v[t][j]);
    }
  __syncthreads();
#pragma unroll
  for (int t = 0; t < kGroupTiles; ++t) {
    const int f0 = fb + t * kTile;
    for (int it = threadIdx.x; it < kTile * 8; it += kTileThreads) {
      const int c = it >> 3, q = it & 7;
      if (f0 + c < C && col0 + q * 8 + 8 <= ld)
        *reinterpret_cast<uint4*>(dst + (size_t)(f0 + c) * ld + col0 + q * 8) =
            tile_get(sm[t], c, q);
    }
  }
}

// ---- the weight-gradient products ---------------------------------------------------
struct alignas(64) WgradArgs {
  CUtensorMap tmL;  // left operand [M_total, R] (rows of the gradient), box {64, 128}
  CUtensorMap tmR;  // right operand [N_total, R] (its columns), box {64, 256}
  CUtensorMap tmOut;  // gradient [G1 * M_total, N_total], box {64, 32}, 128B swizzle
  const int32_t* colbase;  // [G1 + 1] column block of each group
  uint32_t* status;
  int G1, M_total, N_total;
};

__global__ void __launch_bounds__(WThreads, 1) wgrad_gemm_kernel(
    const __grid_constant__ WgradArgs args) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* staging = base + (size_t)WStages * WStageBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(staging + 8 * WStgBytes);
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

  // unit -> group g, left tile m, right tile n (n fastest: units running at the
  // same time write whole rows of the gradient, and an expert's operands stay
  // in L2 while its units run); K blocks of the group's column block
  auto decode = [&](int u, int& g, int& n, int& m, int& kb0, int& kcnt) {
    g = u / per_group;
    const int local = u - g * per_group;
    m = local / NT;
    n = local - m * NT;
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
    // Units are short (a few K blocks) and each stores a 64 KB tile.  Two
    // warps per TMEM lane quadrant drain it, 128 columns each, in 64-column
    // pieces: TMEM -> registers -> bf16 -> this warp's 128B-swizzled staging
    // buffer -> one TMA tensor store of 32 rows x 64 columns (whole 128-byte
    // lines, off the load/store pipeline).
    const int q = warp & 3;
    const int half = (warp - 2) >> 2;
    uint8_t* stg = staging + (size_t)(warp - 2) * WStgBytes;
    int local = 0;
    for (int u = blockIdx.x; u < total; u += gridDim.x, ++local) {
      int g, n, m, kb0, kcnt;
      decode(u, g, n, m, kb0, kcnt);
      const int acc = local & 1;
      if (!mbar_wait_bounded(&tfull[acc], (local >> 1) & 1, args.status, WTimeoutNs)) break;
      tc_fence_after();
      const int grow = g * args.M_total + m * WBM + q * 32;
      const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + acc * WBN;
#pragma unroll 1
      for (int c = half * (WBN / 2); c < (half + 1) * (WBN / 2); c += 64) {
        uint32_t packed[32];
        if (kcnt > 0) {  // a group without rows has a zero gradient
          uint32_t v0[32], v1[32];
          tmem_ld32(taddr + c, v0);
          tmem_ld32(taddr + c + 32, v1);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            packed[i] = bf16x2_bits(__uint_as_float(v0[2 * i]), __uint_as_float(v0[2 * i + 1]));
            packed[16 + i] =
                bf16x2_bits(__uint_as_float(v1[2 * i]), __uint_as_float(v1[2 * i + 1]));
          }
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) packed[i] = 0u;
        }
        if (lane == 0) bulk_wait_read_all();  // the previous piece has left the buffer
        __syncwarp();
        uint8_t* my_row = stg + lane * 128;
#pragma unroll
        for (int j = 0; j < 8; ++j)
          *reinterpret_cast<uint4*>(my_row + ((j ^ (lane & 7)) << 4)) =
              make_uint4(packed[4 * j], packed[4 * j + 1], packed[4 * j + 2], packed[4 * j + 3]);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_2d(&args.tmOut, stg, n * WBN + c, grow);
          bulk_commit_group();
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[acc]);
    }
    if (lane == 0) bulk_wait_all();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 2 * WBN);
  }
}

cudaError_t launch_wgrad(const WgradArgs& a, cudaStream_t st) {
  const size_t smem = WSmemBytes;
  cudaError_t e = note_cuda(cudaFuncSetAttribute(wgrad_gemm_kernel,
                                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 (int)smem),
                            "weight-gradient GEMM: set shared-memory size");
  if (e != cudaSuccess) return e;
  wgrad_gemm_kernel<<<num_sms(), WThreads, smem, st>>>(a);
  return note_cuda(cudaGetLastError(), "weight-gradient GEMM launch");
}

// ---- the same products on CTA pairs -----------------------------------------------
// A unit is one 256 x 256 output tile of one expert, one tcgen05.mma
// cta_group::2 (M=256, N=256, K=16) per K step: CTA r of the pair stages rows
// 128r..128r+127 of the tile's left operand and rows 128r..128r+127 of its
// right operand, so per K block a CTA stages 32 KB instead of 48 KB for the
// same 128 x 256 outputs, and each CTA's TMEM holds its 128 rows of the tile.
// The gradient rows are multiples of 256 (d and 2f are), so no unit is ragged.
// Barriers: full (leader; both CTAs' copies land on it), empty and tfull (each
// CTA; the leader's commits are multicast), edone (each CTA; its eight
// epilogue warps have read the accumulator) and tempty (leader; one arrive per
// use from the peer CTA's warp 1, which forwards its edone).  The leader's MMA
// thread waits on its own edone and on tempty, so one cluster-scope arrive per
// accumulator use crosses the pair instead of one per epilogue warp: the
// release fence each of those arrives carries was the epilogue's largest
// stall.  Both CTAs reach the final cluster barrier, so neither exits while
// its peer may still signal it.
constexpr int QStages = 5;
constexpr int QHalfBytes = WBM * WBK * 2;     // 16 KB: 128 rows x 64 K
constexpr int QStageBytes = 2 * QHalfBytes;   // left rows + right rows
// two staging buffers per epilogue warp: a piece is staged while the store of
// the previous one may still be reading its buffer
constexpr int QSmemBytes = 1024 + QStages * QStageBytes + 16 * WStgBytes + 256;
static_assert(QSmemBytes <= 232448, "pair weight-gradient kernel exceeds the shared-memory opt-in");

__global__ void __launch_bounds__(WThreads, 1) wgrad_pair_kernel(
    const __grid_constant__ WgradArgs args) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* staging = base + (size_t)QStages * QStageBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(staging + 16 * WStgBytes);
  uint64_t* full = bars;               // [QStages] leader
  uint64_t* empty = full + QStages;    // [QStages] each CTA
  uint64_t* tfull = empty + QStages;   // [2] each CTA
  uint64_t* tempty = tfull + 2;        // [2] leader
  uint64_t* drain = tempty + 2;
  uint64_t* edone = drain + 1;         // [2] each CTA: its eight epilogue warps have read
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(edone + 2);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const int MT = args.M_total / (2 * WBM), NT = args.N_total / WBN;
  const int per_group = MT * NT;
  const int total = args.G1 * per_group;

  if (tid == 0) {
    for (int st = 0; st < QStages; ++st) {
      mbar_init(&full[st], 1);
      mbar_init(&empty[st], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 1);   // the peer CTA's forwarded release
      mbar_init(&edone[a], 8);
    }
    mbar_init(drain, 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc_2sm(tmem_holder, 2 * WBN);
    tmem_relinquish_2sm();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // both CTAs' barriers exist before either signals the other
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  auto decode = [&](int u, int& g, int& n, int& m, int& kb0, int& kcnt) {
    g = u / per_group;
    const int local = u - g * per_group;
    m = local / NT;
    n = local - m * NT;
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
      for (int u = pair; u < total && ok; u += npairs) {
        int g, n, m, kb0, kcnt;
        decode(u, g, n, m, kb0, kcnt);
        for (int kb = 0; kb < kcnt; ++kb) {
          if (!mbar_wait_bounded(&empty[stage], phase ^ 1u, args.status, WTimeoutNs)) {
            ok = false;
            break;
          }
          uint8_t* sa = base + (size_t)stage * QStageBytes;
          const uint32_t fbar = mapa_shared(smem_u32(&full[stage]), 0);
          if (leader) mbar_arrive_expect_tx(&full[stage], 2 * QStageBytes);
          tma_load_2d_2sm(sa, &args.tmL, (kb0 + kb) * WBK, m * 2 * WBM + (int)rank * WBM, fbar);
          tma_load_2d_2sm(sa + QHalfBytes, &args.tmR, (kb0 + kb) * WBK,
                          n * WBN + (int)rank * WBM, fbar);
          issued |= 1u << stage;
          issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == QStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok && leader) {  // the copies already issued complete on these barriers
        for (int st = 0; st < QStages; ++st)
          if ((issued >> st) & 1u)
            mbar_wait_bounded(&full[st], (issued_parity >> st) & 1u, args.status,
                              WTimeoutNs / 8);
      }
    }
  } else if (warp == 1) {
    if (leader && lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(2 * WBM, WBN);
      int stage = 0;
      uint32_t phase = 0;
      int local = 0;
      bool ok = true;
      for (int u = pair; u < total && ok; u += npairs, ++local) {
        int g, n, m, kb0, kcnt;
        decode(u, g, n, m, kb0, kcnt);
        const int acc = local & 1;
        if (!mbar_wait_bounded(&edone[acc], ((local >> 1) & 1) ^ 1u, args.status, WTimeoutNs) ||
            !mbar_wait_cluster_bounded(&tempty[acc], ((local >> 1) & 1) ^ 1u, args.status,
                                       WTimeoutNs))
          break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * WBN;
        for (int kb = 0; kb < kcnt; ++kb) {
          if (!mbar_wait_bounded(&full[stage], phase, args.status, WTimeoutNs)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(base + (size_t)stage * QStageBytes);
          const uint32_t b0 = a0 + QHalfBytes;
#pragma unroll
          for (int k = 0; k < WBK / 16; ++k)
            mma_bf16_2sm(d_tmem, smem_desc_sw128(a0 + k * 32), smem_desc_sw128(b0 + k * 32),
                         idesc, (kb | k) != 0);
          mma_commit_2sm_mc(&empty[stage], 0x3);
          if (++stage == QStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (ok) mma_commit_2sm_mc(&tfull[acc], 0x3);  // with no K blocks: arrives at once
      }
      mma_commit_2sm(drain);
      mbar_wait_bounded(drain, 0, args.status, WTimeoutNs / 8);
    } else if (!leader && lane == 0) {
      // forward each accumulator release of this CTA's epilogue warps to the
      // leader with one cluster-scope arrive
      const uint32_t tempty0 = mapa_shared(smem_u32(&tempty[0]), 0);
      int local = 0;
      for (int u = pair; u < total; u += npairs, ++local) {
        const int acc = local & 1;
        if (!mbar_wait_bounded(&edone[acc], (local >> 1) & 1, args.status, WTimeoutNs)) break;
        mbar_arrive_cluster(tempty0 + 8u * (uint32_t)acc);
      }
    }
  } else {
    // each CTA drains its 128 rows of the tile exactly as the one-CTA kernel
    const int q = warp & 3;
    const int half = (warp - 2) >> 2;
    uint8_t* stg0 = staging + (size_t)(warp - 2) * 2 * WStgBytes;
    int local = 0;
    for (int u = pair; u < total; u += npairs, ++local) {
      int g, n, m, kb0, kcnt;
      decode(u, g, n, m, kb0, kcnt);
      const int acc = local & 1;
      if (!mbar_wait_bounded(&tfull[acc], (local >> 1) & 1, args.status, WTimeoutNs)) break;
      tc_fence_after();
      const int grow = g * args.M_total + m * 2 * WBM + (int)rank * WBM + q * 32;
      const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + acc * WBN;
#pragma unroll 1
      for (int c = half * (WBN / 2); c < (half + 1) * (WBN / 2); c += 64) {
        uint32_t packed[32];
        if (kcnt > 0) {
          uint32_t v0[32], v1[32];
          tmem_ld32(taddr + c, v0);
          tmem_ld32(taddr + c + 32, v1);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            packed[i] = bf16x2_bits(__uint_as_float(v0[2 * i]), __uint_as_float(v0[2 * i + 1]));
            packed[16 + i] =
                bf16x2_bits(__uint_as_float(v1[2 * i]), __uint_as_float(v1[2 * i + 1]));
          }
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) packed[i] = 0u;
        }
        uint8_t* stg = stg0 + (c & 64 ? WStgBytes : 0);  // pieces alternate buffers
        if (lane == 0) bulk_wait_read_but_one();  // this buffer's last store has read it
        __syncwarp();
        uint8_t* my_row = stg + lane * 128;
#pragma unroll
        for (int j = 0; j < 8; ++j)
          *reinterpret_cast<uint4*>(my_row + ((j ^ (lane & 7)) << 4)) =
              make_uint4(packed[4 * j], packed[4 * j + 1], packed[4 * j + 2], packed[4 * j + 3]);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_2d(&args.tmOut, stg, n * WBN + c, grow);
          bulk_commit_group();
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&edone[acc]);
    }
    if (lane == 0) bulk_wait_all();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_2sm(tmem_base, 2 * WBN);
  }
}

cudaError_t launch_wgrad_pair(const WgradArgs& a, cudaStream_t st) {
  cudaError_t e = note_cuda(cudaFuncSetAttribute(wgrad_pair_kernel,
                                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 QSmemBytes),
                            "pair weight-gradient GEMM: set shared-memory size");
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(WThreads, 1, 1);
  cfg.dynamicSmemBytes = QSmemBytes;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cfg.gridDim = dim3((unsigned)(num_sms() & ~1), 1, 1);
  // as many pairs as can be resident at once, so no pair waits for a second wave
  static int max_pairs = 0;
  if (max_pairs == 0) {
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, wgrad_pair_kernel, &cfg) != cudaSuccess || n <= 0)
      n = num_sms() / 2;
    max_pairs = n;
  }
  cfg.gridDim = dim3((unsigned)(2 * max_pairs), 1, 1);
  return note_cuda(cudaLaunchKernelEx(&cfg, wgrad_pair_kernel, a),
                   "pair weight-gradient GEMM launch");
}

// MOE_WGRAD=single selects the one-CTA kernel (read once per process).
bool use_pair_wgrad() {
  static int v = -1;
  if (v < 0) {
    const char* e = std::getenv("MOE_WGRAD");
    v = (e != nullptr && std::strcmp(e, "single") == 0) ? 0 : 1;
  }
  return v == 1;
}

}  // namespace

// Columns of the transposed layouts: all rows plus up to 63 of padding per group.
long long wgrad_cols(const moe_shape& s) {
  const long long rows = (long long)s.T * s.K + s.T;
  return (rows + (long long)(s.N + 1) * (WBK - 1) + WBK - 1) / WBK * WBK;
}

// The activations of every product laid out transposed in per-group column
// blocks padded to `pad` (64 for the bf16 MMA's K step, 128 for an FP8 scale
// tile): AT = [A; x]^T (A the dispatched rows, or x gathered through
// perm_tok), dYT = [dy_perm; dy_shared]^T, HT from the stored g, u, and
// dGUT = dGU^T.  colbase [N+2] receives the blocks' first columns.
cudaError_t launch_group_transposes(const moe_shape& s, int pad, const void* a_routed,
                                    const int32_t* a_perm, const void* x, const void* dy_perm,
                                    const void* dy_shared, const __nv_bfloat16* GU,
                                    const __nv_bfloat16* dGU, const int32_t* offsets,
                                    int32_t* colbase, long long R, __nv_bfloat16* AT,
                                    __nv_bfloat16* dYT, __nv_bfloat16* HT, __nv_bfloat16* dGUT,
                                    cudaStream_t st) {
  const int TK = s.T * s.K;
  const int twof = 2 * s.f;
  const auto bf = [](const void* p) { return static_cast<const __nv_bfloat16*>(p); };
  colbase_kernel<<<1, 32, 0, st>>>(offsets, s.N, s.T, pad, colbase);
  const unsigned col_tiles = (unsigned)(R / kTile);
  auto layout = [&](auto kernel, const __nv_bfloat16* routed, const int32_t* perm,
                    const __nv_bfloat16* shared, int C, int src_ld, __nv_bfloat16* dst) {
    const unsigned f_blocks = (unsigned)((C / kTile + kGroupTiles - 1) / kGroupTiles);
    kernel<<<dim3(f_blocks, col_tiles), kTileThreads, 0, st>>>(
        routed, shared, TK, s.T, s.N, C, src_ld, offsets, perm, colbase, R, dst);
  };
  layout(transpose_groups_kernel<false>, bf(a_routed), a_perm, bf(x), s.d, s.d, AT);
  layout(transpose_groups_kernel<false>, bf(dy_perm), nullptr, bf(dy_shared), s.d, s.d, dYT);
  layout(transpose_groups_kernel<true>, GU, nullptr, GU + (size_t)TK * twof, s.f, twof, HT);
  layout(transpose_groups_kernel<false>, dGU, nullptr, dGU + (size_t)TK * twof, twof, twof,
         dGUT);
  return note_cuda(cudaGetLastError(), "weight-gradient layout kernels");
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
  __nv_bfloat16* AT = reinterpret_cast<__nv_bfloat16*>(w + B.at);
  __nv_bfloat16* dYT = reinterpret_cast<__nv_bfloat16*>(w + B.dyt);
  __nv_bfloat16* HT = reinterpret_cast<__nv_bfloat16*>(w + B.ht);
  __nv_bfloat16* dGUT = reinterpret_cast<__nv_bfloat16*>(w + B.dgut);
  const long long R = wgrad_cols(s);
  const int twof = 2 * s.f;
  if (launch_group_transposes(s, WBK, x_perm, nullptr, x, dy_perm, dy_shared, GU, dGU, offsets,
                              colbase, R, AT, dYT, HT, dGUT, st) != cudaSuccess)
    return MOE_ERR_CUDA;

  const auto BF = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const bool pair = use_pair_wgrad();
  const uint32_t rbox = pair ? WBM : WBN;  // right-operand rows per CTA
  // dW2_e [d, f] = dYT_e HT_e^T
  WgradArgs a2{};
  bool ok = make_map(&a2.tmL, dYT, BF, 2, R, s.d, WBK, WBM) &&
            make_map(&a2.tmR, HT, BF, 2, R, s.f, WBK, rbox);
  // dW13_e [2f, d] = dGUT_e AT_e^T (rows in the packed W13 order)
  WgradArgs a13{};
  ok = ok && make_map(&a13.tmL, dGUT, BF, 2, R, twof, WBK, WBM) &&
       make_map(&a13.tmR, AT, BF, 2, R, s.d, WBK, rbox);
  const uint64_t G1 = (uint64_t)s.N + 1;
  ok = ok && make_map(&a2.tmOut, dw2, BF, 2, s.f, G1 * s.d, 64, 32) &&
       make_map(&a13.tmOut, dw13, BF, 2, s.d, G1 * twof, 64, 32);
  if (!ok) {
    note_text("weight-gradient GEMM: tensor-map encoding failed");
    return MOE_ERR_CUDA;
  }
  a2.colbase = a13.colbase = colbase;
  a2.status = a13.status = status;
  a2.G1 = a13.G1 = s.N + 1;
  a2.M_total = s.d;
  a2.N_total = s.f;
  a13.M_total = twof;
  a13.N_total = s.d;
  const auto run = pair ? launch_wgrad_pair : launch_wgrad;
  if (run(a2, st) != cudaSuccess || run(a13, st) != cudaSuccess) return MOE_ERR_CUDA;
  return MOE_OK;
}

}  // namespace moe
