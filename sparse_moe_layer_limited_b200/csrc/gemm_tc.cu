// Grouped bf16 GEMMs on the 5th-generation tensor cores: the SwiGLU expert
// GEMMs and the router score GEMM.
//
// The experts are FFNs (mhpq.cn article §1.1; wenxiaobai §二(一)4) in the
// SwiGLU form y = (silu(a W1^T) * (a W3^T)) W2^T; the routed experts run on
// their dispatched rows and the shared expert on every token, all in one
// persistent launch per GEMM:
//   GEMM1  [rows_g, d] x [d, 2f] -> SwiGLU epilogue -> H [rows_g, f] (bf16)
//   GEMM2  [rows_g, f] x [f, d]  -> Y [rows_g, d] (bf16)
// Group g < N is routed expert g (rows offsets[g]..offsets[g+1]); group N is
// the shared expert (T rows).
//
// Work unit: a 128 x 256 output tile (tcgen05.mma cta_group::1, M=128,
// N=256, K=16 per instruction; M=64 when an expert's last tile has at most
// 64 rows), ordered group-major, then n-tile, then
// m-tile, so CTAs running side by side share the same weight tile through
// L2 and each expert's weights stream from HBM about once.  Each CTA (one
// per SM) walks tiles blockIdx.x, +gridDim.x, ... with three roles:
//   warp 0    one thread issues TMA loads of 64-wide K slices of A and B
//             (128-byte swizzle) into a 4-stage shared-memory ring;
//   warp 1    allocates 512 TMEM columns (two 256-column accumulators) and
//             one thread issues the MMAs, committing each ring slot back to
//             the producer and each finished accumulator to the epilogue;
//   warps 2-5 drain an accumulator with tcgen05.ld (one TMEM lane = one
//             output row per thread) while the next tile accumulates in the
//             other buffer, apply SwiGLU (GEMM1), round to bf16 and store
//             the rows that belong to the group.
// In GEMM1 the packed weight rows hold, per 128-row block j, W1 rows then
// W3 rows, so one accumulator tile holds matching gate and up columns.
// Every mbarrier wait is bounded (~2 s); a wait that gives up sets the
// device status word and the CTA unwinds, frees its TMEM and returns.
//
// The same kernel computes the router scores z = x . e_i (one group of T
// rows, tile width N): the fp32 router matrix is split exactly into three
// bf16 parts R = R0 + R1 + R2 (R0 = bf16(R), R1 = bf16(R - R0), R2 =
// bf16(R - R0 - R1), residual below 2^-27 |R|), stored as one [N, 3d]
// operand whose 64-column blocks run (R0, R1, R2) per 64 columns of d; each
// A tile of x is used for three consecutive K blocks (a_rep = 3), so the
// fp32 accumulator receives x.R0 + x.R1 + x.R2 = x.R.  With only T/128 token
// tiles, the 3d-long K loop is split into k_splits ranges run by separate
// units (the n-tile index carries the split); each writes its fp32 partial
// z to its own [T, N] slab, and the selection kernel adds the slabs in split
// order (deterministic) before the sigmoid.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>

#include <cstdlib>
#include <cstring>
#include <mutex>

#include "epilogue.cuh"
#include "internal.h"
#include "ptx.cuh"

namespace moe {
namespace {

constexpr int BM = 128, BK = 64;  // BK bf16 = 128 bytes = one swizzle row
constexpr int kStages = 4;
constexpr int kABytes = BM * BK * 2;
constexpr int kThreads = 192;
constexpr uint64_t kTimeoutNs = 2000000000ull;

enum Epi { kEpiSwiGLU = 0, kEpiStore = 1, kEpiScores = 2, kEpiSwiGLUBwd = 3,
           kEpiStoreCombine = 4 };

// Row-store epilogues (GEMM1 h, GEMM2 y) write full 32-row groups by TMA:
// per epilogue warp two 2 KB pieces (32 rows x 32 bf16 columns) of shared
// memory in the TMA's 64-byte swizzle, one filled while the other is stored.
constexpr int kOutPiece = 2048;
constexpr int kOutStgBytes = 4 * 2 * kOutPiece;
template <int kEpi, int kBN>
__host__ __device__ constexpr bool tma_out() {
  return (kEpi == kEpiStore || kEpi == kEpiSwiGLU) && kBN == 256;
}

template <int kBN>
struct TileCfg {
  static constexpr int kBBytes = kBN * BK * 2;
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kTmemCols = 2 * kBN;  // two accumulators
  static constexpr size_t smem_bytes(int groups, bool gather, bool staging) {
    return 1024 + (size_t)kStages * kStageBytes + (staging ? kOutStgBytes : 0) + 256 +
           (gather ? (size_t)BM * 8 : 0) + (size_t)(groups + 1) * 4;
  }
};

struct alignas(64) GemmArgs {
  CUtensorMap tmA_routed;  // routed rows (unused when a_rows is set)
  CUtensorMap tmA_shared;
  CUtensorMap tmB;
  CUtensorMap tmOut_routed;  // row-store epilogues: out_routed [rows_routed, out_ld] bf16 and
  CUtensorMap tmOut_shared;  // out_shared [T, out_ld], box {32, 32}, 64-byte swizzle
  int out_tma;               // 1: the two maps above are valid (set by the launcher)
  const int32_t* offsets;
  const int32_t* a_rows;  // when set: routed A row r of a group is a_src row a_rows[offsets[g] + r]
  const __nv_bfloat16* a_src;  // gathered rows' source (x), a_ld elements per row
  int a_ld;
  __nv_bfloat16* out_routed;
  __nv_bfloat16* out_shared;
  float* out_f32;   // score epilogue: fp32 partial sums [k_splits, T, n_valid]
  // SwiGLU-backward epilogue: the stored gate/up products [rows, 2f] (packed
  // like W13: per 128 features, gate columns then up columns), routed rows at
  // offsets[g] + r of aux_routed, shared-expert rows r of aux_shared
  const __nv_bfloat16* aux_routed;
  const __nv_bfloat16* aux_shared;
  uint32_t* status;
  // store-and-combine epilogue (GEMM2 with the COMBINE step fused): the
  // token of every routed row, each token's K slots and gates, the output y
  // [T, d], and one arrival counter per (token, 256-column tile), zero on entry
  const int32_t* perm_tok;
  const int32_t* slot;
  const float* gate;
  __nv_bfloat16* y;
  int32_t* arrive;
  int K;
  int shared_first;  // 1: the shared expert's tiles come before the routed ones
  int N, T;
  int rows_routed;  // T*K
  int a_shared_row0;
  int n_acc;   // accumulator columns per expert (2f for GEMM1, d for GEMM2)
  int k_dim;   // contraction length
  int out_ld;  // output row stride in elements
  int a_rep;   // K blocks that reuse one A tile (3 for the split router, else 1)
  int n_valid; // columns to store (score epilogue)
  int k_splits; // K ranges computed by separate units (score epilogue; else 1)
};

// COMBINE fused into GEMM2's epilogue (the mhpq.cn article §2.2 runs
// DISPATCH -> MLP -> COMBINE as one chunk): after storing its row's 256
// columns of y_perm (or y_shared), a thread counts one arrival for (token,
// column tile).  A token has K routed rows and its shared-expert row; the
// K+1-th arrival sees every one of them stored, and its warp then forms
//   y[t, cols] = y_shared[t] + sum_k gate[t,k] * y_perm[slot[t,k]]
// in k order with fp32 fused multiply-adds and one bf16 rounding -- the same
// operations, in the same order, as the standalone combine kernel, so the
// result is bit-identical.  Each lane handles 8 of the tile's 256 columns.
// The rows are read through L2 (ld.global.cg): they were written by other
// CTAs, made visible by the writers' fence before their counter increment and
// ordered after the last increment by the reader's fence.
__device__ __forceinline__ void combine_arrivals(const GemmArgs& args, int g, int n, int r,
                                                 bool valid, int lane) {
  const int NTd = args.n_acc / 256;
  int tok = -1;
  if (valid) {
    tok = (g < args.N) ? args.perm_tok[args.offsets[g] + r] : r;
    if (tok < 0 || tok >= args.T) {
      atomicOr(args.status, kErrBadIndex);
      tok = -1;
    }
  }
  bool last = false;
  if (tok >= 0) {
    __threadfence();
    last = atomicAdd(&args.arrive[(size_t)tok * NTd + n], 1) == args.K;
  }
  unsigned mask = __ballot_sync(0xffffffffu, last);
  if (mask == 0u) return;
  __threadfence();
  const int d = args.n_acc;
  const int col = n * 256 + 8 * lane;
  const long long TK = (long long)args.T * args.K;
  constexpr int kBatch = 8;  // rows whose loads are in flight together
  while (mask) {
    const int src = __ffs(mask) - 1;
    mask &= mask - 1u;
    const int t = __shfl_sync(0xffffffffu, tok, src);
    // lanes 0..K-1 fetch the token's slots and gates once (kMaxK <= 32)
    int my_sl = 0;
    float my_g = 0.f;
    if (lane < args.K) {
      const int sl = __ldg(args.slot + (size_t)t * args.K + lane);
      const bool ok = sl >= 0 && sl < TK;  // a slot outside the rows adds nothing
      my_sl = ok ? sl : 0;
      my_g = ok ? __ldg(args.gate + (size_t)t * args.K + lane) : 0.f;
    }
    float acc[8];
    const uint4 sh = __ldcg(reinterpret_cast<const uint4*>(args.out_shared + (size_t)t * d + col));
    for (int k0 = 0; k0 < args.K; k0 += kBatch) {
      uint4 rv[kBatch];
#pragma unroll
      for (int j = 0; j < kBatch; ++j) {
        const int sl = __shfl_sync(0xffffffffu, my_sl, (k0 + j) & 31);
        if (k0 + j < args.K)
          rv[j] = __ldcg(reinterpret_cast<const uint4*>(args.out_routed + (size_t)sl * d + col));
      }
      if (k0 == 0) bf16x8_unpack(sh, acc);
#pragma unroll
      for (int j = 0; j < kBatch; ++j) {
        const float gk = __shfl_sync(0xffffffffu, my_g, (k0 + j) & 31);
        if (k0 + j < args.K) {
          float r8[8];
          bf16x8_unpack(rv[j], r8);
#pragma unroll
          for (int i = 0; i < 8; ++i) acc[i] = fmaf(gk, r8[i], acc[i]);
        }
      }
    }
    uint4 o;
    __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&o);
#pragma unroll
    for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(acc[2 * i], acc[2 * i + 1]);
    *reinterpret_cast<uint4*>(args.y + (size_t)t * d + col) = o;
  }
}

template <int kEpi, int kBN, bool kGather>
__global__ void __launch_bounds__(kThreads, 1) grouped_gemm_bf16_kernel(
    const __grid_constant__ GemmArgs args) {
  constexpr int BN = kBN;
  constexpr int kBBytes = TileCfg<kBN>::kBBytes;
  constexpr int kStageBytes = TileCfg<kBN>::kStageBytes;
  constexpr int kTmemCols = TileCfg<kBN>::kTmemCols;
  static_assert(kEpi != kEpiSwiGLU || kBN == 256, "SwiGLU tiles pair 128 gate + 128 up columns");
  (void)kBBytes;
  constexpr bool kTmaOut = tma_out<kEpi, kBN>();
  constexpr size_t kStg = kTmaOut ? kOutStgBytes : 0;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* staging = base + (size_t)kStages * kStageBytes;  // 1024-aligned
  (void)staging;
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + (size_t)kStages * kStageBytes + kStg);
  uint64_t* full = bars;                 // [kStages]
  uint64_t* empty = bars + kStages;      // [kStages]
  uint64_t* tfull = bars + 2 * kStages;  // [2]
  uint64_t* tempty = tfull + 2;          // [2]
  uint64_t* drain = tempty + 2;          // [1]
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
  // gathered tiles: the source address of each of the tile's 128 rows
  const char** rowptr =
      reinterpret_cast<const char**>(base + (size_t)kStages * kStageBytes + kStg + 256);
  int* tile_start = reinterpret_cast<int*>(base + (size_t)kStages * kStageBytes + kStg + 256 +
                                           (kGather ? BM * 8 : 0));

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const bool clock_cta = kEpi != kEpiScores && blockIdx.x == 0 && tid == 0 && args.status;
  ClockMark cm{};
  if (clock_cta) cm = clock_start();
  const int G1 = args.N + 1;
  const int NT = (args.n_acc / BN) * args.k_splits;  // n-tiles x K splits
  const int KB = args.k_dim / BK;
  const int KBs = (KB + args.k_splits - 1) / args.k_splits;  // K blocks per split

  // ---- set-up: barriers, TMEM, tile schedule --------------------------------
  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      // with gathered rows every producer lane also arrives once per stage,
      // when its row copies have landed
      mbar_init(&full[s], kGather ? 33 : 1);
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
  // tiles are laid out group by group in schedule position order; position p
  // holds group p, or with shared_first group (p + N) mod (N + 1): the shared
  // expert first, then the routed experts in order
  auto group_at = [&](int p) { return args.shared_first ? (p + args.N) % G1 : p; };
  for (int p = tid; p < G1; p += kThreads) {
    const int g = group_at(p);
    const int rows = (g < args.N) ? args.offsets[g + 1] - args.offsets[g] : args.T;
    tile_start[p] = rows > 0 ? (rows + BM - 1) / BM : 0;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) {  // exclusive scan of m-tiles per group, times NT
    const int per = (G1 + 31) / 32;
    const int g0 = min(G1, lane * per), g1 = min(G1, g0 + per);
    int sum = 0;
    for (int g = g0; g < g1; ++g) sum += tile_start[g];
    int inc = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, inc, o);
      if (lane >= o) inc += v;
    }
    int run = inc - sum;
    for (int g = g0; g < g1; ++g) {
      const int mt = tile_start[g];
      tile_start[g] = run * NT;
      run += mt;
    }
    if (lane == 31) tile_start[G1] = inc * NT;
  }
  __syncthreads();
  const uint32_t tmem_base = *tmem_holder;
  const int total = tile_start[G1];

  auto decode = [&](int tile, int& g, int& n, int& m, int& mt) {
    int lo = 0, hi = G1;
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (tile_start[mid] <= tile) lo = mid; else hi = mid;
    }
    g = group_at(lo);
    mt = (tile_start[lo + 1] - tile_start[lo]) / NT;
    const int local = tile - tile_start[lo];
    n = local / mt;
    m = local - n * mt;
  };

  if (warp == 0) {
    if constexpr (!kGather) {
      // ---- TMA producer ---------------------------------------------------------
      if (lane == 0) {
        tma_prefetch_desc(&args.tmA_routed);
        tma_prefetch_desc(&args.tmA_shared);
        tma_prefetch_desc(&args.tmB);
        int stage = 0;
        uint32_t phase = 0;
        uint32_t issued = 0, issued_parity = 0;
        bool ok = true;
        for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
          int g, n, m, mt;
          decode(tile, g, n, m, mt);
          const CUtensorMap* am = (g < args.N) ? &args.tmA_routed : &args.tmA_shared;
          const int arow = ((g < args.N) ? args.offsets[g] : args.a_shared_row0) + m * BM;
          const int brow = g * args.n_acc + (n / args.k_splits) * BN;
          const int kb0 = (n % args.k_splits) * KBs, kb1 = min(KB, kb0 + KBs);
          for (int kb = kb0; kb < kb1; ++kb) {
            if (!mbar_wait_bounded(&empty[stage], phase ^ 1u, args.status, kTimeoutNs)) {
              ok = false;
              break;
            }
            uint8_t* sa = base + (size_t)stage * kStageBytes;
            mbar_arrive_expect_tx(&full[stage], kStageBytes);
            tma_load_2d(sa, am, (kb / args.a_rep) * BK, arow, &full[stage]);
            tma_load_2d(sa + kABytes, &args.tmB, kb * BK, brow, &full[stage]);
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
    } else {
      // ---- TMA producer (gathered routed rows) -----------------------------------
      // Lane 0 waits, arms the barrier and loads B (and A for contiguous rows)
      // by TMA.  With a_rows set, the warp gathers a routed tile's 128 token
      // rows itself: per stage 32 cp.async instructions of 16 bytes per lane,
      // four rows of 128 bytes each, written in the 128-byte swizzled layout the
      // MMA reads (16-byte chunk c of row r at chunk c ^ (r mod 8)); each lane's
      // copies complete on the stage's barrier, and no permuted copy of x exists.
      if (lane == 0) {
        tma_prefetch_desc(&args.tmA_routed);
        tma_prefetch_desc(&args.tmA_shared);
        tma_prefetch_desc(&args.tmB);
      }
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued = 0, issued_parity = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
        int g, n, m, mt;
        decode(tile, g, n, m, mt);
        const bool gather = g < args.N;
        const CUtensorMap* am = (g < args.N) ? &args.tmA_routed : &args.tmA_shared;
        const int arow = ((g < args.N) ? args.offsets[g] : args.a_shared_row0) + m * BM;
        const int brow = g * args.n_acc + (n / args.k_splits) * BN;
        const int kb0 = (n % args.k_splits) * KBs, kb1 = min(KB, kb0 + KBs);
        if (gather) {  // rows past the group's end read token 0; they are never stored
          __syncwarp();
          const int rows_g = args.offsets[g + 1] - args.offsets[g];
  #pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int rr = 4 * lane + j;
            const int row = m * BM + rr;
            int t = row < rows_g ? args.a_rows[args.offsets[g] + row] : 0;
            if (t < 0 || t >= args.T) t = 0;
            rowptr[rr] = reinterpret_cast<const char*>(args.a_src + (size_t)t * args.a_ld);
          }
          __syncwarp();
        }
        for (int kb = kb0; kb < kb1; ++kb) {
          bool got = true;
          if (lane == 0) got = mbar_wait_bounded(&empty[stage], phase ^ 1u, args.status, kTimeoutNs);
          if (!__shfl_sync(0xffffffffu, got ? 1 : 0, 0)) {
            ok = false;
            break;
          }
          uint8_t* sa = base + (size_t)stage * kStageBytes;
          if (lane == 0) {
            mbar_arrive_expect_tx(&full[stage], gather ? kBBytes : kStageBytes);
            if (!gather) tma_load_2d(sa, am, (kb / args.a_rep) * BK, arow, &full[stage]);
            tma_load_2d(sa + kABytes, &args.tmB, kb * BK, brow, &full[stage]);
          }
          if (args.a_rows != nullptr) {
            if (gather) {
              const int c = lane & 7;
              const int koff = (kb * BK + c * 8) * 2;  // byte offset of this lane's chunk
  #pragma unroll 8
              for (int i = 0; i < BM / 4; ++i) {
                const int r = 4 * i + (lane >> 3);
                cp_async_16(sa + r * (BK * 2) + ((c ^ (r & 7)) << 4), rowptr[r] + koff);
              }
            }
            cp_async_mbar_arrive_noinc(&full[stage]);
          }
          issued |= 1u << stage;
          issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok && lane == 0) {  // let the copies already issued land before the CTA exits
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
      for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x, ++local) {
        int g, n, m, mt;
        decode(tile, g, n, m, mt);
        const int kb0 = (n % args.k_splits) * KBs, kb1 = min(KB, kb0 + KBs);
        // a tile with at most 64 real rows (an expert's ragged tail) runs the
        // M=64 MMA: the tensor pipe takes as long as for M=128 (tcgen05
        // issue-rate probe), but half the products are computed and drained
        const int rows_g = (g < args.N) ? args.offsets[g + 1] - args.offsets[g] : args.T;
        const uint32_t idesc = idesc_bf16_f32(rows_g - m * BM <= 64 ? 64 : BM, kBN);
        const int acc = local & 1;
        const uint32_t aphase = (local >> 1) & 1;
        if (!mbar_wait_bounded(&tempty[acc], aphase ^ 1u, args.status, kTimeoutNs)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait_bounded(&full[stage], phase, args.status, kTimeoutNs)) {
            ok = false;
            break;
          }
          // rows copied by the producer lanes are generic-proxy writes
          if constexpr (kGather) fence_proxy_async_smem();
          tc_fence_after();
          const uint32_t a0 = smem_u32(base + (size_t)stage * kStageBytes);
          const uint32_t b0 = a0 + kABytes;
#pragma unroll
          for (int k = 0; k < BK / 16; ++k)
            mma_bf16(d_tmem, smem_desc_sw128(a0 + k * 32), smem_desc_sw128(b0 + k * 32), idesc,
                     ((kb - kb0) | k) != 0);
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
    const int q = warp & 3;  // TMEM lane quadrant this warp may access
    const int row = q * 32 + lane;
    int local = 0;
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x, ++local) {
      int g, n, m, mt;
      decode(tile, g, n, m, mt);
      const int acc = local & 1;
      const uint32_t aphase = (local >> 1) & 1;
      if (!mbar_wait_bounded(&tfull[acc], aphase, args.status, kTimeoutNs)) break;
      tc_fence_after();
      const int rows_g = (g < args.N) ? args.offsets[g + 1] - args.offsets[g] : args.T;
      // M=64 tiles (<= 64 rows) hold row 16*q + i in TMEM lane 32*q + i (i < 16)
      const bool m64 = rows_g - m * BM <= 64;
      const int r = m * BM + (m64 ? (lane < 16 ? 16 * q + lane : BM) : row);
      // rows past the group's end belong to the next group (or are padding);
      // the second test keeps a corrupted offsets[] from writing out of range
      const bool valid = r < rows_g && (g == args.N || args.offsets[g] + r < args.rows_routed);
      __nv_bfloat16* orow =
          (g < args.N) ? args.out_routed + (size_t)(args.offsets[g] + r) * args.out_ld
                       : args.out_shared + (size_t)r * args.out_ld;
      const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + acc * BN;
      // a warp whose 32 rows (of a 128-row tile) all lie inside the group
      // stores them by TMA; the others take the row stores
      bool tma_rows = false;
      const CUtensorMap* omap = (g < args.N) ? &args.tmOut_routed : &args.tmOut_shared;
      const int orow0 = ((g < args.N) ? args.offsets[g] : 0) + m * BM + q * 32;
      if constexpr (kTmaOut) {
        const int r0 = m * BM + q * 32;
        tma_rows = args.out_tma != 0 && !m64 && r0 + 32 <= rows_g &&
                   (g == args.N || args.offsets[g] + r0 + 32 <= args.rows_routed);
      }
      // one 32-column piece of this warp's rows -> staging -> TMA store
      auto store_piece = [&](const float* y, int piece, int col) {
        uint8_t* buf = staging + (size_t)(warp - 2) * (2 * kOutPiece) + (piece & 1) * kOutPiece;
        if (lane == 0) bulk_wait_read_but_one();  // the store that last read buf is done
        __syncwarp();
        uint8_t* my = buf + lane * 64;
        const int sw = (lane >> 1) & 3;  // the 64-byte swizzle of row `lane`
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) {
          const float* a = y + 8 * c4;
          *reinterpret_cast<uint4*>(my + ((c4 ^ sw) << 4)) =
              make_uint4(bf16x2_bits(a[0], a[1]), bf16x2_bits(a[2], a[3]),
                         bf16x2_bits(a[4], a[5]), bf16x2_bits(a[6], a[7]));
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_2d(omap, buf, col, orow0);
          bulk_commit_group();
        }
      };
      (void)store_piece;
      (void)omap;
      (void)orow0;
      if constexpr (kEpi == kEpiSwiGLU) {
#pragma unroll 1
        for (int c = 0; c < BN / 2; c += 32) {
          uint32_t ga[32], up[32];
          tmem_ld32(taddr + c, ga);
          tmem_ld32(taddr + BN / 2 + c, up);
          tmem_wait_ld();
          float h[32];
#pragma unroll
          for (int i = 0; i < 32; ++i)
            h[i] = silu_fast(__uint_as_float(ga[i])) * __uint_as_float(up[i]);
          if (tma_rows)
            store_piece(h, c / 32, n * (BN / 2) + c);
          else if (valid)
            store_row32(orow + n * (BN / 2) + c, h);
        }
      } else if constexpr (kEpi == kEpiStore) {
#pragma unroll 1
        for (int c = 0; c < BN; c += 32) {
          uint32_t v[32];
          tmem_ld32(taddr + c, v);
          tmem_wait_ld();
          float y[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) y[i] = __uint_as_float(v[i]);
          if (tma_rows)
            store_piece(y, c / 32, n * BN + c);
          else if (valid)
            store_row32(orow + n * BN + c, y);
        }
      } else if constexpr (kEpi == kEpiStoreCombine) {
#pragma unroll 1
        for (int c = 0; c < BN; c += 32) {
          uint32_t v[32];
          tmem_ld32(taddr + c, v);
          tmem_wait_ld();
          float y[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) y[i] = __uint_as_float(v[i]);
          if (valid) store_row32(orow + n * BN + c, y);
        }
        // the accumulator is drained: hand it back before the combine work
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tempty[acc]);
        combine_arrivals(args, g, n, r, valid, lane);
        continue;
      } else if constexpr (kEpi == kEpiSwiGLUBwd) {
        // the accumulator is dh for hidden features n*BN + c; with g, u the
        // stored gate/up products: dg = dh * u * silu'(g), du = dh * silu(g),
        // written bf16 into the packed [rows, 2f] layout (gate block, up block)
        const __nv_bfloat16* arow =
            (g < args.N) ? args.aux_routed + (size_t)(args.offsets[g] + r) * args.out_ld
                         : args.aux_shared + (size_t)r * args.out_ld;
#pragma unroll 1
        for (int c = 0; c < BN; c += 32) {
          uint32_t v[32];
          tmem_ld32(taddr + c, v);
          tmem_wait_ld();
          const int j0 = n * BN + c;                       // first feature of the chunk
          const int col = (j0 / 128) * 256 + (j0 % 128);   // its gate column; up at +128
          if (valid) {
            float gt[32], up[32], dg[32], du[32];
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
              bf16x8_load(arow + col + 8 * q4, gt + 8 * q4);
              bf16x8_load(arow + col + 128 + 8 * q4, up + 8 * q4);
            }
#pragma unroll
            for (int i = 0; i < 32; ++i)
              swiglu_bwd(__uint_as_float(v[i]), gt[i], up[i], dg[i], du[i]);
            store_row32(orow + col, dg);
            store_row32(orow + col + 128, du);
          }
        }
      } else {  // raw fp32 scores of this K split, columns < n_valid
        float* srow = args.out_f32 +
                      ((size_t)(n % args.k_splits) * args.T + r) * args.n_valid;
#pragma unroll 1
        for (int c = 0; c < BN; c += 32) {
          uint32_t v[32];
          tmem_ld32(taddr + c, v);
          tmem_wait_ld();
          if (valid && c < args.n_valid) {
            if (c + 32 <= args.n_valid) {
#pragma unroll
              for (int i = 0; i < 32; i += 4)
                *reinterpret_cast<float4*>(srow + c + i) =
                    make_float4(__uint_as_float(v[i]), __uint_as_float(v[i + 1]),
                                __uint_as_float(v[i + 2]), __uint_as_float(v[i + 3]));
            } else {
#pragma unroll
              for (int i = 0; i < 32; ++i)
                if (c + i < args.n_valid) srow[c + i] = __uint_as_float(v[i]);
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[acc]);
    }
    // the staging buffers must outlive the stores that read them
    if constexpr (kTmaOut) {
      if (lane == 0) bulk_wait_all();
    }
  }

  // ---- teardown ------------------------------------------------------------------
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
  if (clock_cta)
    clock_stop(cm, reinterpret_cast<unsigned long long*>(
                       reinterpret_cast<uint8_t*>(args.status) + kClockRecordOffset));
}

template <int kEpi, int kBN, bool kGather = false>
cudaError_t launch_gemm(const GemmArgs& a0, cudaStream_t st) {
  constexpr bool kTmaOut = tma_out<kEpi, kBN>();
  const size_t smem = TileCfg<kBN>::smem_bytes(a0.N + 1, kGather, kTmaOut);
  cudaError_t e = note_cuda(cudaFuncSetAttribute(grouped_gemm_bf16_kernel<kEpi, kBN, kGather>,
                                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 (int)smem),
                            "bf16 GEMM: set shared-memory size");
  if (e != cudaSuccess) return e;
  GemmArgs a = a0;
  a.out_tma = 0;
  if constexpr (kTmaOut) {
    // TMA stores need 16-byte aligned outputs; otherwise every row takes the
    // row stores
    const auto BF = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    const bool aligned = (reinterpret_cast<uintptr_t>(a.out_routed) % 16 == 0) &&
                         (reinterpret_cast<uintptr_t>(a.out_shared) % 16 == 0) &&
                         ((size_t)a.out_ld * 2) % 16 == 0;
    if (aligned &&
        make_map_swizzled(&a.tmOut_routed, a.out_routed, BF, 2, a.out_ld, a.rows_routed, 32, 32,
                          CU_TENSOR_MAP_SWIZZLE_64B) &&
        make_map_swizzled(&a.tmOut_shared, a.out_shared, BF, 2, a.out_ld, a.T, 32, 32,
                          CU_TENSOR_MAP_SWIZZLE_64B))
      a.out_tma = 1;
  }
  grouped_gemm_bf16_kernel<kEpi, kBN, kGather><<<num_sms(), kThreads, smem, st>>>(a);
  return note_cuda(cudaGetLastError(), "bf16 GEMM launch");
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

namespace {
// The COMBINE step fused into GEMM2 (store-and-combine epilogue): null when
// the combine runs as its own kernel.
struct FusedCombine {
  const int32_t* perm_tok;
  const int32_t* slot;
  const float* gate;
  void* y;
};

int ffn_tc_bf16(const moe_shape& s, const void* x_perm, const int32_t* perm_tok,
                const int32_t* offsets, const void* x, const void* w13, const void* w2,
                void* y_perm, void* y_shared, void* ws, cudaStream_t st,
                const FusedCombine* fc);
}  // namespace

int launch_ffn_tc_bf16(const moe_shape& s, const void* x_perm, const int32_t* perm_tok,
                       const int32_t* offsets, const void* x, const void* w13, const void* w2,
                       void* y_perm, void* y_shared, void* ws, cudaStream_t st) {
  // MOE_BF16_GEMM selects the expert GEMM kernel: "dual" (two token tiles per
  // weight tile, gemm_dual.cu), "pair" (CTA pairs, gemm2sm.cu); default: this file's
  static const int kind = [] {
    const char* v = std::getenv("MOE_BF16_GEMM");
    if (v != nullptr && std::strcmp(v, "pair") == 0) return 2;
    if (v != nullptr && std::strcmp(v, "dual") == 0) return 1;
    return 0;
  }();
  // rows gathered from x through perm_tok always run on this file's kernel
  if (perm_tok == nullptr && kind == 2)
    return launch_ffn_tc_bf16_pair(s, x_perm, offsets, x, w13, w2, y_perm, y_shared, ws, st);
  if (perm_tok == nullptr && kind == 1)
    return launch_ffn_tc_bf16_dual(s, x_perm, offsets, x, w13, w2, y_perm, y_shared, ws, st);
  return ffn_tc_bf16(s, x_perm, perm_tok, offsets, x, w13, w2, y_perm, y_shared, ws, st,
                     nullptr);
}

int launch_ffn_combine_bf16(const moe_shape& s, const void* x_perm, const int32_t* offsets,
                            const int32_t* perm_tok, const int32_t* slot, const float* gate,
                            const void* x, const void* w13, const void* w2, void* y_perm,
                            void* y_shared, void* y, void* ws, cudaStream_t st) {
  const FusedCombine fc{perm_tok, slot, gate, y};
  return ffn_tc_bf16(s, x_perm, nullptr, offsets, x, w13, w2, y_perm, y_shared, ws, st, &fc);
}

namespace {
int ffn_tc_bf16(const moe_shape& s, const void* x_perm, const int32_t* perm_tok,
                const int32_t* offsets, const void* x, const void* w13, const void* w2,
                void* y_perm, void* y_shared, void* ws, cudaStream_t st,
                const FusedCombine* fc) {
  const WsLayout L = ws_layout(s);
  uint8_t* w = static_cast<uint8_t*>(ws);
  __nv_bfloat16* H = reinterpret_cast<__nv_bfloat16*>(w + L.h);
  const uint64_t TK = (uint64_t)s.T * s.K;
  const auto BF = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;

  GemmArgs g1{};
  // gathered rows are copied by the producer warp; the routed map is then unused
  bool ok = make_map(&g1.tmA_routed, perm_tok ? x : x_perm, BF, 2, s.d, perm_tok ? s.T : TK,
                     BK, BM) &&
            make_map(&g1.tmA_shared, x, BF, 2, s.d, s.T, BK, BM) &&
            make_map(&g1.tmB, w13, BF, 2, s.d, (uint64_t)(s.N + 1) * 2 * s.f, BK, 256);
  if (!ok) {
    note_text("bf16 GEMM: tensor-map encoding failed");
    return MOE_ERR_CUDA;
  }
  g1.offsets = offsets;
  g1.a_rows = perm_tok;
  g1.a_src = static_cast<const __nv_bfloat16*>(x);
  g1.a_ld = s.d;
  g1.out_routed = H;
  g1.out_shared = H + TK * s.f;
  g1.status = reinterpret_cast<uint32_t*>(w + L.status);
  g1.N = s.N;
  g1.T = s.T;
  g1.rows_routed = (int)TK;
  g1.a_shared_row0 = 0;
  g1.n_acc = 2 * s.f;
  g1.k_dim = s.d;
  g1.out_ld = s.f;
  g1.a_rep = 1;
  g1.k_splits = 1;
  if ((perm_tok ? launch_gemm<kEpiSwiGLU, 256, true>(g1, st)
                : launch_gemm<kEpiSwiGLU, 256>(g1, st)) != cudaSuccess)
    return MOE_ERR_CUDA;

  GemmArgs g2{};
  ok = make_map(&g2.tmA_routed, H, BF, 2, s.f, TK + s.T, BK, BM) &&
       make_map(&g2.tmA_shared, H, BF, 2, s.f, TK + s.T, BK, BM) &&
       make_map(&g2.tmB, w2, BF, 2, s.f, (uint64_t)(s.N + 1) * s.d, BK, 256);
  if (!ok) {
    note_text("bf16 GEMM: tensor-map encoding failed");
    return MOE_ERR_CUDA;
  }
  g2.offsets = offsets;
  g2.out_routed = static_cast<__nv_bfloat16*>(y_perm);
  g2.out_shared = static_cast<__nv_bfloat16*>(y_shared);
  g2.status = g1.status;
  g2.N = s.N;
  g2.T = s.T;
  g2.rows_routed = (int)TK;
  g2.a_shared_row0 = (int)TK;
  g2.n_acc = s.d;
  g2.k_dim = s.f;
  g2.out_ld = s.d;
  g2.a_rep = 1;
  g2.k_splits = 1;
  if (fc == nullptr) {
    if (launch_gemm<kEpiStore, 256>(g2, st) != cudaSuccess) return MOE_ERR_CUDA;
    return MOE_OK;
  }
  // store-and-combine: arrival counters start at zero; the shared expert's
  // tiles go first so each token completes with its last routed row
  int32_t* arrive = reinterpret_cast<int32_t*>(w + L.arrive);
  if (note_cuda(cudaMemsetAsync(arrive, 0, (size_t)s.T * (s.d / 256) * sizeof(int32_t), st),
                "fused combine: clear arrival counters") != cudaSuccess)
    return MOE_ERR_CUDA;
  g2.perm_tok = fc->perm_tok;
  g2.slot = fc->slot;
  g2.gate = fc->gate;
  g2.y = static_cast<__nv_bfloat16*>(fc->y);
  g2.arrive = arrive;
  g2.K = s.K;
  g2.shared_first = 1;
  if (launch_gemm<kEpiStoreCombine, 256>(g2, st) != cudaSuccess) return MOE_ERR_CUDA;
  return MOE_OK;
}
}  // namespace

int router_k_splits(const moe_shape& s) {
  const int m_tiles = (s.T + BM - 1) / BM;
  const int KB = 3 * s.d / BK;
  int want = num_sms() / m_tiles;  // fill the SMs with token tiles x K splits
  want = want < 1 ? 1 : (want > 8 ? 8 : want);
  while (want > 1 && KB % want != 0) --want;
  return want;
}

int launch_router_scores_tc(const moe_shape& s, const void* x, const float* router, float* Z,
                            int k_splits, void* ws, cudaStream_t st) {
  const WsLayout L = ws_layout(s);
  uint8_t* w = static_cast<uint8_t*>(ws);
  __nv_bfloat16* Rs = reinterpret_cast<__nv_bfloat16*>(w + L.router_split);
  const long long total = (long long)s.N * s.d;
  long long blocks = (total + 255) / 256;
  if (blocks > 148 * 8) blocks = 148 * 8;
  router_split_kernel<<<(int)blocks, 256, 0, st>>>(router, s.N, s.d, Rs);
  if (cudaGetLastError() != cudaSuccess) return MOE_ERR_CUDA;

  const int bn = s.N <= 64 ? 64 : (s.N <= 128 ? 128 : 256);
  GemmArgs a{};
  const auto BF = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  bool ok = make_map(&a.tmA_routed, x, BF, 2, s.d, s.T, BK, BM) &&
            make_map(&a.tmA_shared, x, BF, 2, s.d, s.T, BK, BM) &&
            make_map(&a.tmB, Rs, BF, 2, 3ull * s.d, s.N, BK, bn);
  if (!ok) {
    note_text("bf16 GEMM: tensor-map encoding failed");
    return MOE_ERR_CUDA;
  }
  a.offsets = nullptr;
  a.out_f32 = Z;
  a.status = reinterpret_cast<uint32_t*>(w + L.status);
  a.N = 0;  // a single group: all T rows of x
  a.T = s.T;
  a.rows_routed = 0;
  a.a_shared_row0 = 0;
  a.n_acc = bn;
  a.k_dim = 3 * s.d;
  a.out_ld = s.N;
  a.a_rep = 3;
  a.n_valid = s.N;
  a.k_splits = k_splits;
  cudaError_t e = bn == 64    ? launch_gemm<kEpiScores, 64>(a, st)
                  : bn == 128 ? launch_gemm<kEpiScores, 128>(a, st)
                              : launch_gemm<kEpiScores, 256>(a, st);
  return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

// Backward of the expert FFNs, input gradients ([P1] §2.2 MLP_B), bf16:
//   GU  = [x_perm | x] W13^T      (GEMM1 recomputed, gate/up stored bf16)
//   dGU = SwiGLU'(dY W2, GU)      (dH in fp32 in TMEM; dg, du bf16 per feature)
//   dX  = dGU W13                 (against W13^T, K = 2f)
// Three launches of the grouped kernel; W2^T and W13^T come from
// moe_transpose_weights.  ws_bwd (bwd_layout): status word, GU and dGU, which
// the weight-gradient pass (gemm_wgrad.cu) reads afterwards.
BwdLayout bwd_layout(const moe_shape& s) {
  auto al = [](size_t v) { return (v + 255) & ~size_t(255); };
  BwdLayout B;
  const size_t rows = (size_t)s.T * s.K + s.T;
  const size_t R = (size_t)wgrad_cols(s);
  size_t off = 256;
  B.gu = off;
  off = al(off + rows * 2 * s.f * 2);
  B.dgu = off;
  off = al(off + rows * 2 * s.f * 2);
  B.colbase = off;
  off = al(off + (size_t)(s.N + 2) * 4);
  B.at = off;
  off = al(off + (size_t)s.d * R * 2);
  B.dyt = off;
  off = al(off + (size_t)s.d * R * 2);
  B.ht = off;
  off = al(off + (size_t)s.f * R * 2);
  B.dgut = off;
  off = al(off + (size_t)2 * s.f * R * 2);
  B.total = off;
  return B;
}

size_t backward_ws_bytes(const moe_shape& s) { return bwd_layout(s).total; }

int launch_ffn_bwd_dx_bf16(const moe_shape& s, const void* x_perm, const int32_t* offsets,
                           const void* x, const void* w13, const void* w13t, const void* w2t,
                           const void* dy_perm, const void* dy_shared, void* dx_perm,
                           void* dx_shared, void* ws_bwd, cudaStream_t st) {
  uint8_t* w = static_cast<uint8_t*>(ws_bwd);
  const uint64_t TK = (uint64_t)s.T * s.K;
  const size_t rows = TK + s.T;
  const BwdLayout B = bwd_layout(s);
  __nv_bfloat16* GU = reinterpret_cast<__nv_bfloat16*>(w + B.gu);
  __nv_bfloat16* dGU = reinterpret_cast<__nv_bfloat16*>(w + B.dgu);
  uint32_t* status = reinterpret_cast<uint32_t*>(w);
  const auto BF = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const uint64_t twof = 2ull * s.f;

  auto base_args = [&](GemmArgs& a) {
    a.offsets = offsets;
    a.status = status;
    a.N = s.N;
    a.T = s.T;
    a.rows_routed = (int)TK;
    a.a_rep = 1;
    a.k_splits = 1;
  };
  // 1. GU = A W13^T (routed rows from x_perm, shared rows from x)
  GemmArgs g1{};
  bool ok = make_map(&g1.tmA_routed, x_perm, BF, 2, s.d, TK, BK, BM) &&
            make_map(&g1.tmA_shared, x, BF, 2, s.d, s.T, BK, BM) &&
            make_map(&g1.tmB, w13, BF, 2, s.d, (uint64_t)(s.N + 1) * twof, BK, 256);
  // 2. dH = dY W2 (B = W2^T, [f, d] per expert), SwiGLU-backward epilogue -> dGU
  GemmArgs g2{};
  ok = ok && make_map(&g2.tmA_routed, dy_perm, BF, 2, s.d, TK, BK, BM) &&
       make_map(&g2.tmA_shared, dy_shared, BF, 2, s.d, s.T, BK, BM) &&
       make_map(&g2.tmB, w2t, BF, 2, s.d, (uint64_t)(s.N + 1) * s.f, BK, 256);
  // 3. dX = dGU W13 (B = W13^T, [d, 2f] per expert)
  GemmArgs g3{};
  ok = ok && make_map(&g3.tmA_routed, dGU, BF, 2, twof, rows, BK, BM) &&
       make_map(&g3.tmA_shared, dGU, BF, 2, twof, rows, BK, BM) &&
       make_map(&g3.tmB, w13t, BF, 2, twof, (uint64_t)(s.N + 1) * s.d, BK, 256);
  if (!ok) {
    note_text("expert backward: tensor-map encoding failed");
    return MOE_ERR_CUDA;
  }
  base_args(g1);
  g1.out_routed = GU;
  g1.out_shared = GU + TK * twof;
  g1.a_shared_row0 = 0;
  g1.n_acc = (int)twof;
  g1.k_dim = s.d;
  g1.out_ld = (int)twof;
  if (launch_gemm<kEpiStore, 256>(g1, st) != cudaSuccess) return MOE_ERR_CUDA;

  base_args(g2);
  g2.aux_routed = GU;
  g2.aux_shared = GU + TK * twof;
  g2.out_routed = dGU;
  g2.out_shared = dGU + TK * twof;
  g2.a_shared_row0 = 0;
  g2.n_acc = s.f;
  g2.k_dim = s.d;
  g2.out_ld = (int)twof;
  if (launch_gemm<kEpiSwiGLUBwd, 256>(g2, st) != cudaSuccess) return MOE_ERR_CUDA;

  base_args(g3);
  g3.out_routed = static_cast<__nv_bfloat16*>(dx_perm);
  g3.out_shared = static_cast<__nv_bfloat16*>(dx_shared);
  g3.a_shared_row0 = (int)TK;
  g3.n_acc = s.d;
  g3.k_dim = (int)twof;
  g3.out_ld = s.d;
  if (launch_gemm<kEpiStore, 256>(g3, st) != cudaSuccess) return MOE_ERR_CUDA;
  return MOE_OK;
}

}  // namespace moe
