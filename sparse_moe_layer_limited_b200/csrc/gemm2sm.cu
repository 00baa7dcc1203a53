// bf16 expert GEMMs on CTA pairs (tcgen05 cta_group::2), one unit per
// (expert, weight tile) covering all of the expert's rows.
//
// Same computation as the one-CTA kernel in gemm_tc.cu (the SwiGLU expert FFN
// of the mhpq.cn article §1.1; GEMM1 with the SwiGLU epilogue, then GEMM2),
// arranged so that no weight byte is fetched twice:
//   * the weights are the MMA's M side: 256 weight rows of one expert per unit,
//     128 in each CTA of the pair;
//   * the tokens are the N side: all of the expert's rows (up to 512) in the
//     same unit, as one or two tcgen05.mma.cta_group::2 per K step (N up to
//     256 each, rounded up to 16 only), written to TMEM columns equal to the
//     token index; each CTA stages half of every MMA's token rows (64-row TMA
//     boxes, only as many as the unit needs);
//   * so a unit streams its weight tile once, a ragged expert costs MMA work in
//     proportion to its rows, and token bytes are split between the pair.
// The accumulator takes all 512 TMEM columns, so the epilogue of one unit does
// not overlap the next unit's MMAs; eight epilogue warps (two per TMEM lane
// quadrant, alternate 32-token chunks) keep that drain short.
// GEMM1 pairing: CTA rank r loads W1 rows 128j+64r..+63 into its TMEM lanes
// 0-63 and the W3 rows of the same hidden features into lanes 64-127 (two
// 64-row boxes of the 128-row-interleaved W13), so each CTA produces 64
// complete hidden features; the up values cross from the lane quadrants 2/3
// to 0/1 through shared memory.
// Roles per CTA: warp 0 TMA producer; warp 1 TMEM owner (both CTAs allocate
// 512 columns with cta_group::2) and, in the leader CTA, the single thread
// that issues the pair MMAs and multicasts the commits to both CTAs' barriers;
// warps 2-9 epilogue.  Loads of both CTAs complete on the leader's "full"
// barrier; "TMEM empty" lives on the leader and counts the 16 epilogue warps
// of the pair.  Every wait is bounded (~2 s); both CTAs always reach the final
// cluster barrier, so neither exits while its peer may still signal it.
#include <cuda.h>
#include <cuda_bf16.h>

#include "internal.h"
#include "ptx.cuh"

namespace moe {
namespace {

constexpr int PW = 128;      // weight rows per CTA (pair: 256)
constexpr int PT = 512;      // max token rows per unit (pair)
constexpr int PK = 64;       // bf16 K slice (128 bytes)
constexpr int PBox = 64;     // token rows per TMA box
constexpr int PStages = 4;
constexpr int PWBytes = PW * PK * 2;              // 16 KB of weights per CTA and stage
constexpr int PRegionBytes = 128 * PK * 2;        // up to 128 token rows per MMA and CTA
constexpr int PBoxBytes = PBox * PK * 2;          // 8 KB
constexpr int PStageBytes = PWBytes + 2 * PRegionBytes;  // 48 KB
constexpr int PThreads = 320;                     // warps 0, 1, then 8 epilogue warps
constexpr uint64_t PTimeoutNs = 2000000000ull;
constexpr int PXchgFloats = 2 * 32 * 64;          // one 32-token x 64-feature buffer per half

enum PEpi { kPSwiGLU = 0, kPStore = 1 };

struct alignas(64) PairArgs {
  CUtensorMap tmW;          // weights [(N+1) * n_feat, k_dim]; box {64, 64} (GEMM1) or {64, 128}
  CUtensorMap tmX_routed;   // token rows, box {64, 64}
  CUtensorMap tmX_shared;
  const int32_t* offsets;
  __nv_bfloat16* out_routed;
  __nv_bfloat16* out_shared;
  uint32_t* status;
  int N, T;
  int rows_routed;
  int x_shared_row0;
  int n_feat;   // weight rows per group (2f for GEMM1, d for GEMM2)
  int k_dim;
  int out_ld;
};

constexpr size_t pair_smem_bytes(int groups) {
  return 1024 + (size_t)PStages * PStageBytes + 512 + (size_t)PXchgFloats * 4 +
         (size_t)(groups + 1) * 4;
}

__device__ __forceinline__ float silu_f(float v) { return v / (1.f + expf(-v)); }

// Token split of a unit: MMA 0 takes tokens [0, n0), MMA 1 tokens [256, 256 + n1);
// each CTA stages half of each.
struct TokSplit {
  int n0, n1;    // MMA widths (multiples of 16; n1 = 0 when the unit has <= 256 rows)
  int b0, b1;    // 64-row boxes per CTA for each MMA
};
__device__ __forceinline__ TokSplit tok_split(int ntok) {
  const int n = (ntok + 15) & ~15;
  TokSplit t;
  t.n0 = min(n, 256);
  t.n1 = n - t.n0;
  t.b0 = (t.n0 / 2 + PBox - 1) / PBox;
  t.b1 = (t.n1 / 2 + PBox - 1) / PBox;
  return t;
}

template <int kEpi>
__global__ void __launch_bounds__(PThreads, 1) pair_gemm_bf16_kernel(
    const __grid_constant__ PairArgs args) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + (size_t)PStages * PStageBytes);
  uint64_t* full = bars;                  // [PStages] (used in the leader)
  uint64_t* empty = bars + PStages;       // [PStages] (each CTA)
  uint64_t* tfull = bars + 2 * PStages;   // [1] (each CTA)
  uint64_t* tempty = tfull + 1;           // [1] (leader; 16 epilogue warps of the pair)
  uint64_t* xfull = tempty + 1;           // [2] per half: up values staged (2 warps)
  uint64_t* xempty = xfull + 2;           // [2] per half: up values consumed (2 warps)
  uint64_t* drain = xempty + 2;           // [1]
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
  float* xchg = reinterpret_cast<float*>(base + (size_t)PStages * PStageBytes + 512);
  int* unit_start = reinterpret_cast<int*>(xchg + PXchgFloats);

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const int G1 = args.N + 1;
  const int NF = args.n_feat / (2 * PW);
  const int KB = args.k_dim / PK;

  if (tid == 0) {
    for (int s = 0; s < PStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(tfull, 1);
    mbar_init(tempty, 16);
    for (int h = 0; h < 2; ++h) {
      mbar_init(&xfull[h], 2);
      mbar_init(&xempty[h], 2);
    }
    mbar_init(drain, 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc_2sm(tmem_holder, 512);
    tmem_relinquish_2sm();
  }
  for (int g = tid; g < G1; g += PThreads) {
    const int rows = (g < args.N) ? args.offsets[g + 1] - args.offsets[g] : args.T;
    unit_start[g] = rows > 0 ? (rows + PT - 1) / PT : 0;
  }
  tc_fence_before();
  __syncthreads();
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
  // both CTAs' barriers are initialised before either signals the other
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  const int total = unit_start[G1];

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
    // ---- TMA producer (both CTAs) ---------------------------------------------
    if (lane == 0) {
      tma_prefetch_desc(&args.tmW);
      tma_prefetch_desc(&args.tmX_routed);
      tma_prefetch_desc(&args.tmX_shared);
      int stage = 0;
      uint32_t phase = 0, issued = 0, issued_parity = 0;
      bool ok = true;
      for (int u = pair; u < total && ok; u += npairs) {
        int g, nf, mt;
        decode(u, g, nf, mt);
        const int ntok = min(PT, group_rows(g) - mt * PT);
        const TokSplit ts = tok_split(ntok);
        const CUtensorMap* xm = (g < args.N) ? &args.tmX_routed : &args.tmX_shared;
        const int row0 = ((g < args.N) ? args.offsets[g] : args.x_shared_row0) + mt * PT;
        const int r0 = row0 + (int)rank * (ts.n0 / 2);
        const int r1 = row0 + 256 + (int)rank * (ts.n1 / 2);
        const int wtile = g * args.n_feat + nf * 2 * PW;
        const uint32_t bytes = 2u * (PWBytes + (uint32_t)(ts.b0 + ts.b1) * PBoxBytes);
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait_bounded(&empty[stage], phase ^ 1u, args.status, PTimeoutNs)) {
            ok = false;
            break;
          }
          uint8_t* sw = base + (size_t)stage * PStageBytes;
          const uint32_t fbar = mapa_shared(smem_u32(&full[stage]), 0);
          if (leader) mbar_arrive_expect_tx(&full[stage], bytes);
          if constexpr (kEpi == kPSwiGLU) {
            // W1 rows 128j + 64r .. +63 (lanes 0-63), W3 rows of the same features (64-127)
            tma_load_2d_2sm(sw, &args.tmW, kb * PK, wtile + 64 * (int)rank, fbar);
            tma_load_2d_2sm(sw + PWBytes / 2, &args.tmW, kb * PK, wtile + PW + 64 * (int)rank,
                            fbar);
          } else {
            tma_load_2d_2sm(sw, &args.tmW, kb * PK, wtile + PW * (int)rank, fbar);
          }
          for (int i = 0; i < ts.b0; ++i)
            tma_load_2d_2sm(sw + PWBytes + i * PBoxBytes, xm, kb * PK, r0 + i * PBox, fbar);
          for (int i = 0; i < ts.b1; ++i)
            tma_load_2d_2sm(sw + PWBytes + PRegionBytes + i * PBoxBytes, xm, kb * PK,
                            r1 + i * PBox, fbar);
          issued |= 1u << stage;
          issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == PStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {  // the copies already issued complete on the leader's barriers
        if (leader)
          for (int s = 0; s < PStages; ++s)
            if ((issued >> s) & 1u)
              mbar_wait_bounded(&full[s], (issued_parity >> s) & 1u, args.status,
                                PTimeoutNs / 8);
      }
    }
  } else if (warp == 1) {
    // ---- MMA issuer (leader CTA only) -----------------------------------------------
    if (leader && lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int local = 0;
      bool ok = true;
      for (int u = pair; u < total && ok; u += npairs, ++local) {
        int g, nf, mt;
        decode(u, g, nf, mt);
        const TokSplit ts = tok_split(min(PT, group_rows(g) - mt * PT));
        const uint32_t idesc0 = idesc_bf16_f32(2 * PW, ts.n0);
        const uint32_t idesc1 = idesc_bf16_f32(2 * PW, ts.n1 > 0 ? ts.n1 : 16);
        if (!mbar_wait_bounded(tempty, (local & 1) ^ 1u, args.status, PTimeoutNs)) break;
        tc_fence_after();
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait_bounded(&full[stage], phase, args.status, PTimeoutNs)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t w0 = smem_u32(base + (size_t)stage * PStageBytes);
          const uint32_t x0 = w0 + PWBytes, x1 = x0 + PRegionBytes;
#pragma unroll
          for (int k = 0; k < PK / 16; ++k) {
            const uint64_t wd = smem_desc_sw128(w0 + k * 32);
            mma_bf16_2sm(tmem_base, wd, smem_desc_sw128(x0 + k * 32), idesc0, (kb | k) != 0);
            if (ts.n1 > 0)
              mma_bf16_2sm(tmem_base + 256, wd, smem_desc_sw128(x1 + k * 32), idesc1,
                           (kb | k) != 0);
          }
          mma_commit_2sm_mc(&empty[stage], 0x3);
          if (++stage == PStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (ok) mma_commit_2sm_mc(tfull, 0x3);
      }
      mma_commit_2sm(drain);
      mbar_wait_bounded(drain, 0, args.status, PTimeoutNs / 8);
    }
  } else {
    // ---- epilogue: warps 2..9 of each CTA (two per lane quadrant) ------------------
    const int q = warp & 3;
    const int half = (warp - 2) >> 2;  // this warp takes chunks 32*half, 32*half + 64, ...
    const int j = q * 32 + lane;       // TMEM lane = weight row of this CTA
    const uint32_t tempty_leader = mapa_shared(smem_u32(tempty), 0);
    float* buf = xchg + half * (32 * 64);
    int local = 0;
    uint32_t xc = 0;  // exchange sequence of this half (GEMM1)
    bool ok = true;
    for (int u = pair; u < total && ok; u += npairs, ++local) {
      int g, nf, mt;
      decode(u, g, nf, mt);
      if (!mbar_wait_bounded(tfull, local & 1, args.status, PTimeoutNs)) break;
      tc_fence_after();
      const int ntok = min(PT, group_rows(g) - mt * PT);
      const long long row0 =
          (g < args.N) ? (long long)args.offsets[g] + mt * PT : (long long)mt * PT;
      const bool in_range =
          (g == args.N) || (args.offsets[g] >= 0 && row0 + ntok <= args.rows_routed);
      __nv_bfloat16* outb = (g < args.N) ? args.out_routed : args.out_shared;
      const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16);
#pragma unroll 1
      for (int c = 32 * half; c < ntok; c += 64) {
        uint32_t v[32];
        tmem_ld32(taddr + c, v);  // TMEM column = token index
        tmem_wait_ld();
        if constexpr (kEpi == kPSwiGLU) {
          const uint32_t xph = xc & 1u;
          ++xc;
          if (q >= 2) {  // up projection: stage [token][feature] for the gate warp
            if (!mbar_wait_bounded(&xempty[half], xph ^ 1u, args.status, PTimeoutNs)) {
              ok = false;
              break;
            }
#pragma unroll
            for (int i = 0; i < 32; ++i) buf[i * 64 + (j - 64)] = __uint_as_float(v[i]);
            __syncwarp();
            if (lane == 0) mbar_arrive(&xfull[half]);
          } else {       // gate: h = silu(gate) * up, stored as bf16
            if (!mbar_wait_bounded(&xfull[half], xph, args.status, PTimeoutNs)) {
              ok = false;
              break;
            }
            if (in_range) {
              __nv_bfloat16* o = outb + (row0 + c) * args.out_ld + nf * PW + 64 * (int)rank + j;
#pragma unroll
              for (int i = 0; i < 32; ++i)
                if (c + i < ntok)
                  o[(long long)i * args.out_ld] =
                      __float2bfloat16_rn(silu_f(__uint_as_float(v[i])) * buf[i * 64 + j]);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&xempty[half]);
          }
        } else {
          if (in_range) {
            __nv_bfloat16* o = outb + (row0 + c) * args.out_ld + nf * 2 * PW + PW * (int)rank + j;
#pragma unroll
            for (int i = 0; i < 32; ++i)
              if (c + i < ntok) o[(long long)i * args.out_ld] = __float2bfloat16_rn(__uint_as_float(v[i]));
          }
        }
      }
      if (!ok) break;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(tempty_leader);
    }
  }

  // ---- teardown: neither CTA leaves while its peer may still signal it ----------------
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_2sm(tmem_base, 512);
  }
}

template <int kEpi>
cudaError_t launch_pair(const PairArgs& a, cudaStream_t st) {
  const size_t smem = pair_smem_bytes(a.N + 1);
  cudaError_t e = note_cuda(cudaFuncSetAttribute(pair_gemm_bf16_kernel<kEpi>,
                                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 (int)smem),
                            "pair GEMM: set shared-memory size");
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(num_sms() & ~1), 1, 1);
  cfg.blockDim = dim3(PThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  // as many pairs as can be resident at once (a GPC with an odd SM count
  // leaves one SM without a partner), so no pair waits for a second wave
  static int max_pairs = 0;
  if (max_pairs == 0) {
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, pair_gemm_bf16_kernel<kEpi>, &cfg) != cudaSuccess ||
        n <= 0)
      n = num_sms() / 2;
    max_pairs = n;
  }
  cfg.gridDim = dim3((unsigned)(2 * max_pairs), 1, 1);
  return note_cuda(cudaLaunchKernelEx(&cfg, pair_gemm_bf16_kernel<kEpi>, a), "pair GEMM launch");
}

}  // namespace

int launch_ffn_tc_bf16_pair(const moe_shape& s, const void* x_perm, const int32_t* offsets,
                            const void* x, const void* w13, const void* w2, void* y_perm,
                            void* y_shared, void* ws, cudaStream_t st) {
  const WsLayout L = ws_layout(s);
  uint8_t* w = static_cast<uint8_t*>(ws);
  __nv_bfloat16* H = reinterpret_cast<__nv_bfloat16*>(w + L.h);
  const uint64_t TK = (uint64_t)s.T * s.K;
  const auto BF = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  uint32_t* status = reinterpret_cast<uint32_t*>(w + L.status);

  PairArgs g1{};
  bool ok = make_map(&g1.tmW, w13, BF, 2, s.d, (uint64_t)(s.N + 1) * 2 * s.f, PK, 64) &&
            make_map(&g1.tmX_routed, x_perm, BF, 2, s.d, TK, PK, PBox) &&
            make_map(&g1.tmX_shared, x, BF, 2, s.d, s.T, PK, PBox);
  if (!ok) {
    note_text("pair GEMM1: tensor-map encoding failed");
    return MOE_ERR_CUDA;
  }
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
  g1.out_ld = s.f;
  if (launch_pair<kPSwiGLU>(g1, st) != cudaSuccess) return MOE_ERR_CUDA;

  PairArgs g2{};
  ok = make_map(&g2.tmW, w2, BF, 2, s.f, (uint64_t)(s.N + 1) * s.d, PK, PW) &&
       make_map(&g2.tmX_routed, H, BF, 2, s.f, TK + s.T, PK, PBox) &&
       make_map(&g2.tmX_shared, H, BF, 2, s.f, TK + s.T, PK, PBox);
  if (!ok) {
    note_text("pair GEMM2: tensor-map encoding failed");
    return MOE_ERR_CUDA;
  }
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
  g2.out_ld = s.d;
  if (launch_pair<kPStore>(g2, st) != cudaSuccess) return MOE_ERR_CUDA;
  return MOE_OK;
}

}  // namespace moe
