// bf16 expert GEMMs on CTA pairs (tcgen05 cta_group::2) with whole-expert
// units and a ring of TMEM columns.
//
// Same computation as the one-CTA kernel in gemm_tc.cu (the SwiGLU expert FFN
// of the mhpq.cn article §1.1: GEMM1 with the SwiGLU epilogue, then GEMM2),
// arranged so that each weight tile crosses from L2 into shared memory once
// per expert and no ragged row count costs a second pass over the weights:
//   * the weights are the MMA's M side: 256 weight rows of one expert per unit,
//     128 in each CTA of the pair;
//   * the tokens are the N side: a unit takes up to UMax of the expert's rows
//     (an expert with more is cut into near-equal units), rounded up to 16
//     columns only, as one to three tcgen05.mma.cta_group::2 per K step; each
//     CTA stages half of every MMA's token rows;
//   * per K step a CTA stages 16 KB of weights and at most 18 KB of tokens, so
//     six stages fit in shared memory.
// TMEM: the 512 accumulator columns form a ring of 32 chunks of 16 columns.
// Unit after unit takes the next chunks of the ring (an MMA is split where the
// ring wraps); the epilogue drains chunk by chunk and frees each one on its own
// barrier, so the next unit's MMAs start as soon as the chunks they overwrite
// are drained instead of after the whole previous epilogue.
// GEMM1 lane layout: in CTA r, TMEM lanes 32q..32q+15 hold the gate rows
// (W1) of hidden features 128j + 64r + 16q + i and lanes 32q+16..32q+31 the
// up rows (W3) of the same features; one copy through a 5-D view of the
// 128-row-interleaved W13 (row = 256 tile + 128 up + 16 block + i) builds this
// order, so SiLU(gate)*up needs one shuffle inside the warp.
// Token rows come in boxes of 64, 32, 16 and 8 rows, so a stage takes one
// weight copy and a few token copies.
// Roles per CTA: warp 0 TMA producer (its lanes issue the stage's copies in
// parallel), warp 1 TMEM owner and, in the leader CTA, the one thread that
// issues the pair MMAs and multicasts the commits to both CTAs; warps 2-17
// epilogue, four per TMEM lane quadrant, taking chunks in turn.  Every wait is
// bounded (~2 s) and sets the device status word when it gives up; both CTAs
// always reach the final cluster barrier, so neither exits while its peer may
// still signal it.
#include <cuda.h>
#include <cuda_bf16.h>

#include "epilogue.cuh"
#include "internal.h"
#include "ptx.cuh"

namespace moe {
namespace {

constexpr int PW = 128;            // weight rows per CTA (pair: 256)
constexpr int PK = 64;             // bf16 K slice (128 bytes)
constexpr int UMax = 288;          // max token rows per unit
constexpr int PStages = 6;
constexpr int PWBytes = PW * PK * 2;                  // 16 KB of weights per CTA and stage
constexpr int PTokBytes = (UMax / 2) * PK * 2;        // 18 KB: half of a unit's tokens
constexpr int PStageBytes = PWBytes + PTokBytes;      // 34 KB
constexpr int PThreads = 576;      // warps 0, 1, then 16 epilogue warps
constexpr int PEpiWarps = 16;
constexpr int PChunks = 32;        // TMEM ring: 32 chunks of 16 columns
constexpr int PUnitSlots = 4;      // units in flight between MMA and epilogue
constexpr uint64_t PTimeoutNs = 2000000000ull;

enum PEpi { kPSwiGLU = 0, kPStore = 1 };

struct alignas(64) PairArgs {
  CUtensorMap tmW;          // weights: GEMM1 the 5-D W13 view, GEMM2 [(N+1) d, f] box {64, 128}
  CUtensorMap tmX[2][4];    // token rows [src: routed, shared][box rows 64, 32, 16, 8]
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
  return 1024 + (size_t)PStages * PStageBytes + 1024 + (size_t)(groups + 1) * 4;
}


// Rows of a group split into near-equal units of at most UMax rows; every unit
// but the last has `size` rows (a multiple of 16).
__device__ __forceinline__ void unit_split(int rows, int& size, int& count) {
  if (rows <= 0) {
    size = 16;
    count = 0;
    return;
  }
  const int n0 = (rows + UMax - 1) / UMax;
  size = (((rows + n0 - 1) / n0) + 15) & ~15;
  count = (rows + size - 1) / size;
}

// Cluster-scope acquire: the arrivals come from both CTAs of the pair.
__device__ __forceinline__ bool mbar_wait_cl(uint64_t* bar, uint32_t parity, uint32_t* err) {
  return mbar_wait_cluster_bounded(bar, parity, err, PTimeoutNs);
}

// One unit as every role sees it.
struct Unit {
  int g, nf;
  int ntok;      // token rows of the unit
  int ncol;      // ntok rounded up to 16
  long long row0;  // first row in the token source (routed rows or x)
};

// The MMA pieces of a unit whose columns start at ring column c0: split where
// the ring wraps and at 256 columns.  Returns the piece count (1..3).
__device__ __forceinline__ int unit_pieces(int c0, int ncol, int (&col)[3], int (&n)[3]) {
  int k = 0, left = ncol, c = c0;
  while (left > 0) {
    const int w = min(min(left, 256), PChunks * 16 - c);
    col[k] = c;
    n[k] = w;
    ++k;
    left -= w;
    c = (c + w) & (PChunks * 16 - 1);
  }
  for (int i = k; i < 3; ++i) {
    col[i] = 0;
    n[i] = 0;
  }
  return k;
}

template <int kEpi>
__global__ void __launch_bounds__(PThreads, 1) pair_gemm_bf16_kernel(
    const __grid_constant__ PairArgs args) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + (size_t)PStages * PStageBytes);
  uint64_t* full = bars;                       // [PStages] leader: both CTAs' copies landed
  uint64_t* empty = full + PStages;            // [PStages] each CTA: stage consumed
  uint64_t* cfree = empty + PStages;           // [PChunks] leader: chunk drained (8 warps)
  uint64_t* ufull = cfree + PChunks;           // [PUnitSlots] each CTA: unit accumulated
  uint64_t* uempty = ufull + PUnitSlots;       // [PUnitSlots] leader: unit taken (32 warps)
  uint64_t* drain = uempty + PUnitSlots;       // [1]
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
  int* unit_start = reinterpret_cast<int*>(base + (size_t)PStages * PStageBytes + 1024);

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
    for (int c = 0; c < PChunks; ++c) mbar_init(&cfree[c], 8);
    for (int i = 0; i < PUnitSlots; ++i) {
      mbar_init(&ufull[i], 1);
      mbar_init(&uempty[i], 2 * PEpiWarps);
    }
    mbar_init(drain, 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc_2sm(tmem_holder, 512);
    tmem_relinquish_2sm();
  }
  auto group_rows = [&](int g) {
    return (g < args.N) ? args.offsets[g + 1] - args.offsets[g] : args.T;
  };
  for (int g = tid; g < G1; g += PThreads) {
    int size, count;
    unit_split(group_rows(g), size, count);
    unit_start[g] = count;
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {  // exclusive scan of units per group, times NF
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
      const int c = unit_start[g];
      unit_start[g] = run * NF;
      run += c;
    }
    if (lane == 31) unit_start[G1] = inc * NF;
  }
  // both CTAs' barriers are initialised before either signals the other
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  const int total = unit_start[G1];

  // unit u -> group, weight tile, token rows; units of a group are ordered
  // (weight tile, token part)
  auto decode = [&](int u) {
    int lo = 0, hi = G1;
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (unit_start[mid] <= u) lo = mid; else hi = mid;
    }
    Unit U;
    U.g = lo;
    const int rows = group_rows(lo);
    int size, count;
    unit_split(rows, size, count);
    const int local = u - unit_start[lo];
    U.nf = local / count;
    const int mt = local - U.nf * count;
    U.ntok = min(size, rows - mt * size);
    U.ncol = (U.ntok + 15) & ~15;
    U.row0 = (long long)mt * size;
    return U;
  };

  if (warp == 0) {
    // ---- TMA producer (both CTAs); lane j issues the j-th box of a stage -------
    if (lane < 9) tma_prefetch_desc(lane == 0 ? &args.tmW : &args.tmX[(lane - 1) >> 2][(lane - 1) & 3]);
    int stage = 0;
    uint32_t phase = 0, issued = 0, issued_parity = 0;
    uint32_t s = 0;  // chunk sequence number of the unit's first column
    bool ok = true;
    for (int u = pair; u < total && ok; u += npairs) {
      const Unit U = decode(u);
      int col[3], n[3];
      const int np = unit_pieces((int)(s % PChunks) * 16, U.ncol, col, n);
      s += U.ncol / 16;
      const int src = U.g < args.N ? 0 : 1;
      const long long srow0 =
          U.row0 + (U.g < args.N ? (long long)args.offsets[U.g] : (long long)args.x_shared_row0);
      // this lane's copy: lane 0 the weights, then each piece's half of the
      // token rows in boxes of 64, 32, 16, 8 rows
      const CUtensorMap* map = nullptr;
      uint32_t soff = 0;
      int row = 0, c3 = 0, c4 = 0;
      if (lane == 0) {
        map = &args.tmW;
        if constexpr (kEpi == kPSwiGLU) {
          c3 = 4 * (int)rank;                          // 16-row block within the 128-row half
          c4 = U.g * NF + U.nf;                        // 256-row tile of W13
        } else {
          row = U.g * args.n_feat + U.nf * 2 * PW + PW * (int)rank;
        }
      } else {
        int i = lane - 1, tok = 0, sm = PWBytes;
        for (int p = 0; p < 3 && map == nullptr; ++p) {
          if (p >= np) break;
          const int h = n[p] / 2;
          int done = 0;
          for (int c = 0; c < 4 && map == nullptr; ++c) {
            const int bs = 64 >> c;
            const int nb = (c == 0) ? (h - done) / 64 : (((h - done) & bs) ? 1 : 0);
            if (i < nb) {
              map = &args.tmX[src][c];
              row = (int)(srow0 + tok + (int)rank * h + done + bs * i);
              soff = (uint32_t)(sm + (done + bs * i) * (PK * 2));
            } else {
              i -= nb;
              done += nb * bs;
            }
          }
          tok += n[p];
          sm += h * (PK * 2);
        }
      }
      const uint32_t bytes = 2u * (uint32_t)(PWBytes + (U.ncol / 2) * (PK * 2));
      for (int kb = 0; kb < KB; ++kb) {
        bool got = true;
        if (lane == 0) got = mbar_wait_bounded(&empty[stage], phase ^ 1u, args.status, PTimeoutNs);
        if (!__shfl_sync(0xffffffffu, got ? 1 : 0, 0)) {
          ok = false;
          break;
        }
        uint8_t* sw = base + (size_t)stage * PStageBytes;
        const uint32_t fbar = mapa_shared(smem_u32(&full[stage]), 0);
        if (leader && lane == 0) mbar_arrive_expect_tx(&full[stage], bytes);
        __syncwarp();
        if (map != nullptr) {
          if (kEpi == kPSwiGLU && lane == 0)
            tma_load_5d_2sm(sw, map, kb * PK, 0, 0, c3, c4, fbar);
          else
            tma_load_2d_2sm(sw + soff, map, kb * PK, row, fbar);
        }
        issued |= 1u << stage;
        issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
        if (++stage == PStages) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
    if (!ok && leader && lane == 0) {  // the copies already issued complete on these barriers
      for (int st = 0; st < PStages; ++st)
        if ((issued >> st) & 1u)
          mbar_wait_bounded(&full[st], (issued_parity >> st) & 1u, args.status, PTimeoutNs / 8);
    }
  } else if (warp == 1) {
    // ---- MMA issuer (leader CTA only) -------------------------------------------
    if (leader && lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t s = 0;
      int lu = 0;
      bool ok = true;
      for (int u = pair; u < total && ok; u += npairs, ++lu) {
        const Unit U = decode(u);
        const int nch = U.ncol / 16;
        for (int c = 0; c < nch && ok; ++c) {
          const uint32_t sc = s + (uint32_t)c;
          ok = mbar_wait_cl(&cfree[sc % PChunks], ((sc / PChunks) & 1u) ^ 1u, args.status);
        }
        if (!ok) break;
        tc_fence_after();
        int col[3], n[3];
        const int np = unit_pieces((int)(s % PChunks) * 16, U.ncol, col, n);
        s += (uint32_t)nch;
        uint32_t idesc[3], xoff[3];
        uint32_t off = PWBytes;
        for (int p = 0; p < 3; ++p) {
          idesc[p] = idesc_bf16_f32(2 * PW, n[p] > 0 ? n[p] : 16);
          xoff[p] = off;
          off += (uint32_t)(n[p] / 2) * (PK * 2);
        }
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait_bounded(&full[stage], phase, args.status, PTimeoutNs)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t w0 = smem_u32(base + (size_t)stage * PStageBytes);
#pragma unroll
          for (int k = 0; k < PK / 16; ++k) {
            const uint64_t wd = smem_desc_sw128(w0 + k * 32);
            const uint32_t acc = (kb | k) != 0;
            mma_bf16_2sm(tmem_base + col[0], wd, smem_desc_sw128(w0 + xoff[0] + k * 32), idesc[0],
                         acc);
            if (np > 1)
              mma_bf16_2sm(tmem_base + col[1], wd, smem_desc_sw128(w0 + xoff[1] + k * 32),
                           idesc[1], acc);
            if (np > 2)
              mma_bf16_2sm(tmem_base + col[2], wd, smem_desc_sw128(w0 + xoff[2] + k * 32),
                           idesc[2], acc);
          }
          mma_commit_2sm_mc(&empty[stage], 0x3);
          if (++stage == PStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        const int us = lu % PUnitSlots;
        if (!mbar_wait_cl(&uempty[us], ((uint32_t)(lu / PUnitSlots) & 1u) ^ 1u, args.status)) break;
        mma_commit_2sm_mc(&ufull[us], 0x3);
      }
      mma_commit_2sm(drain);
      mbar_wait_bounded(drain, 0, args.status, PTimeoutNs / 8);
    }
  } else {
    // ---- epilogue: warps 2..17 of each CTA, four per TMEM lane quadrant ----------
    const int q = warp & 3;              // TMEM lanes 32q..32q+31
    const int wq = (warp - 2) >> 2;      // takes the chunks with sequence number = wq mod 4
    const uint32_t taddr_q = tmem_base + ((uint32_t)(q * 32) << 16);
    const uint32_t cfree0 = mapa_shared(smem_u32(&cfree[0]), 0);
    const uint32_t uempty0 = mapa_shared(smem_u32(&uempty[0]), 0);
    uint32_t s = 0;
    int lu = 0;
    for (int u = pair; u < total; u += npairs, ++lu) {
      const Unit U = decode(u);
      const int nch = U.ncol / 16;
      const int us = lu % PUnitSlots;
      if (!mbar_wait_bounded(&ufull[us], (uint32_t)(lu / PUnitSlots) & 1u, args.status,
                             PTimeoutNs))
        break;
      tc_fence_after();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(uempty0 + 8u * (uint32_t)us);
      const long long orow0 = (U.g < args.N) ? (long long)args.offsets[U.g] + U.row0 : U.row0;
      const bool in_range = (U.g == args.N) ||
                            (args.offsets[U.g] >= 0 && orow0 + U.ntok <= args.rows_routed);
      __nv_bfloat16* outb = (U.g < args.N) ? args.out_routed : args.out_shared;
      // first chunk of this unit that falls to this warp
      int c = (int)((uint32_t)(wq - (int)(s & 3u)) & 3u);
      for (; c < nch; c += 4) {
        const uint32_t sc = s + (uint32_t)c;
        uint32_t v[16];
        tmem_ld16(taddr_q + (sc % PChunks) * 16, v);
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(cfree0 + 8u * (sc % PChunks));
        if (!in_range) continue;
        const int t0 = 16 * c;
        if constexpr (kEpi == kPSwiGLU) {
          // lanes 0-15: gate of feature i, tokens t0..t0+7;
          // lanes 16-31: up of feature i, tokens t0+8..t0+15
          const bool up_lane = (lane & 16) != 0;
          const int feat = U.nf * PW + 64 * (int)rank + 16 * q + (lane & 15);
          const int tb = t0 + (up_lane ? 8 : 0);
          __nv_bfloat16* o = outb + (orow0 + tb) * args.out_ld + feat;
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const float mine_send = __uint_as_float(up_lane ? v[k] : v[8 + k]);
            const float other = __shfl_xor_sync(0xffffffffu, mine_send, 16);
            const float gt = up_lane ? other : __uint_as_float(v[k]);
            const float upv = up_lane ? __uint_as_float(v[8 + k]) : other;
            if (tb + k < U.ntok)
              o[(long long)k * args.out_ld] = __float2bfloat16_rn(silu_fast(gt) * upv);
          }
        } else {
          const int feat = U.nf * 2 * PW + PW * (int)rank + 32 * q + lane;
          __nv_bfloat16* o = outb + (orow0 + t0) * args.out_ld + feat;
#pragma unroll
          for (int k = 0; k < 16; ++k)
            if (t0 + k < U.ntok) o[(long long)k * args.out_ld] = __float2bfloat16_rn(__uint_as_float(v[k]));
        }
      }
      s += (uint32_t)nch;
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

bool token_maps(PairArgs& a, const void* routed, uint64_t routed_rows, const void* shared,
                uint64_t shared_rows, uint64_t k) {
  const auto BF = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  bool ok = true;
  for (int c = 0; c < 4; ++c)
    ok = ok && make_map(&a.tmX[0][c], routed, BF, 2, k, routed_rows, PK, 64u >> c) &&
         make_map(&a.tmX[1][c], shared, BF, 2, k, shared_rows, PK, 64u >> c);
  return ok;
}

// W13 [(N+1) * 2f, d] (W1/W3 interleaved in 128-row blocks) as a 5-D tensor
// (k, i, up, block, tile) with row = 256 tile + 128 up + 16 block + i; the box
// {64, 16, 2, 4, 1} lands as 128 rows ordered (block, up, i).
bool w13_gate_up_map(CUtensorMap* m, const void* w13, const moe_shape& s) {
  const uint64_t rb = (uint64_t)s.d * 2;  // bytes per row
  const uint64_t dims[5] = {(uint64_t)s.d, 16, 2, 8, (uint64_t)(s.N + 1) * 2 * s.f / 256};
  const uint64_t strides[4] = {rb, 128 * rb, 16 * rb, 256 * rb};
  const uint32_t box[5] = {PK, 16, 2, 4, 1};
  return make_map_nd(m, w13, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, dims, strides, box);
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
  bool ok = w13_gate_up_map(&g1.tmW, w13, s) &&
            token_maps(g1, x_perm, TK, x, s.T, s.d);
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
       token_maps(g2, H, TK + s.T, H, TK + s.T, s.f);
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
