// FP8-E4M3 expert GEMMs with fine-grained fp32 block scales.
//
// The FP8 recipe follows the mhpq.cn article §4.1 (精细量化策略 / 在线量化 /
// 高精度累加): activations are scaled per 1x128 tile and weights per
// 128x128 block, each scale taken online from the current max-abs; products
// accumulate in fp32.  Reading taken: scale = amax/448 and inverse
// 448/amax in fp32 (IEEE division), code = E4M3_RNE_satfinite(v * inverse),
// a tile with amax = 0 gets scale 1 and all-zero codes.
//
// GEMM (one persistent launch per expert GEMM, all groups):
//   C[row, col] = sum over 128-wide K slices kb of
//                 sa[row, kb] * sw[col/128, kb] * sum_{k in kb} qa[row,k] qw[col,k]
// The per-slice products come from tcgen05.mma kind::f8f6f4 (E4M3 x E4M3,
// fp32 accumulate, M=128 tokens, N=256 weight columns, K=32 each); every
// 128-wide slice lands in its own TMEM buffer (two 256-column buffers, so
// the tensor core fills one while the other is drained).  Sixteen epilogue
// warps -- four per TMEM lane quadrant, each owning 64 of the 256 columns --
// fold each slice into fp32 register sums with the product of the two
// scales (packed fp32x2 FMAs).  This per-slice promotion is the tcgen05
// counterpart of the article's "accumulate at an interval in fp32 on the CUDA
// cores" (the kaiyunto.com walk-through describes the same H800 step); on
// sm_100 the partial sums already sit in TMEM in fp32, so only the scale
// product is applied per slice.
//
// GEMM1 epilogue: h = silu(gate) * up for the 128 hidden features of the
// tile (gate and up columns of one feature lie in the same tile and thread
// row), then h is quantised per 1x128 tile along f; the four warps that
// share a row exchange their quarter-tile max-abs through shared memory
// under an mbarrier.  GEMM2 epilogue: bf16 output rows.
// Roles: warp 0 TMA producer (4-stage ring: 128 token rows + 256 weight rows
// of 128 bytes), warp 1 TMEM owner and MMA issuer, warps 2-17 epilogue.
// Sixteen epilogue warps (four per TMEM lane quadrant, 64 running sums each)
// keep a thread within the register budget of an 18-warp CTA (five warps
// share some of the SM's four 16K-register banks) and give each scheduler
// four warps to overlap the TMEM-load latency of the per-slice promotion.
// Activation scales are block-major ([K/128][rows rounded up to 4]); for each
// slice the producer copies the tile's 128 scales (a 132-float box starting at
// the tile's first row rounded down to 4) into a ring of eight shared-memory
// slots that the epilogue releases, together with the slice's two weight-block
// scales (two 4-byte cp.async copies completing on the same barrier), so the
// promotion reads every scale from shared memory.
// All waits are bounded (~2 s) and set the device status word on expiry.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include <cstdlib>
#include <cstring>

#include "epilogue.cuh"
#include "fp8_util.cuh"
#include "internal.h"
#include "ptx.cuh"

namespace moe {
namespace {

constexpr int FBM = 128, FBN = 256, FBK = 128;
constexpr int FStages = 4;
constexpr int FABytes = FBM * FBK;      // 16 KB
constexpr int FBBytes = FBN * FBK;      // 32 KB
constexpr int FStageBytes = FABytes + FBBytes;
// warp 0 TMA, warp 1 MMA, then kEpiW epilogue warps (kEpiW / 4 per TMEM lane
// quadrant): 8 by default, each thread holding 128 running sums within the
// per-thread register budget of a 10-warp CTA; 16 (MOE_FP8_EPI=narrow or x32)
// halves the sums per thread
__host__ __device__ constexpr int fp8_threads(int epi_warps) { return 64 + 32 * epi_warps; }
constexpr int FScaleSlots = 8;      // ring of per-slice activation-scale boxes
constexpr int FScaleBox = 132;      // floats per box: 128 rows + up to 3 of alignment
constexpr int FScaleSlotBytes = 640;
constexpr uint64_t FTimeoutNs = 2000000000ull;

enum FEpi { kFEpiSwiGLUQuant = 0, kFEpiStore = 1, kFEpiSwiGLUBwd = 2 };

// x [rows, d] bf16 -> codes [rows, d], scales block-major [d/128][sc_ld]; one
// half-warp per tile.  kE5M2: gradient rows in E5M2 instead of E4M3.
template <bool kE5M2>
__global__ void quant_rows_kernel(const __nv_bfloat16* __restrict__ x, long long rows, int d,
                                  uint8_t* __restrict__ q, float* __restrict__ sc,
                                  long long sc_ld) {
  const int tiles_per_row = d / QB;
  const long long tiles = rows * tiles_per_row;
  const int half = (threadIdx.x >> 4) & 1, l16 = threadIdx.x & 15;
  const long long hw = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 4;
  const long long hw_stride = ((long long)gridDim.x * blockDim.x) >> 4;
  (void)half;
  // every half-warp walks the same number of iterations so shuffles stay converged
  const long long iters = (tiles + hw_stride - 1) / hw_stride;
  for (long long it = 0; it < iters; ++it) {
    const long long tile = hw + it * hw_stride;
    const bool live = tile < tiles;
    const long long r = live ? tile / tiles_per_row : 0;
    const int tc = live ? (int)(tile - r * tiles_per_row) : 0;
    float v[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    if (live)
      bf16x8_to_f32(*reinterpret_cast<const uint4*>(x + r * d + tc * QB + 8 * l16), v);
    uint2 codes;
    const float s = quant_tile_16lanes<kE5M2>(v, codes);
    if (live) {
      *reinterpret_cast<uint2*>(q + r * d + tc * QB + 8 * l16) = codes;
      if (l16 == 0) sc[(long long)tc * sc_ld + r] = s;
    }
  }
}

// ---- 128x128 weight quantisation ---------------------------------------------------
// One CTA (128 threads) per block.  Sixteen lanes cover one 128-column row of
// the block with 16-byte loads (8 values each), so a warp reads two whole
// 256-byte rows per instruction; warp w takes rows 32w .. 32w+31, two at a
// time, and keeps its 16 loads in registers for the second pass.  The block's
// max-abs is reduced over the lanes and warps, then each lane writes its 8
// codes of each of its rows (8 bytes; 128 contiguous bytes per row).
__global__ void __launch_bounds__(128) quant_blocks_kernel(const __nv_bfloat16* __restrict__ w,
                                                           int cols, long long blocks_r,
                                                           int blocks_c,
                                                           uint8_t* __restrict__ q,
                                                           float* __restrict__ sc) {
  __shared__ float red[4];
  const long long b = blockIdx.x;
  const long long br = b / blocks_c;
  const int bc = (int)(b - br * blocks_c);
  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
  const int half = lane >> 4, l16 = lane & 15;  // row parity within a pair, 16-byte piece
  const long long row0 = br * QB + warp * 32 + half;  // this lane's first row
  const __nv_bfloat16* src = w + row0 * (long long)cols + (long long)bc * QB + 8 * l16;
  float amax = 0.f;
  uint4 raw[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) {  // rows row0 + 2i
    raw[i] = __ldg(reinterpret_cast<const uint4*>(src + (long long)(2 * i) * cols));
    float f[8];
    bf16x8_to_f32(raw[i], f);
#pragma unroll
    for (int j = 0; j < 8; ++j) amax = fmaxf(amax, fabsf(f[j]));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if (lane == 0) red[warp] = amax;
  __syncthreads();
  amax = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
  const bool zero = amax == 0.f;
  const float scale = zero ? 1.f : __fdiv_rn(amax, 448.f);
  const float inv = zero ? 0.f : __fdiv_rn(448.f, amax);
  uint8_t* dst = q + row0 * (long long)cols + (long long)bc * QB + 8 * l16;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    float f[8];
    bf16x8_to_f32(raw[i], f);
    uint32_t w2[2] = {0u, 0u};
    if (!zero) {
#pragma unroll
      for (int p = 0; p < 2; ++p)
#pragma unroll
        for (int qq = 0; qq < 2; ++qq) {
          const int k = 4 * p + 2 * qq;
          const __nv_fp8x2_storage_t c2 = __nv_cvt_float2_to_fp8x2(
              make_float2(__fmul_rn(f[k], inv), __fmul_rn(f[k + 1], inv)), __NV_SATFINITE,
              __NV_E4M3);
          w2[p] |= (uint32_t)c2 << (16 * qq);
        }
    }
    *reinterpret_cast<uint2*>(dst + (long long)(2 * i) * cols) = make_uint2(w2[0], w2[1]);
  }
  if (t == 0) sc[br * blocks_c + bc] = scale;
}

// ---- block-scaled FP8 grouped GEMM -------------------------------------------------
struct alignas(64) Fp8Args {
  CUtensorMap tmA_routed;
  CUtensorMap tmA_shared;
  CUtensorMap tmB;
  CUtensorMap tmS_routed;  // activation scales [KB][ld] (row index as in tmA_routed), box {132, 1}
  CUtensorMap tmS_shared;  // the same for tmA_shared's rows
  CUtensorMap tmY_routed;  // store epilogue: y_routed [rows_routed, out_ld] bf16, box {16, 32},
  CUtensorMap tmY_shared;  // 32-byte swizzle; y_shared [T, out_ld] (built by the launcher)
  int y_tma;               // 1: the maps above are valid
  const int32_t* offsets;
  const float* sw;         // [(N+1) * n_acc / 128, KB] weight block scales
  uint8_t* q_routed;       // GEMM1: h codes, row (offsets[g] + r)
  uint8_t* q_shared;       // GEMM1: h codes, row r
  float* qs_routed;        // GEMM1: h scales, block-major [out_ld/128][qs_ld], routed rows
  float* qs_shared;        // ... shared-expert rows (same array, column TK onwards)
  long long qs_ld;
  __nv_bfloat16* y_routed;  // Store / SwiGLU-backward outputs, row (offsets[g] + r)
  __nv_bfloat16* y_shared;  // ... shared-expert row r
  const __nv_bfloat16* aux_routed;  // SwiGLU backward: the stored g, u [rows, 2f], packed
  const __nv_bfloat16* aux_shared;
  int a_format;             // A operand: kF8E4M3 (forward) or kF8E5M2 (gradients)
  uint32_t* status;
  int N, T;
  int rows_routed;
  int a_shared_row0;
  int n_acc;   // weight rows per group (2f or d)
  int k_dim;   // contraction length
  int out_ld;  // f (GEMM1 codes) or d (GEMM2)
};

// Store epilogue staging: per epilogue warp two 1 KB pieces (32 rows x 16
// bf16 columns) in the TMA's 32-byte swizzle, one filled while the other is
// being stored.
constexpr int FStgPiece = 1024;
constexpr int FStgBytes = 8 * 2 * FStgPiece;

constexpr size_t fp8_smem_bytes(int groups, bool staging) {
  return 1024 + (size_t)FStages * FStageBytes + (staging ? FStgBytes : 0) +
         (size_t)FScaleSlots * FScaleSlotBytes + 512 + 2 * 4 * FBM * 4 + (size_t)(groups + 1) * 4;
}

// a0 += x0 * s and a1 += x1 * s as one packed fp32x2 FMA (two independent
// round-to-nearest FMAs, the same results as two fmaf, half the issue slots)
__device__ __forceinline__ void ffma2(float& a0, float& a1, float x0, float x1, float s) {
  asm("{\n\t.reg .b64 ra, rb, rc;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %4};\n\t"
      "mov.b64 rc, {%0, %1};\n\tfma.rn.f32x2 rc, ra, rb, rc;\n\tmov.b64 {%0, %1}, rc;\n\t}"
      : "+f"(a0), "+f"(a1)
      : "f"(x0), "f"(x1), "f"(s));
}


// kEpiW epilogue warps; each reads its slice columns kLd at a time (16 or 32
// columns per tcgen05.ld), kInFlight loads per wait
template <int kEpi, int kEpiW, int kLd, int kInFlight>
__global__ void __launch_bounds__(fp8_threads(kEpiW), 1) grouped_gemm_fp8_kernel(
    const __grid_constant__ Fp8Args args) {
  static_assert(kEpiW == 16 || kEpiW == 8, "four or two epilogue warps per lane quadrant");
  static_assert(kLd == 16 || kLd == 32, "16- or 32-column TMEM loads");
  constexpr int FThreads = fp8_threads(kEpiW);
  constexpr int FEpiWarps = kEpiW;
  constexpr int kSub = kEpiW / 4;          // epilogue warps per TMEM lane quadrant
  constexpr int kCols = FBN / kSub;        // accumulator columns per warp
  constexpr int kFeat = (FBN / 2) / kSub;  // GEMM1: hidden features per warp
  static_assert((kCols / kLd) % (2 * kInFlight) == 0, "gate and up halves split evenly");
  // the bf16 store epilogue writes full 32-row groups by TMA (eight-warp shape)
  constexpr bool kTmaY = kEpi == kFEpiStore && kEpiW == 8;
  constexpr size_t kStg = kTmaY ? FStgBytes : 0;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* staging = base + (size_t)FStages * FStageBytes;  // 1024-aligned
  float* sc_ring = reinterpret_cast<float*>(staging + kStg);
  uint64_t* bars = reinterpret_cast<uint64_t*>(staging + kStg +
                                               (size_t)FScaleSlots * FScaleSlotBytes);
  uint64_t* full = bars;                  // [FStages]
  uint64_t* empty = bars + FStages;       // [FStages]
  uint64_t* sfull = bars + 2 * FStages;   // [2] slice buffer written
  uint64_t* sempty = sfull + 2;           // [2] slice buffer drained (8 warps)
  uint64_t* xbar = sempty + 2;            // [2] amax exchange (8 warps)
  uint64_t* drain = xbar + 2;             // [1]
  uint64_t* scfull = drain + 1;           // [FScaleSlots] scale box landed
  uint64_t* scempty = scfull + FScaleSlots;  // [FScaleSlots] scale box read (16 warps)
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(scempty + FScaleSlots);
  float* xchg = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(bars) + 512);  // [2][4][128]
  int* tile_start = reinterpret_cast<int*>(xchg + 2 * 4 * FBM);

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const bool clock_cta = blockIdx.x == 0 && tid == 0 && args.status;
  ClockMark cm{};
  if (clock_cta) cm = clock_start();
  const int G1 = args.N + 1;
  const int NT = args.n_acc / FBN;
  const int KB = args.k_dim / FBK;

  if (tid == 0) {
    for (int s = 0; s < FStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&sfull[a], 1);
      mbar_init(&sempty[a], FEpiWarps);
      mbar_init(&xbar[a], FEpiWarps);
    }
    mbar_init(drain, 1);
    for (int c = 0; c < FScaleSlots; ++c) {
      mbar_init(&scfull[c], 1);
      mbar_init(&scempty[c], FEpiWarps);
    }
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, 512);
    tmem_relinquish();
  }
  for (int g = tid; g < G1; g += FThreads) {
    const int rows = (g < args.N) ? args.offsets[g + 1] - args.offsets[g] : args.T;
    tile_start[g] = rows > 0 ? (rows + FBM - 1) / FBM : 0;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) {
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

  auto decode = [&](int tile, int& g, int& n, int& m) {
    int lo = 0, hi = G1;
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (tile_start[mid] <= tile) lo = mid; else hi = mid;
    }
    g = lo;
    const int mt = (tile_start[g + 1] - tile_start[g]) / NT;
    const int local = tile - tile_start[g];
    n = local / mt;
    m = local - n * mt;
  };

  if (warp == 0) {
    // ---- TMA producer ----
    if (lane == 0) {
      tma_prefetch_desc(&args.tmA_routed);
      tma_prefetch_desc(&args.tmA_shared);
      tma_prefetch_desc(&args.tmB);
      tma_prefetch_desc(&args.tmS_routed);
      tma_prefetch_desc(&args.tmS_shared);
      int stage = 0;
      uint32_t phase = 0, issued = 0, issued_parity = 0;
      uint32_t sslice = 0, sc_issued = 0, sc_parity = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
        int g, n, m;
        decode(tile, g, n, m);
        const CUtensorMap* am = (g < args.N) ? &args.tmA_routed : &args.tmA_shared;
        const CUtensorMap* smap = (g < args.N) ? &args.tmS_routed : &args.tmS_shared;
        const int arow = ((g < args.N) ? args.offsets[g] : args.a_shared_row0) + m * FBM;
        const int brow = g * args.n_acc + n * FBN;
        // the tile's two 128-row weight blocks, scales [block][KB]
        const float* sw_tile = args.sw + ((long long)brow / QB) * KB;
        for (int kb = 0; kb < KB; ++kb) {
          const uint32_t cs = sslice % FScaleSlots, cph = (sslice / FScaleSlots) & 1u;
          if (!mbar_wait_bounded(&empty[stage], phase ^ 1u, args.status, FTimeoutNs) ||
              !mbar_wait_bounded(&scempty[cs], cph ^ 1u, args.status, FTimeoutNs)) {
            ok = false;
            break;
          }
          uint8_t* sa = base + (size_t)stage * FStageBytes;
          mbar_arrive_expect_tx(&full[stage], FStageBytes);
          tma_load_2d(sa, am, kb * FBK, arow, &full[stage]);
          tma_load_2d(sa + FABytes, &args.tmB, kb * FBK, brow, &full[stage]);
          // this slice's scales: the two weight-block scales by cp.async, whose
          // pending arrival is registered on the slot's barrier before the
          // expect-tx arrival (so the phase cannot complete without them), then
          // the activation box for the tile's rows by TMA
          uint8_t* slot_dst = reinterpret_cast<uint8_t*>(sc_ring) + cs * FScaleSlotBytes;
          cp_async_4(slot_dst + FScaleBox * 4, sw_tile + kb);
          cp_async_4(slot_dst + FScaleBox * 4 + 4, sw_tile + KB + kb);
          cp_async_mbar_arrive(&scfull[cs]);
          mbar_arrive_expect_tx(&scfull[cs], FScaleBox * 4);
          tma_load_2d(slot_dst, smap, arow & ~3, kb, &scfull[cs]);
          issued |= 1u << stage;
          issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
          sc_issued |= 1u << cs;
          sc_parity = (sc_parity & ~(1u << cs)) | (cph << cs);
          ++sslice;
          if (++stage == FStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {
        for (int s = 0; s < FStages; ++s)
          if ((issued >> s) & 1u)
            mbar_wait_bounded(&full[s], (issued_parity >> s) & 1u, args.status, FTimeoutNs / 8);
        for (int c = 0; c < FScaleSlots; ++c)
          if ((sc_issued >> c) & 1u)
            mbar_wait_bounded(&scfull[c], (sc_parity >> c) & 1u, args.status, FTimeoutNs / 8);
      }
    }
  } else if (warp == 1) {
    // ---- MMA issuer: one TMEM slice buffer per 128-wide K slice ----
    if (lane == 0) {
      const uint32_t idesc = idesc_f8_f32(FBM, FBN, (uint32_t)args.a_format, kF8E4M3);
      int stage = 0;
      uint32_t phase = 0;
      uint32_t slice = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
        for (int kb = 0; kb < KB; ++kb, ++slice) {
          const uint32_t sb = slice & 1u, sph = (slice >> 1) & 1u;
          if (!mbar_wait_bounded(&sempty[sb], sph ^ 1u, args.status, FTimeoutNs) ||
              !mbar_wait_bounded(&full[stage], phase, args.status, FTimeoutNs)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(base + (size_t)stage * FStageBytes);
          const uint32_t b0 = a0 + FABytes;
#pragma unroll
          for (int k = 0; k < FBK / 32; ++k)
            mma_e4m3(tmem_base + sb * FBN, smem_desc_sw128(a0 + k * 32),
                     smem_desc_sw128(b0 + k * 32), idesc, k != 0);
          mma_commit(&empty[stage]);
          mma_commit(&sfull[sb]);
          if (++stage == FStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      mma_commit(drain);
      mbar_wait_bounded(drain, 0, args.status, FTimeoutNs / 8);
    }
  } else {
    // ---- epilogue: warps 2 .. kEpiW+1 ----
    // Warp w may read TMEM lanes 32*(w%4)..+31 (its row quadrant); the kSub
    // warps of a quadrant split the 256 columns: in GEMM1 warp `sub` owns the
    // gate columns kFeat*sub.. and the up columns 128+kFeat*sub.. (hidden
    // features kFeat*sub..+kFeat-1 of the tile), in GEMM2 the kCols columns
    // kCols*sub..
    const int q = warp & 3;
    const int sub = (warp - 2) >> 2;
    const int row = q * 32 + lane;
    uint32_t slice = 0;
    int local = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x, ++local) {
      int g, n, m;
      decode(tile, g, n, m);
      const int rows_g = (g < args.N) ? args.offsets[g + 1] - args.offsets[g] : args.T;
      const int r = m * FBM + row;
      const bool valid =
          r < rows_g && (g == args.N || args.offsets[g] + r < args.rows_routed);
      // the scale box starts at the tile's first row rounded down to 4
      const int arow0 = ((g < args.N) ? args.offsets[g] : args.a_shared_row0) + m * FBM;
      const int sc_off = (arow0 & 3) + row;
      // the slot's two weight-block scales follow the activation box: GEMM1
      // uses the gate block for its first 32 columns and the up block for the
      // rest, GEMM2 the block of its 64 columns
      const int wA = (kEpi == kFEpiSwiGLUQuant) ? 0 : (sub * kCols) / FBM;
      const int wB = (kEpi == kFEpiSwiGLUQuant) ? 1 : (sub * kCols) / FBM;
      float acc[kCols];
#pragma unroll
      for (int i = 0; i < kCols; ++i) acc[i] = 0.f;
      for (int kb = 0; kb < KB; ++kb, ++slice) {
        const uint32_t sb = slice & 1u, sph = (slice >> 1) & 1u;
        const uint32_t cs = slice % FScaleSlots, cph = (slice / FScaleSlots) & 1u;
        if (!mbar_wait_bounded(&scfull[cs], cph, args.status, FTimeoutNs)) {
          ok = false;
          break;
        }
        const float* slot_sc = sc_ring + cs * (FScaleSlotBytes / 4);
        const float sa = slot_sc[sc_off];
        const float sA = sa * slot_sc[FScaleBox + wA], sB = sa * slot_sc[FScaleBox + wB];
        __syncwarp();
        if (lane == 0) mbar_arrive(&scempty[cs]);
        // load c (kLd columns) of this warp: GEMM1 gate loads first, then up
        constexpr int kLoads = kCols / kLd;
        if (!mbar_wait_bounded(&sfull[sb], sph, args.status, FTimeoutNs)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + sb * FBN;
#pragma unroll
        for (int c0 = 0; c0 < kLoads; c0 += kInFlight) {
          uint32_t p[kInFlight][kLd];
#pragma unroll
          for (int j = 0; j < kInFlight; ++j) {
            const int c = c0 + j;
            int col;
            if constexpr (kEpi == kFEpiSwiGLUQuant)
              col = (c < kLoads / 2) ? kFeat * sub + kLd * c
                                     : 128 + kFeat * sub + kLd * (c - kLoads / 2);
            else
              col = kCols * sub + kLd * c;
            if constexpr (kLd == 32)
              tmem_ld32(taddr + col, p[j]);
            else
              tmem_ld16(taddr + col, p[j]);
          }
          tmem_wait_ld();
          if (c0 + kInFlight == kLoads) {
            // the whole slice is in registers: hand the buffer back to the
            // MMA before the last multiply-adds
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sempty[sb]);
          }
#pragma unroll
          for (int j = 0; j < kInFlight; ++j) {
            const int c = c0 + j;
            const float sc = (c < kLoads / 2) ? sA : sB;
#pragma unroll
            for (int i = 0; i < kLd; i += 2)
              ffma2(acc[c * kLd + i], acc[c * kLd + i + 1], __uint_as_float(p[j][i]),
                    __uint_as_float(p[j][i + 1]), sc);
          }
        }
      }
      if (!ok) break;

      if constexpr (kEpi == kFEpiSwiGLUQuant) {
        // h for hidden features n*128 + kFeat*sub + i, i < kFeat
        float amax = 0.f;
#pragma unroll
        for (int i = 0; i < kFeat; ++i) {
          acc[i] = silu_fast(acc[i]) * acc[kFeat + i];
          amax = fmaxf(amax, fabsf(acc[i]));
        }
        // the row's 1x128 tile spans the kSub warps of this quadrant
        float* xb = xchg + (local & 1) * 4 * FBM;
        xb[sub * FBM + row] = amax;
        __syncwarp();
        if (lane == 0) mbar_arrive(&xbar[local & 1]);
        if (!mbar_wait_bounded(&xbar[local & 1], (local >> 1) & 1, args.status, FTimeoutNs)) break;
        amax = (kSub == 4) ? fmaxf(fmaxf(xb[row], xb[FBM + row]),
                                   fmaxf(xb[2 * FBM + row], xb[3 * FBM + row]))
                           : fmaxf(xb[row], xb[FBM + row]);
        const bool zero = amax == 0.f;
        const float scale = zero ? 1.f : __fdiv_rn(amax, 448.f);
        const float inv = zero ? 0.f : __fdiv_rn(448.f, amax);
        if (valid) {
          uint8_t* qrow = ((g < args.N) ? args.q_routed + (long long)args.offsets[g] * args.out_ld
                                        : args.q_shared) +
                          (long long)r * args.out_ld + n * QB + kFeat * sub;
#pragma unroll
          for (int v = 0; v < kFeat / 16; ++v) {
            uint32_t w4[4];
#pragma unroll
            for (int wd = 0; wd < 4; ++wd) {
              uint32_t word = 0;
#pragma unroll
              for (int qq = 0; qq < 2; ++qq) {
                const int i = 16 * v + 4 * wd + 2 * qq;
                const __nv_fp8x2_storage_t c2 =
                    zero ? (__nv_fp8x2_storage_t)0
                         : __nv_cvt_float2_to_fp8x2(
                               make_float2(__fmul_rn(acc[i], inv), __fmul_rn(acc[i + 1], inv)),
                               __NV_SATFINITE, __NV_E4M3);
                word |= (uint32_t)c2 << (16 * qq);
              }
              w4[wd] = word;
            }
            reinterpret_cast<uint4*>(qrow)[v] = make_uint4(w4[0], w4[1], w4[2], w4[3]);
          }
          if (sub == 0) {
            float* qs = (g < args.N) ? args.qs_routed + args.offsets[g] : args.qs_shared;
            qs[(long long)n * args.qs_ld + r] = scale;
          }
        }
      } else if constexpr (kEpi == kFEpiSwiGLUBwd) {
        // acc holds dh for hidden features n*256 + kCols*sub + i; g, u and the
        // outputs dg, du sit in the packed [rows, 2f] layout (gate block of
        // 128 features, then their up block)
        if (valid) {
          const long long orow = (g < args.N) ? (long long)args.offsets[g] + r : (long long)r;
          const __nv_bfloat16* arow =
              ((g < args.N) ? args.aux_routed : args.aux_shared) + orow * args.out_ld;
          __nv_bfloat16* drow = ((g < args.N) ? args.y_routed : args.y_shared) + orow * args.out_ld;
#pragma unroll
          for (int i0 = 0; i0 < kCols; i0 += 8) {
            const int j0 = n * FBN + kCols * sub + i0;       // first feature of the 8
            const int col = (j0 / 128) * 256 + (j0 % 128);   // its gate column; up at +128
            float gt[8], up[8], dg[8], du[8];
            bf16x8_load(arow + col, gt);
            bf16x8_load(arow + col + 128, up);
#pragma unroll
            for (int i = 0; i < 8; ++i) swiglu_bwd(acc[i0 + i], gt[i], up[i], dg[i], du[i]);
            uint4 wg, wu;
            __nv_bfloat162* hg = reinterpret_cast<__nv_bfloat162*>(&wg);
            __nv_bfloat162* hu = reinterpret_cast<__nv_bfloat162*>(&wu);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              hg[i] = __floats2bfloat162_rn(dg[2 * i], dg[2 * i + 1]);
              hu[i] = __floats2bfloat162_rn(du[2 * i], du[2 * i + 1]);
            }
            *reinterpret_cast<uint4*>(drow + col) = wg;
            *reinterpret_cast<uint4*>(drow + col + 128) = wu;
          }
        }
      } else {
        // a warp whose 32 rows all lie inside the group stores them by TMA;
        // the ragged last rows of a group take the row stores below
        const int r0 = m * FBM + q * 32;
        bool tma_rows = false;
        if constexpr (kTmaY) {
          tma_rows = args.y_tma != 0 && r0 + 32 <= rows_g &&
                     (g == args.N || args.offsets[g] + r0 + 32 <= args.rows_routed);
          if (tma_rows) {
            uint8_t* stg = staging + (size_t)(warp - 2) * (2 * FStgPiece);
            const CUtensorMap* ym = (g < args.N) ? &args.tmY_routed : &args.tmY_shared;
            const int yrow = ((g < args.N) ? args.offsets[g] : 0) + r0;
            const int ycol = n * FBN + kCols * sub;
            const int sw = (lane >> 2) & 1;  // the 32-byte swizzle of row `lane`
#pragma unroll
            for (int c = 0; c < kCols / 16; ++c) {
              uint8_t* buf = stg + (c & 1) * FStgPiece;
              if (lane == 0) bulk_wait_read_but_one();  // this piece's buffer is free
              __syncwarp();
              uint8_t* my = buf + lane * 32;
              const float* a = acc + 16 * c;
              *reinterpret_cast<uint4*>(my + (sw << 4)) =
                  make_uint4(bf16x2_bits(a[0], a[1]), bf16x2_bits(a[2], a[3]),
                             bf16x2_bits(a[4], a[5]), bf16x2_bits(a[6], a[7]));
              *reinterpret_cast<uint4*>(my + ((sw ^ 1) << 4)) =
                  make_uint4(bf16x2_bits(a[8], a[9]), bf16x2_bits(a[10], a[11]),
                             bf16x2_bits(a[12], a[13]), bf16x2_bits(a[14], a[15]));
              fence_proxy_async_smem();
              __syncwarp();
              if (lane == 0) {
                tma_store_2d(ym, buf, ycol + 16 * c, yrow);
                bulk_commit_group();
              }
            }
          }
        }
        if (!tma_rows && valid) {
          __nv_bfloat16* yrow =
              ((g < args.N) ? args.y_routed + ((long long)args.offsets[g] + r) * args.out_ld
                            : args.y_shared + (long long)r * args.out_ld) +
              n * FBN + kCols * sub;
#pragma unroll
          for (int v = 0; v < kCols / 8; ++v) {
            uint4 w;
            __nv_bfloat162* hb = reinterpret_cast<__nv_bfloat162*>(&w);
#pragma unroll
            for (int i = 0; i < 4; ++i)
              hb[i] = __floats2bfloat162_rn(acc[8 * v + 2 * i], acc[8 * v + 2 * i + 1]);
            reinterpret_cast<uint4*>(yrow)[v] = w;
          }
        }
      }
    }
    // the staging buffers must outlive the stores that read them
    if constexpr (kTmaY) {
      if (lane == 0) bulk_wait_all();
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
  if (clock_cta)
    clock_stop(cm, reinterpret_cast<unsigned long long*>(
                       reinterpret_cast<uint8_t*>(args.status) + kClockRecordOffset + 16));
}

template <int kEpi, int kEpiW, int kLd, int kInFlight>
cudaError_t launch_fp8_gemm_w(const Fp8Args& a0, cudaStream_t st) {
  constexpr bool kTmaY = kEpi == kFEpiStore && kEpiW == 8;
  const size_t smem = fp8_smem_bytes(a0.N + 1, kTmaY);
  auto kernel = grouped_gemm_fp8_kernel<kEpi, kEpiW, kLd, kInFlight>;
  cudaError_t e = note_cuda(cudaFuncSetAttribute(kernel,
                                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 (int)smem),
                            "fp8 GEMM: set shared-memory size");
  if (e != cudaSuccess) return e;
  Fp8Args a = a0;
  a.y_tma = 0;
  if constexpr (kTmaY) {
    // TMA stores need 16-byte aligned outputs; otherwise every row takes the
    // row stores
    const auto BF = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    const bool aligned = (reinterpret_cast<uintptr_t>(a.y_routed) % 16 == 0) &&
                         (reinterpret_cast<uintptr_t>(a.y_shared) % 16 == 0) &&
                         ((size_t)a.out_ld * 2) % 16 == 0;
    if (aligned &&
        make_map_swizzled(&a.tmY_routed, a.y_routed, BF, 2, a.out_ld, a.rows_routed, 16, 32,
                          CU_TENSOR_MAP_SWIZZLE_32B) &&
        make_map_swizzled(&a.tmY_shared, a.y_shared, BF, 2, a.out_ld, a.T, 16, 32,
                          CU_TENSOR_MAP_SWIZZLE_32B))
      a.y_tma = 1;
  }
  kernel<<<num_sms(), fp8_threads(kEpiW), smem, st>>>(a);
  return note_cuda(cudaGetLastError(), "fp8 GEMM launch");
}

// The epilogue's TMEM read shape, chosen once per process by MOE_FP8_EPI:
//   unset   8 warps, 16-column loads, two per wait (128 running sums per thread;
//           measured 2.5-4.5% faster than the 16-warp shape on the V3 FP8 layer)
//   narrow  16 warps, 16-column loads, one per wait (64 running sums per thread)
//   x32     16 warps, 32-column loads, one per wait
//   wide32  8 warps, 32-column loads, one per wait
// (the 16-warp shapes run at 96 registers a thread and spill; x32 and wide32
// spill more and measured slower.  The 18-warp CTA cannot have more registers:
// compiled for 112 a thread, its launch is refused; a 20-warp CTA that moves
// registers from its control warpgroup to the epilogue with setmaxnreg spills
// the TMA and MMA loops instead, 0.6-0.8 KB a thread at 32-56 registers.  A
// 12-warp CTA with a 88/208 setmaxnreg split and four loads in flight, and a
// ring of four 128-column slice buffers fed by N=128 MMAs, were both exact
// and slower: the slice handshake, not the read shape, bounds the kernel)
int fp8_epilogue_kind() {
  static int v = -1;
  if (v < 0) {
    const char* e = std::getenv("MOE_FP8_EPI");
    v = 2;
    if (e != nullptr && std::strcmp(e, "narrow") == 0) v = 0;
    if (e != nullptr && std::strcmp(e, "x32") == 0) v = 1;
    if (e != nullptr && std::strcmp(e, "wide32") == 0) v = 3;
  }
  return v;
}

template <int kEpi>
cudaError_t launch_fp8_gemm(const Fp8Args& a, cudaStream_t st) {
  switch (fp8_epilogue_kind()) {
    case 0: return launch_fp8_gemm_w<kEpi, 16, 16, 1>(a, st);
    case 1: return launch_fp8_gemm_w<kEpi, 16, 32, 1>(a, st);
    case 3: return launch_fp8_gemm_w<kEpi, 8, 32, 1>(a, st);
    default: return launch_fp8_gemm_w<kEpi, 8, 16, 2>(a, st);
  }
}

}  // namespace

namespace {
template <bool kE5M2>
cudaError_t quant_rows(const void* x, long long rows, int d, uint8_t* q, float* sc,
                       long long sc_ld, cudaStream_t st) {
  const long long tiles = rows * (d / QB);
  long long blocks = (tiles * 16 + 255) / 256;
  if (blocks > 148 * 16) blocks = 148 * 16;
  if (blocks < 1) blocks = 1;
  quant_rows_kernel<kE5M2><<<(int)blocks, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(x),
                                                        rows, d, q, sc, sc_ld);
  return note_cuda(cudaGetLastError(), "1x128 quantisation launch");
}
}  // namespace

cudaError_t launch_quant_rows(const void* x, long long rows, int d, uint8_t* q, float* sc,
                              long long sc_ld, cudaStream_t st) {
  return quant_rows<false>(x, rows, d, q, sc, sc_ld, st);
}

cudaError_t launch_quant_rows_e5m2(const void* g, long long rows, int d, uint8_t* q, float* sc,
                                   long long sc_ld, cudaStream_t st) {
  return quant_rows<true>(g, rows, d, q, sc, sc_ld, st);
}

cudaError_t launch_quantize_weights(const moe_shape& s, const void* w13, const void* w2,
                                    void* w13_q, float* w13_scales, void* w2_q,
                                    float* w2_scales, cudaStream_t st) {
  const long long E = s.N + 1;
  // w13 [E * 2f, d]: blocks of 128 rows x 128 columns
  const long long br13 = E * 2 * s.f / QB;
  const int bc13 = s.d / QB;
  quant_blocks_kernel<<<(unsigned)(br13 * bc13), 128, 0, st>>>(
      static_cast<const __nv_bfloat16*>(w13), s.d, br13, bc13, static_cast<uint8_t*>(w13_q),
      w13_scales);
  const long long br2 = E * s.d / QB;
  const int bc2 = s.f / QB;
  quant_blocks_kernel<<<(unsigned)(br2 * bc2), 128, 0, st>>>(
      static_cast<const __nv_bfloat16*>(w2), s.f, br2, bc2, static_cast<uint8_t*>(w2_q),
      w2_scales);
  return cudaGetLastError();
}

// The transposed weights W13^T [N+1, d, 2f] and W2^T [N+1, f, d] (bf16, from
// moe_transpose_weights) quantised per 128x128 block like the forward's: the
// blocks are the forward's blocks transposed, so codes and scales are theirs.
cudaError_t launch_quantize_weights_transposed(const moe_shape& s, const void* w13t,
                                               const void* w2t, void* w13t_q, float* w13t_scales,
                                               void* w2t_q, float* w2t_scales, cudaStream_t st) {
  const long long E = s.N + 1;
  const long long br13 = E * s.d / QB;
  const int bc13 = 2 * s.f / QB;
  quant_blocks_kernel<<<(unsigned)(br13 * bc13), 128, 0, st>>>(
      static_cast<const __nv_bfloat16*>(w13t), 2 * s.f, br13, bc13,
      static_cast<uint8_t*>(w13t_q), w13t_scales);
  const long long br2 = E * s.f / QB;
  const int bc2 = s.d / QB;
  quant_blocks_kernel<<<(unsigned)(br2 * bc2), 128, 0, st>>>(
      static_cast<const __nv_bfloat16*>(w2t), s.d, br2, bc2, static_cast<uint8_t*>(w2t_q),
      w2t_scales);
  return cudaGetLastError();
}

BwdLayoutFp8 bwd_layout_fp8(const moe_shape& s) {
  auto al = [](size_t v) { return (v + 255) & ~size_t(255); };
  const size_t TK = (size_t)s.T * s.K, rows = TK + s.T;
  const size_t ld_rows = (size_t)scale_ld((long long)rows), ld_x = (size_t)scale_ld(s.T);
  const size_t twof = 2 * (size_t)s.f;
  BwdLayoutFp8 B;
  size_t off = 256;
  B.gu = off;
  off = al(off + rows * twof * 2);
  B.dgu = off;
  off = al(off + rows * twof * 2);
  B.xq = off;
  off = al(off + (size_t)s.T * s.d);
  B.xs = off;
  off = al(off + (size_t)(s.d / QB) * ld_x * 4);
  B.dyq = off;
  off = al(off + rows * s.d);
  B.dys = off;
  off = al(off + (size_t)(s.d / QB) * ld_rows * 4);
  B.dguq = off;
  off = al(off + rows * twof);
  B.dgus = off;
  off = al(off + (twof / QB) * ld_rows * 4);
  // weight-gradient pass
  const size_t R = (size_t)wgrad_cols_fp8(s), KT = R / QB;
  const size_t ld_d = (size_t)scale_ld(s.d), ld_f = (size_t)scale_ld(s.f);
  const size_t ld_2f = (size_t)scale_ld((long long)twof);
  B.colbase = off;
  off = al(off + (size_t)(s.N + 2) * 4);
  B.at = off;
  off = al(off + (size_t)s.d * R * 2);
  B.dyt = off;
  off = al(off + (size_t)s.d * R * 2);
  B.ht = off;
  off = al(off + (size_t)s.f * R * 2);
  B.dgut = off;
  off = al(off + twof * R * 2);
  B.atq = off;
  off = al(off + (size_t)s.d * R);
  B.dytq = off;
  off = al(off + (size_t)s.d * R);
  B.htq = off;
  off = al(off + (size_t)s.f * R);
  B.dgutq = off;
  off = al(off + twof * R);
  B.ats = off;
  off = al(off + KT * ld_d * 4);
  B.dyts = off;
  off = al(off + KT * ld_d * 4);
  B.hts = off;
  off = al(off + KT * ld_f * 4);
  B.dguts = off;
  off = al(off + KT * ld_2f * 4);
  B.total = off;
  return B;
}

// The experts' input gradients in FP8 (E5M2 gradients against E4M3 weights):
//   1. g, u recomputed from the forward's E4M3 operands, stored bf16 (Store);
//   2. dY quantised to E5M2 per 1x128 along d;
//   3. dH = dY W2 against W2^T's E4M3 blocks, SwiGLU-backward epilogue -> dg, du bf16;
//   4. dG U quantised to E5M2 per 1x128 along 2f;
//   5. dX = dGU W13 against W13^T's E4M3 blocks (Store).
int launch_ffn_bwd_dx_e4m3(const moe_shape& s, const void* x_perm, const float* x_perm_scales,
                           const int32_t* offsets, const void* x, const void* w13q,
                           const float* w13_scales, const void* w13tq, const float* w13t_scales,
                           const void* w2tq, const float* w2t_scales, const void* dy_perm,
                           const void* dy_shared, void* dx_perm, void* dx_shared, void* ws_bwd,
                           cudaStream_t st) {
  const BwdLayoutFp8 B = bwd_layout_fp8(s);
  uint8_t* w = static_cast<uint8_t*>(ws_bwd);
  uint32_t* status = reinterpret_cast<uint32_t*>(w);
  __nv_bfloat16* GU = reinterpret_cast<__nv_bfloat16*>(w + B.gu);
  __nv_bfloat16* dGU = reinterpret_cast<__nv_bfloat16*>(w + B.dgu);
  uint8_t* xq = w + B.xq;
  float* xs = reinterpret_cast<float*>(w + B.xs);
  uint8_t* dyq = w + B.dyq;
  float* dys = reinterpret_cast<float*>(w + B.dys);
  uint8_t* dguq = w + B.dguq;
  float* dgus = reinterpret_cast<float*>(w + B.dgus);
  const uint64_t TK = (uint64_t)s.T * s.K, rows = TK + s.T;
  const uint64_t twof = 2ull * s.f;
  const auto U8 = CU_TENSOR_MAP_DATA_TYPE_UINT8;
  const long long ld_routed = scale_ld((long long)TK), ld_x = scale_ld(s.T);
  const long long ld_rows = scale_ld((long long)rows);
  auto common = [&](Fp8Args& a, int n_acc, int k_dim, int out_ld, int a_format,
                    int a_shared_row0) {
    a.offsets = offsets;
    a.status = status;
    a.N = s.N;
    a.T = s.T;
    a.rows_routed = (int)TK;
    a.a_shared_row0 = a_shared_row0;
    a.n_acc = n_acc;
    a.k_dim = k_dim;
    a.out_ld = out_ld;
    a.a_format = a_format;
  };

  // 1. g, u = A W13^T in E4M3, stored bf16 [rows, 2f]
  if (launch_quant_rows(x, s.T, s.d, xq, xs, ld_x, st) != cudaSuccess) return MOE_ERR_CUDA;
  Fp8Args g1{};
  bool ok = make_map(&g1.tmA_routed, x_perm, U8, 1, s.d, TK, FBK, FBM) &&
            make_map(&g1.tmA_shared, xq, U8, 1, s.d, s.T, FBK, FBM) &&
            make_map(&g1.tmB, w13q, U8, 1, s.d, (uint64_t)(s.N + 1) * twof, FBK, FBN) &&
            make_map_f32_rows(&g1.tmS_routed, x_perm_scales, ld_routed, s.d / QB, FScaleBox) &&
            make_map_f32_rows(&g1.tmS_shared, xs, ld_x, s.d / QB, FScaleBox);
  if (!ok) {
    note_text("fp8 backward GEMM1: tensor-map encoding failed");
    return MOE_ERR_CUDA;
  }
  common(g1, (int)twof, s.d, (int)twof, kF8E4M3, 0);
  g1.sw = w13_scales;
  g1.y_routed = GU;
  g1.y_shared = GU + TK * twof;
  if (launch_fp8_gemm<kFEpiStore>(g1, st) != cudaSuccess) return MOE_ERR_CUDA;

  // 2. dY -> E5M2, routed rows then shared rows, one block-major scale array
  if (launch_quant_rows_e5m2(dy_perm, (long long)TK, s.d, dyq, dys, ld_rows, st) != cudaSuccess ||
      launch_quant_rows_e5m2(dy_shared, s.T, s.d, dyq + TK * s.d, dys + TK, ld_rows, st) !=
          cudaSuccess)
    return MOE_ERR_CUDA;

  // 3. dH = dY W2 (B = W2^T [(N+1) f, d]), SwiGLU backward into dGU
  Fp8Args g2{};
  ok = make_map(&g2.tmA_routed, dyq, U8, 1, s.d, rows, FBK, FBM) &&
       make_map(&g2.tmA_shared, dyq, U8, 1, s.d, rows, FBK, FBM) &&
       make_map(&g2.tmB, w2tq, U8, 1, s.d, (uint64_t)(s.N + 1) * s.f, FBK, FBN) &&
       make_map_f32_rows(&g2.tmS_routed, dys, ld_rows, s.d / QB, FScaleBox) &&
       make_map_f32_rows(&g2.tmS_shared, dys, ld_rows, s.d / QB, FScaleBox);
  if (!ok) {
    note_text("fp8 backward dH GEMM: tensor-map encoding failed");
    return MOE_ERR_CUDA;
  }
  common(g2, s.f, s.d, (int)twof, kF8E5M2, (int)TK);
  g2.sw = w2t_scales;
  g2.aux_routed = GU;
  g2.aux_shared = GU + TK * twof;
  g2.y_routed = dGU;
  g2.y_shared = dGU + TK * twof;
  if (launch_fp8_gemm<kFEpiSwiGLUBwd>(g2, st) != cudaSuccess) return MOE_ERR_CUDA;

  // 4. dGU -> E5M2 over all rows
  if (launch_quant_rows_e5m2(dGU, (long long)rows, (int)twof, dguq, dgus, ld_rows, st) !=
      cudaSuccess)
    return MOE_ERR_CUDA;

  // 5. dX = dGU W13 (B = W13^T [(N+1) d, 2f])
  Fp8Args g3{};
  ok = make_map(&g3.tmA_routed, dguq, U8, 1, twof, rows, FBK, FBM) &&
       make_map(&g3.tmA_shared, dguq, U8, 1, twof, rows, FBK, FBM) &&
       make_map(&g3.tmB, w13tq, U8, 1, twof, (uint64_t)(s.N + 1) * s.d, FBK, FBN) &&
       make_map_f32_rows(&g3.tmS_routed, dgus, ld_rows, (int)(twof / QB), FScaleBox) &&
       make_map_f32_rows(&g3.tmS_shared, dgus, ld_rows, (int)(twof / QB), FScaleBox);
  if (!ok) {
    note_text("fp8 backward dX GEMM: tensor-map encoding failed");
    return MOE_ERR_CUDA;
  }
  common(g3, s.d, (int)twof, s.d, kF8E5M2, (int)TK);
  g3.sw = w13t_scales;
  g3.y_routed = static_cast<__nv_bfloat16*>(dx_perm);
  g3.y_shared = static_cast<__nv_bfloat16*>(dx_shared);
  if (launch_fp8_gemm<kFEpiStore>(g3, st) != cudaSuccess) return MOE_ERR_CUDA;
  return MOE_OK;
}

int launch_ffn_tc_e4m3(const moe_shape& s, const void* x_perm, const float* x_perm_scales,
                       const int32_t* offsets, const void* x, const void* w13, const void* w2,
                       const float* w13_scales, const float* w2_scales, void* y_perm,
                       void* y_shared, void* ws, cudaStream_t st) {
  const WsLayout L = ws_layout(s);
  uint8_t* w = static_cast<uint8_t*>(ws);
  uint8_t* Hq = w + L.h;
  float* Hs = reinterpret_cast<float*>(w + L.h_scales);
  uint8_t* xq = w + L.xq;
  float* xs = reinterpret_cast<float*>(w + L.xq_scales);
  uint32_t* status = reinterpret_cast<uint32_t*>(w + L.status);
  const uint64_t TK = (uint64_t)s.T * s.K;
  const auto U8 = CU_TENSOR_MAP_DATA_TYPE_UINT8;

  // scale arrays are block-major [K/128][ld]
  const long long ld_routed = scale_ld((long long)TK), ld_x = scale_ld(s.T);
  const long long ld_h = scale_ld((long long)TK + s.T);
  // the shared expert reads x: quantise it per 1x128 tile first
  if (launch_quant_rows(x, s.T, s.d, xq, xs, ld_x, st) != cudaSuccess) return MOE_ERR_CUDA;

  Fp8Args g1{};
  bool ok = make_map(&g1.tmA_routed, x_perm, U8, 1, s.d, TK, FBK, FBM) &&
            make_map(&g1.tmA_shared, xq, U8, 1, s.d, s.T, FBK, FBM) &&
            make_map(&g1.tmB, w13, U8, 1, s.d, (uint64_t)(s.N + 1) * 2 * s.f, FBK, FBN) &&
            make_map_f32_rows(&g1.tmS_routed, x_perm_scales, ld_routed, s.d / QB, FScaleBox) &&
            make_map_f32_rows(&g1.tmS_shared, xs, ld_x, s.d / QB, FScaleBox);
  if (!ok) {
    note_text("fp8 GEMM1: tensor-map encoding failed");
    return MOE_ERR_CUDA;
  }
  g1.offsets = offsets;
  g1.sw = w13_scales;
  g1.q_routed = Hq;
  g1.q_shared = Hq + TK * s.f;
  g1.qs_routed = Hs;
  g1.qs_shared = Hs + TK;
  g1.qs_ld = ld_h;
  g1.status = status;
  g1.N = s.N;
  g1.T = s.T;
  g1.rows_routed = (int)TK;
  g1.a_shared_row0 = 0;
  g1.n_acc = 2 * s.f;
  g1.k_dim = s.d;
  g1.out_ld = s.f;
  if (launch_fp8_gemm<kFEpiSwiGLUQuant>(g1, st) != cudaSuccess) return MOE_ERR_CUDA;

  Fp8Args g2{};
  ok = make_map(&g2.tmA_routed, Hq, U8, 1, s.f, TK + s.T, FBK, FBM) &&
       make_map(&g2.tmA_shared, Hq, U8, 1, s.f, TK + s.T, FBK, FBM) &&
       make_map(&g2.tmB, w2, U8, 1, s.f, (uint64_t)(s.N + 1) * s.d, FBK, FBN) &&
       make_map_f32_rows(&g2.tmS_routed, Hs, ld_h, s.f / QB, FScaleBox) &&
       make_map_f32_rows(&g2.tmS_shared, Hs, ld_h, s.f / QB, FScaleBox);
  if (!ok) {
    note_text("fp8 GEMM2: tensor-map encoding failed");
    return MOE_ERR_CUDA;
  }
  g2.offsets = offsets;
  g2.sw = w2_scales;
  g2.y_routed = static_cast<__nv_bfloat16*>(y_perm);
  g2.y_shared = static_cast<__nv_bfloat16*>(y_shared);
  g2.status = status;
  g2.N = s.N;
  g2.T = s.T;
  g2.rows_routed = (int)TK;
  g2.a_shared_row0 = (int)TK;
  g2.n_acc = s.d;
  g2.k_dim = s.f;
  g2.out_ld = s.d;
  if (launch_fp8_gemm<kFEpiStore>(g2, st) != cudaSuccess) return MOE_ERR_CUDA;
  return MOE_OK;
}

}  // namespace moe
