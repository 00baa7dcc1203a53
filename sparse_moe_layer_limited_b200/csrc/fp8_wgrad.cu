// FP8 weight gradients of the experts: E5M2 gradients against E4M3
// activations (the 10100.com article on the V3 report, FP8 paragraph: E4M3
// forward, E5M2 backward), each operand scaled per 128-row tile along the
// contraction from its online max-abs (the mhpq.cn article §4.1 fine-grained
// scaling, the tile laid along the contraction as in every FP8 product here).
//
// Per expert e (group N = the shared expert):
//   dW2_e  [d, f]  = dY_e^T H_e        dW13_e [2f, d] = [dg du]_e^T A_e
// Layout pass (gemm_wgrad.cu's transposes with 128-column padding, A gathered
// from x through perm_tok), then each transposed operand [C, R] is quantised
// per 1x128 tile of its rows, i.e. per 128 expert rows of one feature:
// scales [R/128][C] block-major.  The GEMM is the K-grouped unit loop of the
// bf16 weight-gradient kernel with the FP8 per-slice promotion of fp8.cu: a
// unit is one 128 x 256 gradient tile of one expert, its K loop the expert's
// column block in 128-row slices; every slice lands in one of two 256-column
// TMEM buffers (tcgen05.mma kind::f8f6f4, E5M2 x E4M3, K=32 per MMA) and
// sixteen epilogue warps (four per TMEM lane quadrant, 64 columns each) fold
// it into fp32 register sums with the slice's scale product, a row scale
// times a column scale.  The producer stages each slice's 128 row scales and
// 256 column scales in a ring of shared-memory slots by TMA.
// All waits are bounded (~2 s) and set the device status word on expiry.
#include <cuda.h>
#include <cuda_bf16.h>

#include <cstdlib>
#include <cstring>

#include "epilogue.cuh"
#include "internal.h"
#include "ptx.cuh"

namespace moe {
namespace {

constexpr int GBM = 128, GBK = 128;  // gradient tile rows; K slice (one scale tile)
constexpr int GABytes = GBM * GBK;   // 16 KB (one byte per element)
// warp 0 TMA, warp 1 MMA, then kEpiW epilogue warps (kEpiW / 4 per TMEM lane quadrant)
__host__ __device__ constexpr int wgrad_threads(int epi_warps) { return 64 + 32 * epi_warps; }
constexpr int GScaleSlots = 8;
constexpr uint64_t GTimeoutNs = 2000000000ull;

// Tile configuration by gradient-tile width kBN (256 or 128 columns): the 512
// TMEM columns hold 512 / kBN slice buffers, so a narrower tile gives the MMA
// more slices of slack and each epilogue thread fewer running sums
// The 128-column tiles store their gradient through shared memory by TMA
// (eight epilogue warps, one 32-row x 64-column 128B-swizzled staging buffer
// each); the 256-column tiles store rows directly.
template <int kBN>
struct WgTile {
  static constexpr int kBufs = 512 / kBN;
  static constexpr int kBBytes = kBN * GBK;
  static constexpr int kStageBytes = GABytes + kBBytes;
  static constexpr bool kTmaStore = kBN == 128;
  static constexpr int kStages = kBN == 256 ? 4 : 5;
  static constexpr int kStgBytes = kTmaStore ? 8 * 32 * 128 : 0;  // all epilogue warps
  static constexpr int kScaleSlotBytes = (GBM + kBN) * 4;  // row scales, then column scales
  static constexpr size_t kSmemBytes = 1024 + (size_t)kStages * kStageBytes + kStgBytes +
                                       (size_t)GScaleSlots * kScaleSlotBytes + 512;
  static_assert(kSmemBytes <= 232448, "FP8 weight-gradient kernel exceeds the shared memory");
};

struct alignas(64) Fp8WgradArgs {
  CUtensorMap tmL;   // left codes [M_total, R] E5M2 (the gradient), box {128, 128}
  CUtensorMap tmR;   // right codes [N_total, R] E4M3 (the activation), box {128, kBN}
  CUtensorMap tmSL;  // left scales [R/128, ld] fp32, box {128, 1}
  CUtensorMap tmSR;  // right scales [R/128, ld] fp32, box {kBN, 1}
  CUtensorMap tmOut; // gradient [G1 * M_total, N_total] bf16, box {64, 32}, 128B swizzle
  const int32_t* colbase;  // [G1 + 1] column block of each group, multiples of 128
  __nv_bfloat16* out;      // [G1, M_total, N_total]
  uint32_t* status;
  int G1, M_total, N_total;
};

// {m0, m1} = {a0 * s, a1 * s} as one packed fp32x2 multiply
__device__ __forceinline__ void fmul2_s(float& m0, float& m1, float a0, float a1, float s) {
  asm("{\n\t.reg .b64 ra, rb, rc;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %4};\n\t"
      "mul.rn.f32x2 rc, ra, rb;\n\tmov.b64 {%0, %1}, rc;\n\t}"
      : "=f"(m0), "=f"(m1)
      : "f"(a0), "f"(a1), "f"(s));
}
// {acc0, acc1} += {x0 * s0, x1 * s1} as one packed fp32x2 fused multiply-add
__device__ __forceinline__ void ffma2_v(float& acc0, float& acc1, float x0, float x1, float s0,
                                       float s1) {
  asm("{\n\t.reg .b64 ra, rb, rc;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "mov.b64 rc, {%0, %1};\n\tfma.rn.f32x2 rc, ra, rb, rc;\n\tmov.b64 {%0, %1}, rc;\n\t}"
      : "+f"(acc0), "+f"(acc1)
      : "f"(x0), "f"(x1), "f"(s0), "f"(s1));
}

// kBN-column gradient tiles; kEpiW epilogue warps, each reading its slice
// columns 16 at a time with kInFlight TMEM loads per wait
template <int kBN, int kEpiW, int kInFlight>
__global__ void __launch_bounds__(wgrad_threads(kEpiW), 1) fp8_wgrad_kernel(
    const __grid_constant__ Fp8WgradArgs args) {
  static_assert(kEpiW == 16 || kEpiW == 8, "four or two epilogue warps per lane quadrant");
  using C = WgTile<kBN>;
  static_assert(!C::kTmaStore || kEpiW == 8, "one staging buffer per epilogue warp, eight warps");
  constexpr int GBN = kBN;
  constexpr int GStages = C::kStages;
  constexpr int GStageBytes = C::kStageBytes;
  constexpr int GScaleSlotBytes = C::kScaleSlotBytes;
  constexpr int kBufs = C::kBufs;
  constexpr int GEpiWarps = kEpiW;
  constexpr int kSub = kEpiW / 4;      // epilogue warps per lane quadrant
  constexpr int kCols = GBN / kSub;    // gradient columns per warp
  constexpr int kLoads = kCols / 16;
  static_assert(kLoads % kInFlight == 0, "loads split evenly into waits");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* staging = base + (size_t)GStages * GStageBytes;  // 1024-aligned (stage sizes)
  float* sc_ring = reinterpret_cast<float*>(staging + C::kStgBytes);
  uint64_t* bars = reinterpret_cast<uint64_t*>(staging + C::kStgBytes +
                                               (size_t)GScaleSlots * GScaleSlotBytes);
  uint64_t* full = bars;                       // [GStages]
  uint64_t* empty = full + GStages;            // [GStages]
  uint64_t* sfull = empty + GStages;           // [kBufs] slice buffer written
  uint64_t* sempty = sfull + kBufs;            // [kBufs] slice buffer drained (epilogue warps)
  uint64_t* scfull = sempty + kBufs;           // [GScaleSlots] scale slot landed
  uint64_t* scempty = scfull + GScaleSlots;    // [GScaleSlots] scale slot read (epilogue warps)
  uint64_t* drain = scempty + GScaleSlots;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int MT = args.M_total / GBM, NT = args.N_total / GBN;
  const int per_group = MT * NT;
  const int total = args.G1 * per_group;

  if (tid == 0) {
    for (int s = 0; s < GStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < kBufs; ++a) {
      mbar_init(&sfull[a], 1);
      mbar_init(&sempty[a], GEpiWarps);
    }
    for (int c = 0; c < GScaleSlots; ++c) {
      mbar_init(&scfull[c], 1);
      mbar_init(&scempty[c], GEpiWarps);
    }
    mbar_init(drain, 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  // unit -> group g, row tile m, column tile n (n fastest); K slices of the
  // group's column block
  auto decode = [&](int u, int& g, int& m, int& n, int& kb0, int& kcnt) {
    g = u / per_group;
    const int local = u - g * per_group;
    m = local / NT;
    n = local - m * NT;
    kb0 = args.colbase[g] / GBK;
    kcnt = (args.colbase[g + 1] - args.colbase[g]) / GBK;
  };

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&args.tmL);
      tma_prefetch_desc(&args.tmR);
      tma_prefetch_desc(&args.tmSL);
      tma_prefetch_desc(&args.tmSR);
      int stage = 0;
      uint32_t phase = 0, issued = 0, issued_parity = 0;
      uint32_t sslice = 0, sc_issued = 0, sc_parity = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < total && ok; u += gridDim.x) {
        int g, m, n, kb0, kcnt;
        decode(u, g, m, n, kb0, kcnt);
        for (int kb = 0; kb < kcnt; ++kb, ++sslice) {
          const uint32_t cs = sslice % GScaleSlots, cph = (sslice / GScaleSlots) & 1u;
          if (!mbar_wait_bounded(&empty[stage], phase ^ 1u, args.status, GTimeoutNs) ||
              !mbar_wait_bounded(&scempty[cs], cph ^ 1u, args.status, GTimeoutNs)) {
            ok = false;
            break;
          }
          uint8_t* sa = base + (size_t)stage * GStageBytes;
          const int k = (kb0 + kb) * GBK;
          mbar_arrive_expect_tx(&full[stage], GStageBytes);
          tma_load_2d(sa, &args.tmL, k, m * GBM, &full[stage]);
          tma_load_2d(sa + GABytes, &args.tmR, k, n * GBN, &full[stage]);
          float* slot = sc_ring + cs * (GScaleSlotBytes / 4);
          mbar_arrive_expect_tx(&scfull[cs], GScaleSlotBytes);
          tma_load_2d(slot, &args.tmSL, m * GBM, kb0 + kb, &scfull[cs]);
          tma_load_2d(slot + GBM, &args.tmSR, n * GBN, kb0 + kb, &scfull[cs]);
          issued |= 1u << stage;
          issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
          sc_issued |= 1u << cs;
          sc_parity = (sc_parity & ~(1u << cs)) | (cph << cs);
          if (++stage == GStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {  // the copies already issued complete on these barriers
        for (int s = 0; s < GStages; ++s)
          if ((issued >> s) & 1u)
            mbar_wait_bounded(&full[s], (issued_parity >> s) & 1u, args.status, GTimeoutNs / 8);
        for (int c = 0; c < GScaleSlots; ++c)
          if ((sc_issued >> c) & 1u)
            mbar_wait_bounded(&scfull[c], (sc_parity >> c) & 1u, args.status, GTimeoutNs / 8);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_f8_f32(GBM, GBN, kF8E5M2, kF8E4M3);
      int stage = 0;
      uint32_t phase = 0, slice = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < total && ok; u += gridDim.x) {
        int g, m, n, kb0, kcnt;
        decode(u, g, m, n, kb0, kcnt);
        for (int kb = 0; kb < kcnt; ++kb, ++slice) {
          const uint32_t sb = slice % kBufs, sph = (slice / kBufs) & 1u;
          if (!mbar_wait_bounded(&sempty[sb], sph ^ 1u, args.status, GTimeoutNs) ||
              !mbar_wait_bounded(&full[stage], phase, args.status, GTimeoutNs)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(base + (size_t)stage * GStageBytes);
          const uint32_t b0 = a0 + GABytes;
#pragma unroll
          for (int k = 0; k < GBK / 32; ++k)
            mma_e4m3(tmem_base + sb * GBN, smem_desc_sw128(a0 + k * 32),
                     smem_desc_sw128(b0 + k * 32), idesc, k != 0);
          mma_commit(&empty[stage]);
          mma_commit(&sfull[sb]);
          if (++stage == GStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      mma_commit(drain);
      mbar_wait_bounded(drain, 0, args.status, GTimeoutNs / 8);
    }
  } else {
    // warps 2..kEpiW+1: warp w reads TMEM lanes 32*(w%4)..+31; the kSub warps
    // of a quadrant own the kCols columns kCols*sub.. of the tile
    const int q = warp & 3;
    const int sub = (warp - 2) >> 2;
    const int row = q * 32 + lane;
    uint32_t slice = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < total && ok; u += gridDim.x) {
      int g, m, n, kb0, kcnt;
      decode(u, g, m, n, kb0, kcnt);
      float acc[kCols];
#pragma unroll
      for (int i = 0; i < kCols; ++i) acc[i] = 0.f;
      for (int kb = 0; kb < kcnt; ++kb, ++slice) {
        const uint32_t sb = slice % kBufs, sph = (slice / kBufs) & 1u;
        const uint32_t cs = slice % GScaleSlots, cph = (slice / GScaleSlots) & 1u;
        if (!mbar_wait_bounded(&scfull[cs], cph, args.status, GTimeoutNs) ||
            !mbar_wait_bounded(&sfull[sb], sph, args.status, GTimeoutNs)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const float* slot = sc_ring + cs * (GScaleSlotBytes / 4);
        const float s_row = slot[row];
        const float* s_col = slot + GBM + kCols * sub;
        const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + sb * GBN + kCols * sub;
#pragma unroll
        for (int c0 = 0; c0 < kLoads; c0 += kInFlight) {
          uint32_t p[kInFlight][16];
#pragma unroll
          for (int j = 0; j < kInFlight; ++j) tmem_ld16(taddr + 16 * (c0 + j), p[j]);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < kInFlight; ++j) {
            const int c = c0 + j;
            // pairs of columns: their two scale products by one packed multiply,
            // then one packed fused multiply-add (two round-to-nearest fp32 ops
            // each, the same results as the scalar fmul and fmaf)
#pragma unroll
            for (int i = 0; i < 16; i += 4) {
              const float4 sc = *reinterpret_cast<const float4*>(s_col + 16 * c + i);
              float m0, m1, m2, m3;
              fmul2_s(m0, m1, sc.x, sc.y, s_row);
              fmul2_s(m2, m3, sc.z, sc.w, s_row);
              ffma2_v(acc[16 * c + i], acc[16 * c + i + 1], __uint_as_float(p[j][i]),
                      __uint_as_float(p[j][i + 1]), m0, m1);
              ffma2_v(acc[16 * c + i + 2], acc[16 * c + i + 3], __uint_as_float(p[j][i + 2]),
                      __uint_as_float(p[j][i + 3]), m2, m3);
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&sempty[sb]);
          mbar_arrive(&scempty[cs]);
        }
      }
      if (!ok) break;
      // an expert without rows stores zeros
      if constexpr (C::kTmaStore) {
        // 64-column pieces: bf16 into this warp's swizzled staging buffer (the
        // 16-byte chunks of row `lane` XOR-permuted like the TMA's 128-byte
        // swizzle), then one TMA store of 32 rows x 64 columns
        uint8_t* stg = staging + (size_t)(warp - 2) * (32 * 128);
        const int grow = g * args.M_total + m * GBM + q * 32;
#pragma unroll
        for (int c = 0; c < kCols; c += 64) {
          if (lane == 0) bulk_wait_read_all();  // the previous piece has left the buffer
          __syncwarp();
          uint8_t* my_row = stg + lane * 128;
#pragma unroll
          for (int jj = 0; jj < 8; ++jj) {
            const float* a8 = acc + c + 8 * jj;
            *reinterpret_cast<uint4*>(my_row + ((jj ^ (lane & 7)) << 4)) =
                make_uint4(bf16x2_bits(a8[0], a8[1]), bf16x2_bits(a8[2], a8[3]),
                           bf16x2_bits(a8[4], a8[5]), bf16x2_bits(a8[6], a8[7]));
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_2d(&args.tmOut, stg, n * GBN + kCols * sub + c, grow);
            bulk_commit_group();
          }
        }
      } else {
        __nv_bfloat16* orow = args.out +
                              ((size_t)g * args.M_total + (size_t)m * GBM + row) * args.N_total +
                              (size_t)n * GBN + kCols * sub;
#pragma unroll
        for (int v = 0; v < kCols / 8; ++v) {
          uint4 w;
          __nv_bfloat162* hb = reinterpret_cast<__nv_bfloat162*>(&w);
#pragma unroll
          for (int i = 0; i < 4; ++i)
            hb[i] = __floats2bfloat162_rn(acc[8 * v + 2 * i], acc[8 * v + 2 * i + 1]);
          reinterpret_cast<uint4*>(orow)[v] = w;
        }
      }
    }
    if constexpr (C::kTmaStore) {
      if (lane == 0) bulk_wait_all();  // every store has completed before the CTA exits
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

template <int kBN, int kEpiW, int kInFlight>
cudaError_t launch_fp8_wgrad_w(const Fp8WgradArgs& a, cudaStream_t st) {
  auto kernel = fp8_wgrad_kernel<kBN, kEpiW, kInFlight>;
  constexpr size_t smem = WgTile<kBN>::kSmemBytes;
  cudaError_t e = note_cuda(cudaFuncSetAttribute(kernel,
                                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 (int)smem),
                            "fp8 weight-gradient GEMM: set shared-memory size");
  if (e != cudaSuccess) return e;
  kernel<<<num_sms(), wgrad_threads(kEpiW), smem, st>>>(a);
  return note_cuda(cudaGetLastError(), "fp8 weight-gradient GEMM launch");
}

// Gradient tile and epilogue shape, chosen once per process by
// MOE_FP8_WGRAD_EPI:
//   unset   128-column tiles, four slice buffers, eight epilogue warps with two
//           16-column loads in flight (64 running sums a thread; four in
//           flight measured the same and spills)
//   wide    256-column tiles, two slice buffers, eight warps, one load in flight
//           (128 running sums a thread)
//   narrow  256-column tiles, sixteen warps, one load in flight
int fp8_wgrad_kind() {
  static int v = -1;
  if (v < 0) {
    const char* e = std::getenv("MOE_FP8_WGRAD_EPI");
    v = 0;
    if (e != nullptr && std::strcmp(e, "wide") == 0) v = 1;
    if (e != nullptr && std::strcmp(e, "narrow") == 0) v = 2;
  }
  return v;
}
int fp8_wgrad_tile_cols() { return fp8_wgrad_kind() == 0 ? 128 : 256; }

cudaError_t launch_fp8_wgrad(const Fp8WgradArgs& a, cudaStream_t st) {
  switch (fp8_wgrad_kind()) {
    case 1: return launch_fp8_wgrad_w<256, 8, 1>(a, st);
    case 2: return launch_fp8_wgrad_w<256, 16, 1>(a, st);
    default: return launch_fp8_wgrad_w<128, 8, 2>(a, st);
  }
}

}  // namespace

// Columns of the FP8 transposed layouts: all rows plus up to 127 of padding
// per group (blocks padded to one 128-row scale tile).
long long wgrad_cols_fp8(const moe_shape& s) {
  const long long rows = (long long)s.T * s.K + s.T;
  return (rows + (long long)(s.N + 1) * 127 + 127) / 128 * 128;
}

int launch_ffn_bwd_dw_e4m3(const moe_shape& s, const int32_t* perm_tok, const int32_t* offsets,
                           const void* x, const void* dy_perm, const void* dy_shared, void* dw13,
                           void* dw2, void* ws_bwd, cudaStream_t st) {
  const BwdLayoutFp8 B = bwd_layout_fp8(s);
  uint8_t* w = static_cast<uint8_t*>(ws_bwd);
  uint32_t* status = reinterpret_cast<uint32_t*>(w);
  const __nv_bfloat16* GU = reinterpret_cast<const __nv_bfloat16*>(w + B.gu);
  const __nv_bfloat16* dGU = reinterpret_cast<const __nv_bfloat16*>(w + B.dgu);
  int32_t* colbase = reinterpret_cast<int32_t*>(w + B.colbase);
  auto bfp = [&](size_t off) { return reinterpret_cast<__nv_bfloat16*>(w + off); };
  auto f32 = [&](size_t off) { return reinterpret_cast<float*>(w + off); };
  const long long R = wgrad_cols_fp8(s);
  const int twof = 2 * s.f;
  // A: the layer input rows, gathered from x through perm_tok (E4M3 mode keeps
  // no bf16 copy of the dispatched rows)
  if (launch_group_transposes(s, GBK, x, perm_tok, x, dy_perm, dy_shared, GU, dGU, offsets,
                              colbase, R, bfp(B.at), bfp(B.dyt), bfp(B.ht), bfp(B.dgut),
                              st) != cudaSuccess)
    return MOE_ERR_CUDA;
  // each transposed operand [C, R] per 1x128 tile of its rows
  const long long ld_d = scale_ld(s.d), ld_f = scale_ld(s.f), ld_2f = scale_ld(twof);
  if (launch_quant_rows_e5m2(bfp(B.dyt), s.d, (int)R, w + B.dytq, f32(B.dyts), ld_d, st) !=
          cudaSuccess ||
      launch_quant_rows(bfp(B.ht), s.f, (int)R, w + B.htq, f32(B.hts), ld_f, st) !=
          cudaSuccess ||
      launch_quant_rows_e5m2(bfp(B.dgut), twof, (int)R, w + B.dgutq, f32(B.dguts), ld_2f, st) !=
          cudaSuccess ||
      launch_quant_rows(bfp(B.at), s.d, (int)R, w + B.atq, f32(B.ats), ld_d, st) != cudaSuccess)
    return MOE_ERR_CUDA;

  const auto U8 = CU_TENSOR_MAP_DATA_TYPE_UINT8;
  const uint64_t KT = (uint64_t)(R / GBK);
  const uint32_t GBN = (uint32_t)fp8_wgrad_tile_cols();
  // dW2_e [d, f] = dYT_e HT_e^T
  Fp8WgradArgs a2{};
  bool ok = make_map(&a2.tmL, w + B.dytq, U8, 1, R, s.d, GBK, GBM) &&
            make_map(&a2.tmR, w + B.htq, U8, 1, R, s.f, GBK, GBN) &&
            make_map_f32_rows(&a2.tmSL, f32(B.dyts), ld_d, KT, GBM) &&
            make_map_f32_rows(&a2.tmSR, f32(B.hts), ld_f, KT, GBN);
  // dW13_e [2f, d] = dGUT_e AT_e^T (rows in the packed W13 order)
  Fp8WgradArgs a13{};
  ok = ok && make_map(&a13.tmL, w + B.dgutq, U8, 1, R, twof, GBK, GBM) &&
       make_map(&a13.tmR, w + B.atq, U8, 1, R, s.d, GBK, GBN) &&
       make_map_f32_rows(&a13.tmSL, f32(B.dguts), ld_2f, KT, GBM) &&
       make_map_f32_rows(&a13.tmSR, f32(B.ats), ld_d, KT, GBN);
  const auto BF = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const uint64_t G1 = (uint64_t)s.N + 1;
  ok = ok && make_map(&a2.tmOut, dw2, BF, 2, s.f, G1 * s.d, 64, 32) &&
       make_map(&a13.tmOut, dw13, BF, 2, s.d, G1 * twof, 64, 32);
  if (!ok) {
    note_text("fp8 weight-gradient GEMM: tensor-map encoding failed");
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
  if (launch_fp8_wgrad(a2, st) != cudaSuccess || launch_fp8_wgrad(a13, st) != cudaSuccess)
    return MOE_ERR_CUDA;
  return MOE_OK;
}

}  // namespace moe
