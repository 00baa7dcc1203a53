// bf16 expert GEMMs with two token tiles per weight tile.
//
// Same computation as the grouped kernel in gemm_tc.cu (the SwiGLU expert FFN
// of the mhpq.cn article §1.1: GEMM1 [rows_g, d] x [d, 2f] with the SwiGLU
// epilogue, GEMM2 [rows_g, f] x [f, d]; group N is the shared expert on all T
// rows).  A work unit is one 256-column weight tile of a group and up to two
// consecutive 128-row token tiles of it: per 64-wide K stage the producer
// loads the weight tile once (32 KB) and both token tiles (16 KB each), and
// the MMA thread issues the four K=16 steps of the first tile's accumulator,
// then the four of the second's (tcgen05.mma cta_group::1, M=128 -- M=64 for
// a token tile of at most 64 rows -- N=256).  Operand bytes per MMA cycle
// drop from 96 to 64 against one token tile per weight tile, and issuing
// each accumulator's K steps back to back keeps the tensor pipe at its full
// rate (the issue-rate probe, csrc/probe/mma_rate.cu: 128 cycles per N=256
// MMA this way, 149.5 when the two accumulators alternate every K step).  An expert with an odd number of token tiles ends
// with a one-tile unit, so a ragged tail costs one tile's MMA work, as in the
// one-tile kernel.
//
// Schedule: units are handed out in order (group, weight tile, token tiles)
// from a counter in the workspace; a unit of two tiles costs twice one of a
// single tile, so a static round-robin split left some SMs ~13% more work on
// the routed loads.  The producer takes the next unit while the current one
// streams and passes each unit index to the MMA thread and the epilogue warps
// through a shared-memory ring; the last CTA to finish puts the counter back
// to zero for the next launch.
// TMEM: two 256-column accumulator slots.  A two-tile unit takes both, a
// one-tile unit the next free one; the slots are taken in turn, and each has
// its own full/empty barriers and use count, so a unit's MMAs start as soon
// as the slots they write have been drained.
// Roles: warp 0 TMA producer (3-stage ring of 64 KB), warp 1 TMEM owner and
// MMA issuer, warps 2-5 drain slot 0 and warps 6-9 slot 1 (one TMEM lane
// quadrant each), apply SwiGLU (GEMM1: the 128-row W1/W3 interleave of the
// packed W13 puts a feature's gate and up columns in the same accumulator)
// and store bf16 rows.  Every mbarrier wait is bounded (~2 s) and sets the
// device status word when it gives up.
#include <cuda.h>
#include <cuda_bf16.h>

#include "epilogue.cuh"
#include "internal.h"
#include "ptx.cuh"

namespace moe {
namespace {

constexpr int DBM = 128, DBN = 256, DBK = 64;
constexpr int DStages = 3;
constexpr int DABytes = DBM * DBK * 2;                   // 16 KB per token tile
constexpr int DBBytes = DBN * DBK * 2;                   // 32 KB weight tile
constexpr int DStageBytes = 2 * DABytes + DBBytes;       // 64 KB
constexpr int DThreads = 320;                            // warps 0, 1, then 2 x 4 epilogue
constexpr int DUnitRing = 8;                             // unit indices in flight
constexpr uint64_t DTimeoutNs = 2000000000ull;

enum DEpi { kDSwiGLU = 0, kDStore = 1 };

struct alignas(64) DualArgs {
  CUtensorMap tmA_routed;
  CUtensorMap tmA_shared;
  CUtensorMap tmB;
  const int32_t* offsets;
  __nv_bfloat16* out_routed;
  __nv_bfloat16* out_shared;
  uint32_t* status;
  uint32_t* sched;    // [0] next unit, [1] CTAs finished (both zero between launches)
  int N, T;
  int rows_routed;    // T*K
  int a_shared_row0;  // first row of the shared expert's rows in its A tensor
  int n_acc;          // weight rows per group (2f for GEMM1, d for GEMM2)
  int k_dim;
  int out_ld;
};

constexpr size_t dual_smem_bytes(int groups) {
  return 1024 + (size_t)DStages * DStageBytes + 512 + (size_t)(groups + 1) * 4;
}

template <int kEpi>
__global__ void __launch_bounds__(DThreads, 1) dual_gemm_bf16_kernel(
    const __grid_constant__ DualArgs args) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + (size_t)DStages * DStageBytes);
  uint64_t* full = bars;                   // [DStages]
  uint64_t* empty = full + DStages;        // [DStages]
  uint64_t* tfull = empty + DStages;       // [2] slot accumulated
  uint64_t* tempty = tfull + 2;            // [2] slot drained (4 warps)
  uint64_t* drain = tempty + 2;            // [1]
  uint64_t* urfull = drain + 1;            // [DUnitRing] unit index written
  uint64_t* urempty = urfull + DUnitRing;  // [DUnitRing] read by the MMA thread + 8 warps
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(urempty + DUnitRing);
  int* uring = reinterpret_cast<int*>(tmem_holder + 1);  // [DUnitRing]
  int* unit_start = reinterpret_cast<int*>(base + (size_t)DStages * DStageBytes + 512);

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int G1 = args.N + 1;
  const int NT = args.n_acc / DBN;
  const int KB = args.k_dim / DBK;

  if (tid == 0) {
    for (int s = 0; s < DStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 4);
    }
    mbar_init(drain, 1);
    for (int i = 0; i < DUnitRing; ++i) {
      mbar_init(&urfull[i], 1);
      mbar_init(&urempty[i], 9);
    }
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, 512);
    tmem_relinquish();
  }
  auto group_rows = [&](int g) {
    return (g < args.N) ? args.offsets[g + 1] - args.offsets[g] : args.T;
  };
  for (int g = tid; g < G1; g += DThreads) {
    const int rows = group_rows(g);
    const int mt = rows > 0 ? (rows + DBM - 1) / DBM : 0;
    unit_start[g] = (mt + 1) / 2;  // units per weight tile
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) {  // exclusive scan of units per group, times NT
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
      unit_start[g] = run * NT;
      run += c;
    }
    if (lane == 31) unit_start[G1] = inc * NT;
  }
  __syncthreads();
  const uint32_t tmem_base = *tmem_holder;
  const int total = unit_start[G1];

  // unit -> group g, weight tile n, first token tile m0 (= 2 j), tiles in it (1 or 2)
  auto decode = [&](int u, int& g, int& n, int& m0, int& ntiles) {
    int lo = 0, hi = G1;
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (unit_start[mid] <= u) lo = mid; else hi = mid;
    }
    g = lo;
    const int per_n = (unit_start[g + 1] - unit_start[g]) / NT;
    const int local = u - unit_start[g];
    n = local / per_n;
    const int j = local - n * per_n;
    const int rows = group_rows(g);
    const int mt = (rows + DBM - 1) / DBM;
    m0 = 2 * j;
    ntiles = min(2, mt - m0);
  };

  // the next unit index from the ring (every consumer warp reads every entry;
  // lane 0 releases it); a value >= total ends the loop
  auto next_unit = [&](uint32_t& seq, int& u) -> bool {
    const uint32_t slot = seq % DUnitRing, ph = (seq / DUnitRing) & 1u;
    if (!mbar_wait_bounded(&urfull[slot], ph, args.status, DTimeoutNs)) return false;
    u = *reinterpret_cast<volatile int*>(&uring[slot]);
    __syncwarp(__activemask());
    if (lane == 0) mbar_arrive(&urempty[slot]);
    ++seq;
    return true;
  };

  if (warp == 0) {
    // ---- TMA producer ---------------------------------------------------------
    if (lane == 0) {
      tma_prefetch_desc(&args.tmA_routed);
      tma_prefetch_desc(&args.tmA_shared);
      tma_prefetch_desc(&args.tmB);
      int stage = 0;
      uint32_t phase = 0, issued = 0, issued_parity = 0;
      uint32_t useq = 0;
      bool ok = true;
      int u_next = (int)atomicAdd(&args.sched[0], 1u);
      for (;;) {
        // after a failed wait the consumers get the end marker (total) at once
        const int u = ok ? u_next : total;
        // publish the unit to the MMA thread and the epilogue warps
        const uint32_t rs = useq % DUnitRing, rph = (useq / DUnitRing) & 1u;
        if (!mbar_wait_bounded(&urempty[rs], rph ^ 1u, args.status, DTimeoutNs)) break;
        uring[rs] = u;
        mbar_arrive(&urfull[rs]);
        ++useq;
        if (u >= total) break;
        u_next = (int)atomicAdd(&args.sched[0], 1u);  // lands while this unit streams
        int g, n, m0, nt;
        decode(u, g, n, m0, nt);
        const CUtensorMap* am = (g < args.N) ? &args.tmA_routed : &args.tmA_shared;
        const int arow = ((g < args.N) ? args.offsets[g] : args.a_shared_row0) + m0 * DBM;
        const int brow = g * args.n_acc + n * DBN;
        const uint32_t bytes = (uint32_t)(DBBytes + nt * DABytes);
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait_bounded(&empty[stage], phase ^ 1u, args.status, DTimeoutNs)) {
            ok = false;
            break;
          }
          uint8_t* st = base + (size_t)stage * DStageBytes;
          mbar_arrive_expect_tx(&full[stage], bytes);
          tma_load_2d(st, &args.tmB, kb * DBK, brow, &full[stage]);
          tma_load_2d(st + DBBytes, am, kb * DBK, arow, &full[stage]);
          if (nt > 1) tma_load_2d(st + DBBytes + DABytes, am, kb * DBK, arow + DBM, &full[stage]);
          issued |= 1u << stage;
          issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == DStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {  // let the copies already issued land before the CTA exits
        for (int s = 0; s < DStages; ++s)
          if ((issued >> s) & 1u)
            mbar_wait_bounded(&full[s], (issued_parity >> s) & 1u, args.status, DTimeoutNs / 8);
      }
    }
  } else if (warp == 1) {
    // ---- MMA issuer -------------------------------------------------------------
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t uses = 0;  // bit s: parity of the next use of accumulator slot s
      int p = 0;          // slot the next unit starts in
      uint32_t useq = 0;
      bool ok = true;
      for (;;) {
        int u;
        if (!next_unit(useq, u) || u >= total) break;
        int g, n, m0, nt;
        decode(u, g, n, m0, nt);
        const int rows_g = group_rows(g);
        const int slot[2] = {p, p ^ 1};
        for (int t = 0; t < nt && ok; ++t)
          ok = mbar_wait_bounded(&tempty[slot[t]], ((uses >> slot[t]) & 1u) ^ 1u, args.status,
                                 DTimeoutNs);
        if (!ok) break;
        tc_fence_after();
        // a token tile with at most 64 rows (an expert's ragged tail) runs M=64
        uint32_t idesc[2];
        for (int t = 0; t < 2; ++t)
          idesc[t] = idesc_bf16_f32(rows_g - (m0 + t) * DBM <= 64 ? 64 : DBM, DBN);
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait_bounded(&full[stage], phase, args.status, DTimeoutNs)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t b0 = smem_u32(base + (size_t)stage * DStageBytes);
          const uint32_t a0 = b0 + DBBytes;
          // each accumulator's four K steps back to back
          for (int t = 0; t < nt; ++t) {
            const uint32_t d_tmem = tmem_base + (uint32_t)(slot[t] * DBN);
#pragma unroll
            for (int k = 0; k < DBK / 16; ++k)
              mma_bf16(d_tmem, smem_desc_sw128(a0 + t * DABytes + k * 32),
                       smem_desc_sw128(b0 + k * 32), idesc[t], (kb | k) != 0);
          }
          mma_commit(&empty[stage]);
          if (++stage == DStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        for (int t = 0; t < nt; ++t) {
          mma_commit(&tfull[slot[t]]);
          uses ^= 1u << slot[t];
        }
        p = (p + nt) & 1;
      }
      mma_commit(drain);
      mbar_wait_bounded(drain, 0, args.status, DTimeoutNs / 8);
    }
  } else {
    // ---- epilogue: warps 2-5 drain slot 0, warps 6-9 slot 1 -----------------------
    const int sg = (warp - 2) >> 2;  // accumulator slot of this warp group
    const int q = warp & 3;          // TMEM lane quadrant this warp may access
    const int row = q * 32 + lane;
    const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(sg * DBN);
    uint32_t uses = 0;
    int p = 0;
    uint32_t useq = 0;
    for (;;) {
      int u;
      if (!next_unit(useq, u) || u >= total) break;
      int g, n, m0, nt;
      decode(u, g, n, m0, nt);
      const int first = p;
      p = (p + nt) & 1;
      int t;  // which of the unit's token tiles sits in this warp's slot
      if (first == sg) t = 0;
      else if (nt == 2) t = 1;
      else continue;
      if (!mbar_wait_bounded(&tfull[sg], uses & 1u, args.status, DTimeoutNs)) break;
      ++uses;
      tc_fence_after();
      const int m = m0 + t;
      const int rows_g = group_rows(g);
      // M=64 tiles (<= 64 rows) hold row 16*q + i in TMEM lane 32*q + i (i < 16)
      const bool m64 = rows_g - m * DBM <= 64;
      const int r = m * DBM + (m64 ? (lane < 16 ? 16 * q + lane : DBM) : row);
      // rows past the group's end belong to the next group (or are padding);
      // the second test keeps a corrupted offsets[] from writing out of range
      const bool valid = r < rows_g && (g == args.N || args.offsets[g] + r < args.rows_routed);
      __nv_bfloat16* orow =
          (g < args.N) ? args.out_routed + (size_t)(args.offsets[g] + r) * args.out_ld
                       : args.out_shared + (size_t)r * args.out_ld;
      if constexpr (kEpi == kDSwiGLU) {
#pragma unroll 1
        for (int c = 0; c < DBN / 2; c += 32) {
          uint32_t ga[32], up[32];
          tmem_ld32(taddr + c, ga);
          tmem_ld32(taddr + DBN / 2 + c, up);
          tmem_wait_ld();
          float h[32];
#pragma unroll
          for (int i = 0; i < 32; ++i)
            h[i] = silu_fast(__uint_as_float(ga[i])) * __uint_as_float(up[i]);
          if (valid) store_row32(orow + n * (DBN / 2) + c, h);
        }
      } else {
#pragma unroll 1
        for (int c = 0; c < DBN; c += 32) {
          uint32_t v[32];
          tmem_ld32(taddr + c, v);
          tmem_wait_ld();
          float y[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) y[i] = __uint_as_float(v[i]);
          if (valid) store_row32(orow + n * DBN + c, y);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[sg]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
  // the last CTA to finish (every unit has been taken) resets the counter
  if (tid == 0) {
    __threadfence();
    if (atomicAdd(&args.sched[1], 1u) == gridDim.x - 1) {
      atomicExch(&args.sched[0], 0u);
      atomicExch(&args.sched[1], 0u);
    }
  }
}

template <int kEpi>
cudaError_t launch_dual(const DualArgs& a, cudaStream_t st) {
  const size_t smem = dual_smem_bytes(a.N + 1);
  cudaError_t e = note_cuda(cudaFuncSetAttribute(dual_gemm_bf16_kernel<kEpi>,
                                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 (int)smem),
                            "expert GEMM: set shared-memory size");
  if (e != cudaSuccess) return e;
  dual_gemm_bf16_kernel<kEpi><<<num_sms(), DThreads, smem, st>>>(a);
  return note_cuda(cudaGetLastError(), "expert GEMM launch");
}

}  // namespace

int launch_ffn_tc_bf16_dual(const moe_shape& s, const void* x_perm, const int32_t* offsets,
                            const void* x, const void* w13, const void* w2, void* y_perm,
                            void* y_shared, void* ws, cudaStream_t st) {
  const WsLayout L = ws_layout(s);
  uint8_t* w = static_cast<uint8_t*>(ws);
  __nv_bfloat16* H = reinterpret_cast<__nv_bfloat16*>(w + L.h);
  const uint64_t TK = (uint64_t)s.T * s.K;
  const auto BF = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  uint32_t* status = reinterpret_cast<uint32_t*>(w + L.status);

  DualArgs g1{};
  bool ok = make_map(&g1.tmA_routed, x_perm, BF, 2, s.d, TK, DBK, DBM) &&
            make_map(&g1.tmA_shared, x, BF, 2, s.d, s.T, DBK, DBM) &&
            make_map(&g1.tmB, w13, BF, 2, s.d, (uint64_t)(s.N + 1) * 2 * s.f, DBK, DBN);
  if (!ok) {
    note_text("expert GEMM1: tensor-map encoding failed");
    return MOE_ERR_CUDA;
  }
  g1.offsets = offsets;
  g1.out_routed = H;
  g1.out_shared = H + TK * s.f;
  g1.status = status;
  g1.sched = status + 16;  // counters in the zero-initialised head of the workspace
  g1.N = s.N;
  g1.T = s.T;
  g1.rows_routed = (int)TK;
  g1.a_shared_row0 = 0;
  g1.n_acc = 2 * s.f;
  g1.k_dim = s.d;
  g1.out_ld = s.f;
  if (launch_dual<kDSwiGLU>(g1, st) != cudaSuccess) return MOE_ERR_CUDA;

  DualArgs g2{};
  ok = make_map(&g2.tmA_routed, H, BF, 2, s.f, TK + s.T, DBK, DBM) &&
       make_map(&g2.tmA_shared, H, BF, 2, s.f, TK + s.T, DBK, DBM) &&
       make_map(&g2.tmB, w2, BF, 2, s.f, (uint64_t)(s.N + 1) * s.d, DBK, DBN);
  if (!ok) {
    note_text("expert GEMM2: tensor-map encoding failed");
    return MOE_ERR_CUDA;
  }
  g2.offsets = offsets;
  g2.out_routed = static_cast<__nv_bfloat16*>(y_perm);
  g2.out_shared = static_cast<__nv_bfloat16*>(y_shared);
  g2.status = status;
  g2.sched = status + 18;
  g2.N = s.N;
  g2.T = s.T;
  g2.rows_routed = (int)TK;
  g2.a_shared_row0 = (int)TK;
  g2.n_acc = s.d;
  g2.k_dim = s.f;
  g2.out_ld = s.d;
  if (launch_dual<kDStore>(g2, st) != cudaSuccess) return MOE_ERR_CUDA;
  return MOE_OK;
}

}  // namespace moe
