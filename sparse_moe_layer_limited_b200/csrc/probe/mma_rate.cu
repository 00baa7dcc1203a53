// Issue-rate probes for the tensor-core path.
// (1) tcgen05.mma: SM cycles per MMA instruction with both
// operands resident in shared memory (no loads, no epilogue), for the
// instruction shapes the expert GEMMs use.  One thread issues `iters` K steps;
// each K step issues `chains` MMAs into separate accumulators (chains = 1 is a
// dependent accumulation chain, as in a GEMM main loop).  With `blocked`, a
// 64-wide K stage issues its four K steps on one accumulator before the next
// (the order a kernel sharing one weight tile between two token tiles uses);
// otherwise the accumulators alternate every K step.  Operand values are
// zero: only the timing is of interest.
// (2) tcgen05.ld: cycles per round of `inflight` loads of 32 lanes x W columns
// followed by one tcgen05.wait::ld, per warp, with 4 or 16 warps per CTA; gives
// the load latency (inflight = 1) and the TMEM read bandwidth per SM.
// Prints one JSON line per configuration.
// Build: nvcc -O3 -std=c++17 -gencode arch=compute_100a,code=sm_100a mma_rate.cu
#include <cstdint>
#include <cstdio>
#include <cuda.h>
#include <cuda_runtime.h>

#include "../ptx.cuh"

using namespace moe;

__device__ unsigned long long g_cycles;
__device__ uint32_t g_err;

template <bool kFp8, bool kPair>
__global__ void __launch_bounds__(128, 1) mma_rate_kernel(int M, int N, int chains, int iters,
                                                          int blocked) {
  extern __shared__ uint8_t sm_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(sm_raw) + 1023) &
                                             ~uintptr_t(1023));
  __shared__ uint64_t bar;
  __shared__ uint32_t holder;
  const int warp = threadIdx.x >> 5;
  const uint32_t rank = kPair ? cluster_ctarank() : 0u;
  for (int i = threadIdx.x; i < 48 * 1024 / 4; i += blockDim.x)
    reinterpret_cast<uint32_t*>(base)[i] = 0u;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
  }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  if (warp == 0) {
    if (kPair) {
      tmem_alloc_2sm(&holder, 512);
      tmem_relinquish_2sm();
    } else {
      tmem_alloc(&holder, 512);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  __syncthreads();
  if (kPair) cluster_sync_all();
  tc_fence_after();
  const uint32_t tb = holder;
  if (threadIdx.x == 0 && rank == 0) {
    // A at +0 (up to 128 rows of 128 B), B at +16 KB (up to 256 rows)
    const uint32_t a0 = smem_u32(base), b0 = a0 + 16384;
    const uint32_t id = kFp8 ? idesc_e4m3_f32(M, N) : idesc_bf16_f32(M, N);
    const unsigned long long t0 = clock64();
    // the issuing thread must stay far below one MMA's duration per
    // instruction: plain loop nests, no division by a runtime value
    auto issue = [&](int k, int c, uint32_t acc) {
      const uint64_t ad = smem_desc_sw128(a0 + 32 * k), bd = smem_desc_sw128(b0 + 32 * k);
      // disjoint accumulators: chain c at column c * max(N, 128)
      const uint32_t d = tb + (uint32_t)(c * (N > 128 ? N : 128));
      if (kPair) {
        mma_bf16_2sm(d, ad, bd, id, acc);
      } else if (kFp8) {
        mma_e4m3(d, ad, bd, id, acc);
      } else {
        mma_bf16(d, ad, bd, id, acc);
      }
    };
    for (int it = 0; it < iters; ++it) {
      if (blocked) {
        for (int c = 0; c < chains; ++c)
#pragma unroll
          for (int k = 0; k < 4; ++k) issue(k, c, (it | k) != 0);
      } else {
#pragma unroll
        for (int k = 0; k < 4; ++k)
          for (int c = 0; c < chains; ++c) issue(k, c, (it | k) != 0);
      }
    }
    if (kPair) mma_commit_2sm(&bar); else mma_commit(&bar);
    mbar_wait_bounded(&bar, 0, &g_err, 2000000000ull);
    g_cycles = clock64() - t0;
  }
  tc_fence_before();
  __syncthreads();
  if (kPair) cluster_sync_all();
  if (warp == 0) {
    tc_fence_after();
    if (kPair) tmem_dealloc_2sm(tb, 512); else tmem_dealloc(tb, 512);
  }
}

template <int W>
__device__ __forceinline__ void ld_cols(uint32_t taddr, uint32_t (&r)[W]) {
  if constexpr (W == 16) {
    tmem_ld16(taddr, r);
  } else {
#pragma unroll
    for (int h = 0; h < W / 32; ++h) {
      uint32_t (&part)[32] = *reinterpret_cast<uint32_t (*)[32]>(&r[32 * h]);
      tmem_ld32(taddr + 32 * h, part);
    }
  }
}

__device__ float g_sink;

template <int W, int kInflight>
__global__ void __launch_bounds__(512, 1) tmem_ld_kernel(int iters) {
  __shared__ uint32_t holder;
  const int warp = threadIdx.x >> 5;
  if (warp == 0) {
    tmem_alloc(&holder, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tb = holder + ((uint32_t)((warp & 3) * 32) << 16);
  float acc = 0.f;
  const unsigned long long t0 = clock64();
  for (int it = 0; it < iters; ++it) {
    uint32_t v[kInflight][W];
#pragma unroll
    for (int j = 0; j < kInflight; ++j) ld_cols<W>(tb + (uint32_t)(((it + j) * W) & 511), v[j]);
    tmem_wait_ld();
#pragma unroll
    for (int j = 0; j < kInflight; ++j) acc += __uint_as_float(v[j][0] ^ v[j][W - 1]);
  }
  const unsigned long long cyc = clock64() - t0;
  if ((threadIdx.x & 31) == 0 && warp == 0) g_cycles = cyc;
  if (acc == 12345.f) g_sink = acc;
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(holder, 512);
  }
}

template <int W, int kInflight>
static int run_ld(int warps) {
  const int iters = 4000;
  tmem_ld_kernel<W, kInflight><<<1, 32 * warps>>>(iters);
  if (cudaDeviceSynchronize() != cudaSuccess) return 1;
  unsigned long long cyc = 0;
  cudaMemcpyFromSymbol(&cyc, g_cycles, sizeof(cyc));
  const double per = (double)cyc / iters;
  const double bytes = (double)warps * kInflight * W * 32 * 4;
  printf("{\"kind\": \"tmem_ld\", \"warps\": %d, \"cols\": %d, \"inflight\": %d, "
         "\"cycles_per_round\": %.1f, \"bytes_per_sm_cycle\": %.0f}\n",
         warps, W, kInflight, per, bytes / per);
  return 0;
}

template <bool kFp8, bool kPair>
static int run(int M, int N, int chains, int blocked = 0, bool print = true) {
  const int iters = 2000;
  const size_t smem = 50 * 1024;
  auto kern = mma_rate_kernel<kFp8, kPair>;
  cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(kPair ? 2 : 1);
  cfg.blockDim = dim3(128);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = kPair ? 2 : 1;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kern, M, N, chains, iters, blocked) != cudaSuccess) return 1;
  if (cudaDeviceSynchronize() != cudaSuccess) return 1;
  unsigned long long cyc = 0;
  uint32_t err = 0;
  cudaMemcpyFromSymbol(&cyc, g_cycles, sizeof(cyc));
  cudaMemcpyFromSymbol(&err, g_err, sizeof(err));
  const double per_step = (double)cyc / (iters * 4.0);
  // MACs per SM and K step: M rows (M/2 per SM for a pair) x N x K
  const double k = kFp8 ? 32.0 : 16.0;
  const double macs = (kPair ? M / 2 : M) * (double)N * k * chains;
  if (print)
    printf("{\"kind\": \"%s\", \"cta_group\": %d, \"M\": %d, \"N\": %d, \"chains\": %d, "
         "\"blocked\": %d, \"cycles_per_mma\": %.1f, \"macs_per_sm_cycle\": %.0f, "
         "\"status\": %u}\n",
         kFp8 ? "f8f6f4" : "f16", kPair ? 2 : 1, M, N, chains, blocked, per_step / chains,
         macs / per_step, err);
  return err != 0;
}

int main() {
  int bad = 0;
  // the tensor pipe of an idle GPU runs slower for a while after it wakes:
  // keep it busy for about a second before measuring anything
  for (int i = 0; i < 200; ++i) bad |= run<false, false>(128, 256, 1, 0, false);
  for (int N : {256, 128, 64, 16})
    for (int c : {1, 2, 3}) {
      if (N > 128 && c > 2) continue;  // accumulators must fit in 512 columns
      bad |= run<false, false>(128, N, c);
      bad |= run<false, false>(64, N, c);
      bad |= run<true, false>(128, N, c);
      bad |= run<false, true>(256, N, c);
    }
  bad |= run<false, false>(128, 256, 2, 1);
  bad |= run<true, false>(128, 256, 2, 1);
  bad |= run<false, true>(256, 256, 2, 1);
  bad |= run<false, false>(128, 128, 3, 1);
  for (int w : {4, 16}) {
    bad |= run_ld<16, 1>(w);
    bad |= run_ld<16, 2>(w);
    bad |= run_ld<16, 4>(w);
    bad |= run_ld<32, 1>(w);
    bad |= run_ld<32, 2>(w);
    bad |= run_ld<64, 1>(w);
  }
  return bad;
}
