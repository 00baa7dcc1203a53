// Row gather for expert parallelism.
//
// With the experts split over GPUs (the mhpq.cn article §2.1: each GPU holds
// a contiguous share of the routed experts; §3.1: tokens reach the experts
// of other GPUs by all-to-all), the rows a GPU receives arrive grouped by
// source GPU, then by expert.  The grouped expert GEMM wants them grouped by
// expert, and the results must go back in arrival order.  Both reorderings
// are one gather, dst[i] = src[idx[i]], with the index table built on the
// host from the exchanged per-expert counts.
//
// One warp per destination row, 16-byte vectors; a row whose index falls
// outside the source is written as zeros.
#include <cuda_runtime.h>

#include <cstdint>

#include "internal.h"

namespace moe {
namespace {

__global__ void __launch_bounds__(256) gather_rows_kernel(const uint4* __restrict__ src,
                                                          long long src_rows,
                                                          const int32_t* __restrict__ idx,
                                                          long long n, int vec_per_row,
                                                          uint4* __restrict__ dst) {
  const long long warps = ((long long)gridDim.x * blockDim.x) >> 5;
  const int lane = threadIdx.x & 31;
  for (long long r = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5; r < n; r += warps) {
    const long long s = idx[r];
    const bool ok = s >= 0 && s < src_rows;
    const uint4* from = src + (ok ? s : 0) * vec_per_row;
    uint4* to = dst + r * vec_per_row;
    for (int v = lane; v < vec_per_row; v += 32)
      to[v] = ok ? __ldg(from + v) : make_uint4(0u, 0u, 0u, 0u);
  }
}

}  // namespace
}  // namespace moe

extern "C" int moe_gather_rows(const void* src, int64_t src_rows, const int32_t* idx, int64_t n,
                               int row_bytes, void* dst, void* stream) {
  using namespace moe;
  auto ok16 = [](const void* p) {
    return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 15u) == 0;
  };
  if (n < 0 || src_rows < 0 || row_bytes <= 0 || row_bytes % 16 != 0) return MOE_ERR_ARG;
  if (n == 0) return MOE_OK;
  if (!ok16(src) || !ok16(dst) || idx == nullptr) return MOE_ERR_ARG;
  const long long warps_needed = n;
  long long blocks = (warps_needed * 32 + 255) / 256;
  const long long cap = (long long)num_sms() * 8;
  if (blocks > cap) blocks = cap;
  gather_rows_kernel<<<(unsigned)blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint4*>(src), src_rows, idx, n, row_bytes / 16,
      static_cast<uint4*>(dst));
  return note_cuda(cudaGetLastError(), "row gather launch") == cudaSuccess ? MOE_OK
                                                                           : MOE_ERR_CUDA;
}
