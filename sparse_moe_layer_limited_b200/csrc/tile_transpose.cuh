// 64 x 64 bf16 tile transposes through shared memory, 16-byte vectors on both
// sides of HBM.
//
// A tile is 64 source rows (the destination's columns) by 64 features (the
// destination's rows).  256 threads, two items per thread per phase:
//   load phase:  item (i, p) reads source row i, features 8p .. 8p+7
//                (8 lanes per 128-byte source segment, 4 rows per warp);
//   store phase: item (c, q) writes destination row c, columns 8q .. 8q+7
//                (8 lanes per 128-byte destination segment, 4 rows per warp).
// In shared memory feature c's 64 values are one 128-byte line whose 16-byte
// chunk q sits at chunk q ^ ((c ^ (c >> 3)) & 7).  In the load phase the 8
// lanes of one source row hold features whose c >> 3 differ, so their 2-byte
// stores land in 8 different chunks (16 banks, two lanes per word); in the
// store phase the 8 lanes of one destination row read the 8 chunks of one line.
#pragma once
#include <cuda_bf16.h>
#include <cstdint>

namespace moe {

constexpr int kTile = 64;
constexpr int kTileThreads = 256;
constexpr int kTileBytes = kTile * kTile * 2;

__host__ __device__ __forceinline__ uint32_t tile_chunk(int c, int q) {
  return (uint32_t)c * 128u + ((uint32_t)((q ^ c ^ (c >> 3)) & 7) << 4);
}

// Source row i of the tile, features 8p .. 8p+7, into the shared tile.
__device__ __forceinline__ void tile_put(uint8_t* sm, int i, int p, const uint4& v) {
  const uint16_t* h = reinterpret_cast<const uint16_t*>(&v);
#pragma unroll
  for (int e = 0; e < 8; ++e)
    *reinterpret_cast<uint16_t*>(sm + tile_chunk(p * 8 + e, i >> 3) + (i & 7) * 2) = h[e];
}

// Destination row c of the tile, columns 8q .. 8q+7.
__device__ __forceinline__ uint4 tile_get(const uint8_t* sm, int c, int q) {
  return *reinterpret_cast<const uint4*>(sm + tile_chunk(c, q));
}

}  // namespace moe
