// Whole-block copy: the copy-on-write copy inside one pool and the swap
// between a device pool and a pinned host pool ("4. vLLM核心机制" sections
// 4.2 and 4.4).  Pure data movement, bound by HBM (inside the device) or by
// the host link (swap).
#pragma once

#include <cstdint>

#include "pa_kernels.cuh"

namespace pa {

struct CopyArgs {
  const uint4 *src_k;
  const uint4 *src_v;
  uint4 *dst_k;
  uint4 *dst_v;
  const int64_t *mapping;  // [num_pairs][2] (source block, destination block)
  long long num_pairs, chunks_per_block, src_blocks, dst_blocks;
};

// Work is cut into warp tiles of COPY_UNROLL * 32 16-byte chunks of one
// block of one cache.  Load u of lane l moves chunk u * 32 + l of the tile,
// so each warp instruction covers 512 contiguous bytes: whole 128-byte lines
// for HBM and full-size requests on the host link, where partial lines cost
// a request each.  All loads of a tile are issued before its stores.
// A pair with a negative entry is skipped; one outside its pool is skipped
// and flagged.  Either pool may be pinned host memory (unified addressing).
constexpr int COPY_UNROLL = 4;
constexpr int COPY_TILE = COPY_UNROLL * 32;  // chunks; every supported block is a multiple of it

__global__ void __launch_bounds__(256) copy_blocks_kernel(const CopyArgs a) {
  grid_dependency_wait();
  grid_launch_dependents();
  const int lane = threadIdx.x & 31;
  const long long tiles_per_block = (a.chunks_per_block + COPY_TILE - 1) / COPY_TILE;
  const long long total = a.num_pairs * 2 * tiles_per_block;
  const long long warps = (long long)gridDim.x * (blockDim.x >> 5);
  for (long long w = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5; w < total; w += warps) {
    const long long pair = w / (2 * tiles_per_block);
    const long long rem = w - pair * 2 * tiles_per_block;
    const bool is_v = rem >= tiles_per_block;
    const long long tile = is_v ? rem - tiles_per_block : rem;
    const long long src = a.mapping[2 * pair], dst = a.mapping[2 * pair + 1];  // may be host memory
    if (src < 0 || dst < 0) continue;
    if (src >= a.src_blocks || dst >= a.dst_blocks) {
      if (tile == 0 && !is_v && lane == 0) atomicOr(&g_status, PA_DEV_ERR_BLOCK_ID);
      continue;
    }
    const long long base = tile * COPY_TILE + lane;
    const uint4 *from = (is_v ? a.src_v : a.src_k) + src * a.chunks_per_block;
    uint4 *to = (is_v ? a.dst_v : a.dst_k) + dst * a.chunks_per_block;
    uint4 v[COPY_UNROLL];
#pragma unroll
    for (int u = 0; u < COPY_UNROLL; ++u)
      if (base + u * 32 < a.chunks_per_block) v[u] = from[base + u * 32];
#pragma unroll
    for (int u = 0; u < COPY_UNROLL; ++u)
      if (base + u * 32 < a.chunks_per_block) to[base + u * 32] = v[u];
  }
}

}  // namespace pa
