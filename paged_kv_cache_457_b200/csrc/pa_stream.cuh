// Read-only streaming probe: the rate at which this GPU's SMs can pull bytes
// out of HBM when they only read.  The decode path is such a stream (K/V
// tiles in, a few hundred kilobytes out), so this rate, measured in the same
// process as the decode kernels, is the tightest of the roofline's
// denominators; a copy (read + write) peak is the looser one.
#pragma once

#include <cstdint>

#include "pa_kernels.cuh"

namespace pa {

// 16-byte load that bypasses L1 (the data is used once).
__device__ __forceinline__ uint4 ld_stream16(const uint4 *p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

constexpr int STREAM_UNROLL = 8;  // independent 16-byte loads in flight per thread
constexpr int STREAM_THREADS = 512;

// Every thread reads STREAM_UNROLL chunks a grid stride apart per round (each
// warp instruction covers 512 contiguous bytes), folds them with XOR and the
// block's warps fold their words into *sink, so no load can be dropped.
__global__ void __launch_bounds__(STREAM_THREADS) stream_read_kernel(const uint4 *src, long long n16,
                                                                     unsigned int *sink) {
  const long long stride = (long long)gridDim.x * blockDim.x;
  long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  uint32_t x = 0;
  for (; i + (STREAM_UNROLL - 1) * stride < n16; i += STREAM_UNROLL * stride) {
    uint4 v[STREAM_UNROLL];
#pragma unroll
    for (int u = 0; u < STREAM_UNROLL; ++u) v[u] = ld_stream16(src + i + u * stride);
#pragma unroll
    for (int u = 0; u < STREAM_UNROLL; ++u) x ^= v[u].x ^ v[u].y ^ v[u].z ^ v[u].w;
  }
  for (; i < n16; i += stride) {
    const uint4 v = ld_stream16(src + i);
    x ^= v.x ^ v.y ^ v.z ^ v.w;
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) x ^= __shfl_xor_sync(FULL, x, off);
  if ((threadIdx.x & 31) == 0) atomicXor(sink, x);
}

}  // namespace pa
