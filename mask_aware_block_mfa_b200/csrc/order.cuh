// Work ordering shared by the tile-map kernels: longest work first.
#pragma once

#include <cstdint>

namespace mfa {

// Stable counting sort of E entries by count[e] in [0, max_count], largest
// first, by one block (all of its threads call it). Histogram and bucket
// offsets live in shared memory (s_buf, max_count + 1 ints); warp 0 then
// places the entries 32 at a time in index order, so equal counts keep
// ascending indices.
__device__ __forceinline__ void order_by_count_desc(const int32_t* __restrict__ count, int E, int max_count,
                                                    int32_t* __restrict__ order, int* s_buf) {
  const int t = threadIdx.x;
  for (int c = t; c <= max_count; c += blockDim.x) s_buf[c] = 0;
  __syncthreads();
  for (int e = t; e < E; e += blockDim.x) atomicAdd(&s_buf[count[e]], 1);
  __syncthreads();
  if (t == 0) {  // offsets for descending counts
    int acc = 0;
    for (int c = max_count; c >= 0; --c) {
      const int h = s_buf[c];
      s_buf[c] = acc;
      acc += h;
    }
  }
  __syncthreads();
  if (t < 32) {
    const int lane = t;
    for (int base = 0; base < E; base += 32) {
      const int e = base + lane;
      const int c = e < E ? count[e] : -1;
      const unsigned peers = __match_any_sync(0xffffffffu, c);
      const int rank = __popc(peers & ((1u << lane) - 1u));
      const int leader = __ffs(peers) - 1;
      int off = 0;
      if (c >= 0 && lane == leader) off = s_buf[c];
      off = __shfl_sync(0xffffffffu, off, leader);
      if (c >= 0) order[off + rank] = e;
      __syncwarp();
      if (c >= 0 && lane == leader) s_buf[c] = off + __popc(peers);
      __syncwarp();
    }
  }
}

}  // namespace mfa
