// Register bitonic sort of 64-bit keys across one warp, shared by the
// selection and the scheduler.
#pragma once

#include <stdint.h>

namespace omni {

__device__ __forceinline__ uint64_t shfl_xor64(uint64_t v, int m) {
  const uint32_t lo = __shfl_xor_sync(0xffffffffu, static_cast<uint32_t>(v), m);
  const uint32_t hi = __shfl_xor_sync(0xffffffffu, static_cast<uint32_t>(v >> 32), m);
  return (static_cast<uint64_t>(hi) << 32) | lo;
}

// Bitonic sort into descending order of the 32*W keys a warp holds W per lane
// (element i = w*32 + lane in key[w]); partners closer than 32 are exchanged
// with shuffles, farther ones sit in the same lane.
template <int W>
__device__ __forceinline__ void reg_sort_desc(uint64_t (&key)[W]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int s = 2; s <= 32 * W; s <<= 1) {
#pragma unroll
    for (int j = s >> 1; j > 0; j >>= 1) {
      if (j >= 32) {
#pragma unroll
        for (int w = 0; w < W; ++w) {
          const int wj = w ^ (j >> 5);
          if (wj > w) {
            const bool desc = ((w * 32) & s) == 0;
            const uint64_t a = key[w], b = key[wj];
            const bool sw = desc ? (a < b) : (a > b);
            key[w] = sw ? b : a;
            key[wj] = sw ? a : b;
          }
        }
      } else {
#pragma unroll
        for (int w = 0; w < W; ++w) {
          const uint64_t o = shfl_xor64(key[w], j);
          const bool desc = ((w * 32 + lane) & s) == 0;
          const bool lower = (lane & j) == 0;
          const bool mine_max = key[w] > o;
          key[w] = (lower == desc) == mine_max ? key[w] : o;
        }
      }
    }
  }
}

}  // namespace omni
