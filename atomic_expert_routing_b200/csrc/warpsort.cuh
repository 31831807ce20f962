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

__device__ __forceinline__ uint32_t shfl_xor_key(uint32_t v, int m) {
  return __shfl_xor_sync(0xffffffffu, v, m);
}
__device__ __forceinline__ uint64_t shfl_xor_key(uint64_t v, int m) { return shfl_xor64(v, m); }

// Bitonic sort into descending order of the 32*W keys (32- or 64-bit) a warp
// holds W per lane (element i = w*32 + lane in key[w]); partners closer than
// 32 are exchanged with shuffles, farther ones sit in the same lane.  With
// P < 32*W (a power of two) every run of P consecutive elements is sorted on
// its own.
template <int W, int P = 32 * W, typename Key>
__device__ __forceinline__ void reg_sort_desc(Key (&key)[W]) {
  static_assert(P >= 1 && P <= 32 * W && (P & (P - 1)) == 0, "segment: a power of two");
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int s = 2; s <= P; s <<= 1) {
#pragma unroll
    for (int j = s >> 1; j > 0; j >>= 1) {
      if (j >= 32) {
#pragma unroll
        for (int w = 0; w < W; ++w) {
          const int wj = w ^ (j >> 5);
          if (wj > w) {
            const bool desc = s == P || ((w * 32) & s) == 0;
            const Key a = key[w], b = key[wj];
            const bool sw = desc ? (a < b) : (a > b);
            key[w] = sw ? b : a;
            key[wj] = sw ? a : b;
          }
        }
      } else {
#pragma unroll
        for (int w = 0; w < W; ++w) {
          const Key o = shfl_xor_key(key[w], j);
          const bool desc = s == P || ((w * 32 + lane) & s) == 0;
          const bool lower = (lane & j) == 0;
          const bool mine_max = key[w] > o;
          key[w] = (lower == desc) == mine_max ? key[w] : o;
        }
      }
    }
  }
}

}  // namespace omni
