// CTA-wide building blocks shared by the scheduler and the executor: an
// exclusive scan over the threads of a block and one stable LSD radix pass
// over up to kBlockSortMax keys held in shared memory.
#pragma once

#include "common.cuh"

namespace omni {

constexpr int kBlockSortMax = 8192;      // keys per CTA-wide sort
constexpr int kBlockSortThreads = 1024;  // threads of a CTA that sorts
constexpr int kBlockSortWarps = kBlockSortThreads / 32;
constexpr int kBlockSortRounds = kBlockSortMax / kBlockSortThreads;  // 32-key rounds per warp

// Exclusive prefix sum of v (int or a 64-bit unsigned) over the threads of
// the block (any blockDim that is a multiple of 32, up to 1024); *total
// receives the block's sum.  warp_tot: 32 values of shared memory.  Every
// thread of the block must call it.
template <typename V>
__device__ __forceinline__ V block_exclusive_scan(V v, V* warp_tot, V* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  V incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const V u = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += u;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int nw = blockDim.x >> 5;
    V w = lane < nw ? warp_tot[lane] : V(0);
    V wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const V u = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += u;
    }
    if (lane < nw) warp_tot[lane] = wi - w;
    if (lane == nw - 1) *total = wi;
  }
  __syncthreads();
  return incl - v + warp_tot[warp];
}

// One stable LSD radix pass (8-bit digit at `shift`) of n <= kBlockSortMax
// keys with 16-bit payloads, in shared memory, by a CTA of kBlockSortThreads
// threads.  Warp w ranks keys [w*256, w*256+256) in order (match_any groups
// equal digits), then the per-warp digit counts are scanned (warp-major
// inside each digit, then over digits) and every key is scattered to its
// final slot.  wcount: kBlockSortWarps*256 words; dbase: 256 words;
// warp_tot: 32 ints; total: one int -- all shared memory.
__device__ __forceinline__ void block_radix_pass(const uint32_t* kin, const uint16_t* vin,
                                                 uint32_t* kout, uint16_t* vout, int n, int shift,
                                                 uint32_t* wcount, uint32_t* dbase, int* warp_tot,
                                                 int* total) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  for (int j = tid; j < kBlockSortWarps * 256; j += kBlockSortThreads) wcount[j] = 0u;
  __syncthreads();
  uint32_t dig[kBlockSortRounds], rnk[kBlockSortRounds];
#pragma unroll
  for (int r = 0; r < kBlockSortRounds; ++r) {
    const int i = warp * (kBlockSortRounds * 32) + r * 32 + lane;
    const bool valid = i < n;
    dig[r] = valid ? ((kin[i] >> shift) & 255u) : 0xffffffffu;
    const uint32_t peers = __match_any_sync(0xffffffffu, dig[r]);
    const int leader = __ffs(peers) - 1;
    uint32_t old = 0;
    if (valid && lane == leader) {
      old = wcount[warp * 256 + dig[r]];
      wcount[warp * 256 + dig[r]] = old + __popc(peers);
    }
    old = __shfl_sync(0xffffffffu, old, leader);
    rnk[r] = old + __popc(peers & lanemask_lt());
    __syncwarp();
  }
  __syncthreads();
  if (tid < 256) {
    uint32_t acc = 0;
    for (int w = 0; w < kBlockSortWarps; ++w) {
      const uint32_t c = wcount[w * 256 + tid];
      wcount[w * 256 + tid] = acc;
      acc += c;
    }
    dbase[tid] = acc;
  }
  __syncthreads();
  {
    const int v = tid < 256 ? static_cast<int>(dbase[tid]) : 0;
    const int ex = block_exclusive_scan(v, warp_tot, total);
    if (tid < 256) dbase[tid] = static_cast<uint32_t>(ex);
  }
  __syncthreads();
#pragma unroll
  for (int r = 0; r < kBlockSortRounds; ++r) {
    const int i = warp * (kBlockSortRounds * 32) + r * 32 + lane;
    if (i < n) {
      const uint32_t pos = dbase[dig[r]] + wcount[warp * 256 + dig[r]] + rnk[r];
      kout[pos] = kin[i];
      vout[pos] = vin[i];
    }
  }
  __syncthreads();
}

}  // namespace omni
