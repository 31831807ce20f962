// A persistent bf16 GEMM on the 5th-generation tensor cores, D = A B^T with
// A [M x K] and B [Nn x K] both K-major (row-major with K contiguous), fp32
// accumulation in TMEM, and a caller-supplied epilogue.
//
// CTA c takes the tiles c, c + gridDim.x, ... of a tile source (128 rows of A
// by BN rows of B).  Warp 4 (one elected lane) streams 128 x 64 tiles of A
// and BN x 64 tiles of B into a 4-stage shared-memory ring with TMA (128-byte
// swizzle, no multicast) without a break between tiles; warp 5 (one lane)
// issues tcgen05.mma (M = 128, N = BN, K = 16) into one of two TMEM
// accumulators and frees each stage with tcgen05.commit; warps 0-3 drain the
// other accumulator with tcgen05.ld, 32 columns at a time, into the
// epilogue, so a tile's epilogue overlaps the next tile's products.  Rows of
// a tile past the end of A or B read as zeros (TMA out-of-bounds fill).
// Every mbarrier wait is bounded: a time-out sets OMNI_DEV_TIMEOUT, the roles
// leave their loops, and the CTA waits (bounded again) for its own loads and
// MMAs in flight before it frees TMEM.
//
// Tile source: int count() (tiles, read after the kernel ahead finished) and
// void at(int t, int* a_row0, int* b_row0) (first rows of tile t).
// Epilogue: static constexpr size_t kStageBytes (shared memory it may use,
// 0 for none); void operator()(int t, int a_row0, int b_row0, int r, int c,
// const uint32_t* v, float* stage) -- row r (0..127) of tile t, fp32 bit
// patterns of its columns c .. c + 31 (0 <= c < BN); and, when kStageBytes
// > 0, void tile_end(int t, int a_row0, int b_row0, int i, float* stage),
// called by the 128 epilogue threads (i = 0..127) once every row of the tile
// has been handed over (the stage is theirs until the next tile's rows).
#pragma once

#include "internal.h"
#include "tc_common.cuh"

namespace omni {
namespace tc {

template <int BN>
constexpr size_t gemm_smem_bytes() {
  return 1024 /* alignment slack */ +
         static_cast<size_t>(TC_STAGES) * (TC_BM * TC_BK * 2 + BN * TC_BK * 2) +
         (2 * TC_STAGES + 5) * 8 + 16;
}

// named barrier of the four epilogue warps (barrier 0 is __syncthreads)
__device__ __forceinline__ void epilogue_sync() {
  asm volatile("bar.sync 1, 128;" ::: "memory");
}

template <int BN, class Tiles, class Epi>
__global__ void __launch_bounds__(TC_THREADS, 1)
    k_gemm_tc(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
              int nk, Tiles T, Epi epi, int32_t* status) {
  pdl_wait();
  constexpr uint32_t A_BYTES = TC_BM * TC_BK * 2;
  constexpr uint32_t B_BYTES = BN * TC_BK * 2;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + TC_STAGES * A_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sB + TC_STAGES * B_BYTES);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * TC_STAGES + 5);
  uint32_t* aborted = tmem_slot + 1;  // a wait of this CTA timed out
  float* stage = reinterpret_cast<float*>(aborted + 3);  // Epi::kStageBytes (4-byte aligned)
  const uint32_t full0 = smem_u32(bars);
  const uint32_t empty0 = smem_u32(bars + TC_STAGES);
  const uint32_t tfull0 = smem_u32(bars + 2 * TC_STAGES);       // accumulator b ready
  const uint32_t tempty0 = smem_u32(bars + 2 * TC_STAGES + 2);  // accumulator b drained
  const uint32_t drain = smem_u32(bars + 2 * TC_STAGES + 4);    // MMAs in flight, after a time-out
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ntiles = T.count();

  if (threadIdx.x == 0) {
    for (int s = 0; s < TC_STAGES; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(tfull0 + 8 * b, 1);
      mbar_init(tempty0 + 8 * b, 128);
    }
    mbar_init(drain, 1);
    *aborted = 0u;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(2 * BN)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t tmem = *tmem_slot;

  bool timed_out = false;
  uint32_t issued = 0;  // producer: TMA stages loaded
  if (warp == 4 && lane == 0) {
    uint32_t it = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
      int a0, b0;
      T.at(t, &a0, &b0);
      for (int kb = 0; kb < nk; ++kb, ++it) {
        const int s = it % TC_STAGES;
        const uint32_t ph = (it / TC_STAGES) & 1;
        if (!mbar_wait(empty0 + 8 * s, ph ^ 1, status)) {
          ok = false;
          break;
        }
        mbar_expect_tx(full0 + 8 * s, A_BYTES + B_BYTES);
        tma_load_2d(smem_u32(sA + s * A_BYTES), &tmA, full0 + 8 * s, kb * TC_BK, a0);
        tma_load_2d(smem_u32(sB + s * B_BYTES), &tmB, full0 + 8 * s, kb * TC_BK, b0);
      }
    }
    timed_out = !ok;
    issued = it;
  } else if (warp == 5 && lane == 0) {
    // tile j of this CTA accumulates in TMEM columns (j & 1) * BN
    constexpr uint32_t idesc = idesc_bf16<BN>();
    uint32_t it = 0;
    bool ok = true;
    int j = 0;
    for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x, ++j) {
      const int b = j & 1;
      const uint32_t use = static_cast<uint32_t>(j >> 1);
      if (!mbar_wait(tempty0 + 8 * b, (use & 1) ^ 1, status)) {  // drained by the epilogue
        ok = false;
        break;
      }
      asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
      const uint32_t acc = tmem + static_cast<uint32_t>(b * BN);
      for (int kb = 0; kb < nk; ++kb, ++it) {
        const int s = it % TC_STAGES;
        const uint32_t ph = (it / TC_STAGES) & 1;
        if (!mbar_wait(full0 + 8 * s, ph, status)) {
          ok = false;
          break;
        }
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        const uint32_t sa = smem_u32(sA + s * A_BYTES);
        const uint32_t sb = smem_u32(sB + s * B_BYTES);
#pragma unroll
        for (int kk = 0; kk < TC_BK / 16; ++kk)
          umma_bf16(acc, sw128_desc(sa + kk * 32), sw128_desc(sb + kk * 32), idesc,
                    (kb | kk) != 0 ? 1u : 0u);
        umma_commit(empty0 + 8 * s);
      }
      umma_commit(tfull0 + 8 * b);
    }
    timed_out = !ok;
  } else if (warp < 4) {
    // epilogue: TMEM lane (32 * warp + lane) holds row 32 * warp + lane of the tile
    int j = 0;
    for (int t = blockIdx.x; t < ntiles; t += gridDim.x, ++j) {
      int a0, b0;
      T.at(t, &a0, &b0);
      const int b = j & 1;
      const uint32_t use = static_cast<uint32_t>(j >> 1);
      // the wait's outcome is made warp-uniform: tcgen05.ld below is .sync.aligned
      if (!__all_sync(0xffffffffu, mbar_wait(tfull0 + 8 * b, use & 1, status))) {
        timed_out = true;
        break;
      }
      asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
      for (int c = 0; c < BN; c += 32) {
        uint32_t r[32];
        tmem_ld32(tmem + (static_cast<uint32_t>(warp * 32) << 16) + b * BN + c, r);
        epi(t, a0, b0, warp * 32 + lane, c, r, stage);
      }
      asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
      mbar_arrive(tempty0 + 8 * b);  // TMEM is free once every row is read
      if constexpr (Epi::kStageBytes > 0) {
        epilogue_sync();  // every row is in the stage
        epi.tile_end(t, a0, b0, warp * 32 + lane, stage);
        epilogue_sync();  // the stage is free for the next tile
      }
    }
  }
  if (timed_out) *aborted = 1u;
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  if (*aborted != 0u) {
    // a wait timed out: this CTA's own TMA loads and MMAs still in flight
    // land (each wait bounded again) before TMEM is freed and the CTA exits
    if (warp == 4 && lane == 0) {
      const uint32_t first = issued > TC_STAGES ? issued - TC_STAGES : 0u;
      for (uint32_t i = first; i < issued; ++i)
        mbar_wait(full0 + 8 * (i % TC_STAGES), (i / TC_STAGES) & 1, status);
    } else if (warp == 5 && lane == 0) {
      umma_commit(drain);
      mbar_wait(drain, 0, status);
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
  }
  pdl_trigger();
  if (warp == 0) {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(2 * BN)
                 : "memory");
  }
}

// Every 128 x BN tile of an [M x Nn] product, B tiles fastest (the CTAs at
// work share their A rows in L2).
template <int BN>
struct DenseTiles {
  int mt, nt;
  __device__ __forceinline__ int count() const { return mt * nt; }
  __device__ __forceinline__ void at(int t, int* a0, int* b0) const {
    *a0 = (t / nt) * TC_BM;
    *b0 = (t % nt) * BN;
  }
};

// Launch k_gemm_tc<BN> over the tiles T on min(tiles, SMs) persistent CTAs
// (tiles_hint: the host's bound on T.count()).
template <int BN, class Tiles, class Epi>
cudaError_t launch_gemm_tc(const CUtensorMap& a, const CUtensorMap& b, int nk, const Tiles& T,
                           int64_t tiles_hint, const Epi& epi, int32_t* status, cudaStream_t s) {
  const size_t smem = gemm_smem_bytes<BN>() + Epi::kStageBytes;
  cudaError_t err = cudaFuncSetAttribute(k_gemm_tc<BN, Tiles, Epi>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
  if (err != cudaSuccess) return err;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  int64_t grid = tiles_hint < sms ? tiles_hint : sms;
  if (grid < 1) grid = 1;
  OMNI_TRY(launch_k(k_gemm_tc<BN, Tiles, Epi>, static_cast<unsigned>(grid), TC_THREADS, smem, s,
                    a, b, nk, T, epi, status));
  return cudaGetLastError();
}

// One GEMM D = A B^T (A [rows x K], B [cols x K], bf16, K-major, rows of K
// elements 16-byte aligned) with epilogue epi: 256-wide B tiles when they
// still give every SM a tile, else 128-wide.
template <class Epi>
cudaError_t gemm_bf16(const void* A, const void* Bm, int64_t rows, int64_t cols, int64_t K,
                      const Epi& epi, int32_t* status, cudaStream_t s) {
  const int64_t mt = (rows + TC_BM - 1) / TC_BM;
  const int nk = static_cast<int>((K + TC_BK - 1) / TC_BK);
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  CUtensorMap a, b;
  if (!make_map(&a, A, rows, K, TC_BM)) return cudaErrorInvalidValue;
  if (mt * ((cols + 255) / 256) >= sms) {
    if (!make_map(&b, Bm, cols, K, 256)) return cudaErrorInvalidValue;
    DenseTiles<256> T{static_cast<int>(mt), static_cast<int>((cols + 255) / 256)};
    return launch_gemm_tc<256>(a, b, nk, T, mt * T.nt, epi, status, s);
  }
  if (!make_map(&b, Bm, cols, K, 128)) return cudaErrorInvalidValue;
  DenseTiles<128> T{static_cast<int>(mt), static_cast<int>((cols + 127) / 128)};
  return launch_gemm_tc<128>(a, b, nk, T, mt * T.nt, epi, status, s);
}

}  // namespace tc
}  // namespace omni
