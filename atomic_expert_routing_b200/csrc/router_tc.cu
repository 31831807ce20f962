// Router logits on the 5th-generation tensor cores (bf16 in, fp32 out):
// Z[t, :Nr] = x[t] Wr^T and Z[t, Nr:] = x[t] Wc^T, the two projections of the
// Cartesian Product Router ("OmniMoE: An Efficient MoE by Orchestrating
// Atomic Experts at Scale" (gist.science), Technisch Overzicht section 2.2).
// This is the one dense contraction of the routed layer: 2*d*(Nr+Nc) flops
// per token.
//
// Persistent: CTA c computes the 128 x BN tiles c, c + gridDim.x, ... of Z
// (N tile fastest, so the CTAs working at one time share their x rows in L2).
// Warp 4 (one elected lane) streams 128 x 64 tiles of x and BN x 64 tiles of
// the axis keys into a shared-memory ring with TMA (128-byte swizzle, no
// multicast), without a break between tiles; warp 5 (one lane) issues
// tcgen05.mma (M=128, N=BN, K=16, bf16 -> fp32) into one of two TMEM
// accumulators and releases each stage with tcgen05.commit; warps 0-3 drain
// the other accumulator with tcgen05.ld (one row per thread) and store fp32
// logits, so a tile's epilogue overlaps the next tile's products.
// Every mbarrier wait is bounded; a time-out sets OMNI_DEV_TIMEOUT and the
// roles leave their loops.
#include <cuda.h>

#include "common.cuh"
#include "internal.h"
#include "tc_common.cuh"

namespace omni {
namespace {

using namespace tc;

template <int BN>
constexpr size_t tc_smem_bytes() {
  return 1024 /* alignment slack */ +
         static_cast<size_t>(TC_STAGES) * (TC_BM * TC_BK * 2 + BN * TC_BK * 2) +
         (2 * TC_STAGES + 5) * 8 + 16;
}

// Tile t of the grid of tiles: M block, N tile (rows then columns of the
// grid of experts), K split.
struct RouterTiles {
  int mt, ntn, tiles_r, ks, kper, nk_all;
  __device__ __forceinline__ void at(int t, int* m, int* n, int* z) const {
    const int per = mt * ntn;
    *z = t / per;
    const int rem = t - *z * per;
    *m = rem / ntn;
    *n = rem - *m * ntn;
  }
};

template <int BN>
__global__ void __launch_bounds__(TC_THREADS, 1)
    k_router_tc(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmBr,
                const __grid_constant__ CUtensorMap tmBc, float* __restrict__ Z, int L, int Nr,
                int Nc, RouterTiles T, int32_t* status) {
  pdl_wait();
  // let the selection launch early only for a single wave of tiles (small L):
  // for many waves its waiting CTAs would sit beside the last tiles
  if (T.mt * T.ntn * T.ks <= 296) pdl_trigger();
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
  const uint32_t full0 = smem_u32(bars);
  const uint32_t empty0 = smem_u32(bars + TC_STAGES);
  const uint32_t tfull0 = smem_u32(bars + 2 * TC_STAGES);       // accumulator b ready
  const uint32_t tempty0 = smem_u32(bars + 2 * TC_STAGES + 2);  // accumulator b drained
  const uint32_t drain = smem_u32(bars + 2 * TC_STAGES + 4);    // MMAs in flight, after a time-out

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t ld = static_cast<int64_t>(Nr) + Nc;
  const int ntiles = T.mt * T.ntn * T.ks;

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
    // producer: TMA loads, one ring of stages across all of this CTA's tiles
    uint32_t it = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
      int m, n, z;
      T.at(t, &m, &n, &z);
      const bool colax = n >= T.tiles_r;
      const CUtensorMap* tmB = colax ? &tmBc : &tmBr;
      const int n0 = (colax ? n - T.tiles_r : n) * BN;
      const int kb0 = z * T.kper;
      const int nk = (T.nk_all - kb0 < T.kper ? T.nk_all - kb0 : T.kper);
      for (int kb = 0; kb < nk; ++kb, ++it) {
        const int s = it % TC_STAGES;
        const uint32_t ph = (it / TC_STAGES) & 1;
        if (!mbar_wait(empty0 + 8 * s, ph ^ 1, status)) {
          ok = false;
          break;
        }
        mbar_expect_tx(full0 + 8 * s, A_BYTES + B_BYTES);
        tma_load_2d(smem_u32(sA + s * A_BYTES), &tmA, full0 + 8 * s, (kb0 + kb) * TC_BK,
                    m * TC_BM);
        tma_load_2d(smem_u32(sB + s * B_BYTES), tmB, full0 + 8 * s, (kb0 + kb) * TC_BK, n0);
      }
    }
    timed_out = !ok;
    issued = it;
  } else if (warp == 5 && lane == 0) {
    // MMA issuer: tile j of this CTA accumulates in TMEM columns (j & 1) * BN
    constexpr uint32_t idesc = idesc_bf16<BN>();
    uint32_t it = 0;
    bool ok = true;
    int j = 0;
    for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x, ++j) {
      int m, n, z;
      T.at(t, &m, &n, &z);
      const int kb0 = z * T.kper;
      const int nk = (T.nk_all - kb0 < T.kper ? T.nk_all - kb0 : T.kper);
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
        const uint32_t a0 = smem_u32(sA + s * A_BYTES);
        const uint32_t b0 = smem_u32(sB + s * B_BYTES);
#pragma unroll
        for (int kk = 0; kk < TC_BK / 16; ++kk)
          umma_bf16(acc, sw128_desc(a0 + kk * 32), sw128_desc(b0 + kk * 32), idesc,
                    (kb | kk) != 0 ? 1u : 0u);
        umma_commit(empty0 + 8 * s);
      }
      umma_commit(tfull0 + 8 * b);
    }
    timed_out = !ok;
  } else if (warp < 4) {
    // epilogue: TMEM lane (32*warp + lane) holds row m0 + 32*warp + lane
    int j = 0;
    for (int t = blockIdx.x; t < ntiles; t += gridDim.x, ++j) {
      int m, n, z;
      T.at(t, &m, &n, &z);
      const int b = j & 1;
      const uint32_t use = static_cast<uint32_t>(j >> 1);
      // the wait's outcome is made warp-uniform: tcgen05.ld below is .sync.aligned
      if (!__all_sync(0xffffffffu, mbar_wait(tfull0 + 8 * b, use & 1, status))) {
        timed_out = true;
        break;
      }
      asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
      const bool colax = n >= T.tiles_r;
      const int n0 = (colax ? n - T.tiles_r : n) * BN;
      const int naxis = colax ? Nc : Nr;
      const int zc0 = (colax ? Nr : 0) + n0;
      float* Zs = Z + static_cast<int64_t>(z) * L * ld;  // split z writes its own partials
      const int64_t grow = static_cast<int64_t>(m) * TC_BM + warp * 32 + lane;
      const bool vec_ok = (ld % 4 == 0) && (zc0 % 4 == 0);  // 16-byte aligned rows
      for (int c = 0; c < BN; c += 32) {
        uint32_t r[32];
        tmem_ld32(tmem + (static_cast<uint32_t>(warp * 32) << 16) + b * BN + c, r);
        if (grow < L) {
          float* zp = Zs + grow * ld + zc0 + c;
          if (n0 + c + 32 <= naxis && vec_ok) {
#pragma unroll
            for (int q = 0; q < 32; q += 4)
              *reinterpret_cast<float4*>(zp + q) =
                  make_float4(__uint_as_float(r[q]), __uint_as_float(r[q + 1]),
                              __uint_as_float(r[q + 2]), __uint_as_float(r[q + 3]));
          } else {
            for (int q = 0; q < 32; ++q)
              if (n0 + c + q < naxis) zp[q] = __uint_as_float(r[q]);
          }
        }
      }
      asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
      mbar_arrive(tempty0 + 8 * b);
    }
  }
  if (timed_out) *aborted = 1u;
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  if (*aborted != 0u) {
    // a wait timed out: this CTA's own TMA loads and MMAs still in flight
    // land (each wait bounded again) before TMEM is freed and the CTA exits.
    // The last TC_STAGES loads went to distinct stages, each in its latest
    // phase; one commit tracks every MMA the issuing thread started.
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
  if (warp == 0) {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(2 * BN)
                 : "memory");
  }
}

// N tile: the widest the axes allow, narrowed while a few row tiles (small L)
// would leave most SMs to split-K partials instead of output tiles.
int pick_bn(const Dims& D) {
  const int64_t m = D.Nr < D.Nc ? D.Nr : D.Nc;
  int bn = m >= 256 ? 256 : (m >= 128 ? 128 : 64);
  const int64_t mt = (D.L + TC_BM - 1) / TC_BM;
  while (bn > 64 && mt * ((D.Nr + bn - 1) / bn + (D.Nc + bn - 1) / bn) < 74) bn >>= 1;
  return bn;
}

template <int BN>
cudaError_t launch_bn(const Dims& D, const CUtensorMap& a, const CUtensorMap& br,
                      const CUtensorMap& bc, float* Z, int32_t* status, cudaStream_t s) {
  const size_t smem = tc_smem_bytes<BN>();
  cudaError_t err = cudaFuncSetAttribute(k_router_tc<BN>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
  if (err != cudaSuccess) return err;
  RouterTiles T;
  T.tiles_r = static_cast<int>((D.Nr + BN - 1) / BN);
  T.ntn = T.tiles_r + static_cast<int>((D.Nc + BN - 1) / BN);
  T.mt = static_cast<int>((D.L + TC_BM - 1) / TC_BM);
  T.nk_all = static_cast<int>((D.d + TC_BK - 1) / TC_BK);
  T.ks = router_splits(D);
  T.kper = (T.nk_all + T.ks - 1) / T.ks;
  const int64_t ntiles = static_cast<int64_t>(T.mt) * T.ntn * T.ks;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t grid = ntiles < sms ? ntiles : sms;  // persistent: one CTA per SM
  OMNI_TRY(launch_k(k_router_tc<BN>, static_cast<unsigned>(grid), TC_THREADS, smem, s, a, br, bc,
      Z, static_cast<int>(D.L), static_cast<int>(D.Nr), static_cast<int>(D.Nc), T, status));
  return cudaGetLastError();
}

}  // namespace

// K-splits from the dims alone (so workspace sizes are known on the host):
// enough CTAs for about one per SM of a 148-SM B200, at most 16 partials.
int router_splits(const Dims& D) {
  if (D.dtype != OMNI_BF16 || (D.flags & OMNI_FLAG_ROUTER_SIMT)) return 1;
  const int bn = pick_bn(D);
  const int64_t tiles = ((D.L + TC_BM - 1) / TC_BM) *
                        ((D.Nr + bn - 1) / bn + (D.Nc + bn - 1) / bn);
  const int nk = static_cast<int>((D.d + TC_BK - 1) / TC_BK);
  int ks = tiles >= 148 ? 1 : static_cast<int>(148 / tiles);
  ks = ks < 1 ? 1 : (ks > 16 ? 16 : ks);
  ks = ks > nk ? nk : ks;
  const int kper = (nk + ks - 1) / ks;
  return (nk + kper - 1) / kper;
}

namespace {
__global__ void __launch_bounds__(256) k_sum_partials(float* __restrict__ Z, int splits, int64_t n) {
  pdl_wait();
  pdl_trigger();
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= n) return;
  float acc = Z[i];
  for (int s = 1; s < splits; ++s) acc += Z[s * n + i];
  Z[i] = acc;
}
}  // namespace

cudaError_t launch_sum_partials(float* Z, int splits, int64_t n, cudaStream_t s) {
  if (splits <= 1 || n == 0) return cudaSuccess;
  OMNI_TRY(launch_k(k_sum_partials, static_cast<unsigned>((n + 255) / 256), 256, 0, s, Z, splits,
      n));
  return cudaGetLastError();
}

bool router_tc_supported(const Dims& D, const void* x, const void* Wr, const void* Wc) {
  if (D.dtype != OMNI_BF16 || (D.flags & OMNI_FLAG_ROUTER_SIMT)) return false;
  if (D.d % 8 != 0 || D.L > (1ll << 30)) return false;  // TMA row pitch: multiple of 16 bytes
  auto al16 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; };
  return al16(x) && al16(Wr) && al16(Wc) && encode_fn() != nullptr;
}

cudaError_t launch_router_tc(const Dims& D, const void* x, const void* Wr, const void* Wc,
                             float* Z, int32_t* status, cudaStream_t s) {
  if (D.L == 0) return cudaSuccess;
  const int bn = pick_bn(D);
  CUtensorMap a, br, bc;
  if (!make_map(&a, x, D.L, D.d, TC_BM) || !make_map(&br, Wr, D.Nr, D.d, bn) ||
      !make_map(&bc, Wc, D.Nc, D.d, bn))
    return cudaErrorInvalidValue;
  switch (bn) {
    case 256: return launch_bn<256>(D, a, br, bc, Z, status, s);
    case 128: return launch_bn<128>(D, a, br, bc, Z, status, s);
    default: return launch_bn<64>(D, a, br, bc, Z, status, s);
  }
}

}  // namespace omni
