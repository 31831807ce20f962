// Expert-Centric Scheduling and grouped execution of a small batch in two
// kernels ("OmniMoE: An Efficient MoE by Orchestrating Atomic Experts at
// Scale" (gist.science), Technisch Overzicht section 2.2; the OmniMoE
// explainer on manus.space, Expert-Centric Scheduling steps 1-4).
//
// For a decode-sized batch (a few thousand tasks) the separate scheduling and
// execution kernels are each bound by their own latency, not by bytes, and
// scatter-adding every task's d-vector into the few rows of y piles fp32
// reductions onto the same lines.  Here:
//
// k_sched_act -- scheduling and the activations, split by expert id (gated
// experts, with a gate matrix U: c also times x[t] . U[e]):
//  1. The ids are cut into kSeTiles tiles of consecutive ids; kSeParts CTAs
//     share a tile.  Every CTA of a tile reads the whole routing (L*K ids)
//     and keeps the tasks whose expert lies in its tile; the tile's CTAs ask
//     L2 to prefetch an eighth of its W rows each.
//  2. It sorts them by expert: a bitmap over the tile's ids and its popcount
//     prefix give every task's expert its rank among the tile's active ids
//     (so the tile's count of active ids), per-rank counts and their scan
//     give every expert its first position.  Tasks of one expert (each for a
//     different token) are placed in any order: that changes no result.
//  3. Part r of the tile computes c = gate * SiLU(x[t] . W[e]) for a
//     contiguous share of that list, cut at expert boundaries, so an
//     expert's W row is read once for all its tokens; c goes to the task's
//     slot t*K + k.  A group of B consecutive active ids is thus executed
//     expert by expert by the CTAs its ids fall to; no CTA needs the global
//     ranks for its part.
//  4. |U| is the sum of the tiles' counts of active ids (atomic adds); the
//     tile that finishes last writes it and the group count ceil(|U| / B).
//
// k_gather_v -- the value rows: CTA (t, s) forms columns s of
//  y[t] = sum over k of c[t, k] * V[idx[t, k]] in registers (each warp a
//  share of the K tasks, then a sum over the warps in shared memory) and
//  stores them in the storage type (bf16: nearest even).  Each output
//  element is written once: no reductions into y, no accumulator to clear.
//
// Tiles have a fixed count, so the split of the ids does not depend on the
// device; no CTA waits on another.  Ids outside [0, N) raise
// OMNI_DEV_BAD_INDEX and are executed as expert 0, as omni_schedule treats
// them.
#include "common.cuh"
#include "blocksort.cuh"
#include "internal.h"

namespace omni {
namespace {

constexpr int kSeThreads = 512;
constexpr int kSeWarps = kSeThreads / 32;
constexpr int kSeTiles = 18;              // tiles of consecutive ids
constexpr int kSeParts = 8;               // CTAs per tile
constexpr int64_t kSeMaxM = 8192;         // tasks (13 bits of a packed task)
constexpr int64_t kSeMaxN = int64_t(1) << 20;  // tile spans below 2^16 ids

__device__ __forceinline__ void prefetch_l2(const void* p, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

__device__ __forceinline__ float dot16(uint4 a, uint4 b, const __nv_bfloat16*) {
  float s0 = 0.0f, s1 = 0.0f;
  s0 = fmaf(bf16lo(a.x), bf16lo(b.x), s0); s1 = fmaf(bf16hi(a.x), bf16hi(b.x), s1);
  s0 = fmaf(bf16lo(a.y), bf16lo(b.y), s0); s1 = fmaf(bf16hi(a.y), bf16hi(b.y), s1);
  s0 = fmaf(bf16lo(a.z), bf16lo(b.z), s0); s1 = fmaf(bf16hi(a.z), bf16hi(b.z), s1);
  s0 = fmaf(bf16lo(a.w), bf16lo(b.w), s0); s1 = fmaf(bf16hi(a.w), bf16hi(b.w), s1);
  return s0 + s1;
}
__device__ __forceinline__ float dot16(uint4 a, uint4 b, const float*) {
  return __uint_as_float(a.x) * __uint_as_float(b.x) + __uint_as_float(a.y) * __uint_as_float(b.y) +
         __uint_as_float(a.z) * __uint_as_float(b.z) + __uint_as_float(a.w) * __uint_as_float(b.w);
}
// a[0 : 16 / sizeof(T)] += c * v
__device__ __forceinline__ void axpy16(float c, uint4 v, float* a, const __nv_bfloat16*) {
  a[0] = fmaf(c, bf16lo(v.x), a[0]); a[1] = fmaf(c, bf16hi(v.x), a[1]);
  a[2] = fmaf(c, bf16lo(v.y), a[2]); a[3] = fmaf(c, bf16hi(v.y), a[3]);
  a[4] = fmaf(c, bf16lo(v.z), a[4]); a[5] = fmaf(c, bf16hi(v.z), a[5]);
  a[6] = fmaf(c, bf16lo(v.w), a[6]); a[7] = fmaf(c, bf16hi(v.w), a[7]);
}
__device__ __forceinline__ void axpy16(float c, uint4 v, float* a, const float*) {
  a[0] = fmaf(c, __uint_as_float(v.x), a[0]); a[1] = fmaf(c, __uint_as_float(v.y), a[1]);
  a[2] = fmaf(c, __uint_as_float(v.z), a[2]); a[3] = fmaf(c, __uint_as_float(v.w), a[3]);
}
// four values to the storage type (bf16: nearest even)
__device__ __forceinline__ void store4(__nv_bfloat16* p, float4 v) {
  const __nv_bfloat162 lo2 = __floats2bfloat162_rn(v.x, v.y);
  const __nv_bfloat162 hi2 = __floats2bfloat162_rn(v.z, v.w);
  uint2 u;
  u.x = *reinterpret_cast<const uint32_t*>(&lo2);
  u.y = *reinterpret_cast<const uint32_t*>(&hi2);
  *reinterpret_cast<uint2*>(p) = u;
}
__device__ __forceinline__ void store4(float* p, float4 v) { *reinterpret_cast<float4*>(p) = v; }

// Global scratch of one call, zeroed before the kernel: the sum of the
// tiles' active ids, finished tiles.
struct SeScratch {
  uint32_t* uacc;
  uint32_t* tiles_done;
};

struct SePlan {
  int64_t span;   // ids per tile
  int words;      // bitmap words of a tile
  size_t smem;
};

// d = NV * 32 * (16 / sizeof(T)): every lane holds NV 16-byte vectors of a row.
// Every phase issues its global loads before it uses any of them.  GLU: gated
// experts, c also times x[t] . U[e].
template <typename T, int NV, bool GLU>
__global__ void __launch_bounds__(kSeThreads, 1)
    k_sched_act(const T* __restrict__ x, const T* __restrict__ W, const T* __restrict__ U,
                const int32_t* __restrict__ idx,
                const float* __restrict__ gate, int L, int K, int64_t N, int B, SePlan P,
                ShardIds sh, float* __restrict__ cbuf, SeScratch sc,
                int32_t* __restrict__ counts) {
  constexpr int EPV = 16 / sizeof(T);
  constexpr int kPer = kSeMaxM / kSeThreads;  // routing ids per thread
  constexpr uint32_t kIdxMask = (1u << 13) - 1u;
  const int d = NV * 32 * EPV;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int M = L * K;
  const int tile = blockIdx.x / kSeParts, part = blockIdx.x % kSeParts;
  // the tile's ids [lo, hi) within this process' ids [sh.lo, sh.hi); the
  // row of id e is e - sh.lo
  const int64_t lo = sh.lo + static_cast<int64_t>(tile) * P.span;
  const int64_t hi = lo + P.span < sh.hi ? lo + P.span : sh.hi;
  extern __shared__ __align__(16) uint8_t sm[];
  uint32_t* own = reinterpret_cast<uint32_t*>(sm);   // [M] (e - lo) << 13 | task index
  uint32_t* sorted = own + M;                        // [M] the same, by expert
  int* ecnt = reinterpret_cast<int*>(sorted + M);    // [M] tasks per expert rank, then first position
  int* ecur = ecnt + M;                              // [M] placement cursors
  uint32_t* lbits = reinterpret_cast<uint32_t*>(ecur + M);  // [words] the tile's active ids
  int* lpre = reinterpret_cast<int*>(lbits + P.words);      // [words] rank before each word
  __shared__ int warp_tot[32];
  __shared__ int total, nown;
  int32_t* status = counts + 2;

  for (int j = tid; j < P.words; j += kSeThreads) lbits[j] = 0u;
  if (tid == 0) nown = 0;
  pdl_wait();
  pdl_trigger();
  __syncthreads();

  // (1) the tile's tasks: every routing id of this thread loaded first
  {
    int ev[kPer];
#pragma unroll
    for (int q = 0; q < kPer; ++q) {
      const int i = tid + q * kSeThreads;
      ev[q] = i < M ? idx[i] : 0;
    }
#pragma unroll
    for (int q = 0; q < kPer; ++q) {
      const int i = tid + q * kSeThreads;
      if (i < M) {
        int64_t e = ev[q];
        if (e < 0 || e >= N) {
          if (blockIdx.x == 0) raise_status(status, OMNI_DEV_BAD_INDEX);
          e = 0;
        }
        if (e >= lo && e < hi) {
          const uint32_t el = static_cast<uint32_t>(e - lo);
          own[atomicAdd(&nown, 1)] = (el << 13) | static_cast<uint32_t>(i);
          atomicOr(&lbits[el >> 5], 1u << (el & 31));
        }
      }
    }
  }
  __syncthreads();
  const int n = nown;
  // the tile's W rows, whole (d * sizeof(T) bytes, 16-byte multiples): part
  // r asks L2 for those of own tasks r, r + parts, ... while the tile is
  // sorted
  for (int q = part + kSeParts * tid; q < n; q += kSeParts * kSeThreads)
    prefetch_l2(W + (lo - sh.lo + (own[q] >> 13)) * d, static_cast<uint32_t>(d * sizeof(T)));

  // (2) rank of every active id of the tile (popcount prefix of the bitmap)
  {
    const int per = (P.words + kSeThreads - 1) / kSeThreads;
    const int w0 = tid * per;
    const int w1 = w0 + per < P.words ? w0 + per : P.words;
    int mine = 0;
    for (int w = w0; w < w1; ++w) mine += __popc(lbits[w]);
    int run = block_exclusive_scan(mine, warp_tot, &total);
    for (int w = w0; w < w1; ++w) {
      lpre[w] = run;
      run += __popc(lbits[w]);
    }
  }
  __syncthreads();
  const int u_tile = total;
  auto rank_of = [&](uint32_t el) {
    return lpre[el >> 5] + __popc(lbits[el >> 5] & ((1u << (el & 31)) - 1u));
  };
  for (int r = tid; r < u_tile; r += kSeThreads) {
    ecnt[r] = 0;
    ecur[r] = 0;
  }
  __syncthreads();
  for (int j = tid; j < n; j += kSeThreads) atomicAdd(&ecnt[rank_of(own[j] >> 13)], 1);
  __syncthreads();
  // first position of every expert (exclusive scan of the counts, in place)
  {
    const int per = (u_tile + kSeThreads - 1) / kSeThreads;
    const int r0 = tid * per;
    const int r1 = r0 + per < u_tile ? r0 + per : u_tile;
    int mine = 0;
    for (int r = r0; r < r1; ++r) mine += ecnt[r];
    int run = block_exclusive_scan(mine, warp_tot, &total);
    for (int r = r0; r < r1; ++r) {
      const int c = ecnt[r];
      ecnt[r] = run;
      run += c;
    }
  }
  __syncthreads();
  for (int j = tid; j < n; j += kSeThreads) {
    const uint32_t v = own[j];
    const int r = rank_of(v >> 13);
    sorted[ecnt[r] + atomicAdd(&ecur[r], 1)] = v;
  }
  // |U| and the group count: part 0 of every tile adds its count; the tile
  // that finishes last writes both
  if (part == 0 && tid == 0) {
    atomicAdd(sc.uacc, static_cast<uint32_t>(u_tile));
    __threadfence();
    if (atomicAdd(sc.tiles_done, 1u) == kSeTiles - 1) {
      __threadfence();
      const uint32_t u = atomicAdd(sc.uacc, 0u);
      counts[0] = static_cast<int32_t>(u);
      counts[1] = static_cast<int32_t>((static_cast<int64_t>(u) + B - 1) / B);
    }
  }
  __syncthreads();

  // (3) this part's share [b0, b1) of the expert-sorted list, cut where an
  // expert starts (the first expert starting at or after part * n / parts)
  auto cut = [&](int q) {
    if (q >= kSeParts) return n;
    const int want = static_cast<int>((static_cast<int64_t>(q) * n + kSeParts - 1) / kSeParts);
    int l = 0, h = u_tile;  // first rank whose start is >= want
    while (l < h) {
      const int m = (l + h) >> 1;
      if (ecnt[m] >= want) h = m; else l = m + 1;
    }
    return l < u_tile ? ecnt[l] : n;
  };
  const int b0 = cut(part), b1 = cut(part + 1);

  // (4) activations; warp w takes positions b0 + w, b0 + w + 16, ..., PAIR at
  // a time (their x and W rows loaded together; one at d = 256 vectors, which
  // fill the registers)
  constexpr int PAIR = (NV >= 8 || (GLU && NV >= 4)) ? 1 : 2;
  constexpr int NU = GLU ? NV : 1;  // vectors of the U row held per lane
  for (int p0 = b0 + warp; p0 < b1; p0 += PAIR * kSeWarps) {
    uint4 xv[PAIR][NV], wv[PAIR][NV], uv[PAIR][NU];
    int ii[PAIR];
#pragma unroll
    for (int r = 0; r < PAIR; ++r) {
      const int pos = p0 + r * kSeWarps;
      ii[r] = -1;
      if (pos >= b1) continue;
      const uint32_t v = sorted[pos];  // warp-uniform
      ii[r] = static_cast<int>(v & kIdxMask);
      const int64_t e = lo - sh.lo + (v >> 13);  // the row
      const uint4* xr = reinterpret_cast<const uint4*>(x + static_cast<int64_t>(ii[r] / K) * d);
      const uint4* wr = reinterpret_cast<const uint4*>(W + e * d);
#pragma unroll
      for (int q = 0; q < NV; ++q) {
        xv[r][q] = xr[q * 32 + lane];
        wv[r][q] = wr[q * 32 + lane];
      }
      if constexpr (GLU) {
        const uint4* ur = reinterpret_cast<const uint4*>(U + e * d);
#pragma unroll
        for (int q = 0; q < NV; ++q) uv[r][q] = ur[q * 32 + lane];
      }
    }
#pragma unroll
    for (int r = 0; r < PAIR; ++r) {
      if (ii[r] < 0) continue;
      float sdot = 0.0f;
#pragma unroll
      for (int q = 0; q < NV; ++q) sdot += dot16(xv[r][q], wv[r][q], static_cast<const T*>(nullptr));
      sdot = warp_sum(sdot);
      float c = gate[ii[r]] * silu(sdot);
      if constexpr (GLU) {
        float su = 0.0f;
#pragma unroll
        for (int q = 0; q < NV; ++q) su += dot16(xv[r][q], uv[r][q], static_cast<const T*>(nullptr));
        c *= warp_sum(su);
      }
      if (lane == 0) cbuf[ii[r]] = c;
    }
  }
}

// CTA (t, s): y[t, s*cols : (s+1)*cols] = sum_k c[t, k] * V[idx[t, k], same
// columns], cols = NS * 32 * (16 / sizeof(T)).  Warp w sums tasks w, w + 16,
// ... in registers; the warps' partial rows are added in shared memory in a
// fixed order (the result does not depend on timing).
template <typename T, int NS, typename O>
__global__ void __launch_bounds__(kSeThreads)
    k_gather_v(const T* __restrict__ V, const int32_t* __restrict__ idx,
               const float* __restrict__ cbuf, int K, int64_t N, int d, ShardIds sh,
               O* __restrict__ y, int32_t* __restrict__ status) {
  constexpr int EPV = 16 / sizeof(T);
  constexpr int COLS = NS * 32 * EPV;
  __shared__ __align__(16) float part[kSeWarps][COLS];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t t = blockIdx.x;
  const int col0 = blockIdx.y * COLS;
  pdl_wait();
  pdl_trigger();
  float a[NS][EPV];
#pragma unroll
  for (int q = 0; q < NS; ++q)
#pragma unroll
    for (int u = 0; u < EPV; ++u) a[q][u] = 0.0f;
  for (int k0 = warp; k0 < K; k0 += 2 * kSeWarps) {
    uint4 vv[2][NS];
    float cc[2];
    bool live[2];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int k = k0 + r * kSeWarps;
      cc[r] = 0.0f;
      live[r] = false;
      if (k >= K) continue;
      int64_t e = idx[t * K + k];
      if (e < 0 || e >= N) {
        if (lane == 0) raise_status(status, OMNI_DEV_BAD_INDEX);
        e = 0;
      }
      if (!sh.has(e)) continue;  // another shard's task
      live[r] = true;
      cc[r] = cbuf[t * K + k];
      const uint4* vr = reinterpret_cast<const uint4*>(V + (e - sh.lo) * d + col0);
#pragma unroll
      for (int q = 0; q < NS; ++q) vv[r][q] = vr[q * 32 + lane];
    }
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      if (!live[r]) continue;
#pragma unroll
      for (int q = 0; q < NS; ++q) axpy16(cc[r], vv[r][q], a[q], static_cast<const T*>(nullptr));
    }
  }
#pragma unroll
  for (int q = 0; q < NS; ++q)
#pragma unroll
    for (int u = 0; u < EPV; u += 4)
      *reinterpret_cast<float4*>(&part[warp][(q * 32 + lane) * EPV + u]) =
          make_float4(a[q][u], a[q][u + 1], a[q][u + 2], a[q][u + 3]);
  __syncthreads();
  // thread j sums columns [j*EPV/... ): COLS columns over kSeThreads threads
  for (int c = tid * 4; c < COLS; c += kSeThreads * 4) {
    float4 s4 = *reinterpret_cast<const float4*>(&part[0][c]);
#pragma unroll
    for (int w = 1; w < kSeWarps; ++w) {
      const float4 p = *reinterpret_cast<const float4*>(&part[w][c]);
      s4.x += p.x; s4.y += p.y; s4.z += p.z; s4.w += p.w;
    }
    store4(y + t * d + col0 + c, s4);
  }
}

int se_nv(const Dims& D) {
  const int64_t row = D.dtype == OMNI_F32 ? 128 : 256;  // elements of one 16-byte vector per lane
  if (D.d % row != 0) return 0;
  const int64_t nv = D.d / row;
  return (nv == 1 || nv == 2 || nv == 4 || nv == 8) ? static_cast<int>(nv) : 0;
}

// A function of the dims alone (not of the device), so that the workspace
// sized from it holds for a launch on any device.
bool se_plan(const Dims& D, SePlan* P) {
  const int64_t M = D.M();
  if (D.L < 1 || M > kSeMaxM || D.N() > kSeMaxN || se_nv(D) == 0) return false;
  if (D.B > (int64_t(1) << 30)) return false;
  // supported or not by the whole layer's ids (a shard's tiles are no
  // larger), so that the decision and the workspace do not depend on the
  // shard; the tiles then split this process' ids
  auto plan = [&](int64_t ids) {
    P->span = (ids + kSeTiles - 1) / kSeTiles;
    P->words = static_cast<int>((P->span + 31) / 32);
    P->smem = static_cast<size_t>(M) * 16 + static_cast<size_t>(P->words) * 8;
    return P->smem <= 200 * 1024;
  };
  if (!plan(D.N())) return false;
  return plan(D.shard_hi() - D.shard_lo());
}

// workspace words: the two scratch counters (cleared before the call), then
// c [M] floats from the next 256-byte boundary
constexpr size_t kSeCbufOff = 64;

template <typename T, int NV, bool GLU>
cudaError_t launch_se_t(const Dims& D, const SePlan& P, const void* x, const void* W,
                        const void* V, const int32_t* idx, const float* gate, void* y,
                        uint32_t* ws, int32_t* counts, cudaStream_t s, const void* U) {
  cudaError_t err = cudaFuncSetAttribute(k_sched_act<T, NV, GLU>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(P.smem));
  if (err != cudaSuccess) return err;
  SeScratch sc;
  sc.uacc = ws;
  sc.tiles_done = ws + 1;
  float* cbuf = reinterpret_cast<float*>(ws + kSeCbufOff);
  OMNI_TRY(launch_k(k_sched_act<T, NV, GLU>, kSeTiles * kSeParts, kSeThreads, P.smem, s,
      static_cast<const T*>(x), static_cast<const T*>(W), static_cast<const T*>(U), idx, gate,
      static_cast<int>(D.L),
      static_cast<int>(D.K), D.N(), static_cast<int>(D.B), P, shard_ids(D), cbuf, sc, counts));
  // value rows: NS vectors per lane and CTA, 2 when the row has them
  constexpr int NS = NV < 2 ? NV : 2;
  constexpr int COLS = NS * 32 * (16 / sizeof(T));
  const dim3 grid(static_cast<unsigned>(D.L), static_cast<unsigned>(D.d / COLS));
  // a shard's partial sum stays in fp32
  if (D.sharded()) {
    OMNI_TRY(launch_k(k_gather_v<T, NS, float>, grid, kSeThreads, 0, s, static_cast<const T*>(V),
        idx, static_cast<const float*>(cbuf), static_cast<int>(D.K), D.N(),
        static_cast<int>(D.d), shard_ids(D), static_cast<float*>(y), counts + 2));
  } else {
    OMNI_TRY(launch_k(k_gather_v<T, NS, T>, grid, kSeThreads, 0, s, static_cast<const T*>(V), idx,
        static_cast<const float*>(cbuf), static_cast<int>(D.K), D.N(), static_cast<int>(D.d),
        shard_ids(D), static_cast<T*>(y), counts + 2));
  }
  return cudaGetLastError();
}

}  // namespace

bool sched_exec_supported(const Dims& D) {
  if (D.flags & OMNI_FLAG_STAGED_SMALL) return false;
  SePlan P;
  return se_plan(D, &P) && D.L <= 65535;
}

size_t sched_exec_ws_words(const Dims& D) { return kSeCbufOff + static_cast<size_t>(D.M()); }

cudaError_t launch_sched_exec(const Dims& D, const void* x, const void* W, const void* V,
                              const int32_t* idx, const float* gate, void* y, uint32_t* ws,
                              int32_t* counts, cudaStream_t s, const void* U) {
  SePlan P;
  if (!se_plan(D, &P)) return cudaErrorInvalidValue;
#define OMNI_SE(T_, NV_)                                                                  \
  return U != nullptr                                                                     \
             ? launch_se_t<T_, NV_, true>(D, P, x, W, V, idx, gate, y, ws, counts, s, U)  \
             : launch_se_t<T_, NV_, false>(D, P, x, W, V, idx, gate, y, ws, counts, s, U);
  if (D.dtype == OMNI_F32) {
    switch (se_nv(D)) {
      case 1: OMNI_SE(float, 1)
      case 2: OMNI_SE(float, 2)
      case 4: OMNI_SE(float, 4)
      default: OMNI_SE(float, 8)
    }
  }
  switch (se_nv(D)) {
    case 1: OMNI_SE(__nv_bfloat16, 1)
    case 2: OMNI_SE(__nv_bfloat16, 2)
    case 4: OMNI_SE(__nv_bfloat16, 4)
    default: OMNI_SE(__nv_bfloat16, 8)
  }
#undef OMNI_SE
}

}  // namespace omni
