// Grouped execution of a small batch in two kernels, straight from the
// routing ("OmniMoE: An Efficient MoE by Orchestrating Atomic Experts at
// Scale" (gist.science), Technisch Overzicht section 2.2; the OmniMoE
// explainer on manus.space, Expert-Centric Scheduling steps 1-4).
//
// Expert-Centric Scheduling orders the tasks by expert so that each active
// expert's W and V rows leave HBM once for all its tokens.  A batch touches
// at most min(N, L*K) rows of each matrix; when those fit in 64 MiB (decode:
// 4096 rows of 4 KiB each at d = 2048 in bf16), the 126 MB L2 of a B200 holds
// them, so in any task order a row leaves HBM once and later reads of it are
// L2 hits.  A batch whose tasks read at most 1 GiB of rows even without any
// reuse (L*K rows of each matrix) takes the same path: its worst case, about
// 0.16 ms of HBM traffic, is below the cost of sorting its tasks, and the
// rows it shares come from L2.  For such a batch the tasks are not sorted;
// the schedule's counts (|U| and the group count) are still formed, from a
// bitmap of the active ids:
//
// k_task_act -- one warp per task (t, k) in routing order: marks its id in
//   the bitmap (the first task to set a bit counts the id), then
//   c = gate * SiLU(x[t] . W[e]) (gated experts, with a gate matrix U: c also
//   times x[t] . U[e]) into the task's slot t*K + k.  The CTA that finishes
//   last writes |U| and ceil(|U| / B).
//
// k_gather_v -- the value rows: CTA (t, s) forms columns s of
//  y[t] = sum over k of c[t, k] * V[idx[t, k]] in registers (each warp a
//  share of the K tasks, then a sum over the warps in shared memory) and
//  stores them in the storage type (bf16: nearest even).  Each output
//  element is written once: no reductions into y, no accumulator to clear.
//
// No CTA waits on another.  Ids outside [0, N) raise OMNI_DEV_BAD_INDEX and
// are executed as expert 0, as omni_schedule treats them.
#include "common.cuh"
#include "internal.h"

namespace omni {
namespace {

constexpr int kSeThreads = 512;  // k_gather_v
constexpr int kSeWarps = kSeThreads / 32;
constexpr int kTaThreads = 256;  // k_task_act: a task per warp
constexpr int kTaWarps = kTaThreads / 32;
// The bytes of W and V rows a batch can touch (min(N, L*K) rows each) that
// L2 is trusted to hold while the batch runs; and the most row bytes a batch
// may read from HBM if no row of it were reused from L2 (a row per task).
constexpr int64_t kSeRowBudget = int64_t(64) << 20;
constexpr int64_t kSeTaskBudget = int64_t(1) << 30;
constexpr int64_t kSeMaxN = int64_t(1) << 20;  // ids: a bitmap of at most 128 KiB

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

// Global scratch of one call, zeroed before the kernel (the zero words of
// sched_exec_zero_words): the active ids counted, finished CTAs, and the
// bitmap of this process' ids.
struct SeScratch {
  uint32_t* uacc;
  uint32_t* ctas_done;
  uint32_t* bits;
};

// d = NV * 32 * (16 / sizeof(T)): every lane holds NV 16-byte vectors of a
// row.  GLU: gated experts, c also times x[t] . U[e].
template <typename T, int NV, bool GLU>
__global__ void __launch_bounds__(kTaThreads, GLU ? 2 : 4)
    k_task_act(const T* __restrict__ x, const T* __restrict__ W, const T* __restrict__ U,
               const int32_t* __restrict__ idx, const float* __restrict__ gate, int L, int K,
               int64_t N, int B, ShardIds sh, float* __restrict__ cbuf, SeScratch sc,
               int32_t* __restrict__ counts) {
  constexpr int EPV = 16 / sizeof(T);
  const int d = NV * 32 * EPV;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __shared__ uint32_t cta_new;
  if (threadIdx.x == 0) cta_new = 0u;
  pdl_wait();
  pdl_trigger();
  __syncthreads();
  const int64_t M = static_cast<int64_t>(L) * K;
  const int64_t i = static_cast<int64_t>(blockIdx.x) * kTaWarps + warp;  // the task's slot
  if (i < M) {
    int64_t e = idx[i];
    if (e < 0 || e >= N) {
      if (lane == 0) raise_status(counts + 2, OMNI_DEV_BAD_INDEX);
      e = 0;
    }
    if (sh.has(e)) {  // warp-uniform
      const int64_t row = e - sh.lo;
      const uint4* xr = reinterpret_cast<const uint4*>(x + (i / K) * d);
      const uint4* wr = reinterpret_cast<const uint4*>(W + row * d);
      const uint4* ur = GLU ? reinterpret_cast<const uint4*>(U + row * d) : nullptr;
      if (lane == 0) {  // the first task to set the id's bit counts the id
        const uint32_t m = 1u << (row & 31);
        if ((atomicOr(&sc.bits[row >> 5], m) & m) == 0u) atomicAdd(&cta_new, 1u);
      }
      // the row in chunks of CH vectors per lane, each chunk's loads issued
      // together (registers for every task of the batch to be resident)
      constexpr int CH = NV > 4 ? 4 : NV;
      float sdot = 0.0f, su = 0.0f;
#pragma unroll
      for (int q0 = 0; q0 < NV; q0 += CH) {
        uint4 xv[CH], wv[CH], uv[GLU ? CH : 1];
#pragma unroll
        for (int q = 0; q < CH; ++q) {
          xv[q] = xr[(q0 + q) * 32 + lane];
          wv[q] = wr[(q0 + q) * 32 + lane];
          if constexpr (GLU) uv[q] = ur[(q0 + q) * 32 + lane];
        }
#pragma unroll
        for (int q = 0; q < CH; ++q) {
          sdot += dot16(xv[q], wv[q], static_cast<const T*>(nullptr));
          if constexpr (GLU) su += dot16(xv[q], uv[q], static_cast<const T*>(nullptr));
        }
      }
      sdot = warp_sum(sdot);
      float c = gate[i] * silu(sdot);
      if constexpr (GLU) c *= warp_sum(su);
      if (lane == 0) cbuf[i] = c;
    }
  }
  // |U| and the group count: every CTA adds its newly counted ids; the CTA
  // that finishes last writes both
  __syncthreads();
  if (threadIdx.x == 0) {
    atomicAdd(sc.uacc, cta_new);
    __threadfence();
    if (atomicAdd(sc.ctas_done, 1u) == gridDim.x - 1) {
      __threadfence();
      const uint32_t u = atomicAdd(sc.uacc, 0u);
      counts[0] = static_cast<int32_t>(u);
      counts[1] = static_cast<int32_t>((static_cast<int64_t>(u) + B - 1) / B);
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
bool se_ok(const Dims& D) {
  if (D.L < 1 || D.L > 65535 || D.N() > kSeMaxN || se_nv(D) == 0 || D.B > (int64_t(1) << 30))
    return false;
  const int64_t rows = D.N() < D.M() ? D.N() : D.M();  // distinct ids a batch can use
  const int64_t esize = D.dtype == OMNI_F32 ? 4 : 2;
  return rows * D.d * esize * 2 <= kSeRowBudget || D.M() * D.d * esize * 2 <= kSeTaskBudget;
}

// workspace words: the two counters, the bitmap of the ids (all zeroed
// before the call), then c [M] floats, each part on a 256-byte boundary
constexpr size_t kSeBitsOff = 64;
size_t se_bits_words(const Dims& D) { return (static_cast<size_t>(D.N()) + 31) / 32; }
size_t se_cbuf_off(const Dims& D) { return (kSeBitsOff + se_bits_words(D) + 63) / 64 * 64; }

template <typename T, int NV, bool GLU>
cudaError_t launch_se_t(const Dims& D, const void* x, const void* W, const void* V,
                        const int32_t* idx, const float* gate, void* y, uint32_t* ws,
                        int32_t* counts, cudaStream_t s, const void* U) {
  SeScratch sc;
  sc.uacc = ws;
  sc.ctas_done = ws + 1;
  sc.bits = ws + kSeBitsOff;
  float* cbuf = reinterpret_cast<float*>(ws + se_cbuf_off(D));
  const unsigned blocks = static_cast<unsigned>((D.M() + kTaWarps - 1) / kTaWarps);
  OMNI_TRY(launch_k(k_task_act<T, NV, GLU>, blocks, kTaThreads, 0, s, static_cast<const T*>(x),
      static_cast<const T*>(W), static_cast<const T*>(U), idx, gate, static_cast<int>(D.L),
      static_cast<int>(D.K), D.N(), static_cast<int>(D.B), shard_ids(D), cbuf, sc, counts));
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
  return (D.flags & OMNI_FLAG_STAGED_SMALL) == 0 && se_ok(D);
}

size_t sched_exec_ws_words(const Dims& D) { return se_cbuf_off(D) + static_cast<size_t>(D.M()); }

size_t sched_exec_zero_words(const Dims& D) { return kSeBitsOff + se_bits_words(D); }

cudaError_t launch_sched_exec(const Dims& D, const void* x, const void* W, const void* V,
                              const int32_t* idx, const float* gate, void* y, uint32_t* ws,
                              int32_t* counts, cudaStream_t s, const void* U) {
  if (!se_ok(D)) return cudaErrorInvalidValue;
#define OMNI_SE(T_, NV_)                                                               \
  return U != nullptr                                                                  \
             ? launch_se_t<T_, NV_, true>(D, x, W, V, idx, gate, y, ws, counts, s, U)  \
             : launch_se_t<T_, NV_, false>(D, x, W, V, idx, gate, y, ws, counts, s, U);
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
