// Execution of the routed atomic experts.
//
// An atomic expert e is the vector pair (W[e], V[e]) and computes
// sigma(x . W[e]) V[e] with sigma the scalar SiLU ("OmniMoE: An Efficient MoE
// by Orchestrating Atomic Experts at Scale" (gist.science), Technisch
// Overzicht section 2.1).  The layer output of token t is
//   y[t] = sum over its tasks (t, e, g) of g * SiLU(x[t] . W[e]) * V[e].
//
// Expert-centric order (section 2.2 "Grouped GEMM"; the OmniMoE explainer on
// manus.space, Expert-Centric Scheduling, last step): CTA g executes group g
// of the schedule.  Inside a group the tasks are sorted by token, so tasks of
// one token form a run; one warp takes one run, keeps x[t] in shared memory,
// computes the SiLU activations of the run's experts and accumulates
// sum g*h*V[e] in registers, then adds the run's d-vector into the fp32
// accumulator with vector reductions (red.global.add.v4.f32).  The group's
// expert rows are fetched from HBM once and re-read by the group's other runs
// from L2 while the group is in flight.
//
// The activations are scattered, one (token, expert) pair at a time: a
// group's B experts see only a few tokens each, so a dense B x T_g tile would
// multiply the useful work by roughly B and the stage is bound by the
// 2*d*|E_active| parameter bytes, not by arithmetic.  CUDA cores with 16-byte
// coalesced row loads are used instead of tensor cores.
//
// Token-centric order (the ablation the scheduling replaces, section 2.2):
// CTA t gathers the rows of its own K experts; no reductions across CTAs.
#include "common.cuh"
#include "internal.h"

namespace omni {
namespace {

constexpr int kExpWarps = 8;
constexpr int kExpChunk = kExpWarps * 32;  // tasks scanned for pieces per step
constexpr int kPieceMax = 16;              // tasks of one token per piece (one reduction)

// Elements per 16-byte vector.
template <typename T> constexpr int kEpv = 16 / sizeof(T);

// Dot product contribution of one 16-byte vector pair, widened to fp32.
__device__ __forceinline__ float dot_vec(uint4 a, uint4 b, __nv_bfloat16*) {
  return bf16lo(a.x) * bf16lo(b.x) + bf16hi(a.x) * bf16hi(b.x) + bf16lo(a.y) * bf16lo(b.y) +
         bf16hi(a.y) * bf16hi(b.y) + bf16lo(a.z) * bf16lo(b.z) + bf16hi(a.z) * bf16hi(b.z) +
         bf16lo(a.w) * bf16lo(b.w) + bf16hi(a.w) * bf16hi(b.w);
}
__device__ __forceinline__ float dot_vec(uint4 a, uint4 b, float*) {
  return __uint_as_float(a.x) * __uint_as_float(b.x) + __uint_as_float(a.y) * __uint_as_float(b.y) +
         __uint_as_float(a.z) * __uint_as_float(b.z) + __uint_as_float(a.w) * __uint_as_float(b.w);
}
__device__ __forceinline__ void axpy_vec(float c, uint4 v, float* acc, __nv_bfloat16*) {
  acc[0] = fmaf(c, bf16lo(v.x), acc[0]); acc[1] = fmaf(c, bf16hi(v.x), acc[1]);
  acc[2] = fmaf(c, bf16lo(v.y), acc[2]); acc[3] = fmaf(c, bf16hi(v.y), acc[3]);
  acc[4] = fmaf(c, bf16lo(v.z), acc[4]); acc[5] = fmaf(c, bf16hi(v.z), acc[5]);
  acc[6] = fmaf(c, bf16lo(v.w), acc[6]); acc[7] = fmaf(c, bf16hi(v.w), acc[7]);
}
__device__ __forceinline__ void axpy_vec(float c, uint4 v, float* acc, float*) {
  acc[0] = fmaf(c, __uint_as_float(v.x), acc[0]); acc[1] = fmaf(c, __uint_as_float(v.y), acc[1]);
  acc[2] = fmaf(c, __uint_as_float(v.z), acc[2]); acc[3] = fmaf(c, __uint_as_float(v.w), acc[3]);
}

// Round EPV fp32 values to one 16-byte vector of T (bf16: nearest even).
__device__ __forceinline__ uint4 pack_vec(const float* a, __nv_bfloat16*) {
  uint4 r;
  auto p = [](float lo, float hi) {
    const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&v);
  };
  r.x = p(a[0], a[1]); r.y = p(a[2], a[3]); r.z = p(a[4], a[5]); r.w = p(a[6], a[7]);
  return r;
}
__device__ __forceinline__ uint4 pack_vec(const float* a, float*) {
  return make_uint4(__float_as_uint(a[0]), __float_as_uint(a[1]), __float_as_uint(a[2]),
                    __float_as_uint(a[3]));
}

// Grouped execution over the schedule, taken as one task list in schedule
// order (group after group; inside a group by token, then expert).  A CTA
// scans chunks of kExpChunk consecutive tasks; a piece is a maximal stretch of
// one token's tasks inside a chunk, at most kPieceMax long; each warp executes
// pieces: x[t] is read once, every task reads W[e] and V[e] (a group's rows
// come from HBM once and are re-read by its other pieces from L2), and the
// piece adds its sum g*SiLU(x[t].W[e])*V[e] to the fp32 row y[t] with 16-byte
// vector reductions.  NV > 0: d = NV * 32 * (16 / sizeof(T)), x[t] lives in
// registers; NV == 0: any d that is a multiple of 16 bytes, x[t] in shared
// memory.  Every index read from memory is range-checked before it is used
// (a bad one sets OMNI_DEV_BAD_INDEX and the task is skipped).
template <typename T, int NV>
__global__ void __launch_bounds__(kExpWarps * 32)
    k_expert_pieces(const T* __restrict__ x, const T* __restrict__ W, const T* __restrict__ V,
                    const int32_t* __restrict__ task_token,
                    const int32_t* __restrict__ task_expert,
                    const float* __restrict__ task_gate, int64_t M, int64_t L, int64_t N, int d,
                    float* __restrict__ yacc, int32_t* status) {
  constexpr int EPV = kEpv<T>;
  extern __shared__ __align__(16) uint8_t smem[];  // NV == 0: kExpWarps rows of x
  __shared__ int pstart[kExpChunk + 1];
  __shared__ int wcnt[kExpWarps];
  __shared__ int npieces;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nvec = d / EPV;  // 16-byte vectors per row
  uint4* xs = reinterpret_cast<uint4*>(smem) + static_cast<size_t>(warp) * nvec;
  const int64_t nchunks = (M + kExpChunk - 1) / kExpChunk;
  for (int64_t ch = blockIdx.x; ch < nchunks; ch += gridDim.x) {
    const int64_t c0 = ch * kExpChunk;
    const int64_t c1 = (M - c0 < kExpChunk) ? M : c0 + kExpChunk;
    {
      const int64_t i = c0 + threadIdx.x;
      bool st = false;
      if (i < c1) {
        const int64_t off = i - c0;
        st = (off == 0) || task_token[i] != task_token[i - 1];
        if (!st) {
          // cut a long run every kPieceMax tasks (counted from the run start)
          int64_t k0 = i - 1;
          while (k0 > c0 && task_token[k0 - 1] == task_token[i]) --k0;
          st = ((i - k0) % kPieceMax) == 0;
        }
      }
      const uint32_t m = __ballot_sync(0xffffffffu, st);
      if (lane == 0) wcnt[warp] = __popc(m);
      __syncthreads();
      int wbase = 0;
      for (int w = 0; w < warp; ++w) wbase += wcnt[w];
      const int pos = wbase + __popc(m & lanemask_lt());
      if (st && pos < kExpChunk) pstart[pos] = static_cast<int>(i - c0);
      if (threadIdx.x == kExpChunk - 1) {
        const int n = wbase + __popc(m);
        npieces = n;
        pstart[n < kExpChunk ? n : kExpChunk] = static_cast<int>(c1 - c0);
      }
    }
    __syncthreads();
    const int np = npieces;
    for (int p = warp; p < np; p += kExpWarps) {
      const int pa = pstart[p], pb = pstart[p + 1];
      if (pa < 0 || pb > kExpChunk || pa >= pb) {
        if (lane == 0) raise_status(status, OMNI_DEV_BAD_INDEX);
        continue;
      }
      const int64_t a = c0 + pa, b = c0 + pb;
      const int64_t t = task_token[a];
      if (t < 0 || t >= L) {
        if (lane == 0) raise_status(status, OMNI_DEV_BAD_INDEX);
        continue;
      }
      const uint4* xr = reinterpret_cast<const uint4*>(x + t * d);
      // this lane's task of the piece (pieces are <= kPieceMax <= 32 long)
      int64_t my_e = -1;
      float my_g = 0.0f;
      if (lane < b - a) {
        my_e = task_expert[a + lane];
        my_g = task_gate[a + lane];
        if (my_e < 0 || my_e >= N) {
          raise_status(status, OMNI_DEV_BAD_INDEX);
          my_e = -1;
        }
      }
      const int nt = static_cast<int>(b - a);
      if constexpr (NV > 0) {
        uint4 xv[NV];
#pragma unroll
        for (int v = 0; v < NV; ++v) xv[v] = xr[v * 32 + lane];
        float acc[NV * EPV];
#pragma unroll
        for (int u = 0; u < NV * EPV; ++u) acc[u] = 0.0f;
        for (int j = 0; j < nt; ++j) {
          const int64_t e = __shfl_sync(0xffffffffu, my_e, j);
          const float gj = __shfl_sync(0xffffffffu, my_g, j);
          if (e < 0 || e >= N) continue;  // warp-uniform
          const uint4* wr = reinterpret_cast<const uint4*>(W + e * d);
          const uint4* vr = reinterpret_cast<const uint4*>(V + e * d);
          uint4 wv[NV], vv[NV];
#pragma unroll
          for (int v = 0; v < NV; ++v) wv[v] = wr[v * 32 + lane];
#pragma unroll
          for (int v = 0; v < NV; ++v) vv[v] = vr[v * 32 + lane];
          float s = 0.0f;
#pragma unroll
          for (int v = 0; v < NV; ++v) s += dot_vec(xv[v], wv[v], static_cast<T*>(nullptr));
          s = warp_sum(s);
          const float c = gj * silu(s);
#pragma unroll
          for (int v = 0; v < NV; ++v) axpy_vec(c, vv[v], acc + v * EPV, static_cast<T*>(nullptr));
        }
        float* yr = yacc + t * d;
#pragma unroll
        for (int v = 0; v < NV; ++v) {
          float* q = yr + static_cast<int64_t>(v * 32 + lane) * EPV;
#pragma unroll
          for (int u = 0; u < EPV; u += 4)
            red_add_v4(q + u, acc[v * EPV + u], acc[v * EPV + u + 1], acc[v * EPV + u + 2],
                       acc[v * EPV + u + 3]);
        }
      } else {
        // generic d: x[t] in this warp's shared-memory row
        for (int v = lane; v < nvec; v += 32) xs[v] = xr[v];
        __syncwarp();
        float my_c = 0.0f;
        for (int j = 0; j < nt; ++j) {
          const int64_t e = __shfl_sync(0xffffffffu, my_e, j);
          float s = 0.0f;
          if (e >= 0 && e < N) {  // warp-uniform; the loop below holds no shuffle
            const uint4* wr = reinterpret_cast<const uint4*>(W + e * d);
            for (int v = lane; v < nvec; v += 32) s += dot_vec(xs[v], wr[v], static_cast<T*>(nullptr));
          }
          s = warp_sum(s);
          if (lane == j) my_c = (e >= 0) ? my_g * silu(s) : 0.0f;
        }
        float* yr = yacc + t * d;
        // the trip count is the same for every lane: the shuffles below need
        // all 32 lanes; only the memory accesses are predicated
        for (int v0 = 0; v0 < nvec; v0 += 32) {
          const int v = v0 + lane;
          const bool act = v < nvec;
          float acc[EPV];
#pragma unroll
          for (int u = 0; u < EPV; ++u) acc[u] = 0.0f;
          for (int j = 0; j < nt; ++j) {
            const int64_t e = __shfl_sync(0xffffffffu, my_e, j);
            const float c = __shfl_sync(0xffffffffu, my_c, j);
            if (!act || e < 0 || e >= N) continue;
            const uint4* vr = reinterpret_cast<const uint4*>(V + e * d);
            axpy_vec(c, vr[v], acc, static_cast<T*>(nullptr));
          }
          if (act) {
#pragma unroll
            for (int u = 0; u < EPV; u += 4)
              red_add_v4(yr + static_cast<int64_t>(v) * EPV + u, acc[u], acc[u + 1], acc[u + 2],
                         acc[u + 3]);
          }
        }
        __syncwarp();
      }
    }
    __syncthreads();
  }
}

template <typename T>
__global__ void __launch_bounds__(256) k_cast(const float* __restrict__ src, T* __restrict__ dst,
                                              int64_t n) {
  const int64_t i = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) * 8;
  if (i >= n) return;
  const float4 a = *reinterpret_cast<const float4*>(src + i);
  const float4 b = *reinterpret_cast<const float4*>(src + i + 4);
  const float f[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
  for (int u = 0; u < 8; ++u) dst[i + u] = from_float<T>(f[u]);
}

constexpr int kTokThreads = 128;

// Token-centric execution: CTA t gathers the rows of its own K experts.
// Phase 1: each warp takes tasks q = warp, warp+4, ... and computes
// c_q = gate * SiLU(x[t] . W[e_q]) (x[t] as 16-byte vectors in shared memory);
// phase 2: each thread owns 16-byte vectors of the output row and sums
// c_q * V[e_q] over the K tasks.  No reductions across CTAs.
template <typename T>
__global__ void __launch_bounds__(kTokThreads)
    k_token_centric(const T* __restrict__ x, const T* __restrict__ W, const T* __restrict__ V,
                    const int32_t* __restrict__ idx, const float* __restrict__ gate, int K, int d,
                    int64_t N, T* __restrict__ y, int32_t* status) {
  constexpr int EPV = kEpv<T>;
  extern __shared__ __align__(16) uint8_t smem[];
  const int nvec = d / EPV;
  uint4* xs = reinterpret_cast<uint4*>(smem);
  float* cq = reinterpret_cast<float*>(xs + nvec);
  int64_t* es = reinterpret_cast<int64_t*>(cq + ((K + 3) & ~3));
  const int64_t t = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint4* xr = reinterpret_cast<const uint4*>(x + t * d);
  for (int v = threadIdx.x; v < nvec; v += kTokThreads) xs[v] = xr[v];
  for (int q = threadIdx.x; q < K; q += kTokThreads) {
    int64_t e = idx[t * K + q];
    if (e < 0 || e >= N) {
      raise_status(status, OMNI_DEV_BAD_INDEX);
      e = -1;
    }
    es[q] = e;
  }
  __syncthreads();
  for (int q = warp; q < K; q += kTokThreads / 32) {
    const int64_t e = es[q];
    float s = 0.0f;
    if (e >= 0) {
      const uint4* wr = reinterpret_cast<const uint4*>(W + e * d);
      for (int v = lane; v < nvec; v += 32) s += dot_vec(xs[v], wr[v], static_cast<T*>(nullptr));
    }
    s = warp_sum(s);
    if (lane == 0) cq[q] = (e >= 0) ? gate[t * K + q] * silu(s) : 0.0f;
  }
  __syncthreads();
  uint4* yr = reinterpret_cast<uint4*>(y + t * d);
  for (int v = threadIdx.x; v < nvec; v += kTokThreads) {
    float acc[EPV];
#pragma unroll
    for (int u = 0; u < EPV; ++u) acc[u] = 0.0f;
    for (int q = 0; q < K; ++q) {
      const int64_t e = es[q];
      if (e < 0) continue;
      const uint4* vr = reinterpret_cast<const uint4*>(V + e * d);
      axpy_vec(cq[q], vr[v], acc, static_cast<T*>(nullptr));
    }
    yr[v] = pack_vec(acc, static_cast<T*>(nullptr));
  }
}

}  // namespace

size_t expert_ws_bytes(const Dims& D) {
  if (D.dtype == OMNI_F32) return 0;
  return static_cast<size_t>(D.L) * D.d * sizeof(float);
}

template <typename T, int NV>
cudaError_t launch_pieces(const Dims& D, const void* x, const void* W, const void* V,
                          const int32_t* tt, const int32_t* te, const float* tg, float* acc,
                          int32_t* status, cudaStream_t s) {
  const size_t smem = NV > 0 ? 0 : static_cast<size_t>(kExpWarps) * D.d * sizeof(T);
  cudaError_t err = cudaFuncSetAttribute(k_expert_pieces<T, NV>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
  if (err != cudaSuccess) return err;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t nchunks = (D.M() + kExpChunk - 1) / kExpChunk;
  const int64_t cap = static_cast<int64_t>(sms) * 8;
  const unsigned grid = static_cast<unsigned>(nchunks < cap ? nchunks : cap);
  k_expert_pieces<T, NV><<<grid, kExpWarps * 32, smem, s>>>(
      static_cast<const T*>(x), static_cast<const T*>(W), static_cast<const T*>(V), tt, te, tg,
      D.M(), D.L, D.N(), static_cast<int>(D.d), acc, status);
  return cudaGetLastError();
}

template <typename T>
cudaError_t dispatch_pieces(const Dims& D, const void* x, const void* W, const void* V,
                            const int32_t* tt, const int32_t* te, const float* tg, float* acc,
                            int32_t* status, cudaStream_t s) {
  constexpr int row = 32 * kEpv<T>;  // elements covered by one vector per lane
  switch (D.d == row * 8 ? 8 : D.d == row * 4 ? 4 : D.d == row * 2 ? 2 : D.d == row ? 1 : 0) {
    case 8: return launch_pieces<T, 8>(D, x, W, V, tt, te, tg, acc, status, s);
    case 4: return launch_pieces<T, 4>(D, x, W, V, tt, te, tg, acc, status, s);
    case 2: return launch_pieces<T, 2>(D, x, W, V, tt, te, tg, acc, status, s);
    case 1: return launch_pieces<T, 1>(D, x, W, V, tt, te, tg, acc, status, s);
    default: return launch_pieces<T, 0>(D, x, W, V, tt, te, tg, acc, status, s);
  }
}

cudaError_t launch_expert(const Dims& D, const void* x, const void* W, const void* V,
                          const int32_t* task_token, const int32_t* task_expert,
                          const float* task_gate, const int32_t* group_off,
                          const int32_t* counts, void* y, void* ws, cudaStream_t s) {
  (void)group_off;
  if (D.L == 0) return cudaSuccess;
  const bool f32 = D.dtype == OMNI_F32;
  float* acc = f32 ? static_cast<float*>(y) : static_cast<float*>(ws);
  const size_t ybytes = static_cast<size_t>(D.L) * D.d * sizeof(float);
  cudaError_t err = cudaMemsetAsync(acc, 0, ybytes, s);
  if (err != cudaSuccess) return err;
  int32_t* status = const_cast<int32_t*>(counts) + 2;
  err = f32 ? dispatch_pieces<float>(D, x, W, V, task_token, task_expert, task_gate, acc, status, s)
            : dispatch_pieces<__nv_bfloat16>(D, x, W, V, task_token, task_expert, task_gate, acc,
                                             status, s);
  if (err != cudaSuccess || f32) return err;
  const int64_t n = D.L * D.d;
  k_cast<__nv_bfloat16><<<static_cast<unsigned>((n / 8 + 255) / 256), 256, 0, s>>>(
      acc, static_cast<__nv_bfloat16*>(y), n);
  return cudaGetLastError();
}

cudaError_t launch_token(const Dims& D, const void* x, const void* W, const void* V,
                         const int32_t* idx, const float* gate, void* y, int32_t* status,
                         cudaStream_t s) {
  if (D.L == 0) return cudaSuccess;
  const size_t esz = D.dtype == OMNI_F32 ? 4 : 2;
  const size_t smem = static_cast<size_t>(D.d) * esz +
                      static_cast<size_t>((D.K + 3) & ~3) * sizeof(float) +
                      static_cast<size_t>(D.K) * sizeof(int64_t);
  cudaError_t err;
  if (D.dtype == OMNI_F32) {
    err = cudaFuncSetAttribute(k_token_centric<float>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (err != cudaSuccess) return err;
    k_token_centric<float><<<static_cast<unsigned>(D.L), kTokThreads, smem, s>>>(
        static_cast<const float*>(x), static_cast<const float*>(W), static_cast<const float*>(V),
        idx, gate, static_cast<int>(D.K), static_cast<int>(D.d), D.N(), static_cast<float*>(y),
        status);
  } else {
    err = cudaFuncSetAttribute(k_token_centric<__nv_bfloat16>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (err != cudaSuccess) return err;
    k_token_centric<__nv_bfloat16><<<static_cast<unsigned>(D.L), kTokThreads, smem, s>>>(
        static_cast<const __nv_bfloat16*>(x), static_cast<const __nv_bfloat16*>(W),
        static_cast<const __nv_bfloat16*>(V), idx, gate, static_cast<int>(D.K),
        static_cast<int>(D.d), D.N(), static_cast<__nv_bfloat16*>(y), status);
  }
  return cudaGetLastError();
}

}  // namespace omni
