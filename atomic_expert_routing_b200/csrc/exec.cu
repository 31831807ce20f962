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
constexpr int kExpChunk = kExpWarps * 32;  // tasks scanned for run starts per step

template <typename T>
__global__ void __launch_bounds__(kExpWarps * 32)
    k_expert_grouped(const T* __restrict__ x, const T* __restrict__ W, const T* __restrict__ V,
                     const int32_t* __restrict__ task_token,
                     const int32_t* __restrict__ task_expert,
                     const float* __restrict__ task_gate, const int32_t* __restrict__ group_off,
                     const int32_t* __restrict__ counts, int64_t N, int d,
                     float* __restrict__ yacc, int32_t* status) {
  extern __shared__ __align__(16) uint8_t smem[];
  __shared__ int starts[kExpChunk + 1];
  __shared__ int nruns;
  __shared__ int wcnt[kExpWarps];
  const int g = blockIdx.x;
  if (g >= counts[1]) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  T* xs = reinterpret_cast<T*>(smem) + static_cast<size_t>(warp) * d;
  const int off0 = group_off[g], off1 = group_off[g + 1];
  for (int c0 = off0; c0 < off1; c0 += kExpChunk) {
    const int c1 = min(off1, c0 + kExpChunk);
    {
      // run starts of this chunk, compacted in task order
      const int i = c0 + threadIdx.x;
      const bool st = i < c1 && (i == c0 || task_token[i] != task_token[i - 1]);
      const uint32_t m = __ballot_sync(0xffffffffu, st);
      if (lane == 0) wcnt[warp] = __popc(m);
      __syncthreads();
      int wbase = 0;
      for (int w = 0; w < warp; ++w) wbase += wcnt[w];
      if (st) starts[wbase + __popc(m & lanemask_lt())] = i;
      if (threadIdx.x == kExpChunk - 1) {
        const int n = wbase + __popc(m);
        nruns = n;
        starts[n] = c1;
      }
    }
    __syncthreads();
    const int n = nruns;
    for (int r = warp; r < n; r += kExpWarps) {
      const int a = starts[r], b = starts[r + 1];
      const int64_t t = task_token[a];
      const T* xr = x + t * d;
      for (int m = lane * 8; m < d; m += 256)
        *reinterpret_cast<uint4*>(reinterpret_cast<uint8_t*>(xs + m)) =
            *reinterpret_cast<const uint4*>(reinterpret_cast<const uint8_t*>(xr + m));
      if (sizeof(T) == 4)
        for (int m = lane * 8 + 4; m < d; m += 256)
          *reinterpret_cast<uint4*>(reinterpret_cast<uint8_t*>(xs + m)) =
              *reinterpret_cast<const uint4*>(reinterpret_cast<const uint8_t*>(xr + m));
      __syncwarp();
      for (int j0 = a; j0 < b; j0 += 32) {
        const int nb = min(32, b - j0);
        int64_t my_e = 0;
        float my_g = 0.0f;
        if (lane < nb) {
          my_e = task_expert[j0 + lane];
          my_g = task_gate[j0 + lane];
          if (my_e < 0 || my_e >= N) {
            raise_status(status, OMNI_DEV_BAD_INDEX);
            my_e = 0;
            my_g = 0.0f;
          }
        }
        // activations h = SiLU(x[t] . W[e]) of the batch
        float my_gh = 0.0f;
        for (int jj = 0; jj < nb; ++jj) {
          const int64_t e = __shfl_sync(0xffffffffu, my_e, jj);
          const T* wr = W + e * d;
          float s = 0.0f;
          for (int m = lane * 8; m < d; m += 256) {
            float w8[8], x8[8];
            load8(wr + m, w8);
            load8(xs + m, x8);
#pragma unroll
            for (int u = 0; u < 8; ++u) s = fmaf(w8[u], x8[u], s);
          }
          s = warp_sum(s);
          const float gj = __shfl_sync(0xffffffffu, my_g, jj);
          if (lane == jj) my_gh = gj * silu(s);
        }
        // sum of g*h*V[e] over the batch, added into y[t]
        float* yr = yacc + t * d;
        for (int m = lane * 8; m < d; m += 256) {
          float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
          for (int jj = 0; jj < nb; ++jj) {
            const int64_t e = __shfl_sync(0xffffffffu, my_e, jj);
            const float c = __shfl_sync(0xffffffffu, my_gh, jj);
            float v8[8];
            load8(V + e * d + m, v8);
#pragma unroll
            for (int u = 0; u < 8; ++u) acc[u] = fmaf(c, v8[u], acc[u]);
          }
          red_add_v4(yr + m, acc[0], acc[1], acc[2], acc[3]);
          red_add_v4(yr + m + 4, acc[4], acc[5], acc[6], acc[7]);
        }
      }
      __syncwarp();
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

template <typename T>
__global__ void __launch_bounds__(kTokThreads)
    k_token_centric(const T* __restrict__ x, const T* __restrict__ W, const T* __restrict__ V,
                    const int32_t* __restrict__ idx, const float* __restrict__ gate, int K, int d,
                    int64_t N, T* __restrict__ y, int32_t* status) {
  extern __shared__ __align__(16) uint8_t smem[];
  T* xs = reinterpret_cast<T*>(smem);
  float* gh = reinterpret_cast<float*>(smem + ((static_cast<size_t>(d) * sizeof(T) + 15) & ~size_t(15)));
  int64_t* es = reinterpret_cast<int64_t*>(gh + ((K + 3) & ~3));
  const int64_t t = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int m = threadIdx.x; m < d; m += kTokThreads) xs[m] = x[t * d + m];
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
    if (e >= 0)
      for (int m = lane * 8; m < d; m += 256) {
        float w8[8], x8[8];
        load8(W + e * d + m, w8);
        load8(xs + m, x8);
#pragma unroll
        for (int u = 0; u < 8; ++u) s = fmaf(w8[u], x8[u], s);
      }
    s = warp_sum(s);
    if (lane == 0) gh[q] = (e >= 0) ? gate[t * K + q] * silu(s) : 0.0f;
  }
  __syncthreads();
  for (int m = threadIdx.x * 8; m < d; m += kTokThreads * 8) {
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int q = 0; q < K; ++q) {
      const int64_t e = es[q];
      if (e < 0) continue;
      const float c = gh[q];
      float v8[8];
      load8(V + e * d + m, v8);
#pragma unroll
      for (int u = 0; u < 8; ++u) acc[u] = fmaf(c, v8[u], acc[u]);
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) y[t * d + m + u] = from_float<T>(acc[u]);
  }
}

}  // namespace

size_t expert_ws_bytes(const Dims& D) {
  if (D.dtype == OMNI_F32) return 0;
  return static_cast<size_t>(D.L) * D.d * sizeof(float);
}

cudaError_t launch_expert(const Dims& D, const void* x, const void* W, const void* V,
                          const int32_t* task_token, const int32_t* task_expert,
                          const float* task_gate, const int32_t* group_off,
                          const int32_t* counts, void* y, void* ws, cudaStream_t s) {
  if (D.L == 0) return cudaSuccess;
  const bool f32 = D.dtype == OMNI_F32;
  float* acc = f32 ? static_cast<float*>(y) : static_cast<float*>(ws);
  const size_t ybytes = static_cast<size_t>(D.L) * D.d * sizeof(float);
  cudaError_t err = cudaMemsetAsync(acc, 0, ybytes, s);
  if (err != cudaSuccess) return err;
  const size_t esz = f32 ? 4 : 2;
  const size_t smem = static_cast<size_t>(kExpWarps) * D.d * esz;
  const unsigned grid = static_cast<unsigned>(D.gmax());
  int32_t* status = const_cast<int32_t*>(counts) + 2;
  if (f32) {
    err = cudaFuncSetAttribute(k_expert_grouped<float>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (err != cudaSuccess) return err;
    k_expert_grouped<float><<<grid, kExpWarps * 32, smem, s>>>(
        static_cast<const float*>(x), static_cast<const float*>(W), static_cast<const float*>(V),
        task_token, task_expert, task_gate, group_off, counts, D.N(), static_cast<int>(D.d), acc,
        status);
  } else {
    err = cudaFuncSetAttribute(k_expert_grouped<__nv_bfloat16>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (err != cudaSuccess) return err;
    k_expert_grouped<__nv_bfloat16><<<grid, kExpWarps * 32, smem, s>>>(
        static_cast<const __nv_bfloat16*>(x), static_cast<const __nv_bfloat16*>(W),
        static_cast<const __nv_bfloat16*>(V), task_token, task_expert, task_gate, group_off,
        counts, D.N(), static_cast<int>(D.d), acc, status);
    err = cudaGetLastError();
    if (err != cudaSuccess) return err;
    const int64_t n = D.L * D.d;
    k_cast<__nv_bfloat16><<<static_cast<unsigned>((n / 8 + 255) / 256), 256, 0, s>>>(
        acc, static_cast<__nv_bfloat16*>(y), n);
  }
  return cudaGetLastError();
}

cudaError_t launch_token(const Dims& D, const void* x, const void* W, const void* V,
                         const int32_t* idx, const float* gate, void* y, int32_t* status,
                         cudaStream_t s) {
  if (D.L == 0) return cudaSuccess;
  const size_t esz = D.dtype == OMNI_F32 ? 4 : 2;
  const size_t smem = ((static_cast<size_t>(D.d) * esz + 15) & ~size_t(15)) +
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
