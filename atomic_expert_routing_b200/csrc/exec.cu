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

constexpr int kExpThreads = 128;  // 4 warps per CTA, each executing its own task slice

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
// order (group after group; inside a group by token, then expert).  Warp w
// owns the slice of S consecutive tasks [w*S, (w+1)*S); inside its slice a
// piece is a maximal stretch of one token's tasks.  For every piece the warp
// reads x[t] once, and for every task of the piece the rows W[e] and V[e]
// (issued together; a group's rows come from HBM once and are re-read by its
// other pieces from L2 while the group is in flight), computes
// c = g * SiLU(x[t] . W[e]) and accumulates c * V[e] in registers; the piece
// then adds its d-vector to the fp32 row y[t] with 16-byte vector reductions.
// NV > 0: d = NV * 32 * (16 / sizeof(T)), x[t] held in registers; NV == 0: any
// d that is a multiple of 16 bytes (x[t] streamed from L2 per task).  Every
// index read from memory is range-checked before use (a bad one sets
// OMNI_DEV_BAD_INDEX and the task is skipped).  All warp shuffles sit at
// warp-uniform points.
template <typename T, int NV>
__global__ void __launch_bounds__(kExpThreads, (NV >= 8 ? 3 : 4))
    k_expert_slices(const T* __restrict__ x, const T* __restrict__ W, const T* __restrict__ V,
                    const int32_t* __restrict__ task_token,
                    const int32_t* __restrict__ task_expert,
                    const float* __restrict__ task_gate, int64_t M, int64_t L, int64_t N, int d,
                    int S, float* __restrict__ yacc, int32_t* status) {
  constexpr int EPV = kEpv<T>;
  const int lane = threadIdx.x & 31;
  const int64_t wid = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t a0 = wid * S;
  if (a0 >= M) return;  // whole warp
  const int n = static_cast<int>(M - a0 < S ? M - a0 : S);
  const int nvec = d / EPV;
  // one task per lane (S <= 32): token, expert, gate
  int64_t my_t = -1, my_e = -1;
  float my_g = 0.0f;
  if (lane < n) {
    my_t = task_token[a0 + lane];
    my_e = task_expert[a0 + lane];
    my_g = task_gate[a0 + lane];
    if (my_t < 0 || my_t >= L || my_e < 0 || my_e >= N) {
      raise_status(status, OMNI_DEV_BAD_INDEX);
      my_e = -1;
    }
  }
  const int64_t prev_t = __shfl_up_sync(0xffffffffu, my_t, 1);
  const bool start = lane < n && (lane == 0 || prev_t != my_t);
  uint32_t starts = __ballot_sync(0xffffffffu, start);
  while (starts) {
    const int p = __ffs(starts) - 1;
    starts &= starts - 1;
    const int q = starts ? __ffs(starts) - 1 : n;  // piece = lanes [p, q)
    const int64_t t = __shfl_sync(0xffffffffu, my_t, p);
    if (t < 0 || t >= L) continue;  // warp-uniform
    float* yr = yacc + t * d;
    if constexpr (NV > 0) {
      const uint4* xr = reinterpret_cast<const uint4*>(x + t * d);
      uint4 xv[NV];
#pragma unroll
      for (int v = 0; v < NV; ++v) xv[v] = xr[v * 32 + lane];
      float acc[NV * EPV];
#pragma unroll
      for (int u = 0; u < NV * EPV; ++u) acc[u] = 0.0f;
      for (int j = p; j < q; ++j) {
        const int64_t e = __shfl_sync(0xffffffffu, my_e, j);
        const float gj = __shfl_sync(0xffffffffu, my_g, j);
        if (e < 0) continue;  // warp-uniform
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
#pragma unroll
      for (int v = 0; v < NV; ++v) {
        float* o = yr + static_cast<int64_t>(v * 32 + lane) * EPV;
#pragma unroll
        for (int u = 0; u < EPV; u += 4)
          red_add_v4(o + u, acc[v * EPV + u], acc[v * EPV + u + 1], acc[v * EPV + u + 2],
                     acc[v * EPV + u + 3]);
      }
    } else {
      // generic d: activations first (x re-read from L2 per task), then the
      // value rows vector block by vector block; trip counts are warp-uniform
      const uint4* xr = reinterpret_cast<const uint4*>(x + t * d);
      float my_c = 0.0f;
      for (int j = p; j < q; ++j) {
        const int64_t e = __shfl_sync(0xffffffffu, my_e, j);
        float sacc = 0.0f;
        if (e >= 0) {  // warp-uniform; no shuffle inside
          const uint4* wr = reinterpret_cast<const uint4*>(W + e * d);
          for (int v = lane; v < nvec; v += 32) sacc += dot_vec(xr[v], wr[v], static_cast<T*>(nullptr));
        }
        sacc = warp_sum(sacc);
        const float gj = __shfl_sync(0xffffffffu, my_g, j);
        if (lane == j) my_c = (e >= 0) ? gj * silu(sacc) : 0.0f;
      }
      for (int v0 = 0; v0 < nvec; v0 += 32) {
        const int v = v0 + lane;
        const bool act = v < nvec;
        float acc[EPV];
#pragma unroll
        for (int u = 0; u < EPV; ++u) acc[u] = 0.0f;
        for (int j = p; j < q; ++j) {
          const int64_t e = __shfl_sync(0xffffffffu, my_e, j);
          const float c = __shfl_sync(0xffffffffu, my_c, j);
          if (!act || e < 0) continue;
          axpy_vec(c, reinterpret_cast<const uint4*>(V + e * d)[v], acc, static_cast<T*>(nullptr));
        }
        if (act) {
#pragma unroll
          for (int u = 0; u < EPV; u += 4)
            red_add_v4(yr + static_cast<int64_t>(v) * EPV + u, acc[u], acc[u + 1], acc[u + 2],
                       acc[u + 3]);
        }
      }
    }
  }
}

// L2 eviction policies (createpolicy): rows of W and V are streamed once
// (evict first), the fp32 accumulator y is re-used by many pieces (evict last).
__device__ __forceinline__ uint64_t policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ uint64_t policy_evict_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint64_t pol) {
  asm volatile("cp.async.cg.shared.global.L2::cache_hint [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
               "l"(pol)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void red_add_v4_keep(float* addr, float a, float b, float c, float d,
                                                uint64_t pol) {
  asm volatile("red.global.add.L2::cache_hint.v4.f32 [%0], {%1, %2, %3, %4}, %5;" ::"l"(addr),
               "f"(a), "f"(b), "f"(c), "f"(d), "l"(pol)
               : "memory");
}

constexpr int kAsyncWarps = 8;

// The same grouped execution as k_expert_slices for d = NV * 32 * (16 /
// sizeof(T)), with the row traffic decoupled from the arithmetic: every warp
// streams the W and V rows of its next R-1 tasks into its own shared-memory
// ring with cp.async (each lane copies, and later reads, only its own 16-byte
// vectors, so no cross-lane synchronisation is needed), prefetches x of the
// next piece into registers one task ahead, and computes the current task
// from shared memory.  Warps run a grid-stride loop over task slices; the
// pipeline restarts at every slice.
template <typename T, int NV, int R>
__global__ void __launch_bounds__(kAsyncWarps * 32, 1)
    k_expert_async(const T* __restrict__ x, const T* __restrict__ W, const T* __restrict__ V,
                   const int32_t* __restrict__ task_token,
                   const int32_t* __restrict__ task_expert,
                   const float* __restrict__ task_gate, int64_t M, int64_t L, int64_t N, int d,
                   int S, int64_t nslices, float* __restrict__ yacc, int32_t* status) {
  constexpr int EPV = kEpv<T>;
  constexpr int SLOT = 2 * NV * 32;  // uint4 per ring slot: W vectors, then V vectors
  extern __shared__ __align__(16) uint4 ring[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint4* wring = ring + static_cast<size_t>(warp) * R * SLOT;
  const uint32_t wring_s = static_cast<uint32_t>(__cvta_generic_to_shared(wring));
  const uint64_t pol_stream = policy_evict_first();
  const uint64_t pol_keep = policy_evict_last();
  const int64_t nw = static_cast<int64_t>(gridDim.x) * kAsyncWarps;
  for (int64_t sl = static_cast<int64_t>(blockIdx.x) * kAsyncWarps + warp; sl < nslices; sl += nw) {
    const int64_t a0 = sl * S;
    const int n = static_cast<int>(M - a0 < S ? M - a0 : S);
    int64_t my_t = -1, my_e = -1;
    float my_g = 0.0f;
    if (lane < n) {
      my_t = task_token[a0 + lane];
      my_e = task_expert[a0 + lane];
      my_g = task_gate[a0 + lane];
      if (my_t < 0 || my_t >= L || my_e < 0 || my_e >= N) {
        raise_status(status, OMNI_DEV_BAD_INDEX);
        my_e = -1;
        my_t = -1;
      }
    }
    const int64_t prev_t = __shfl_up_sync(0xffffffffu, my_t, 1);
    const int64_t next_t = __shfl_down_sync(0xffffffffu, my_t, 1);
    const uint32_t starts = __ballot_sync(0xffffffffu, lane < n && (lane == 0 || prev_t != my_t));
    const uint32_t ends = __ballot_sync(0xffffffffu, lane < n && (lane == n - 1 || next_t != my_t));

    // issue the row copies of task j into slot j % R (one commit group per task)
    auto issue = [&](int j) {
      if (j < n) {
        const int64_t e = __shfl_sync(0xffffffffu, my_e, j);
        if (e >= 0) {
          const uint4* wr = reinterpret_cast<const uint4*>(W + e * d);
          const uint4* vr = reinterpret_cast<const uint4*>(V + e * d);
          const uint32_t base = wring_s + static_cast<uint32_t>((j % R) * SLOT) * 16u;
#pragma unroll
          for (int v = 0; v < NV; ++v) {
            cp_async16(base + static_cast<uint32_t>(v * 32 + lane) * 16u, wr + v * 32 + lane, pol_stream);
            cp_async16(base + static_cast<uint32_t>((NV + v) * 32 + lane) * 16u, vr + v * 32 + lane,
                       pol_stream);
          }
        }
      }
      cp_async_commit();
    };
#pragma unroll
    for (int j = 0; j < R - 1; ++j) issue(j);

    uint4 xc[NV], xn[NV];
    {
      const int64_t t0 = __shfl_sync(0xffffffffu, my_t, 0);
      const uint4* xr = reinterpret_cast<const uint4*>(x + (t0 < 0 ? 0 : t0) * d);
#pragma unroll
      for (int v = 0; v < NV; ++v) xn[v] = xr[v * 32 + lane];
    }
    float acc[NV * EPV];
    for (int j = 0; j < n; ++j) {
      issue(j + R - 1);
      const bool st = (starts >> j) & 1u;
      if (st) {
#pragma unroll
        for (int v = 0; v < NV; ++v) xc[v] = xn[v];
#pragma unroll
        for (int u = 0; u < NV * EPV; ++u) acc[u] = 0.0f;
        // x of the next piece, one task ahead
        const uint32_t later = starts & ~((2u << j) - 1u);
        if (later) {
          const int jn = __ffs(later) - 1;
          const int64_t tn = __shfl_sync(0xffffffffu, my_t, jn);
          const uint4* xr = reinterpret_cast<const uint4*>(x + (tn < 0 ? 0 : tn) * d);
#pragma unroll
          for (int v = 0; v < NV; ++v) xn[v] = xr[v * 32 + lane];
        }
      }
      cp_async_wait<R - 1>();
      const int64_t e = __shfl_sync(0xffffffffu, my_e, j);
      const float gj = __shfl_sync(0xffffffffu, my_g, j);
      const int64_t t = __shfl_sync(0xffffffffu, my_t, j);
      if (e >= 0) {  // warp-uniform
        const uint4* slot = wring + (j % R) * SLOT;
        float sdot = 0.0f;
#pragma unroll
        for (int v = 0; v < NV; ++v) sdot += dot_vec(xc[v], slot[v * 32 + lane], static_cast<T*>(nullptr));
        sdot = warp_sum(sdot);
        const float c = gj * silu(sdot);
#pragma unroll
        for (int v = 0; v < NV; ++v)
          axpy_vec(c, slot[(NV + v) * 32 + lane], acc + v * EPV, static_cast<T*>(nullptr));
      }
      if (((ends >> j) & 1u) && t >= 0) {
        float* yr = yacc + t * d;
#pragma unroll
        for (int v = 0; v < NV; ++v) {
          float* o = yr + static_cast<int64_t>(v * 32 + lane) * EPV;
#pragma unroll
          for (int u = 0; u < EPV; u += 4)
            red_add_v4_keep(o + u, acc[v * EPV + u], acc[v * EPV + u + 1], acc[v * EPV + u + 2],
                            acc[v * EPV + u + 3], pol_keep);
        }
      }
    }
    cp_async_wait<0>();
  }
}

// ---- large batches: activations, then accumulation sweeps over slices of d ----
//
// When the fp32 accumulator y (L x d) is larger than about a third of L2, the
// scatter-adds of the grouped execution miss L2 and every reduction turns
// into DRAM traffic.  The grouped execution is then split: k_act computes the
// scalar c = gate * SiLU(x[t] . W[e]) of every task (W rows streamed group by
// group, as in k_expert_async), and Q sweeps of k_acc each add c * V[e] for
// one slice of Q columns of d -- only that slice of y is live, and it stays in
// L2 while the V rows stream past it.  Every task still reads its rows of W
// and V once, in schedule order, and the group's tokens still get their
// contributions by scatter-add.

constexpr int kActWarps = 8;

template <typename T, int NV, int R>
__global__ void __launch_bounds__(kActWarps * 32, 1)
    k_act(const T* __restrict__ x, const T* __restrict__ W, const int32_t* __restrict__ task_token,
          const int32_t* __restrict__ task_expert, const float* __restrict__ task_gate,
          int64_t M, int64_t L, int64_t N, int d, int S, int64_t nslices, float* __restrict__ cbuf,
          int32_t* status) {
  constexpr int SLOT = NV * 32;  // uint4 per ring slot: one W row
  extern __shared__ __align__(16) uint4 ring[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint4* wring = ring + static_cast<size_t>(warp) * R * SLOT;
  const uint32_t wring_s = static_cast<uint32_t>(__cvta_generic_to_shared(wring));
  const uint64_t pol_stream = policy_evict_first();
  const int64_t nw = static_cast<int64_t>(gridDim.x) * kActWarps;
  for (int64_t sl = static_cast<int64_t>(blockIdx.x) * kActWarps + warp; sl < nslices; sl += nw) {
    const int64_t a0 = sl * S;
    const int n = static_cast<int>(M - a0 < S ? M - a0 : S);
    int64_t my_t = -1, my_e = -1;
    float my_g = 0.0f, my_c = 0.0f;
    if (lane < n) {
      my_t = task_token[a0 + lane];
      my_e = task_expert[a0 + lane];
      my_g = task_gate[a0 + lane];
      if (my_t < 0 || my_t >= L || my_e < 0 || my_e >= N) {
        raise_status(status, OMNI_DEV_BAD_INDEX);
        my_e = -1;
        my_t = -1;
      }
    }
    const int64_t prev_t = __shfl_up_sync(0xffffffffu, my_t, 1);
    const uint32_t starts = __ballot_sync(0xffffffffu, lane < n && (lane == 0 || prev_t != my_t));
    auto issue = [&](int j) {
      if (j < n) {
        const int64_t e = __shfl_sync(0xffffffffu, my_e, j);
        if (e >= 0) {
          const uint4* wr = reinterpret_cast<const uint4*>(W + e * d);
          const uint32_t base = wring_s + static_cast<uint32_t>((j % R) * SLOT) * 16u;
#pragma unroll
          for (int v = 0; v < NV; ++v)
            cp_async16(base + static_cast<uint32_t>(v * 32 + lane) * 16u, wr + v * 32 + lane, pol_stream);
        }
      }
      cp_async_commit();
    };
#pragma unroll
    for (int j = 0; j < R - 1; ++j) issue(j);
    uint4 xc[NV], xn[NV];
    {
      const int64_t t0 = __shfl_sync(0xffffffffu, my_t, 0);
      const uint4* xr = reinterpret_cast<const uint4*>(x + (t0 < 0 ? 0 : t0) * d);
#pragma unroll
      for (int v = 0; v < NV; ++v) xn[v] = xr[v * 32 + lane];
    }
    for (int j = 0; j < n; ++j) {
      issue(j + R - 1);
      if ((starts >> j) & 1u) {
#pragma unroll
        for (int v = 0; v < NV; ++v) xc[v] = xn[v];
        const uint32_t later = starts & ~((2u << j) - 1u);
        if (later) {
          const int jn = __ffs(later) - 1;
          const int64_t tn = __shfl_sync(0xffffffffu, my_t, jn);
          const uint4* xr = reinterpret_cast<const uint4*>(x + (tn < 0 ? 0 : tn) * d);
#pragma unroll
          for (int v = 0; v < NV; ++v) xn[v] = xr[v * 32 + lane];
        }
      }
      cp_async_wait<R - 1>();
      const int64_t e = __shfl_sync(0xffffffffu, my_e, j);
      const float gj = __shfl_sync(0xffffffffu, my_g, j);
      if (e >= 0) {  // warp-uniform
        const uint4* slot = wring + (j % R) * SLOT;
        float sdot = 0.0f;
#pragma unroll
        for (int v = 0; v < NV; ++v) sdot += dot_vec(xc[v], slot[v * 32 + lane], static_cast<T*>(nullptr));
        sdot = warp_sum(sdot);
        if (lane == j) my_c = gj * silu(sdot);
      }
    }
    cp_async_wait<0>();
    if (lane < n) cbuf[a0 + lane] = my_c;
  }
}

constexpr int kAccThreads = 128;
constexpr int kAccUnroll = 4;  // value-row loads in flight per warp

// One sweep: y[t, col0 : col0 + 32*NVQ*EPV] += sum over the piece of c * V[e, same columns].
template <typename T, int NVQ>
__global__ void __launch_bounds__(kAccThreads)
    k_acc(const T* __restrict__ V, const int32_t* __restrict__ task_token,
          const int32_t* __restrict__ task_expert, const float* __restrict__ cbuf, int64_t M,
          int64_t L, int64_t N, int d, int col0, int S, float* __restrict__ yacc) {
  constexpr int EPV = kEpv<T>;
  const int lane = threadIdx.x & 31;
  const int64_t wid = (static_cast<int64_t>(blockIdx.x) * kAccThreads + threadIdx.x) >> 5;
  const int64_t a0 = wid * S;
  if (a0 >= M) return;
  const int n = static_cast<int>(M - a0 < S ? M - a0 : S);
  const uint64_t pol_stream = policy_evict_first();
  const uint64_t pol_keep = policy_evict_last();
  int64_t my_t = -1, my_e = -1;
  float my_c = 0.0f;
  if (lane < n) {
    my_t = task_token[a0 + lane];
    my_e = task_expert[a0 + lane];
    my_c = cbuf[a0 + lane];
    if (my_t < 0 || my_t >= L || my_e < 0 || my_e >= N) {
      my_e = -1;
      my_t = -1;
    }
  }
  const int64_t prev_t = __shfl_up_sync(0xffffffffu, my_t, 1);
  uint32_t starts = __ballot_sync(0xffffffffu, lane < n && (lane == 0 || prev_t != my_t));
  while (starts) {
    const int p = __ffs(starts) - 1;
    starts &= starts - 1;
    const int q = starts ? __ffs(starts) - 1 : n;
    const int64_t t = __shfl_sync(0xffffffffu, my_t, p);
    float acc[NVQ * EPV];
#pragma unroll
    for (int u = 0; u < NVQ * EPV; ++u) acc[u] = 0.0f;
    for (int j0 = p; j0 < q; j0 += kAccUnroll) {
      uint4 vv[kAccUnroll][NVQ];
      float cc[kAccUnroll];
#pragma unroll
      for (int u = 0; u < kAccUnroll; ++u) {
        const int j = j0 + u;
        const int64_t e = __shfl_sync(0xffffffffu, my_e, j < q ? j : p);
        cc[u] = __shfl_sync(0xffffffffu, my_c, j < q ? j : p);
        const bool ok = j < q && e >= 0;
        if (!ok) cc[u] = 0.0f;
        const uint4* vr = reinterpret_cast<const uint4*>(V + (ok ? e : 0) * d + col0);
#pragma unroll
        for (int v = 0; v < NVQ; ++v) {
          if (ok) {
            asm volatile("ld.global.L2::cache_hint.v4.u32 {%0, %1, %2, %3}, [%4], %5;"
                         : "=r"(vv[u][v].x), "=r"(vv[u][v].y), "=r"(vv[u][v].z), "=r"(vv[u][v].w)
                         : "l"(vr + v * 32 + lane), "l"(pol_stream));
          } else {
            vv[u][v] = make_uint4(0u, 0u, 0u, 0u);
          }
        }
      }
#pragma unroll
      for (int u = 0; u < kAccUnroll; ++u)
#pragma unroll
        for (int v = 0; v < NVQ; ++v) axpy_vec(cc[u], vv[u][v], acc + v * EPV, static_cast<T*>(nullptr));
    }
    if (t >= 0) {
      float* yr = yacc + t * d + col0;
#pragma unroll
      for (int v = 0; v < NVQ; ++v) {
        float* o = yr + static_cast<int64_t>(v * 32 + lane) * EPV;
#pragma unroll
        for (int u = 0; u < EPV; u += 4)
          red_add_v4_keep(o + u, acc[v * EPV + u], acc[v * EPV + u + 1], acc[v * EPV + u + 2],
                          acc[v * EPV + u + 3], pol_keep);
      }
    }
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

// Number of accumulation sweeps: 1 keeps the fused kernel; Q > 1 splits the
// columns of d so that each live slice of the fp32 accumulator is <= ~40 MiB.
int expert_sweeps(const Dims& D) {
  const int epv = D.dtype == OMNI_F32 ? 4 : 8;
  const int64_t ybytes = D.L * D.d * 4;
  const int64_t limit = int64_t(40) << 20;
  if (ybytes <= limit) return 1;
  const int64_t nv = D.d % (32 * epv) == 0 ? D.d / (32 * epv) : 0;
  if (nv != 2 && nv != 4 && nv != 8) return 1;  // row shapes the sweep kernels are built for
  for (int Q = 2; Q <= 16; Q *= 2) {
    if (D.d % Q != 0) break;
    const int64_t cols = D.d / Q;
    if (cols % (32 * epv) != 0) break;
    const int64_t nvq = cols / (32 * epv);
    if (nvq > 4) continue;
    if (ybytes / Q <= limit) return (nvq == 1 || nvq == 2 || nvq == 4) ? Q : 1;
  }
  return 1;
}

size_t expert_ws_bytes(const Dims& D) {
  size_t b = D.dtype == OMNI_F32 ? 0 : static_cast<size_t>(D.L) * D.d * sizeof(float);
  if (expert_sweeps(D) > 1) b = ((b + 255) & ~size_t(255)) + static_cast<size_t>(D.M()) * sizeof(float);
  return b;
}

template <typename T, int NV>
cudaError_t launch_slices(const Dims& D, const void* x, const void* W, const void* V,
                          const int32_t* tt, const int32_t* te, const float* tg, float* acc,
                          int32_t* status, cudaStream_t s) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  // slice length: about 16 warps per SM, at most 32 tasks (one per lane)
  const int64_t M = D.M();
  const int64_t want_warps = static_cast<int64_t>(sms) * 16;
  int S = static_cast<int>((M + want_warps - 1) / want_warps);
  S = S < 1 ? 1 : (S > 32 ? 32 : S);
  const int64_t warps = (M + S - 1) / S;
  const int64_t blocks = (warps + kExpThreads / 32 - 1) / (kExpThreads / 32);
  k_expert_slices<T, NV><<<static_cast<unsigned>(blocks), kExpThreads, 0, s>>>(
      static_cast<const T*>(x), static_cast<const T*>(W), static_cast<const T*>(V), tt, te, tg,
      M, D.L, D.N(), static_cast<int>(D.d), S, acc, status);
  return cudaGetLastError();
}

template <typename T, int NV, int R>
cudaError_t launch_async(const Dims& D, const void* x, const void* W, const void* V,
                         const int32_t* tt, const int32_t* te, const float* tg, float* acc,
                         int32_t* status, cudaStream_t s) {
  constexpr size_t smem = static_cast<size_t>(kAsyncWarps) * R * 2 * NV * 32 * 16;
  cudaError_t err = cudaFuncSetAttribute(k_expert_async<T, NV, R>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
  if (err != cudaSuccess) return err;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t M = D.M();
  const int64_t warps_all = static_cast<int64_t>(sms) * kAsyncWarps;
  int S = static_cast<int>((M + warps_all - 1) / warps_all);
  S = S < 1 ? 1 : (S > 32 ? 32 : S);
  const int64_t nslices = (M + S - 1) / S;
  int64_t blocks = (nslices + kAsyncWarps - 1) / kAsyncWarps;
  if (blocks > sms) blocks = sms;  // persistent: one CTA per SM (shared-memory bound)
  k_expert_async<T, NV, R><<<static_cast<unsigned>(blocks), kAsyncWarps * 32, smem, s>>>(
      static_cast<const T*>(x), static_cast<const T*>(W), static_cast<const T*>(V), tt, te, tg, M,
      D.L, D.N(), static_cast<int>(D.d), S, nslices, acc, status);
  return cudaGetLastError();
}

template <typename T>
cudaError_t dispatch_slices(const Dims& D, const void* x, const void* W, const void* V,
                            const int32_t* tt, const int32_t* te, const float* tg, float* acc,
                            int32_t* status, cudaStream_t s) {
  constexpr int row = 32 * kEpv<T>;  // elements covered by one vector per lane
  switch (D.d == row * 8 ? 8 : D.d == row * 4 ? 4 : D.d == row * 2 ? 2 : D.d == row ? 1 : 0) {
    case 8: return launch_async<T, 8, 3>(D, x, W, V, tt, te, tg, acc, status, s);
    case 4: return launch_async<T, 4, 4>(D, x, W, V, tt, te, tg, acc, status, s);
    case 2: return launch_async<T, 2, 4>(D, x, W, V, tt, te, tg, acc, status, s);
    case 1: return launch_async<T, 1, 4>(D, x, W, V, tt, te, tg, acc, status, s);
    default: return launch_slices<T, 0>(D, x, W, V, tt, te, tg, acc, status, s);
  }
}

template <typename T, int NV, int NVQ>
cudaError_t sweeps_nv(const Dims& D, int Q, const void* x, const void* W, const void* V,
                      const int32_t* tt, const int32_t* te, const float* tg, float* cbuf,
                      float* acc, int32_t* status, cudaStream_t s) {
  constexpr int R = 6;
  constexpr size_t smem = static_cast<size_t>(kActWarps) * R * NV * 32 * 16;
  cudaError_t err = cudaFuncSetAttribute(k_act<T, NV, R>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
  if (err != cudaSuccess) return err;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t M = D.M();
  const int S = 32;
  const int64_t nslices = (M + S - 1) / S;
  int64_t blocks = (nslices + kActWarps - 1) / kActWarps;
  if (blocks > sms) blocks = sms;
  k_act<T, NV, R><<<static_cast<unsigned>(blocks), kActWarps * 32, smem, s>>>(
      static_cast<const T*>(x), static_cast<const T*>(W), tt, te, tg, M, D.L, D.N(),
      static_cast<int>(D.d), S, nslices, cbuf, status);
  err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  const int64_t ablocks = (nslices + kAccThreads / 32 - 1) / (kAccThreads / 32);
  const int cols = static_cast<int>(D.d / Q);
  for (int q = 0; q < Q; ++q) {
    k_acc<T, NVQ><<<static_cast<unsigned>(ablocks), kAccThreads, 0, s>>>(
        static_cast<const T*>(V), tt, te, cbuf, M, D.L, D.N(), static_cast<int>(D.d), q * cols, S,
        acc);
    err = cudaGetLastError();
    if (err != cudaSuccess) return err;
  }
  return cudaSuccess;
}

template <typename T>
cudaError_t launch_sweeps(const Dims& D, int Q, const void* x, const void* W, const void* V,
                          const int32_t* tt, const int32_t* te, const float* tg, float* cbuf,
                          float* acc, int32_t* status, cudaStream_t s) {
  constexpr int row = 32 * kEpv<T>;
  const int64_t nv = D.d / row;             // vectors per lane for a whole row
  const int64_t nvq = (D.d / Q) / row;      // ... for one slice
  if (D.d % row != 0) return cudaErrorInvalidValue;
#define OMNI_SWEEP(NV_, NVQ_)                                                               \
  if (nv == NV_ && nvq == NVQ_)                                                             \
    return sweeps_nv<T, NV_, NVQ_>(D, Q, x, W, V, tt, te, tg, cbuf, acc, status, s);
  OMNI_SWEEP(8, 4) OMNI_SWEEP(8, 2) OMNI_SWEEP(8, 1) OMNI_SWEEP(4, 2) OMNI_SWEEP(4, 1)
  OMNI_SWEEP(2, 1)
#undef OMNI_SWEEP
  return cudaErrorInvalidValue;
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
  const int Q = expert_sweeps(D);
  if (Q > 1) {
    size_t off = f32 ? 0 : ((ybytes + 255) & ~size_t(255));
    float* cbuf = reinterpret_cast<float*>(static_cast<char*>(ws) + off);
    err = f32 ? launch_sweeps<float>(D, Q, x, W, V, task_token, task_expert, task_gate, cbuf, acc,
                                     status, s)
              : launch_sweeps<__nv_bfloat16>(D, Q, x, W, V, task_token, task_expert, task_gate,
                                             cbuf, acc, status, s);
  } else {
    err = f32 ? dispatch_slices<float>(D, x, W, V, task_token, task_expert, task_gate, acc, status, s)
              : dispatch_slices<__nv_bfloat16>(D, x, W, V, task_token, task_expert, task_gate, acc,
                                               status, s);
  }
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
