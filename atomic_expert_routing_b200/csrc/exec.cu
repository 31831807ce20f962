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
#include "blocksort.cuh"
#include "common.cuh"
#include "internal.h"

namespace omni {
namespace {

constexpr int kExpThreads = 128;  // 4 warps per CTA, each executing its own task slice

// Elements per 16-byte vector.
template <typename T> constexpr int kEpv = 16 / sizeof(T);

// s0 += a.lo * b.lo, s1 += a.hi * b.hi for two bf16 pairs, with the
// mixed-precision fma (bf16 operands, fp32 addend and result, one rounding):
// the same value as widening both operands to fp32 and using fmaf.
__device__ __forceinline__ void fma_bf16x2(float& s0, float& s1, uint32_t a, uint32_t b) {
  asm("{\n .reg .b16 al, ah, bl, bh;\n"
      " mov.b32 {al, ah}, %2;\n"
      " mov.b32 {bl, bh}, %3;\n"
      " fma.rn.f32.bf16 %0, al, bl, %0;\n"
      " fma.rn.f32.bf16 %1, ah, bh, %1;\n}"
      : "+f"(s0), "+f"(s1)
      : "r"(a), "r"(b));
}

// Dot product contribution of one 16-byte vector pair, in fp32.
__device__ __forceinline__ float dot_vec(uint4 a, uint4 b, __nv_bfloat16*) {
  float s0 = 0.0f, s1 = 0.0f;
  fma_bf16x2(s0, s1, a.x, b.x);
  fma_bf16x2(s0, s1, a.y, b.y);
  fma_bf16x2(s0, s1, a.z, b.z);
  fma_bf16x2(s0, s1, a.w, b.w);
  return s0 + s1;
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
    k_expert_slices(const T* __restrict__ x, const T* __restrict__ W, const T* __restrict__ U,
                    const T* __restrict__ V, const int32_t* __restrict__ task_token,
                    const int32_t* __restrict__ task_expert,
                    const float* __restrict__ task_gate, int64_t M, int64_t L, int64_t N, int d,
                    int S, ShardIds sh, float* __restrict__ yacc, int32_t* status) {
  pdl_wait();
  pdl_trigger();
  constexpr int EPV = kEpv<T>;
  const int lane = threadIdx.x & 31;
  const int64_t wid = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t a0 = wid * S;
  if (a0 >= M) return;  // whole warp
  {
    int64_t s0, s1;  // a shard's slices (all of them unsharded)
    sh.slices(S, (M + S - 1) / S, &s0, &s1);
    if (wid < s0 || wid >= s1) return;
  }
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
    } else if (!sh.has(my_e)) {  // another shard's task: nothing to add
      my_e = -1;
      my_t = -1;
    } else {
      my_e -= sh.lo;
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
        float c = gj * silu(s);
        if (U != nullptr) {  // gated expert: times x[t] . U[e]
          const uint4* ur = reinterpret_cast<const uint4*>(U + e * d);
          float su = 0.0f;
#pragma unroll
          for (int v = 0; v < NV; ++v) su += dot_vec(xv[v], ur[v * 32 + lane], static_cast<T*>(nullptr));
          c *= warp_sum(su);
        }
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
        float sacc = 0.0f, uacc = 0.0f;
        if (e >= 0) {  // warp-uniform; no shuffle inside
          const uint4* wr = reinterpret_cast<const uint4*>(W + e * d);
          for (int v = lane; v < nvec; v += 32) sacc += dot_vec(xr[v], wr[v], static_cast<T*>(nullptr));
          if (U != nullptr) {
            const uint4* ur = reinterpret_cast<const uint4*>(U + e * d);
            for (int v = lane; v < nvec; v += 32) uacc += dot_vec(xr[v], ur[v], static_cast<T*>(nullptr));
          }
        }
        sacc = warp_sum(sacc);
        uacc = warp_sum(uacc);
        const float gj = __shfl_sync(0xffffffffu, my_g, j);
        if (lane == j) my_c = (e >= 0) ? gj * silu(sacc) * (U != nullptr ? uacc : 1.0f) : 0.0f;
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
__device__ __forceinline__ uint64_t policy_evict_normal() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_normal.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ uint64_t policy_evict_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ void cp_async16_plain(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ uint4 ld_v4_hint(const void* p, uint64_t pol) {
  uint4 r;
  asm volatile("ld.global.nc.L2::cache_hint.v4.u32 {%0, %1, %2, %3}, [%4], %5;"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p), "l"(pol));
  return r;
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
// pipeline restarts at every slice.  With dense != nullptr, a task with
// dense[a] set takes its activation c from cpre[a] (formed on the tensor
// cores) and fetches only its V row.  GLU: gated experts, c also times
// x[t] . U[e]; a ring slot then holds the U row after the W and V rows.
template <typename T, int NV, int R, bool GLU>
__global__ void __launch_bounds__(kAsyncWarps * 32, 1)
    k_expert_async(const T* __restrict__ x, const T* __restrict__ W, const T* __restrict__ U,
                   const T* __restrict__ V,
                   const int32_t* __restrict__ task_token,
                   const int32_t* __restrict__ task_expert,
                   const float* __restrict__ task_gate, int64_t M, int64_t L, int64_t N, int d,
                   int S, int64_t nslices, ShardIds sh, float* __restrict__ yacc,
                   int32_t* status, const uint8_t* __restrict__ dense,
                   const float* __restrict__ cpre) {
  pdl_wait();
  pdl_trigger();
  constexpr int EPV = kEpv<T>;
  constexpr int SLOT = (GLU ? 3 : 2) * NV * 32;  // uint4 per ring slot: W, V (, U) vectors
  extern __shared__ __align__(16) uint4 ring[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint4* wring = ring + static_cast<size_t>(warp) * R * SLOT;
  const uint32_t wring_s = static_cast<uint32_t>(__cvta_generic_to_shared(wring));
  const uint64_t pol_stream = policy_evict_first();
  const uint64_t pol_keep = policy_evict_last();
  const int64_t nw = static_cast<int64_t>(gridDim.x) * kAsyncWarps;
  int64_t s0, s1;  // a shard's slices (all of them unsharded)
  sh.slices(S, nslices, &s0, &s1);
  for (int64_t sl = s0 + static_cast<int64_t>(blockIdx.x) * kAsyncWarps + warp; sl < s1; sl += nw) {
    const int64_t a0 = sl * S;
    const int n = static_cast<int>(M - a0 < S ? M - a0 : S);
    int64_t my_t = -1, my_e = -1;
    float my_g = 0.0f, my_cp = 0.0f;
    bool my_dense = false;
    if (lane < n) {
      my_t = task_token[a0 + lane];
      my_e = task_expert[a0 + lane];
      my_g = task_gate[a0 + lane];
      if (dense != nullptr && dense[a0 + lane] != 0) {
        my_dense = true;
        my_cp = cpre[a0 + lane];
      }
      if (my_t < 0 || my_t >= L || my_e < 0 || my_e >= N) {
        raise_status(status, OMNI_DEV_BAD_INDEX);
        my_e = -1;
        my_t = -1;
      } else if (!sh.has(my_e)) {  // another shard's task: nothing to add
        my_e = -1;
        my_t = -1;
      } else {
        my_e -= sh.lo;
      }
    }
    const uint32_t dmask = __ballot_sync(0xffffffffu, my_dense);
    const int64_t prev_t = __shfl_up_sync(0xffffffffu, my_t, 1);
    const int64_t next_t = __shfl_down_sync(0xffffffffu, my_t, 1);
    const uint32_t starts = __ballot_sync(0xffffffffu, lane < n && (lane == 0 || prev_t != my_t));
    const uint32_t ends = __ballot_sync(0xffffffffu, lane < n && (lane == n - 1 || next_t != my_t));

    // issue the row copies of task j into slot j % R (one commit group per
    // task; a dense task needs only its V row)
    auto issue = [&](int j) {
      if (j < n) {
        const int64_t e = __shfl_sync(0xffffffffu, my_e, j);
        if (e >= 0) {
          const bool need_w = !((dmask >> j) & 1u);
          const uint4* wr = reinterpret_cast<const uint4*>(W + e * d);
          const uint4* vr = reinterpret_cast<const uint4*>(V + e * d);
          const uint32_t base = wring_s + static_cast<uint32_t>((j % R) * SLOT) * 16u;
#pragma unroll
          for (int v = 0; v < NV; ++v) {
            if (need_w)
              cp_async16(base + static_cast<uint32_t>(v * 32 + lane) * 16u, wr + v * 32 + lane,
                         pol_stream);
            cp_async16(base + static_cast<uint32_t>((NV + v) * 32 + lane) * 16u, vr + v * 32 + lane,
                       pol_stream);
            if constexpr (GLU)
              cp_async16(base + static_cast<uint32_t>((2 * NV + v) * 32 + lane) * 16u,
                         reinterpret_cast<const uint4*>(U + e * d) + v * 32 + lane, pol_stream);
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
        float c;
        if ((dmask >> j) & 1u) {  // warp-uniform
          c = __shfl_sync(0xffffffffu, my_cp, j);
        } else {
          float sdot = 0.0f;
#pragma unroll
          for (int v = 0; v < NV; ++v)
            sdot += dot_vec(xc[v], slot[v * 32 + lane], static_cast<T*>(nullptr));
          sdot = warp_sum(sdot);
          c = gj * silu(sdot);
          if constexpr (GLU) {
            float su = 0.0f;
#pragma unroll
            for (int v = 0; v < NV; ++v)
              su += dot_vec(xc[v], slot[(2 * NV + v) * 32 + lane], static_cast<T*>(nullptr));
            c *= warp_sum(su);
          }
        }
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
// into DRAM traffic.  The grouped execution is then split: k_wsort merges
// consecutive groups into windows ordered by token, k_act computes the scalar
// c = gate * SiLU(x[t] . W[e]) of every task (W rows streamed window by
// window, as in k_expert_async), and Q sweeps of k_acc each add
// c * V[e] for one slice of Q columns of d -- only that slice of y is live,
// and it stays in L2 while the V rows stream past it.  Every task still
// reads its rows of W and V once, and the tokens of a window still get their
// contributions by scatter-add.

constexpr int kActWarps = 8;

// c[dst[a]] = g[a] * SiLU(H[hidx[a]] . F[fidx[a]]) over a task list in which
// tasks that share a held row H[h] are adjacent (a run).  Warp w takes slices
// of S consecutive tasks; the run's held row sits in registers (the next
// run's row is fetched while the current one is used), and the rows of F
// stream through a ring of R shared-memory slots per warp (cp.async, R - 1
// rows in flight), one per run of tasks that share it.  HOLD_KEEP: the held
// rows are re-read by later tasks (x by token) -- keep them in L2
// (evict-last) and read the F rows, each fetched once, evict-first.  dst ==
// nullptr writes c[a].  Indices are range-checked (OMNI_DEV_BAD_INDEX; the
// task gets c = 0).  GLU: gated experts, c also times H[h] . G[f]; a ring
// slot then holds the row of G after the row of F (one CTA per SM).
template <typename T, int NV, int R, bool HOLD_KEEP, bool GLU>
__global__ void __launch_bounds__(kActWarps * 32, GLU ? 1 : 2)
    k_act(const T* __restrict__ H, const int32_t* __restrict__ hidx, int64_t nh,
          const T* __restrict__ F, const T* __restrict__ G, const int32_t* __restrict__ fidx,
          int64_t nf, ShardIds fs, const float* __restrict__ task_gate,
          const int32_t* __restrict__ dst, int64_t M, int d, int S, int64_t nslices,
          float* __restrict__ cbuf, int32_t* status) {
  pdl_wait();
  constexpr int SLOT = (GLU ? 2 : 1) * NV * 32;  // uint4 per ring slot: a row of F (and of G)
  extern __shared__ __align__(16) uint4 ring[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint4* fring = ring + static_cast<size_t>(warp) * R * SLOT;
  const uint32_t fring_s = static_cast<uint32_t>(__cvta_generic_to_shared(fring));
  const uint64_t pol_once = policy_evict_first();
  const uint64_t pol_keep = policy_evict_last();
  const int64_t nw = static_cast<int64_t>(gridDim.x) * kActWarps;
  int64_t s0, s1;  // a shard's slices (all of them unsharded)
  fs.slices(S, nslices, &s0, &s1);
  for (int64_t sl = s0 + static_cast<int64_t>(blockIdx.x) * kActWarps + warp; sl < s1; sl += nw) {
    const int64_t a0 = sl * S;
    const int n = static_cast<int>(M - a0 < S ? M - a0 : S);
    int64_t my_h = -1, my_f = -1, my_d = -1;
    float my_g = 0.0f, my_c = 0.0f;
    if (lane < n) {
      my_h = hidx[a0 + lane];
      my_f = fidx[a0 + lane];
      my_g = task_gate[a0 + lane];
      my_d = dst != nullptr ? dst[a0 + lane] : a0 + lane;
      if (my_h < 0 || my_h >= nh || my_f < 0 || my_f >= nf || my_d < 0 || my_d >= M) {
        raise_status(status, OMNI_DEV_BAD_INDEX);
        my_h = -1;
        my_f = -1;
        if (my_d < 0 || my_d >= M) my_d = -1;
      } else if (!fs.has(my_f)) {  // a row of another shard: c = 0
        my_h = -1;
        my_f = -1;
      } else {
        my_f -= fs.lo;
      }
    }
    const int64_t prev_h = __shfl_up_sync(0xffffffffu, my_h, 1);
    const uint32_t starts = __ballot_sync(0xffffffffu, lane < n && (lane == 0 || prev_h != my_h));
    const int64_t prev_f = __shfl_up_sync(0xffffffffu, my_f, 1);
    const uint32_t fstarts = __ballot_sync(0xffffffffu, lane < n && (lane == 0 || prev_f != my_f));
    // the ring is filled run by run of F: a row repeated by adjacent tasks is
    // fetched once.  Run r sits in slot r % R; every issue commits one group.
    uint32_t pending = fstarts;
    int issued = 0;
    auto issue = [&]() {
      if (pending != 0u) {
        const int j = __ffs(pending) - 1;
        pending &= pending - 1u;
        const int64_t f = __shfl_sync(0xffffffffu, my_f, j);
        if (f >= 0) {
          const uint4* fr = reinterpret_cast<const uint4*>(F + f * d);
          const uint32_t base = fring_s + static_cast<uint32_t>((issued % R) * SLOT) * 16u;
#pragma unroll
          for (int v = 0; v < NV; ++v) {
            if (HOLD_KEEP)
              cp_async16(base + static_cast<uint32_t>(v * 32 + lane) * 16u, fr + v * 32 + lane, pol_once);
            else
              cp_async16_plain(base + static_cast<uint32_t>(v * 32 + lane) * 16u, fr + v * 32 + lane);
            if constexpr (GLU)
              cp_async16(base + static_cast<uint32_t>((NV + v) * 32 + lane) * 16u,
                         reinterpret_cast<const uint4*>(G + f * d) + v * 32 + lane, pol_once);
          }
        }
      }
      ++issued;
      cp_async_commit();
    };
#pragma unroll
    for (int j = 0; j < R - 1; ++j) issue();
    uint4 hc[NV], hn[NV];
    auto load_held = [&](int64_t h) {
      const uint4* hr = reinterpret_cast<const uint4*>(H + (h < 0 ? 0 : h) * d);
#pragma unroll
      for (int v = 0; v < NV; ++v) hn[v] = HOLD_KEEP ? ld_v4_hint(hr + v * 32 + lane, pol_keep) : hr[v * 32 + lane];
    };
    load_held(__shfl_sync(0xffffffffu, my_h, 0));
    int run = -1;
    for (int j = 0; j < n; ++j) {
      if ((fstarts >> j) & 1u) {  // F run `run` is complete once R - 1 later ones are issued
        ++run;
        issue();
        cp_async_wait<R - 1>();
      }
      if ((starts >> j) & 1u) {
#pragma unroll
        for (int v = 0; v < NV; ++v) hc[v] = hn[v];
        const uint32_t later = starts & ~((2u << j) - 1u);
        if (later) load_held(__shfl_sync(0xffffffffu, my_h, __ffs(later) - 1));
      }
      const int64_t h = __shfl_sync(0xffffffffu, my_h, j);
      const float gj = __shfl_sync(0xffffffffu, my_g, j);
      if (h >= 0) {  // warp-uniform
        const uint4* slot = fring + (run % R) * SLOT;
        float sdot = 0.0f;
#pragma unroll
        for (int v = 0; v < NV; ++v) sdot += dot_vec(hc[v], slot[v * 32 + lane], static_cast<T*>(nullptr));
        sdot = warp_sum(sdot);
        float cj = gj * silu(sdot);
        if constexpr (GLU) {
          float su = 0.0f;
#pragma unroll
          for (int v = 0; v < NV; ++v)
            su += dot_vec(hc[v], slot[(NV + v) * 32 + lane], static_cast<T*>(nullptr));
          cj *= warp_sum(su);
        }
        if (lane == j) my_c = cj;
      }
    }
    cp_async_wait<0>();
    if (lane < n && my_d >= 0) cbuf[my_d] = my_c;
  }
}

// ---- windows: consecutive groups merged per token --------------------------
//
// A token's K experts lie in few rows of the Nr x Nc grid, so they fall into
// far fewer windows of consecutive groups than groups.  Inside a window of
// whole groups (about kWinTasks tasks) k_wsort orders the tasks by token
// (stable: a token's tasks keep their group and expert order), so the sweeps
// below can add a token's contributions from the whole window with one
// scatter-add instead of one per group.  Every group is still executed as a
// unit -- its rows are read while its window is in flight -- and every task
// exactly once.
constexpr int kWinTasks = 7168;
constexpr int kWinCountBins = 2 * kBlockSortMax;  // counters of the counting expert order

// The first sweep's fp32 slice (zrows x zcols floats, rows zld apart;
// nullptr: nothing) is cleared by the window sort.
__device__ __forceinline__ void clear_slice(float* zslice, int64_t zrows, int zcols, int64_t zld) {
  if (zslice == nullptr) return;
  const int per_row = zcols / 4;
  const int64_t n = zrows * per_row;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    reinterpret_cast<float4*>(zslice + (i / per_row) * zld)[i % per_row] =
        make_float4(0.f, 0.f, 0.f, 0.f);
}

// Window w takes the groups whose first task lies in [w*T, (w+1)*T).  Two
// orders of its tasks are written: by token (wt/we/wg, for the accumulation
// sweeps) and by expert (xt/xe/xg, for the activations, so that the tasks of
// one expert are adjacent and its W row leaves HBM once), with xdst the
// token-order position of each expert-order task.  Both sorts are stable
// (a window arrives in (group, token, expert) order).  Windows larger than
// the CTA sort (a single very large group) and the whole batch when the
// group count on the device is out of range are passed through in schedule
// order (the latter with OMNI_DEV_BAD_INDEX raised).
struct WinOut {
  int32_t *wt, *we;
  float* wg;
  int32_t *xt, *xe;
  float* xg;
  int32_t* xdst;
};

__global__ void __launch_bounds__(kBlockSortThreads)
    k_wsort(const int32_t* __restrict__ tt, const int32_t* __restrict__ te,
            const float* __restrict__ tg, const int32_t* __restrict__ group_off,
            const int32_t* __restrict__ counts, int64_t M, int64_t gmax, int T, int passes,
            WinOut o, int32_t* status, float* __restrict__ zslice, int64_t zrows, int zcols,
            int64_t zld) {
  pdl_wait();  // the kernel ahead may be a previous call's last use of the slice
  pdl_trigger();
  clear_slice(zslice, zrows, zcols, zld);
  extern __shared__ __align__(16) uint8_t wsm[];
  uint32_t* kA = reinterpret_cast<uint32_t*>(wsm);
  uint32_t* kB = kA + kBlockSortMax;
  uint16_t* vA = reinterpret_cast<uint16_t*>(kB + kBlockSortMax);
  uint16_t* vB = vA + kBlockSortMax;
  uint16_t* inv = vB + kBlockSortMax;  // token-order position of each task
  uint32_t* wcount = reinterpret_cast<uint32_t*>(inv + kBlockSortMax);
  __shared__ uint32_t dbase[256];
  __shared__ int warp_tot[32];
  __shared__ int total;
  __shared__ int64_t rng[2];
  __shared__ int emin, emax;
  const int64_t lo = static_cast<int64_t>(blockIdx.x) * T;
  const int64_t hi = M - lo < T ? M : lo + T;
  if (threadIdx.x == 0) {
    const int64_t G = counts[1];
    int64_t a0 = lo, a1 = hi;
    if (G < 1 || G > gmax) {
      raise_status(status, OMNI_DEV_BAD_INDEX);
    } else {
      // first group starting at or after v (group_off[G] == M closes the list)
      auto first_at = [&](int64_t v) {
        int64_t l = 0, h = G;
        while (l < h) {
          const int64_t m = (l + h) >> 1;
          if (group_off[m] >= v) h = m; else l = m + 1;
        }
        return l;
      };
      const int64_t g0 = first_at(lo), g1 = first_at(hi);
      const int64_t b0 = g0 >= G ? M : group_off[g0];
      const int64_t b1 = g1 >= G ? M : group_off[g1];
      if (b0 < 0 || b1 > M || b0 > b1) {
        raise_status(status, OMNI_DEV_BAD_INDEX);
      } else {
        a0 = b0;
        a1 = b1;
      }
    }
    rng[0] = a0;
    rng[1] = a1;
    emin = INT_MAX;
    emax = INT_MIN;
  }
  __syncthreads();
  const int64_t a0 = rng[0];
  const int64_t n = rng[1] - a0;
  if (n <= 0) return;
  if (n > kBlockSortMax) {
    for (int64_t i = threadIdx.x; i < n; i += blockDim.x) {
      const int32_t t = tt[a0 + i], e = te[a0 + i];
      const float g = tg[a0 + i];
      o.wt[a0 + i] = t; o.we[a0 + i] = e; o.wg[a0 + i] = g;
      o.xt[a0 + i] = t; o.xe[a0 + i] = e; o.xg[a0 + i] = g;
      o.xdst[a0 + i] = static_cast<int32_t>(a0 + i);
    }
    return;
  }
  const int nn = static_cast<int>(n);
  int lmin = INT_MAX, lmax = INT_MIN;
  for (int i = threadIdx.x; i < nn; i += blockDim.x) {
    kA[i] = static_cast<uint32_t>(tt[a0 + i]);
    vA[i] = static_cast<uint16_t>(i);
    const int e = te[a0 + i];
    lmin = e < lmin ? e : lmin;
    lmax = e > lmax ? e : lmax;
  }
  atomicMin(&emin, lmin);
  atomicMax(&emax, lmax);
  __syncthreads();
  // by token
  uint32_t* kin = kA; uint32_t* kout = kB;
  uint16_t* vin = vA; uint16_t* vout = vB;
  for (int p = 0; p < passes; ++p) {
    block_radix_pass(kin, vin, kout, vout, nn, 8 * p, wcount, dbase, warp_tot, &total);
    uint32_t* tk = kin; kin = kout; kout = tk;
    uint16_t* tv = vin; vin = vout; vout = tv;
  }
  for (int i = threadIdx.x; i < nn; i += blockDim.x) {
    const int src = vin[i];
    inv[src] = static_cast<uint16_t>(i);
    o.wt[a0 + i] = tt[a0 + src];
    o.we[a0 + i] = te[a0 + src];
    o.wg[a0 + i] = tg[a0 + src];
  }
  __syncthreads();  // the key/value buffers are reused below
  // by expert (ids relative to the window's smallest)
  const int64_t span = static_cast<int64_t>(emax) - emin;
  int ebits = 0;
  while (ebits < 32 && (int64_t(1) << ebits) <= span) ++ebits;
  const int epasses = (ebits + 7) / 8;
  for (int i = threadIdx.x; i < nn; i += blockDim.x) {
    kA[i] = static_cast<uint32_t>(te[a0 + i] - emin);
    vA[i] = static_cast<uint16_t>(i);
  }
  __syncthreads();
  kin = kA; kout = kB; vin = vA; vout = vB;
  for (int p = 0; p < epasses; ++p) {
    block_radix_pass(kin, vin, kout, vout, nn, 8 * p, wcount, dbase, warp_tot, &total);
    uint32_t* tk = kin; kin = kout; kout = tk;
    uint16_t* tv = vin; vin = vout; vout = tv;
  }
  for (int i = threadIdx.x; i < nn; i += blockDim.x) {
    const int src = vin[i];
    o.xt[a0 + i] = tt[a0 + src];
    o.xe[a0 + i] = te[a0 + src];
    o.xg[a0 + i] = tg[a0 + src];
    o.xdst[a0 + i] = static_cast<int32_t>(a0 + inv[src]);
  }
}

// The same window orders when the tasks already arrive in window token order
// (wt/we/wg, windows [win_lo[w], win_lo[w+1])): only the expert order is
// left.  The activation pass needs an expert's tasks adjacent, not in any
// order among themselves (each task's activation is its own dot product), so
// a window whose ids span at most kWinCountBins is ordered by one counting
// pass (shared-memory counters, then placement by atomic cursors); a wider
// one by the stable radix sort.  Windows larger than the CTA sort keep token
// order.
__global__ void __launch_bounds__(kBlockSortThreads)
    k_wsort_x(const int32_t* __restrict__ win_lo, WinOut o, float* __restrict__ zslice,
              int64_t zrows, int zcols, int64_t zld) {
  // the kernel ahead is the window scatter of the same forward, which does
  // not touch the slice: clear it before the wait
  clear_slice(zslice, zrows, zcols, zld);
  pdl_wait();
  pdl_trigger();
  extern __shared__ __align__(16) uint8_t wsm[];
  uint32_t* kA = reinterpret_cast<uint32_t*>(wsm);
  uint32_t* kB = kA + kBlockSortMax;
  uint16_t* vA = reinterpret_cast<uint16_t*>(kB + kBlockSortMax);
  uint16_t* vB = vA + kBlockSortMax;
  uint32_t* wcount = reinterpret_cast<uint32_t*>(vB + 2 * kBlockSortMax);
  __shared__ uint32_t dbase[256];
  __shared__ int warp_tot[32];
  __shared__ int total;
  __shared__ int emin, emax;
  const int64_t a0 = win_lo[blockIdx.x];
  const int64_t n = win_lo[blockIdx.x + 1] - a0;
  if (n <= 0) return;
  if (n > kBlockSortMax) {
    for (int64_t i = threadIdx.x; i < n; i += blockDim.x) {
      o.xt[a0 + i] = o.wt[a0 + i];
      o.xe[a0 + i] = o.we[a0 + i];
      o.xg[a0 + i] = o.wg[a0 + i];
      o.xdst[a0 + i] = static_cast<int32_t>(a0 + i);
    }
    return;
  }
  if (threadIdx.x == 0) {
    emin = INT_MAX;
    emax = INT_MIN;
  }
  __syncthreads();
  const int nn = static_cast<int>(n);
  // this thread's tasks i = threadIdx.x + q * blockDim.x, read once
  constexpr int kPer = kBlockSortMax / kBlockSortThreads;
  int te_r[kPer], tt_r[kPer];
  float tg_r[kPer];
  int lmin = INT_MAX, lmax = INT_MIN;
#pragma unroll
  for (int q = 0; q < kPer; ++q) {
    const int i = threadIdx.x + q * kBlockSortThreads;
    te_r[q] = 0;
    if (i < nn) {
      te_r[q] = o.we[a0 + i];
      tt_r[q] = o.wt[a0 + i];
      tg_r[q] = o.wg[a0 + i];
      lmin = te_r[q] < lmin ? te_r[q] : lmin;
      lmax = te_r[q] > lmax ? te_r[q] : lmax;
    }
  }
  atomicMin(&emin, lmin);
  atomicMax(&emax, lmax);
  __syncthreads();
  const int64_t span = static_cast<int64_t>(emax) - emin;
  if (span < kWinCountBins) {
    int* cnt = reinterpret_cast<int*>(kA);  // kA and kB: kWinCountBins counters
    const int bins = static_cast<int>(span) + 1;
    for (int b = threadIdx.x; b < bins; b += blockDim.x) cnt[b] = 0;
    __syncthreads();
#pragma unroll
    for (int q = 0; q < kPer; ++q)
      if (threadIdx.x + q * kBlockSortThreads < nn) atomicAdd(&cnt[te_r[q] - emin], 1);
    __syncthreads();
    // exclusive scan of the counters: thread k takes bins [k*per, k*per + per)
    const int per = (bins + kBlockSortThreads - 1) / kBlockSortThreads;
    int mine = 0;
    for (int b = threadIdx.x * per; b < bins && b < threadIdx.x * per + per; ++b) mine += cnt[b];
    int run = block_exclusive_scan(mine, warp_tot, &total);
    for (int b = threadIdx.x * per; b < bins && b < threadIdx.x * per + per; ++b) {
      const int c = cnt[b];
      cnt[b] = run;
      run += c;
    }
    __syncthreads();
#pragma unroll
    for (int q = 0; q < kPer; ++q) {
      const int i = threadIdx.x + q * kBlockSortThreads;
      if (i < nn) {
        const int pos = atomicAdd(&cnt[te_r[q] - emin], 1);
        o.xt[a0 + pos] = tt_r[q];
        o.xe[a0 + pos] = te_r[q];
        o.xg[a0 + pos] = tg_r[q];
        o.xdst[a0 + pos] = static_cast<int32_t>(a0 + i);
      }
    }
    return;
  }
  int ebits = 0;
  while (ebits < 32 && (int64_t(1) << ebits) <= span) ++ebits;
  const int epasses = (ebits + 7) / 8;
  for (int i = threadIdx.x; i < nn; i += blockDim.x) {
    kA[i] = static_cast<uint32_t>(o.we[a0 + i] - emin);
    vA[i] = static_cast<uint16_t>(i);
  }
  __syncthreads();
  uint32_t* kin = kA; uint32_t* kout = kB;
  uint16_t* vin = vA; uint16_t* vout = vB;
  for (int p = 0; p < epasses; ++p) {
    block_radix_pass(kin, vin, kout, vout, nn, 8 * p, wcount, dbase, warp_tot, &total);
    uint32_t* tk = kin; kin = kout; kout = tk;
    uint16_t* tv = vin; vin = vout; vout = tv;
  }
  for (int i = threadIdx.x; i < nn; i += blockDim.x) {
    const int src = vin[i];
    o.xt[a0 + i] = o.wt[a0 + src];
    o.xe[a0 + i] = o.we[a0 + src];
    o.xg[a0 + i] = o.wg[a0 + src];
    o.xdst[a0 + i] = static_cast<int32_t>(a0 + src);
  }
}

constexpr int kAccWarps = 4;

// Four consecutive elements of T as one load: bf16 -> 8 bytes, fp32 -> 16 bytes.
template <typename T> struct Quad;
template <> struct Quad<__nv_bfloat16> { using type = uint2; };
template <> struct Quad<float> { using type = uint4; };

__device__ __forceinline__ uint2 ld_quad(const __nv_bfloat16* p, uint64_t pol) {
  uint2 r;
  asm volatile("ld.global.nc.L2::cache_hint.v2.u32 {%0, %1}, [%2], %3;"
               : "=r"(r.x), "=r"(r.y) : "l"(p), "l"(pol));
  return r;
}
__device__ __forceinline__ uint4 ld_quad(const float* p, uint64_t pol) {
  uint4 r;
  asm volatile("ld.global.nc.L2::cache_hint.v4.u32 {%0, %1, %2, %3}, [%4], %5;"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p), "l"(pol));
  return r;
}
__device__ __forceinline__ void fma_quad(float c, uint2 v, float* a) {
  a[0] = fmaf(c, bf16lo(v.x), a[0]); a[1] = fmaf(c, bf16hi(v.x), a[1]);
  a[2] = fmaf(c, bf16lo(v.y), a[2]); a[3] = fmaf(c, bf16hi(v.y), a[3]);
}
__device__ __forceinline__ void fma_quad(float c, uint4 v, float* a) {
  a[0] = fmaf(c, __uint_as_float(v.x), a[0]); a[1] = fmaf(c, __uint_as_float(v.y), a[1]);
  a[2] = fmaf(c, __uint_as_float(v.z), a[2]); a[3] = fmaf(c, __uint_as_float(v.w), a[3]);
}

// One sweep over the window-ordered tasks: yacc[t, 0 : 128*NB] (rows ld
// floats apart) += c * V[e, col0 : col0 + 128*NB], summed over each run of one token's tasks in a
// 32-task slice and added with one vector reduction per run and 128 columns.
// Lane l owns columns col0 + 128*b + 4*l .. +3 of every block b, so each
// reduction instruction covers 512 contiguous bytes of y (whole sectors).
// Warps take slices round-robin (the whole grid moves through the task list
// together, so a window's re-used V rows are still in L2); the V loads run D
// tasks ahead in registers, across run and slice boundaries.
template <typename T, int NB, int D>
__global__ void __launch_bounds__(kAccWarps * 32, (NB >= 8 ? 4 : 5))
    k_acc(const T* __restrict__ V, const int32_t* __restrict__ task_token,
          const int32_t* __restrict__ task_expert, const float* __restrict__ cbuf, int64_t M,
          int64_t L, int64_t N, int d, int col0, int64_t nslices, ShardIds sh,
          float* __restrict__ yacc, int64_t ld) {
  pdl_wait();
  static_assert(32 % D == 0, "the prefetch distance divides the slice");
  using QT = typename Quad<T>::type;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // V rows of a window's repeated experts are re-read soon: normal priority
  const uint64_t pol_stream = policy_evict_normal();
  const uint64_t pol_keep = policy_evict_last();
  const int64_t nw = static_cast<int64_t>(gridDim.x) * kAccWarps;
  int64_t s0, s1;  // a shard's slices (all of them unsharded)
  sh.slices(32, nslices, &s0, &s1);
  int64_t sl = s0 + static_cast<int64_t>(blockIdx.x) * kAccWarps + warp;
  if (sl >= s1) return;
  struct Meta {
    int n, t, e;
    float c;
  };
  auto load_meta = [&](int64_t s) {
    Meta m{0, -1, -1, 0.0f};
    if (s < s1) {
      const int64_t a0 = s * 32;
      m.n = static_cast<int>(M - a0 < 32 ? M - a0 : 32);
      if (lane < m.n) {
        const int64_t t = task_token[a0 + lane];
        const int64_t e = task_expert[a0 + lane];
        // (other shards' tasks are skipped like bad indices, silently)
        if (t >= 0 && t < L && e >= 0 && e < N && sh.has(e)) {
          m.t = static_cast<int>(t);
          m.e = static_cast<int>(e - sh.lo);
          m.c = cbuf[a0 + lane];
        }
      }
    }
    return m;
  };
  Meta cur = load_meta(sl);
  Meta nxt = load_meta(sl + nw);
  // position p counts from the current slice's first task; p >= 32 lies in
  // the warp's next slice (only a full slice is followed by another)
  auto issue = [&](int p, QT (&b)[NB]) {
    int e = -1;
    if (p < cur.n) {
      e = __shfl_sync(0xffffffffu, cur.e, p);
    } else if (cur.n == 32 && p - 32 < nxt.n) {
      e = __shfl_sync(0xffffffffu, nxt.e, p - 32);
    }
    if (e >= 0) {  // warp-uniform
      const T* row = V + static_cast<int64_t>(e) * d + col0 + 4 * lane;
#pragma unroll
      for (int bb = 0; bb < NB; ++bb) b[bb] = ld_quad(row + 128 * bb, pol_stream);
    }
  };
  QT buf[D][NB];
#pragma unroll
  for (int q = 0; q < D; ++q) issue(q, buf[q]);
  float acc[NB][4];
#pragma unroll
  for (int bb = 0; bb < NB; ++bb) acc[bb][0] = acc[bb][1] = acc[bb][2] = acc[bb][3] = 0.0f;
  while (true) {
    const int next_t = __shfl_down_sync(0xffffffffu, cur.t, 1);
    const uint32_t ends =
        __ballot_sync(0xffffffffu, lane < cur.n && (lane == cur.n - 1 || next_t != cur.t));
    for (int j0 = 0; j0 < 32; j0 += D) {
#pragma unroll
      for (int q = 0; q < D; ++q) {
        const int j = j0 + q;
        if (j < cur.n) {  // warp-uniform
          const int e = __shfl_sync(0xffffffffu, cur.e, j);
          const float c = __shfl_sync(0xffffffffu, cur.c, j);
          if (e >= 0) {
#pragma unroll
            for (int bb = 0; bb < NB; ++bb) fma_quad(c, buf[q][bb], acc[bb]);
          }
          issue(j + D, buf[q]);
          if ((ends >> j) & 1u) {
            const int t = __shfl_sync(0xffffffffu, cur.t, j);
            if (t >= 0) {
              float* yr = yacc + static_cast<int64_t>(t) * ld + 4 * lane;
#pragma unroll
              for (int bb = 0; bb < NB; ++bb)
                red_add_v4_keep(yr + 128 * bb, acc[bb][0], acc[bb][1], acc[bb][2], acc[bb][3],
                                pol_keep);
            }
#pragma unroll
            for (int bb = 0; bb < NB; ++bb) acc[bb][0] = acc[bb][1] = acc[bb][2] = acc[bb][3] = 0.0f;
          }
        }
      }
    }
    sl += nw;
    if (sl >= s1) break;
    cur = nxt;
    nxt = load_meta(sl + nw);
  }
}

// fp32 accumulator -> bf16 output (round to nearest even), 8 values per thread.
__global__ void __launch_bounds__(256) k_cast(const float* __restrict__ src,
                                              __nv_bfloat16* __restrict__ dst, int64_t n) {
  pdl_wait();
  pdl_trigger();
  const int64_t i = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) * 8;
  if (i >= n) return;
  const float4 a = *reinterpret_cast<const float4*>(src + i);
  const float4 b = *reinterpret_cast<const float4*>(src + i + 4);
  const float f[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
  *reinterpret_cast<uint4*>(dst + i) = pack_vec(f, static_cast<__nv_bfloat16*>(nullptr));
}

// Bookkeeping between accumulation sweeps on an fp32 slice of cols columns
// of L rows, 8 columns per thread:
//  - src != nullptr: the slice (rows src_ld floats apart) is final -- round
//    it to bf16 into y (rows y_ld apart); with discard, the accumulator being
//    scratch, drop its 128-byte lines from L2 without writing them back
//    (discard.global.L2);
//  - zdst != nullptr: zero the slice at zdst (rows z_ld apart) for the next
//    sweep; the stores leave it in L2.  zdst may be src: each thread reads
//    its eight values before it zeroes them.
__global__ void __launch_bounds__(256)
    k_slice_finish(const float* __restrict__ src, int64_t src_ld, __nv_bfloat16* __restrict__ y,
                   int64_t y_ld, float* zdst, int64_t z_ld, int64_t L, int cols, int discard) {
  pdl_wait();
  pdl_trigger();
  const int per_row = cols / 8;
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t row = i / per_row;
  const int c8 = static_cast<int>(i % per_row) * 8;
  const bool active = row < L;
  if (src != nullptr) {
    const float* p = src + row * src_ld + c8;
    if (active) {
      const float4 a = *reinterpret_cast<const float4*>(p);
      const float4 b = *reinterpret_cast<const float4*>(p + 4);
      const float f[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
      *reinterpret_cast<uint4*>(y + row * y_ld + c8) =
          pack_vec(f, static_cast<__nv_bfloat16*>(nullptr));
    }
    if (discard) {
      __syncwarp();  // the four threads of a line have read it
      if (active && (c8 & 31) == 0) asm volatile("discard.global.L2 [%0], 128;" ::"l"(p) : "memory");
    }
  }
  if (zdst != nullptr && active) {
    float4* dst = reinterpret_cast<float4*>(zdst + row * z_ld + c8);
    dst[0] = make_float4(0.f, 0.f, 0.f, 0.f);
    dst[1] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
}

constexpr int kTokThreads = 128;

// Token-centric execution: CTA t gathers the rows of its own K experts.
// Phase 1: each warp takes tasks q = warp, warp+4, ... and computes
// c_q = gate * SiLU(x[t] . W[e_q]) (x[t] as 16-byte vectors in shared memory);
// phase 2: each thread owns 16-byte vectors of the output row and sums
// c_q * V[e_q] over the K tasks.  No reductions across CTAs.
template <typename T>
__global__ void __launch_bounds__(kTokThreads)
    k_token_centric(const T* __restrict__ x, const T* __restrict__ W, const T* __restrict__ U,
                    const T* __restrict__ V,
                    const int32_t* __restrict__ idx, const float* __restrict__ gate, int K, int d,
                    int64_t N, T* __restrict__ y, int32_t* status) {
  pdl_wait();
  pdl_trigger();
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
    float s = 0.0f, su = 0.0f;
    if (e >= 0) {
      const uint4* wr = reinterpret_cast<const uint4*>(W + e * d);
      for (int v = lane; v < nvec; v += 32) s += dot_vec(xs[v], wr[v], static_cast<T*>(nullptr));
      if (U != nullptr) {  // gated expert: times x[t] . U[e]
        const uint4* ur = reinterpret_cast<const uint4*>(U + e * d);
        for (int v = lane; v < nvec; v += 32) su += dot_vec(xs[v], ur[v], static_cast<T*>(nullptr));
      }
    }
    s = warp_sum(s);
    su = warp_sum(su);
    if (lane == 0)
      cq[q] = (e >= 0) ? gate[t * K + q] * silu(s) * (U != nullptr ? su : 1.0f) : 0.0f;
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

// Workspace of the sweeps path, after the fp32 accumulator: the activations
// c and the window-ordered copy of the task list.
struct SweepWs {
  float* cbuf;
  WinOut win;
  int32_t* win_lo;  // [nwin + 1] window starts, when the tasks come in window order
};

size_t acc_bytes(const Dims& D) {
  return D.dtype == OMNI_F32 ? 0 : static_cast<size_t>(D.L) * D.d * sizeof(float);
}

SweepWs carve_sweeps(const Dims& D, void* ws, size_t* bytes) {
  Carver c(ws);
  c.take<char>(acc_bytes(D) / expert_sweeps(D));  // bf16: one fp32 slice of d / Q columns
  SweepWs w;
  const size_t M = static_cast<size_t>(D.M());
  w.cbuf = c.take<float>(M);
  w.win.wt = c.take<int32_t>(M);
  w.win.we = c.take<int32_t>(M);
  w.win.wg = c.take<float>(M);
  w.win.xt = c.take<int32_t>(M);
  w.win.xe = c.take<int32_t>(M);
  w.win.xg = c.take<float>(M);
  w.win.xdst = c.take<int32_t>(M);
  const int64_t T = window_tasks(D);
  w.win_lo = c.take<int32_t>(static_cast<size_t>((D.M() + T - 1) / T) + 1);
  if (bytes) *bytes = c.off;
  return w;
}

// bf16 batches without sweeps whose row width has a k_expert_async instance
// run the activations of dense groups on the tensor cores first.
bool dense_path(const Dims& D) {
  if (!dense_supported(D) || expert_sweeps(D) > 1) return false;
  return D.d == 256 || D.d == 512 || D.d == 1024 || D.d == 2048;
}

size_t dense_ws_offset(const Dims& D) { return (acc_bytes(D) + 255) & ~size_t(255); }

size_t expert_ws_bytes(const Dims& D) {
  if (expert_sweeps(D) <= 1)
    return dense_path(D) ? dense_ws_offset(D) + dense_ws_bytes(D) : acc_bytes(D);
  size_t b = 0;
  carve_sweeps(D, nullptr, &b);
  return b;
}

template <typename T, int NV>
cudaError_t launch_slices(const Dims& D, const void* x, const void* W, const void* V,
                          const int32_t* tt, const int32_t* te, const float* tg, float* acc,
                          int32_t* status, cudaStream_t s, const void* U) {
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
  OMNI_TRY(launch_k(k_expert_slices<T, NV>, static_cast<unsigned>(blocks), kExpThreads, 0, s,
      static_cast<const T*>(x), static_cast<const T*>(W), static_cast<const T*>(U),
      static_cast<const T*>(V), tt, te, tg, M,
      D.L, D.N(), static_cast<int>(D.d), S, shard_ids(D), acc, status));
  return cudaGetLastError();
}

template <typename T, int NV, int R, bool GLU>
cudaError_t launch_async(const Dims& D, const void* x, const void* W, const void* V,
                         const int32_t* tt, const int32_t* te, const float* tg, float* acc,
                         int32_t* status, cudaStream_t s, const DenseFlags& df, const void* U) {
  constexpr size_t smem = static_cast<size_t>(kAsyncWarps) * R * (GLU ? 3 : 2) * NV * 32 * 16;
  cudaError_t err = cudaFuncSetAttribute(k_expert_async<T, NV, R, GLU>,
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
  OMNI_TRY(launch_k(k_expert_async<T, NV, R, GLU>, static_cast<unsigned>(blocks), kAsyncWarps * 32,
      smem, s, static_cast<const T*>(x), static_cast<const T*>(W), static_cast<const T*>(U),
      static_cast<const T*>(V), tt, te, tg,
      M, D.L, D.N(), static_cast<int>(D.d), S, nslices, shard_ids(D), acc, status, df.flag,
      df.cbuf));
  return cudaGetLastError();
}

// df: the dense-group activations (flag == nullptr: none).  Row widths
// without a k_expert_async instance take k_expert_slices, which forms every
// activation itself; the dense path is only run for widths that have one.
// U != nullptr: gated experts (a third row per task; fewer ring slots at the
// widest rows so that the ring still fits the shared memory).
template <typename T>
cudaError_t dispatch_slices(const Dims& D, const void* x, const void* W, const void* V,
                            const int32_t* tt, const int32_t* te, const float* tg, float* acc,
                            int32_t* status, cudaStream_t s, const DenseFlags& df,
                            const void* U) {
  constexpr int row = 32 * kEpv<T>;  // elements covered by one vector per lane
  const int nv = D.d == row * 8 ? 8 : D.d == row * 4 ? 4 : D.d == row * 2 ? 2 : D.d == row ? 1 : 0;
  if (U != nullptr) {
    switch (nv) {
      case 8: return launch_async<T, 8, 2, true>(D, x, W, V, tt, te, tg, acc, status, s, df, U);
      case 4: return launch_async<T, 4, 3, true>(D, x, W, V, tt, te, tg, acc, status, s, df, U);
      case 2: return launch_async<T, 2, 4, true>(D, x, W, V, tt, te, tg, acc, status, s, df, U);
      case 1: return launch_async<T, 1, 4, true>(D, x, W, V, tt, te, tg, acc, status, s, df, U);
      default: return launch_slices<T, 0>(D, x, W, V, tt, te, tg, acc, status, s, U);
    }
  }
  switch (nv) {
    case 8: return launch_async<T, 8, 3, false>(D, x, W, V, tt, te, tg, acc, status, s, df, U);
    case 4: return launch_async<T, 4, 4, false>(D, x, W, V, tt, te, tg, acc, status, s, df, U);
    case 2: return launch_async<T, 2, 4, false>(D, x, W, V, tt, te, tg, acc, status, s, df, U);
    case 1: return launch_async<T, 1, 4, false>(D, x, W, V, tt, te, tg, acc, status, s, df, U);
    default: return launch_slices<T, 0>(D, x, W, V, tt, te, tg, acc, status, s, U);
  }
}

int sm_count() {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return sms;
}

// About one window per SM of a B200 (148), within what one CTA sorts.  A
// function of the batch alone, not of the device queried: workspace sizes
// computed before a launch hold for it on any device.
int64_t window_tasks(const Dims& D) {
  constexpr int64_t kWindowsPerBatch = 148;
  const int64_t T = (D.M() + kWindowsPerBatch - 1) / kWindowsPerBatch;
  return T < 1024 ? 1024 : (T > kWinTasks ? kWinTasks : T);
}

constexpr size_t kWsortSmem = static_cast<size_t>(kBlockSortMax) * (2 * 4 + 3 * 2) +
                              static_cast<size_t>(kBlockSortWarps) * 256 * 4;

// win_lo != nullptr: the tasks are in window token order already (wt/we/wg),
// and only the expert order is left to make
cudaError_t launch_wsort(const Dims& D, const int32_t* tt, const int32_t* te, const float* tg,
                         const int32_t* group_off, const int32_t* counts, const SweepWs& w,
                         const int32_t* win_lo, float* zslice, int zcols, int64_t zld,
                         int32_t* status, cudaStream_t s) {
  const int64_t M = D.M();
  const int64_t T = window_tasks(D);
  const int64_t nwin = (M + T - 1) / T;
  if (win_lo != nullptr) {
    cudaError_t err = cudaFuncSetAttribute(k_wsort_x, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           static_cast<int>(kWsortSmem));
    if (err != cudaSuccess) return err;
    OMNI_TRY(launch_k(k_wsort_x, static_cast<unsigned>(nwin), kBlockSortThreads, kWsortSmem, s,
        win_lo, w.win, zslice, D.L, zcols, zld));
    return cudaGetLastError();
  }
  constexpr size_t smem = kWsortSmem;
  cudaError_t err = cudaFuncSetAttribute(k_wsort, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
  if (err != cudaSuccess) return err;
  int bits = 0;
  while ((int64_t(1) << bits) < D.L) ++bits;
  const int passes = (bits + 7) / 8;
  OMNI_TRY(launch_k(k_wsort, static_cast<unsigned>(nwin), kBlockSortThreads, smem, s, tt, te, tg,
      group_off, counts, M, D.gmax(), static_cast<int>(T), passes, w.win, status, zslice, D.L,
      zcols, zld));
  return cudaGetLastError();
}

template <typename T, int NB, int D>
cudaError_t launch_acc(const Dims& D_, int col0, const void* V, const SweepWs& w, float* acc,
                       int64_t ld, cudaStream_t s) {
  int per_sm = 1;
  cudaError_t err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_acc<T, NB, D>,
                                                                  kAccWarps * 32, 0);
  if (err != cudaSuccess) return err;
  if (per_sm < 1) per_sm = 1;
  const int64_t M = D_.M();
  const int64_t nslices = (M + 31) / 32;
  int64_t blocks = (nslices + kAccWarps - 1) / kAccWarps;
  const int64_t cap = static_cast<int64_t>(sm_count()) * per_sm;
  if (blocks > cap) blocks = cap;
  OMNI_TRY(launch_k(k_acc<T, NB, D>, static_cast<unsigned>(blocks), kAccWarps * 32, 0, s,
      static_cast<const T*>(V), w.win.wt, w.win.we, w.cbuf, M, D_.L, D_.N(), static_cast<int>(D_.d),
      col0, nslices, shard_ids(D_), acc, ld));
  return cudaGetLastError();
}

cudaError_t launch_finish(const Dims& D, const float* src, int64_t src_ld, __nv_bfloat16* y,
                          float* zdst, int64_t z_ld, int cols, bool discard, cudaStream_t s) {
  if (src == nullptr && zdst == nullptr) return cudaSuccess;
  const int64_t threads = D.L * (cols / 8);
  OMNI_TRY(launch_k(k_slice_finish, static_cast<unsigned>((threads + 255) / 256), 256, 0, s, src,
      src_ld, y, static_cast<int64_t>(D.d), zdst, z_ld, D.L, cols, discard ? 1 : 0));
  return cudaGetLastError();
}

// ycast: the bf16 output (nullptr for fp32, whose accumulator is y itself).
template <typename T, int NV, int NVQ>
cudaError_t sweeps_nv(const Dims& D, int Q, const void* x, const void* W, const void* V,
                      const int32_t* tt, const int32_t* te, const float* tg,
                      const int32_t* group_off, const int32_t* counts, const SweepWs& w,
                      const int32_t* win_lo, float* acc, __nv_bfloat16* ycast, int32_t* status,
                      cudaStream_t s, const void* U) {
  const int cols = static_cast<int>(D.d / Q);
  // bf16: one compact fp32 slice [L x cols] serves every sweep -- zeroed
  // before the first, then rounded into y's columns and zeroed in place
  // (its lines stay in L2) between sweeps, and dropped after the last.
  // fp32: the slices are y's own columns.  The window sort clears the first
  // slice.
  const int64_t ld = ycast ? cols : D.d;
  auto slice = [&](int q) { return ycast ? acc : acc + static_cast<int64_t>(q) * cols; };
  cudaError_t err = launch_wsort(D, tt, te, tg, group_off, counts, w, win_lo, slice(0), cols, ld,
                                 status, s);
  if (err != cudaSuccess) return err;
  // three ring slots per warp: two rows in flight, two CTAs (16 warps) per SM
  // (gated experts: a W and a U row per slot, one CTA per SM)
  constexpr int R = 3;
  const int64_t M = D.M();
  const int S = 32;
  const int64_t nslices = (M + S - 1) / S;
  int64_t blocks = (nslices + kActWarps - 1) / kActWarps;
  // tasks by expert: x[t] held per run of one token, the W rows through the
  // ring (an expert's repeated row comes from L2 right after its first read)
  auto act = [&](auto kernel, int per_sm, size_t smem) -> cudaError_t {
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    const int64_t b = blocks > per_sm * sm_count() ? per_sm * sm_count() : blocks;
    OMNI_TRY(launch_k(kernel, static_cast<unsigned>(b), kActWarps * 32, smem, s,
        static_cast<const T*>(x), w.win.xt, D.L, static_cast<const T*>(W),
        static_cast<const T*>(U), w.win.xe, D.N(), shard_ids(D), w.win.xg, w.win.xdst, M,
        static_cast<int>(D.d), S, nslices, w.cbuf, status));
    return cudaGetLastError();
  };
  err = U != nullptr
            ? act(k_act<T, NV, R, true, true>, 1, static_cast<size_t>(kActWarps) * R * 2 * NV * 32 * 16)
            : act(k_act<T, NV, R, true, false>, 2, static_cast<size_t>(kActWarps) * R * NV * 32 * 16);
  if (err != cudaSuccess) return err;
  // 128-column blocks per slice and the prefetch distance (about 16 vectors
  // of loads in flight per lane)
  constexpr int NB = NVQ * 32 * kEpv<T> / 128;
  constexpr int PD = 8 / NVQ;
  for (int q = 0; q < Q && err == cudaSuccess; ++q) {
    err = launch_acc<T, NB, PD>(D, q * cols, V, w, slice(q), ld, s);
    if (err != cudaSuccess) break;
    const bool last = q + 1 == Q;
    err = launch_finish(D, ycast ? acc : nullptr, ld, ycast ? ycast + static_cast<int64_t>(q) * cols : nullptr,
                        last ? nullptr : slice(q + 1), ld, cols, last, s);
  }
  return err;
}

template <typename T>
cudaError_t launch_sweeps(const Dims& D, int Q, const void* x, const void* W, const void* V,
                          const int32_t* tt, const int32_t* te, const float* tg,
                          const int32_t* group_off, const int32_t* counts, const SweepWs& w,
                          const int32_t* win_lo, float* acc, __nv_bfloat16* ycast,
                          int32_t* status, cudaStream_t s, const void* U) {
  constexpr int row = 32 * kEpv<T>;
  const int64_t nv = D.d / row;             // vectors per lane for a whole row
  const int64_t nvq = (D.d / Q) / row;      // ... for one slice
  if (D.d % row != 0) return cudaErrorInvalidValue;
#define OMNI_SWEEP(NV_, NVQ_)                                                               \
  if (nv == NV_ && nvq == NVQ_)                                                             \
    return sweeps_nv<T, NV_, NVQ_>(D, Q, x, W, V, tt, te, tg, group_off, counts, w, win_lo, \
                                   acc, ycast, status, s, U);
  OMNI_SWEEP(8, 4) OMNI_SWEEP(8, 2) OMNI_SWEEP(8, 1) OMNI_SWEEP(4, 2) OMNI_SWEEP(4, 1)
  OMNI_SWEEP(2, 1)
#undef OMNI_SWEEP
  return cudaErrorInvalidValue;
}

cudaError_t launch_expert(const Dims& D, const void* x, const void* W, const void* V,
                          const int32_t* task_token, const int32_t* task_expert,
                          const float* task_gate, const int32_t* uniq, const int32_t* group_off,
                          const int32_t* counts, void* y, void* ws, cudaStream_t s,
                          bool acc_zeroed, bool allow_dense, const void* U) {
  if (D.L == 0) return cudaSuccess;
  const bool f32 = D.dtype == OMNI_F32;
  // fp32 storage and a shard's partial sum accumulate in y itself
  const bool out32 = f32 || D.sharded();
  float* acc = out32 ? static_cast<float*>(y) : static_cast<float*>(ws);
  int32_t* status = const_cast<int32_t*>(counts) + 2;
  const int Q = expert_sweeps(D);
  if (Q > 1) {  // the sweeps zero, accumulate and cast slice by slice
    const SweepWs w = carve_sweeps(D, ws, nullptr);
    __nv_bfloat16* ycast = out32 ? nullptr : static_cast<__nv_bfloat16*>(y);
    return f32 ? launch_sweeps<float>(D, Q, x, W, V, task_token, task_expert, task_gate,
                                      group_off, counts, w, nullptr, acc, ycast, status, s, U)
               : launch_sweeps<__nv_bfloat16>(D, Q, x, W, V, task_token, task_expert, task_gate,
                                              group_off, counts, w, nullptr, acc, ycast, status,
                                              s, U);
  }
  cudaError_t err = acc_zeroed ? cudaSuccess
                               : launch_zero(acc, static_cast<size_t>(expert_acc_words(D)), s);
  if (err != cudaSuccess) return err;
  DenseFlags df{nullptr, nullptr};
  if (allow_dense && U == nullptr && !D.sharded() && uniq != nullptr && dense_path(D)) {
    void* dws = static_cast<char*>(ws) + dense_ws_offset(D);
    OMNI_TRY(launch_dense_activations(D, x, W, task_token, task_expert, task_gate, uniq,
                                      group_off, const_cast<int32_t*>(counts), dws, s));
    df = dense_flags(D, dws);
  }
  err = f32 ? dispatch_slices<float>(D, x, W, V, task_token, task_expert, task_gate, acc, status,
                                     s, df, U)
            : dispatch_slices<__nv_bfloat16>(D, x, W, V, task_token, task_expert, task_gate, acc,
                                             status, s, df, U);
  if (err != cudaSuccess || out32) return err;
  const int64_t n = D.L * D.d;
  OMNI_TRY(launch_k(k_cast, static_cast<unsigned>((n / 8 + 255) / 256), 256, 0, s, acc,
      static_cast<__nv_bfloat16*>(y), n));
  return cudaGetLastError();
}

int64_t expert_acc_words(const Dims& D) {
  return expert_sweeps(D) > 1 ? 0 : D.L * D.d;
}

WinTasks expert_windows(const Dims& D, void* ws) {
  const SweepWs w = carve_sweeps(D, ws, nullptr);
  return WinTasks{w.win.wt, w.win.we, w.win.wg, w.win_lo};
}

cudaError_t launch_expert_windows(const Dims& D, const void* x, const void* W, const void* V,
                                  int32_t* counts, void* y, void* ws, cudaStream_t s,
                                  const void* U) {
  const int Q = expert_sweeps(D);
  if (D.L == 0 || Q <= 1) return cudaErrorInvalidValue;
  const bool f32 = D.dtype == OMNI_F32;
  const bool out32 = f32 || D.sharded();  // the accumulator is y itself
  float* acc = out32 ? static_cast<float*>(y) : static_cast<float*>(ws);
  int32_t* status = counts + 2;
  const SweepWs w = carve_sweeps(D, ws, nullptr);
  __nv_bfloat16* ycast = out32 ? nullptr : static_cast<__nv_bfloat16*>(y);
  return f32 ? launch_sweeps<float>(D, Q, x, W, V, nullptr, nullptr, nullptr, nullptr, counts, w,
                                    w.win_lo, acc, ycast, status, s, U)
             : launch_sweeps<__nv_bfloat16>(D, Q, x, W, V, nullptr, nullptr, nullptr, nullptr,
                                            counts, w, w.win_lo, acc, ycast, status, s, U);
}

namespace {
__global__ void __launch_bounds__(256) k_zero_words(uint32_t* __restrict__ p, int64_t n) {
  pdl_wait();
  pdl_trigger();
  const int64_t i = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) * 4;
  if (i + 3 < n && (reinterpret_cast<uintptr_t>(p) & 15) == 0) {
    *reinterpret_cast<uint4*>(p + i) = make_uint4(0u, 0u, 0u, 0u);
  } else {
    for (int64_t j = i; j < n && j < i + 4; ++j) p[j] = 0u;
  }
}
}  // namespace

cudaError_t launch_zero(void* p, size_t n_words, cudaStream_t s) {
  if (n_words == 0) return cudaSuccess;
  const int64_t n = static_cast<int64_t>(n_words);
  return launch_k(k_zero_words, static_cast<unsigned>((n / 4 + 256) / 256), 256, 0, s,
                  static_cast<uint32_t*>(p), n);
}

cudaError_t launch_cast_output(const Dims& D, const float* src, void* y, cudaStream_t s) {
  const int64_t n = D.L * D.d;
  if (n == 0) return cudaSuccess;
  if (D.dtype == OMNI_F32) {
    if (src == y) return cudaSuccess;
    return cudaMemcpyAsync(y, src, static_cast<size_t>(n) * sizeof(float),
                           cudaMemcpyDeviceToDevice, s);
  }
  OMNI_TRY(launch_k(k_cast, static_cast<unsigned>((n / 8 + 255) / 256), 256, 0, s, src,
      static_cast<__nv_bfloat16*>(y), n));
  return cudaGetLastError();
}

cudaError_t launch_token(const Dims& D, const void* x, const void* W, const void* V,
                         const int32_t* idx, const float* gate, void* y, int32_t* status,
                         cudaStream_t s, const void* U) {
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
    OMNI_TRY(launch_k(k_token_centric<float>, static_cast<unsigned>(D.L), kTokThreads, smem, s,
        static_cast<const float*>(x), static_cast<const float*>(W), static_cast<const float*>(U),
        static_cast<const float*>(V), idx, gate, static_cast<int>(D.K), static_cast<int>(D.d),
        D.N(), static_cast<float*>(y), status));
  } else {
    err = cudaFuncSetAttribute(k_token_centric<__nv_bfloat16>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (err != cudaSuccess) return err;
    OMNI_TRY(launch_k(k_token_centric<__nv_bfloat16>, static_cast<unsigned>(D.L), kTokThreads, smem,
        s, static_cast<const __nv_bfloat16*>(x), static_cast<const __nv_bfloat16*>(W),
        static_cast<const __nv_bfloat16*>(U), static_cast<const __nv_bfloat16*>(V), idx, gate,
        static_cast<int>(D.K),
        static_cast<int>(D.d), D.N(), static_cast<__nv_bfloat16*>(y), status));
  }
  return cudaGetLastError();
}

}  // namespace omni
