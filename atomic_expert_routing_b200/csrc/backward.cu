// Backward of the routed branch: the gradients of the loss sum(dy * y) with
// the forward's routing fixed (the pages train the model: "OmniMoE: An
// Efficient MoE by Orchestrating Atomic Experts at Scale" (gist.science),
// section 4).  Per task (t, k), e = idx[t,k], with a = x[t] . W[e],
// h = SiLU(a), s = dy[t] . V[e]:
//   dV[e] += gate h dy[t],   dW[e] += da x[t],   dx[t] += da W[e],
//   da = gate s SiLU'(a),    dgate = h s;
// per token, through gate = softmax of the selected joint scores
// S_k = lr[i_k] + lc[j_k]:  dS_k = gate_k (dgate_k - sum_q gate_q dgate_q),
// added to the row logit i_k and the column logit j_k.  The per-axis
// log-softmax adds -softmax(z) * sum(dS) to the logit gradients, and sum(dS)
// is zero (the gates sum to one), so the logit gradients are the dS sums
// themselves.  Then, with dZ = [dzr | dzc] [L x (Nr + Nc)]:
//   dx += dZ [Wr; Wc],   [dWr; dWc] += dZ^T x,   dbias += column sums of dZ.
//
// Kernels, all on one stream:
//  1. the schedule with groups of one expert (omni_schedule with B = 1):
//     each expert's tasks adjacent, in token order;
//  2. k_bwd_expert: a warp per expert reads its W and V rows, computes every
//     task's scalars (a, s, da, dgate), writes da and dgate to the task's
//     slot t*K + k, and adds its row gradients dW[e], dV[e] (fp32) once per
//     32 tasks -- no atomics, an expert belongs to one warp.  A call that
//     does not accumulate writes the rows with the first 32 tasks instead of
//     adding to them, without reading them;
//  3. k_bwd_token: a CTA per token forms dS, its dZ row (bf16, the GEMM
//     operand; fp32 atomics into the bias gradients) and dx[t] = sum_k da_k
//     W[e_k] (fp32);
//  4. transposes to K-major bf16 operands, then two tcgen05 GEMMs with fp32
//     accumulation: dx += dZ [Wr; Wc] and [dWr; dWc] += dZ^T x (= when the
//     call does not accumulate; the bias gradients are then cleared first).
// bf16 storage only (the GEMM operands; dZ is rounded to bf16 for them).
#include "common.cuh"
#include "gemm_tc.cuh"
#include "internal.h"

namespace omni {
namespace {

using namespace tc;
using bf16 = __nv_bfloat16;

constexpr int kBwdWarps = 8;
constexpr int kTokThreadsB = 256;
static_assert(kTokThreadsB >= OMNI_MAX_TOPK, "k_bwd_token: a thread per task of a token");

__device__ __forceinline__ float silu_grad(float z) {
  const float sg = 1.0f / (1.0f + expf(-z));
  return sg * (1.0f + z * (1.0f - sg));
}

// dot of two vectors of 8 bf16
__device__ __forceinline__ float dot8(uint4 a, uint4 b) {
  const uint32_t* pa = reinterpret_cast<const uint32_t*>(&a);
  const uint32_t* pb = reinterpret_cast<const uint32_t*>(&b);
  float s = 0.0f;
#pragma unroll
  for (int q = 0; q < 4; ++q) s += bf16lo(pa[q]) * bf16lo(pb[q]) + bf16hi(pa[q]) * bf16hi(pb[q]);
  return s;
}

// acc[0..8) += c * v (8 bf16)
__device__ __forceinline__ void axpy8(float c, uint4 v, float* acc) {
  const uint32_t* p = reinterpret_cast<const uint32_t*>(&v);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    acc[2 * q] += c * bf16lo(p[q]);
    acc[2 * q + 1] += c * bf16hi(p[q]);
  }
}

// o[0..8) += acc, or = acc without reading o (add == false); fp32,
// 32-byte aligned
__device__ __forceinline__ void put8(float* o, const float* acc, bool add) {
  float4* p = reinterpret_cast<float4*>(o);
  float4 u = make_float4(acc[0], acc[1], acc[2], acc[3]);
  float4 w = make_float4(acc[4], acc[5], acc[6], acc[7]);
  if (add) {
    const float4 a = p[0], b = p[1];
    u.x += a.x; u.y += a.y; u.z += a.z; u.w += a.w;
    w.x += b.x; w.y += b.y; w.z += b.z; w.w += b.w;
  }
  p[0] = u;
  p[1] = w;
}

// One warp per group of a B = 1 schedule (one expert, its tasks in token
// order), 32 tasks at a time.  Lane j keeps task j's da and gate * h.
__global__ void __launch_bounds__(kBwdWarps * 32)
    k_bwd_expert(const bf16* __restrict__ x, const bf16* __restrict__ W,
                 const bf16* __restrict__ V, const bf16* __restrict__ dy,
                 const int32_t* __restrict__ task_token, const int32_t* __restrict__ task_expert,
                 const float* __restrict__ task_gate, const int32_t* __restrict__ group_off,
                 const int32_t* __restrict__ counts, const int32_t* __restrict__ idx, int64_t L,
                 int K, int64_t N, int d, int64_t gmax, int accumulate, float* __restrict__ dW,
                 float* __restrict__ dV, float* __restrict__ da_slot,
                 float* __restrict__ dg_slot, int32_t* status) {
  pdl_wait();
  pdl_trigger();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t M = L * K;
  int64_t G = counts[1];
  G = G < 0 ? 0 : (G > gmax ? gmax : G);
  const int nvec = d / 8;
  const int64_t nw = static_cast<int64_t>(gridDim.x) * kBwdWarps;
  for (int64_t g = static_cast<int64_t>(blockIdx.x) * kBwdWarps + warp; g < G; g += nw) {
    const int64_t a0 = group_off[g], a1 = group_off[g + 1];
    if (a0 < 0 || a1 > M || a1 <= a0) {  // warp-uniform
      if (lane == 0) raise_status(status, OMNI_DEV_BAD_INDEX);
      continue;
    }
    const int64_t e = task_expert[a0];
    if (e < 0 || e >= N) {
      if (lane == 0) raise_status(status, OMNI_DEV_BAD_INDEX);
      continue;
    }
    const uint4* wr = reinterpret_cast<const uint4*>(W + e * d);
    const uint4* vr = reinterpret_cast<const uint4*>(V + e * d);
    for (int64_t c0 = a0; c0 < a1; c0 += 32) {
      const int n = static_cast<int>(a1 - c0 < 32 ? a1 - c0 : 32);
      int64_t my_t = -1;
      float my_g = 0.0f;
      if (lane < n) {
        my_t = task_token[c0 + lane];
        my_g = task_gate[c0 + lane];
        if (my_t < 0 || my_t >= L || task_expert[c0 + lane] != e) {
          raise_status(status, OMNI_DEV_BAD_INDEX);
          my_t = -1;
        }
      }
      float my_da = 0.0f, my_cv = 0.0f;
      // the scalars of every task
      for (int j = 0; j < n; ++j) {
        const int64_t t = __shfl_sync(0xffffffffu, my_t, j);
        const float gj = __shfl_sync(0xffffffffu, my_g, j);
        if (t < 0) continue;  // warp-uniform
        const uint4* xr = reinterpret_cast<const uint4*>(x + t * d);
        const uint4* dr = reinterpret_cast<const uint4*>(dy + t * d);
        float sa = 0.0f, ss = 0.0f;
        for (int v = lane; v < nvec; v += 32) {
          sa += dot8(xr[v], wr[v]);
          ss += dot8(dr[v], vr[v]);
        }
        sa = warp_sum(sa);
        ss = warp_sum(ss);
        const float h = silu(sa);
        const float dav = gj * ss * silu_grad(sa);
        if (lane == j) {
          my_da = dav;
          my_cv = gj * h;
        }
        // the task's slot: the position of e among the token's K ids
        int kpos = -1;
        for (int k0 = 0; k0 < K; k0 += 32) {
          const int k = k0 + lane;
          const uint32_t m = __ballot_sync(0xffffffffu, k < K && idx[t * K + k] == e);
          if (m != 0u) {
            kpos = k0 + __ffs(m) - 1;
            break;
          }
        }
        if (kpos < 0) {  // warp-uniform: e is not among the token's ids
          if (lane == 0) raise_status(status, OMNI_DEV_BAD_INDEX);
          continue;
        }
        if (lane == 0) {
          da_slot[t * K + kpos] = dav;
          dg_slot[t * K + kpos] = h * ss;
        }
      }
      // the row gradients, 8 columns per lane and step
      for (int v0 = 0; v0 < nvec; v0 += 32) {
        const int v = v0 + lane;
        float aw[8], av[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) aw[u] = av[u] = 0.0f;
        for (int j = 0; j < n; ++j) {
          const int64_t t = __shfl_sync(0xffffffffu, my_t, j);
          const float daj = __shfl_sync(0xffffffffu, my_da, j);
          const float cvj = __shfl_sync(0xffffffffu, my_cv, j);
          if (t < 0 || v >= nvec) continue;
          axpy8(daj, reinterpret_cast<const uint4*>(x + t * d)[v], aw);
          axpy8(cvj, reinterpret_cast<const uint4*>(dy + t * d)[v], av);
        }
        if (v < nvec) {
          // the expert's first 32 tasks overwrite its rows unless the call
          // accumulates; later ones add to what the first wrote
          const bool add = accumulate != 0 || c0 > a0;
          put8(dW + e * d + static_cast<int64_t>(v) * 8, aw, add);
          put8(dV + e * d + static_cast<int64_t>(v) * 8, av, add);
        }
      }
    }
  }
}

// One CTA per token: dS of its K tasks, its dZ row (bf16, zero-padded to Kp
// columns), the bias gradients (fp32 atomics), and dx[t] = sum_k da_k W[e_k].
__global__ void __launch_bounds__(kTokThreadsB)
    k_bwd_token(const bf16* __restrict__ W, const int32_t* __restrict__ idx,
                const float* __restrict__ gate, const float* __restrict__ da_slot,
                const float* __restrict__ dg_slot, int K, int64_t Nr, int64_t Nc, int d,
                int64_t Kp, float* __restrict__ dx, bf16* __restrict__ dzb,
                float* __restrict__ dbr, float* __restrict__ dbc, int32_t* status) {
  extern __shared__ float dz[];  // [Nr + Nc]
  __shared__ int64_t es[256];
  __shared__ float das[256];
  __shared__ float red[kTokThreadsB / 32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t t = blockIdx.x;
  const int64_t N = Nr * Nc, nz = Nr + Nc;
  for (int64_t i = tid; i < nz; i += kTokThreadsB) dz[i] = 0.0f;
  pdl_wait();
  pdl_trigger();
  float gk = 0.0f, dgk = 0.0f;
  int64_t ek = -1;
  if (tid < K) {
    ek = idx[t * K + tid];
    if (ek < 0 || ek >= N) {
      raise_status(status, OMNI_DEV_BAD_INDEX);
      ek = -1;
    } else {
      gk = gate[t * K + tid];
      dgk = dg_slot[t * K + tid];
    }
    es[tid] = ek;
    das[tid] = ek >= 0 ? da_slot[t * K + tid] : 0.0f;
  }
  // sum_q gate_q dgate_q
  float p = warp_sum(gk * dgk);
  if (lane == 0) red[warp] = p;
  __syncthreads();
  float gdg = 0.0f;
#pragma unroll
  for (int w = 0; w < kTokThreadsB / 32; ++w) gdg += red[w];
  if (ek >= 0) {
    const float dS = gk * (dgk - gdg);
    atomicAdd(&dz[ek / Nc], dS);
    atomicAdd(&dz[Nr + ek % Nc], dS);
  }
  __syncthreads();
  for (int64_t i = tid; i < Kp; i += kTokThreadsB) {
    const float v = i < nz ? dz[i] : 0.0f;
    dzb[t * Kp + i] = __float2bfloat16_rn(v);
    if (v != 0.0f) {
      if (i < Nr) {
        if (dbr != nullptr) atomicAdd(&dbr[i], v);
      } else if (dbc != nullptr) {
        atomicAdd(&dbc[i - Nr], v);
      }
    }
  }
  // dx (the experts' part)
  const int nvec = d / 8;
  for (int v = tid; v < nvec; v += kTokThreadsB) {
    float acc[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) acc[u] = 0.0f;
    for (int k = 0; k < K; ++k) {
      const int64_t e = es[k];
      if (e < 0) continue;
      axpy8(das[k], reinterpret_cast<const uint4*>(W + e * d)[v], acc);
    }
    float4* o = reinterpret_cast<float4*>(dx + t * d + static_cast<int64_t>(v) * 8);
    o[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
    o[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
  }
}

// dst[c * ld_dst + r] = r < rows ? src[r * ld_src + c] : 0, for c < cols and
// r < rows_out: a 32 x 32 tile per CTA through shared memory.
__global__ void __launch_bounds__(256)
    k_transpose16(const uint16_t* __restrict__ src, int64_t rows, int64_t cols, int64_t ld_src,
                  uint16_t* __restrict__ dst, int64_t ld_dst, int64_t rows_out) {
  __shared__ uint16_t tile[32][33];
  pdl_wait();
  pdl_trigger();
  const int64_t r0 = static_cast<int64_t>(blockIdx.x) * 32, c0 = static_cast<int64_t>(blockIdx.y) * 32;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;  // 32 x 8
  for (int i = ty; i < 32; i += 8) {
    const int64_t r = r0 + i, c = c0 + tx;
    tile[i][tx] = (r < rows && c < cols) ? src[r * ld_src + c] : static_cast<uint16_t>(0);
  }
  __syncthreads();
  for (int i = ty; i < 32; i += 8) {
    const int64_t c = c0 + i, r = r0 + tx;
    if (c < cols && r < rows_out) dst[c * ld_dst + r] = tile[tx][i];
  }
}

// GEMM epilogue: D[row, col] += acc (accumulate != 0) or = acc (fp32; rows
// of ld floats), rows below `split` in D0 and the others in D1 (row - split).
struct AddF32Split {
  static constexpr size_t kStageBytes = 0;
  float* D0;
  float* D1;
  int64_t split, ld;
  int rows, cols, accumulate;
  __device__ __forceinline__ void operator()(int, int a0, int b0, int r, int c,
                                             const uint32_t* v, float*) const {
    const int row = a0 + r;
    if (row >= rows) return;
    const int col = b0 + c;
    float* o = row < split ? D0 + static_cast<int64_t>(row) * ld + col
                           : D1 + static_cast<int64_t>(row - split) * ld + col;
    if (col + 32 <= cols) {
#pragma unroll
      for (int q = 0; q < 32; q += 4) {
        float4 u = make_float4(__uint_as_float(v[q]), __uint_as_float(v[q + 1]),
                               __uint_as_float(v[q + 2]), __uint_as_float(v[q + 3]));
        if (accumulate) {
          const float4 a = *reinterpret_cast<const float4*>(o + q);
          u.x += a.x; u.y += a.y; u.z += a.z; u.w += a.w;
        }
        *reinterpret_cast<float4*>(o + q) = u;
      }
    } else {
#pragma unroll
      for (int q = 0; q < 32; ++q)
        if (col + q < cols) o[q] = __uint_as_float(v[q]) + (accumulate ? o[q] : 0.0f);
    }
  }
};

// The contraction lengths of the two products (Nr + Nc and L) padded with
// zeros to whole 64-element k-blocks: no TMA box reaches past a row's end.
int64_t pad_k(int64_t v) { return (v + TC_BK - 1) / TC_BK * TC_BK; }

}  // namespace

BwdWs carve_backward(const Dims& D, void* base, size_t* bytes) {
  Dims D1 = D;
  D1.B = 1;
  Carver c(base);
  BwdWs w{};
  const size_t M = static_cast<size_t>(D.M());
  const int64_t Kp = pad_k(D.Nr + D.Nc), Lp = pad_k(D.L);
  w.task_token = c.take<int32_t>(M);
  w.task_expert = c.take<int32_t>(M);
  w.task_gate = c.take<float>(M);
  w.uniq = c.take<int32_t>(static_cast<size_t>(D1.ucap() > 0 ? D1.ucap() : 1));
  w.group_off = c.take<int32_t>(static_cast<size_t>(D1.gmax()) + 1);
  w.sched = c.take<char>(schedule_ws_bytes(D1));
  w.da = c.take<float>(M);
  w.dg = c.take<float>(M);
  w.dzb = c.take<uint16_t>(static_cast<size_t>(D.L * Kp));
  w.dzT = c.take<uint16_t>(static_cast<size_t>((D.Nr + D.Nc) * Lp));
  w.xT = c.take<uint16_t>(static_cast<size_t>(D.d * Lp));
  w.WrcT = c.take<uint16_t>(static_cast<size_t>(D.d * Kp));
  if (bytes) *bytes = c.off;
  return w;
}

cudaError_t launch_backward(const Dims& D, const void* x, const void* Wr, const void* Wc,
                            const void* W, const void* V, const int32_t* idx, const float* gate,
                            const void* dy, float* dx, float* dW, float* dV, float* dWr,
                            float* dWc, float* dbr, float* dbc, bool accumulate,
                            int32_t* counts, void* ws, cudaStream_t s) {
  if (D.L == 0) return cudaSuccess;
  if (D.dtype != OMNI_BF16 || encode_fn() == nullptr) return cudaErrorNotSupported;
  const BwdWs w = carve_backward(D, ws, nullptr);
  Dims D1 = D;
  D1.B = 1;
  int32_t* status = counts + 2;
  const int64_t Kp = pad_k(D.Nr + D.Nc), Lp = pad_k(D.L);
  const int K = static_cast<int>(D.K);
  const int d = static_cast<int>(D.d);
  // 1. each expert's tasks adjacent
  OMNI_TRY(launch_schedule(D1, idx, gate, w.task_token, w.task_expert, w.task_gate, w.uniq,
                           w.group_off, counts, w.sched, s));
  // 2. per expert: the task scalars and dW, dV
  {
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t want = (D1.gmax() + kBwdWarps - 1) / kBwdWarps;
    const int64_t cap = static_cast<int64_t>(sms) * 8;
    const unsigned blocks = static_cast<unsigned>(want < cap ? (want < 1 ? 1 : want) : cap);
    OMNI_TRY(launch_k(k_bwd_expert, blocks, kBwdWarps * 32, 0, s, static_cast<const bf16*>(x),
        static_cast<const bf16*>(W), static_cast<const bf16*>(V), static_cast<const bf16*>(dy),
        static_cast<const int32_t*>(w.task_token), static_cast<const int32_t*>(w.task_expert),
        static_cast<const float*>(w.task_gate), static_cast<const int32_t*>(w.group_off),
        static_cast<const int32_t*>(counts), idx, D.L, K, D.N(), d, D1.gmax(), accumulate ? 1 : 0,
        dW, dV, w.da, w.dg, status));
  }
  // 3. per token: dS, the dZ row, the bias gradients, dx (experts)
  if (!accumulate) {  // the bias gradients are sums of atomic adds
    if (dbr != nullptr) OMNI_TRY(launch_zero(dbr, static_cast<size_t>(D.Nr), s));
    if (dbc != nullptr) OMNI_TRY(launch_zero(dbc, static_cast<size_t>(D.Nc), s));
  }
  {
    const size_t smem = static_cast<size_t>(D.Nr + D.Nc) * sizeof(float);
    cudaError_t err = cudaFuncSetAttribute(k_bwd_token, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           static_cast<int>(smem));
    if (err != cudaSuccess) return err;
    OMNI_TRY(launch_k(k_bwd_token, static_cast<unsigned>(D.L), kTokThreadsB, smem, s,
        static_cast<const bf16*>(W), idx, gate, static_cast<const float*>(w.da),
        static_cast<const float*>(w.dg), K, D.Nr, D.Nc, d, Kp, dx, reinterpret_cast<bf16*>(w.dzb),
        dbr, dbc, status));
  }
  // 4. K-major operands, then the two products on the tensor cores
  auto transpose = [&](const void* src, int64_t rows, int64_t cols, int64_t ld_src, void* dst,
                       int64_t ld_dst, int64_t rows_out) -> cudaError_t {
    const dim3 grid(static_cast<unsigned>((rows_out + 31) / 32),
                    static_cast<unsigned>((cols + 31) / 32));
    OMNI_TRY(launch_k(k_transpose16, grid, 256, 0, s, static_cast<const uint16_t*>(src), rows,
        cols, ld_src, static_cast<uint16_t*>(dst), ld_dst, rows_out));
    return cudaGetLastError();
  };
  OMNI_TRY(transpose(Wr, D.Nr, D.d, D.d, w.WrcT, Kp, D.Nr));
  OMNI_TRY(transpose(Wc, D.Nc, D.d, D.d, w.WrcT + D.Nr, Kp, Kp - D.Nr));
  OMNI_TRY(transpose(w.dzb, D.L, D.Nr + D.Nc, Kp, w.dzT, Lp, Lp));
  OMNI_TRY(transpose(x, D.L, D.d, D.d, w.xT, Lp, Lp));
  // dx [L x d] += dZ [L x Kp] . WrcT [d x Kp]^T
  OMNI_TRY(gemm_bf16(w.dzb, w.WrcT, D.L, D.d, Kp,
                     AddF32Split{dx, dx, D.L, D.d, static_cast<int>(D.L), d, 1}, status, s));
  // [dWr; dWc] [(Nr + Nc) x d] += dZ^T [(Nr + Nc) x Lp] . xT [d x Lp]^T
  return gemm_bf16(w.dzT, w.xT, D.Nr + D.Nc, D.d, Lp,
                   AddF32Split{dWr, dWc, D.Nr, D.d, static_cast<int>(D.Nr + D.Nc), d,
                               accumulate ? 1 : 0},
                   status, s);
}

}  // namespace omni
