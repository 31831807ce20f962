// The shared dense MLP branch of the OmniMoE layer ("OmniMoE: An Efficient MoE
// by Orchestrating Atomic Experts at Scale" (gist.science), Technisch
// Overzicht section 2.1: an always-on dense MLP beside the routed atomic
// experts; the OmniMoE explainer's ablation table removes it as "w/o shared
// MLP").  With one hidden layer of F units and the experts' scalar SiLU:
//   H = SiLU(x W1^T)  [L x F],   y (+)= H W2^T  [L x d],
// W1 [F x d], W2 [d x F].  Both products are dense, so both run on the
// tensor cores (tcgen05, TMEM accumulators, TMA-staged tiles): the first
// GEMM's epilogue applies SiLU and stores H in bf16 (the second GEMM's A
// operand); the second's adds the product to y -- the routed branch's output
// when the layer is fused -- and rounds once to bf16.
#include "common.cuh"
#include "internal.h"
#include "gemm_tc.cuh"

namespace omni {
namespace {

using namespace tc;

// Eight fp32 values to eight bf16 (nearest even), as one 16-byte vector.
__device__ __forceinline__ uint4 pack8_bf16(const float* f) {
  uint4 u;
  uint32_t* w = reinterpret_cast<uint32_t*>(&u);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const __nv_bfloat162 p = __floats2bfloat162_rn(f[2 * q], f[2 * q + 1]);
    w[q] = *reinterpret_cast<const uint32_t*>(&p);
  }
  return u;
}

// First GEMM: H[row, col] = bf16(SiLU(acc)).  Rows of H are ld elements apart
// (ld a multiple of 8, so 32-column chunks are 16-byte aligned).
struct SiluToHidden {
  static constexpr size_t kStageBytes = 0;
  __nv_bfloat16* H;
  int64_t ld;
  int rows, cols;
  __device__ __forceinline__ void operator()(int, int a0, int b0, int r, int c,
                                             const uint32_t* v, float*) const {
    const int row = a0 + r;
    if (row >= rows) return;
    const int col = b0 + c;
    __nv_bfloat16* o = H + static_cast<int64_t>(row) * ld + col;
    if (col + 32 <= cols) {
#pragma unroll
      for (int q = 0; q < 32; q += 8) {
        float f[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) f[u] = silu(__uint_as_float(v[q + u]));
        *reinterpret_cast<uint4*>(o + q) = pack8_bf16(f);
      }
    } else {
#pragma unroll
      for (int q = 0; q < 32; ++q)
        if (col + q < cols) o[q] = __float2bfloat16_rn(silu(__uint_as_float(v[q])));
    }
  }
};

// Second GEMM: y[row, col] = bf16(acc + (accumulate ? y[row, col] : 0)).
struct AddToOutput {
  static constexpr size_t kStageBytes = 0;
  __nv_bfloat16* Y;
  int64_t ld;
  int rows, cols, accumulate;
  __device__ __forceinline__ void operator()(int, int a0, int b0, int r, int c,
                                             const uint32_t* v, float*) const {
    const int row = a0 + r;
    if (row >= rows) return;
    const int col = b0 + c;
    __nv_bfloat16* o = Y + static_cast<int64_t>(row) * ld + col;
    if (col + 32 <= cols) {
#pragma unroll
      for (int q = 0; q < 32; q += 8) {
        float f[8];
        if (accumulate) {
          const uint4 u = *reinterpret_cast<const uint4*>(o + q);
          f[0] = bf16lo(u.x); f[1] = bf16hi(u.x); f[2] = bf16lo(u.y); f[3] = bf16hi(u.y);
          f[4] = bf16lo(u.z); f[5] = bf16hi(u.z); f[6] = bf16lo(u.w); f[7] = bf16hi(u.w);
        } else {
#pragma unroll
          for (int u = 0; u < 8; ++u) f[u] = 0.0f;
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) f[u] += __uint_as_float(v[q + u]);
        *reinterpret_cast<uint4*>(o + q) = pack8_bf16(f);
      }
    } else {
#pragma unroll
      for (int q = 0; q < 32; ++q) {
        if (col + q >= cols) continue;
        const float base = accumulate ? __bfloat162float(o[q]) : 0.0f;
        o[q] = __float2bfloat16_rn(base + __uint_as_float(v[q]));
      }
    }
  }
};

}  // namespace

size_t mlp_ws_bytes(const Dims& D, int64_t F) {
  return static_cast<size_t>(D.L) * static_cast<size_t>(F) * sizeof(__nv_bfloat16);
}

cudaError_t launch_shared_mlp(const Dims& D, int64_t F, const void* x, const void* W1,
                              const void* W2, void* y, bool accumulate, void* ws, int32_t* status,
                              cudaStream_t s) {
  if (D.L == 0) return cudaSuccess;
  if (D.dtype != OMNI_BF16 || encode_fn() == nullptr) return cudaErrorNotSupported;
  __nv_bfloat16* H = static_cast<__nv_bfloat16*>(ws);
  OMNI_TRY(gemm_bf16(x, W1, D.L, F, D.d,
                     SiluToHidden{H, F, static_cast<int>(D.L), static_cast<int>(F)}, status, s));
  return gemm_bf16(H, W2, D.L, D.d, F,
              AddToOutput{static_cast<__nv_bfloat16*>(y), D.d, static_cast<int>(D.L),
                          static_cast<int>(D.d), accumulate ? 1 : 0},
              status, s);
}

}  // namespace omni
