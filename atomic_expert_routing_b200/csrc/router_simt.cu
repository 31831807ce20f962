// Router logits on CUDA cores: Z[t, :Nr] = x[t] Wr^T, Z[t, Nr:] = x[t] Wc^T
// (fp32 accumulation).  Used for fp32 storage -- tf32 tensor cores would not
// keep the fp32 logits exact enough -- and as a diagnostic path for bf16.
//
// "OmniMoE: An Efficient MoE by Orchestrating Atomic Experts at Scale"
// (gist.science), Technisch Overzicht section 2.2: two low-dimensional
// projections give the row and column logits of the Cartesian Product Router.
#include "common.cuh"
#include "internal.h"

namespace omni {
namespace {

constexpr int TM = 64, TN = 64, TK = 16;

template <typename T>
__global__ void __launch_bounds__(256) k_router_simt(const T* __restrict__ x,
                                                     const T* __restrict__ Wr,
                                                     const T* __restrict__ Wc,
                                                     float* __restrict__ Z, int64_t L, int Nr,
                                                     int Nc, int d, int tiles_r) {
  pdl_wait();
  pdl_trigger();
  __shared__ float As[TK][TM + 4];
  __shared__ float Bs[TK][TN + 4];
  const int tid = threadIdx.x;
  const int64_t m0 = static_cast<int64_t>(blockIdx.x) * TM;
  const bool colax = static_cast<int>(blockIdx.y) >= tiles_r;
  const int n0 = (colax ? static_cast<int>(blockIdx.y) - tiles_r : static_cast<int>(blockIdx.y)) * TN;
  const int naxis = colax ? Nc : Nr;
  const T* Wa = colax ? Wc : Wr;
  const int ty = tid / 16, tx = tid % 16;  // 16 x 16 threads, 4 x 4 outputs each
  float acc[4][4] = {};
  for (int k0 = 0; k0 < d; k0 += TK) {
    // 64 x 16 tiles of x and of the axis keys: 4 elements per thread each
    for (int r = 0; r < 4; ++r) {
      const int li = tid + 256 * r;
      const int row = li / TK, kk = li % TK;
      const int64_t gm = m0 + row;
      const int gk = k0 + kk;
      As[kk][row] = (gm < L && gk < d) ? to_float(x[gm * d + gk]) : 0.0f;
      const int gn = n0 + row;
      Bs[kk][row] = (gn < naxis && gk < d) ? to_float(Wa[static_cast<int64_t>(gn) * d + gk]) : 0.0f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < TK; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        a[i] = As[kk][ty * 4 + i];
        b[i] = Bs[kk][tx * 4 + i];
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
  const int64_t ld = Nr + Nc;
  const int zc0 = (colax ? Nr : 0);
  for (int i = 0; i < 4; ++i) {
    const int64_t gm = m0 + ty * 4 + i;
    if (gm >= L) continue;
    for (int j = 0; j < 4; ++j) {
      const int gn = n0 + tx * 4 + j;
      if (gn < naxis) Z[gm * ld + zc0 + gn] = acc[i][j];
    }
  }
}

}  // namespace

cudaError_t launch_router_simt(const Dims& D, const void* x, const void* Wr, const void* Wc,
                               float* Z, cudaStream_t s) {
  if (D.L == 0) return cudaSuccess;
  const int tiles_r = static_cast<int>((D.Nr + TN - 1) / TN);
  const int tiles_c = static_cast<int>((D.Nc + TN - 1) / TN);
  dim3 grid(static_cast<unsigned>((D.L + TM - 1) / TM), tiles_r + tiles_c);
  if (D.dtype == OMNI_F32)
    OMNI_TRY(launch_k(k_router_simt<float>, grid, 256, 0, s, static_cast<const float*>(x),
        static_cast<const float*>(Wr), static_cast<const float*>(Wc), Z, D.L,
        static_cast<int>(D.Nr), static_cast<int>(D.Nc), static_cast<int>(D.d), tiles_r));
  else
    OMNI_TRY(launch_k(k_router_simt<__nv_bfloat16>, grid, 256, 0, s,
        static_cast<const __nv_bfloat16*>(x), static_cast<const __nv_bfloat16*>(Wr),
        static_cast<const __nv_bfloat16*>(Wc), Z, D.L, static_cast<int>(D.Nr),
        static_cast<int>(D.Nc), static_cast<int>(D.d), tiles_r));
  return cudaGetLastError();
}

}  // namespace omni
