// Cartesian Product Router, selection half.
//
// "OmniMoE: An Efficient MoE by Orchestrating Atomic Experts at Scale"
// (gist.science), Technisch Overzicht section 2.2, and the OmniMoE explainer
// (manus.space), Cartesian product router section: the router predicts a row
// distribution and a column distribution over an Nr x Nc grid of experts and
// scores expert (i, j) by S_ij = lr[i] + lc[j] in log space, without forming
// the N joint scores.
//
// Per token, two warps work side by side: warp 0 takes the Nr row logits,
// warp 1 the Nc column logits.  Each computes its axis' log-sum-exp and its
// top-k entries by a warp radix select over 64-bit keys
// (order-preserving bits of the logit << 32 | ~index), so ties fall to the
// smaller index.  Warp 0 then forms the joint scores of the k x k candidate
// pairs that can reach the top-K -- pair (a, b) of the sorted axis lists has
// (a+1)(b+1) - 1 pairs that score at least as high, so only pairs with
// (a+1)(b+1) <= K are needed -- and selects the K best by (S desc, e asc),
// again by radix select over (bits of S << 32 | ~e).  The gate is the
// softmax of the K selected joint scores.
//
// Ordering uses the raw fp32 logit sums z_r[i] + z_c[j] (the per-token
// log-sum-exp terms are constants and only enter the reported score), so no
// rounding of a log-sum-exp subtraction can tie two distinct logits.
#include "common.cuh"
#include "internal.h"

namespace omni {
namespace {

__device__ __forceinline__ uint32_t f2ord(float f) {
  uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float ord2f(uint32_t o) {
  uint32_t u = (o & 0x80000000u) ? (o & 0x7fffffffu) : ~o;
  return __uint_as_float(u);
}
__device__ __forceinline__ uint64_t make_key(float v, uint32_t id) {
  return (static_cast<uint64_t>(f2ord(v)) << 32) | static_cast<uint32_t>(~id);
}
__device__ __forceinline__ float key_val(uint64_t k) { return ord2f(static_cast<uint32_t>(k >> 32)); }
__device__ __forceinline__ uint32_t key_id(uint64_t k) { return ~static_cast<uint32_t>(k); }

// Radix select by one warp: the `want` largest of n distinct 64-bit keys
// key(i), written unordered to out[0..want).  hist: 256 words of scratch.
template <typename KeyFn>
__device__ void warp_select_top(KeyFn key, int n, int want, uint64_t* out, uint32_t* hist) {
  const int lane = threadIdx.x & 31;
  if (want >= n) {
    for (int i = lane; i < n; i += 32) out[i] = key(i);
    __syncwarp();
    return;
  }
  uint64_t prefix = 0;
  int need = want;
  int fixed = 0;  // low bit of the key bits fixed so far (64 = none)
  for (int shift = 56; shift >= 0; shift -= 8) {
    for (int b = lane; b < 256; b += 32) hist[b] = 0;
    __syncwarp();
    for (int i = lane; i < n; i += 32) {
      const uint64_t kk = key(i);
      if (shift == 56 || (kk >> (shift + 8)) == (prefix >> (shift + 8)))
        atomicAdd(&hist[(kk >> shift) & 255u], 1u);
    }
    __syncwarp();
    // bins in descending order: lane l owns bins 255-8l ... 248-8l
    uint32_t c[8];
    uint32_t tot = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      c[j] = hist[255 - 8 * lane - j];
      tot += c[j];
    }
    uint32_t incl = tot;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    const uint32_t excl = incl - tot;
    int digit = -1;
    uint32_t above = 0;
    if (excl < static_cast<uint32_t>(need) && static_cast<uint32_t>(need) <= incl) {
      uint32_t run = excl;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (digit < 0 && run + c[j] >= static_cast<uint32_t>(need)) {
          digit = 255 - 8 * lane - j;
          above = run;
        }
        run += c[j];
      }
    }
    const uint32_t who = __ballot_sync(0xffffffffu, digit >= 0);
    const int src = __ffs(who) - 1;
    digit = __shfl_sync(0xffffffffu, digit, src);
    above = __shfl_sync(0xffffffffu, above, src);
    prefix |= static_cast<uint64_t>(digit) << shift;
    need -= static_cast<int>(above);
    fixed = shift;
    const uint32_t at = hist[digit];
    __syncwarp();
    if (at == static_cast<uint32_t>(need)) break;  // every key with this prefix is taken
  }
  // keys whose bits [fixed, 64) are >= the prefix are the selection
  const uint64_t thr = prefix >> fixed;
  int base = 0;
  for (int i0 = 0; i0 < n; i0 += 32) {
    const int i = i0 + lane;
    uint64_t kk = 0;
    bool take = false;
    if (i < n) {
      kk = key(i);
      take = (kk >> fixed) >= thr;
    }
    const uint32_t m = __ballot_sync(0xffffffffu, take);
    const int pos = base + __popc(m & lanemask_lt());
    if (take && pos < want) out[pos] = kk;
    base += __popc(m);
  }
  __syncwarp();
}

// Bitonic sort of s[0..P) (P a power of two) into descending order, one warp.
__device__ void warp_sort_desc(uint64_t* s, int P) {
  const int lane = threadIdx.x & 31;
  for (int size = 2; size <= P; size <<= 1)
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = lane; i < P / 2; i += 32) {
        const int lo = 2 * i - (i & (stride - 1));
        const int hi = lo + stride;
        const bool desc = (lo & size) == 0;
        const uint64_t a = s[lo], b = s[hi];
        if ((a < b) == desc) {
          s[lo] = b;
          s[hi] = a;
        }
      }
      __syncwarp();
    }
}

struct SelPlan {
  int nr_pad, nc_pad, kp, Kp, cand;  // sizes (elements)
  int off_vr, off_vc, off_hr, off_hc, off_sr, off_sc, off_cand, off_out, off_misc;
  int pair_bytes;
};

// bytes per token pair, each array 16-byte aligned
SelPlan make_plan(const Dims& D) {
  SelPlan p{};
  auto al = [](int v) { return (v + 15) & ~15; };
  p.kp = static_cast<int>(next_pow2(D.k));
  p.Kp = static_cast<int>(next_pow2(D.K));
  int cand = 0;
  for (int64_t a = 0; a < D.k; ++a) {
    int64_t nb = D.K / (a + 1);
    if (nb > D.k) nb = D.k;
    if (nb <= 0) break;
    cand += static_cast<int>(nb);
  }
  p.cand = cand;
  int off = 0;
  p.off_vr = off; off = al(off + 4 * static_cast<int>(D.Nr));
  p.off_vc = off; off = al(off + 4 * static_cast<int>(D.Nc));
  p.off_hr = off; off = al(off + 4 * 256);
  p.off_hc = off; off = al(off + 4 * 256);
  p.off_sr = off; off = al(off + 8 * p.kp);
  p.off_sc = off; off = al(off + 8 * p.kp);
  p.off_cand = off; off = al(off + 8 * cand);
  p.off_out = off; off = al(off + 8 * p.Kp);
  p.off_misc = off; off = al(off + 16);
  p.pair_bytes = off;
  return p;
}

__global__ void __launch_bounds__(256) k_select(const float* __restrict__ Z, int64_t L, int Nr,
                                                int Nc, int k, int K,
                                                const float* __restrict__ br,
                                                const float* __restrict__ bc,
                                                int32_t* __restrict__ idx,
                                                float* __restrict__ gate,
                                                float* __restrict__ score, SelPlan P) {
  extern __shared__ __align__(16) uint8_t smem[];
  const int lane = threadIdx.x & 31;
  const int pair = threadIdx.x >> 6;
  const int role = (threadIdx.x >> 5) & 1;  // 0: rows, 1: columns
  const int pairs = blockDim.x >> 6;
  const int64_t t = static_cast<int64_t>(blockIdx.x) * pairs + pair;
  if (t >= L) return;  // both warps of the pair leave together
  uint8_t* base = smem + static_cast<size_t>(pair) * P.pair_bytes;
  float* misc = reinterpret_cast<float*>(base + P.off_misc);

  // ---- per-axis: log-sum-exp and top-k ----
  {
    const int n = role ? Nc : Nr;
    const float* z = Z + t * static_cast<int64_t>(Nr + Nc) + (role ? Nr : 0);
    const float* bias = role ? bc : br;
    float* vals = reinterpret_cast<float*>(base + (role ? P.off_vc : P.off_vr));
    uint32_t* hist = reinterpret_cast<uint32_t*>(base + (role ? P.off_hc : P.off_hr));
    uint64_t* sel = reinterpret_cast<uint64_t*>(base + (role ? P.off_sc : P.off_sr));
    float mx = -INFINITY;
    for (int i = lane; i < n; i += 32) {
      float v = z[i];
      if (bias != nullptr) v += bias[i];
      v = (v == 0.0f) ? 0.0f : v;  // one zero (no -0) so equal logits tie
      vals[i] = v;
      mx = fmaxf(mx, v);
    }
    mx = warp_max(mx);
    float s = 0.0f;
    for (int i = lane; i < n; i += 32) s += expf(vals[i] - mx);
    s = warp_sum(s);
    __syncwarp();
    if (lane == 0) misc[role] = mx + logf(s);
    auto key = [&](int i) { return make_key(vals[i], static_cast<uint32_t>(i)); };
    warp_select_top(key, n, k, sel, hist);
    for (int i = k + lane; i < P.kp; i += 32) sel[i] = 0;
    __syncwarp();
    warp_sort_desc(sel, P.kp);
  }
  asm volatile("bar.sync %0, %1;" ::"r"(1 + pair), "r"(64) : "memory");
  if (role != 0) return;

  // ---- k x k merge over the pairs that can reach the top-K ----
  const uint64_t* sr = reinterpret_cast<const uint64_t*>(base + P.off_sr);
  const uint64_t* sc = reinterpret_cast<const uint64_t*>(base + P.off_sc);
  uint64_t* cand = reinterpret_cast<uint64_t*>(base + P.off_cand);
  uint64_t* out = reinterpret_cast<uint64_t*>(base + P.off_out);
  uint32_t* hist = reinterpret_cast<uint32_t*>(base + P.off_hr);
  int nc = 0;
  for (int a = 0; a < k; ++a) {
    int nb = K / (a + 1);
    if (nb > k) nb = k;
    if (nb <= 0) break;
    const uint64_t ra = sr[a];
    const float za = key_val(ra);
    const uint32_t ia = key_id(ra);
    for (int b = lane; b < nb; b += 32) {
      const uint64_t cb = sc[b];
      const float sv = za + key_val(cb);
      const uint32_t e = ia * static_cast<uint32_t>(Nc) + key_id(cb);
      cand[nc + b] = make_key(sv, e);
    }
    nc += nb;
  }
  __syncwarp();
  auto ckey = [&](int i) { return cand[i]; };
  warp_select_top(ckey, nc, K, out, hist);
  for (int i = K + lane; i < P.Kp; i += 32) out[i] = 0;
  __syncwarp();
  warp_sort_desc(out, P.Kp);

  // ---- gate = softmax of the K selected joint scores ----
  const float s0 = key_val(out[0]);
  float wsum = 0.0f;
  for (int q = lane; q < K; q += 32) wsum += expf(key_val(out[q]) - s0);
  wsum = warp_sum(wsum);
  const float lse = misc[0] + misc[1];
  for (int q = lane; q < K; q += 32) {
    const uint64_t kk = out[q];
    const float v = key_val(kk);
    idx[t * K + q] = static_cast<int32_t>(key_id(kk));
    gate[t * K + q] = expf(v - s0) / wsum;
    if (score != nullptr) score[t * K + q] = v - lse;
  }
}

}  // namespace

cudaError_t launch_select(const Dims& D, const float* Z, const float* br, const float* bc,
                          int32_t* idx, float* gate, float* score, cudaStream_t s) {
  if (D.L == 0) return cudaSuccess;
  SelPlan P = make_plan(D);
  int pairs = 4;
  while (pairs > 1 && pairs * P.pair_bytes > 100 * 1024) pairs >>= 1;
  const size_t smem = static_cast<size_t>(pairs) * P.pair_bytes;
  cudaError_t err =
      cudaFuncSetAttribute(k_select, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem));
  if (err != cudaSuccess) return err;
  const int64_t grid = (D.L + pairs - 1) / pairs;
  k_select<<<static_cast<unsigned>(grid), 64 * pairs, smem, s>>>(
      Z, D.L, static_cast<int>(D.Nr), static_cast<int>(D.Nc), static_cast<int>(D.k),
      static_cast<int>(D.K), br, bc, idx, gate, score, P);
  return cudaGetLastError();
}

}  // namespace omni
