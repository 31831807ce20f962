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
    // histogram of the next digit; lanes holding the same digit add once
    // (one shared-memory atomic per distinct digit and step, not per key)
    for (int i0 = 0; i0 < n; i0 += 32) {
      const int i = i0 + lane;
      bool part = false;
      uint32_t dig = 0;
      if (i < n) {
        const uint64_t kk = key(i);
        part = shift == 56 || (kk >> (shift + 8)) == (prefix >> (shift + 8));
        dig = static_cast<uint32_t>(kk >> shift) & 255u;
      }
      const uint32_t pm = __ballot_sync(0xffffffffu, part);
      if (part) {
        const uint32_t peers = __match_any_sync(pm, dig);
        if ((peers & lanemask_lt()) == 0) atomicAdd(&hist[dig], static_cast<uint32_t>(__popc(peers)));
      }
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

constexpr int kCandMax = 64;  // keys of the threshold bin resolved by sorting

// Top `want` of n keys by (value desc, id asc), one warp, written sorted
// (descending composite key) to out[0..P) (P = next power of two >= want,
// padded with 0).  Value-range binning: with lo/hi the smallest/largest value,
// bin(v) = floor((v - lo) * 256 / (hi - lo)) is monotone in v, so every key in
// a bin above the threshold bin is selected and equal values share a bin; the
// keys of the threshold bin (at most kCandMax) are ordered exactly by their
// 64-bit keys.  Otherwise (threshold bin too full, non-finite scale) the radix
// select decides.  hist: 256 words; cand: kCandMax keys.
template <typename ValFn, typename IdFn>
__device__ void warp_topk_sorted(ValFn val, IdFn id, int n, int want, int P, float lo, float hi,
                                 uint64_t* out, uint32_t* hist, uint64_t* cand) {
  const int lane = threadIdx.x & 31;
  auto key = [&](int i) { return make_key(val(i), id(i)); };
  const float range = hi - lo;
  const float scale = 256.0f / range;
  bool fast = want < n && range > 0.0f && isfinite(scale) && isfinite(range);
  if (fast) {
    for (int b = lane; b < 256; b += 32) hist[b] = 0;
    __syncwarp();
    auto bin = [&](float v) {
      const float f = (v - lo) * scale;
      return f >= 255.0f ? 255u : (f > 0.0f ? static_cast<uint32_t>(f) : 0u);
    };
    for (int i0 = 0; i0 < n; i0 += 32) {
      const int i = i0 + lane;
      const bool part = i < n;
      const uint32_t dig = part ? bin(val(i)) : 0u;
      const uint32_t pm = __ballot_sync(0xffffffffu, part);
      if (part) {
        const uint32_t peers = __match_any_sync(pm, dig);
        if ((peers & lanemask_lt()) == 0) atomicAdd(&hist[dig], static_cast<uint32_t>(__popc(peers)));
      }
    }
    __syncwarp();
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
    int tb = -1;
    uint32_t above = 0;
    if (excl < static_cast<uint32_t>(want) && static_cast<uint32_t>(want) <= incl) {
      uint32_t run = excl;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (tb < 0 && run + c[j] >= static_cast<uint32_t>(want)) {
          tb = 255 - 8 * lane - j;
          above = run;
        }
        run += c[j];
      }
    }
    const uint32_t who = __ballot_sync(0xffffffffu, tb >= 0);
    const int src = __ffs(who) - 1;
    tb = __shfl_sync(0xffffffffu, tb, src);
    above = __shfl_sync(0xffffffffu, above, src);
    const uint32_t at = hist[tb];
    __syncwarp();
    fast = at <= kCandMax;
    if (fast) {
      // keys above the threshold bin -> out[0..above), the threshold bin -> cand
      int nb = 0, nc = 0;
      for (int i0 = 0; i0 < n; i0 += 32) {
        const int i = i0 + lane;
        uint32_t b = 0;
        uint64_t kk = 0;
        if (i < n) {
          const float v = val(i);
          b = bin(v);
          kk = make_key(v, id(i));
        }
        const bool up = i < n && static_cast<int>(b) > tb;
        const bool eq = i < n && static_cast<int>(b) == tb;
        const uint32_t mu = __ballot_sync(0xffffffffu, up);
        const uint32_t me = __ballot_sync(0xffffffffu, eq);
        if (up) out[nb + __popc(mu & lanemask_lt())] = kk;
        if (eq) cand[nc + __popc(me & lanemask_lt())] = kk;
        nb += __popc(mu);
        nc += __popc(me);
      }
      // order the threshold bin and take what is still needed
      int cp = 1;
      while (cp < nc) cp <<= 1;
      for (int i = nc + lane; i < cp; i += 32) cand[i] = 0;
      __syncwarp();
      warp_sort_desc(cand, cp);
      const int need = want - nb;
      for (int i = lane; i < need; i += 32) out[nb + i] = cand[i];
      __syncwarp();
    }
  }
  if (!fast) warp_select_top(key, n, want, out, hist);
  for (int i = want + lane; i < P; i += 32) out[i] = 0;
  __syncwarp();
  warp_sort_desc(out, P);
}

// The same selection as warp_topk_sorted for values held in registers: lane l
// holds values v[j] of indices j*32 + l (indices >= n are absent).  The rare
// fallback copies the values to `spill` (n floats) and runs the radix select.
template <int NPL>
__device__ void warp_topk_regs(const float (&v)[NPL], int n, int want, int P, float lo, float hi,
                               uint64_t* out, uint32_t* hist, uint64_t* cand, float* spill) {
  const int lane = threadIdx.x & 31;
  const float range = hi - lo;
  const float scale = 256.0f / range;
  bool fast = want < n && range > 0.0f && isfinite(scale) && isfinite(range);
  if (fast) {
    for (int b = lane; b < 256; b += 32) hist[b] = 0;
    __syncwarp();
    auto bin = [&](float x) {
      const float f = (x - lo) * scale;
      return f >= 255.0f ? 255u : (f > 0.0f ? static_cast<uint32_t>(f) : 0u);
    };
#pragma unroll
    for (int j = 0; j < NPL; ++j) {
      const bool part = j * 32 + lane < n;
      const uint32_t dig = part ? bin(v[j]) : 0u;
      const uint32_t pm = __ballot_sync(0xffffffffu, part);
      if (part) {
        const uint32_t peers = __match_any_sync(pm, dig);
        if ((peers & lanemask_lt()) == 0) atomicAdd(&hist[dig], static_cast<uint32_t>(__popc(peers)));
      }
    }
    __syncwarp();
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
      const uint32_t t = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += t;
    }
    const uint32_t excl = incl - tot;
    int tb = -1;
    uint32_t above = 0;
    if (excl < static_cast<uint32_t>(want) && static_cast<uint32_t>(want) <= incl) {
      uint32_t run = excl;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (tb < 0 && run + c[j] >= static_cast<uint32_t>(want)) {
          tb = 255 - 8 * lane - j;
          above = run;
        }
        run += c[j];
      }
    }
    const uint32_t who = __ballot_sync(0xffffffffu, tb >= 0);
    const int src = __ffs(who) - 1;
    tb = __shfl_sync(0xffffffffu, tb, src);
    above = __shfl_sync(0xffffffffu, above, src);
    const uint32_t at = hist[tb];
    __syncwarp();
    fast = at <= kCandMax;
    if (fast) {
      int nb = 0, nc = 0;
#pragma unroll
      for (int j = 0; j < NPL; ++j) {
        const int i = j * 32 + lane;
        const bool valid = i < n;
        const uint32_t b = valid ? bin(v[j]) : 0u;
        const bool up = valid && static_cast<int>(b) > tb;
        const bool eq = valid && static_cast<int>(b) == tb;
        const uint64_t kk = make_key(v[j], static_cast<uint32_t>(i));
        const uint32_t mu = __ballot_sync(0xffffffffu, up);
        const uint32_t me = __ballot_sync(0xffffffffu, eq);
        if (up) out[nb + __popc(mu & lanemask_lt())] = kk;
        if (eq) cand[nc + __popc(me & lanemask_lt())] = kk;
        nb += __popc(mu);
        nc += __popc(me);
      }
      int cp = 1;
      while (cp < nc) cp <<= 1;
      for (int i = nc + lane; i < cp; i += 32) cand[i] = 0;
      __syncwarp();
      warp_sort_desc(cand, cp);
      const int need = want - nb;
      for (int i = lane; i < need; i += 32) out[nb + i] = cand[i];
      __syncwarp();
    }
  }
  if (!fast) {
#pragma unroll
    for (int j = 0; j < NPL; ++j)
      if (j * 32 + lane < n) spill[j * 32 + lane] = v[j];
    __syncwarp();
    warp_select_top([&](int i) { return make_key(spill[i], static_cast<uint32_t>(i)); }, n, want,
                    out, hist);
  }
  for (int i = want + lane; i < P; i += 32) out[i] = 0;
  __syncwarp();
  warp_sort_desc(out, P);
}

struct SelPlan {
  int nr_pad, nc_pad, kp, Kp, cand;  // sizes (elements)
  int off_vr, off_vc, off_hr, off_hc, off_sr, off_sc, off_cand, off_out, off_misc, off_tr, off_tc,
      off_roff;
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
  p.off_tr = off; off = al(off + 8 * kCandMax);
  p.off_tc = off; off = al(off + 8 * kCandMax);
  p.off_roff = off; off = al(off + 4 * static_cast<int>(D.k));
  p.pair_bytes = off;
  return p;
}

template <int NPL>
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
    uint64_t* tbin = reinterpret_cast<uint64_t*>(base + (role ? P.off_tc : P.off_tr));
    float v[NPL];
    float mx = -INFINITY, mn = INFINITY;
#pragma unroll
    for (int j = 0; j < NPL; ++j) {
      const int i = j * 32 + lane;
      float x = 0.0f;
      if (i < n) {
        x = z[i];
        if (bias != nullptr) x += bias[i];
        x = (x == 0.0f) ? 0.0f : x;  // one zero (no -0) so equal logits tie
        mx = fmaxf(mx, x);
        mn = fminf(mn, x);
      }
      v[j] = x;
    }
    mx = warp_max(mx);
    mn = -warp_max(-mn);
    float s = 0.0f;
#pragma unroll
    for (int j = 0; j < NPL; ++j)
      if (j * 32 + lane < n) s += expf(v[j] - mx);
    s = warp_sum(s);
    if (lane == 0) misc[role] = mx + logf(s);
    warp_topk_regs<NPL>(v, n, k, P.kp, mn, mx, sel, hist, tbin, vals);
  }
  asm volatile("bar.sync %0, %1;" ::"r"(1 + pair), "r"(64) : "memory");
  if (role != 0) return;

  // ---- k x k merge over the pairs that can reach the top-K ----
  const uint64_t* sr = reinterpret_cast<const uint64_t*>(base + P.off_sr);
  const uint64_t* sc = reinterpret_cast<const uint64_t*>(base + P.off_sc);
  uint64_t* cand = reinterpret_cast<uint64_t*>(base + P.off_cand);
  uint64_t* out = reinterpret_cast<uint64_t*>(base + P.off_out);
  uint32_t* hist = reinterpret_cast<uint32_t*>(base + P.off_hr);
  uint64_t* tbin = reinterpret_cast<uint64_t*>(base + P.off_tr);
  // candidate (a, b) pairs with (a+1)(b+1) <= K, one per lane: row a's pairs
  // start at roff[a] (prefix of min(k, K/(a+1)) over the rows)
  int32_t* roff = reinterpret_cast<int32_t*>(base + P.off_roff);
  int na = 0;
  for (int a0 = 0; a0 < k; a0 += 32) {
    const int a = a0 + lane;
    int nb = 0;
    if (a < k) {
      nb = K / (a + 1);
      if (nb > k) nb = k;
    }
    int incl = nb;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t2 = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += t2;
    }
    if (a < k) roff[a] = na + incl - nb;
    na += __shfl_sync(0xffffffffu, incl, 31);
  }
  __syncwarp();
  const int nc = na;
  float cmx = -INFINITY, cmn = INFINITY;
  for (int c = lane; c < nc; c += 32) {
    int lo = 0, hi = k - 1;  // last row a with roff[a] <= c
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (roff[mid] <= c) lo = mid; else hi = mid - 1;
    }
    const int a = lo, b = c - roff[a];
    const uint64_t ra = sr[a], cb = sc[b];
    const float sv = key_val(ra) + key_val(cb);
    const uint32_t e = key_id(ra) * static_cast<uint32_t>(Nc) + key_id(cb);
    cand[c] = make_key(sv, e);
    cmx = fmaxf(cmx, sv);
    cmn = fminf(cmn, sv);
  }
  cmx = warp_max(cmx);
  cmn = -warp_max(-cmn);
  __syncwarp();
  warp_topk_sorted([&](int i) { return key_val(cand[i]); }, [&](int i) { return key_id(cand[i]); },
                   nc, K, P.Kp, cmn, cmx, out, hist, tbin);

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

template <int NPL>
cudaError_t launch_select_npl(const Dims& D, const float* Z, const float* br, const float* bc,
                              int32_t* idx, float* gate, float* score, cudaStream_t s) {
  SelPlan P = make_plan(D);
  int pairs = 4;
  while (pairs > 1 && pairs * P.pair_bytes > 100 * 1024) pairs >>= 1;
  const size_t smem = static_cast<size_t>(pairs) * P.pair_bytes;
  cudaError_t err =
      cudaFuncSetAttribute(k_select<NPL>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem));
  if (err != cudaSuccess) return err;
  const int64_t grid = (D.L + pairs - 1) / pairs;
  k_select<NPL><<<static_cast<unsigned>(grid), 64 * pairs, smem, s>>>(
      Z, D.L, static_cast<int>(D.Nr), static_cast<int>(D.Nc), static_cast<int>(D.k),
      static_cast<int>(D.K), br, bc, idx, gate, score, P);
  return cudaGetLastError();
}

cudaError_t launch_select(const Dims& D, const float* Z, int parts, const float* br,
                          const float* bc, int32_t* idx, float* gate, float* score,
                          cudaStream_t s) {
  if (D.L == 0) return cudaSuccess;
  if (parts > 1) {  // split-K partial logits: sum them first, in a fixed order
    cudaError_t e = launch_sum_partials(const_cast<float*>(Z), parts, D.L * (D.Nr + D.Nc), s);
    if (e != cudaSuccess) return e;
  }
  const int64_t n = D.Nr > D.Nc ? D.Nr : D.Nc;
  if (n <= 256) return launch_select_npl<8>(D, Z, br, bc, idx, gate, score, s);
  if (n <= 1024) return launch_select_npl<32>(D, Z, br, bc, idx, gate, score, s);
  if (n <= 2048) return launch_select_npl<64>(D, Z, br, bc, idx, gate, score, s);
  return launch_select_npl<128>(D, Z, br, bc, idx, gate, score, s);
}

}  // namespace omni
