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
// top-k entries over 64-bit keys (order-preserving bits of the logit << 32 |
// ~index, so ties fall to the smaller index): a 256-bin histogram over the
// value range finds the bin that holds the k-th key, the keys above it are
// compacted, the bin itself is sorted for the rest, and the k keys are sorted
// by a register bitonic network.  Warp 0 then forms the joint scores of the
// k x k candidate pairs that can reach the top-K -- pair (a, b) of the sorted
// axis lists has (a+1)(b+1) - 1 pairs that score at least as high, so only
// pairs with (a+1)(b+1) <= K are needed -- and selects the K best by
// (S desc, e asc) the same way.  The gate is the softmax of the K selected
// joint scores.  A radix select over the keys takes over when the value
// range is degenerate or the threshold bin holds too many keys.
//
// Ordering uses the raw fp32 logit sums z_r[i] + z_c[j] (the per-token
// log-sum-exp terms are constants and only enter the reported score), so no
// rounding of a log-sum-exp subtraction can tie two distinct logits.
#include "common.cuh"
#include "internal.h"
#include "warpsort.cuh"

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

constexpr int kCandMax = 64;  // keys of the threshold bin resolved by sorting

// out[0 .. 32*W) := the first `m` keys of out sorted descending, then zeros.
template <int W>
__device__ __forceinline__ void sort_out(uint64_t* out, int m) {
  const int lane = threadIdx.x & 31;
  uint64_t key[W];
#pragma unroll
  for (int w = 0; w < W; ++w) key[w] = w * 32 + lane < m ? out[w * 32 + lane] : 0ull;
  __syncwarp();
  reg_sort_desc<W>(key);
#pragma unroll
  for (int w = 0; w < W; ++w) out[w * 32 + lane] = key[w];
  __syncwarp();
}

template <int NW>
__device__ __forceinline__ void group_sync(int bar_id) {
  if (NW == 1) {
    __syncwarp();
  } else {
    asm volatile("bar.sync %0, %1;" ::"r"(bar_id), "r"(NW * 32) : "memory");
  }
}

// Top `want` (<= 32*W) of the n keys make_key(value, id) held by a group of
// NW warps (gw: this warp's index in the group, bar_id: the group's named
// barrier), by (value desc, id asc), written sorted to out[0 .. 32*W)
// (padded with 0); out is complete for every warp of the group on return.
//
// for_each(f) calls f(value, id) for every element of the calling thread (in
// any order; elements are split over the group's threads), key_at(i) gives
// the key of element i < n (used only by the fallback, after every thread
// has called prepare()).  Value-range binning with lo/hi the smallest/largest
// value: bin(v) = floor((v - lo) * 256 / (hi - lo)) is monotone in v, so
// every key in a bin above the threshold bin is selected and equal values
// share a bin.  A 256-bin histogram (shared-memory atomics) finds the
// threshold bin; the histogram, scanned from the top bin down, gives every
// bin at or above it its first output position, and each of those keys
// (about want of n, the threshold bin at most kCandMax) is placed at its
// bin's position plus the number of larger keys of its bin: the output is
// sorted without a sorting network.  A threshold bin that is too full, or a
// non-finite range, falls back to the radix select.  hist: 256 words; tbk:
// kCandMax keys.
template <int W, int NW, typename ForEach, typename Prepare, typename KeyAt>
__device__ void group_topk(int gw, int bar_id, ForEach for_each, Prepare prepare, KeyAt key_at,
                           int n, int want, float lo, float hi, uint64_t* out, uint32_t* hist,
                           uint64_t* tbk) {
  const int lane = threadIdx.x & 31;
  const int gt = gw * 32 + lane;
  const float range = hi - lo;
  const float scale = 256.0f / range;
  bool fast = want < n && range > 0.0f && isfinite(scale) && isfinite(range);
  if (fast) {
    const float off = -lo * scale;
    auto bin = [&](float v) -> int {  // monotone in v: one fma, clamped to [0, 255]
      return __float2int_rz(fminf(fmaxf(fmaf(v, scale, off), 0.0f), 255.0f));
    };
    for (int b = gt; b < 256; b += NW * 32) hist[b] = 0u;
    group_sync<NW>(bar_id);
    for_each([&](float v, uint32_t) { atomicAdd(&hist[bin(v)], 1u); });
    group_sync<NW>(bar_id);
    // every warp scans the bins in descending order: lane l owns bins
    // 255-8l ... 248-8l
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
    uint32_t above = 0, at = 0;
    if (excl < static_cast<uint32_t>(want) && static_cast<uint32_t>(want) <= incl) {
      uint32_t run = excl;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (tb < 0 && run + c[j] >= static_cast<uint32_t>(want)) {
          tb = 255 - 8 * lane - j;
          above = run;
          at = c[j];
        }
        run += c[j];
      }
    }
    const uint32_t who = __ballot_sync(0xffffffffu, tb >= 0);
    const int src = __ffs(who) - 1;
    tb = __shfl_sync(0xffffffffu, tb, src);
    above = __shfl_sync(0xffffffffu, above, src);
    at = __shfl_sync(0xffffffffu, at, src);
    fast = at <= static_cast<uint32_t>(kCandMax);
    if (fast) {
      // the keys of bins >= tb in bin order: bin b starts after the keys of
      // the bins above it (warp 0 turns the histogram into those offsets)
      group_sync<NW>(bar_id);  // every warp has read the histogram
      if (gw == 0) {
        uint32_t run = excl;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int b = 255 - 8 * lane - j;
          if (b >= tb) hist[b] = run;
          run += c[j];
        }
      }
      group_sync<NW>(bar_id);
      // slots [0, above) live in out, [above, above + at) in tbk
      auto slot = [&](uint32_t q) -> uint64_t& { return q < above ? out[q] : tbk[q - above]; };
      for_each([&](float v, uint32_t id) {
        const int b = bin(v);
        if (b >= tb) slot(atomicAdd(&hist[b], 1u)) = make_key(v, id);
      });
      group_sync<NW>(bar_id);
      // hist[b] now ends bin b, so bin b spans [hist[b + 1], hist[b]) (255: from 0);
      // a key's rank is its bin's start plus the larger keys of its bin
      constexpr int PER = (32 * W + kCandMax + NW * 32 - 1) / (NW * 32);
      const uint32_t staged = above + at;
      uint64_t kk[PER];
      int rk[PER];
#pragma unroll
      for (int q = 0; q < PER; ++q) {
        const uint32_t s0 = static_cast<uint32_t>(gt + q * NW * 32);
        rk[q] = -1;
        kk[q] = 0ull;
        if (s0 < staged) {
          kk[q] = slot(s0);
          const int b = bin(key_val(kk[q]));
          const uint32_t lo_s = b == 255 ? 0u : hist[b + 1], hi_s = hist[b];
          uint32_t r = lo_s;
          for (uint32_t s1 = lo_s; s1 < hi_s; ++s1) r += slot(s1) > kk[q] ? 1u : 0u;
          rk[q] = static_cast<int>(r);
        }
      }
      group_sync<NW>(bar_id);  // every staged key is read before out is rewritten
#pragma unroll
      for (int q = 0; q < PER; ++q)
        if (rk[q] >= 0 && rk[q] < want) out[rk[q]] = kk[q];
      for (int p = want + gt; p < 32 * W; p += NW * 32) out[p] = 0ull;
    }
  }
  if (!fast) {
    prepare();
    group_sync<NW>(bar_id);
    if (gw == 0) {
      warp_select_top(key_at, n, want, out, hist);
      sort_out<W>(out, want < n ? want : n);
    }
  }
  group_sync<NW>(bar_id);  // out is complete for every warp of the group
}

struct SelPlan {
  int cand;                           // (a, b) candidate pairs of the k x k merge
  int off_vr, off_vc, off_hr, off_hc, off_sr, off_sc, off_cand, off_out, off_misc, off_tr, off_tc;
  int pair_bytes;
  int table_bytes;                    // per CTA: the (a, b) pair table
  int bias_bytes;                     // per CTA: cached row/column biases (0 without bias)
};

int merge_candidates(const Dims& D) {
  int cand = 0;
  for (int64_t a = 0; a < D.k; ++a) {
    int64_t nb = D.K / (a + 1);
    if (nb > D.k) nb = D.k;
    if (nb <= 0) break;
    cand += static_cast<int>(nb);
  }
  return cand;
}

// bytes per token pair, each array 16-byte aligned
SelPlan make_plan(const Dims& D, int W, int WK) {
  SelPlan p{};
  auto al = [](int v) { return (v + 15) & ~15; };
  p.cand = merge_candidates(D);
  int off = 0;
  p.off_vr = off; off = al(off + 4 * static_cast<int>(D.Nr));
  p.off_vc = off; off = al(off + 4 * static_cast<int>(D.Nc));
  p.off_hr = off; off = al(off + 4 * 256);
  p.off_hc = off; off = al(off + 4 * 256);
  p.off_sr = off; off = al(off + 8 * 32 * W);
  p.off_sc = off; off = al(off + 8 * 32 * W);
  p.off_cand = off; off = al(off + 8 * p.cand);
  p.off_out = off; off = al(off + 8 * 32 * WK);
  p.off_misc = off; off = al(off + 32);
  p.off_tr = off; off = al(off + 8 * kCandMax);
  p.off_tc = off; off = al(off + 8 * kCandMax);
  p.pair_bytes = off;
  p.table_bytes = al(4 * p.cand);
  p.bias_bytes = 0;
  return p;
}

__device__ __forceinline__ void cp_async4(float* dst, const float* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(
                   static_cast<uint32_t>(__cvta_generic_to_shared(dst))),
               "l"(src)
               : "memory");
}

// NPL: logits per lane and axis (n <= 32*NPL); W, WK: sorted lengths 32*W >=
// k and 32*WK >= K.  Persistent: pair p of CTA b takes tokens b*pairs + p,
// + gridDim.x*pairs, ...; while it merges one token, each warp's logits of
// its next token land in shared memory (cp.async, each lane its own
// elements), and the biases sit in shared memory for the whole CTA.
template <int NPL, int W, int WK>
__global__ void __launch_bounds__(256, 3) k_select(const float* __restrict__ Z, int64_t L, int Nr,
                                                int Nc, int k, int K,
                                                const float* __restrict__ br,
                                                const float* __restrict__ bc,
                                                int32_t* __restrict__ idx,
                                                float* __restrict__ gate,
                                                float* __restrict__ score, SelPlan P) {
  pdl_wait();
  extern __shared__ __align__(16) uint8_t smem[];
  const int lane = threadIdx.x & 31;
  const int pair = threadIdx.x >> 6;
  const int role = (threadIdx.x >> 5) & 1;  // 0: rows, 1: columns
  const int pairs = blockDim.x >> 6;

  // (a, b) pairs with (a+1)(b+1) <= K, row by row: pair c of row a sits at
  // roff(a) + b, roff the prefix sum of min(k, K/(a+1)); built once per CTA
  uint32_t* cab = reinterpret_cast<uint32_t*>(smem);
  float* bias_s = reinterpret_cast<float*>(smem + P.table_bytes);  // [Nr + Nc] when biased
  if (threadIdx.x < 32) {
    int base = 0;
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
      const int off = base + incl - nb;
      for (int b = 0; b < nb; ++b) cab[off + b] = (static_cast<uint32_t>(a) << 16) | b;
      base += __shfl_sync(0xffffffffu, incl, 31);
    }
  }
  if (P.bias_bytes > 0) {
    for (int i = threadIdx.x; i < Nr + Nc; i += blockDim.x)
      bias_s[i] = i < Nr ? (br != nullptr ? br[i] : 0.0f) : (bc != nullptr ? bc[i - Nr] : 0.0f);
  }
  __syncthreads();

  const int64_t stride = static_cast<int64_t>(gridDim.x) * pairs;
  int64_t t = static_cast<int64_t>(blockIdx.x) * pairs + pair;
  if (t >= L) return;  // both warps of the pair leave together
  uint8_t* base = smem + P.table_bytes + P.bias_bytes + static_cast<size_t>(pair) * P.pair_bytes;
  float* misc = reinterpret_cast<float*>(base + P.off_misc);
  const int n = role ? Nc : Nr;
  const int zoff = role ? Nr : 0;
  // this warp's logits of one token (raw, before bias); the radix fallback
  // also reads values from here
  float* vals = reinterpret_cast<float*>(base + (role ? P.off_vc : P.off_vr));
  auto prefetch = [&](int64_t tt) {
    const float* z = Z + tt * static_cast<int64_t>(Nr + Nc) + zoff;
#pragma unroll
    for (int j = 0; j < NPL; ++j) {
      const int i = j * 32 + lane;
      if (i < n) cp_async4(vals + i, z + i);
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };
  prefetch(t);

  for (; t < L; t += stride) {
  // ---- per-axis: log-sum-exp and top-k ----
  {
    uint32_t* hist = reinterpret_cast<uint32_t*>(base + (role ? P.off_hc : P.off_hr));
    uint64_t* sel = reinterpret_cast<uint64_t*>(base + (role ? P.off_sc : P.off_sr));
    uint64_t* tbin = reinterpret_cast<uint64_t*>(base + (role ? P.off_tc : P.off_tr));
    const float* bias = P.bias_bytes > 0 ? bias_s + zoff : nullptr;
    asm volatile("cp.async.wait_all;" ::: "memory");  // this lane's copies of token t
    float v[NPL];
    float mx = -INFINITY, mn = INFINITY;
#pragma unroll
    for (int j = 0; j < NPL; ++j) {
      const int i = j * 32 + lane;
      float x = 0.0f;
      if (i < n) {
        x = vals[i];
        if (bias != nullptr) x += bias[i];
        x = (x == 0.0f) ? 0.0f : x;  // one zero (no -0) so equal logits tie
        mx = fmaxf(mx, x);
        mn = fminf(mn, x);
      }
      v[j] = x;
    }
    mx = warp_max(mx);
    mn = -warp_max(-mn);
    if (score != nullptr) {  // the log-sum-exp moves only the scores, not ids or gates
      float s = 0.0f;
#pragma unroll
      for (int j = 0; j < NPL; ++j)
        if (j * 32 + lane < n) s += __expf(v[j] - mx);
      s = warp_sum(s);
      if (lane == 0) misc[role] = mx + logf(s);
    }
    group_topk<W, 1>(
        0, 0,
        [&](auto f) {
#pragma unroll
          for (int j = 0; j < NPL; ++j)
            if (j * 32 + lane < n) f(v[j], static_cast<uint32_t>(j * 32 + lane));
        },
        [&]() {  // the radix fallback reads values by index
#pragma unroll
          for (int j = 0; j < NPL; ++j)
            if (j * 32 + lane < n) vals[j * 32 + lane] = v[j];
        },
        [&](int i) { return make_key(vals[i], static_cast<uint32_t>(i)); }, n, k, mn, mx, sel,
        hist, tbin);
    __syncwarp();
    if (t + stride < L) prefetch(t + stride);  // lands while the pair merges
  }
  asm volatile("bar.sync %0, %1;" ::"r"(1 + pair), "r"(64) : "memory");
  const float lse = misc[0] + misc[1];  // read before the next token rewrites them

  // ---- k x k merge over the pairs that can reach the top-K (both warps) ----
  const uint64_t* sr = reinterpret_cast<const uint64_t*>(base + P.off_sr);
  const uint64_t* sc = reinterpret_cast<const uint64_t*>(base + P.off_sc);
  uint64_t* cand = reinterpret_cast<uint64_t*>(base + P.off_cand);
  uint64_t* out = reinterpret_cast<uint64_t*>(base + P.off_out);
  uint32_t* hist = reinterpret_cast<uint32_t*>(base + P.off_hr);
  uint64_t* tbin = reinterpret_cast<uint64_t*>(base + P.off_tr);
  const int nc = P.cand;
  const int pt = role * 32 + lane;  // thread of the pair
  float cmx = -INFINITY, cmn = INFINITY;
  for (int c = pt; c < nc; c += 64) {
    const uint32_t ab = cab[c];
    const uint64_t ra = sr[ab >> 16], cb = sc[ab & 0xffffu];
    const float sv = key_val(ra) + key_val(cb);
    const uint32_t e = key_id(ra) * static_cast<uint32_t>(Nc) + key_id(cb);
    cand[c] = make_key(sv, e);
    cmx = fmaxf(cmx, sv);
    cmn = fminf(cmn, sv);
  }
  cmx = warp_max(cmx);
  cmn = -warp_max(-cmn);
  if (lane == 0) {
    misc[2 + role] = cmx;
    misc[4 + role] = cmn;
  }
  asm volatile("bar.sync %0, %1;" ::"r"(1 + pair), "r"(64) : "memory");
  cmx = fmaxf(misc[2], misc[3]);
  cmn = fminf(misc[4], misc[5]);
  group_topk<WK, 2>(
      role, 1 + pair,
      [&](auto f) {
        for (int c = pt; c < nc; c += 64) {
          const uint64_t kk = cand[c];
          f(key_val(kk), key_id(kk));
        }
      },
      []() {}, [&](int i) { return cand[i]; }, nc, K, cmn, cmx, out, hist, tbin);
  if (role == 0) {
    // ---- gate = softmax of the K selected joint scores ----
    const float s0 = key_val(out[0]);
    float wsum = 0.0f;
    for (int q = lane; q < K; q += 32) wsum += __expf(key_val(out[q]) - s0);
    wsum = warp_sum(wsum);
    for (int q = lane; q < K; q += 32) {
      const uint64_t kk = out[q];
      const float v = key_val(kk);
      idx[t * K + q] = static_cast<int32_t>(key_id(kk));
      gate[t * K + q] = __expf(v - s0) / wsum;
      if (score != nullptr) score[t * K + q] = v - lse;
    }
  }
  // the next token's merge reuses out/cand/hist: both warps meet first
  asm volatile("bar.sync %0, %1;" ::"r"(1 + pair), "r"(64) : "memory");
  }
  asm volatile("cp.async.wait_all;" ::: "memory");
}

// ---- small batches: one CTA of 8 warps per token ---------------------------
//
// The same selection with more warps per token, for batches too small to
// fill the GPU with two warps per token: warps 0-3 take the row logits and
// warps 4-7 the column logits (each warp NPW values per lane; named barriers
// 1 and 2), and all eight warps form the merge candidates and their
// histogram.  The sorted lists, the threshold bins and the gate are the work
// of one warp, as in k_select.
struct WidePlan {
  int cand;
  int off_vals, off_hist, off_sel, off_tbk, off_red, off_roff, off_cand, off_out, off_misc;
  int bytes;
};

WidePlan make_wide_plan(const Dims& D, int W, int WK) {
  WidePlan p{};
  auto al = [](int v) { return (v + 15) & ~15; };
  p.cand = merge_candidates(D);
  const int nmax = static_cast<int>(D.Nr > D.Nc ? D.Nr : D.Nc);
  int off = 0;
  p.off_vals = off; off = al(off + 2 * 4 * nmax);
  p.off_hist = off; off = al(off + 2 * 4 * 256);
  p.off_sel = off; off = al(off + 2 * 8 * 32 * W);
  p.off_tbk = off; off = al(off + 2 * 8 * kCandMax);
  p.off_red = off; off = al(off + 4 * 3 * 8);
  p.off_roff = off; off = al(off + 4 * static_cast<int>(D.k));
  p.off_cand = off; off = al(off + 8 * p.cand);
  p.off_out = off; off = al(off + 8 * 32 * WK);
  p.off_misc = off; off = al(off + 16);
  p.bytes = off;
  return p;
}

template <int NPW, int W, int WK>
__global__ void __launch_bounds__(256) k_select_wide(const float* __restrict__ Z, int parts,
                                                     int64_t L, int Nr, int Nc, int k, int K,
                                                     const float* __restrict__ br,
                                                     const float* __restrict__ bc,
                                                     int32_t* __restrict__ idx,
                                                     float* __restrict__ gate,
                                                     float* __restrict__ score, WidePlan P,
                                                     float* __restrict__ zero, int64_t zero_words) {
  // The buffer to clear (passed by the fused forward only) is cleared before
  // the wait.  The kernel ahead is that forward's router, which lets this
  // one start only after its own wait, so every earlier user of the buffer
  // has finished.
  if (zero != nullptr) {
    const int64_t i0 = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    if ((reinterpret_cast<uintptr_t>(zero) & 15) == 0) {
      for (int64_t i = i0; i < zero_words / 4; i += stride)
        reinterpret_cast<float4*>(zero)[i] = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int64_t i = (zero_words / 4) * 4 + i0; i < zero_words; i += stride) zero[i] = 0.0f;
    } else {
      for (int64_t i = i0; i < zero_words; i += stride) zero[i] = 0.0f;
    }
  }
  pdl_wait();
  pdl_trigger();
  extern __shared__ __align__(16) uint8_t smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int axis = warp >> 2, gw = warp & 3;
  const int64_t t = blockIdx.x;
  if (t >= L) return;  // the whole CTA leaves
  const int nmax = Nr > Nc ? Nr : Nc;
  float* red = reinterpret_cast<float*>(smem + P.off_red);   // [3][8]: max, min, sum
  float* misc = reinterpret_cast<float*>(smem + P.off_misc);

  // ---- per-axis: log-sum-exp and top-k, four warps per axis ----
  {
    const int n = axis ? Nc : Nr;
    const float* z = Z + t * static_cast<int64_t>(Nr + Nc) + (axis ? Nr : 0);
    const float* bias = axis ? bc : br;
    float* vals = reinterpret_cast<float*>(smem + P.off_vals) + axis * nmax;
    uint32_t* hist = reinterpret_cast<uint32_t*>(smem + P.off_hist) + axis * 256;
    uint64_t* sel = reinterpret_cast<uint64_t*>(smem + P.off_sel) + axis * 32 * W;
    uint64_t* tbk = reinterpret_cast<uint64_t*>(smem + P.off_tbk) + axis * kCandMax;
    const int bar = 1 + axis;
    // split-K partial logits (parts > 1) are summed here, in order
    const int64_t zs = L * static_cast<int64_t>(Nr + Nc);
    float v[NPW];
#pragma unroll
    for (int j = 0; j < NPW; ++j) {
      const int i = (j * 4 + gw) * 32 + lane;
      v[j] = i < n ? z[i] : 0.0f;
    }
#pragma unroll 4
    for (int p = 1; p < parts; ++p) {
#pragma unroll
      for (int j = 0; j < NPW; ++j) {
        const int i = (j * 4 + gw) * 32 + lane;
        if (i < n) v[j] += z[p * zs + i];
      }
    }
    float mx = -INFINITY, mn = INFINITY;
#pragma unroll
    for (int j = 0; j < NPW; ++j) {
      const int i = (j * 4 + gw) * 32 + lane;
      float x = 0.0f;
      if (i < n) {
        x = v[j];
        if (bias != nullptr) x += bias[i];
        x = (x == 0.0f) ? 0.0f : x;  // one zero (no -0) so equal logits tie
        mx = fmaxf(mx, x);
        mn = fminf(mn, x);
      }
      v[j] = x;
    }
    mx = warp_max(mx);
    mn = -warp_max(-mn);
    if (lane == 0) {
      red[warp] = mx;
      red[8 + warp] = mn;
    }
    group_sync<4>(bar);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      mx = fmaxf(mx, red[axis * 4 + q]);
      mn = fminf(mn, red[8 + axis * 4 + q]);
    }
    if (score != nullptr) {  // the log-sum-exp moves only the scores, not ids or gates
      float s = 0.0f;
#pragma unroll
      for (int j = 0; j < NPW; ++j)
        if ((j * 4 + gw) * 32 + lane < n) s += __expf(v[j] - mx);
      s = warp_sum(s);
      if (lane == 0) red[16 + warp] = s;
      group_sync<4>(bar);
      if (gw == 0 && lane == 0) {
        float tot = 0.0f;
#pragma unroll
        for (int q = 0; q < 4; ++q) tot += red[16 + axis * 4 + q];
        misc[axis] = mx + logf(tot);
      }
    }
    group_topk<W, 4>(
        gw, bar,
        [&](auto f) {
#pragma unroll
          for (int j = 0; j < NPW; ++j) {
            const int i = (j * 4 + gw) * 32 + lane;
            if (i < n) f(v[j], static_cast<uint32_t>(i));
          }
        },
        [&]() {  // the radix fallback reads values by index
#pragma unroll
          for (int j = 0; j < NPW; ++j) {
            const int i = (j * 4 + gw) * 32 + lane;
            if (i < n) vals[i] = v[j];
          }
        },
        [&](int i) { return make_key(vals[i], static_cast<uint32_t>(i)); }, n, k, mn, mx, sel,
        hist, tbk);
  }
  __syncthreads();

  // ---- k x k merge, all eight warps ----
  const uint64_t* sr = reinterpret_cast<const uint64_t*>(smem + P.off_sel);
  const uint64_t* sc = sr + 32 * W;
  int32_t* roff = reinterpret_cast<int32_t*>(smem + P.off_roff);
  uint64_t* cand = reinterpret_cast<uint64_t*>(smem + P.off_cand);
  uint64_t* out = reinterpret_cast<uint64_t*>(smem + P.off_out);
  uint32_t* hist = reinterpret_cast<uint32_t*>(smem + P.off_hist);
  uint64_t* tbk = reinterpret_cast<uint64_t*>(smem + P.off_tbk);
  if (warp == 0) {
    // pairs of row a start at roff[a] (prefix of min(k, K/(a+1)))
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
  }
  __syncthreads();
  const int nc = P.cand;
  float cmx = -INFINITY, cmn = INFINITY;
  for (int c = threadIdx.x; c < nc; c += 256) {
    int lo = 0, hi = k - 1;  // last row a with roff[a] <= c
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (roff[mid] <= c) lo = mid; else hi = mid - 1;
    }
    const uint64_t ra = sr[lo], cb = sc[c - roff[lo]];
    const float sv = key_val(ra) + key_val(cb);
    cand[c] = make_key(sv, key_id(ra) * static_cast<uint32_t>(Nc) + key_id(cb));
    cmx = fmaxf(cmx, sv);
    cmn = fminf(cmn, sv);
  }
  cmx = warp_max(cmx);
  cmn = -warp_max(-cmn);
  if (lane == 0) {
    red[warp] = cmx;
    red[8 + warp] = cmn;
  }
  __syncthreads();
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    cmx = fmaxf(cmx, red[q]);
    cmn = fminf(cmn, red[8 + q]);
  }
  group_topk<WK, 8>(
      warp, 0,
      [&](auto f) {
        for (int c = threadIdx.x; c < nc; c += 256) {
          const uint64_t kk = cand[c];
          f(key_val(kk), key_id(kk));
        }
      },
      []() {}, [&](int i) { return cand[i]; }, nc, K, cmn, cmx, out, hist, tbk);
  if (warp != 0) return;

  // ---- gate = softmax of the K selected joint scores ----
  const float s0 = key_val(out[0]);
  float wsum = 0.0f;
  for (int q = lane; q < K; q += 32) wsum += __expf(key_val(out[q]) - s0);
  wsum = warp_sum(wsum);
  const float lse = misc[0] + misc[1];
  for (int q = lane; q < K; q += 32) {
    const uint64_t kk = out[q];
    const float v = key_val(kk);
    idx[t * K + q] = static_cast<int32_t>(key_id(kk));
    gate[t * K + q] = __expf(v - s0) / wsum;
    if (score != nullptr) score[t * K + q] = v - lse;
  }
}

template <int NPW, int W, int WK>
cudaError_t launch_wide_t(const Dims& D, const float* Z, int parts, const float* br,
                          const float* bc, int32_t* idx, float* gate, float* score,
                          float* zero, int64_t zero_words, cudaStream_t s) {
  const WidePlan P = make_wide_plan(D, W, WK);
  cudaError_t err = cudaFuncSetAttribute(k_select_wide<NPW, W, WK>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, P.bytes);
  if (err != cudaSuccess) return err;
  OMNI_TRY(launch_k(k_select_wide<NPW, W, WK>, static_cast<unsigned>(D.L), 256, P.bytes, s, Z,
      parts, D.L, static_cast<int>(D.Nr), static_cast<int>(D.Nc), static_cast<int>(D.k),
      static_cast<int>(D.K), br, bc, idx, gate, score, P, zero, zero_words));
  return cudaGetLastError();
}

template <int NPW>
cudaError_t launch_wide(const Dims& D, const float* Z, int parts, const float* br,
                        const float* bc, int32_t* idx, float* gate, float* score, cudaStream_t s);

int sort_width(int64_t m) {
  int w = 1;
  while (32 * w < m) w <<= 1;
  return w;
}

template <int NPL, int W, int WK>
cudaError_t launch_select_t(const Dims& D, const float* Z, const float* br, const float* bc,
                            int32_t* idx, float* gate, float* score, cudaStream_t s) {
  SelPlan P = make_plan(D, W, WK);
  if (br != nullptr || bc != nullptr) P.bias_bytes = static_cast<int>((4 * (D.Nr + D.Nc) + 15) & ~15);
  // up to four tokens per CTA, fewer when that leaves SMs idle (small batches)
  int sms = 148, dev = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  int pairs = 4;
  while (pairs > 1 && (D.L + pairs - 1) / pairs < sms) pairs >>= 1;
  while (pairs > 1 && P.table_bytes + P.bias_bytes + pairs * P.pair_bytes > 100 * 1024) pairs >>= 1;
  const size_t smem = static_cast<size_t>(P.table_bytes) + P.bias_bytes +
                      static_cast<size_t>(pairs) * P.pair_bytes;
  cudaError_t err =
      cudaFuncSetAttribute(k_select<NPL, W, WK>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem));
  if (err != cudaSuccess) return err;
  int per_sm = 1;
  err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_select<NPL, W, WK>, 64 * pairs,
                                                      smem);
  if (err != cudaSuccess) return err;
  if (per_sm < 1) per_sm = 1;
  int64_t grid = (D.L + pairs - 1) / pairs;
  if (grid > static_cast<int64_t>(sms) * per_sm) grid = static_cast<int64_t>(sms) * per_sm;
  OMNI_TRY(launch_k(k_select<NPL, W, WK>, static_cast<unsigned>(grid), 64 * pairs, smem, s, Z, D.L,
      static_cast<int>(D.Nr), static_cast<int>(D.Nc), static_cast<int>(D.k), static_cast<int>(D.K),
      br, bc, idx, gate, score, P));
  return cudaGetLastError();
}

template <int NPL>
cudaError_t launch_select_npl(const Dims& D, const float* Z, const float* br, const float* bc,
                              int32_t* idx, float* gate, float* score, cudaStream_t s) {
  // one sort width for both lists (32*W >= max(k, K))
  switch (sort_width(D.k > D.K ? D.k : D.K)) {
    case 1: return launch_select_t<NPL, 1, 1>(D, Z, br, bc, idx, gate, score, s);
    case 2: return launch_select_t<NPL, 2, 2>(D, Z, br, bc, idx, gate, score, s);
    case 4: return launch_select_t<NPL, 4, 4>(D, Z, br, bc, idx, gate, score, s);
    default: return launch_select_t<NPL, 8, 8>(D, Z, br, bc, idx, gate, score, s);
  }
}

template <int NPW>
cudaError_t launch_wide(const Dims& D, const float* Z, int parts, const float* br,
                        const float* bc, int32_t* idx, float* gate, float* score, float* zero,
                        int64_t zero_words, cudaStream_t s) {
  switch (sort_width(D.k > D.K ? D.k : D.K)) {
    case 1: return launch_wide_t<NPW, 1, 1>(D, Z, parts, br, bc, idx, gate, score, zero, zero_words, s);
    case 2: return launch_wide_t<NPW, 2, 2>(D, Z, parts, br, bc, idx, gate, score, zero, zero_words, s);
    case 4: return launch_wide_t<NPW, 4, 4>(D, Z, parts, br, bc, idx, gate, score, zero, zero_words, s);
    default: return launch_wide_t<NPW, 8, 8>(D, Z, parts, br, bc, idx, gate, score, zero, zero_words, s);
  }
}

}  // namespace

cudaError_t launch_select(const Dims& D, const float* Z, int parts, const float* br,
                          const float* bc, int32_t* idx, float* gate, float* score,
                          cudaStream_t s, float* zero, int64_t zero_words, bool* zeroed) {
  if (zeroed != nullptr) *zeroed = false;
  if (D.L == 0) return cudaSuccess;
  const int64_t n = D.Nr > D.Nc ? D.Nr : D.Nc;
  int sms = 148, dev = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (D.L <= sms) {  // too few tokens for two warps each to fill the GPU
    if (zeroed != nullptr) *zeroed = zero != nullptr;
    if (n <= 256) return launch_wide<2>(D, Z, parts, br, bc, idx, gate, score, zero, zero_words, s);
    if (n <= 1024) return launch_wide<8>(D, Z, parts, br, bc, idx, gate, score, zero, zero_words, s);
    return launch_wide<32>(D, Z, parts, br, bc, idx, gate, score, zero, zero_words, s);
  }
  if (parts > 1) {  // split-K partial logits: sum them first, in a fixed order
    cudaError_t e = launch_sum_partials(const_cast<float*>(Z), parts, D.L * (D.Nr + D.Nc), s);
    if (e != cudaSuccess) return e;
  }
  if (n <= 256) return launch_select_npl<8>(D, Z, br, bc, idx, gate, score, s);
  if (n <= 1024) return launch_select_npl<32>(D, Z, br, bc, idx, gate, score, s);
  if (n <= 2048) return launch_select_npl<64>(D, Z, br, bc, idx, gate, score, s);
  return launch_select_npl<128>(D, Z, br, bc, idx, gate, score, s);
}

}  // namespace omni
