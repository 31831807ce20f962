// Expert-Centric Scheduling on the device.
//
// "OmniMoE: An Efficient MoE by Orchestrating Atomic Experts at Scale"
// (gist.science), Technisch Overzicht section 2.2 (task collection; grouping
// and sorting; grouped execution) and the OmniMoE explainer (manus.space),
// Expert-Centric Scheduling steps: flatten the L*K (token, expert, weight)
// triples into tasks; collect the unique active experts, sort them by id and
// cut every B into a group; sort tasks by group id, then token id.
//
// Steps (all on `stream`, data-dependent counts stay on the device):
//  1. prep    one warp per token sorts its K (expert, gate) pairs by expert
//             id, so the task list is in (token, expert) order, and counts
//             the tasks of every expert in an N-long array;
//  2. scan    one exclusive prefix sum over the ids of (active, tasks) gives
//             each active expert its rank in U (sorted unique ids), U itself,
//             |U|, the group count ceil(|U| / B) and every group's first task;
//  3. sort    stable LSD radix sort of the tasks by group = rank / B with
//             8-bit digits (as many passes as the group-count bound needs),
//             one kernel per pass (decoupled look-back over tiles) after one
//             histogram kernel for all passes; stability keeps (token,
//             expert) order inside each group;
//  4. emit    gather the sorted tasks.
// The fused forward of a large batch replaces 3-4 by the window order its
// expert stage consumes (launch_schedule_windows, at the end of this file).
#include <cooperative_groups.h>

#include "blocksort.cuh"
#include "common.cuh"
#include "internal.h"
#include "warpsort.cuh"

namespace cg = cooperative_groups;

namespace omni {
namespace {

constexpr int kPrepWarps = 8;
constexpr int kScanThreads = 1024;
constexpr int kScanItems = 4;
constexpr int kScanTile = kScanThreads * kScanItems;
constexpr int kRsThreads = 256;
constexpr int kRsWarps = kRsThreads / 32;
constexpr int kRsPerWarp = 512;  // consecutive tasks per warp in a tile
constexpr int kRsTile = kRsWarps * kRsPerWarp;

// ---- 1. per-token sort by expert id + task counts ------------------------
// One warp per token: its K (expert, slot) keys sorted ascending in registers
// (32*W >= K; a descending network over complemented keys); mult[e] counts
// the tasks of expert e (active: mult > 0).
template <int W>
__global__ void __launch_bounds__(kPrepWarps * 32)
    k_prep(const int32_t* __restrict__ idx, const float* __restrict__ gate, int64_t L, int K,
           int64_t N, int32_t* __restrict__ mult, int32_t* __restrict__ tmp_e,
           float* __restrict__ tmp_g, int32_t* status) {
  pdl_wait();
  pdl_trigger();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t t = static_cast<int64_t>(blockIdx.x) * kPrepWarps + warp;
  if (t >= L) return;  // warp-uniform
  uint64_t key[W];
#pragma unroll
  for (int w = 0; w < W; ++w) {
    const int q = w * 32 + lane;
    key[w] = 0ull;  // complement of the largest key: sorts last
    if (q < K) {
      int64_t e = idx[t * K + q];
      if (e < 0 || e >= N) {
        raise_status(status, OMNI_DEV_BAD_INDEX);
        e = 0;
      }
      atomicAdd(&mult[e], 1);
      key[w] = ~((static_cast<uint64_t>(e) << 32) | static_cast<uint32_t>(q));
    }
  }
  reg_sort_desc<W>(key);
#pragma unroll
  for (int w = 0; w < W; ++w) {
    const int j = w * 32 + lane;
    if (j < K) {
      const uint64_t k = ~key[w];
      tmp_e[t * K + j] = static_cast<int32_t>(k >> 32);
      tmp_g[t * K + j] = gate[t * K + static_cast<uint32_t>(k)];
    }
  }
}

// ---- 2. scan of the (active, task count) pairs over the ids ----------------
// A 64-bit item packs (active ids) << 32 | (tasks): both sums stay below 2^31,
// so one 64-bit scan carries both.  The rank of an id is the active ids
// before it; the first task of group g is the task count before the id of
// rank g * B.
__device__ __forceinline__ uint64_t mult_item(int32_t m) {
  return m > 0 ? ((uint64_t(1) << 32) | static_cast<uint32_t>(m)) : 0ull;
}

__global__ void __launch_bounds__(kScanThreads)
    k_scan_reduce(const int32_t* __restrict__ mult, int64_t N, uint64_t* __restrict__ tile_sum) {
  pdl_wait();
  pdl_trigger();
  __shared__ uint64_t warp_tot[32];
  __shared__ uint64_t total;
  const int64_t base = static_cast<int64_t>(blockIdx.x) * kScanTile + threadIdx.x * kScanItems;
  uint64_t v = 0;
#pragma unroll
  for (int j = 0; j < kScanItems; ++j)
    if (base + j < N) v += mult_item(mult[base + j]);
  block_exclusive_scan(v, warp_tot, &total);
  if (threadIdx.x == 0) tile_sum[blockIdx.x] = total;
}

// single block: exclusive scan of the tile sums; counts[0] = |U|, counts[1] = groups
__global__ void __launch_bounds__(kScanThreads)
    k_scan_tiles(uint64_t* __restrict__ tile_sum, int ntiles, int64_t B, int32_t* counts) {
  pdl_wait();
  pdl_trigger();
  __shared__ uint64_t warp_tot[32];
  __shared__ uint64_t total;
  __shared__ uint64_t carry;
  if (threadIdx.x == 0) carry = 0;
  __syncthreads();
  for (int c0 = 0; c0 < ntiles; c0 += kScanThreads) {
    const int i = c0 + threadIdx.x;
    const uint64_t v = i < ntiles ? tile_sum[i] : 0ull;
    const uint64_t ex = block_exclusive_scan(v, warp_tot, &total);
    if (i < ntiles) tile_sum[i] = carry + ex;
    __syncthreads();
    if (threadIdx.x == 0) carry += total;
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    const int64_t n_active = static_cast<int64_t>(carry >> 32);
    counts[0] = static_cast<int32_t>(n_active);
    counts[1] = static_cast<int32_t>((n_active + B - 1) / B);
  }
}

// rank[e], U, and group_off (every group start; group_off[G] = M)
__global__ void __launch_bounds__(kScanThreads)
    k_scan_finish(const int32_t* __restrict__ mult, int64_t N,
                  const uint64_t* __restrict__ tile_off, int64_t B, int64_t M,
                  const int32_t* __restrict__ counts, int32_t* __restrict__ rank,
                  int32_t* __restrict__ uniq, int32_t* __restrict__ group_off) {
  pdl_wait();
  pdl_trigger();
  __shared__ uint64_t warp_tot[32];
  __shared__ uint64_t total;
  const int64_t base = static_cast<int64_t>(blockIdx.x) * kScanTile + threadIdx.x * kScanItems;
  uint64_t f[kScanItems];
  uint64_t v = 0;
#pragma unroll
  for (int j = 0; j < kScanItems; ++j) {
    f[j] = (base + j < N) ? mult_item(mult[base + j]) : 0ull;
    v += f[j];
  }
  uint64_t r = block_exclusive_scan(v, warp_tot, &total) + tile_off[blockIdx.x];
#pragma unroll
  for (int j = 0; j < kScanItems; ++j) {
    if (base + j < N) {
      const int64_t rk = static_cast<int64_t>(r >> 32);
      rank[base + j] = static_cast<int32_t>(rk);
      if (f[j] != 0ull) {
        uniq[rk] = static_cast<int32_t>(base + j);
        if (rk % B == 0) group_off[rk / B] = static_cast<int32_t>(r & 0xffffffffull);
      }
    }
    r += f[j];
  }
  if (blockIdx.x == 0 && threadIdx.x == 0) group_off[counts[1]] = static_cast<int32_t>(M);
}

// ---- 3. stable radix sort by group id ---------------------------------------
struct KeySrc {
  const uint32_t* keys;    // previous pass output (nullptr on the first pass)
  const int32_t* tmp_e;    // first pass: key = rank[tmp_e[i]] / B
  const int32_t* rank;
  int64_t B;
  __device__ __forceinline__ uint32_t operator()(int64_t i) const {
    if (keys != nullptr) return keys[i];
    return static_cast<uint32_t>(rank[tmp_e[i]] / B);
  }
};

// One-kernel radix pass (decoupled look-back).  A global histogram of every
// pass's digits is taken once up front; then each pass is one kernel whose
// CTAs take tiles in start order (an atomic tile counter), rank their keys
// stably per warp, publish their per-digit counts, and find the counts of
// all earlier tiles by walking back through the published words: a word
// holds a 2-bit state (0 none, 1 this tile's count, 2 count of all tiles up
// to and including this one) and a 30-bit count.  A tile only waits on tiles
// that started before it; every wait is bounded (OMNI_DEV_TIMEOUT).
constexpr uint32_t kLbAgg = 1u << 30, kLbIncl = 2u << 30, kLbCount = (1u << 30) - 1;

__global__ void __launch_bounds__(kRsThreads)
    k_rs_ghist(KeySrc src, int64_t M, int passes, uint32_t* __restrict__ dgh) {
  pdl_wait();
  pdl_trigger();
  __shared__ uint32_t h[4][256];
  for (int j = threadIdx.x; j < 4 * 256; j += kRsThreads) (&h[0][0])[j] = 0u;
  __syncthreads();
  const int64_t t0 = static_cast<int64_t>(blockIdx.x) * kRsTile;
  for (int j = threadIdx.x; j < kRsTile; j += kRsThreads) {
    const int64_t i = t0 + j;
    if (i < M) {
      const uint32_t key = src(i);
      for (int p = 0; p < passes; ++p) atomicAdd(&h[p][(key >> (8 * p)) & 255u], 1u);
    }
  }
  __syncthreads();
  for (int p = 0; p < passes; ++p) {
    const uint32_t c = h[p][threadIdx.x];
    if (c) atomicAdd(&dgh[p * 256 + threadIdx.x], c);
  }
}

__device__ __forceinline__ uint32_t ld_relaxed(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_relaxed(uint32_t* p, uint32_t v) {
  asm volatile("st.relaxed.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__global__ void __launch_bounds__(kRsThreads)
    k_rs_onesweep(KeySrc src, const uint32_t* __restrict__ vals_in, int64_t M, int shift,
                  const uint32_t* __restrict__ dgh, uint32_t* __restrict__ look,
                  uint32_t* __restrict__ tile_ctr, uint32_t* __restrict__ keys_out,
                  uint32_t* __restrict__ vals_out, int32_t* status) {
  pdl_wait();
  pdl_trigger();
  __shared__ uint32_t wcount[kRsWarps][256];
  __shared__ uint32_t tbase[256];
  __shared__ int warp_tot[32];
  __shared__ int total;
  __shared__ int64_t tile_s;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int j = threadIdx.x; j < kRsWarps * 256; j += kRsThreads) (&wcount[0][0])[j] = 0;
  if (threadIdx.x == 0) tile_s = atomicAdd(tile_ctr, 1u);
  __syncthreads();
  const int64_t tile = tile_s;
  const int64_t w0 = tile * kRsTile + warp * kRsPerWarp;
  constexpr int R = kRsPerWarp / 32;
  uint32_t key[R], rnk[R];
  // per-warp stable ranks, in element order
#pragma unroll
  for (int r = 0; r < R; ++r) {
    const int64_t i = w0 + r * 32 + lane;
    const bool valid = i < M;
    key[r] = valid ? src(i) : 0u;
    const uint32_t dig = valid ? ((key[r] >> shift) & 255u) : 0xffffffffu;
    const uint32_t peers = __match_any_sync(0xffffffffu, dig);
    const int leader = __ffs(peers) - 1;
    uint32_t old = 0;
    if (valid && lane == leader) {
      old = wcount[warp][dig];
      wcount[warp][dig] = old + __popc(peers);
    }
    old = __shfl_sync(0xffffffffu, old, leader);
    rnk[r] = old + __popc(peers & lanemask_lt());
    __syncwarp();
  }
  __syncthreads();
  const int d = threadIdx.x;  // one digit per thread
  uint32_t local = 0;
  for (int w = 0; w < kRsWarps; ++w) {
    const uint32_t c = wcount[w][d];
    wcount[w][d] = local;
    local += c;
  }
  uint32_t* mine = look + tile * 256 + d;
  uint32_t excl = 0;
  if (tile == 0) {
    st_relaxed(mine, kLbIncl | local);
  } else {
    st_relaxed(mine, kLbAgg | local);
    const uint64_t t0 = global_ns();
    uint32_t polls = 0;
    for (int64_t pt = tile - 1; pt >= 0;) {
      const uint32_t v = ld_relaxed(look + pt * 256 + d);
      const uint32_t state = v & ~kLbCount;
      if (state == 0u) {
        if (++polls >= kWaitMaxPolls || global_ns() - t0 > kWaitLimitNs) {
          raise_status(status, OMNI_DEV_TIMEOUT);
          break;
        }
        __nanosleep(32);
        continue;
      }
      excl += v & kLbCount;
      if (state == kLbIncl) break;
      --pt;
    }
    st_relaxed(mine, kLbIncl | (excl + local));
  }
  // global base of each digit: exclusive scan of the histogram
  const int gex = block_exclusive_scan(static_cast<int>(dgh[d]), warp_tot, &total);
  tbase[d] = static_cast<uint32_t>(gex) + excl;
  __syncthreads();
#pragma unroll
  for (int r = 0; r < R; ++r) {
    const int64_t i = w0 + r * 32 + lane;
    if (i < M) {
      const uint32_t dig = (key[r] >> shift) & 255u;
      const uint32_t pos = tbase[dig] + wcount[warp][dig] + rnk[r];
      if (pos < static_cast<uint64_t>(M)) {
        keys_out[pos] = key[r];
        vals_out[pos] = vals_in ? vals_in[i] : static_cast<uint32_t>(i);
      } else {
        raise_status(status, OMNI_DEV_TIMEOUT);  // only after a timed-out wait
      }
    }
  }
}

// ---- 4. emit ---------------------------------------------------------------
__global__ void __launch_bounds__(256)
    k_emit(const uint32_t* __restrict__ vals, int64_t M, int K,
           const int32_t* __restrict__ tmp_e, const float* __restrict__ tmp_g,
           int32_t* __restrict__ task_token, int32_t* __restrict__ task_expert,
           float* __restrict__ task_gate) {
  pdl_wait();
  pdl_trigger();
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= M) return;
  const uint32_t pos = vals ? vals[i] : static_cast<uint32_t>(i);
  task_token[i] = static_cast<int32_t>(pos / static_cast<uint32_t>(K));
  task_expert[i] = tmp_e[pos];
  task_gate[i] = tmp_g[pos];
}

// ---- small batches (M <= kSmallMax): the whole schedule in one cluster -------
//
// Eight CTAs of one thread-block cluster each own a contiguous eighth of the
// tasks in shared memory.  Every stable LSD radix pass (8-bit digits) ranks
// each CTA's keys per warp in element order, exchanges the per-CTA digit
// totals through distributed shared memory, and scatters every key straight
// into the shared memory of the CTA that owns its new position.  (1) Sort by
// expert id; the "new id" flags, counted across the cluster, give U and the
// rank of each task's expert.  (2) Stable sort of the expert-ordered tasks
// by group * L + token: equal keys keep their expert order, so the tasks end
// up ordered by (group, token, expert).  (3) Emit.  Every CTA takes the same
// sequence of cluster barriers; none waits on a flag.
constexpr int kSmallMax = kBlockSortMax;
constexpr int kClCtas = 8;
constexpr int kClThreads = 512;
constexpr int kClWarps = kClThreads / 32;
constexpr int kClChunk = kSmallMax / kClCtas;      // keys per CTA at most
constexpr int kClRounds = kClChunk / kClThreads;   // 32-key rounds per warp at most

struct ClSmem {
  uint32_t key[2][kClChunk];
  uint16_t val[2][kClChunk];
  uint32_t wcnt[kClWarps][256];
  uint32_t tot[256];    // this CTA's digit totals, read by the other CTAs
  uint32_t base[256];
  int warp_tot[32];
  int total;
  int news;             // "new id" flags in this CTA, read by the other CTAs
};

// One stable radix pass over the cluster: keys move from buffer `in` to
// buffer in ^ 1 (of whichever CTA owns their new position).
__device__ void cl_radix_pass(cg::cluster_group& cl, ClSmem& S, int in, int n_local, int chunk,
                              int shift) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int rank = static_cast<int>(cl.block_rank());
  const int rounds = (n_local + kClThreads - 1) / kClThreads;
  for (int j = tid; j < kClWarps * 256; j += kClThreads) (&S.wcnt[0][0])[j] = 0u;
  __syncthreads();
  uint32_t dig[kClRounds], rnk[kClRounds];
#pragma unroll
  for (int r = 0; r < kClRounds; ++r) {
    dig[r] = 0xffffffffu;
    rnk[r] = 0u;
    if (r < rounds) {  // block-uniform
      const int j = (warp * rounds + r) * 32 + lane;
      const bool valid = j < n_local;
      dig[r] = valid ? ((S.key[in][j] >> shift) & 255u) : 0xffffffffu;
      const uint32_t peers = __match_any_sync(0xffffffffu, dig[r]);
      const int leader = __ffs(peers) - 1;
      uint32_t old = 0;
      if (valid && lane == leader) {
        old = S.wcnt[warp][dig[r]];
        S.wcnt[warp][dig[r]] = old + __popc(peers);
      }
      old = __shfl_sync(0xffffffffu, old, leader);
      rnk[r] = old + __popc(peers & lanemask_lt());
      __syncwarp();
    }
  }
  __syncthreads();
  if (tid < 256) {
    uint32_t run = 0;
    for (int w = 0; w < kClWarps; ++w) {
      const uint32_t c = S.wcnt[w][tid];
      S.wcnt[w][tid] = run;
      run += c;
    }
    S.tot[tid] = run;
  }
  cl.sync();  // every CTA's digit totals are visible
  int all = 0;
  if (tid < 256) {
    uint32_t before = 0, sum = 0;
    for (int c = 0; c < kClCtas; ++c) {
      const uint32_t v = cl.map_shared_rank(S.tot, c)[tid];
      sum += v;
      if (c < rank) before += v;
    }
    S.base[tid] = before;
    all = static_cast<int>(sum);
  }
  const int ex = block_exclusive_scan(all, S.warp_tot, &S.total);
  if (tid < 256) S.base[tid] += static_cast<uint32_t>(ex);
  __syncthreads();
#pragma unroll
  for (int r = 0; r < kClRounds; ++r) {
    if (r < rounds) {
      const int j = (warp * rounds + r) * 32 + lane;
      if (j < n_local) {
        const uint32_t pos = S.base[dig[r]] + S.wcnt[warp][dig[r]] + rnk[r];
        const int dst = static_cast<int>(pos / static_cast<uint32_t>(chunk));
        const int off = static_cast<int>(pos - static_cast<uint32_t>(dst) * chunk);
        cl.map_shared_rank(&S.key[in ^ 1][0], dst)[off] = S.key[in][j];
        cl.map_shared_rank(&S.val[in ^ 1][0], dst)[off] = S.val[in][j];
      }
    }
  }
  cl.sync();  // every key has landed in its new owner's buffer
}

__global__ void __cluster_dims__(kClCtas, 1, 1) __launch_bounds__(kClThreads)
    k_sched_cluster(const int32_t* __restrict__ idx, const float* __restrict__ gate, int64_t L,
                    int K, int64_t N, int64_t B, int epasses, int kpasses,
                    int32_t* __restrict__ task_token, int32_t* __restrict__ task_expert,
                    float* __restrict__ task_gate, int32_t* __restrict__ uniq,
                    int32_t* __restrict__ group_off, int32_t* counts) {
  pdl_wait();
  pdl_trigger();
  __shared__ ClSmem S;
  cg::cluster_group cl = cg::this_cluster();
  const int tid = threadIdx.x;
  const int rank = static_cast<int>(cl.block_rank());
  const int M = static_cast<int>(L * K);
  const int chunk = (M + kClCtas - 1) / kClCtas;
  const int first = rank * chunk;
  const int n_local = M - first < 0 ? 0 : (M - first < chunk ? M - first : chunk);
  int32_t* status = counts + 2;
  // (1) load this CTA's tasks: key = expert id, value = task index
  for (int j = tid; j < n_local; j += kClThreads) {
    int64_t e = idx[first + j];
    if (e < 0 || e >= N) {
      raise_status(status, OMNI_DEV_BAD_INDEX);
      e = 0;
    }
    S.key[0][j] = static_cast<uint32_t>(e);
    S.val[0][j] = static_cast<uint16_t>(first + j);
  }
  __syncthreads();
  int cur = 0;
  for (int p = 0; p < epasses; ++p) {
    cl_radix_pass(cl, S, cur, n_local, chunk, 8 * p);
    cur ^= 1;
  }
  // ranks: thread tid takes elements 2*tid, 2*tid + 1 of this CTA (position order)
  const uint32_t prev_last =
      (rank > 0 && n_local > 0) ? cl.map_shared_rank(&S.key[cur][0], rank - 1)[chunk - 1] : 0u;
  int nnew = 0;
  bool isnew[kClChunk / kClThreads];
#pragma unroll
  for (int q = 0; q < kClChunk / kClThreads; ++q) {
    const int j = tid * (kClChunk / kClThreads) + q;
    isnew[q] = false;
    if (j < n_local) {
      const uint32_t prev = j > 0 ? S.key[cur][j - 1] : prev_last;
      isnew[q] = (first + j == 0) || S.key[cur][j] != prev;
      nnew += isnew[q];
    }
  }
  const int ex = block_exclusive_scan(nnew, S.warp_tot, &S.total);
  if (tid == 0) S.news = S.total;
  cl.sync();
  int before = 0, n_active = 0;
  for (int c = 0; c < kClCtas; ++c) {
    const int v = *cl.map_shared_rank(&S.news, c);
    n_active += v;
    if (c < rank) before += v;
  }
  const int64_t G = (n_active + B - 1) / B;
  if (rank == 0 && tid == 0) {
    counts[0] = n_active;
    counts[1] = static_cast<int32_t>(G);
  }
  // (2) key g * L + t in place of the expert id (same positions, same CTA)
  int r = before + ex - 1;
#pragma unroll
  for (int q = 0; q < kClChunk / kClThreads; ++q) {
    const int j = tid * (kClChunk / kClThreads) + q;
    if (j < n_local) {
      if (isnew[q]) {
        ++r;
        uniq[r] = static_cast<int32_t>(S.key[cur][j]);
      }
      const uint32_t i = S.val[cur][j];
      const uint32_t g = static_cast<uint32_t>(r / B);
      S.key[cur][j] = g * static_cast<uint32_t>(L) + i / static_cast<uint32_t>(K);
    }
  }
  cl.sync();  // no CTA still reads a neighbour's last expert id
  for (int p = 0; p < kpasses; ++p) {
    cl_radix_pass(cl, S, cur, n_local, chunk, 8 * p);
    cur ^= 1;
  }
  // (3) emit
  const uint32_t prev_key =
      (rank > 0 && n_local > 0) ? cl.map_shared_rank(&S.key[cur][0], rank - 1)[chunk - 1] : 0u;
  for (int j = tid; j < n_local; j += kClThreads) {
    const int p = first + j;
    const int i = S.val[cur][j];
    const uint32_t g = S.key[cur][j] / static_cast<uint32_t>(L);
    task_token[p] = i / K;
    int32_t e = idx[i];
    if (e < 0 || e >= N) e = 0;
    task_expert[p] = e;
    task_gate[p] = gate[i];
    const uint32_t pk = j > 0 ? S.key[cur][j - 1] : prev_key;
    if (p == 0 || pk / static_cast<uint32_t>(L) != g) group_off[g] = p;
    if (p == M - 1) group_off[G] = M;
  }
  cl.sync();  // keep this CTA's shared memory alive until its neighbour has read it
}

// ---- small batches: a bitmap of the active ids across a cluster -----------
//
// One thread-block cluster of 8 CTAs.  CTA c holds tokens [c*Lc, (c+1)*Lc)
// and the bitmap of ids [c*S, (c+1)*S); the CTAs reach each other's shared
// memory directly.  Warps hold whole tokens, 32*W/P per pass (P = K rounded
// up to a power of two).
//  (A) Each token's K ids are sorted in registers and set their bits in the
//      bitmap of the CTA that owns them.
//  (B) Each CTA counts its bits in 8-word chunks and scans them; the CTA
//      totals, summed across the cluster, give |U| and the first rank of each
//      CTA's ids.  Each CTA writes its part of U.  The rank of any id is then
//      its CTA's first rank plus its chunk's prefix plus the popcounts of the
//      chunk's earlier words and of its own word below it.
//  (C) Per token, the rank and group g = rank / B of every task.  A token's
//      tasks of one group are consecutive in its sorted list, so a task's
//      place among them is its distance to the first of them; the last one
//      writes their count into the cell (g, token).  Each CTA sums its cells
//      per group.
//  (D) The group sums of all CTAs give the first position of every group and
//      of every cell: groups in order, inside a group the tokens of CTA 0,
//      then CTA 1, ..., each CTA's tokens in order.
//  (E) Every task goes to its position: (group, token, expert) order, with
//      equal ids of one token (only out-of-range ids, read as 0) in slot order.
// The cluster takes the same five barriers on every path; no CTA waits on a
// flag.  Batches beyond its limits take the radix cluster sort above.
constexpr int kCbCtas = 8;
constexpr int kCbThreads = 512;
constexpr int kCbWarps = kCbThreads / 32;
constexpr int kCbChunk = 8;             // bitmap words per chunk prefix
constexpr int64_t kCbSlice = 1024;      // ids per CTA: a multiple of this
constexpr int64_t kCbMaxWords = 16384;  // bitmap words per CTA: N <= 2^22
constexpr int64_t kCbMaxTokens = 64;    // tokens per CTA
constexpr int64_t kCbMaxCells = 8192;   // gmax * tokens per CTA
constexpr int kCbMaxK = 256;
constexpr int kCbSlotBits = 8;          // se = e << 8 | slot; info = g << 8 | place
constexpr size_t kCbMaxSmem = 200 * 1024;

__device__ __forceinline__ void cluster_arrive_release() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait_acquire() {
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

template <int P>
__global__ void __cluster_dims__(kCbCtas, 1, 1) __launch_bounds__(kCbThreads)
    k_sched_bits(const int32_t* __restrict__ idx, const float* __restrict__ gate, int L, int K,
                 int64_t N, int64_t B, uint32_t Bq, int S, int words, int Lc, int gmax,
                 int32_t* __restrict__ task_token, int32_t* __restrict__ task_expert,
                 float* __restrict__ task_gate, int32_t* __restrict__ uniq,
                 int32_t* __restrict__ group_off, int32_t* counts) {
  constexpr int W = P > 32 ? P / 32 : 1;  // keys per lane: one token spans W rows
  constexpr int TP = 32 * W / P;          // tokens per warp and pass
  constexpr int WIDTH = P < 32 ? P : 32;  // lanes of one token in a row
  constexpr uint32_t kSlotMask = (1u << kCbSlotBits) - 1u;
  constexpr uint32_t kFull = 0xffffffffu;
  extern __shared__ __align__(16) uint32_t csm[];
  __shared__ int warp_tot[32];
  __shared__ int total;
  __shared__ int tot_local;               // this CTA's active ids, read by the others
  __shared__ int first_rank[kCbCtas + 1]; // first rank of each CTA's ids; [8] = |U|
  cg::cluster_group cl = cg::this_cluster();
  const int crank = static_cast<int>(cl.block_rank());
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int M = L * K;
  const int t_lo = crank * Lc;
  const int t_hi = L < t_lo + Lc ? L : t_lo + Lc;
  const int Mc = t_hi > t_lo ? (t_hi - t_lo) * K : 0;
  const int nchunks = words / kCbChunk;
  uint32_t* bits = csm;                         // ids [crank*S, crank*S + S)
  int* cpre = reinterpret_cast<int*>(bits + words);
  int* cells = cpre + nchunks;                  // [gmax][Lc]
  int* sg = cells + gmax * Lc;                  // [gmax] this CTA's tasks per group
  int* gtot = sg + gmax;                        // [gmax] all CTAs' tasks per group
  int* gbef = gtot + gmax;                      // [gmax] the earlier CTAs' tasks per group
  uint32_t* se = reinterpret_cast<uint32_t*>(gbef + gmax);  // [Lc*K] e << 8 | slot
  uint32_t* info = se + Lc * K;                 // [Lc*K] g << 8 | place
  int32_t* status = counts + 2;
  const int t_first = t_lo + warp * TP;
  const int t_step = kCbWarps * TP;

  // clearing the bitmaps and the cells needs nothing from the kernel before
  // this one: it runs while that kernel finishes
  for (int j = tid; j < words / 4; j += kCbThreads)
    reinterpret_cast<uint4*>(bits)[j] = make_uint4(0u, 0u, 0u, 0u);
  for (int j = tid; j < gmax * Lc; j += kCbThreads) cells[j] = 0;
  cl.sync();  // (1) every bitmap is clear
  pdl_wait();
  pdl_trigger();
  uint32_t key[W];
  int eid[W];
  auto load_keys = [&](int t0) {
#pragma unroll
    for (int w = 0; w < W; ++w) {
      const int i = w * 32 + lane;
      const int t = t0 + i / P, q = i % P;
      key[w] = 0u;  // complement of the largest key: sorts last
      eid[w] = -1;
      if (t < t_hi && q < K) {
        int64_t e = idx[static_cast<int64_t>(t) * K + q];
        if (e < 0 || e >= N) {
          raise_status(status, OMNI_DEV_BAD_INDEX);
          e = 0;
        }
        eid[w] = static_cast<int>(e);
        key[w] = ~((static_cast<uint32_t>(e) << kCbSlotBits) | static_cast<uint32_t>(q));
      }
    }
  };
  // (A)
  for (int t0 = t_first; t0 < t_hi; t0 += t_step) {
    load_keys(t0);
#pragma unroll
    for (int w = 0; w < W; ++w) {
      if (eid[w] >= 0) {
        const int o = eid[w] / S;
        atomicOr(cl.map_shared_rank(bits, o) + ((eid[w] - o * S) >> 5), 1u << (eid[w] & 31));
      }
    }
    reg_sort_desc<W, P>(key);
#pragma unroll
    for (int w = 0; w < W; ++w) {
      const int i = w * 32 + lane;
      const int t = t0 + i / P, q = i % P;
      if (t < t_hi && q < K) se[(t - t_lo) * K + q] = ~key[w];
    }
  }
  cl.sync();  // (2) every bit is set
  // (B) chunk popcounts (a warp reads 128 consecutive words a step), then their scan
  for (int base = warp * 128; base < words; base += kCbWarps * 128) {
    const int wd = base + lane * 4;
    int c = 0;
    if (wd < words) {
      const uint4 v = *reinterpret_cast<const uint4*>(bits + wd);
      c = __popc(v.x) + __popc(v.y) + __popc(v.z) + __popc(v.w);
    }
    c += __shfl_xor_sync(kFull, c, 1);
    if (wd < words && (lane & 1) == 0) cpre[wd / kCbChunk] = c;
  }
  __syncthreads();
  {
    int4 v = make_int4(0, 0, 0, 0);
    if (tid * 4 < nchunks) v = reinterpret_cast<const int4*>(cpre)[tid];
    const int ex = block_exclusive_scan(v.x + v.y + v.z + v.w, warp_tot, &total);
    if (tid * 4 < nchunks)
      reinterpret_cast<int4*>(cpre)[tid] =
          make_int4(ex, ex + v.x, ex + v.x + v.y, ex + v.x + v.y + v.z);
    if (tid == 0) tot_local = total;
  }
  cl.sync();  // (3) every CTA's total is visible
  if (warp == 0) {
    const int v = lane < kCbCtas ? *cl.map_shared_rank(&tot_local, lane) : 0;
    int incl = v;
#pragma unroll
    for (int o = 1; o < kCbCtas; o <<= 1) {
      const int x = __shfl_up_sync(kFull, incl, o);
      if (lane >= o) incl += x;
    }
    if (lane < kCbCtas) first_rank[lane] = incl - v;
    if (lane == kCbCtas - 1) first_rank[kCbCtas] = incl;
  }
  __syncthreads();
  const int n_active = first_rank[kCbCtas];
  const int64_t G = (n_active + B - 1) / B;
  if (crank == 0 && tid == 0) {
    counts[0] = n_active;
    counts[1] = static_cast<int32_t>(G);
    group_off[G] = M;
  }
  // this CTA's part of U, a chunk per thread
  for (int ch = tid; ch < nchunks; ch += kCbThreads) {
    int r = first_rank[crank] + cpre[ch];
    const uint4 lo = reinterpret_cast<const uint4*>(bits)[ch * 2];
    const uint4 hi = reinterpret_cast<const uint4*>(bits)[ch * 2 + 1];
    const uint32_t wv[kCbChunk] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
#pragma unroll
    for (int u = 0; u < kCbChunk; ++u) {
      uint32_t v = wv[u];
      while (v != 0u) {
        const int b = __ffs(v) - 1;
        v &= v - 1u;
        uniq[r++] = crank * S + (ch * kCbChunk + u) * 32 + b;
      }
    }
  }
  // (C) per token: ranks, groups, places and cell counts
  for (int t0 = t_first; t0 < t_hi; t0 += t_step) {
    int g[W];
#pragma unroll
    for (int w = 0; w < W; ++w) {
      const int i = w * 32 + lane;
      const int t = t0 + i / P, q = i % P;
      g[w] = -1;
      if (t < t_hi && q < K) {
        const uint32_t e = se[(t - t_lo) * K + q] >> kCbSlotBits;
        const int o = static_cast<int>(e) / S;
        const int wd = (static_cast<int>(e) - o * S) >> 5, c0 = wd & ~(kCbChunk - 1);
        const uint4* rb = reinterpret_cast<const uint4*>(cl.map_shared_rank(bits, o) + c0);
        const uint4 lo = rb[0], hi = rb[1];
        const uint32_t wv[kCbChunk] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
        int r = first_rank[o] + cl.map_shared_rank(cpre, o)[wd / kCbChunk];
        const int jw = wd - c0;
        const uint32_t below = (1u << (e & 31)) - 1u;
#pragma unroll
        for (int u = 0; u < kCbChunk; ++u)
          r += __popc(wv[u] & (u < jw ? kFull : (u == jw ? below : 0u)));
        g[w] = static_cast<int>(static_cast<uint32_t>(r) / Bq);
      }
    }
    int carry = 0;  // first place of the run that reaches into this row
#pragma unroll
    for (int w = 0; w < W; ++w) {
      const int i = w * 32 + lane;
      const int t = t0 + i / P, q = i % P;
      const int row_prev = __shfl_sync(kFull, g[w > 0 ? w - 1 : 0], 31);
      const int row_next = __shfl_sync(kFull, g[w + 1 < W ? w + 1 : W - 1], 0);
      int gp = __shfl_up_sync(kFull, g[w], 1, WIDTH);
      int gn = __shfl_down_sync(kFull, g[w], 1, WIDTH);
      if (w > 0 && lane == 0) gp = row_prev;
      if (w + 1 < W && lane == 31) gn = row_next;
      int first = (q == 0 || gp != g[w]) ? q : 0;
#pragma unroll
      for (int o = 1; o < WIDTH; o <<= 1) {
        const int f = __shfl_up_sync(kFull, first, o, WIDTH);
        if ((lane % WIDTH) >= o) first = f > first ? f : first;
      }
      first = first > carry ? first : carry;
      carry = __shfl_sync(kFull, first, 31);
      if (t < t_hi && q < K) {
        const int place = q - first;
        info[(t - t_lo) * K + q] =
            (static_cast<uint32_t>(g[w]) << kCbSlotBits) | static_cast<uint32_t>(place);
        if (q == K - 1 || gn != g[w]) cells[g[w] * Lc + (t - t_lo)] = place + 1;
      }
    }
  }
  __syncthreads();
  for (int g = tid; g < G; g += kCbThreads) {
    int sum = 0;
    for (int tl = 0; tl < Lc; ++tl) sum += cells[g * Lc + tl];
    sg[g] = sum;
  }
  cl.sync();  // (4) every CTA's group sums are visible
  // (D) group totals (thread k takes groups [k*per, k*per + per)), their scan, cell bases
  const int per = static_cast<int>((G + kCbThreads - 1) / kCbThreads);
  int mine = 0;
  for (int g = tid * per; g < G && g < tid * per + per; ++g) {
    int all = 0, before = 0;
    for (int c = 0; c < kCbCtas; ++c) {
      const int v = cl.map_shared_rank(sg, c)[g];
      all += v;
      if (c < crank) before += v;
    }
    gtot[g] = all;
    gbef[g] = before;
    mine += all;
  }
  cluster_arrive_release();  // this CTA reads no other CTA's shared memory from here on
  {
    int run = block_exclusive_scan(mine, warp_tot, &total);
    for (int g = tid * per; g < G && g < tid * per + per; ++g) {
      if (crank == 0) group_off[g] = run;
      int pos = run + gbef[g];
      for (int tl = 0; tl < Lc; ++tl) {
        const int v = cells[g * Lc + tl];
        cells[g * Lc + tl] = pos;
        pos += v;
      }
      run += gtot[g];
    }
  }
  __syncthreads();
  // (E)
  for (int j = tid; j < Mc; j += kCbThreads) {
    const int tl = j / K;
    const uint32_t a = se[j], b = info[j];
    const int pos = cells[static_cast<int>(b >> kCbSlotBits) * Lc + tl] + static_cast<int>(b & kSlotMask);
    if (pos < 0 || pos >= M) {  // unreachable for consistent inputs; never write outside
      raise_status(status, OMNI_DEV_BAD_INDEX);
      continue;
    }
    const int t = t_lo + tl;
    task_token[pos] = t;
    task_expert[pos] = static_cast<int32_t>(a >> kCbSlotBits);
    task_gate[pos] = gate[static_cast<int64_t>(t) * K + (a & kSlotMask)];
  }
  cluster_wait_acquire();  // (5) no CTA still reads this CTA's shared memory
}

// The bitmap cluster scheduler's layout, or false when it does not apply.
struct CbPlan {
  int S, words, Lc, gmax;
  size_t smem;
};
bool bits_plan(const Dims& D, CbPlan* p) {
  const int64_t N = D.N(), M = D.M();
  if (M > kSmallMax || D.K > kCbMaxK) return false;
  const int64_t S = (N + kCbCtas * kCbSlice - 1) / (kCbCtas * kCbSlice) * kCbSlice;
  const int64_t words = S / 32;
  const int64_t Lc = (D.L + kCbCtas - 1) / kCbCtas;
  const int64_t gmax = D.gmax();
  if (words > kCbMaxWords || Lc > kCbMaxTokens || gmax * Lc > kCbMaxCells) return false;
  const size_t smem = sizeof(uint32_t) *
      static_cast<size_t>(words + words / kCbChunk + gmax * Lc + 3 * gmax + 2 * Lc * D.K);
  if (smem > kCbMaxSmem) return false;
  *p = CbPlan{static_cast<int>(S), static_cast<int>(words), static_cast<int>(Lc),
              static_cast<int>(gmax), smem};
  return true;
}

template <int P>
cudaError_t launch_bits(const Dims& D, const CbPlan& p, const int32_t* idx, const float* gate,
                        int32_t* task_token, int32_t* task_expert, float* task_gate,
                        int32_t* uniq, int32_t* group_off, int32_t* counts, cudaStream_t s) {
  cudaError_t err = cudaFuncSetAttribute(k_sched_bits<P>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(p.smem));
  if (err != cudaSuccess) return err;
  // ranks are below 2^22: any B beyond 2^30 puts every expert in group 0
  const uint32_t Bq = static_cast<uint32_t>(D.B < (int64_t(1) << 30) ? D.B : (int64_t(1) << 30));
  OMNI_TRY(launch_k(k_sched_bits<P>, kCbCtas, kCbThreads, p.smem, s, idx, gate,
      static_cast<int>(D.L), static_cast<int>(D.K), D.N(), D.B, Bq, p.S, p.words, p.Lc, p.gmax,
      task_token, task_expert, task_gate, uniq, group_off, counts));
  return cudaGetLastError();
}

struct SchedWs {
  int32_t *mult, *rank, *tmp_e;
  uint64_t* tile_sum;
  float* tmp_g;
  int32_t* cnt;  // windows: [nwin][L] tasks per (window, token)
  uint32_t *ka, *va, *kb, *vb, *sweep;  // sweep: [passes][256] histogram, [passes] tile
                                        // counters, [passes][ntiles][256] look-back words
  size_t sweep_words;
  int64_t nscan, ntiles;
  int passes;
};

// windows: the scratch of launch_schedule_windows (no radix buffers; the
// (window, token) counts instead)
SchedWs carve(const Dims& D, void* base, size_t* bytes, bool windows = false) {
  Carver c(base);
  SchedWs w{};
  const int64_t N = D.N(), M = D.M();
  if (M <= kSmallMax && !windows) {  // the cluster paths work in shared memory only
    if (bytes) *bytes = 0;
    return w;
  }
  w.nscan = (N + kScanTile - 1) / kScanTile;
  w.ntiles = (M + kRsTile - 1) / kRsTile;
  int bits = 0;
  while ((int64_t(1) << bits) < D.gmax()) ++bits;
  w.passes = (bits + 7) / 8;
  w.mult = c.take<int32_t>(N);
  w.rank = c.take<int32_t>(N);
  w.tile_sum = c.take<uint64_t>(w.nscan + 1);
  w.tmp_e = c.take<int32_t>(M);
  w.tmp_g = c.take<float>(M);
  if (windows) {
    const int64_t T = window_tasks(D);
    w.cnt = c.take<int32_t>(static_cast<size_t>((M + T - 1) / T) * D.L);
  } else if (w.passes > 0) {
    w.ka = c.take<uint32_t>(M);
    w.va = c.take<uint32_t>(M);
    w.kb = c.take<uint32_t>(M);
    w.vb = c.take<uint32_t>(M);
    w.sweep_words = static_cast<size_t>(w.passes) * (256 + 1 + 256 * w.ntiles);
    w.sweep = c.take<uint32_t>(w.sweep_words);
  }
  if (bytes) *bytes = c.off;
  return w;
}

// zero the task counts, sort every token's tasks, scan the counts: ranks,
// U, |U|, G and the group offsets
cudaError_t prep_and_scan(const Dims& D, const int32_t* idx, const float* gate, int32_t* uniq,
                          int32_t* group_off, int32_t* counts, const SchedWs& w, cudaStream_t s) {
  const int64_t N = D.N();
  int32_t* status = counts + 2;
  cudaError_t err = launch_zero(w.mult, static_cast<size_t>(N), s);
  if (err != cudaSuccess) return err;
  const unsigned prep_blocks = static_cast<unsigned>((D.L + kPrepWarps - 1) / kPrepWarps);
  auto prep = [&](auto kern) {
    return launch_k(kern, prep_blocks, kPrepWarps * 32, 0, s, idx, gate, D.L,
                    static_cast<int>(D.K), N, w.mult, w.tmp_e, w.tmp_g, status);
  };
  OMNI_TRY(D.K <= 32 ? prep(k_prep<1>) : D.K <= 64 ? prep(k_prep<2>)
           : D.K <= 128 ? prep(k_prep<4>) : prep(k_prep<8>));
  OMNI_TRY(launch_k(k_scan_reduce, static_cast<unsigned>(w.nscan), kScanThreads, 0, s, w.mult, N,
      w.tile_sum));
  OMNI_TRY(launch_k(k_scan_tiles, 1, kScanThreads, 0, s, w.tile_sum, static_cast<int>(w.nscan), D.B,
      counts));
  OMNI_TRY(launch_k(k_scan_finish, static_cast<unsigned>(w.nscan), kScanThreads, 0, s, w.mult, N,
      w.tile_sum, D.B, D.M(), static_cast<const int32_t*>(counts), w.rank, uniq, group_off));
  return cudaGetLastError();
}

// ---- the fused forward's windows: the tasks in window token order --------
//
// Window w holds the groups whose first task lies in [w*T, (w+1)*T); the
// expert stage wants its tasks by token, a token's tasks by expert.  A
// token's tasks, sorted by expert, visit the windows in order, so the tasks
// of one (window, token) pair are consecutive in its list.  cnt[w][t] counts
// them; scanned along t it gives the pair's first position inside the
// window, whose own first position is its first group's.  The order equals
// that of a stable sort by token of the window's tasks in schedule order.
constexpr int64_t kWinCellsMax = int64_t(1) << 23;  // nwin * L

// Token t's task j (sorted by expert): its window, and the index of the first
// task of its (window, token) run.  One warp per token, element j = w*32 + lane.
template <int W>
__device__ __forceinline__ void token_windows(const int32_t* __restrict__ tmp_e,
                                              const int32_t* __restrict__ rank,
                                              const int32_t* __restrict__ group_off, int64_t t,
                                              int K, int64_t B, int64_t T, int (&win)[W],
                                              int (&first)[W], uint32_t (&last)[W]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int w = 0; w < W; ++w) {
    const int j = w * 32 + lane;
    win[w] = -1;
    if (j < K) {
      const int32_t e = tmp_e[t * K + j];
      const int64_t g = rank[e] / B;
      win[w] = static_cast<int>(group_off[g] / T);
    }
  }
  int carry = 0;
#pragma unroll
  for (int w = 0; w < W; ++w) {
    const int j = w * 32 + lane;
    const int row_prev = __shfl_sync(0xffffffffu, win[w > 0 ? w - 1 : 0], 31);
    const int row_next = __shfl_sync(0xffffffffu, win[w + 1 < W ? w + 1 : W - 1], 0);
    int wp = __shfl_up_sync(0xffffffffu, win[w], 1);
    int wn = __shfl_down_sync(0xffffffffu, win[w], 1);
    if (w > 0 && lane == 0) wp = row_prev;
    if (w + 1 < W && lane == 31) wn = row_next;
    int f = (j == 0 || wp != win[w]) ? j : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int x = __shfl_up_sync(0xffffffffu, f, o);
      if (lane >= o) f = x > f ? x : f;
    }
    f = f > carry ? f : carry;
    carry = __shfl_sync(0xffffffffu, f, 31);
    first[w] = f;
    last[w] = (j < K && (j == K - 1 || wn != win[w])) ? 1u : 0u;
  }
}

template <int W>
__global__ void __launch_bounds__(kPrepWarps * 32)
    k_wincount(const int32_t* __restrict__ tmp_e, const int32_t* __restrict__ rank,
               const int32_t* __restrict__ group_off, int64_t L, int K, int64_t B, int64_t T,
               int32_t* __restrict__ cnt) {
  pdl_wait();
  pdl_trigger();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t t = static_cast<int64_t>(blockIdx.x) * kPrepWarps + warp;
  if (t >= L) return;  // warp-uniform
  int win[W], first[W];
  uint32_t last[W];
  token_windows<W>(tmp_e, rank, group_off, t, K, B, T, win, first, last);
#pragma unroll
  for (int w = 0; w < W; ++w)
    if (last[w]) cnt[static_cast<int64_t>(win[w]) * L + t] = w * 32 + lane - first[w] + 1;
}

// One CTA per window: the exclusive scan of its row of L counts, in place,
// and win_lo[w], the window's first task (that of the first group starting at
// or after w*T; M when none does), with win_lo[nwin] = M.
__global__ void __launch_bounds__(kScanThreads)
    k_rowscan(int32_t* __restrict__ cnt, int64_t L, const int32_t* __restrict__ group_off,
              const int32_t* __restrict__ counts, int64_t M, int64_t T,
              int32_t* __restrict__ win_lo) {
  pdl_wait();
  pdl_trigger();
  __shared__ int warp_tot[32];
  __shared__ int total;
  if (threadIdx.x < 32) {  // warp 0: a 32-way search for the first group starting at >= w*T
    const int lane = threadIdx.x;
    const int64_t G = counts[1];
    const int64_t v = static_cast<int64_t>(blockIdx.x) * T;
    int64_t lo = 0, hi = G;  // the answer lies in [lo, hi]; G: no such group
    while (lo < hi) {
      const int64_t step = (hi - lo + 31) / 32;
      const int64_t pos = lo + lane * step;
      const uint32_t ge = __ballot_sync(0xffffffffu, pos < hi && group_off[pos] >= v);
      const uint32_t in = __ballot_sync(0xffffffffu, pos < hi);
      if (ge != 0u) {
        const int f = __ffs(ge) - 1;
        hi = lo + f * step;
        lo = f > 0 ? lo + (f - 1) * step + 1 : hi;
      } else {
        lo = lo + (31 - __clz(in)) * step + 1;
      }
    }
    if (lane == 0) {
      win_lo[blockIdx.x] = lo < G ? group_off[lo] : static_cast<int32_t>(M);
      if (blockIdx.x == gridDim.x - 1) win_lo[gridDim.x] = static_cast<int32_t>(M);
    }
  }
  int32_t* row = cnt + static_cast<int64_t>(blockIdx.x) * L;
  int carry = 0;
  for (int64_t b0 = 0; b0 < L; b0 += kScanTile) {
    const int64_t base = b0 + threadIdx.x * kScanItems;
    int v[kScanItems];
    int sum = 0;
#pragma unroll
    for (int j = 0; j < kScanItems; ++j) {
      v[j] = base + j < L ? row[base + j] : 0;
      sum += v[j];
    }
    int run = carry + block_exclusive_scan(sum, warp_tot, &total);
#pragma unroll
    for (int j = 0; j < kScanItems; ++j) {
      if (base + j < L) row[base + j] = run;
      run += v[j];
    }
    carry += total;
    __syncthreads();  // total is rewritten by the next chunk's scan
  }
}

template <int W>
__global__ void __launch_bounds__(kPrepWarps * 32)
    k_winscatter(const int32_t* __restrict__ tmp_e, const float* __restrict__ tmp_g,
                 const int32_t* __restrict__ rank, const int32_t* __restrict__ group_off,
                 const int32_t* __restrict__ win_lo, const int32_t* __restrict__ cnt, int64_t L,
                 int K, int64_t B, int64_t T, int64_t M, int32_t* __restrict__ wt,
                 int32_t* __restrict__ we, float* __restrict__ wg, int32_t* status) {
  pdl_wait();
  pdl_trigger();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t t = static_cast<int64_t>(blockIdx.x) * kPrepWarps + warp;
  if (t >= L) return;  // warp-uniform
  int win[W], first[W];
  uint32_t last[W];
  token_windows<W>(tmp_e, rank, group_off, t, K, B, T, win, first, last);
#pragma unroll
  for (int w = 0; w < W; ++w) {
    const int j = w * 32 + lane;
    if (j < K) {
      const int64_t pos = static_cast<int64_t>(win_lo[win[w]]) +
                          cnt[static_cast<int64_t>(win[w]) * L + t] + (j - first[w]);
      if (pos < 0 || pos >= M) {  // unreachable for consistent counts; never write outside
        raise_status(status, OMNI_DEV_BAD_INDEX);
        continue;
      }
      wt[pos] = static_cast<int32_t>(t);
      we[pos] = tmp_e[t * K + j];
      wg[pos] = tmp_g[t * K + j];
    }
  }
}

}  // namespace

size_t schedule_ws_bytes(const Dims& D) {
  size_t b = 0;
  carve(D, nullptr, &b);
  return b;
}

cudaError_t launch_schedule(const Dims& D, const int32_t* idx, const float* gate,
                            int32_t* task_token, int32_t* task_expert, float* task_gate,
                            int32_t* uniq, int32_t* group_off, int32_t* counts, void* ws,
                            cudaStream_t s) {
  const int64_t N = D.N(), M = D.M();
  int32_t* status = counts + 2;
  if (M == 0) {
    cudaError_t e = cudaMemsetAsync(counts, 0, 2 * sizeof(int32_t), s);
    if (e == cudaSuccess) e = cudaMemsetAsync(group_off, 0, sizeof(int32_t), s);
    return e;
  }
  CbPlan cp;
  if (bits_plan(D, &cp)) {
#define OMNI_BITS(P_) \
  if (D.K <= P_)      \
    return launch_bits<P_>(D, cp, idx, gate, task_token, task_expert, task_gate, uniq, group_off, \
                           counts, s);
    OMNI_BITS(1) OMNI_BITS(2) OMNI_BITS(4) OMNI_BITS(8) OMNI_BITS(16) OMNI_BITS(32) OMNI_BITS(64)
    OMNI_BITS(128) OMNI_BITS(256)
#undef OMNI_BITS
  }
  if (M <= kSmallMax) {
    auto nbits = [](uint64_t v) {
      int b = 0;
      while ((uint64_t(1) << b) < v) ++b;
      return b;
    };
    const int epasses = (nbits(static_cast<uint64_t>(N)) + 7) / 8;
    // key g * L + t < gmax * L
    const int kpasses =
        (nbits(static_cast<uint64_t>(D.gmax()) * static_cast<uint64_t>(D.L)) + 7) / 8;
    OMNI_TRY(launch_k(k_sched_cluster, kClCtas, kClThreads, 0, s, idx, gate, D.L,
        static_cast<int>(D.K), N, D.B, epasses, kpasses, task_token, task_expert, task_gate, uniq,
        group_off, counts));
    return cudaGetLastError();
  }
  SchedWs w = carve(D, ws, nullptr);
  cudaError_t err = prep_and_scan(D, idx, gate, uniq, group_off, counts, w, s);
  if (err != cudaSuccess) return err;
  const uint32_t* keys = nullptr;
  const uint32_t* vals = nullptr;
  uint32_t *ko = w.ka, *vo = w.va;
  if (w.passes > 0) {
    uint32_t* dgh = w.sweep;
    uint32_t* ctr = dgh + 256 * w.passes;
    uint32_t* look = ctr + w.passes;
    err = launch_zero(w.sweep, w.sweep_words, s);
    if (err != cudaSuccess) return err;
    KeySrc src0{nullptr, w.tmp_e, w.rank, D.B};
    OMNI_TRY(launch_k(k_rs_ghist, static_cast<unsigned>(w.ntiles), kRsThreads, 0, s, src0, M,
        w.passes, dgh));
    for (int p = 0; p < w.passes; ++p) {
      KeySrc src{keys, w.tmp_e, w.rank, D.B};
      OMNI_TRY(launch_k(k_rs_onesweep, static_cast<unsigned>(w.ntiles), kRsThreads, 0, s, src, vals,
          M, 8 * p, dgh + 256 * p, look + static_cast<size_t>(p) * 256 * w.ntiles, ctr + p, ko, vo,
          status));
      keys = ko;
      vals = vo;
      ko = (ko == w.ka) ? w.kb : w.ka;
      vo = (vo == w.va) ? w.vb : w.va;
    }
    err = cudaGetLastError();
    if (err != cudaSuccess) return err;
  }
  OMNI_TRY(launch_k(k_emit, static_cast<unsigned>((M + 255) / 256), 256, 0, s, vals, M,
      static_cast<int>(D.K), w.tmp_e, w.tmp_g, task_token, task_expert, task_gate));
  return cudaGetLastError();
}

size_t windows_ws_bytes(const Dims& D) {
  size_t b = 0;
  carve(D, nullptr, &b, true);
  return b;
}

bool windows_supported(const Dims& D) {
  const int64_t T = window_tasks(D);
  const int64_t nwin = (D.M() + T - 1) / T;
  return D.M() > 0 && nwin * D.L <= kWinCellsMax && D.K <= 256;
}

cudaError_t launch_schedule_windows(const Dims& D, const int32_t* idx, const float* gate,
                                    int32_t* uniq, int32_t* group_off, int32_t* counts, void* ws,
                                    const WinTasks& out, cudaStream_t s) {
  const int64_t M = D.M();
  const int64_t T = window_tasks(D);
  const int nwin = static_cast<int>((M + T - 1) / T);
  SchedWs w = carve(D, ws, nullptr, true);
  cudaError_t err = prep_and_scan(D, idx, gate, uniq, group_off, counts, w, s);
  if (err != cudaSuccess) return err;
  err = launch_zero(w.cnt, static_cast<size_t>(nwin) * D.L, s);
  if (err != cudaSuccess) return err;
  const unsigned blocks = static_cast<unsigned>((D.L + kPrepWarps - 1) / kPrepWarps);
  const int K = static_cast<int>(D.K);
  auto count = [&](auto kern) {
    return launch_k(kern, blocks, kPrepWarps * 32, 0, s, w.tmp_e, w.rank, group_off, D.L, K, D.B,
                    T, w.cnt);
  };
  OMNI_TRY(K <= 32 ? count(k_wincount<1>) : K <= 64 ? count(k_wincount<2>)
           : K <= 128 ? count(k_wincount<4>) : count(k_wincount<8>));
  OMNI_TRY(launch_k(k_rowscan, static_cast<unsigned>(nwin), kScanThreads, 0, s, w.cnt, D.L,
      static_cast<const int32_t*>(group_off), static_cast<const int32_t*>(counts), M, T,
      out.win_lo));
  auto scatter = [&](auto kern) {
    return launch_k(kern, blocks, kPrepWarps * 32, 0, s, w.tmp_e, w.tmp_g, w.rank, group_off,
                    static_cast<const int32_t*>(out.win_lo), static_cast<const int32_t*>(w.cnt),
                    D.L, K, D.B, T, M, out.wt, out.we, out.wg, counts + 2);
  };
  OMNI_TRY(K <= 32 ? scatter(k_winscatter<1>) : K <= 64 ? scatter(k_winscatter<2>)
           : K <= 128 ? scatter(k_winscatter<4>) : scatter(k_winscatter<8>));
  return cudaGetLastError();
}

namespace {
// First position of the sorted ids uniq[0, n) holding an id >= v.
__device__ __forceinline__ int64_t lower_id(const int32_t* uniq, int64_t n, int64_t v) {
  int64_t l = 0, h = n;
  while (l < h) {
    const int64_t m = (l + h) >> 1;
    if (uniq[m] < v) l = m + 1; else h = m;
  }
  return l;
}

// T > 0: the window order (window w holds the groups whose first task lies
// in [w*T, (w+1)*T) and starts at the first of them); the range is widened
// to whole windows.
__global__ void k_shard_range(const int32_t* __restrict__ uniq,
                              const int32_t* __restrict__ group_off,
                              const int32_t* __restrict__ counts, int64_t T, int64_t lo,
                              int64_t hi, int64_t ucap, int64_t gmax, int64_t B, int64_t M,
                              int64_t* __restrict__ arange) {
  pdl_wait();
  pdl_trigger();
  if (threadIdx.x != 0) return;
  int64_t n = counts[0], G = counts[1];
  n = n < 0 ? 0 : (n > ucap ? ucap : n);
  G = G < 0 ? 0 : (G > gmax ? gmax : G);
  const int64_t r0 = lower_id(uniq, n, lo), r1 = lower_id(uniq, n, hi);
  int64_t a0 = 0, a1 = 0;
  if (r1 > r0) {
    const int64_t g0 = r0 / B, g1 = (r1 - 1) / B;  // first and last group of the shard
    a0 = group_off[g0];
    a1 = g1 + 1 < G ? group_off[g1 + 1] : M;
    if (T > 0) {
      // first task of the window holding task position v: that of the first
      // group starting at or after the window's start (M if none)
      auto window_start = [&](int64_t v) {
        const int64_t w0 = (v / T) * T;
        int64_t l = 0, h = G;
        while (l < h) {
          const int64_t m = (l + h) >> 1;
          if (group_off[m] >= w0) h = m; else l = m + 1;
        }
        return l < G ? static_cast<int64_t>(group_off[l]) : M;
      };
      a0 = window_start(a0);
      // the end of the window holding the last group: the start of the next
      const int64_t last = group_off[g1];
      const int64_t next = (last / T + 1) * T;
      a1 = next >= M ? M : window_start(next);
    }
  }
  arange[0] = a0;
  arange[1] = a1;
}

// counts[0] (|U| of the whole batch) and counts[1] replaced by those of the
// shard's ids [lo, hi): the active ids in U (sorted) between the two bounds.
__global__ void k_shard_counts(const int32_t* __restrict__ uniq, int32_t* __restrict__ counts,
                               int64_t lo, int64_t hi, int64_t ucap, int64_t B) {
  pdl_wait();
  pdl_trigger();
  if (threadIdx.x != 0) return;
  int64_t n = counts[0];
  if (n < 0) n = 0;
  if (n > ucap) n = ucap;
  const int64_t u = lower_id(uniq, n, hi) - lower_id(uniq, n, lo);
  counts[0] = static_cast<int32_t>(u);
  counts[1] = static_cast<int32_t>((u + B - 1) / B);
}
}  // namespace

cudaError_t launch_shard_range(const Dims& D, const int32_t* uniq, const int32_t* group_off,
                               const int32_t* counts, int64_t T, int64_t* arange,
                               cudaStream_t s) {
  OMNI_TRY(launch_k(k_shard_range, 1, 32, 0, s, uniq, group_off, counts, T, D.shard_lo(),
      D.shard_hi(), D.ucap(), D.gmax(), D.B, D.M(), arange));
  return cudaGetLastError();
}

cudaError_t launch_shard_counts(const Dims& D, const int32_t* uniq, int32_t* counts,
                                cudaStream_t s) {
  OMNI_TRY(launch_k(k_shard_counts, 1, 32, 0, s, uniq, counts, D.shard_lo(), D.shard_hi(),
      D.ucap(), D.B));
  return cudaGetLastError();
}

}  // namespace omni
