// The activations of dense groups on the tensor cores.
//
// Grouped execution ("OmniMoE: An Efficient MoE by Orchestrating Atomic
// Experts at Scale" (gist.science), Technisch Overzicht section 2.2, grouped
// GEMMs; the OmniMoE explainer on manus.space, Expert-Centric Scheduling):
// group g holds B consecutive active experts and the tasks routed to them,
// sorted by token.  For a block of 128 consecutive tokens the activations
// the group needs are entries of the dense product
//   S = X[block] W_g^T   (128 tokens x B experts, K = d),
// which the tensor cores compute whole; only the entries of actual tasks are
// kept, c = gate * SiLU(S[t, e]).  That can only pay when a group's tiles are
// well filled: a group is dense when its tasks average at least
// kDenseMinTasks per touched block (a batch routed to a few hundred experts
// by many tokens; never a batch whose experts are nearly all distinct, where
// the tile would be > 99.9% waste).  Measured on B200, even a batch of 8192
// tokens routed to 256 experts (two groups, 512 tasks per tile, 3% of it
// used) runs its grouped execution in 0.158 ms this way against 0.099 ms
// with every activation formed on the CUDA cores from L2-resident rows, so
// the path is taken only on request (OMNI_FLAG_DENSE_TENSOR_CORES).  The
// decision is taken on the device, from the schedule:
//
//  1. k_plan_dense (one CTA per group): tasks and touched 128-token blocks of
//     the group; a dense group takes a slot (at most kDenseCap), every task
//     of it gets its column (its expert's rank inside the group, a binary
//     search in the group's slice of U) and every touched block one tile
//     (slot, block, its task range); every task is flagged dense or not.
//  2. k_gather_dense: the W rows of each slot's group, in rank order, into a
//     contiguous panel [B x d] (rows past the group's experts are zero).
//  3. k_gemm_tc over the tile list: A = x (TMA tiles of 128 token rows), B =
//     the panel; the epilogue stages the 128 x 128 tile of S in shared memory
//     and then reads, for every task of the tile (in parallel), the entry of
//     its row and column and writes its c.
// The value rows are added by the grouped-execution kernel, which takes the
// c of flagged tasks instead of forming them itself.
#include "common.cuh"
#include "internal.h"
#include "gemm_tc.cuh"

namespace omni {
namespace {

using namespace tc;

constexpr int kDenseCap = 64;          // dense groups per call (panels in the workspace)
// Tasks per touched 128-token block for a group to be dense (2.3% of a 128 x
// 128 tile): a tile streams at about 6.8 us per SM (the product and its
// staged epilogue, d = 1024), an activation formed on the CUDA cores from
// L2-resident rows at about 22 ns per task per SM.
constexpr int kDenseMinTasks = 384;
constexpr int kDenseBlock = TC_BM;     // tokens per tile
constexpr int kDenseBN = 128;          // experts per tile (B <= 128)
constexpr int kStageLd = kDenseBN + 1; // staged row stride: rows on distinct banks

// Workspace of the dense path: counters, flags, activations, tile list, panels.
struct DenseWs {
  uint32_t* ctr;      // [4]: dense groups, tiles
  uint8_t* flag;      // [M] task of a dense group
  float* cbuf;        // [M] activations of the flagged tasks
  int32_t* col;       // [M] column of a flagged task in its group's tile
  int4* tiles;        // [kDenseCap * blocks] (slot, block, first task, end task)
  int32_t* slot_group;  // [kDenseCap] group of each slot
  __nv_bfloat16* panel;  // [kDenseCap * kDenseBN x d]
};

DenseWs carve_dense(const Dims& D, void* ws, size_t* bytes) {
  Carver c(ws);
  DenseWs w;
  const int64_t M = D.M();
  const int64_t blocks = (D.L + kDenseBlock - 1) / kDenseBlock;
  w.ctr = c.take<uint32_t>(4);
  w.flag = c.take<uint8_t>(static_cast<size_t>(M));
  w.cbuf = c.take<float>(static_cast<size_t>(M));
  w.col = c.take<int32_t>(static_cast<size_t>(M));
  w.tiles = c.take<int4>(static_cast<size_t>(kDenseCap * blocks));
  w.slot_group = c.take<int32_t>(kDenseCap);
  w.panel = c.take<__nv_bfloat16>(static_cast<size_t>(kDenseCap) * kDenseBN * D.d);
  if (bytes) *bytes = c.off;
  return w;
}

constexpr int kPlanThreads = 1024;
constexpr int kPlanMaxBlocks = 4096;  // 128-token blocks a batch may have (L <= 2^19)

// One CTA per group g (< gmax; groups past counts[1] exit), every loop over
// the group's tasks spread over the CTA's threads with independent loads.
__global__ void __launch_bounds__(kPlanThreads)
    k_plan_dense(const int32_t* __restrict__ task_token, const int32_t* __restrict__ task_expert,
                 const int32_t* __restrict__ uniq, const int32_t* __restrict__ group_off,
                 const int32_t* __restrict__ counts, int64_t M, int64_t gmax, int64_t B,
                 int64_t blocks, DenseWs w) {
  pdl_wait();
  pdl_trigger();
  __shared__ int nb_sh, slot_sh;
  __shared__ int32_t ids[kDenseBN];               // the group's experts, in rank order
  __shared__ int32_t run_lo[kPlanMaxBlocks], run_hi[kPlanMaxBlocks];
  const int64_t g = blockIdx.x;
  const int64_t G = counts[1];
  if (g >= G || G > gmax) return;  // whole CTA
  const int64_t lo = group_off[g], hi = group_off[g + 1];
  if (lo < 0 || hi > M || lo > hi) return;
  if (threadIdx.x == 0) nb_sh = 0;
  __syncthreads();
  // a task starts (ends) a block's run when the task before (after) it is of
  // another block
  int nb = 0;
#pragma unroll 8
  for (int64_t p = lo + threadIdx.x; p < hi; p += kPlanThreads)
    nb += (p == lo || task_token[p - 1] / kDenseBlock != task_token[p] / kDenseBlock) ? 1 : 0;
  nb = __reduce_add_sync(0xffffffffu, nb);
  if ((threadIdx.x & 31) == 0 && nb != 0) atomicAdd(&nb_sh, nb);
  __syncthreads();
  if (threadIdx.x == 0) {
    int slot = -1;
    if (hi - lo >= static_cast<int64_t>(kDenseMinTasks) * nb_sh) {
      const uint32_t s = atomicAdd(&w.ctr[0], 1u);
      if (s < static_cast<uint32_t>(kDenseCap)) {
        slot = static_cast<int>(s);
        w.slot_group[slot] = static_cast<int32_t>(g);
      }
    }
    slot_sh = slot;
  }
  const int64_t u0 = g * B;
  int64_t nbg = static_cast<int64_t>(counts[0]) - u0;
  nbg = nbg < B ? nbg : B;
  for (int j = threadIdx.x; j < nbg; j += kPlanThreads) ids[j] = uniq[u0 + j];
  for (int64_t j = threadIdx.x; j < blocks; j += kPlanThreads) run_lo[j] = -1;
  __syncthreads();
  const int slot = slot_sh;
  const uint8_t f = slot >= 0 ? 1 : 0;
#pragma unroll 8
  for (int64_t p = lo + threadIdx.x; p < hi; p += kPlanThreads) w.flag[p] = f;
  if (slot < 0) return;
  // columns (the expert's rank inside the group) and the blocks' task runs
#pragma unroll 4
  for (int64_t p = lo + threadIdx.x; p < hi; p += kPlanThreads) {
    const int32_t e = task_expert[p];
    const int b = task_token[p] / kDenseBlock;
    const bool first = p == lo || task_token[p - 1] / kDenseBlock != b;
    const bool last = p + 1 == hi || task_token[p + 1] / kDenseBlock != b;
    int l = 0, h = static_cast<int>(nbg);
    while (l < h) {
      const int m = (l + h) >> 1;
      if (ids[m] < e) l = m + 1; else h = m;
    }
    w.col[p] = l;
    if (first) run_lo[b] = static_cast<int32_t>(p);
    if (last) run_hi[b] = static_cast<int32_t>(p + 1);
  }
  __syncthreads();
  for (int64_t b = threadIdx.x; b < blocks; b += kPlanThreads) {
    if (run_lo[b] < 0) continue;
    const uint32_t t = atomicAdd(&w.ctr[1], 1u);
    if (t < static_cast<uint32_t>(kDenseCap * blocks))
      w.tiles[t] = make_int4(slot, static_cast<int>(b), run_lo[b], run_hi[b]);
  }
}

// Panel rows: slot s, row j = W[U[g*B + j]] for j < the group's experts, else 0.
__global__ void __launch_bounds__(256)
    k_gather_dense(const __nv_bfloat16* __restrict__ W, const int32_t* __restrict__ uniq,
                   int32_t* __restrict__ counts, int64_t N, int64_t B, int bn, int d, DenseWs w) {
  int32_t* status = counts + 2;
  pdl_wait();
  pdl_trigger();
  const uint32_t ndense = w.ctr[0] < static_cast<uint32_t>(kDenseCap) ? w.ctr[0] : kDenseCap;
  const int slot = blockIdx.y;
  if (blockIdx.x == 0 && threadIdx.x == 0 && slot == 0) counts[3] = static_cast<int32_t>(ndense);
  if (slot >= static_cast<int>(ndense)) return;
  const int64_t g = w.slot_group[slot];
  const int64_t n_active = counts[0];
  const int nvec = d / 8;  // 16-byte vectors per row
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
       i < static_cast<int64_t>(bn) * nvec; i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int j = static_cast<int>(i / nvec), v = static_cast<int>(i % nvec);
    const int64_t r = g * B + j;
    uint4 val = make_uint4(0u, 0u, 0u, 0u);
    if (j < B && r < n_active) {
      const int64_t e = uniq[r];
      if (e >= 0 && e < N) {
        val = reinterpret_cast<const uint4*>(W + e * d)[v];
      } else {
        raise_status(status, OMNI_DEV_BAD_INDEX);
      }
    }
    reinterpret_cast<uint4*>(w.panel + (static_cast<int64_t>(slot) * bn + j) * d)[v] = val;
  }
}

// The device-side tile list (count read after the planner finished).
struct ListTiles {
  const int4* tiles;
  const uint32_t* ctr;
  int cap, bn;
  __device__ __forceinline__ int count() const {
    const uint32_t n = ctr[1];
    return n < static_cast<uint32_t>(cap) ? static_cast<int>(n) : cap;
  }
  __device__ __forceinline__ void at(int t, int* a0, int* b0) const {
    const int4 v = tiles[t];
    *a0 = v.y * kDenseBlock;  // token block
    *b0 = v.x * bn;           // the slot's panel
  }
};

// The tile of S is staged row by row in shared memory; then the 128
// epilogue threads take the tile's tasks in parallel: task p reads the entry
// of its token's row and its column and writes c = gate * SiLU(S).
struct TaskActivations {
  static constexpr size_t kStageBytes = sizeof(float) * TC_BM * kStageLd;
  const int4* tiles;
  const int32_t* task_token;
  const float* task_gate;
  const int32_t* col;
  float* cbuf;
  __device__ __forceinline__ void operator()(int, int, int, int r, int c, const uint32_t* v,
                                             float* stage) const {
#pragma unroll
    for (int q = 0; q < 32; ++q) stage[r * kStageLd + c + q] = __uint_as_float(v[q]);
  }
  __device__ __forceinline__ void tile_end(int t, int a0, int, int i, float* stage) const {
    const int4 tl = tiles[t];
    for (int p = tl.z + i; p < tl.w; p += TC_BM) {
      const int row = task_token[p] - a0, cc = col[p];
      cbuf[p] = task_gate[p] * silu(stage[row * kStageLd + cc]);
    }
  }
};

cudaError_t launch_dense_gemm(const Dims& D, const void* x, const int32_t* tt, const float* tg,
                              const DenseWs& w, int64_t blocks, int32_t* status, cudaStream_t s) {
  CUtensorMap a, b;
  if (!make_map(&a, x, D.L, D.d, TC_BM) ||
      !make_map(&b, w.panel, static_cast<int64_t>(kDenseCap) * kDenseBN, D.d, kDenseBN))
    return cudaErrorInvalidValue;
  const int cap = static_cast<int>(kDenseCap * blocks);
  ListTiles T{w.tiles, w.ctr, cap, kDenseBN};
  TaskActivations epi{w.tiles, tt, tg, w.col, w.cbuf};
  return launch_gemm_tc<kDenseBN>(a, b, static_cast<int>((D.d + TC_BK - 1) / TC_BK), T, cap, epi,
                                  status, s);
}

}  // namespace

bool dense_supported(const Dims& D) {
  return D.dtype == OMNI_BF16 && D.d % 64 == 0 && D.B <= kDenseBN && D.d <= 16384 &&
         D.L <= static_cast<int64_t>(kPlanMaxBlocks) * kDenseBlock &&
         (D.flags & OMNI_FLAG_DENSE_TENSOR_CORES) != 0;
}

size_t dense_ws_bytes(const Dims& D) {
  size_t b = 0;
  carve_dense(D, nullptr, &b);
  return b;
}

DenseFlags dense_flags(const Dims& D, void* ws) {
  const DenseWs w = carve_dense(D, ws, nullptr);
  return DenseFlags{w.flag, w.cbuf};
}

cudaError_t launch_dense_activations(const Dims& D, const void* x, const void* W,
                                     const int32_t* task_token, const int32_t* task_expert,
                                     const float* task_gate, const int32_t* uniq,
                                     const int32_t* group_off, int32_t* counts, void* ws,
                                     cudaStream_t s) {
  const DenseWs w = carve_dense(D, ws, nullptr);
  const int64_t blocks = (D.L + kDenseBlock - 1) / kDenseBlock;
  const int64_t gmax = D.gmax();
  int32_t* status = counts + 2;
  OMNI_TRY(launch_zero(w.ctr, 4, s));
  OMNI_TRY(launch_k(k_plan_dense, static_cast<unsigned>(gmax), kPlanThreads, 0, s, task_token,
                    task_expert, uniq, group_off, static_cast<const int32_t*>(counts), D.M(), gmax,
                    D.B, blocks, w));
  const dim3 ggrid(static_cast<unsigned>((kDenseBN * (D.d / 8) + 255) / 256), kDenseCap);
  OMNI_TRY(launch_k(k_gather_dense, ggrid, 256, 0, s, static_cast<const __nv_bfloat16*>(W), uniq,
                    counts, D.N(), D.B, kDenseBN, static_cast<int>(D.d), w));
  return launch_dense_gemm(D, x, task_token, task_gate, w, blocks, status, s);
}

}  // namespace omni
