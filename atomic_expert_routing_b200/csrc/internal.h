// Internal launch interface between the C-ABI layer (api.cu) and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <utility>

#include <nvtx3/nvToolsExt.h>

namespace omni {

// NVTX range over one ABI call or one stage of it, on the host: it spans the
// launches the call enqueues, so a profiler can select a stage's kernels by
// range.  A no-op unless a profiling tool is attached.
struct CallRange {
  explicit CallRange(const char* name) { nvtxRangePushA(name); }
  ~CallRange() { nvtxRangePop(); }
  CallRange(const CallRange&) = delete;
  CallRange& operator=(const CallRange&) = delete;
};

// OMNI_OK for cudaSuccess; otherwise records e as this host thread's last
// CUDA error (omni_last_cuda_error_name) and returns OMNI_ERR_CUDA.
int cuda_status(cudaError_t e);

struct Dims {
  int64_t L, d, Nr, Nc, k, K, B;
  int dtype;
  int flags;
  // Expert shard: this process holds the W/V (and U) rows of ids
  // [e_lo, e_hi), id e in row e - e_lo.  A sharded execution skips the tasks
  // of other ids (silently: they are not bad indices) and leaves its partial
  // sum in fp32, whatever the storage type.  e_hi < 0: not sharded.
  int64_t e_lo = 0, e_hi = -1;
  // device [2] (nullable): the task positions the execution visits for the
  // shard (launch_shard_range); nullptr: every task
  const int64_t* shard_range = nullptr;
  bool sharded() const { return e_hi >= 0; }
  int64_t shard_lo() const { return sharded() ? e_lo : 0; }
  int64_t shard_hi() const { return sharded() ? e_hi : N(); }
  int64_t N() const { return Nr * Nc; }
  int64_t M() const { return L * K; }
  int64_t ucap() const { return N() < M() ? N() : M(); }       // bound on |U|
  int64_t gmax() const { return (ucap() + B - 1) / B; }        // bound on #groups
};

// The ids whose rows this process holds, as the kernels see them: a task of
// id e outside [lo, hi) belongs to another shard and is skipped; row e - lo
// otherwise.  Unsharded: [0, N).
// arange (device, nullable): the task positions [arange[0], arange[1]) of
// the execution order that can hold the shard's tasks (launch_shard_range);
// execution kernels visit only the slices that overlap it.
struct ShardIds {
  int64_t lo, hi;
  const int64_t* arange;
  __host__ __device__ bool has(int64_t e) const { return e >= lo && e < hi; }
  // the slices [*s0, *s1) of S tasks (of nslices) to visit; read on the
  // device after the kernel's dependency wait
  __device__ void slices(int S, int64_t nslices, int64_t* s0, int64_t* s1) const {
    *s0 = 0;
    *s1 = nslices;
    if (arange == nullptr) return;
    const int64_t a0 = arange[0], a1 = arange[1];
    const int64_t b0 = a0 < 0 ? 0 : a0 / S;
    const int64_t b1 = a1 <= 0 ? 0 : (a1 + S - 1) / S;
    *s0 = b0 < nslices ? b0 : nslices;
    *s1 = b1 < nslices ? b1 : nslices;
    if (*s1 < *s0) *s1 = *s0;
  }
};
inline ShardIds shard_ids(const Dims& D) {
  return ShardIds{D.shard_lo(), D.shard_hi(), D.sharded() ? D.shard_range : nullptr};
}

// ---- router logits: Z [L x (Nr + Nc)] fp32 -------------------------------
cudaError_t launch_router_simt(const Dims& D, const void* x, const void* Wr, const void* Wc,
                               float* Z, cudaStream_t s);
bool router_tc_supported(const Dims& D, const void* x, const void* Wr, const void* Wc);
// Number of K-splits of the tensor-core router for these dims (1: no split).
// Split partial logits are written to Z + s * L * (Nr + Nc), s < splits.
int router_splits(const Dims& D);
cudaError_t launch_router_tc(const Dims& D, const void* x, const void* Wr, const void* Wc,
                             float* Z, int32_t* status, cudaStream_t s);
// Z[i] = sum over s < splits of Z[s * n + i] (fixed order), written in place.
cudaError_t launch_sum_partials(float* Z, int splits, int64_t n, cudaStream_t s);

// ---- selection: per-axis top-k, k x k merge, top-K, gate ----------------
// Z holds `parts` consecutive partial logit arrays, summed in order on load.
// zero (nullable, zero_words floats): a buffer the small-batch kernel clears
// before it waits on the kernel ahead of it; *zeroed says whether it did.
cudaError_t launch_select(const Dims& D, const float* Z, int parts, const float* br,
                          const float* bc, int32_t* idx, float* gate, float* score,
                          cudaStream_t s, float* zero = nullptr, int64_t zero_words = 0,
                          bool* zeroed = nullptr);

// ---- windows of consecutive groups (the sweep path of the execution) ------
// Window w holds the groups whose first task lies in [w*T, (w+1)*T).
int64_t window_tasks(const Dims& D);  // T
struct WinTasks {
  int32_t *wt, *we;  // token and expert of every task, in window token order
  float* wg;         // its gate
  int32_t* win_lo;   // [nwin + 1] first task of every window
};

// ---- scheduling ----------------------------------------------------------
size_t schedule_ws_bytes(const Dims& D);
// The fused forward of a large batch: the schedule's ranks, U, counts and
// group offsets, then every task straight into window token order (the
// (group, token) order of omni_schedule is never formed).
bool windows_supported(const Dims& D);
size_t windows_ws_bytes(const Dims& D);
cudaError_t launch_schedule_windows(const Dims& D, const int32_t* idx, const float* gate,
                                    int32_t* uniq, int32_t* group_off, int32_t* counts, void* ws,
                                    const WinTasks& out, cudaStream_t s);
cudaError_t launch_schedule(const Dims& D, const int32_t* idx, const float* gate,
                            int32_t* task_token, int32_t* task_expert, float* task_gate,
                            int32_t* uniq, int32_t* group_off, int32_t* counts, void* ws,
                            cudaStream_t s);

// ---- execution of a small batch straight from the routing: two kernels -----
// Supported: min(N, L*K) rows of W and V within 64 MiB (they stay in L2) or
// L*K rows within 1 GiB, N <= 2^20, 1 <= L <= 65535, d of 256/512/1024/2048 bf16 or
// 128/256/512/1024 fp32 elements; not with OMNI_FLAG_STAGED_SMALL.  A
// function of the dims alone.
bool sched_exec_supported(const Dims& D);
// 32-bit words of workspace (256-byte aligned) the two kernels need; the
// first sched_exec_zero_words(D) words must be zero at the call (the rest is
// scratch).
size_t sched_exec_ws_words(const Dims& D);
size_t sched_exec_zero_words(const Dims& D);
// Writes y [L x d] completely, and counts[0], [1].
cudaError_t launch_sched_exec(const Dims& D, const void* x, const void* W, const void* V,
                              const int32_t* idx, const float* gate, void* y, uint32_t* ws,
                              int32_t* counts, cudaStream_t s, const void* U = nullptr);

// ---- activations of dense groups on the tensor cores ----------------------
// bf16, d a multiple of 64, B <= 256.  The planner flags the tasks of dense
// groups and the tensor-core pass writes their activations c (both in the
// dense workspace); counts[3] receives the number of dense groups.
bool dense_supported(const Dims& D);
size_t dense_ws_bytes(const Dims& D);
struct DenseFlags {
  const uint8_t* flag;  // [M] task of a dense group (its c is in cbuf)
  const float* cbuf;    // [M]
};
DenseFlags dense_flags(const Dims& D, void* ws);
cudaError_t launch_dense_activations(const Dims& D, const void* x, const void* W,
                                     const int32_t* task_token, const int32_t* task_expert,
                                     const float* task_gate, const int32_t* uniq,
                                     const int32_t* group_off, int32_t* counts, void* ws,
                                     cudaStream_t s);

// ---- execution -----------------------------------------------------------
size_t expert_ws_bytes(const Dims& D);
int expert_sweeps(const Dims& D);                // slices of d (1: no sweeps)
WinTasks expert_windows(const Dims& D, void* ws);  // the window buffers of an expert workspace
// The sweeps from tasks already in window token order (expert_windows(ws)).
// U (nullable): the gate matrix of gated experts, h = SiLU(x.W[e]) * (x.U[e]).
cudaError_t launch_expert_windows(const Dims& D, const void* x, const void* W, const void* V,
                                  int32_t* counts, void* y, void* ws, cudaStream_t s,
                                  const void* U = nullptr);
// uniq: the schedule's U (the dense-group path reads it); allow_dense: run
// the activations of dense groups on the tensor cores when the workspace is
// the full OMNI_WS_EXPERT size (false: ws holds only the accumulator).
cudaError_t launch_expert(const Dims& D, const void* x, const void* W, const void* V,
                          const int32_t* task_token, const int32_t* task_expert,
                          const float* task_gate, const int32_t* uniq, const int32_t* group_off,
                          const int32_t* counts, void* y, void* ws, cudaStream_t s,
                          bool acc_zeroed = false, bool allow_dense = true,
                          const void* U = nullptr);
// The accumulator launch_expert clears before a batch without sweeps (its fp32
// partial sums: y itself for fp32, else the head of ws), in floats; 0 for
// batches with sweeps.
int64_t expert_acc_words(const Dims& D);
// y [L x d] in the storage type <- src fp32 (bf16: nearest even; fp32: a
// copy unless src == y).
cudaError_t launch_cast_output(const Dims& D, const float* src, void* y, cudaStream_t s);
// Before a sharded execution: the range of task positions that can hold the
// shard's tasks, arange[0..1], from the schedule (U sorted, group_off) --
// the groups from the one holding the shard's first active id to the one
// holding its last -- and, for the window order of the sweeps (T =
// window_tasks(D); 0 for the schedule's own order), widened to whole
// windows.  Empty ([0, 0)) when the shard has no active id.
cudaError_t launch_shard_range(const Dims& D, const int32_t* uniq, const int32_t* group_off,
                               const int32_t* counts, int64_t T, int64_t* arange,
                               cudaStream_t s);
// After a sharded execution of a schedule: counts[0], counts[1] replaced by
// the shard's active ids in uniq and their group count.
cudaError_t launch_shard_counts(const Dims& D, const int32_t* uniq, int32_t* counts,
                                cudaStream_t s);
cudaError_t launch_token(const Dims& D, const void* x, const void* W, const void* V,
                         const int32_t* idx, const float* gate, void* y, int32_t* status,
                         cudaStream_t s, const void* U = nullptr);

// ---- backward of the routed branch (bf16 storage) --------------------------
struct BwdWs {
  int32_t *task_token, *task_expert, *uniq, *group_off;
  float *task_gate, *da, *dg;
  void* sched;
  uint16_t *dzb, *dzT, *xT, *WrcT;  // bf16 bit patterns
};
// The workspace's buffers (base == nullptr: sizes only, total in *bytes).
BwdWs carve_backward(const Dims& D, void* base, size_t* bytes);
// dx [L x d] fp32 overwritten; dW, dV [N x d] (active rows), dWr [Nr x d],
// dWc [Nc x d], dbr [Nr], dbc [Nc] (nullable) fp32 added to (accumulate) or
// overwritten.  counts[0], [1]: the active experts (twice: groups of one);
// counts[2] status bits.
cudaError_t launch_backward(const Dims& D, const void* x, const void* Wr, const void* Wc,
                            const void* W, const void* V, const int32_t* idx, const float* gate,
                            const void* dy, float* dx, float* dW, float* dV, float* dWr,
                            float* dWc, float* dbr, float* dbc, bool accumulate,
                            int32_t* counts, void* ws, cudaStream_t s);

// ---- shared dense MLP: y (+)= SiLU(x W1^T) W2^T on the tensor cores ---------
// bf16 storage only; ws holds the hidden activations H [L x F] (bf16).
size_t mlp_ws_bytes(const Dims& D, int64_t F);
cudaError_t launch_shared_mlp(const Dims& D, int64_t F, const void* x, const void* W1,
                              const void* W2, void* y, bool accumulate, void* ws, int32_t* status,
                              cudaStream_t s);

// Launch with programmatic stream serialisation (see pdl_wait/pdl_trigger):
// the kernel may be scheduled while its predecessor on the stream finishes.
// Arguments are converted to the kernel's parameter types.
template <typename... KArgs, typename... Args>
cudaError_t launch_k(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                     Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Return the error of a CUDA call from the enclosing launch function.
#define OMNI_TRY(expr)                              \
  do {                                              \
    const cudaError_t omni_try_e_ = (expr);         \
    if (omni_try_e_ != cudaSuccess) return omni_try_e_; \
  } while (0)

// Zero n 32-bit words (a kernel, so that it joins the programmatic chain).
cudaError_t launch_zero(void* p, size_t n_words, cudaStream_t s);

// 256-byte aligned carving of a workspace (base == nullptr: size only)
struct Carver {
  char* base;
  size_t off = 0;
  explicit Carver(void* b) : base(static_cast<char*>(b)) {}
  template <typename T>
  T* take(size_t n) {
    off = (off + 255) & ~size_t(255);
    T* p = base ? reinterpret_cast<T*>(base + off) : nullptr;
    off += n * sizeof(T);
    return p;
  }
};

inline int64_t next_pow2(int64_t v) {
  int64_t p = 1;
  while (p < v) p <<= 1;
  return p;
}

}  // namespace omni
