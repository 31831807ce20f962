// C ABI of the routed atomic-expert layer: argument checks, workspace
// carving and the launch sequence of every entry point (declared and
// documented in include/omnimoe.h).  No call allocates memory, synchronises
// the host or keeps state.
#include <stdint.h>

#include "common.cuh"
#include "internal.h"

using omni::Carver;
using omni::cuda_status;
using omni::Dims;

namespace {
// last failing CUDA call of this host thread (diagnostics only)
thread_local cudaError_t g_last_cuda = cudaSuccess;
}  // namespace

int omni::cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return OMNI_OK;
  g_last_cuda = e;
  return OMNI_ERR_CUDA;
}

namespace {

bool al(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

int check_dims(const omni_dims* in, Dims* D) {
  if (in == nullptr) return OMNI_ERR_INVALID_ARG;
  D->L = in->L; D->d = in->d; D->Nr = in->Nr; D->Nc = in->Nc;
  D->k = in->k; D->K = in->K; D->B = in->B; D->dtype = in->dtype; D->flags = in->flags;
  if (D->L < 0 || D->d < 1 || D->Nr < 1 || D->Nc < 1 || D->k < 1 || D->K < 1 || D->B < 1)
    return OMNI_ERR_INVALID_ARG;
  if (D->dtype != OMNI_F32 && D->dtype != OMNI_BF16) return OMNI_ERR_INVALID_ARG;
  if ((D->flags & ~(OMNI_FLAG_ROUTER_SIMT | OMNI_FLAG_STAGED_SMALL | OMNI_FLAG_DENSE_TENSOR_CORES)) != 0)
    return OMNI_ERR_INVALID_ARG;
  // k*k in 128 bits: k is only bounded by the axes here
  if (D->k > D->Nr || D->k > D->Nc ||
      static_cast<__int128>(D->K) > static_cast<__int128>(D->k) * D->k)
    return OMNI_ERR_INVALID_ARG;
  if (D->Nr > OMNI_MAX_AXIS || D->Nc > OMNI_MAX_AXIS) return OMNI_ERR_UNSUPPORTED;
  if (D->k > OMNI_MAX_TOPK || D->K > OMNI_MAX_TOPK) return OMNI_ERR_UNSUPPORTED;
  // task counts travel in 30-bit fields of the scheduler's look-back words
  // (L is bounded first, so L*K cannot overflow)
  if (D->N() >= (int64_t(1) << 31) || D->L >= (int64_t(1) << 30) ||
      D->M() >= (int64_t(1) << 30))
    return OMNI_ERR_UNSUPPORTED;
  if (D->d % 8 != 0 || D->d > (int64_t(1) << 16)) return OMNI_ERR_UNSUPPORTED;
  return OMNI_OK;
}

// The calls that select experts take the top-K of the k x k candidate pairs.
// That equals the top-K over all N joint scores only when k >= K (a row
// outside the top-k is beaten by at least k >= K others), so they refuse
// K > k.  Scheduling and execution do not use k and take any K <= k*k.
int check_route_dims(const omni_dims* in, Dims* D) {
  const int rc = check_dims(in, D);
  if (rc != OMNI_OK) return rc;
  return D->K > D->k ? OMNI_ERR_UNSUPPORTED : OMNI_OK;
}

// workspace layouts
struct RouteWs {
  float* Z;
};
RouteWs carve_route(const Dims& D, Carver& c) {
  RouteWs w;
  w.Z = c.take<float>(static_cast<size_t>(omni::router_splits(D)) * D.L * (D.Nr + D.Nc));
  return w;
}

struct FusedWs {
  RouteWs route;
  int32_t *idx, *task_token, *task_expert, *uniq, *group_off;
  float *gate, *task_gate;
  int64_t* shard_range;  // [2]: the task range a sharded execution visits
  void* sched;
  void* expert;
};
// A large bf16/fp32 batch on the sweep path: the fused forward goes from the
// routing straight to the window order of the sweeps.
bool fused_windows(const Dims& D) {
  return omni::expert_sweeps(D) > 1 && omni::windows_supported(D);
}

FusedWs carve_fused(const Dims& D, Carver& c) {
  FusedWs w;
  w.route = carve_route(D, c);
  const size_t M = static_cast<size_t>(D.M());
  w.idx = c.take<int32_t>(M);
  w.gate = c.take<float>(M);
  w.task_token = c.take<int32_t>(M);
  w.task_expert = c.take<int32_t>(M);
  w.task_gate = c.take<float>(M);
  w.uniq = c.take<int32_t>(static_cast<size_t>(D.ucap() > 0 ? D.ucap() : 1));
  w.group_off = c.take<int32_t>(static_cast<size_t>(D.gmax()) + 1);
  w.sched = c.take<char>(fused_windows(D) ? omni::windows_ws_bytes(D)
                                           : omni::schedule_ws_bytes(D));
  // the routing-order tail (activations per task, value gather) uses the
  // expert workspace for its counters and activations
  const size_t tail = omni::sched_exec_supported(D) ? omni::sched_exec_ws_words(D) * 4 : 0;
  const size_t ex = omni::expert_ws_bytes(D);
  w.expert = c.take<char>(ex > tail ? ex : tail);
  w.shard_range = c.take<int64_t>(2);
  return w;
}

size_t ws_size(const Dims& D, int which) {
  Carver c(nullptr);
  switch (which) {
    case OMNI_WS_ROUTE: carve_route(D, c); break;
    case OMNI_WS_SCHEDULE: c.take<char>(omni::schedule_ws_bytes(D)); break;
    case OMNI_WS_EXPERT: c.take<char>(omni::expert_ws_bytes(D)); break;
    case OMNI_WS_FUSED: carve_fused(D, c); break;
    case OMNI_WS_BACKWARD: {
      size_t b = 0;
      omni::carve_backward(D, nullptr, &b);
      c.take<char>(b);
      break;
    }
    default: break;
  }
  return c.off;
}

int ws_ok(const Dims& D, int which, const void* ws, size_t ws_bytes) {
  const size_t need = ws_size(D, which);
  if (need == 0) return OMNI_OK;
  if (ws == nullptr || !al(ws, 256) || ws_bytes < need) return OMNI_ERR_WORKSPACE;
  return OMNI_OK;
}


int route_impl(const Dims& D, const void* x, const void* Wr, const void* Wc, const float* br,
               const float* bc, int32_t* idx, float* gate, float* score, int32_t* status,
               float* Z, cudaStream_t s, float* zero = nullptr, int64_t zero_words = 0,
               bool* zeroed = nullptr) {
  cudaError_t e;
  int parts = 1;
  if (omni::router_tc_supported(D, x, Wr, Wc)) {
    e = omni::launch_router_tc(D, x, Wr, Wc, Z, status, s);
    parts = omni::router_splits(D);
  } else {
    e = omni::launch_router_simt(D, x, Wr, Wc, Z, s);
  }
  if (e != cudaSuccess) return cuda_status(e);
  return cuda_status(
      omni::launch_select(D, Z, parts, br, bc, idx, gate, score, s, zero, zero_words, zeroed));
}

// Diagnostic: one thread waits on a shared-memory barrier that expects one
// arrival nobody makes.  The library's bounded wait gives up, ORs
// OMNI_DEV_TIMEOUT into *status and the kernel returns.
__global__ void k_wait_selftest(int32_t* status) {
  __shared__ __align__(8) uint64_t bar;
  omni::pdl_wait();  // the caller's writes to *status come first
  if (threadIdx.x != 0) return;
  const uint32_t b = omni::smem_u32(&bar);
  omni::mbar_init(b, 1);
  omni::mbar_wait(b, 0, status);
}

bool tensors_ok(const void* const* p16, int n16) {
  for (int i = 0; i < n16; ++i)
    if (p16[i] == nullptr || !al(p16[i], 16)) return false;
  return true;
}

// The staged grouped execution, plain or gated (then U is checked like the
// other tensors).
int expert_forward_impl(const omni_dims* dims, bool gated, const void* x, const void* W,
                        const void* U, const void* V, const int32_t* task_token,
                        const int32_t* task_expert, const float* task_gate, const int32_t* uniq,
                        const int32_t* group_off, int32_t* counts, void* y, void* ws,
                        size_t ws_bytes, void* stream) {
  Dims D;
  int rc = check_dims(dims, &D);
  if (rc != OMNI_OK) return rc;
  if (D.L == 0) return OMNI_OK;
  const void* t16[] = {x, W, V, y, gated ? U : x};
  if (!tensors_ok(t16, 5) || task_token == nullptr || task_expert == nullptr ||
      task_gate == nullptr || group_off == nullptr || counts == nullptr)
    return OMNI_ERR_INVALID_ARG;
  if ((rc = ws_ok(D, OMNI_WS_EXPERT, ws, ws_bytes)) != OMNI_OK) return rc;
  return cuda_status(omni::launch_expert(D, x, W, V, task_token, task_expert, task_gate, uniq,
                                         group_off, counts, y, ws,
                                         static_cast<cudaStream_t>(stream), false, true,
                                         gated ? U : nullptr));
}

// The token-centric ablation, plain or gated.
int token_forward_impl(const omni_dims* dims, bool gated, const void* x, const void* W,
                       const void* U, const void* V, const int32_t* idx, const float* gate,
                       void* y, int32_t* counts, void* stream) {
  Dims D;
  int rc = check_dims(dims, &D);
  if (rc != OMNI_OK) return rc;
  if (D.L == 0) return OMNI_OK;
  const void* t16[] = {x, W, V, y, gated ? U : x};
  if (!tensors_ok(t16, 5) || idx == nullptr || gate == nullptr) return OMNI_ERR_INVALID_ARG;
  return cuda_status(omni::launch_token(D, x, W, V, idx, gate, y, counts ? counts + 2 : nullptr,
                                        static_cast<cudaStream_t>(stream),
                                        gated ? U : nullptr));
}

}  // namespace

extern "C" {

int omni_abi_version(void) { return OMNI_ABI_VERSION; }

int omni_wait_selftest(int32_t* counts, void* stream) {
  omni::CallRange range("omni_wait_selftest");
  if (counts == nullptr || !al(counts, 4)) return OMNI_ERR_INVALID_ARG;
  return cuda_status(omni::launch_k(k_wait_selftest, 1, 32, 0,
                                    static_cast<cudaStream_t>(stream), counts + 2));
}

const char* omni_last_cuda_error_name(void) { return cudaGetErrorName(g_last_cuda); }

const char* omni_status_string(int status) {
  switch (status) {
    case OMNI_OK: return "ok";
    case OMNI_ERR_INVALID_ARG: return "invalid argument";
    case OMNI_ERR_UNSUPPORTED: return "unsupported by this build";
    case OMNI_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case OMNI_ERR_CUDA: return "CUDA call failed";
    default: return "unknown status";
  }
}

int omni_workspace_size(const omni_dims* dims, int which, size_t* bytes) {
  Dims D;
  int rc = check_dims(dims, &D);
  if (rc != OMNI_OK) return rc;
  if (bytes == nullptr || which < OMNI_WS_ROUTE || which > OMNI_WS_BACKWARD) return OMNI_ERR_INVALID_ARG;
  *bytes = ws_size(D, which);
  return OMNI_OK;
}

int omni_route(const omni_dims* dims, const void* x, const void* Wr, const void* Wc,
               const float* bias_r, const float* bias_c, int32_t* idx, float* gate, float* score,
               int32_t* counts, void* ws, size_t ws_bytes, void* stream) {
  omni::CallRange range("omni_route");
  Dims D;
  int rc = check_route_dims(dims, &D);
  if (rc != OMNI_OK) return rc;
  if (D.L == 0) return OMNI_OK;
  const void* t16[] = {x, Wr, Wc};
  if (!tensors_ok(t16, 3) || idx == nullptr || gate == nullptr) return OMNI_ERR_INVALID_ARG;
  if ((rc = ws_ok(D, OMNI_WS_ROUTE, ws, ws_bytes)) != OMNI_OK) return rc;
  Carver c(ws);
  RouteWs w = carve_route(D, c);
  return route_impl(D, x, Wr, Wc, bias_r, bias_c, idx, gate, score,
                    counts ? counts + 2 : nullptr, w.Z, static_cast<cudaStream_t>(stream));
}

int omni_router_logits(const omni_dims* dims, const void* x, const void* Wr, const void* Wc,
                       float* logits, int32_t* counts, void* ws, size_t ws_bytes, void* stream) {
  omni::CallRange range("omni_router_logits");
  Dims D;
  int rc = check_dims(dims, &D);
  if (rc != OMNI_OK) return rc;
  if (D.L == 0) return OMNI_OK;
  const void* t16[] = {x, Wr, Wc, logits};
  if (!tensors_ok(t16, 4)) return OMNI_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (!omni::router_tc_supported(D, x, Wr, Wc))
    return cuda_status(omni::launch_router_simt(D, x, Wr, Wc, logits, s));
  const int parts = omni::router_splits(D);
  if (parts > 1 && (ws == nullptr || !al(ws, 256) ||
                    ws_bytes < static_cast<size_t>(parts) * D.L * (D.Nr + D.Nc) * sizeof(float)))
    return OMNI_ERR_WORKSPACE;
  float* Z = parts > 1 ? static_cast<float*>(ws) : logits;
  cudaError_t e = omni::launch_router_tc(D, x, Wr, Wc, Z, counts ? counts + 2 : nullptr, s);
  if (e == cudaSuccess && parts > 1) {
    e = omni::launch_sum_partials(Z, parts, D.L * (D.Nr + D.Nc), s);
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(logits, Z, static_cast<size_t>(D.L) * (D.Nr + D.Nc) * sizeof(float),
                          cudaMemcpyDeviceToDevice, s);
  }
  return cuda_status(e);
}

int omni_route_select(const omni_dims* dims, const float* logits, const float* bias_r,
                      const float* bias_c, int32_t* idx, float* gate, float* score,
                      int32_t* counts, void* ws, size_t ws_bytes, void* stream) {
  omni::CallRange range("omni_route_select");
  (void)counts;
  (void)ws;
  (void)ws_bytes;
  Dims D;
  int rc = check_route_dims(dims, &D);
  if (rc != OMNI_OK) return rc;
  if (D.L == 0) return OMNI_OK;
  if (logits == nullptr || !al(logits, 16) || idx == nullptr || gate == nullptr)
    return OMNI_ERR_INVALID_ARG;
  return cuda_status(omni::launch_select(D, logits, 1, bias_r, bias_c, idx, gate, score,
                                         static_cast<cudaStream_t>(stream)));
}

int omni_schedule(const omni_dims* dims, const int32_t* idx, const float* gate,
                  int32_t* task_token, int32_t* task_expert, float* task_gate, int32_t* uniq,
                  int32_t* group_off, int32_t* counts, void* ws, size_t ws_bytes, void* stream) {
  omni::CallRange range("omni_schedule");
  Dims D;
  int rc = check_dims(dims, &D);
  if (rc != OMNI_OK) return rc;
  if (counts == nullptr || group_off == nullptr) return OMNI_ERR_INVALID_ARG;
  if (D.L > 0 && (idx == nullptr || gate == nullptr || task_token == nullptr ||
                  task_expert == nullptr || task_gate == nullptr || uniq == nullptr))
    return OMNI_ERR_INVALID_ARG;
  if ((rc = ws_ok(D, OMNI_WS_SCHEDULE, ws, ws_bytes)) != OMNI_OK) return rc;
  return cuda_status(omni::launch_schedule(D, idx, gate, task_token, task_expert, task_gate, uniq,
                                           group_off, counts, ws,
                                           static_cast<cudaStream_t>(stream)));
}

int omni_expert_forward(const omni_dims* dims, const void* x, const void* W, const void* V,
                        const int32_t* task_token, const int32_t* task_expert,
                        const float* task_gate, const int32_t* uniq, const int32_t* group_off,
                        int32_t* counts, void* y, void* ws, size_t ws_bytes, void* stream) {
  omni::CallRange range("omni_expert_forward");
  return expert_forward_impl(dims, false, x, W, nullptr, V, task_token, task_expert, task_gate, uniq,
                             group_off, counts, y, ws, ws_bytes, stream);
}

int omni_expert_forward_glu(const omni_dims* dims, const void* x, const void* W, const void* U,
                            const void* V, const int32_t* task_token, const int32_t* task_expert,
                            const float* task_gate, const int32_t* uniq, const int32_t* group_off,
                            int32_t* counts, void* y, void* ws, size_t ws_bytes, void* stream) {
  omni::CallRange range("omni_expert_forward_glu");
  return expert_forward_impl(dims, true, x, W, U, V, task_token, task_expert, task_gate, uniq,
                             group_off, counts, y, ws, ws_bytes, stream);
}

}  // extern "C"

namespace {

// The fused routed branch; dims, pointers and workspace already checked.
// routed: idx_out / gate_out hold the batch's routing already (the route is
// skipped and they are only read).
int moe_forward_impl(const Dims& D, const void* x, const void* Wr, const void* Wc,
                     const float* bias_r, const float* bias_c, const void* W, const void* V,
                     void* y, int32_t* idx_out, float* gate_out, int32_t* counts, void* ws,
                     cudaStream_t s, const void* U = nullptr, bool routed = false) {
  int rc = OMNI_OK;
  Carver c(ws);
  FusedWs w = carve_fused(D, c);
  int32_t* idx = idx_out ? idx_out : w.idx;
  float* gate = gate_out ? gate_out : w.gate;
  // a batch without sweeps accumulates into a buffer the selection can clear
  // while the router runs (y itself for fp32, else the expert workspace)
  const int64_t acc_words = omni::expert_acc_words(D);
  float* acc = acc_words == 0 ? nullptr
               : static_cast<float*>(D.dtype == OMNI_F32 || D.sharded() ? y : w.expert);
  // a batch whose rows fit in L2 runs the two-kernel tail; its counters and id bitmap are
  // cleared by the selection kernel in place of the accumulator
  const bool tail = omni::sched_exec_supported(D);
  float* zero = tail ? static_cast<float*>(w.expert) : acc;
  const int64_t zero_words =
      tail ? static_cast<int64_t>(omni::sched_exec_zero_words(D)) : acc_words;
  bool acc_zeroed = false;
  if (!routed) {
    omni::CallRange stage("route");
    rc = route_impl(D, x, Wr, Wc, bias_r, bias_c, idx, gate, nullptr, counts + 2, w.route.Z, s,
                    zero, zero_words, &acc_zeroed);
  }
  if (rc != OMNI_OK) return rc;
  if (tail) {
    omni::CallRange stage("schedule+expert");
    if (!acc_zeroed &&
        (rc = cuda_status(omni::launch_zero(zero, static_cast<size_t>(zero_words), s))) != OMNI_OK)
      return rc;
    return cuda_status(omni::launch_sched_exec(D, x, W, V, idx, gate, y,
                                               static_cast<uint32_t*>(w.expert), counts, s, U));
  }
  if (fused_windows(D)) {
    {
      omni::CallRange stage("schedule");
      rc = cuda_status(omni::launch_schedule_windows(D, idx, gate, w.uniq, w.group_off, counts,
                                                     w.sched, omni::expert_windows(D, w.expert),
                                                     s));
    }
    if (rc != OMNI_OK) return rc;
    omni::CallRange stage("expert");
    Dims De = D;
    if (D.sharded()) {
      if ((rc = cuda_status(omni::launch_shard_range(D, w.uniq, w.group_off, counts,
                                                     omni::window_tasks(D), w.shard_range, s))) !=
          OMNI_OK)
        return rc;
      De.shard_range = w.shard_range;
    }
    if ((rc = cuda_status(omni::launch_expert_windows(De, x, W, V, counts, y, w.expert, s, U))) !=
        OMNI_OK)
      return rc;
    return D.sharded() ? cuda_status(omni::launch_shard_counts(D, w.uniq, counts, s)) : OMNI_OK;
  }
  {
    omni::CallRange stage("schedule");
    rc = cuda_status(omni::launch_schedule(D, idx, gate, w.task_token, w.task_expert, w.task_gate,
                                           w.uniq, w.group_off, counts, w.sched, s));
  }
  if (rc != OMNI_OK) return rc;
  omni::CallRange stage("expert");
  Dims De = D;
  if (D.sharded()) {
    // the sweeps (if any) visit whole windows of the schedule's order
    const int64_t T = omni::expert_sweeps(D) > 1 ? omni::window_tasks(D) : 0;
    if ((rc = cuda_status(omni::launch_shard_range(D, w.uniq, w.group_off, counts, T,
                                                   w.shard_range, s))) != OMNI_OK)
      return rc;
    De.shard_range = w.shard_range;
  }
  if ((rc = cuda_status(omni::launch_expert(De, x, W, V, w.task_token, w.task_expert,
                                            w.task_gate, w.uniq, w.group_off, counts, y, w.expert,
                                            s, acc_zeroed, true, U))) != OMNI_OK)
    return rc;
  return D.sharded() ? cuda_status(omni::launch_shard_counts(D, w.uniq, counts, s)) : OMNI_OK;
}

// The checks of the shared MLP's width: F >= 1; a multiple of 8 (16-byte
// rows of H and W2) and at most 65536, else unsupported; bf16 storage only.
int check_mlp(const Dims& D, int64_t F) {
  if (F < 1) return OMNI_ERR_INVALID_ARG;
  if (F % 8 != 0 || F > 65536 || D.dtype != OMNI_BF16) return OMNI_ERR_UNSUPPORTED;
  return OMNI_OK;
}

}  // namespace

extern "C" {

int omni_moe_forward(const omni_dims* dims, const void* x, const void* Wr, const void* Wc,
                     const float* bias_r, const float* bias_c, const void* W, const void* V,
                     void* y, int32_t* idx_out, float* gate_out, int32_t* counts, void* ws,
                     size_t ws_bytes, void* stream) {
  omni::CallRange range("omni_moe_forward");
  Dims D;
  int rc = check_route_dims(dims, &D);
  if (rc != OMNI_OK) return rc;
  if (counts == nullptr) return OMNI_ERR_INVALID_ARG;
  if (D.L == 0) return OMNI_OK;
  const void* t16[] = {x, Wr, Wc, W, V, y};
  if (!tensors_ok(t16, 6)) return OMNI_ERR_INVALID_ARG;
  if ((rc = ws_ok(D, OMNI_WS_FUSED, ws, ws_bytes)) != OMNI_OK) return rc;
  return moe_forward_impl(D, x, Wr, Wc, bias_r, bias_c, W, V, y, idx_out, gate_out, counts, ws,
                          static_cast<cudaStream_t>(stream));
}

int omni_mlp_workspace_size(const omni_dims* dims, int64_t F, int with_routed, size_t* bytes) {
  Dims D;
  int rc = with_routed ? check_route_dims(dims, &D) : check_dims(dims, &D);
  if (rc != OMNI_OK) return rc;
  if ((rc = check_mlp(D, F)) != OMNI_OK) return rc;
  if (bytes == nullptr) return OMNI_ERR_INVALID_ARG;
  Carver c(nullptr);
  if (with_routed) c.take<char>(ws_size(D, OMNI_WS_FUSED));
  c.take<char>(omni::mlp_ws_bytes(D, F));
  *bytes = c.off;
  return OMNI_OK;
}

int omni_shared_mlp(const omni_dims* dims, int64_t F, const void* x, const void* W1,
                    const void* W2, void* y, int accumulate, int32_t* counts, void* ws,
                    size_t ws_bytes, void* stream) {
  omni::CallRange range("omni_shared_mlp");
  Dims D;
  int rc = check_dims(dims, &D);
  if (rc != OMNI_OK) return rc;
  if ((rc = check_mlp(D, F)) != OMNI_OK) return rc;
  if (D.L == 0) return OMNI_OK;
  const void* t16[] = {x, W1, W2, y};
  if (!tensors_ok(t16, 4)) return OMNI_ERR_INVALID_ARG;
  if (ws == nullptr || !al(ws, 256) || ws_bytes < omni::mlp_ws_bytes(D, F))
    return OMNI_ERR_WORKSPACE;
  return cuda_status(omni::launch_shared_mlp(D, F, x, W1, W2, y, accumulate != 0, ws,
                                             counts ? counts + 2 : nullptr,
                                             static_cast<cudaStream_t>(stream)));
}

int omni_moe_mlp_forward(const omni_dims* dims, int64_t F, const void* x, const void* Wr,
                         const void* Wc, const float* bias_r, const float* bias_c, const void* W,
                         const void* V, const void* W1, const void* W2, void* y,
                         int32_t* idx_out, float* gate_out, int32_t* counts, void* ws,
                         size_t ws_bytes, void* stream) {
  omni::CallRange range("omni_moe_mlp_forward");
  Dims D;
  int rc = check_route_dims(dims, &D);
  if (rc != OMNI_OK) return rc;
  if ((rc = check_mlp(D, F)) != OMNI_OK) return rc;
  if (counts == nullptr) return OMNI_ERR_INVALID_ARG;
  if (D.L == 0) return OMNI_OK;
  const void* t16[] = {x, Wr, Wc, W, V, W1, W2, y};
  if (!tensors_ok(t16, 8)) return OMNI_ERR_INVALID_ARG;
  size_t need = 0;
  omni_mlp_workspace_size(dims, F, 1, &need);
  if (ws == nullptr || !al(ws, 256) || ws_bytes < need) return OMNI_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  Carver c(ws);
  void* ws_routed = c.take<char>(ws_size(D, OMNI_WS_FUSED));
  void* ws_mlp = c.take<char>(omni::mlp_ws_bytes(D, F));
  if ((rc = moe_forward_impl(D, x, Wr, Wc, bias_r, bias_c, W, V, y, idx_out, gate_out, counts,
                             ws_routed, s)) != OMNI_OK)
    return rc;
  omni::CallRange stage("shared_mlp");
  return cuda_status(omni::launch_shared_mlp(D, F, x, W1, W2, y, true, ws_mlp, counts + 2, s));
}

int omni_token_centric_forward(const omni_dims* dims, const void* x, const void* W,
                               const void* V, const int32_t* idx, const float* gate, void* y,
                               int32_t* counts, void* ws, size_t ws_bytes, void* stream) {
  omni::CallRange range("omni_token_centric_forward");
  (void)ws;
  (void)ws_bytes;
  return token_forward_impl(dims, false, x, W, nullptr, V, idx, gate, y, counts, stream);
}

int omni_token_centric_forward_glu(const omni_dims* dims, const void* x, const void* W,
                                   const void* U, const void* V, const int32_t* idx,
                                   const float* gate, void* y, int32_t* counts, void* ws,
                                   size_t ws_bytes, void* stream) {
  omni::CallRange range("omni_token_centric_forward_glu");
  (void)ws;
  (void)ws_bytes;
  return token_forward_impl(dims, true, x, W, U, V, idx, gate, y, counts, stream);
}

int omni_moe_forward_glu(const omni_dims* dims, const void* x, const void* Wr, const void* Wc,
                         const float* bias_r, const float* bias_c, const void* W, const void* U,
                         const void* V, void* y, int32_t* idx_out, float* gate_out,
                         int32_t* counts, void* ws, size_t ws_bytes, void* stream) {
  omni::CallRange range("omni_moe_forward_glu");
  Dims D;
  int rc = check_route_dims(dims, &D);
  if (rc != OMNI_OK) return rc;
  if (counts == nullptr) return OMNI_ERR_INVALID_ARG;
  if (D.L == 0) return OMNI_OK;
  const void* t16[] = {x, Wr, Wc, W, U, V, y};
  if (!tensors_ok(t16, 7)) return OMNI_ERR_INVALID_ARG;
  if ((rc = ws_ok(D, OMNI_WS_FUSED, ws, ws_bytes)) != OMNI_OK) return rc;
  return moe_forward_impl(D, x, Wr, Wc, bias_r, bias_c, W, V, y, idx_out, gate_out, counts, ws,
                          static_cast<cudaStream_t>(stream), U);
}

int omni_moe_forward_shard(const omni_dims* dims, int64_t e_lo, int64_t e_hi, const void* x,
                           const void* Wr, const void* Wc, const float* bias_r,
                           const float* bias_c, const void* W, const void* U, const void* V,
                           float* y_part, int32_t* idx_out, float* gate_out, int32_t* counts,
                           void* ws, size_t ws_bytes, void* stream) {
  omni::CallRange range("omni_moe_forward_shard");
  Dims D;
  int rc = check_route_dims(dims, &D);
  if (rc != OMNI_OK) return rc;
  if (e_lo < 0 || e_hi <= e_lo || e_hi > D.N() || counts == nullptr) return OMNI_ERR_INVALID_ARG;
  if (D.L == 0) return OMNI_OK;
  const void* t16[] = {x, Wr, Wc, W, V, y_part, U != nullptr ? U : x};
  if (!tensors_ok(t16, 7)) return OMNI_ERR_INVALID_ARG;
  if ((rc = ws_ok(D, OMNI_WS_FUSED, ws, ws_bytes)) != OMNI_OK) return rc;
  D.e_lo = e_lo;
  D.e_hi = e_hi;
  return moe_forward_impl(D, x, Wr, Wc, bias_r, bias_c, W, V, y_part, idx_out, gate_out, counts,
                          ws, static_cast<cudaStream_t>(stream), U);
}

int omni_cast_output(const omni_dims* dims, const float* src, void* y, void* stream) {
  omni::CallRange range("omni_cast_output");
  Dims D;
  int rc = check_dims(dims, &D);
  if (rc != OMNI_OK) return rc;
  if (D.L == 0) return OMNI_OK;
  const void* t16[] = {src, y};
  if (!tensors_ok(t16, 2)) return OMNI_ERR_INVALID_ARG;
  if (D.dtype == OMNI_BF16 && static_cast<const void*>(src) == y) return OMNI_ERR_INVALID_ARG;
  return cuda_status(omni::launch_cast_output(D, src, y, static_cast<cudaStream_t>(stream)));
}

int omni_moe_backward(const omni_dims* dims, const void* x, const void* Wr, const void* Wc,
                      const void* W, const void* V, const int32_t* idx, const float* gate,
                      const void* dy, float* dx, float* dW, float* dV, float* dWr, float* dWc,
                      float* dbias_r, float* dbias_c, int accumulate, int32_t* counts, void* ws,
                      size_t ws_bytes, void* stream) {
  omni::CallRange range("omni_moe_backward");
  Dims D;
  int rc = check_dims(dims, &D);
  if (rc != OMNI_OK) return rc;
  if (D.dtype != OMNI_BF16) return OMNI_ERR_UNSUPPORTED;
  if (D.L == 0) return OMNI_OK;
  const void* t16[] = {x, Wr, Wc, W, V, dy, dx, dW, dV, dWr, dWc};
  if (!tensors_ok(t16, 11) || idx == nullptr || gate == nullptr || counts == nullptr ||
      !al(dbias_r, 4) || !al(dbias_c, 4))
    return OMNI_ERR_INVALID_ARG;
  if ((rc = ws_ok(D, OMNI_WS_BACKWARD, ws, ws_bytes)) != OMNI_OK) return rc;
  return cuda_status(omni::launch_backward(D, x, Wr, Wc, W, V, idx, gate, dy, dx, dW, dV, dWr,
                                           dWc, dbias_r, dbias_c, accumulate != 0, counts, ws,
                                           static_cast<cudaStream_t>(stream)));
}

int omni_moe_forward_shard_routed(const omni_dims* dims, int64_t e_lo, int64_t e_hi,
                                  const void* x, const void* W, const void* U, const void* V,
                                  const int32_t* idx, const float* gate, float* y_part,
                                  int32_t* counts, void* ws, size_t ws_bytes, void* stream) {
  omni::CallRange range("omni_moe_forward_shard_routed");
  Dims D;
  int rc = check_dims(dims, &D);
  if (rc != OMNI_OK) return rc;
  if (e_lo < 0 || e_hi <= e_lo || e_hi > D.N() || counts == nullptr) return OMNI_ERR_INVALID_ARG;
  if (D.L == 0) return OMNI_OK;
  const void* t16[] = {x, W, V, y_part, U != nullptr ? U : x};
  if (!tensors_ok(t16, 5) || idx == nullptr || gate == nullptr) return OMNI_ERR_INVALID_ARG;
  if ((rc = ws_ok(D, OMNI_WS_FUSED, ws, ws_bytes)) != OMNI_OK) return rc;
  D.e_lo = e_lo;
  D.e_hi = e_hi;
  return moe_forward_impl(D, x, nullptr, nullptr, nullptr, nullptr, W, V, y_part,
                          const_cast<int32_t*>(idx), const_cast<float*>(gate), counts, ws,
                          static_cast<cudaStream_t>(stream), U, true);
}

}  // extern "C"
