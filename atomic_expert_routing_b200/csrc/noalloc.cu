// Grouped (expert-centric) execution without a caller-provided workspace.
//
// omni_expert_forward needs an fp32 accumulator of L*d floats (bf16 storage)
// that the caller allocates.  Some callers cannot allocate device memory at
// the point where they run the layer: code that runs while a CUDA graph is
// being captured (cudaMalloc is not allowed there), inference runtimes that
// plan every device buffer ahead of time and forbid allocation in the step,
// and plugin hosts that own all device memory and hand an operator only its
// inputs and outputs.  For them this file holds the accumulator as a
// file-scope device array of a fixed size: every GPU that loads the library
// keeps these bytes until the process exits.
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace {

// fp32 accumulator shared by every call (L * d <= kNoAllocMaxElems)
constexpr size_t kNoAllocMaxElems = size_t(1) << 22;  // 4 Mi floats = 16 MiB
static __device__ __align__(256) float g_noalloc_acc[kNoAllocMaxElems];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
float* g_acc_addr[kMaxDevices] = {};  // device address of g_noalloc_acc, per device

// Device address of the accumulator on the current device, looked up once per
// device (the host-side name of the array is not a device address).  The
// cached address is not refreshed after a cudaDeviceReset of that device.
cudaError_t acc_address(float** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_acc_addr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_acc);
    if (e != cudaSuccess) return e;
    g_acc_addr[dev] = static_cast<float*>(p);
  }
  *out = g_acc_addr[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" int omni_expert_forward_noalloc(const omni_dims* dims, const void* x, const void* W,
                                           const void* V, const int32_t* task_token,
                                           const int32_t* task_expert, const float* task_gate,
                                           const int32_t* uniq, const int32_t* group_off,
                                           int32_t* counts, void* y, void* stream) {
  omni::CallRange range("omni_expert_forward_noalloc");
  if (dims == nullptr) return OMNI_ERR_INVALID_ARG;
  size_t need = 0;
  int rc = omni_workspace_size(dims, OMNI_WS_EXPERT, &need);  // validates dims
  if (rc != OMNI_OK) return rc;
  if (dims->L == 0) return OMNI_OK;
  if (static_cast<size_t>(dims->L) * static_cast<size_t>(dims->d) > kNoAllocMaxElems)
    return OMNI_ERR_UNSUPPORTED;  // batch too large for the fixed scratch
  auto al16 = [](const void* p) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 15) == 0; };
  if (!al16(x) || !al16(W) || !al16(V) || !al16(y) || task_token == nullptr ||
      task_expert == nullptr || task_gate == nullptr || group_off == nullptr || counts == nullptr)
    return OMNI_ERR_INVALID_ARG;
  omni::Dims D;
  D.L = dims->L; D.d = dims->d; D.Nr = dims->Nr; D.Nc = dims->Nc;
  D.k = dims->k; D.K = dims->K; D.B = dims->B; D.dtype = dims->dtype; D.flags = dims->flags;
  // the array holds the accumulator only: the sweep path and the dense-group
  // path need more scratch than that
  if (omni::expert_sweeps(D) > 1) return OMNI_ERR_UNSUPPORTED;
  float* acc = nullptr;
  if (omni::expert_acc_words(D) > 0) {
    const cudaError_t e = acc_address(&acc);
    if (e != cudaSuccess) return omni::cuda_status(e);
  }
  // launch_expert zeroes the accumulator before use (it keeps the previous
  // call's contents otherwise)
  const cudaError_t e = omni::launch_expert(D, x, W, V, task_token, task_expert, task_gate,
                                            uniq, group_off, counts, y, acc,
                                            static_cast<cudaStream_t>(stream), false, false);
  return omni::cuda_status(e);
}
