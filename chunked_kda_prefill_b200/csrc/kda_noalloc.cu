// kda_noalloc.cu -- kda_forward_noalloc: the forward pass for callers that cannot allocate.
//
// Some callers have no way to provide the device workspace kda_forward needs:
// - a plugin interface that hands the library only its input and output tensors;
// - a host runtime that owns every device byte through its own pool and forbids extra
//   cudaMalloc calls (cudaMalloc can also synchronise the device, which some schedulers must
//   avoid).
// For them the library keeps one fixed scratch region per GPU: a file-scope static __device__
// array of KDA_NOALLOC_SCRATCH_BYTES. Every GPU that loads the library holds it until the
// process exits. The entry point calls no cudaMalloc, cudaFree or allocating library routine.
#include <cuda_runtime.h>

#include <mutex>

#include "kda_internal.h"
#include "kda_layout.cuh"

namespace {

// The scratch itself.  In host code this name is only a host-side stand-in for the symbol, not a
// device address; the device address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_kda_noalloc_scratch[KDA_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
void* g_scratch_dev_ptr[kMaxDevices] = {};
std::mutex g_scratch_mu;

// Device address of the scratch on the current device, looked up once per device (with that
// device current) on the first call and cached.
kda_status_t scratch_on_current_device(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return KDA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return KDA_ERR_DEVICE;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_dev_ptr[dev] == nullptr) {
    void* ptr = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&ptr, g_kda_noalloc_scratch);
    if (e != cudaSuccess || ptr == nullptr) return KDA_ERR_CUDA;
    g_scratch_dev_ptr[dev] = ptr;
  }
  *out = g_scratch_dev_ptr[dev];
  return KDA_OK;
}

}  // namespace

using namespace kda;

extern "C" kda_status_t kda_forward_noalloc(const kda_shape_t* shape, const int32_t* plan_host,
                                            const int32_t* plan_dev, size_t n_int32,
                                            const void* q, const void* k, const void* v,
                                            const void* g, const void* beta, float scale,
                                            const float* initial_state, const float* A_log,
                                            const float* dt_bias, float lower_bound, void* out,
                                            float* final_state, kda_stream_t stream) {
  kda_status_t st = validate_shape(shape);
  if (st != KDA_OK) return st;
  if (!plan_host) return KDA_ERR_NULL;
  st = validate_plan(plan_host, n_int32, shape);
  if (st != KDA_OK) return st;
  const size_t need = fused_workspace_bytes(plan_host);
  if (need > (size_t)KDA_NOALLOC_SCRATCH_BYTES) return KDA_ERR_CAPACITY;
  void* scratch = nullptr;
  st = scratch_on_current_device(&scratch);
  if (st != KDA_OK) return st;
  // Exactly kda_forward, with the scratch as its workspace: the device status word at its start
  // is cleared on every call, and under a segmented plan the segment state slots that follow it
  // are written before they are read within the same call.
  return forward_impl(PATH_FUSED, shape, plan_host, plan_dev, n_int32, q, k, v, g, beta, scale,
                      initial_state, A_log, dt_bias, lower_bound, scratch,
                      (size_t)KDA_NOALLOC_SCRATCH_BYTES, out, final_state,
                      reinterpret_cast<cudaStream_t>(stream), nullptr);
}

// The device status word of the last kda_forward_noalloc on the current device: it lives at the
// start of that device's scratch, so this is kda_device_status on the scratch.
extern "C" kda_status_t kda_noalloc_status(kda_stream_t stream) {
  void* scratch = nullptr;
  const kda_status_t st = scratch_on_current_device(&scratch);
  if (st != KDA_OK) return st;
  return kda_device_status(scratch, stream);
}
