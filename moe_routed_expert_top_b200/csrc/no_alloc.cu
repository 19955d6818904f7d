// no_alloc.cu - moe_experts_forward_noalloc: the whole routed-experts forward
// for callers that cannot allocate device memory (a plug-in whose host program
// owns every device allocation, a service with a device-memory budget fixed at
// start-up). The workspace the forward needs lives in a file-scope device
// array inside this library instead of a caller-supplied buffer.
//
// The array's name is only a host-side stand-in in host code: its device
// address comes from cudaGetSymbolAddress, looked up once per device with that
// device current (on the first call there) and cached. The forward itself is
// the unchanged moe_experts_forward, given that address as its workspace.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "moe.h"

namespace {

// Every GPU that loads the library holds this array until the process exits.
static __device__ __align__(256) uint8_t g_noalloc_scratch[MOE_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
void* g_scratch_ptr[kMaxDevices] = {nullptr};
std::mutex g_scratch_mu;

// Device address of g_noalloc_scratch on the current device (nullptr on error).
void* scratch_for_current_device(cudaError_t* err) {
  int dev = -1;
  *err = cudaGetDevice(&dev);
  if (*err != cudaSuccess) return nullptr;
  if (dev < 0 || dev >= kMaxDevices) {
    *err = cudaErrorInvalidDevice;
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    *err = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (*err != cudaSuccess) return nullptr;
    g_scratch_ptr[dev] = p;
  }
  *err = cudaSuccess;
  return g_scratch_ptr[dev];
}

}  // namespace

extern "C" moe_status moe_experts_forward_noalloc(const moe_problem* prob, const void* hidden,
                                                  const int32_t* topk_ids,
                                                  const float* topk_weights,
                                                  const void* w_gate_up, const void* w_down,
                                                  const float* w_down_scales,
                                                  const void* ws_gate_up, const void* ws_down,
                                                  float scale, void* out, moe_stream_t stream) {
  // too large for the built-in scratch area: rejected before anything is enqueued
  const size_t need = moe_workspace_bytes(prob);  // 0 for a problem the forward rejects
  if (need > static_cast<size_t>(MOE_NOALLOC_SCRATCH_BYTES)) return MOE_ERR_WORKSPACE;
  // an invalid problem, or T == 0: moe_experts_forward decides the status
  // (check_problem's error, or MOE_OK with nothing enqueued) without the device
  if (need == 0 || prob->T == 0)
    return moe_experts_forward(prob, hidden, topk_ids, topk_weights, w_gate_up, w_down,
                               w_down_scales, ws_gate_up, ws_down, scale, out, nullptr, 0, stream);
  cudaError_t err = cudaSuccess;
  void* ws = scratch_for_current_device(&err);
  if (ws == nullptr) return MOE_ERR_CUDA;
  // moe_experts_forward zeroes the status word at the array's start itself;
  // every other region is fully rewritten before it is read.
  return moe_experts_forward(prob, hidden, topk_ids, topk_weights, w_gate_up, w_down,
                             w_down_scales, ws_gate_up, ws_down, scale, out, ws,
                             static_cast<size_t>(MOE_NOALLOC_SCRATCH_BYTES), stream);
}

extern "C" moe_status moe_noalloc_read_status(int32_t* host_status, moe_stream_t stream) {
  if (host_status == nullptr) return MOE_ERR_INVALID_ARG;
  cudaError_t err = cudaSuccess;
  void* ws = scratch_for_current_device(&err);
  if (ws == nullptr) return MOE_ERR_CUDA;
  // the status word is the first int32 of the forward's workspace
  err = cudaMemcpyAsync(host_status, ws, sizeof(int32_t), cudaMemcpyDeviceToHost,
                        reinterpret_cast<cudaStream_t>(stream));
  return err == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
