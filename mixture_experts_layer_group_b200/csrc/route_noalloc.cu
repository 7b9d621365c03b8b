// moe_route_noalloc: the router for callers that cannot hand the library
// any device memory of its own to use as scratch.
//
// Some callers cannot allocate: a plugin whose host framework owns all
// device memory and gives the plugin no workspace, or a serving loop with a
// fixed memory budget that must not call cudaMalloc (which can synchronise
// the device) once it is running. For them the router's only scratch -- the
// fp32 logits, T x n_routed values -- lives in a fixed array in this file,
// reserved on every GPU that loads the library until the process exits.
// The caller still passes the inputs and the outputs.
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

// Largest scratch a call may use: the router's fp32 logits, T * n_routed * 4
// bytes (the router splits its reduction only as far as the array allows).
constexpr size_t kNoallocScratchBytes = size_t(8) << 20;  // 8 MiB

__device__ __align__(256) unsigned char g_route_scratch[kNoallocScratchBytes];

std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of g_route_scratch on the current device, looked up once
// per device with that device current. In host code the symbol itself is
// only a host-side stand-in and must never be handed to a kernel.
cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_route_scratch);
    if (e != cudaSuccess) return e;
    if (!p) return cudaErrorInvalidSymbol;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return cudaSuccess;
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" moe_status moe_route_noalloc(const moe_cfg* cfg, int64_t T, const void* x,
                                        const void* W_r, const float* b, int32_t* topk_idx,
                                        float* gates, void* stream) {
  Problem p;
  moe_status st = make_problem(cfg, T, &p);
  if (st != MOE_OK) return st;
  if (T == 0) return MOE_OK;
  if (!x || !W_r || !topk_idx || !gates) return MOE_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(x) & 15u) || (reinterpret_cast<uintptr_t>(W_r) & 15u))
    return MOE_ERR_INVALID_ARG;
  if ((size_t)T * (size_t)p.N * sizeof(float) > kNoallocScratchBytes) return MOE_ERR_UNSUPPORTED;
  void* scratch = nullptr;
  cudaError_t e = scratch_address(&scratch);
  if (e == cudaSuccess)
    e = launch_router(p, x, W_r, b, static_cast<float*>(scratch), kNoallocScratchBytes, topk_idx, gates,
                      nullptr, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) {
    record_cuda_error(e);
    return MOE_ERR_CUDA;
  }
  return MOE_OK;
}
