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

// Size of the fixed scratch array. A call needs T * n_routed * 4 bytes of it
// at least (one plane of fp32 logits for every token); a call that needs
// more planes than fit (moe_route splits the reduction over d into S ranges,
// one plane each) runs the router over slices of the tokens in turn, each
// slice with the same S, so the logits are bitwise those of moe_route.
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
  // moe_route's split count for the whole batch, and the largest token slice
  // whose S planes fit the array (a multiple of 64 tokens, the router's tile
  // height; at least 256 tokens since S <= 16 and n_routed <= 512)
  const int S = router_k_splits(p);
  int64_t slice = (int64_t)(kNoallocScratchBytes / ((size_t)S * (size_t)p.N * sizeof(float)));
  if (slice < T) slice = slice / 64 * 64;
  if (slice < 1) return MOE_ERR_UNSUPPORTED;
  void* scratch = nullptr;
  cudaError_t e = scratch_address(&scratch);
  const uint8_t* xb = static_cast<const uint8_t*>(x);
  for (int64_t t0 = 0; e == cudaSuccess && t0 < T; t0 += slice) {
    Problem ps = p;  // the same layer on tokens [t0, t0 + slice)
    ps.T = T - t0 < slice ? T - t0 : slice;
    ps.R = ps.T * p.k;
    e = launch_router(ps, xb + t0 * (int64_t)p.d * p.elem, W_r, b, static_cast<float*>(scratch),
                      kNoallocScratchBytes, topk_idx + t0 * p.k, gates + t0 * p.k, nullptr,
                      static_cast<cudaStream_t>(stream), S);
  }
  if (e != cudaSuccess) {
    record_cuda_error(e);
    return MOE_ERR_CUDA;
  }
  return MOE_OK;
}
