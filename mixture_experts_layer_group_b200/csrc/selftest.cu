// Self-check of the library's failure path: every wait of the pipelines is
// bounded (mbar_wait_bounded and its cluster variant give up after
// kWaitLimitNs), and a kernel whose wait gave up records MOE_DEV_WAIT_TIMEOUT
// and returns instead of hanging. This entry point makes one such wait run
// out on purpose -- an mbarrier that nothing ever completes -- without any
// fault, trap or unbounded loop.
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

// One status word per device, shared by every call: calls are serialised by
// g_selftest_mu (each call synchronises its stream before it returns), so no
// two calls in this process ever touch the word at the same time.
__device__ unsigned g_selftest_status;
std::mutex g_selftest_mu;

__global__ void wait_timeout_probe(unsigned* status) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);  // one arrival expected; none ever comes
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int no_abort = 0;
    if (!mbar_wait_bounded(&bar, 0, &no_abort)) set_status(status, MOE_DEV_WAIT_TIMEOUT);
  }
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" moe_status moe_selftest_wait_timeout(uint32_t* bits, void* stream) {
  if (!bits) return MOE_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  std::lock_guard<std::mutex> lock(g_selftest_mu);
  void* status = nullptr;
  cudaError_t e = cudaGetSymbolAddress(&status, g_selftest_status);
  if (e == cudaSuccess) e = cudaMemsetAsync(status, 0, sizeof(unsigned), s);
  if (e == cudaSuccess) {
    wait_timeout_probe<<<1, 32, 0, s>>>(static_cast<unsigned*>(status));
    e = cudaGetLastError();
  }
  unsigned host = 0;
  if (e == cudaSuccess) e = cudaMemcpyAsync(&host, status, sizeof(unsigned), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) {
    record_cuda_error(e);
    return MOE_ERR_CUDA;
  }
  *bits = host;
  return MOE_OK;
}
