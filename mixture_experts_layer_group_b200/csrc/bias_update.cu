// Auxiliary-loss-free load balancing: the per-batch nudge of the selection
// bias b (grasp.study lesson on DeepSeek-V3's MoE design, section "3.2.
// Auxiliary-Loss-Free Load Balancing"; "The DeepSeekMoE Architecture.",
// configuration table row "balancing: aux-loss-free bias"). After a batch,
// an expert that received more than the mean load T * k / N has its bias
// lowered by gamma, one that received fewer has it raised by gamma, one at
// exactly the mean keeps it. The pages give neither the rate nor the exact
// rule beyond the direction; gamma is the caller's.
#include <cmath>

#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

__global__ void bias_update_kernel(const int32_t* __restrict__ counts, int N, int64_t Tk, float gamma,
                                   float* __restrict__ b) {
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= N) return;
  // compare counts[e] with Tk / N exactly, in integers
  const int64_t over = (int64_t)counts[e] * N - Tk;
  if (over > 0)
    b[e] -= gamma;
  else if (over < 0)
    b[e] += gamma;
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" moe_status moe_bias_update(const moe_cfg* cfg, int64_t T, const int32_t* counts, float gamma,
                                      float* b, void* stream) {
  Problem p;
  moe_status st = make_problem(cfg, T, &p);
  if (st != MOE_OK) return st;
  if (!counts || !b || (reinterpret_cast<uintptr_t>(counts) & 3u) || (reinterpret_cast<uintptr_t>(b) & 3u))
    return MOE_ERR_INVALID_ARG;
  if (!std::isfinite(gamma)) return MOE_ERR_INVALID_ARG;
  const int threads = 256;
  bias_update_kernel<<<(p.N + threads - 1) / threads, threads, 0, static_cast<cudaStream_t>(stream)>>>(
      counts, p.N, p.T * (int64_t)p.k, gamma, b);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    record_cuda_error(e);
    return MOE_ERR_CUDA;
  }
  return MOE_OK;
}
