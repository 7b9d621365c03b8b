// Seeded synthetic inputs, device side: the same definition as gen_host.c,
// producing the same bits (integer hashing, then explicitly rounded IEEE
// multiplies and adds, so no FMA contraction can change a value).
//
// Shared test/bench infrastructure, not part of the layer: it lets large
// weight tensors be created directly in HBM instead of being copied from the
// host. The tests check it bit for bit against the host generator.
#include <cstdint>
#include <cuda_runtime.h>

namespace {

__device__ __forceinline__ uint64_t splitmix64_out(uint64_t z) {
  z += 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

__device__ __forceinline__ uint64_t gen_counter(uint32_t seed, uint32_t tid, uint64_t index) {
  return ((uint64_t)(seed & 0xFF) << 56) | ((uint64_t)(tid & 0xFF) << 48) |
         (index & 0xFFFFFFFFFFFFull);
}

__device__ __forceinline__ uint16_t f32_to_bf16_rne(float f) {
  uint32_t u = __float_as_uint(f);
  if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu)) return (uint16_t)((u >> 16) | 0x40u);
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

__global__ void gen_kernel(uint32_t seed, uint32_t tid, uint32_t kind, uint32_t out_bf16,
                           uint64_t offset, uint64_t n, double a, double b, void* out) {
  uint64_t stride = (uint64_t)gridDim.x * blockDim.x;
  for (uint64_t i = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride) {
    uint64_t h = splitmix64_out(gen_counter(seed, tid, offset + i));
    double v;
    if (kind == 0) {
      int64_t s = (int64_t)(h & 0xFFFF) + (int64_t)((h >> 16) & 0xFFFF) +
                  (int64_t)((h >> 32) & 0xFFFF) + (int64_t)(h >> 48);
      v = __dmul_rn((double)(s - 131070), a);
    } else {
      double u = __dmul_rn((double)(h >> 11), 1.0 / 9007199254740992.0);
      v = __dadd_rn(a, __dmul_rn(__dsub_rn(b, a), u));
    }
    float f = __double2float_rn(v);
    if (out_bf16) ((uint16_t*)out)[i] = f32_to_bf16_rne(f);
    else ((float*)out)[i] = f;
  }
}

int launch(uint32_t seed, uint32_t tid, uint32_t kind, int out_bf16, uint64_t offset, uint64_t n,
           double a, double b, void* out, void* stream) {
  if (n == 0) return 0;
  if (!out) return 1;
  int blocks = (int)((n + 255) / 256);
  if (blocks > 148 * 16) blocks = 148 * 16;
  gen_kernel<<<blocks, 256, 0, (cudaStream_t)stream>>>(seed, tid, kind, (uint32_t)out_bf16, offset,
                                                       n, a, b, out);
  return (int)cudaGetLastError();
}

}  // namespace

extern "C" {

// Approximately normal values (see gen_host.c); returns a cudaError_t value, 0 on success.
int gen_normal_device(uint32_t seed, uint32_t tid, uint64_t offset, uint64_t n, double factor,
                      int out_bf16, void* out, void* stream) {
  return launch(seed, tid, 0, out_bf16, offset, n, factor, 0.0, out, stream);
}

// Uniform values in [lo, hi); returns a cudaError_t value, 0 on success.
int gen_uniform_device(uint32_t seed, uint32_t tid, uint64_t offset, uint64_t n, double lo,
                       double hi, int out_bf16, void* out, void* stream) {
  return launch(seed, tid, 1, out_bf16, offset, n, lo, hi, out, stream);
}

}  // extern "C"
