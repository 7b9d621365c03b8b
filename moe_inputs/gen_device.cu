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

// FP8 (e4m3) weights with one power-of-two scale per 128 x 128 block: the
// definition of gen_fp8 in gen_host.c, with the same integer hashing and
// exactly rounded fp64 steps (rint ties to even, exact power-of-two scaling).
__device__ __forceinline__ uint8_t e4m3_rne(double x) {
  const uint8_t sign = (x < 0.0) ? 0x80 : 0x00;
  const double a = fabs(x);
  if (a >= 464.0) return (uint8_t)(sign | 0x7E);
  if (a < 0.015625) {
    const int m = (int)rint(__dmul_rn(a, 512.0));
    return (uint8_t)(sign | m);
  }
  int e;
  const double f = frexp(a, &e);
  e -= 1;
  int mant = (int)rint(__dmul_rn(__dsub_rn(ldexp(f, 1), 1.0), 8.0));
  if (mant == 8) { mant = 0; e += 1; }
  if (e > 8 || (e == 8 && mant > 6)) return (uint8_t)(sign | 0x7E);
  return (uint8_t)(sign | ((e + 7) << 3) | mant);
}

__global__ void gen_fp8_kernel(uint32_t seed, uint32_t tid, uint32_t tid_scale, int e0, uint64_t cols,
                               uint64_t offset, uint64_t n, double factor, uint8_t* out) {
  const uint64_t stride = (uint64_t)gridDim.x * blockDim.x;
  const uint64_t bcols = cols / 128;
  for (uint64_t i = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride) {
    const uint64_t g = offset + i, r = g / cols, c = g % cols;
    const int e = e0 + (int)(splitmix64_out(gen_counter(seed, tid_scale, (r / 128) * bcols + c / 128)) & 3u);
    const uint64_t h = splitmix64_out(gen_counter(seed, tid, g));
    const int64_t s = (int64_t)(h & 0xFFFF) + (int64_t)((h >> 16) & 0xFFFF) + (int64_t)((h >> 32) & 0xFFFF) +
                      (int64_t)(h >> 48);
    const double v = __dmul_rn((double)(s - 131070), factor);
    out[i] = e4m3_rne(ldexp(v, -e));
  }
}

__global__ void gen_fp8_scales_kernel(uint32_t seed, uint32_t tid_scale, int e0, uint64_t offset, uint64_t n,
                                      uint8_t* out) {
  const uint64_t stride = (uint64_t)gridDim.x * blockDim.x;
  for (uint64_t i = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride)
    out[i] = (uint8_t)(e0 + (int)(splitmix64_out(gen_counter(seed, tid_scale, offset + i)) & 3u) + 127);
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

// e4m3 codes of elements [offset, offset + n) of a [rows, cols] matrix (see gen_host.c).
int gen_fp8_device(uint32_t seed, uint32_t tid, uint32_t tid_scale, int e0, uint64_t cols, uint64_t offset,
                   uint64_t n, double factor, void* out, void* stream) {
  if (n == 0) return 0;
  if (!out || cols % 128) return 1;
  int blocks = (int)((n + 255) / 256);
  if (blocks > 148 * 16) blocks = 148 * 16;
  gen_fp8_kernel<<<blocks, 256, 0, (cudaStream_t)stream>>>(seed, tid, tid_scale, e0, cols, offset, n, factor,
                                                           (uint8_t*)out);
  return (int)cudaGetLastError();
}

// UE8M0 scale bytes of blocks [offset, offset + n).
int gen_fp8_scales_device(uint32_t seed, uint32_t tid_scale, int e0, uint64_t offset, uint64_t n, void* out,
                          void* stream) {
  if (n == 0) return 0;
  if (!out) return 1;
  int blocks = (int)((n + 255) / 256);
  if (blocks > 148 * 4) blocks = 148 * 4;
  gen_fp8_scales_kernel<<<blocks, 256, 0, (cudaStream_t)stream>>>(seed, tid_scale, e0, offset, n, (uint8_t*)out);
  return (int)cudaGetLastError();
}

}  // extern "C"
