// Combine: y[t] = sum of the gated expert rows of token t, in ascending
// expert index, plus the shared-MLP row, accumulated in fp32 and rounded
// once. This is the last step of the "All 19 steps" list on the
// "DeepSeek-V3.2-Exp · Mixture of experts" page (Delta_ffn = y_routed +
// y_shared, with y_routed the gate-weighted sum over the selected experts);
// the fp32 accumulator and the ascending expert order follow the same page's
// quoted forward excerpt. A fixed order and no atomics make the result
// bitwise reproducible.
#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

template <typename TE>
struct Io;
template <>
struct Io<__nv_bfloat16> {
  static constexpr int kPerVec = 8;
  static MOE_DEV void add(const uint4& v, float* acc) {
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float2 f = __bfloat1622float2(h[i]);
      acc[2 * i] += f.x;
      acc[2 * i + 1] += f.y;
    }
  }
  static MOE_DEV uint4 pack(const float* acc) {
    uint4 o;
    o.x = pack_bf16x2(acc[0], acc[1]);
    o.y = pack_bf16x2(acc[2], acc[3]);
    o.z = pack_bf16x2(acc[4], acc[5]);
    o.w = pack_bf16x2(acc[6], acc[7]);
    return o;
  }
};
template <>
struct Io<float> {
  static constexpr int kPerVec = 4;
  static MOE_DEV void add(const uint4& v, float* acc) {
    acc[0] += __uint_as_float(v.x);
    acc[1] += __uint_as_float(v.y);
    acc[2] += __uint_as_float(v.z);
    acc[3] += __uint_as_float(v.w);
  }
  static MOE_DEV uint4 pack(const float* acc) {
    return make_uint4(__float_as_uint(acc[0]), __float_as_uint(acc[1]), __float_as_uint(acc[2]),
                      __float_as_uint(acc[3]));
  }
};

// One CTA per token; each thread owns 16-byte column vectors. slot_pos
// lists the token's rows in ascending expert order (written that way by the
// dispatch), -1 for a pair that was never placed.
template <typename TE, int KMAX>
__global__ void __launch_bounds__(256) combine_kernel(const uint4* __restrict__ y_rows,
                                                      const uint4* __restrict__ shared_rows,
                                                      const int32_t* __restrict__ slot_pos, int64_t T,
                                                      int k, int64_t R, int vecs, uint4* __restrict__ y) {
  constexpr int P = Io<TE>::kPerVec;
  for (int64_t t = blockIdx.x; t < T; t += gridDim.x) {
    int32_t rows[KMAX];  // routed row indices < R < 2^31
#pragma unroll
    for (int s = 0; s < KMAX; ++s) {
      const int32_t pos = s < k ? __ldg(slot_pos + t * k + s) : -1;
      rows[s] = (pos >= 0 && pos < R) ? pos : -1;
    }
    for (int v = threadIdx.x; v < vecs; v += blockDim.x) {
      uint4 buf[KMAX + 1];
#pragma unroll
      for (int s = 0; s < KMAX; ++s)
        if (rows[s] >= 0) buf[s] = __ldg(y_rows + (int64_t)rows[s] * vecs + v);
      if (shared_rows) buf[KMAX] = __ldg(shared_rows + t * vecs + v);
      float acc[P];
#pragma unroll
      for (int i = 0; i < P; ++i) acc[i] = 0.f;
#pragma unroll
      for (int s = 0; s < KMAX; ++s)
        if (rows[s] >= 0) Io<TE>::add(buf[s], acc);
      if (shared_rows) Io<TE>::add(buf[KMAX], acc);
      y[t * vecs + v] = Io<TE>::pack(acc);
    }
  }
}

}  // namespace

cudaError_t launch_combine_rows(const Problem& p, const void* routed_rows, const void* shared_rows,
                                const int32_t* slot_pos, void* y, cudaStream_t s) {
  const int vecs = (int)((int64_t)p.d * p.elem / 16);
  const int threads = vecs >= 256 ? 256 : (vecs >= 128 ? 128 : 64);
  int64_t cap = (int64_t)device_sm_count() * 16;
  unsigned blocks = (unsigned)(p.T < cap ? p.T : cap);
  const uint4* yr = (const uint4*)routed_rows;
  const uint4* ys = (const uint4*)shared_rows;
  if (p.dtype == MOE_BF16) {
    if (p.k <= 8)
      combine_kernel<__nv_bfloat16, 8><<<blocks, threads, 0, s>>>(yr, ys, slot_pos, p.T, p.k, p.R, vecs, (uint4*)y);
    else
      combine_kernel<__nv_bfloat16, kMaxTopK><<<blocks, threads, 0, s>>>(yr, ys, slot_pos, p.T, p.k, p.R, vecs,
                                                                        (uint4*)y);
  } else {
    if (p.k <= 8)
      combine_kernel<float, 8><<<blocks, threads, 0, s>>>(yr, ys, slot_pos, p.T, p.k, p.R, vecs, (uint4*)y);
    else
      combine_kernel<float, kMaxTopK><<<blocks, threads, 0, s>>>(yr, ys, slot_pos, p.T, p.k, p.R, vecs, (uint4*)y);
  }
  return cudaGetLastError();
}

cudaError_t launch_combine(const Problem& p, const void* y_rows, const int32_t* slot_pos, void* y,
                           cudaStream_t s) {
  // y_rows: the R gated routed rows, then (with a shared MLP) its T rows
  const void* shared = p.ns > 0 ? static_cast<const uint8_t*>(y_rows) + p.R * (int64_t)p.d * p.elem : nullptr;
  return launch_combine_rows(p, y_rows, shared, slot_pos, y, s);
}

}  // namespace moe
