// Combine: y[t] = sum of the gated expert rows of token t, in ascending
// expert index, plus the shared-MLP row, accumulated in fp32 and rounded
// once (the quoted MoE.forward's fp32 accumulator and its expert loop in
// ascending index, then "y += shared_experts(x)"; "DeepSeek-V3.2-Exp ·
// Mixture of experts", Delta_ffn = y_routed + y_shared). A fixed order and
// no atomics make the result bitwise reproducible.
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

// One CTA per token; each thread owns 16-byte column vectors.
template <typename TE>
__global__ void __launch_bounds__(128) combine_kernel(const uint4* __restrict__ y_rows,
                                                      const int32_t* __restrict__ slot_pos,
                                                      const int32_t* __restrict__ idx, int64_t T,
                                                      int k, int N, int has_shared, int64_t R,
                                                      int vecs, uint4* __restrict__ y) {
  constexpr int P = Io<TE>::kPerVec;
  for (int64_t t = blockIdx.x; t < T; t += gridDim.x) {
    // slots sorted by ascending expert index (k <= 16, insertion sort)
    int64_t rows[kMaxTopK + 1];
    int experts[kMaxTopK];
    int n = 0;
    for (int s = 0; s < k; ++s) {
      const int e = idx[t * k + s];
      const int32_t pos = slot_pos[t * k + s];
      if (e < 0 || e >= N || pos < 0 || pos >= R) continue;  // unplaced pair: contributes nothing
      int j = n++;
      while (j > 0 && experts[j - 1] > e) {
        experts[j] = experts[j - 1];
        rows[j] = rows[j - 1];
        --j;
      }
      experts[j] = e;
      rows[j] = pos;
    }
    if (has_shared) rows[n++] = R + t;
    for (int v = threadIdx.x; v < vecs; v += blockDim.x) {
      float acc[P];
#pragma unroll
      for (int i = 0; i < P; ++i) acc[i] = 0.f;
      uint4 buf[kMaxTopK + 1];
#pragma unroll
      for (int s = 0; s < kMaxTopK + 1; ++s)
        if (s < n) buf[s] = y_rows[rows[s] * vecs + v];
#pragma unroll
      for (int s = 0; s < kMaxTopK + 1; ++s)
        if (s < n) Io<TE>::add(buf[s], acc);
      y[t * vecs + v] = Io<TE>::pack(acc);
    }
  }
}

}  // namespace

cudaError_t launch_combine(const Problem& p, const void* y_rows, const int32_t* slot_pos,
                           const int32_t* idx, void* y, cudaStream_t s) {
  const int vecs = (int)((int64_t)p.d * p.elem / 16);
  int64_t cap = (int64_t)device_sm_count() * 16;
  unsigned blocks = (unsigned)(p.T < cap ? p.T : cap);
  if (p.dtype == MOE_BF16)
    combine_kernel<__nv_bfloat16><<<blocks, 128, 0, s>>>((const uint4*)y_rows, slot_pos, idx, p.T,
                                                        p.k, p.N, p.ns > 0, p.R, vecs, (uint4*)y);
  else
    combine_kernel<float><<<blocks, 128, 0, s>>>((const uint4*)y_rows, slot_pos, idx, p.T, p.k,
                                                p.N, p.ns > 0, p.R, vecs, (uint4*)y);
  return cudaGetLastError();
}

}  // namespace moe
