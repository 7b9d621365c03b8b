// fp32 grouped expert GEMMs on CUDA cores, for layers stored in fp32 (the
// GShard-style toy layer): tensor cores would round the operands (TF32) far
// beyond the fp32 tolerance. Same grouping, unit tables and epilogues as the
// tensor-core path: SwiGLU GEMM h = silu(x W1^T) * (x W3^T), then gate GEMM
// E = (h W2^T) * G, written to the token slot's row.
#include <cmath>

#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int kBM = kSimtBM;   // 64 rows
constexpr int kBN = kSimtBN;   // 64 columns
constexpr int kBK = 16;
constexpr int kThreads = 256;  // 16 x 16 threads, 4 x 4 outputs each

struct SimtParams {
  const float* a_routed;  // x_perm [R, K] | h_perm [R, F]
  const float* a_shared;  // x [T, d]      | h_sh [T, nsF]
  const float* b0_routed; // W1 [N*F, d]   | W2 [N*d, F]
  const float* b1_routed; // W3            | unused
  const float* b0_shared; // Ws1           | Ws2
  const float* b1_shared; // Ws3           | unused
  const int32_t* unit_base;
  const int32_t* grp_row0;
  const int32_t* grp_rows;
  int N;
  int k_routed, k_shared;
  int cols_routed, cols_shared;
  int b_rows_per_expert;
  float* out_routed;
  int64_t ld_routed;
  float* out_shared;
  int64_t ld_shared;
  const float* gate_perm;
};

template <bool kSwiGLU>
__global__ void __launch_bounds__(kThreads) expert_gemm_simt_kernel(SimtParams p) {
  __shared__ float As[kBK][kBM + 4];
  __shared__ float Bs0[kBK][kBN + 4];
  __shared__ float Bs1[kBK][kBN + 4];
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  const int total = p.unit_base[p.N + 1];
  for (int u = blockIdx.x; u < total; u += gridDim.x) {
    int lo = 0, hi = p.N;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (p.unit_base[mid] <= u) lo = mid;
      else hi = mid - 1;
    }
    const int g = lo;
    const int rows = p.grp_rows[g];
    const int mt = (rows + kBM - 1) / kBM;
    const int local = u - p.unit_base[g];
    const int f = local / mt, m = local % mt;
    const bool shared = g == p.N;
    const int K = shared ? p.k_shared : p.k_routed;
    const int cols = shared ? p.cols_shared : p.cols_routed;
    const int64_t row0 = shared ? 0 : p.grp_row0[g];
    const float* A = (shared ? p.a_shared : p.a_routed) + row0 * K;
    const int64_t brow0 = (shared ? 0 : (int64_t)g * p.b_rows_per_expert) + (int64_t)f * kBN;
    const float* B0 = (shared ? p.b0_shared : p.b0_routed) + brow0 * K;
    const float* B1 = kSwiGLU ? (shared ? p.b1_shared : p.b1_routed) + brow0 * K : nullptr;
    const int rows_here = rows - m * kBM;        // valid A rows in this tile (>= 1)
    const int cols_here = cols - f * kBN;        // valid B rows (output columns)

    float acc0[4][4] = {}, acc1[4][4] = {};
    for (int k0 = 0; k0 < K; k0 += kBK) {
      __syncthreads();
      // 64 x 16 tiles: 1024 elements each, 4 per thread, stored K-major in smem
      for (int i = tid; i < kBM * kBK; i += kThreads) {
        const int r = i / kBK, kk = i % kBK;
        const int gk = k0 + kk;
        As[kk][r] = (r < rows_here && gk < K) ? A[(int64_t)(m * kBM + r) * K + gk] : 0.f;
        Bs0[kk][r] = (r < cols_here && gk < K) ? B0[(int64_t)r * K + gk] : 0.f;
        if (kSwiGLU) Bs1[kk][r] = (r < cols_here && gk < K) ? B1[(int64_t)r * K + gk] : 0.f;
      }
      __syncthreads();
#pragma unroll
      for (int kk = 0; kk < kBK; ++kk) {
        float a[4], b0[4], b1[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          a[i] = As[kk][ty + 16 * i];
          b0[i] = Bs0[kk][tx + 16 * i];
          if (kSwiGLU) b1[i] = Bs1[kk][tx + 16 * i];
        }
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            acc0[i][j] = fmaf(a[i], b0[j], acc0[i][j]);
            if (kSwiGLU) acc1[i][j] = fmaf(a[i], b1[j], acc1[i][j]);
          }
      }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int r = ty + 16 * i;
      if (r >= rows_here) continue;
      const int64_t row = row0 + (int64_t)m * kBM + r;
      float* out = shared ? p.out_shared + row * p.ld_shared : p.out_routed + row * p.ld_routed;
      const float gate = (kSwiGLU || shared || !p.gate_perm) ? 1.f : p.gate_perm[row];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int c = tx + 16 * j;
        if (c >= cols_here) continue;
        float v;
        if (kSwiGLU) {
          const float gv = acc0[i][j];
          v = gv / (1.0f + expf(-gv)) * acc1[i][j];
        } else {
          v = acc0[i][j] * gate;
        }
        out[(int64_t)f * kBN + c] = v;
      }
    }
  }
}

}  // namespace

cudaError_t launch_expert_gemms_simt(const Problem& p, const GemmArgs& a, cudaStream_t s,
                                   cudaEvent_t between) {
  const int sms = device_sm_count();
  const int grid = sms * 4;
  SimtParams g1{(const float*)a.x_perm, (const float*)a.x, (const float*)a.W1, (const float*)a.W3,
                (const float*)a.Ws1, (const float*)a.Ws3, a.unit_base1, a.grp_row0, a.grp_rows,
                p.N, p.d, p.d, p.F, p.nsF, p.F, (float*)a.h_perm, p.F, (float*)a.h_sh, p.nsF,
                nullptr};
  expert_gemm_simt_kernel<true><<<grid, kThreads, 0, s>>>(g1);
  cudaError_t err = cudaGetLastError();
  if (err == cudaSuccess && between) err = cudaEventRecord(between, s);
  if (err != cudaSuccess) return err;
  SimtParams g2{(const float*)a.h_perm, (const float*)a.h_sh, (const float*)a.W2, nullptr,
                (const float*)a.Ws2, nullptr, a.unit_base2, a.grp_row0, a.grp_rows, p.N, p.F, p.nsF,
                p.d, p.d, p.d, (float*)a.y_rows, p.d, (float*)a.y_rows + p.R * (int64_t)p.d, p.d,
                a.gate_perm};
  expert_gemm_simt_kernel<false><<<grid, kThreads, 0, s>>>(g2);
  return cudaGetLastError();
}

}  // namespace moe
