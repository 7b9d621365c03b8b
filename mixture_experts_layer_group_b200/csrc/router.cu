// Router: z = x W_r^T (fp32 layers on CUDA cores here; bf16 layers on the
// tensor cores, router_tc.cu), then score, group-limited top-k and gates by
// warp shuffles (router steps of the "All 19 steps" list on the
// "DeepSeek-V3.2-Exp · Mixture of experts" page; the softmax top-k variant is
// the GShard router of the "DeepSeekMoE" walkthrough, Step 2).
//
// The CUDA-core logits are accumulated in fp32 over 32-element K chunks and
// carried across chunks in fp64, which keeps the logit error near 1e-7 at d = 7168 (a plain
// fp32 running sum is an order of magnitude worse and would turn near-ties
// into routing differences). bf16 products are exact in fp32. When the
// token count alone gives too few CTAs (decode), K is split into S ranges
// whose partial logits the selection kernel adds in a fixed order, so the
// result stays deterministic.
#include <cfloat>
#include <cmath>

#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int kLBT = 64;   // tokens per CTA tile
constexpr int kLBN = 64;   // experts per CTA tile
constexpr int kLBK = 32;   // K chunk
constexpr int kLPitch = kLBK + 4;  // smem row pitch (floats): conflict-free strided float4 reads
constexpr int kLThreads = 256;

template <typename TIn>
struct Vec16 {
  static constexpr int kElems = 16 / sizeof(TIn);
};

// Loads 16 bytes of row `row` (row pitch d) at column k (zero outside
// [0, rows) x [0, k_end)).
template <typename TIn>
MOE_DEV void load_vec(const TIn* base, int64_t rows, int k_end, int d, int64_t row, int k, float* out) {
  constexpr int E = Vec16<TIn>::kElems;
  if (row < rows && k < k_end) {
    uint4 v = *reinterpret_cast<const uint4*>(base + row * (int64_t)d + k);
    if constexpr (sizeof(TIn) == 2) {
      const __nv_bfloat16* h = reinterpret_cast<const __nv_bfloat16*>(&v);
#pragma unroll
      for (int i = 0; i < E; ++i) out[i] = __bfloat162float(h[i]);
    } else {
      const float* f = reinterpret_cast<const float*>(&v);
#pragma unroll
      for (int i = 0; i < E; ++i) out[i] = f[i];
    }
  } else {
#pragma unroll
    for (int i = 0; i < E; ++i) out[i] = 0.f;
  }
}

// One CTA computes a 64-token x 64-expert tile of logits. Thread (tx, ty)
// owns tokens ty + 16a and experts tx + 16b (a, b in 0..3) so that the
// strided float4 reads of each K step are bank-conflict free.
template <typename TIn>
__global__ void __launch_bounds__(kLThreads) router_logits_kernel(const TIn* __restrict__ x,
                                                                  const TIn* __restrict__ W,
                                                                  int64_t T, int N, int d, int k_len,
                                                                  float* __restrict__ logits) {
  constexpr int E = Vec16<TIn>::kElems;          // elements per 16-byte vector
  constexpr int kVecPerRow = kLBK / E;           // vectors per row per chunk
  constexpr int kVecPerTile = kLBT * kVecPerRow; // vectors per operand tile
  constexpr int kLoads = kVecPerTile / kLThreads;
  static_assert(kVecPerTile % kLThreads == 0, "tile / thread mismatch");

  __shared__ __align__(16) float xs[kLBT][kLPitch];
  __shared__ __align__(16) float ws[kLBN][kLPitch];

  const int tid = threadIdx.x;
  const int tx = tid & 15, ty = tid >> 4;
  const int64_t t0 = (int64_t)blockIdx.y * kLBT;
  const int64_t e0 = (int64_t)blockIdx.x * kLBN;
  // this CTA's K range [k_begin, k_end) and its partial-logit plane
  const int k_begin = blockIdx.z * k_len;
  const int k_end = min(d, k_begin + k_len);
  logits += (int64_t)blockIdx.z * T * N;

  float xr[kLoads][E], wr[kLoads][E];
  auto fetch = [&](int kbase) {
#pragma unroll
    for (int i = 0; i < kLoads; ++i) {
      int v = tid + i * kLThreads;
      int row = v / kVecPerRow, kv = (v % kVecPerRow) * E;
      load_vec<TIn>(x, T, k_end, d, t0 + row, kbase + kv, xr[i]);
      load_vec<TIn>(W, N, k_end, d, e0 + row, kbase + kv, wr[i]);
    }
  };
  auto stash = [&]() {
#pragma unroll
    for (int i = 0; i < kLoads; ++i) {
      int v = tid + i * kLThreads;
      int row = v / kVecPerRow, kv = (v % kVecPerRow) * E;
#pragma unroll
      for (int j = 0; j < E; j += 4) {
        *reinterpret_cast<float4*>(&xs[row][kv + j]) =
            make_float4(xr[i][j], xr[i][j + 1], xr[i][j + 2], xr[i][j + 3]);
        *reinterpret_cast<float4*>(&ws[row][kv + j]) =
            make_float4(wr[i][j], wr[i][j + 1], wr[i][j + 2], wr[i][j + 3]);
      }
    }
  };

  double total[4][4];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int b = 0; b < 4; ++b) total[a][b] = 0.0;

  const int nk = (k_end - k_begin + kLBK - 1) / kLBK;
  fetch(k_begin);
  for (int kc = 0; kc < nk; ++kc) {
    __syncthreads();
    stash();
    __syncthreads();
    if (kc + 1 < nk) fetch(k_begin + (kc + 1) * kLBK);
    float acc[4][4];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int b = 0; b < 4; ++b) acc[a][b] = 0.f;
#pragma unroll
    for (int kk = 0; kk < kLBK; kk += 4) {
      float4 xv[4], wv[4];
#pragma unroll
      for (int a = 0; a < 4; ++a) xv[a] = *reinterpret_cast<const float4*>(&xs[ty + 16 * a][kk]);
#pragma unroll
      for (int b = 0; b < 4; ++b) wv[b] = *reinterpret_cast<const float4*>(&ws[tx + 16 * b][kk]);
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) {
          acc[a][b] = fmaf(xv[a].x, wv[b].x, acc[a][b]);
          acc[a][b] = fmaf(xv[a].y, wv[b].y, acc[a][b]);
          acc[a][b] = fmaf(xv[a].z, wv[b].z, acc[a][b]);
          acc[a][b] = fmaf(xv[a].w, wv[b].w, acc[a][b]);
        }
    }
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int b = 0; b < 4; ++b) total[a][b] += (double)acc[a][b];
  }
#pragma unroll
  for (int a = 0; a < 4; ++a) {
    int64_t t = t0 + ty + 16 * a;
    if (t >= T) continue;
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      int64_t e = e0 + tx + 16 * b;
      if (e < N) logits[t * N + e] = (float)total[a][b];
    }
  }
}

struct Cand {
  float v;
  int e;
};

// Larger value first; among equal values the lower index.
MOE_DEV bool better(float v, int e, float bv, int be) { return v > bv || (v == bv && e < be); }

MOE_DEV Cand warp_best(Cand c) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    float ov = __shfl_xor_sync(0xffffffffu, c.v, off);
    int oe = __shfl_xor_sync(0xffffffffu, c.e, off);
    if (better(ov, oe, c.v, c.e)) {
      c.v = ov;
      c.e = oe;
    }
  }
  return c;
}

MOE_DEV float warp_max(float v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, off));
  return v;
}

MOE_DEV float warp_sum(float v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  return v;
}

// The two largest of {a1 >= a2} and {b1 >= b2}.
MOE_DEV void merge_top2(float& a1, float& a2, float b1, float b2) {
  if (b1 > a1) {
    a2 = fmaxf(a1, b2);
    a1 = b1;
  } else {
    a2 = fmaxf(a2, b1);
  }
}

struct SelectArgs {
  const float* logits;  // [S, T, N] partial logits
  int S;
  const float* bias;
  int64_t T;
  int N, k, G, TG, score_fn, group_score, normalize;
  float route_scale;
  int32_t* idx;
  float* gates;
};

// One warp per token. Lane l holds experts e = 32 j + l, j < V.
template <int V>
__global__ void __launch_bounds__(256) router_select_kernel(SelectArgs a) {
  const int lane = threadIdx.x & 31;
  const int64_t t = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (t >= a.T) return;
  const int N = a.N;
  const float* zrow = a.logits + t * N;

  float s[V], key[V];
#pragma unroll
  for (int j = 0; j < V; ++j) {
    int e = 32 * j + lane;
    if (e < N) {
      float z = zrow[e];
      for (int sp = 1; sp < a.S; ++sp) z += zrow[(int64_t)sp * a.T * N + e];  // fixed order
      s[j] = z;
    } else {
      s[j] = -INFINITY;
    }
  }
  if (a.score_fn == MOE_SOFTMAX) {
    float m = -INFINITY;
#pragma unroll
    for (int j = 0; j < V; ++j) m = fmaxf(m, s[j]);
    m = warp_max(m);
    float sum = 0.f;
#pragma unroll
    for (int j = 0; j < V; ++j) {
      s[j] = (32 * j + lane < N) ? expf(s[j] - m) : 0.f;
      sum += s[j];
    }
    sum = warp_sum(sum);
#pragma unroll
    for (int j = 0; j < V; ++j) s[j] = s[j] / sum;
  } else {
#pragma unroll
    for (int j = 0; j < V; ++j) s[j] = (32 * j + lane < N) ? 1.0f / (1.0f + expf(-s[j])) : 0.f;
  }
#pragma unroll
  for (int j = 0; j < V; ++j) {
    int e = 32 * j + lane;
    key[j] = e < N ? s[j] + (a.bias ? a.bias[e] : 0.f) : -INFINITY;
  }

  if (a.G > 1) {
    // group scores: lane g keeps the score of group g (G <= 32)
    const int S = N / a.G;
    float my_gs = -INFINITY;
    for (int g = 0; g < a.G; ++g) {
      float t1 = -INFINITY, t2 = -INFINITY;
#pragma unroll
      for (int j = 0; j < V; ++j) {
        int e = 32 * j + lane;
        if (e < N && e / S == g) merge_top2(t1, t2, key[j], -INFINITY);
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        float o1 = __shfl_xor_sync(0xffffffffu, t1, off);
        float o2 = __shfl_xor_sync(0xffffffffu, t2, off);
        merge_top2(t1, t2, o1, o2);
      }
      float gsc = a.group_score == MOE_GROUP_MAX ? t1 : t1 + t2;
      if (lane == g) my_gs = gsc;
    }
    uint32_t allowed = 0;
    for (int r = 0; r < a.TG; ++r) {
      Cand c = warp_best(Cand{lane < a.G ? my_gs : -INFINITY, lane < a.G ? lane : 1 << 30});
      allowed |= 1u << (c.e & 31);
      if (lane == c.e) my_gs = -INFINITY;
    }
#pragma unroll
    for (int j = 0; j < V; ++j) {
      int e = 32 * j + lane;
      if (e < N && !((allowed >> (e / S)) & 1u)) key[j] = -INFINITY;
    }
  }

  int sel_e = 0;
  float sel_s = 0.f, ssum = 0.f;
  for (int slot = 0; slot < a.k; ++slot) {
    Cand c{-INFINITY, 1 << 30};
#pragma unroll
    for (int j = 0; j < V; ++j) {
      int e = 32 * j + lane;
      if (e < N && better(key[j], e, c.v, c.e)) c = Cand{key[j], e};
    }
    c = warp_best(c);
    int owner = c.e & 31, jj = c.e >> 5;
    float sv = 0.f;
#pragma unroll
    for (int j = 0; j < V; ++j)
      if (lane == owner && j == jj) {
        sv = s[j];
        key[j] = -INFINITY;
      }
    sv = __shfl_sync(0xffffffffu, sv, owner);
    ssum += sv;
    if (lane == slot) {
      sel_e = c.e;
      sel_s = sv;
    }
  }
  if (lane < a.k) {
    float g = a.normalize ? a.route_scale * sel_s / ssum : a.route_scale * sel_s;
    a.idx[t * a.k + lane] = sel_e;
    a.gates[t * a.k + lane] = g;
  }
}

}  // namespace

int router_k_splits(const Problem& p) {
  // enough CTAs to fill the SMs (tensor cores: once, one CTA per SM; SIMT:
  // twice), each split keeping >= 4 K chunks
  const bool tc = p.dtype == MOE_BF16;
  const int64_t tn = tc ? kRtcExperts : kLBN, tt = tc ? kRtcTokens : kLBT, kc = tc ? kRtcChunk : kLBK;
  const int64_t base = (int64_t)((p.N + tn - 1) / tn) * ((p.T + tt - 1) / tt);
  const int64_t target = (tc ? 1 : 2) * (int64_t)kRouterTargetSms;
  int64_t S = base > 0 ? target / base : 1;
  const int64_t by_k = p.d / (4 * kc);
  if (S > by_k) S = by_k;
  if (S > 16) S = 16;
  return S < 1 ? 1 : (int)S;
}

size_t router_scratch_bytes(const Problem& p) {
  return (size_t)router_k_splits(p) * (size_t)p.T * (size_t)p.N * sizeof(float);
}

cudaError_t launch_router(const Problem& p, const void* x, const void* W_r, const float* b,
                          float* logits, size_t logits_bytes, int32_t* idx, float* gates,
                          unsigned* status, cudaStream_t s) {
  // as many K splits as router_k_splits(p) asks for and the scratch can hold
  const size_t plane = (size_t)p.T * (size_t)p.N * sizeof(float);
  int S = router_k_splits(p);
  if ((size_t)S * plane > logits_bytes) S = (int)(logits_bytes / plane);
  if (S < 1) return cudaErrorInvalidValue;
  cudaError_t err;
  if (p.dtype == MOE_BF16) {
    const int k_len = ((p.d + S - 1) / S + kRtcChunk - 1) / kRtcChunk * kRtcChunk;
    err = launch_router_logits_tc(p, x, W_r, S, k_len, logits, status, s);
  } else {
    const int k_len = ((p.d + S - 1) / S + kLBK - 1) / kLBK * kLBK;
    dim3 grid((unsigned)((p.N + kLBN - 1) / kLBN), (unsigned)((p.T + kLBT - 1) / kLBT), (unsigned)S);
    router_logits_kernel<float><<<grid, kLThreads, 0, s>>>((const float*)x, (const float*)W_r, p.T,
                                                           p.N, p.d, k_len, logits);
    err = cudaGetLastError();
  }
  if (err != cudaSuccess) return err;

  SelectArgs a{logits, S, b, p.T, p.N, p.k, p.G, p.TG, p.score_fn, p.group_score, p.normalize,
               p.route_scale, idx, gates};
  const int warps = 8;
  unsigned blocks = (unsigned)((p.T + warps - 1) / warps);
  int V = (p.N + 31) / 32;
  if (V <= 1) router_select_kernel<1><<<blocks, 32 * warps, 0, s>>>(a);
  else if (V <= 2) router_select_kernel<2><<<blocks, 32 * warps, 0, s>>>(a);
  else if (V <= 4) router_select_kernel<4><<<blocks, 32 * warps, 0, s>>>(a);
  else if (V <= 8) router_select_kernel<8><<<blocks, 32 * warps, 0, s>>>(a);
  else router_select_kernel<16><<<blocks, 32 * warps, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace moe
