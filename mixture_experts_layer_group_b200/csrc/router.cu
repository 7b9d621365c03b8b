// Router: z = x W_r^T on the FP32 pipes (CUDA cores), then score,
// group-limited top-k and gates by warp shuffles (router steps of the "All 19 steps" list on the
// "DeepSeek-V3.2-Exp · Mixture of experts" page; the softmax top-k variant is
// the GShard router of the "DeepSeekMoE" walkthrough, Step 2).
//
// Logits are accumulated in fp32 over 128-element K runs and carried across
// runs in fp64, which keeps the logit error near 1e-7 at d = 7168 (a plain
// fp32 running sum is an order of magnitude worse and would turn near-ties
// into routing differences). bf16 products are exact in fp32. When the
// token count alone gives too few CTAs (decode), K is split into S ranges
// whose partial logits the selection kernel adds in a fixed order, so the
// result stays deterministic.
#include <cfloat>
#include <cmath>
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int kLBT = 64;   // tokens per CTA tile
constexpr int kLBN = 64;   // experts per CTA tile
constexpr int kLBK = 32;   // K chunk (one shared-memory buffer)
constexpr int kLCarry = 4; // chunks summed in fp32 before each fp64 carry (128 K elements)
constexpr int kLPitch = kLBK + 4;  // smem row pitch (floats): conflict-free strided float4 reads
constexpr int kLThreads = 128;
constexpr int kLTA = kLBT / 8;   // tokens per thread (8 thread rows)
constexpr int kLTB = kLBN / 16;  // experts per thread (16 thread columns)
constexpr int kLBufFloats = (kLBT + kLBN) * kLPitch;
constexpr int kLSmemBytes = 2 * kLBufFloats * (int)sizeof(float);
constexpr int kLCtasPerSm = 2;

template <typename TIn>
struct Vec16 {
  static constexpr int kElems = 16 / sizeof(TIn);
};

// 16 bytes of row `row` (row pitch d) at column k, zero outside
// [0, rows) x [0, k_end).
template <typename TIn>
MOE_DEV uint4 load_raw(const TIn* base, int64_t rows, int k_end, int d, int64_t row, int k) {
  if (row < rows && k < k_end) return __ldg(reinterpret_cast<const uint4*>(base + row * (int64_t)d + k));
  return make_uint4(0u, 0u, 0u, 0u);
}

// Widens 16 raw bytes to fp32 (exact for bf16) and stores them at dst.
template <typename TIn>
MOE_DEV void store_widened(float* dst, uint4 v) {
  if constexpr (sizeof(TIn) == 2) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; i += 2) {
      *reinterpret_cast<float4*>(dst + 2 * i) =
          make_float4(__uint_as_float(w[i] << 16), __uint_as_float(w[i] & 0xffff0000u),
                      __uint_as_float(w[i + 1] << 16), __uint_as_float(w[i + 1] & 0xffff0000u));
    }
  } else {
    *reinterpret_cast<uint4*>(dst) = v;
  }
}

// One CTA computes a 64-token x 64-expert tile of logits over one K range
// on the FP32 pipes. Thread (tx, ty) owns tokens ty + 8a (a < 8) and
// experts tx + 16b (b < 4): per 4 K elements it reads 8 + 4 float4 from
// shared memory (one wavefront each: broadcast within the warp and
// conflict-free with the padded pitch) for 128 FMAs. Operand tiles are widened to fp32 once, when staged;
// the two shared-memory buffers alternate so each chunk needs one barrier,
// and the global loads of chunk c + 2 are in flight while chunk c computes.
// Two CTAs share an SM. The products go through the paired FP32 FMA
// (__ffma2_rn: one instruction, two lanes of fp32 FMA), which halves the
// issue slots the arithmetic needs: acc holds the running sums over the even
// and the odd K positions of each (token, expert), added at each carry.
template <typename TIn>
__global__ void __launch_bounds__(kLThreads, kLCtasPerSm) router_logits_kernel(const TIn* __restrict__ x,
                                                                     const TIn* __restrict__ W,
                                                                     int64_t T, int N, int d, int k_len,
                                                                     float* __restrict__ logits) {
  constexpr int E = Vec16<TIn>::kElems;          // elements per 16-byte vector
  constexpr int kVecPerRow = kLBK / E;           // vectors per row per chunk
  constexpr int kXLoads = kLBT * kVecPerRow / kLThreads;
  constexpr int kWLoads = (kLBN * kVecPerRow + kLThreads - 1) / kLThreads;
  static_assert(kLBT * kVecPerRow % kLThreads == 0, "tile / threads");
  constexpr int kWVecs = kLBN * kVecPerRow;      // W vectors per chunk (may be < threads)

  extern __shared__ __align__(16) float lsm[];

  const int tid = threadIdx.x;
  // a warp covers 4 token rows x 8 expert rows of the 8 x 16 thread grid, so
  // each float4 read touches 4 (x) or 8 (W) distinct rows: one wavefront
  const int warp = tid >> 5, lane = tid & 31;
  const int tx = (warp & 1) * 8 + (lane & 7), ty = (warp >> 1) * 4 + (lane >> 3);
  const int64_t t0 = (int64_t)blockIdx.y * kLBT;
  const int64_t e0 = (int64_t)blockIdx.x * kLBN;
  // this CTA's K range [k_begin, k_end) and its partial-logit plane
  const int k_begin = blockIdx.z * k_len;
  const int k_end = min(d, k_begin + k_len);
  logits += (int64_t)blockIdx.z * T * N;

  uint4 xr[kXLoads], wr[kWLoads];
  auto fetch = [&](int kbase) {
#pragma unroll
    for (int i = 0; i < kXLoads; ++i) {
      const int v = tid + i * kLThreads;
      xr[i] = load_raw<TIn>(x, T, k_end, d, t0 + v / kVecPerRow, kbase + (v % kVecPerRow) * E);
    }
#pragma unroll
    for (int i = 0; i < kWLoads; ++i) {
      const int v = tid + i * kLThreads;
      if (v < kWVecs) wr[i] = load_raw<TIn>(W, N, k_end, d, e0 + v / kVecPerRow, kbase + (v % kVecPerRow) * E);
    }
  };
  auto stash = [&](int buf) {
    float* xs = lsm + buf * kLBufFloats;
    float* ws = xs + kLBT * kLPitch;
#pragma unroll
    for (int i = 0; i < kXLoads; ++i) {
      const int v = tid + i * kLThreads;
      store_widened<TIn>(xs + (v / kVecPerRow) * kLPitch + (v % kVecPerRow) * E, xr[i]);
    }
#pragma unroll
    for (int i = 0; i < kWLoads; ++i) {
      const int v = tid + i * kLThreads;
      if (v < kWVecs) store_widened<TIn>(ws + (v / kVecPerRow) * kLPitch + (v % kVecPerRow) * E, wr[i]);
    }
  };


  double total[kLTA][kLTB];
  float2 acc[kLTA][kLTB];
#pragma unroll
  for (int a = 0; a < kLTA; ++a)
#pragma unroll
    for (int b = 0; b < kLTB; ++b) {
      total[a][b] = 0.0;
      acc[a][b] = make_float2(0.f, 0.f);
    }

  const int nk = k_end > k_begin ? (k_end - k_begin + kLBK - 1) / kLBK : 0;
  if (nk > 0) {
    fetch(k_begin);
    stash(0);
    __syncthreads();
    if (nk > 1) fetch(k_begin + kLBK);
  }
  for (int kc = 0; kc < nk; ++kc) {
    const float* xs = lsm + (kc & 1) * kLBufFloats;
    const float* ws = xs + kLBT * kLPitch;
#pragma unroll
    for (int kk = 0; kk < kLBK; kk += 4) {
      float4 wv[kLTB];
#pragma unroll
      for (int b = 0; b < kLTB; ++b) wv[b] = *reinterpret_cast<const float4*>(ws + (tx + 16 * b) * kLPitch + kk);
#pragma unroll
      for (int a = 0; a < kLTA; ++a) {
        const float4 xv = *reinterpret_cast<const float4*>(xs + (ty + 8 * a) * kLPitch + kk);
#pragma unroll
        for (int b = 0; b < kLTB; ++b) {
          acc[a][b] = __ffma2_rn(make_float2(xv.x, xv.y), make_float2(wv[b].x, wv[b].y), acc[a][b]);
          acc[a][b] = __ffma2_rn(make_float2(xv.z, xv.w), make_float2(wv[b].z, wv[b].w), acc[a][b]);
        }
      }
    }
    if ((kc + 1) % kLCarry == 0 || kc + 1 == nk) {
#pragma unroll
      for (int a = 0; a < kLTA; ++a)
#pragma unroll
        for (int b = 0; b < kLTB; ++b) {
          total[a][b] += (double)acc[a][b].x + (double)acc[a][b].y;
          acc[a][b] = make_float2(0.f, 0.f);
        }
    }
    // the other buffer was last read before the previous barrier
    if (kc + 1 < nk) stash((kc + 1) & 1);
    __syncthreads();
    if (kc + 2 < nk) fetch(k_begin + (kc + 2) * kLBK);
  }
#pragma unroll
  for (int a = 0; a < kLTA; ++a) {
    const int64_t t = t0 + ty + 8 * a;
    if (t >= T) continue;
#pragma unroll
    for (int b = 0; b < kLTB; ++b) {
      const int64_t e = e0 + tx + 16 * b;
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
  unsigned* status;     // MOE_DEV_* bits (may be null)
};

// One warp per token. Lane l holds experts e = 32 j + l, j < V.
template <int V>
__global__ void __launch_bounds__(256) router_select_kernel(SelectArgs a) {
  const int lane = threadIdx.x & 31;
  const int64_t t = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (t >= a.T) return;
  const int N = a.N;
  const float* zrow = a.logits + t * N;

  // z = plane 0 + plane 1 + ... in this order for every expert; the loads
  // of four planes are issued before their adds, so a token's 4 V loads are
  // in flight together instead of one dependent L2 round trip per plane
  const int64_t plane = a.T * N;
  float s[V], key[V];
#pragma unroll
  for (int j = 0; j < V; ++j) s[j] = 32 * j + lane < N ? zrow[32 * j + lane] : 0.f;
  int sp = 1;
  for (; sp + 4 <= a.S; sp += 4) {
    float v[4][V];
#pragma unroll
    for (int q = 0; q < 4; ++q)
#pragma unroll
      for (int j = 0; j < V; ++j) v[q][j] = 32 * j + lane < N ? zrow[(sp + q) * plane + 32 * j + lane] : 0.f;
#pragma unroll
    for (int q = 0; q < 4; ++q)
#pragma unroll
      for (int j = 0; j < V; ++j) s[j] += v[q][j];
  }
  for (; sp < a.S; ++sp) {
#pragma unroll
    for (int j = 0; j < V; ++j) s[j] += 32 * j + lane < N ? zrow[sp * plane + 32 * j + lane] : 0.f;
  }
#pragma unroll
  for (int j = 0; j < V; ++j)
    if (32 * j + lane >= N) s[j] = -INFINITY;
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
  // A NaN or infinite logit or key (from non-finite x, W_r or b) is
  // recorded in the status word; its key is replaced by the lowest finite
  // value, so the token still gets k distinct experts below N (which ones is
  // then arbitrary) and every other token is unaffected.
  bool bad = false;
#pragma unroll
  for (int j = 0; j < V; ++j) {
    int e = 32 * j + lane;
    if (e < N) {
      float kv = s[j] + (a.bias ? a.bias[e] : 0.f);
      if (!isfinite(kv) || !isfinite(s[j])) {
        bad = true;
        if (kv != kv) kv = -FLT_MAX;
      }
      key[j] = kv;
    } else {
      key[j] = -INFINITY;
    }
  }
  if (__any_sync(0xffffffffu, bad) && lane == 0) set_status(a.status, MOE_DEV_NONFINITE);

  if (a.G > 1) {
    // group scores: lane g keeps the score of group g (G <= 32)
    const int S = N / a.G;
    int grp[V];  // group of each of this lane's experts
#pragma unroll
    for (int j = 0; j < V; ++j) grp[j] = (32 * j + lane) / S;
    float my_gs = -INFINITY;
    for (int g = 0; g < a.G; ++g) {
      float t1 = -INFINITY, t2 = -INFINITY;
#pragma unroll
      for (int j = 0; j < V; ++j)
        if (32 * j + lane < N && grp[j] == g) merge_top2(t1, t2, key[j], -INFINITY);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        float o1 = __shfl_xor_sync(0xffffffffu, t1, off);
        float o2 = __shfl_xor_sync(0xffffffffu, t2, off);
        merge_top2(t1, t2, o1, o2);
      }
      float gsc = a.group_score == MOE_GROUP_MAX ? t1 : t1 + t2;
      if (gsc != gsc) gsc = -FLT_MAX;  // +inf + -inf keys of a non-finite token
      if (lane == g) my_gs = gsc;
    }
    uint32_t allowed = 0;
    bool g_taken = lane >= a.G;  // lane g: group g already kept (or no such group)
    for (int r = 0; r < a.TG; ++r) {
      Cand c = warp_best(Cand{g_taken ? -INFINITY : my_gs, g_taken ? 1 << 30 : lane});
      allowed |= 1u << (c.e & 31);
      if (lane == c.e) g_taken = true;
    }
#pragma unroll
    for (int j = 0; j < V; ++j)
      if (32 * j + lane < N && !((allowed >> grp[j]) & 1u)) key[j] = -INFINITY;
  }

  int sel_e = 0;
  float sel_s = 0.f, ssum = 0.f;
  uint32_t taken = 0;  // bit j: this lane's expert 32 j + lane is already selected
  for (int slot = 0; slot < a.k; ++slot) {
    Cand c{-INFINITY, 1 << 30};
#pragma unroll
    for (int j = 0; j < V; ++j) {
      int e = 32 * j + lane;
      if (e < N && !((taken >> j) & 1u) && better(key[j], e, c.v, c.e)) c = Cand{key[j], e};
    }
    c = warp_best(c);
    int owner = c.e & 31, jj = c.e >> 5;
    float sv = 0.f;
#pragma unroll
    for (int j = 0; j < V; ++j)
      if (lane == owner && j == jj) {
        sv = s[j];
        taken |= 1u << j;
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
  // The split count with the fewest CTA waves per unit of K work (a split adds a T x N plane for the selection kernel to read, so
  // a larger count must win by more than 1%), each split keeping >= 4 chunks.
  const int64_t base = (int64_t)((p.N + kLBN - 1) / kLBN) * ((p.T + kLBT - 1) / kLBT);
  if (base <= 0) return 1;
  int64_t max_s = p.d / (4 * kLBK);
  if (max_s > 16) max_s = 16;
  int best = 1;
  double best_cost = 1e30;
  for (int64_t S = 1; S <= max_s; ++S) {
    const int64_t slots = (int64_t)kRouterTargetSms * kLCtasPerSm;
    const int64_t waves = (base * S + slots - 1) / slots;
    const double cost = (double)waves / (double)S;
    if (cost < best_cost * 0.99) {
      best_cost = cost;
      best = (int)S;
    }
  }
  return best;
}

size_t router_scratch_bytes(const Problem& p) {
  return (size_t)router_k_splits(p) * (size_t)p.T * (size_t)p.N * sizeof(float);
}

cudaError_t launch_router(const Problem& p, const void* x, const void* W_r, const float* b,
                          float* logits, size_t logits_bytes, int32_t* idx, float* gates,
                          unsigned* status, cudaStream_t s, int splits) {
  // K splits: `splits` when given, else router_k_splits(p); the scratch must
  // hold one [T, N] plane of partial logits per split
  const size_t plane = (size_t)p.T * (size_t)p.N * sizeof(float);
  const int S = splits > 0 ? splits : router_k_splits(p);
  if (S > 16 || (size_t)S * plane > logits_bytes) return cudaErrorInvalidValue;
  const int k_len = ((p.d + S - 1) / S + kLBK - 1) / kLBK * kLBK;
  dim3 grid((unsigned)((p.N + kLBN - 1) / kLBN), (unsigned)((p.T + kLBT - 1) / kLBT), (unsigned)S);
  static std::mutex mu;
  static bool configured[kMaxDevices] = {};  // shared-memory opt-in done, per device
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  {
    std::lock_guard<std::mutex> lock(mu);
    if (!configured[dev]) {
      err = cudaFuncSetAttribute(router_logits_kernel<__nv_bfloat16>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, kLSmemBytes);
      if (err == cudaSuccess)
        err = cudaFuncSetAttribute(router_logits_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   kLSmemBytes);
      if (err != cudaSuccess) return err;
      configured[dev] = true;
    }
  }
  if (p.dtype == MOE_BF16)
    router_logits_kernel<__nv_bfloat16><<<grid, kLThreads, kLSmemBytes, s>>>(
        (const __nv_bfloat16*)x, (const __nv_bfloat16*)W_r, p.T, p.N, p.d, k_len, logits);
  else
    router_logits_kernel<float><<<grid, kLThreads, kLSmemBytes, s>>>((const float*)x, (const float*)W_r, p.T,
                                                                     p.N, p.d, k_len, logits);
  err = cudaGetLastError();
  if (err != cudaSuccess) return err;

  SelectArgs a{logits, S, b, p.T, p.N, p.k, p.G, p.TG, p.score_fn, p.group_score, p.normalize,
               p.route_scale, idx, gates, status};
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
