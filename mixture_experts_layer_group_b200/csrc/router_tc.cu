// Router logits z = x W_r^T on the tensor cores (bf16 layers): the affinity
// step of the router ("DeepSeek-V3.2-Exp · Mixture of experts", "All 19
// steps": the token-to-centroid products that feed the scores).
//
// One CTA computes a 128-token x 64-expert tile over one K range. TMA brings
// 64-wide K slices of x and W_r into shared memory (128-byte swizzle); one
// thread issues four 128 x 64 x 16 UMMAs per slice into a fresh fp32 TMEM
// accumulator (eight rotating buffers of 64 columns); the epilogue warps read
// each slice's partial product and add it into per-thread fp64 totals. The
// tensor core thus never sums more than 64 products into one fp32 value, and
// the carries across slices are fp64, so the logit error stays near the
// final fp32 rounding (the bf16 products themselves are exact). The selection
// kernel adds the K ranges' planes in a fixed order, so results are
// deterministic.
//
// Roles (192 threads, one CTA per SM):
//   warp 0     TMA producer (one lane), kStages-deep ring of 24 KB stages
//   warp 1     TMEM owner and UMMA issuer (one lane)
//   warps 2-5  epilogue: warp w reads TMEM lane quadrant w % 4 (32 tokens),
//              64 experts per thread, fp64 totals in registers
// Every wait is bounded; on a timeout the CTA records MOE_DEV_WAIT_TIMEOUT,
// waits (bounded) for its own copies and MMAs, frees TMEM and exits.
#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int kM = kRtcTokens;
constexpr int kN = kRtcExperts;
constexpr int kKC = kRtcChunk;
constexpr int kStages = 8;
constexpr int kXBytes = kM * kKC * 2;      // 16 KB
constexpr int kWBytes = kN * kKC * 2;      // 8 KB
constexpr int kStageBytes = kXBytes + kWBytes;
constexpr int kAccBufs = 8;                // TMEM accumulators of kN columns
constexpr int kTmemCols = kAccBufs * kN;   // 512
constexpr int kThreads = 192;
constexpr int kEpiWarps = 4;

struct RtcParams {
  CUtensorMap x;   // [T, d], box 64 x 128
  CUtensorMap w;   // [N, d], box 64 x 64
  int64_t T;
  int N, d, k_len;
  float* logits;   // [S, T, N]
  unsigned* status;
};

struct RtcShared {
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t acc_full[kAccBufs];
  uint64_t acc_empty[kAccBufs];
  uint64_t drained;
  uint32_t tmem_base;
  int abort_flag;
  uint32_t consumed;   // stages the MMA issuer saw complete
  uint32_t issued;     // stages the producer issued
};

constexpr int kBarrierBytes = 512;
constexpr int kSmemBytes = kStages * kStageBytes + 1024 + kBarrierBytes;
static_assert(sizeof(RtcShared) <= kBarrierBytes, "barrier block");
static_assert(kSmemBytes <= 232448, "shared memory budget");
static_assert(kTmemCols == 512, "whole TMEM");

__global__ void __launch_bounds__(kThreads, 1) router_logits_tc_kernel(const __grid_constant__ RtcParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  RtcShared& sh = *reinterpret_cast<RtcShared*>(smem + kStages * kStageBytes);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  const int e0 = blockIdx.x * kN;
  const int64_t t0 = (int64_t)blockIdx.y * kM;
  const int k_begin = blockIdx.z * p.k_len;
  const int k_end = min(p.d, k_begin + p.k_len);
  const int nk = k_end > k_begin ? (k_end - k_begin + kKC - 1) / kKC : 0;
  float* out = p.logits + (size_t)blockIdx.z * (size_t)p.T * (size_t)p.N;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&sh.full[i], 1);
      mbar_init(&sh.empty[i], 1);
    }
    for (int i = 0; i < kAccBufs; ++i) {
      mbar_init(&sh.acc_full[i], 1);
      mbar_init(&sh.acc_empty[i], kEpiWarps);
    }
    mbar_init(&sh.drained, 1);
    sh.abort_flag = 0;
    sh.consumed = 0;
    sh.issued = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&p.x);
    tma_prefetch_desc(&p.w);
  }
  if (warp == 1) {
    tmem_alloc(&sh.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = sh.tmem_base;
  volatile int* abort_flag = &sh.abort_flag;

  if (warp == 0) {
    // ---------------------------------------------------------- producer --
    if (lane == 0) {
      uint32_t issued = 0;
      for (int c = 0; c < nk; ++c) {
        const int s = c % kStages;
        if (c >= kStages && !mbar_wait_bounded(&sh.empty[s], ((c / kStages) - 1) & 1, abort_flag)) {
          *abort_flag = 1;
          set_status(p.status, MOE_DEV_WAIT_TIMEOUT);
          break;
        }
        uint8_t* st = smem + s * kStageBytes;
        mbar_arrive_expect_tx(&sh.full[s], kStageBytes);
        const int k = k_begin + c * kKC;
        tma_load_2d(st, &p.x, &sh.full[s], k, (int32_t)t0);
        tma_load_2d(st + kXBytes, &p.w, &sh.full[s], k, e0);
        ++issued;
      }
      sh.issued = issued;
    }
  } else if (warp == 1) {
    // --------------------------------------------------------------- MMA --
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(kM, kN);
      uint32_t consumed = 0;
      for (int c = 0; c < nk; ++c) {
        const int s = c % kStages, b = c % kAccBufs;
        bool ok = mbar_wait_bounded(&sh.full[s], (c / kStages) & 1, abort_flag);
        if (ok) ++consumed;
        if (ok && c >= kAccBufs) ok = mbar_wait_bounded(&sh.acc_empty[b], ((c / kAccBufs) - 1) & 1, abort_flag);
        if (!ok) {
          *abort_flag = 1;
          set_status(p.status, MOE_DEV_WAIT_TIMEOUT);
          break;
        }
        tc_fence_after();
        const uint32_t xs = smem_u32(smem + s * kStageBytes);
        const uint64_t da = smem_desc_sw128(xs), db = smem_desc_sw128(xs + kXBytes);
#pragma unroll
        for (int kk = 0; kk < kKC / 16; ++kk)
          umma_bf16(tmem_base + (uint32_t)(b * kN), da + 2 * kk, db + 2 * kk, idesc, kk > 0 ? 1u : 0u);
        umma_commit(&sh.empty[s]);
        umma_commit(&sh.acc_full[b]);
      }
      sh.consumed = consumed;
      umma_commit(&sh.drained);  // fires once every MMA issued above has completed
      int no_abort = 0;
      if (!mbar_wait_bounded(&sh.drained, 0, &no_abort)) set_status(p.status, MOE_DEV_WAIT_TIMEOUT);
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------- epilogue --
    const int q = warp & 3;  // TMEM lane quadrant this warp may read
    double tot[kN];
#pragma unroll
    for (int j = 0; j < kN; ++j) tot[j] = 0.0;
    const uint32_t t_q = tmem_base + ((uint32_t)(q * 32) << 16);
    bool ok = true;
    for (int c = 0; c < nk; ++c) {
      const int b = c % kAccBufs;
      if (lane == 0) ok = mbar_wait_bounded(&sh.acc_full[b], (c / kAccBufs) & 1, abort_flag);
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      if (!ok) break;
      tc_fence_after();
#pragma unroll
      for (int h = 0; h < kN / 32; ++h) {
        uint32_t r[32];
        tmem_ld32(t_q + (uint32_t)(b * kN + 32 * h), r);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 32; ++j) tot[32 * h + j] += (double)__uint_as_float(r[j]);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh.acc_empty[b]);
    }
    if (!ok) {
      *abort_flag = 1;
      set_status(p.status, MOE_DEV_WAIT_TIMEOUT);
    } else {
      const int64_t t = t0 + 32 * q + lane;
      if (t < p.T) {
        float* row = out + t * p.N + e0;
        if (e0 + kN <= p.N && (p.N & 3) == 0) {
#pragma unroll
          for (int j = 0; j < kN; j += 4)
            *reinterpret_cast<float4*>(row + j) =
                make_float4((float)tot[j], (float)tot[j + 1], (float)tot[j + 2], (float)tot[j + 3]);
        } else {
#pragma unroll
          for (int j = 0; j < kN; ++j)
            if (e0 + j < p.N) row[j] = (float)tot[j];
        }
      }
    }
  }

  __syncthreads();
  if (warp == 0 && lane == 0) {
    // copies issued but never consumed (only after a timeout) must land
    // before this CTA's shared memory is released
    for (uint32_t j = sh.consumed; j < sh.issued; ++j) {
      const uint32_t s = j % kStages, ph = (j / kStages) & 1u;
      int no_abort = 0;
      if (!mbar_wait_bounded(&sh.full[s], ph, &no_abort)) {
        set_status(p.status, MOE_DEV_WAIT_TIMEOUT);
        break;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

}  // namespace

cudaError_t launch_router_logits_tc(const Problem& p, const void* x, const void* W_r, int S, int k_len,
                                    float* logits, unsigned* status, cudaStream_t s) {
  if (k_len % kKC != 0 || S < 1) return cudaErrorInvalidValue;
  RtcParams prm;
  if (!make_tmap_bf16(&prm.x, x, (uint64_t)p.T, (uint64_t)p.d, kKC, kM, true) ||
      !make_tmap_bf16(&prm.w, W_r, (uint64_t)p.N, (uint64_t)p.d, kKC, kN, true))
    return cudaErrorInvalidValue;
  prm.T = p.T;
  prm.N = p.N;
  prm.d = p.d;
  prm.k_len = k_len;
  prm.logits = logits;
  prm.status = status;
  static int configured_device = -1;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (configured_device != dev) {
    e = cudaFuncSetAttribute(router_logits_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    configured_device = dev;
  }
  dim3 grid((unsigned)((p.N + kN - 1) / kN), (unsigned)((p.T + kM - 1) / kM), (unsigned)S);
  router_logits_tc_kernel<<<grid, kThreads, kSmemBytes, s>>>(prm);
  return cudaGetLastError();
}

}  // namespace moe
