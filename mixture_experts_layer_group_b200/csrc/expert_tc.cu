// Grouped expert GEMMs on the 5th-generation tensor cores (tcgen05 + TMEM,
// operands staged by TMA). Two launches per layer:
//
//   SwiGLU GEMM  per group: g = X W1^T, u = X W3^T (one UMMA of N = 256 whose
//                B tile stacks 128 rows of W1 over the same 128 rows of W3),
//                epilogue h = silu(g) * u -> bf16
//                ("Routed expert:" / "Shared expert:" steps g = x W1, u = x W3,
//                a = g sigma(g), h = a (.) u)
//   gate GEMM    per group: E = h W2^T (UMMA N = 256 model columns), epilogue
//                E * G (the row's gate; 1 for the shared MLP) -> bf16 row of
//                the token's slot ("E_i = h W2", "y_routed = sum G_i E_i")
//
// Groups 0..N-1 are the routed experts over their expert-contiguous token
// rows; group N is the fused shared MLP over all T tokens, scheduled in the
// same persistent launch. A unit of work is (group, output-column tile,
// 128-row tile); units of one group are consecutive and ordered column-tile
// major so that concurrent CTAs share each weight tile through L2.
//
// CTA roles (192 threads, one CTA per SM, persistent over units):
//   warp 0      TMA producer (one lane): A tile 128 x 64 and B tile 256 x 64
//               per stage, 4-stage ring of 48 KB
//   warp 1      TMEM owner + UMMA issuer (one lane): 4 x (128 x 256 x 16)
//               per stage into one of two 256-column fp32 accumulators
//   warps 2..5  epilogue: tcgen05.ld of the accumulator quadrant the warp may
//               access, fused SwiGLU / gate, predicated row stores
// Every mbarrier wait is bounded; on a timeout the CTA records
// MOE_DEV_WAIT_TIMEOUT, drains its own copies and MMAs (bounded again),
// frees its tensor memory and exits.
#include <cuda.h>

#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int kStages = 4;
constexpr int kBK = 64;                              // bf16 per K chunk: one 128 B swizzle row
constexpr int kATileBytes = kTcBM * kBK * 2;         // 16 KB
constexpr int kBTileBytes = 256 * kBK * 2;           // 32 KB
constexpr int kStageBytes = kATileBytes + kBTileBytes;
constexpr int kAccCols = 256;                        // fp32 columns per accumulator
constexpr int kTmemCols = 2 * kAccCols;
constexpr int kThreads = 192;
constexpr int kBarrierBytes = 256;
constexpr int kSmemBytes = kStages * kStageBytes + 1024 + kBarrierBytes;
constexpr uint32_t kIdesc = idesc_bf16_f32(kTcBM, 256);

enum Mode : int { kSwiGLU = 0, kGateDown = 1 };

struct TcParams {
  CUtensorMap a_routed;   // x_perm [R, d]   | h_perm [R, F]
  CUtensorMap a_shared;   // x [T, d]        | h_sh [T, nsF]
  CUtensorMap b0_routed;  // W1 [N*F, d]     | W2 [N*d, F]
  CUtensorMap b1_routed;  // W3 [N*F, d]     | unused
  CUtensorMap b0_shared;  // Ws1 [nsF, d]    | Ws2 [d, nsF]
  CUtensorMap b1_shared;  // Ws3 [nsF, d]    | unused
  const int32_t* unit_base;  // [N + 2]: units before group g; [N + 1] = total
  const int32_t* grp_row0;   // [N + 1]
  const int32_t* grp_rows;   // [N + 1]
  int N;
  int k_routed, k_shared;        // reduction length (d | F, d | nsF)
  int cols_routed, cols_shared;  // output columns (F, nsF | d, d)
  int b_rows_per_expert;         // rows of the stacked B per routed expert (F | d)
  int bn;                        // output columns per tile (128 | 256)
  __nv_bfloat16* out_routed;
  int64_t ld_routed;
  __nv_bfloat16* out_shared;
  int64_t ld_shared;
  const float* gate_perm;        // [R] (gate-down mode)
  unsigned* status;
};

struct Unit {
  int g, f, m;
};

MOE_DEV Unit decode_unit(const TcParams& p, int u) {
  int lo = 0, hi = p.N;  // largest g with unit_base[g] <= u
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (__ldg(p.unit_base + mid) <= u) lo = mid;
    else hi = mid - 1;
  }
  const int local = u - __ldg(p.unit_base + lo);
  const int rows = __ldg(p.grp_rows + lo);
  const int mt = (rows + kTcBM - 1) / kTcBM;
  return Unit{lo, local / mt, local % mt};
}

struct Shared {
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint64_t drained;
  uint32_t tmem_base;
  int abort_flag;
  uint32_t consumed;  // stage fills the MMA issuer observed complete
};

// Stores 32 consecutive values of one row as bf16 (16-byte stores), or the
// first ncols of them at a ragged right edge.
MOE_DEV void store_cols(__nv_bfloat16* dst, int ncols, const float (&v)[32]) {
  if (ncols >= 32) {
    uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
    for (int i = 0; i < 4; ++i)
      d4[i] = make_uint4(pack_bf16x2(v[8 * i + 0], v[8 * i + 1]), pack_bf16x2(v[8 * i + 2], v[8 * i + 3]),
                         pack_bf16x2(v[8 * i + 4], v[8 * i + 5]), pack_bf16x2(v[8 * i + 6], v[8 * i + 7]));
  } else {
#pragma unroll
    for (int j = 0; j < 32; ++j)
      if (j < ncols) dst[j] = __float2bfloat16_rn(v[j]);
  }
}

template <int MODE>
__global__ void __launch_bounds__(kThreads, 1) expert_gemm_tc_kernel(const __grid_constant__ TcParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Shared& sh = *reinterpret_cast<Shared*>(smem + kStages * kStageBytes);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int total_units = __ldg(p.unit_base + p.N + 1);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sh.full[s], 1);
      mbar_init(&sh.empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sh.acc_full[b], 1);
      mbar_init(&sh.acc_empty[b], 4);
    }
    mbar_init(&sh.drained, 1);
    sh.abort_flag = 0;
    sh.consumed = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&p.a_routed);
    tma_prefetch_desc(&p.b0_routed);
    if (MODE == kSwiGLU) tma_prefetch_desc(&p.b1_routed);
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

  uint32_t fills = 0;  // producer: stage fills issued
  if (warp == 0) {
    // ------------------------------------------------------------ producer --
    if (lane == 0) {
      const uint64_t pol_w = policy_evict_first();  // weights: each tile is streamed once
      for (int u = blockIdx.x; u < total_units; u += gridDim.x) {
        const Unit un = decode_unit(p, u);
        const bool shared = un.g == p.N;
        const int K = shared ? p.k_shared : p.k_routed;
        const int nk = (K + kBK - 1) / kBK;
        const int rowA = __ldg(p.grp_row0 + un.g) + un.m * kTcBM;
        const int rowB = (shared ? 0 : un.g * p.b_rows_per_expert) + un.f * p.bn;
        const CUtensorMap* ta = shared ? &p.a_shared : &p.a_routed;
        const CUtensorMap* tb0 = shared ? &p.b0_shared : &p.b0_routed;
        const CUtensorMap* tb1 = shared ? &p.b1_shared : &p.b1_routed;
        bool ok = true;
        for (int kc = 0; kc < nk; ++kc, ++fills) {
          const uint32_t s = fills % kStages, ph = (fills / kStages) & 1u;
          if (!mbar_wait_bounded(&sh.empty[s], ph ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          uint8_t* a_dst = smem + s * kStageBytes;
          uint8_t* b_dst = a_dst + kATileBytes;
          mbar_arrive_expect_tx(&sh.full[s], kStageBytes);
          tma_load_2d(a_dst, ta, &sh.full[s], kc * kBK, rowA);
          if (MODE == kSwiGLU) {
            tma_load_2d_hint(b_dst, tb0, &sh.full[s], kc * kBK, rowB, pol_w);
            tma_load_2d_hint(b_dst + kBTileBytes / 2, tb1, &sh.full[s], kc * kBK, rowB, pol_w);
          } else {
            tma_load_2d_hint(b_dst, tb0, &sh.full[s], kc * kBK, rowB, pol_w);
          }
        }
        if (!ok) {
          *abort_flag = 1;
          set_status(p.status, MOE_DEV_WAIT_TIMEOUT);
          break;
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer --
    if (lane == 0) {
      uint32_t consumed = 0;
      int i = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < total_units && ok; u += gridDim.x, ++i) {
        const Unit un = decode_unit(p, u);
        const int K = un.g == p.N ? p.k_shared : p.k_routed;
        const int nk = (K + kBK - 1) / kBK;
        const uint32_t buf = i & 1, aph = (i >> 1) & 1;
        if (!mbar_wait_bounded(&sh.acc_empty[buf], aph ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + buf * kAccCols;
        for (int kc = 0; kc < nk; ++kc) {
          const uint32_t s = consumed % kStages, ph = (consumed / kStages) & 1u;
          if (!mbar_wait_bounded(&sh.full[s], ph, abort_flag)) {
            ok = false;
            break;
          }
          ++consumed;
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smem + s * kStageBytes);
          const uint32_t b_addr = a_addr + kATileBytes;
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk) {
            umma_bf16(d_tmem, smem_desc_sw128(a_addr + kk * 32), smem_desc_sw128(b_addr + kk * 32),
                      kIdesc, (kc | kk) != 0);
          }
          umma_commit(&sh.empty[s]);
        }
        if (ok) umma_commit(&sh.acc_full[buf]);
      }
      if (!ok) {
        *abort_flag = 1;
        set_status(p.status, MOE_DEV_WAIT_TIMEOUT);
      }
      // all MMAs issued by this thread have completed once `drained` fires
      umma_commit(&sh.drained);
      int no_abort = 0;  // wait for the MMAs even when unwinding
      if (!mbar_wait_bounded(&sh.drained, 0, &no_abort)) set_status(p.status, MOE_DEV_WAIT_TIMEOUT);
      sh.consumed = consumed;
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue --
    const int q = warp & 3;          // TMEM lane quadrant this warp may access
    const int r = q * 32 + lane;     // row of the 128-row tile
    int i = 0;
    for (int u = blockIdx.x; u < total_units; u += gridDim.x, ++i) {
      const Unit un = decode_unit(p, u);
      const bool shared = un.g == p.N;
      const uint32_t buf = i & 1, aph = (i >> 1) & 1;
      if (!mbar_wait_bounded(&sh.acc_full[buf], aph, abort_flag)) {
        *abort_flag = 1;
        set_status(p.status, MOE_DEV_WAIT_TIMEOUT);
        break;
      }
      tc_fence_after();
      const int row_in_group = un.m * kTcBM + r;
      const bool valid = row_in_group < __ldg(p.grp_rows + un.g);
      const int64_t row = shared ? row_in_group : (int64_t)__ldg(p.grp_row0 + un.g) + row_in_group;
      __nv_bfloat16* out = shared ? p.out_shared + row * p.ld_shared : p.out_routed + row * p.ld_routed;
      const int cols = shared ? p.cols_shared : p.cols_routed;
      const int col0 = un.f * p.bn;
      const uint32_t t_row = tmem_base + ((uint32_t)(q * 32) << 16) + buf * kAccCols;
      if (MODE == kSwiGLU) {
#pragma unroll 1
        for (int c = 0; c < 128; c += 32) {
          uint32_t gv[32], uv[32];
          tmem_ld32(t_row + c, gv);
          tmem_ld32(t_row + 128 + c, uv);
          tmem_wait_ld();
          float h[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) h[j] = silu_f32(__uint_as_float(gv[j])) * __uint_as_float(uv[j]);
          const int ncols = cols - (col0 + c);
          if (valid && ncols > 0) store_cols(out + col0 + c, ncols, h);
        }
      } else {
        const float gate = shared ? 1.0f : (valid ? __ldg(p.gate_perm + row) : 0.f);
#pragma unroll 1
        for (int c = 0; c < 256; c += 32) {
          uint32_t v[32];
          tmem_ld32(t_row + c, v);
          tmem_wait_ld();
          float o[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) o[j] = __uint_as_float(v[j]) * gate;
          const int ncols = cols - (col0 + c);
          if (valid && ncols > 0) store_cols(out + col0 + c, ncols, o);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh.acc_empty[buf]);
    }
  }

  __syncthreads();
  if (warp == 0 && lane == 0) {
    // wait for any stage fill that was issued but never observed complete
    for (uint32_t j = sh.consumed; j < fills; ++j) {
      const uint32_t s = j % kStages, ph = (j / kStages) & 1u;
      int dummy = 0;
      if (!mbar_wait_bounded(&sh.full[s], ph, &dummy)) {
        set_status(p.status, MOE_DEV_WAIT_TIMEOUT);
        break;
      }
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

// bf16 row-major [rows, cols] viewed as a 2-D tensor map with a box of
// 64 columns x box_rows rows and 128-byte swizzle. Rows/columns beyond the
// tensor read as zero.
bool make_tmap(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
  memset(m, 0, sizeof(*m));
  if (!base || rows == 0 || cols == 0) return true;  // never referenced
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {(cuuint32_t)kBK, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int MODE>
cudaError_t launch_one(const TcParams& prm, int grid, cudaStream_t s) {
  static int configured_device = -1;
  int dev = 0;
  cudaGetDevice(&dev);
  if (configured_device != dev) {
    cudaError_t e = cudaFuncSetAttribute(expert_gemm_tc_kernel<MODE>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    configured_device = dev;
  }
  expert_gemm_tc_kernel<MODE><<<grid, kThreads, kSmemBytes, s>>>(prm);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_expert_gemms_tc(const Problem& p, const GemmArgs& a, cudaStream_t s,
                                   cudaEvent_t between) {
  const int sms = device_sm_count();
  const int64_t mt_bound = (p.R + kTcBM - 1) / kTcBM + p.N + (p.ns > 0 ? (p.T + kTcBM - 1) / kTcBM : 0);

  TcParams g1{};
  bool ok = make_tmap(&g1.a_routed, a.x_perm, (uint64_t)p.R, p.d, kTcBM) &&
            make_tmap(&g1.a_shared, p.ns ? a.x : nullptr, (uint64_t)p.T, p.d, kTcBM) &&
            make_tmap(&g1.b0_routed, a.W1, (uint64_t)p.N * p.F, p.d, 128) &&
            make_tmap(&g1.b1_routed, a.W3, (uint64_t)p.N * p.F, p.d, 128) &&
            make_tmap(&g1.b0_shared, a.Ws1, (uint64_t)p.nsF, p.d, 128) &&
            make_tmap(&g1.b1_shared, a.Ws3, (uint64_t)p.nsF, p.d, 128);
  if (!ok) return cudaErrorInvalidValue;
  g1.unit_base = a.unit_base1;
  g1.grp_row0 = a.grp_row0;
  g1.grp_rows = a.grp_rows;
  g1.N = p.N;
  g1.k_routed = p.d;
  g1.k_shared = p.d;
  g1.cols_routed = p.F;
  g1.cols_shared = p.nsF;
  g1.b_rows_per_expert = p.F;
  g1.bn = kTcBN1;
  g1.out_routed = (__nv_bfloat16*)a.h_perm;
  g1.ld_routed = p.F;
  g1.out_shared = (__nv_bfloat16*)a.h_sh;
  g1.ld_shared = p.nsF;
  g1.gate_perm = nullptr;
  g1.status = a.status;
  const int64_t max_cols1 = p.F > p.nsF ? p.F : p.nsF;
  const int64_t units1 = mt_bound * ((max_cols1 + kTcBN1 - 1) / kTcBN1);
  const int grid1 = (int)(units1 < sms ? units1 : sms);
  cudaError_t err = launch_one<kSwiGLU>(g1, grid1 > 0 ? grid1 : 1, s);
  if (err == cudaSuccess && between) err = cudaEventRecord(between, s);
  if (err != cudaSuccess) return err;

  TcParams g2{};
  ok = make_tmap(&g2.a_routed, a.h_perm, (uint64_t)p.R, p.F, kTcBM) &&
       make_tmap(&g2.a_shared, p.ns ? a.h_sh : nullptr, (uint64_t)p.T, p.nsF, kTcBM) &&
       make_tmap(&g2.b0_routed, a.W2, (uint64_t)p.N * p.d, p.F, 256) &&
       make_tmap(&g2.b0_shared, a.Ws2, (uint64_t)p.d, p.nsF, 256);
  if (!ok) return cudaErrorInvalidValue;
  g2.unit_base = a.unit_base2;
  g2.grp_row0 = a.grp_row0;
  g2.grp_rows = a.grp_rows;
  g2.N = p.N;
  g2.k_routed = p.F;
  g2.k_shared = p.nsF;
  g2.cols_routed = p.d;
  g2.cols_shared = p.d;
  g2.b_rows_per_expert = p.d;
  g2.bn = kTcBN2;
  g2.out_routed = (__nv_bfloat16*)a.y_rows;
  g2.ld_routed = p.d;
  g2.out_shared = (__nv_bfloat16*)a.y_rows + p.R * (int64_t)p.d;
  g2.ld_shared = p.d;
  g2.gate_perm = a.gate_perm;
  g2.status = a.status;
  const int64_t nt2 = (p.d + kTcBN2 - 1) / kTcBN2;
  const int64_t units2 = mt_bound * nt2;
  const int grid2 = (int)(units2 < sms ? units2 : sms);
  return launch_one<kGateDown>(g2, grid2 > 0 ? grid2 : 1, s);
}

}  // namespace moe
