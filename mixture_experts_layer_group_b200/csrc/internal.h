// Host-side declarations shared by the library's translation units:
// validated problem description, workspace layout and kernel launchers.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/moe_b200.h"

namespace moe {

// Tile sizes of the tensor-core grouped GEMMs (rows x columns of one output
// tile) and of the fp32 SIMT grouped GEMMs.
constexpr int kTcBM = 128;      // token rows per tile (UMMA M)
constexpr int kTcBN1 = 128;     // SwiGLU GEMM: features per tile (g and u: UMMA N = 256)
constexpr int kTcBN2 = 256;     // down-projection GEMM: model columns per tile (UMMA N)
constexpr int kSimtBM = 64;
constexpr int kSimtBN = 64;
constexpr int kChunkTokens = 32;  // dispatch: tokens per warp chunk
constexpr int kMaxRouted = 512;
constexpr int kMaxTopK = 16;

struct Problem {
  int64_t T;
  int d, F, N, ns, k, G, TG;
  int score_fn, normalize, group_score, dtype;
  float route_scale;
  int64_t R;          // routed rows = T * k
  int nsF;            // shared MLP width
  int elem;           // bytes per element of x / weights / y
};

// Byte offsets of every workspace region (all 256-byte aligned).
struct Layout {
  size_t status, logits, idx, gates, chunk_counts, chunk_base, counts, offsets;
  size_t grp_row0, grp_rows, unit_base1, unit_base2, perm, slot_pos, gate_perm;
  size_t x_perm, h_perm, h_sh, y_rows, x_stage, y_stage;
  size_t total, total_host;
  int64_t n_chunks;
};

moe_status make_problem(const moe_cfg* cfg, int64_t T, Problem* p);
Layout make_layout(const Problem& p);

struct DispatchBuffers {
  const int32_t* idx;
  int32_t* chunk_counts;
  int32_t* chunk_base;
  int32_t* counts;
  int32_t* offsets;
  int32_t* grp_row0;
  int32_t* grp_rows;
  int32_t* unit_base1;
  int32_t* unit_base2;
  int32_t* perm;
  int32_t* slot_pos;
  float* gate_perm;
  const float* gates;
  unsigned* status;
};

// Router: logits (SIMT fp32) then selection.
cudaError_t launch_router(const Problem& p, const void* x, const void* W_r, const float* b,
                          float* logits, int32_t* idx, float* gates, cudaStream_t s);

// Histogram / scan / scatter; bm, bn1, bn2 select the GEMM tile grid that
// the unit tables describe.
cudaError_t launch_dispatch(const Problem& p, const DispatchBuffers& db, int bm, int bn1, int bn2,
                            cudaStream_t s);

// x_perm[r] = x[perm[r] / k]
cudaError_t launch_gather(const Problem& p, const void* x, const int32_t* perm,
                          const int32_t* n_rows, void* x_perm, cudaStream_t s);

struct GemmArgs {
  const void* x;        // [T, d]
  const void* x_perm;   // [R, d]
  const void* W1;       // [N, F, d]
  const void* W3;
  const void* W2;       // [N, d, F]
  const void* Ws1;      // [nsF, d]
  const void* Ws3;
  const void* Ws2;      // [d, nsF]
  void* h_perm;         // [R, F]
  void* h_sh;           // [T, nsF]
  void* y_rows;         // [R + T, d]
  const int32_t* grp_row0;
  const int32_t* grp_rows;
  const int32_t* unit_base1;
  const int32_t* unit_base2;
  const float* gate_perm;
  unsigned* status;
};

// Tensor-core (bf16) expert GEMMs: SwiGLU projection then gated down
// projection; `between` (optional) is recorded on s between the two launches.
cudaError_t launch_expert_gemms_tc(const Problem& p, const GemmArgs& a, cudaStream_t s,
                                   cudaEvent_t between);
// fp32 SIMT expert GEMMs.
cudaError_t launch_expert_gemms_simt(const Problem& p, const GemmArgs& a, cudaStream_t s,
                                     cudaEvent_t between);

// y[t] = sum over slots (ascending expert) of y_rows[slot_pos] + y_rows[R + t]
cudaError_t launch_combine(const Problem& p, const void* y_rows, const int32_t* slot_pos,
                           const int32_t* idx, void* y, cudaStream_t s);

int device_sm_count();

// Keeps e as this host thread's moe_last_cuda_error() value.
void record_cuda_error(cudaError_t e);

}  // namespace moe
