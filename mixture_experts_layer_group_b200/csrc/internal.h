// Host-side declarations shared by the library's translation units:
// validated problem description, workspace layout and kernel launchers.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/moe_b200.h"

namespace moe {

// Tile sizes of the tensor-core grouped GEMMs (run by CTA pairs): a unit
// covers at most kTcBM token rows of one group (UMMA N) and kTcBN1 SwiGLU
// features (two pair UMMAs of M = 256: W1 rows and the same W3 rows) or
// kTcBN2 model columns of the down projection (two pair UMMAs of M = 256).
// With FP8 weights a unit covers at most kTcBM8 token rows: its bf16 weight
// tiles live in tensor memory beside the accumulators.
// The fp32 SIMT GEMMs use 64 x 64 tiles.
constexpr int kTcBM = 256;
constexpr int kTcBM8 = 160;
constexpr int kTcBN1 = 256;
constexpr int kTcBN2 = 512;
constexpr int kSimtBM = 64;
constexpr int kSimtBN = 64;
constexpr int kChunkTokens = 32;  // dispatch: tokens per warp chunk
constexpr int kMaxRouted = 512;
constexpr int kMaxTopK = 16;
constexpr int kMaxDevices = 64;   // devices a process may use the library on

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
  size_t status, sched, logits, idx, gates, chunk_counts, chunk_base, counts, offsets;
  size_t grp_row0, grp_rows, unit_base1, unit_base2, perm, slot_pos, gate_perm;
  size_t x_perm, h_perm, h_sh, y_rows, x_stage[2], y_stage[2];
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
  int32_t* slot_pos;   // [T, k]: permuted rows of the token's experts, ascending expert
  float* gate_perm;
  const float* gates;
  unsigned* status;
};

// bf16 row-major [rows, cols] as a 2-D TMA tensor map with a box of
// box_cols x box_rows (128-byte swizzle and 256-byte L2 promotion when
// swizzle128, else dense). Elements outside the matrix load as zero; a null
// base or an empty matrix gives a zeroed map that must not be used.
bool make_tmap_bf16(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_cols,
                    uint32_t box_rows, bool swizzle128);
// uint8 row-major [rows, cols] (FP8 codes) with a box of box_cols bytes x
// box_rows rows, 256-byte L2 promotion, zero fill outside; swizzle_bytes 64
// gives the 64-byte swizzle (box_cols must then be 64), 0 none.
bool make_tmap_u8(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_cols,
                  uint32_t box_rows, int swizzle_bytes = 0);
// The same with a swizzle of 0, 64 or 128 bytes.
bool make_tmap_bf16_swz(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_cols,
                        uint32_t box_rows, int swizzle_bytes);

// Router: logits (FP32 pipes) then selection. The reduction over d is cut
// into S contiguous K ranges (S = `splits`, or router_k_splits(p) when
// splits is 0) whose partial logits land in S planes of [T, N] fp32 in
// `logits` (logits_bytes must cover them) and are added in a fixed order.
// A token's logits depend only on its own row, d and S, so every S gives
// deterministic bits and equal S gives equal bits at any T. `status` (may be
// null) receives MOE_DEV_* bits.
constexpr int kRouterTargetSms = 148;
int router_k_splits(const Problem& p);
size_t router_scratch_bytes(const Problem& p);
cudaError_t launch_router(const Problem& p, const void* x, const void* W_r, const float* b,
                          float* logits, size_t logits_bytes, int32_t* idx, float* gates,
                          unsigned* status, cudaStream_t s, int splits = 0);

// Histogram / scan / scatter; bm, bn1, bn2 select the GEMM tile grid that
// the unit tables describe.
cudaError_t launch_dispatch(const Problem& p, const DispatchBuffers& db, int bm, int bn1, int bn2,
                            cudaStream_t s);

// Unit tables of the grouped GEMMs straight from per-group row counts
// [p.N] (groups in order, rows contiguous): counts, offsets, grp_row0,
// grp_rows and unit bases in db; db.chunk_base needs p.N ints of scratch.
cudaError_t launch_unit_tables(const Problem& p, const int32_t* counts, const DispatchBuffers& db, int bm, int bn1,
                               int bn2, cudaStream_t s);

// Expert-parallel row reorder between source-major and expert-major order
// of the blocks counts[W, E] (see ep_reorder_kernel).
cudaError_t launch_ep_reorder(const int32_t* counts, int W, int E, int64_t row_bytes, const void* src, void* dst,
                              bool to_expert_major, cudaStream_t s);

// x_perm[slot_pos[t, s]] = x[t] for every placed (token, slot) pair
// (status: the workspace's device status word, for the debug build's bounds checks)
cudaError_t launch_gather(const Problem& p, const void* x, const int32_t* slot_pos, void* x_perm,
                          unsigned* status, cudaStream_t s);

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
  int* sched;           // [2] unit counters of the two tensor-core launches
  // FP8 expert weights: W1 .. Ws2 above hold the e4m3 codes (uint8, same
  // shapes) and these their UE8M0 scales, one byte per 128 x 128 block
  bool fp8 = false;
  const uint8_t* W1s = nullptr;
  const uint8_t* W3s = nullptr;
  const uint8_t* W2s = nullptr;
  const uint8_t* Ws1s = nullptr;
  const uint8_t* Ws3s = nullptr;
  const uint8_t* Ws2s = nullptr;
};

// Tensor-core (bf16) expert GEMMs: SwiGLU projection then gated down
// projection. `between` (optional) is recorded on s between the two
// launches; without it the down projection is launched with programmatic
// dependent launch and overlaps the SwiGLU GEMM's drain.
cudaError_t launch_expert_gemms_tc(const Problem& p, const GemmArgs& a, cudaStream_t s,
                                   cudaEvent_t between);
// fp32 SIMT expert GEMMs.
cudaError_t launch_expert_gemms_simt(const Problem& p, const GemmArgs& a, cudaStream_t s,
                                     cudaEvent_t between);

// y[t] = sum over the token's rows slot_pos[t, 0..k) (ascending expert) of
// y_rows, plus the shared row y_rows[R + t]
cudaError_t launch_combine(const Problem& p, const void* y_rows, const int32_t* slot_pos, void* y,
                           cudaStream_t s);
// The same with the routed rows [R, d] and the shared rows [T, d] (or null) apart.
cudaError_t launch_combine_rows(const Problem& p, const void* routed_rows, const void* shared_rows,
                                const int32_t* slot_pos, void* y, cudaStream_t s);

int device_sm_count();

// Keeps e as this host thread's moe_last_cuda_error() value.
void record_cuda_error(cudaError_t e);

}  // namespace moe
