// Grouped expert GEMMs on the 5th-generation tensor cores (tcgen05 + TMEM,
// operands staged by TMA), run by CTA pairs (clusters of 2) with pair UMMAs
// (cta_group::2) in "weights as M" orientation. Every pair MMA takes 256
// weight rows as its A operand (128 in each CTA's shared memory, M = 256)
// and the group's token rows as B (N = the tokens of the unit rounded up to
// 16, at most 256, half of them in each CTA), so each SM streams its own
// weight rows but only half of the token rows, and the MMA work follows the
// real number of tokens per expert instead of a padded row tile. A unit
// issues two pair MMAs (its two 128-row A halves per CTA) per K step on one
// shared token tile. Two launches per layer:
//
//   SwiGLU GEMM  unit = (group, 256 features, <= 256 tokens): CTA r holds
//                features 128 r .. 128 r + 127 of the unit; half 0 of its
//                rows is W1, half 1 the same rows of W3, so TMEM lane i holds
//                g and u of one feature for every token column; epilogue
//                h = silu(g) * u -> bf16
//                ("Routed expert:" / "Shared expert:" steps g = x W1,
//                u = x W3, a = g sigma(g), h = a (.) u)
//   gate GEMM    unit = (group, 512 model columns, <= 256 tokens):
//                E^T = W2 h^T; epilogue E * G (the token slot's gate; 1 for
//                the shared MLP) -> bf16 row of the slot
//                ("E_i = h W2", "y_routed = sum G_i E_i")
//
// Groups 0..N-1 are the routed experts over their expert-contiguous token
// rows; group N is the fused shared MLP over all T tokens, in the same
// persistent launch. A group of more than 256 rows is cut into equal chunks.
// Units of one group are consecutive, weight-tile major and token-chunk
// minor. The pair's first CTA takes units from a global counter, so the
// chunks that share a weight tile start together (they read it once through
// L2) and the last units balance across SMs. The gate GEMM is launched with
// programmatic stream serialization and waits for the SwiGLU grid before its
// first load.
//
// CTA roles (320 threads, one CTA per SM, persistent; the same roles in both
// CTAs of a pair except the MMA issuer, which only the first CTA has):
//   warp 0      TMA producer (one lane). In CTA 0 it also takes unit ids and
//               hands them to both CTAs through shared-memory rings (the
//               peer's by an asynchronous store, see below). Stages
//               are variable-size pieces of a 208 KB byte ring: per 64-wide
//               K block, 32 KB of weights (two 128-row boxes) and one token
//               box of 32, 64 or 128 rows (4 / 8 / 16 KB; the TMA engine's
//               cost is per box); the bytes of both CTAs complete on CTA 0's
//               stage barrier; weights read by one unit only are evict-first
//   warp 1      TMEM owner (both CTAs, pair allocation) + UMMA issuer (CTA 0,
//               one lane): 2 x 4 pair MMAs (256 x N x 16) per stage. Each
//               CTA's TMEM holds two buffers of 2 x 128 fp32 columns: a unit
//               of <= 128 tokens takes one buffer (the next unit's MMAs
//               overlap its epilogue), a larger unit takes both (2 x 256)
//   warps 2..9  epilogue, two warps per TMEM lane quadrant taking turns on
//               32-token blocks: each warp reads its quadrant in the m16n8
//               layout (tcgen05.ld 16x256b), applies SwiGLU or the gate,
//               transposes the 32 x 32 block into its own 64-byte-swizzled
//               shared-memory tile with stmatrix.trans and writes it with one
//               TMA tensor store (a ragged last block with 64-byte row
//               stores); no barrier between epilogue warps per block
// With FP8 (e4m3) weights the same kernel runs 448 threads: the producer
// loads the codes (64-byte swizzled rows) and the token box into the ring,
// eight converter warps (one per TMEM lane quadrant and weight half)
// dequantise each stage's codes exactly into bf16 in tensor memory, and the
// pair MMAs read A from there and B from the ring (kind::f16 as above); four
// epilogue warps, one per quadrant.
// Every signal from one CTA of the pair to the other (a unit id, the
// release of a unit-ring slot or of an accumulator, an FP8 slot report) is
// an asynchronous store that completes transaction bytes on the receiving
// CTA's mbarrier (st.async), so no thread waits for a cross-CTA arrive; the
// MMA commits reach both CTAs' barriers by multicast.
// Every mbarrier wait is bounded; on a timeout a CTA records
// MOE_DEV_WAIT_TIMEOUT, drains its own copies and MMAs (bounded again),
// frees its tensor memory and exits.

#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int kSlots = 8;                         // stages in flight at most
constexpr int kBK = 64;                           // bf16 per K chunk: one 128 B swizzle row
constexpr int kMaxTok = kTcBM;                    // tokens per unit (<= 256)
constexpr int kTokBox = 32;                       // token-row granule of a stage
constexpr int kBoxBytes = kTokBox * kBK * 2;      // 4 KB
constexpr int kTokMaps = 3;                       // token boxes of 32, 64 and 128 rows
constexpr int kHalfBytes = 128 * kBK * 2;         // 16 KB: 128 weight rows of one half
constexpr int kATileBytes = 2 * kHalfBytes;       // 32 KB: this CTA's rows of both halves
constexpr int kMaxTokBytes = (kMaxTok / 2 / kTokBox) * kBoxBytes;  // 16 KB: a CTA's largest token box
constexpr int kMaxStageBytes = kATileBytes + kMaxTokBytes;          // 48 KB
constexpr int kTmemCols = 512;                    // the pair allocation in each CTA
constexpr int kRing = 8;                          // unit ids in flight between the roles
constexpr int kTileBytes = 32 * 32 * 2;           // a warp's dense 32 x 32 bf16 tile (TMA store box)
constexpr int kA8Bytes = 2 * 128 * kBK;           // 16 KB: the fp8 codes of a CTA's 256 weight rows x 64 K
constexpr int kFp8Block = 128;                    // FP8 scale block (rows and columns)
constexpr int kASlots = 3;                        // FP8: dequantised weight stages in tensor memory
constexpr int kASlotCols = 2 * kBK / 2;           // FP8: columns of one slot (two halves x 64 bf16 / 2)

// Shared-memory and tensor-memory plan. bf16 weights: one ring of
// variable-size stages (this CTA's 256 weight rows x 64 K in bf16, then the
// token box), which the MMAs read in place; TMEM holds two accumulator
// buffers of 256 columns. FP8 weights: the ring holds the fp8 codes (16 KB,
// 64-byte swizzled rows) and the token box; the converter warps dequantise
// each stage's codes in registers into one of two weight slots in tensor
// memory (three slots, columns 320..511), from which the pair MMAs take A
// (B, the token box, stays in the ring); the accumulators share columns
// 0..319, so a unit covers at most 160 tokens.
template <bool FP8>
struct Plan;
template <>
struct Plan<false> {
  static constexpr int kEpiWarps = 8;            // two per TMEM lane quadrant
  static constexpr int kCvtWarps = 4;            // (no converters; 4 keeps the arithmetic defined)
  static constexpr int kThreads = 64 + 32 * kEpiWarps;
  static constexpr int kRingBytes = 52 * 4096;   // 208 KB
  static constexpr int kABytes = kATileBytes;    // weight bytes at the head of a stage
  static constexpr int kChunk = kTcBM;           // token rows of a unit at most
  static constexpr int kTokAlign = 16;           // MMA N granule
  static constexpr uint32_t kAccCols = 512;      // accumulator columns: two buffers of 256
  static constexpr int kBarrierBytes = 512;
};
template <>
struct Plan<true> {
  static constexpr int kEpiWarps = 4;            // one per TMEM lane quadrant
  static constexpr int kCvtWarps = 8;            // two per TMEM lane quadrant: one per weight half
  static constexpr int kThreads = 64 + 32 * (kEpiWarps + kCvtWarps);
  static constexpr int kRingBytes = 54 * 4096;   // 216 KB
  static constexpr int kABytes = kA8Bytes;
  static constexpr int kChunk = kTcBM8;
  static constexpr int kTokAlign = 32;           // N of an MMA with A in tensor memory
  static constexpr uint32_t kAccCols = 320;      // two buffers of 160; then the weight slots
  static constexpr int kBarrierBytes = 1024;
};
template <bool FP8>
__host__ __device__ constexpr int tile_bytes() {
  return Plan<FP8>::kEpiWarps * kTileBytes;  // one transpose tile per epilogue warp
}
template <bool FP8>
constexpr int smem_bytes() {
  return Plan<FP8>::kRingBytes + tile_bytes<FP8>() + 1024 + Plan<FP8>::kBarrierBytes;
}
static_assert(smem_bytes<false>() <= 232448 && smem_bytes<true>() <= 232448, "shared memory budget");
static_assert(kMaxStageBytes * 3 <= Plan<false>::kRingBytes, "ring holds three full stages");
static_assert((kA8Bytes + kMaxTokBytes) * 4 <= Plan<true>::kRingBytes, "FP8 ring holds four full stages");
static_assert(Plan<false>::kEpiWarps % 4 == 0 && Plan<true>::kEpiWarps % 4 == 0, "whole quadrants");
static_assert(Plan<true>::kCvtWarps == 8, "one converter warp per (TMEM lane quadrant, weight half)");
static_assert(2 * Plan<false>::kChunk <= (int)Plan<false>::kAccCols && 2 * Plan<true>::kChunk <= (int)Plan<true>::kAccCols &&
                  Plan<true>::kAccCols % 64 == 0 &&
                  Plan<true>::kAccCols + kASlots * kASlotCols <= (uint32_t)kTmemCols,
              "accumulators and weight slots fit the tensor memory");
static_assert(kMaxTok % (2 * kTokBox) == 0 && Plan<false>::kChunk <= kMaxTok && Plan<true>::kChunk <= kMaxTok &&
                  Plan<true>::kChunk % Plan<true>::kTokAlign == 0,
              "token chunk");

enum Mode : int { kSwiGLU = 0, kGateDown = 1 };

struct TcParams {
  // bf16 weights: bf16 maps of 64 x 128 boxes (128-byte swizzle; the down
  // GEMM's A maps have 256-row boxes). FP8 weights: uint8 maps of the e4m3
  // codes, 64-byte x 128-row boxes (256 rows for the down GEMM), unswizzled.
  CUtensorMap a0_routed;  // W1 [N*F, d]      | W2 [N*d, F]
  CUtensorMap a1_routed;  // W3 [N*F, d]      | unused
  CUtensorMap a0_shared;  // Ws1 [nsF, d]     | Ws2 [d, nsF]
  CUtensorMap a1_shared;  // Ws3 [nsF, d]     | unused
  CUtensorMap b_routed[kTokMaps];  // x_perm [R, d] | h_perm [R, F]   (boxes of 32 / 64 / 128 rows)
  CUtensorMap b_shared[kTokMaps];  // x [T, d]      | h_sh [T, nsF]
  CUtensorMap o_routed;   // h_perm [R, F]    | y_rows [R + T, d]   (32 x 32 store box)
  CUtensorMap o_shared;   // h_sh [T, nsF]    | y_rows [R + T, d]
  const int32_t* unit_base;  // [N + 2]: units before group g; [N + 1] = total
  const int32_t* grp_row0;   // [N + 1]
  const int32_t* grp_rows;   // [N + 1]
  int* sched;                // unit counter, zero at launch
  int N;
  int k_routed, k_shared;        // reduction length (d | F, d | nsF)
  int cols_routed, cols_shared;  // output columns (F, nsF | d, d)
  int a_rows_per_expert;         // rows of the stacked weight tensor per routed expert (F | d)
  int tile_cols;                 // output columns per unit (256 | 512)
  __nv_bfloat16* out_routed;
  int64_t ld_routed;
  __nv_bfloat16* out_shared;
  int64_t ld_shared;
  int out_row0_shared;           // first row of the shared MLP's rows in o_shared (0 | R)
  const float* gate_perm;        // [R] (gate-down mode)
  unsigned* status;
  // FP8 weights: UE8M0 block scales [rows / 128, K / 128] of a0 / a1 (routed,
  // shared), and the number of 128-row blocks of each (for clamping)
  const uint8_t* s0_routed;
  const uint8_t* s1_routed;
  const uint8_t* s0_shared;
  const uint8_t* s1_shared;
  int sblocks_routed, sblocks_shared;
  int chunk_rows;                // token rows of a unit at most (Plan::kChunk)
  // rows of the token operand, weight and output tensors (routed | shared
  // group), for the debug build's bounds checks
  int64_t tok_rows_routed, tok_rows_shared;
  int64_t a_rows_routed, a_rows_shared;
  int64_t out_rows_routed, out_rows_shared;
};

struct Unit {
  int g;        // group (N = shared MLP)
  int f;        // output-column tile
  int tok0;     // first token row of the chunk within the group
  int ntok;     // tokens in the chunk (1..256)
  int nchunks;  // chunks of the group
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
  // a group's rows split into nc chunks of (almost) equal size, so the
  // chunks that share a weight tile run at the same pace and keep reading
  // its lines from L2 together
  const int nc = (rows + p.chunk_rows - 1) / p.chunk_rows;
  const int cs = (rows + nc - 1) / nc;
  Unit un;
  un.g = lo;
  un.f = local / nc;
  un.tok0 = (local % nc) * cs;
  const int left = rows - un.tok0;
  un.ntok = left < cs ? left : cs;
  un.nchunks = nc;
  return un;
}

// Accumulator placement over kCols columns (identical in both CTAs), by the
// unit's MMA width n (its tokens rounded up to the N granule): a unit with
// n <= kHalf (kCols / 4 rounded down to 32 columns) takes one of two
// buffers, at 0 or kCols / 2 (its halves at base and base + kHalf), so the
// next unit's MMAs overlap its epilogue; a wider unit takes both (halves at
// 0 and kCols / 2). bf16 (512 columns): buffers for n <= 128; FP8 (320):
// n <= 64. The MMA issuer and every epilogue thread replay the same
// sequence, so they agree on every placement.
template <uint32_t kCols>
struct AccPlan {
  static constexpr uint32_t kHalf = (kCols / 4) & ~31u;
  uint32_t next = 0;
  MOE_DEV void place(int n, uint32_t& mask, uint32_t& base, uint32_t& stride) const {
    if (n > (int)kHalf) {
      mask = 3u;
      base = 0;
      stride = kCols / 2;
    } else {
      mask = 1u << next;
      base = next * (kCols / 2);
      stride = kHalf;
    }
  }
  MOE_DEV void advance(int n) { next = n > (int)kHalf ? 0u : next ^ 1u; }
};
// MMA width (N) of a unit of ntok tokens.
template <bool FP8>
MOE_DEV int mma_n(int ntok) { return (ntok + Plan<FP8>::kTokAlign - 1) & ~(Plan<FP8>::kTokAlign - 1); }

struct Shared {
  uint64_t full[kSlots];       // CTA 0: stage bytes of both CTAs landed
  uint64_t empty[kSlots];      // both: the pair MMAs finished reading the stage
  uint64_t acc_full[2];        // both: accumulator buffer complete
  uint64_t acc_empty[2];       // CTA 0: both CTAs' epilogues released the buffer (CTA 0's epilogue
                               // warps arrive, CTA 1's complete 4 transaction bytes each)
  uint64_t ring_full[kRing];   // both: unit id published
  uint64_t ring_empty[kRing];  // CTA 0: every reader of the pair took the id (CTA 0's readers
                               // arrive, CTA 1's complete 4 transaction bytes each)
  uint64_t drained;            // both: all pair MMAs completed
  uint32_t slot_off[kSlots];   // byte offset of each stage in the ring
  int ring[kRing];
  int epi_unit[2];             // the epilogue leader's unit for the epilogue warps
  int epi_info[2][5];          // its decoded (g, f, tok0, ntok) and first output row
  uint32_t tmem_base;
  int abort_flag;
  uint32_t consumed;           // stage fills the MMA issuer observed complete
  uint32_t sink;               // CTA 0: target of CTA 1's signalling stores (never read)
};
static_assert(sizeof(Shared) <= 512, "barrier block");

// The FP8 path's extra state (after Shared, inside the barrier block).
struct SharedFp8 {
  uint64_t conv_full[kASlots];   // CTA 0: both CTAs' converters wrote the weight slot in TMEM (CTA 0's
                                 // converters arrive, CTA 1's complete 4 transaction bytes)
  uint64_t conv_empty[kASlots];  // both: the pair MMAs finished reading the slot
  int cvt_unit[2];             // the converter leader's unit for the converter warps
  int cvt_info[2][2];          // its (g, f)
  int cvt_ok;                  // the leader's waits for the current stage succeeded
  uint32_t seen;               // stage fills this CTA's converters observed complete
  uint32_t peer_word[kASlots];   // CTA 0: target of CTA 1's signalling stores (never read)
};
static_assert(512 + sizeof(SharedFp8) <= Plan<true>::kBarrierBytes, "FP8 barrier block");

// Barrier among the epilogue warps only (id 1; id 0 is __syncthreads).
template <int kWarps>
MOE_DEV void epi_sync() { asm volatile("bar.sync 1, %0;" ::"n"(32 * kWarps) : "memory"); }
// Barrier among the FP8 converter warps only (id 2).
template <int kWarps>
MOE_DEV void cvt_sync() { asm volatile("bar.sync 2, %0;" ::"n"(32 * kWarps) : "memory"); }

// Two e4m3 codes (bytes i and i + 1 of w, i = 0 or 2) -> the bf16 pair of
// their values times 2^-120. For a code s eeee mmm the bf16 bit pattern
// s 0000 eeee mmm 0000 has exponent field e and mantissa m / 8, i.e. the
// value 2^(e - 127) (1 + m / 8) for e > 0 and the bf16 subnormal 2^-126 m / 8
// for e = 0 (e4m3: 2^(e - 7) (1 + m / 8) and 2^-6 m / 8), and zero stays zero.
// One byte permute spreads the two codes into 16-bit lanes with the sign
// replicated into each high byte; a shift and a mask place the fields.
template <int kSel>
MOE_DEV uint32_t e4m3x2_to_bf16x2_scaled(uint32_t w) {
  uint32_t t;
  asm("prmt.b32 %0, %1, 0, %2;" : "=r"(t) : "r"(w), "n"(kSel));
  return (t << 4) & 0x87F087F0u;
}

MOE_DEV uint32_t mul_bf16x2(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

// bf16 pair (f, f) with f = 2^e, -126 <= e <= 127.
MOE_DEV uint32_t bf16x2_pow2(int e) {
  const uint32_t b = (uint32_t)(e + 127) << 7;
  return b | (b << 16);
}

// 16 e4m3 codes -> 16 bf16 values, each code value times 2^(sb - 127):
// the values times 2^-120, multiplied by 2^(sb - 7) in one or (for
// sb - 7 > 127) two exact steps (a power of two times a bf16 with 4
// significant bits, subnormal or not, lands on a normal bf16).
MOE_DEV void dequant16(const uint4 w, int sb, uint32_t (&o)[8]) {
  const int e = sb - 7;                     // exponent of the total factor (>= -7)
  const int e1 = e > 127 ? 127 : e;
  const uint32_t f1 = bf16x2_pow2(e1);
  const uint32_t words[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    // bytes [b0, sign b0, b1, sign b1] and [b2, sign b2, b3, sign b3]
    o[2 * i] = mul_bf16x2(e4m3x2_to_bf16x2_scaled<0x9180>(words[i]), f1);
    o[2 * i + 1] = mul_bf16x2(e4m3x2_to_bf16x2_scaled<0xB3A2>(words[i]), f1);
  }
  if (e > 127) {
    const uint32_t f2 = bf16x2_pow2(e - 127);
#pragma unroll
    for (int i = 0; i < 8; ++i) o[i] = mul_bf16x2(o[i], f2);
  }
}

MOE_DEV int load_volatile(const int* p) { return *reinterpret_cast<const volatile int*>(p); }

// Writes one 64-byte token-row segment (32 bf16 from the transpose tile),
// or the first ncols of it at a ragged right edge.
MOE_DEV void store_row32(__nv_bfloat16* dst, int ncols, const uint4 (&v)[4]) {
  if (ncols >= 32) {
    uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
    for (int c = 0; c < 4; ++c) d4[c] = v[c];
  } else {
    const __nv_bfloat16* e = reinterpret_cast<const __nv_bfloat16*>(v);
#pragma unroll
    for (int c = 0; c < 32; ++c)
      if (c < ncols) dst[c] = e[c];
  }
}

template <int MODE, bool FP8>
__global__ void __launch_bounds__(Plan<FP8>::kThreads, 1) expert_gemm_tc_kernel(const __grid_constant__ TcParams p) {
  using PL = Plan<FP8>;
  constexpr int kRingBytes = PL::kRingBytes;
  constexpr int kEpiWarps = PL::kEpiWarps, kCvtWarps = PL::kCvtWarps, kTBytes = tile_bytes<FP8>();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float* tiles = reinterpret_cast<float*>(smem + kRingBytes);
  Shared& sh = *reinterpret_cast<Shared*>(reinterpret_cast<uint8_t*>(tiles) + kTBytes);
  SharedFp8& shf = *reinterpret_cast<SharedFp8*>(reinterpret_cast<uint8_t*>(&sh) + 512);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();  // 0: issues the pair MMAs and takes the units
  const bool first = rank == 0;
  const int total_units = __ldg(p.unit_base + p.N + 1);
  // Weight rows of this CTA. SwiGLU: rows 128 r .. 128 r + 127 of the unit's
  // 256 features, taken from W1 (half 0) and from W3 (half 1). Down GEMM:
  // rows 256 r .. 256 r + 255 of the unit's 512 output columns, one
  // contiguous 256-row box whose first and second 128 rows are halves 0 and
  // 1; so TMEM lane l of half h in CTA r is output column 256 r + 128 h + l.
  const int rank_rows = (MODE == kSwiGLU ? 128 : 256) * (int)rank;
  // Readers of each unit id in each CTA (producer or MMA issuer, epilogue
  // leader, FP8 converter leader). The pair's cross-CTA signals are
  // asynchronous stores that complete transaction bytes on the other CTA's
  // barrier (st.async): a blocking cluster-scope mbarrier arrive costs the
  // signalling thread about 1000 cycles.
  constexpr int kRingReaders = FP8 ? 3 : 2;
  const int half_cols = MODE == kSwiGLU ? 0 : 128;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kSlots; ++s) {
      mbar_init(&sh.full[s], 1);
      mbar_init(&sh.empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sh.acc_full[b], 1);
      mbar_init(&sh.acc_empty[b], kEpiWarps);
    }
    for (int q = 0; q < kRing; ++q) {
      mbar_init(&sh.ring_full[q], 1);
      // CTA 0's readers: MMA issuer, epilogue leader (and FP8 converter leader)
      mbar_init(&sh.ring_empty[q], kRingReaders);
    }
    mbar_init(&sh.drained, 1);
    sh.abort_flag = 0;
    sh.consumed = 0;
    if (FP8) {
      for (int c = 0; c < kASlots; ++c) {
        mbar_init(&shf.conv_full[c], 1);
        mbar_init(&shf.conv_empty[c], 1);
      }
      shf.seen = 0;
    }
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&p.a0_routed);
    for (int m = 0; m < kTokMaps; ++m) tma_prefetch_desc(&p.b_routed[m]);
    if (MODE == kSwiGLU) tma_prefetch_desc(&p.a1_routed);
  }
  if (warp == 1) {
    tmem_alloc_pair(&sh.tmem_base, kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();  // barriers and tensor memory of both CTAs are ready
  tc_fence_after();
  const uint32_t tmem_base = sh.tmem_base;
  volatile int* abort_flag = &sh.abort_flag;
  auto peer = [&](const void* local) { return map_to_rank(smem_u32(local), rank ^ 1u); };
  auto in_first = [&](const void* local) { return map_to_rank(smem_u32(local), 0u); };

  uint32_t fills = 0;  // producer: stage fills issued
  if (warp == 0) {
    // ------------------------------------------------- scheduler + producer --
    if (lane == 0) {
      // the down GEMM may start while the SwiGLU GEMM drains (programmatic
      // launch): nothing it loads may be read before that grid has finished
      if (MODE == kGateDown) griddep_wait();
      // a weight tile read by one unit only is streamed once: evict it first;
      // tiles shared by the chunks of a large group, and the token rows (read
      // by every feature tile of their group), are kept in L2 as long as possible
      const uint64_t pol_once = policy_evict_first();
      const uint64_t pol_last = policy_evict_last();
      // Ring allocation (identical in both CTAs, so stage offsets match).
      // Stages are placed back to back in fill order and freed in the same
      // order by the pair MMAs' commits, so the bytes in use form one circular
      // interval [offset of the oldest unfreed fill, head). A stage that does
      // not fit before the end restarts at 0.
      uint32_t off_of[kSlots];
      uint32_t head = 0, oldest = 0;
      auto acquire = [&](uint32_t j, uint32_t sz, uint32_t& pos) -> bool {
        for (;;) {
          const uint32_t inflight = j - oldest;
          bool fits = false;
          if (inflight == 0) {
            pos = head + sz <= (uint32_t)kRingBytes ? head : 0u;
            fits = true;
          } else if (inflight < (uint32_t)kSlots) {
            const uint32_t tail = off_of[oldest % kSlots];
            if (tail < head) {  // in use: [tail, head)
              if (head + sz <= (uint32_t)kRingBytes) {
                pos = head;
                fits = true;
              } else if (sz <= tail) {
                pos = 0;
                fits = true;
              }
            } else if (head + sz <= tail) {  // in use wraps: [tail, end) + [0, head)
              pos = head;
              fits = true;
            }
          }
          if (fits) return true;
          // wait for the oldest fill to be consumed
          if (!mbar_wait_cluster_bounded(&sh.empty[oldest % kSlots], (oldest / kSlots) & 1u, abort_flag))
            return false;
          ++oldest;
        }
      };
      bool ok = true;
      for (int i = 0;; ++i) {
        const int q = i % kRing;
        int u;
        if (first) {
          if (!mbar_wait_cluster_bounded(&sh.ring_empty[q], ((i / kRing) & 1) ^ 1, abort_flag)) {
            ok = false;
            break;
          }
          u = atomicAdd(p.sched, 1);
          if (u >= total_units) u = -1;
          sh.ring[q] = u;
          mbar_arrive(&sh.ring_full[q]);
          // the id itself is the 4 transaction bytes of the peer's ring_full
          st_async_u32(peer(&sh.ring[q]), (uint32_t)u, peer(&sh.ring_full[q]));
        } else {
          // this CTA's ring_full phase: one arrival (here) and the 4 bytes of CTA 0's store
          mbar_arrive_expect_tx(&sh.ring_full[q], 4);
          if (!mbar_wait_cluster_bounded(&sh.ring_full[q], (i / kRing) & 1, abort_flag)) {
            ok = false;
            break;
          }
          u = load_volatile(&sh.ring[q]);
          st_async_u32(in_first(&sh.sink), 0u, in_first(&sh.ring_empty[q]));
        }
        if (u < 0) {
          // no units left for this CTA: the down GEMM may start on SMs as
          // they free up
          if (MODE == kSwiGLU) griddep_launch_dependents();
          break;
        }
        const Unit un = decode_unit(p, u);
        const bool shared = un.g == p.N;
        const int K = shared ? p.k_shared : p.k_routed;
        const int nk = (K + kBK - 1) / kBK;
        const int half_n = mma_n<FP8>(un.ntok) / 2;  // token rows per CTA
        // one token box per stage, the smallest of 32 / 64 / 128 rows that
        // covers this CTA's rows (the TMA engine's cost is per box, so a
        // single box beats several small ones even with rows to spare)
        const int tmap = half_n <= kTokBox ? 0 : (half_n <= 2 * kTokBox ? 1 : 2);
        const int nbox = 1 << tmap;  // in 32-row granules
        const uint32_t tx = PL::kABytes + nbox * kBoxBytes;
        const int rowA = (shared ? 0 : un.g * p.a_rows_per_expert) + un.f * p.tile_cols + rank_rows;
        const int rowB = __ldg(p.grp_row0 + un.g) + un.tok0 + (int)rank * half_n;
        // the unit's rows lie inside the group and its tensors (TMA clips a
        // box that reaches past them, and the last column tile of a matrix
        // whose height is not a multiple of the tile may start past it)
        (void)MOE_IN_BOUNDS(un.ntok >= 1 && un.ntok <= p.chunk_rows && un.tok0 >= 0 &&
                                __ldg(p.grp_row0 + un.g) + un.tok0 + un.ntok <=
                                    (shared ? p.tok_rows_shared : p.tok_rows_routed) &&
                                rowA >= 0 && rowA < (shared ? p.a_rows_shared : p.a_rows_routed) + p.tile_cols,
                            p.status);
        const CUtensorMap* ta0 = shared ? &p.a0_shared : &p.a0_routed;
        const CUtensorMap* ta1 = MODE == kSwiGLU ? (shared ? &p.a1_shared : &p.a1_routed) : ta0;
        const CUtensorMap* tb = shared ? &p.b_shared[tmap] : &p.b_routed[tmap];
        const uint64_t pol = un.nchunks == 1 ? pol_once : pol_last;
        for (int kc = 0; kc < nk; ++kc, ++fills) {
          const uint32_t s = fills % kSlots;
          uint32_t pos = 0;
          if (!acquire(fills, tx, pos)) {
            ok = false;
            break;
          }
          off_of[s] = pos;
          head = pos + tx;
          (void)MOE_IN_BOUNDS(pos + tx <= (uint32_t)kRingBytes, p.status);
          sh.slot_off[s] = pos;
          uint8_t* a_dst = smem + pos;
          uint8_t* b_dst = a_dst + PL::kABytes;
          if (FP8) {
            // every CTA's bytes complete on its own stage barrier, which its
            // converter warps wait on; the codes are 64 bytes per row
            mbar_arrive_expect_tx(&sh.full[s], tx);
            tma_load_2d_hint(a_dst, ta0, &sh.full[s], kc * kBK, rowA, pol);
            if (MODE == kSwiGLU) tma_load_2d_hint(a_dst + kA8Bytes / 2, ta1, &sh.full[s], kc * kBK, rowA, pol);
            tma_load_2d_hint(b_dst, tb, &sh.full[s], kc * kBK, rowB, pol_last);
          } else {
            const uint32_t full_bar = in_first(&sh.full[s]);
            if (first) mbar_arrive_expect_tx(&sh.full[s], 2 * tx);  // this CTA's bytes and the peer's
            tma_load_2d_pair(a_dst, ta0, full_bar, kc * kBK, rowA, pol);  // SwiGLU: 128 W1 rows; down: 256 rows
            if (MODE == kSwiGLU) tma_load_2d_pair(a_dst + kHalfBytes, ta1, full_bar, kc * kBK, rowA, pol);
            tma_load_2d_pair(b_dst, tb, full_bar, kc * kBK, rowB, pol_last);
          }
        }
        if (!ok) break;
      }
      if (!ok) {
        *abort_flag = 1;
        set_status(p.status, MOE_DEV_WAIT_TIMEOUT);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------- MMA issuer (CTA 0) --
    if (lane == 0 && first) {
      uint32_t consumed = 0;
      uint32_t uses[2] = {0u, 0u};
      AccPlan<PL::kAccCols> plan;
      bool ok = true;
      for (int i = 0; ok; ++i) {
        const int q = i % kRing;
        if (!mbar_wait_cluster_bounded(&sh.ring_full[q], (i / kRing) & 1, abort_flag)) {
          ok = false;
          break;
        }
        const int u = load_volatile(&sh.ring[q]);
        mbar_arrive_expect_tx(&sh.ring_empty[q], 4 * kRingReaders);  // and CTA 1's readers' stores
        if (u < 0) break;
        const Unit un = decode_unit(p, u);
        const int K = un.g == p.N ? p.k_shared : p.k_routed;
        const int nk = (K + kBK - 1) / kBK;
        const int n = mma_n<FP8>(un.ntok);
        const uint32_t idesc = idesc_bf16_f32(256, (uint32_t)n);
        uint32_t mask, base, stride;
        plan.place(n, mask, base, stride);
        (void)MOE_IN_BOUNDS(n <= p.chunk_rows + PL::kTokAlign && base + stride + n <= PL::kAccCols, p.status);
        plan.advance(n);
        for (int b = 0; b < 2 && ok; ++b)
          if ((mask >> b) & 1u) {
            ok = mbar_wait_cluster_bounded(&sh.acc_empty[b], (uses[b] & 1u) ^ 1u, abort_flag);
            ++uses[b];
          }
        if (!ok) break;
        tc_fence_after();
        const uint32_t d0 = tmem_base + base, d1 = tmem_base + base + stride;
        for (int kc = 0; kc < nk; ++kc) {
          const uint32_t s = consumed % kSlots, ph = (consumed / kSlots) & 1u;
          // FP8: the converted slot of this fill (both CTAs' converters have
          // observed its bytes land before they released it)
          const uint32_t c = FP8 ? consumed % kASlots : 0u;
          const bool landed = FP8 ? mbar_wait_cluster_bounded(&shf.conv_full[c], (consumed / kASlots) & 1u, abort_flag)
                                  : mbar_wait_cluster_bounded(&sh.full[s], ph, abort_flag);
          if (!landed) {
            ok = false;
            break;
          }
          ++consumed;
          tc_fence_after();
          const uint32_t stage_addr = smem_u32(smem + *reinterpret_cast<volatile uint32_t*>(&sh.slot_off[s]));
          const uint32_t b_addr = stage_addr + PL::kABytes;  // the token box follows the weights
          if (FP8) {
            // A: the converted slot in tensor memory, 8 columns per 16 K
            const uint32_t a_t = tmem_base + PL::kAccCols + c * kASlotCols;
#pragma unroll
            for (int kk = 0; kk < kBK / 16; ++kk) {
              const uint64_t bdesc = smem_desc_sw128(b_addr + kk * 32);
              umma_bf16_pair_ts(d0, a_t + kk * 8, bdesc, idesc, (kc | kk) != 0);
              umma_bf16_pair_ts(d1, a_t + kBK / 2 + kk * 8, bdesc, idesc, (kc | kk) != 0);
            }
          } else {
#pragma unroll
            for (int kk = 0; kk < kBK / 16; ++kk) {
              const uint64_t bdesc = smem_desc_sw128(b_addr + kk * 32);
              umma_bf16_pair(d0, smem_desc_sw128(stage_addr + kk * 32), bdesc, idesc, (kc | kk) != 0);
              umma_bf16_pair(d1, smem_desc_sw128(stage_addr + kHalfBytes + kk * 32), bdesc, idesc, (kc | kk) != 0);
            }
          }
          umma_commit_pair_both(smem_u32(&sh.empty[s]));
          if (FP8) umma_commit_pair_both(smem_u32(&shf.conv_empty[c]));
        }
        if (ok) {
          for (int b = 0; b < 2; ++b)
            if ((mask >> b) & 1u) {
              umma_commit_pair_both(smem_u32(&sh.acc_full[b]));
            }
        }
      }
      if (!ok) {
        *abort_flag = 1;
        set_status(p.status, MOE_DEV_WAIT_TIMEOUT);
      }
      // all pair MMAs have completed once `drained` fires (in both CTAs)
      umma_commit_pair_both(smem_u32(&sh.drained));
      sh.consumed = consumed;
    }
    if (lane == 0) {
      int no_abort = 0;  // wait for the MMAs even when unwinding
      if (!mbar_wait_cluster_bounded(&sh.drained, 0, &no_abort)) set_status(p.status, MOE_DEV_WAIT_TIMEOUT);
    }
    __syncwarp();
  } else if (warp < 2 + kEpiWarps) {
    // ------------------------------------------------------------ epilogue --
    const int q = warp & 3;                  // TMEM lane quadrant this warp may access
    const int ew = warp - 2;                 // epilogue warp: its transpose tile
    const int sub = ew >> 2;                 // which of the quadrant's warps
    __nv_bfloat16* tile = reinterpret_cast<__nv_bfloat16*>(reinterpret_cast<uint8_t*>(tiles) + ew * kTileBytes);
    const bool leader = threadIdx.x == 64;
    uint32_t uses[2] = {0u, 0u};
    AccPlan<PL::kAccCols> plan;
    for (int i = 0;; ++i) {
      // the leader takes the next unit and waits for its accumulator(s); the
      // epilogue warps then agree on the outcome and all run the unit or all leave
      if (leader) {
        int u = -2;
        const int qr = i % kRing;
        if (mbar_wait_cluster_bounded(&sh.ring_full[qr], (i / kRing) & 1, abort_flag)) {
          u = load_volatile(&sh.ring[qr]);
          if (first) mbar_arrive(&sh.ring_empty[qr]);
          else st_async_u32(in_first(&sh.sink), 0u, in_first(&sh.ring_empty[qr]));
          if (u >= 0) {
            const Unit un = decode_unit(p, u);
            sh.epi_info[i & 1][0] = un.g;
            sh.epi_info[i & 1][1] = un.f;
            sh.epi_info[i & 1][2] = un.tok0;
            sh.epi_info[i & 1][3] = un.ntok;
            sh.epi_info[i & 1][4] = un.g == p.N ? un.tok0 : __ldg(p.grp_row0 + un.g) + un.tok0;
            uint32_t mask, base, stride;
            plan.place(mma_n<FP8>(un.ntok), mask, base, stride);
            bool ok = true;
            for (int b = 0; b < 2 && ok; ++b)
              if ((mask >> b) & 1u) ok = mbar_wait_cluster_bounded(&sh.acc_full[b], uses[b] & 1u, abort_flag);
            if (!ok) u = -2;
          }
        }
        if (u == -2) {
          *abort_flag = 1;
          set_status(p.status, MOE_DEV_WAIT_TIMEOUT);
        }
        sh.epi_unit[i & 1] = u;
      }
      epi_sync<kEpiWarps>();
      const int u = load_volatile(&sh.epi_unit[i & 1]);
      if (u < 0) break;
      Unit un;
      un.g = load_volatile(&sh.epi_info[i & 1][0]);
      un.f = load_volatile(&sh.epi_info[i & 1][1]);
      un.tok0 = load_volatile(&sh.epi_info[i & 1][2]);
      un.ntok = load_volatile(&sh.epi_info[i & 1][3]);
      uint32_t mask, base, stride;
      plan.place(mma_n<FP8>(un.ntok), mask, base, stride);
      plan.advance(mma_n<FP8>(un.ntok));
      uses[0] += mask & 1u;
      uses[1] += (mask >> 1) & 1u;
      tc_fence_after();
      const bool shared = un.g == p.N;
      const int64_t row_base = load_volatile(&sh.epi_info[i & 1][4]);
      __nv_bfloat16* out_base = shared ? p.out_shared : p.out_routed;
      const int64_t ld = shared ? p.ld_shared : p.ld_routed;
      const int cols = shared ? p.cols_shared : p.cols_routed;
      const uint32_t t_q = tmem_base + ((uint32_t)(q * 32) << 16) + base;
      constexpr int kHalves = MODE == kSwiGLU ? 1 : 2;
#pragma unroll 1
      for (int hh = 0; hh < kHalves; ++hh) {
        // this warp's 32 output columns of the unit
        const int c0 = un.f * p.tile_cols + rank_rows + half_cols * hh + 32 * q;
#pragma unroll 1
        for (int j0 = 32 * sub; j0 < un.ntok; j0 += 32 * (kEpiWarps / 4)) {
          const int tok = j0 + lane;
          const int64_t row = row_base + tok;
          // gate of this lane's token, spread to the lanes that hold it below
          float my_gate = 1.0f;
          if (MODE == kGateDown && !shared && p.gate_perm && tok < un.ntok &&
              MOE_IN_BOUNDS(row < p.tok_rows_routed, p.status))
            my_gate = __ldg(p.gate_perm + row);
          // The block (32 features = this quadrant's TMEM lanes, x 32 tokens =
          // columns j0..j0+31) in the m16n8 layout: lane half hf and column
          // group r give this thread features 16 hf + 8 e + lane / 4 (e = 0, 1)
          // and tokens 8 r + 2 (lane % 4) + 0..1, packed as bf16 pairs.
          uint32_t pk[2][4][2];
          const int tq = 2 * (lane & 3);
#pragma unroll
          for (int hf = 0; hf < 2; ++hf) {
            uint32_t a[16];
            tmem_ld16x256b_x4(t_q + ((uint32_t)(16 * hf) << 16) + hh * stride + j0, a);
            if (MODE == kSwiGLU) {
              uint32_t b[16];
              tmem_ld16x256b_x4(t_q + ((uint32_t)(16 * hf) << 16) + stride + j0, b);  // u of the same features
              tmem_wait_ld();
#pragma unroll
              for (int r = 0; r < 4; ++r)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                  const int x = 4 * r + 2 * e;
                  pk[hf][r][e] = pack_bf16x2(silu_tanh(__uint_as_float(a[x])) * __uint_as_float(b[x]),
                                             silu_tanh(__uint_as_float(a[x + 1])) * __uint_as_float(b[x + 1]));
                }
            } else {
              tmem_wait_ld();
#pragma unroll
              for (int r = 0; r < 4; ++r) {
                const float g0 = __shfl_sync(0xffffffffu, my_gate, 8 * r + tq);
                const float g1 = __shfl_sync(0xffffffffu, my_gate, 8 * r + tq + 1);
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                  const int x = 4 * r + 2 * e;
                  pk[hf][r][e] = pack_bf16x2(__uint_as_float(a[x]) * g0, __uint_as_float(a[x + 1]) * g1);
                }
              }
            }
          }
          // Transpose into this warp's [32 tokens][32 features] tile, 64-byte
          // swizzled (16-byte chunk c of token row t sits at chunk c ^ ((t >> 1) & 3)),
          // with four transposing matrix stores: matrix m of store (hf, rp) is
          // column group r = 2 rp + m / 2 and feature octet e = m % 2.
          if (lane == 0) bulk_wait_group_read<0>();  // the previous block's store has read the tile
          __syncwarp();
          const uint32_t tile_addr = smem_u32(tile);
          {
            const int m = lane >> 3, k = lane & 7;
#pragma unroll
            for (int hf = 0; hf < 2; ++hf)
#pragma unroll
              for (int rp = 0; rp < 2; ++rp) {
                const int t = 8 * (2 * rp + (m >> 1)) + k;  // token row this lane addresses
                const int c = 2 * hf + (m & 1);             // feature chunk
                stmatrix_x4_trans(tile_addr + t * 64 + ((c ^ ((t >> 1) & 3)) << 4), pk[hf][2 * rp][0],
                                  pk[hf][2 * rp][1], pk[hf][2 * rp + 1][0], pk[hf][2 * rp + 1][1]);
              }
          }
          const bool full_block = j0 + 32 <= un.ntok && c0 + 32 <= cols;
          if (full_block) {
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              (void)MOE_IN_BOUNDS(row_base + j0 < (shared ? p.out_rows_shared : p.out_rows_routed), p.status);
              tma_store_2d(shared ? &p.o_shared : &p.o_routed, tile, c0,
                           (int)(row_base + j0) + (shared ? p.out_row0_shared : 0));
              bulk_commit_group();
            }
          } else {
            __syncwarp();
            uint4 rowv[4];
#pragma unroll
            for (int c = 0; c < 4; ++c)
              rowv[c] = *reinterpret_cast<const uint4*>(reinterpret_cast<const uint8_t*>(tile) + lane * 64 +
                                                        ((c ^ ((lane >> 1) & 3)) << 4));
            // (columns at or past the matrix's width belong to a tile that
            // reaches past it: nothing to store)
            if (tok < un.ntok && c0 < cols &&
                MOE_IN_BOUNDS(row < (shared ? p.out_rows_shared : p.out_rows_routed), p.status))
              store_row32(out_base + row * ld + c0, cols - c0, rowv);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        for (int b = 0; b < 2; ++b)
          if ((mask >> b) & 1u) {
            if (!first) st_async_u32(in_first(&sh.sink), 0u, in_first(&sh.acc_empty[b]));
            else if (ew == 0) mbar_arrive_expect_tx(&sh.acc_empty[b], 4 * kEpiWarps);  // and CTA 1's warps' stores
            else mbar_arrive(&sh.acc_empty[b]);
          }
      }
    }
  } else if (FP8) {
    // ----------------------------------------- FP8 converters (kCvtWarps) --
    // Warp cw writes weight half cw / 4 of the rows in its TMEM lane quadrant:
    // per fill, in the producer's order, it waits (through a leader) for this
    // CTA's bytes and for a free weight slot, then each thread dequantises its
    // row's 64 codes (the 64-byte-swizzled box row: chunk c at c ^ (row / 2 % 4))
    // exactly into 32 columns of bf16 pairs, stores them to its TMEM lane and
    // the leader tells the MMA issuer once every converter's stores are done.
    const int cw = warp - (2 + kEpiWarps);   // 0 .. kCvtWarps - 1
    const int q = warp & 3;                  // TMEM lane quadrant this warp may access
    const int hsel = cw >> 2;                // weight half
    const int row = hsel * 128 + 32 * q + lane;  // row of the stage's code tile
    const bool cleader = cw == 0 && lane == 0;
    uint32_t j = 0;  // fills converted
    bool alive = true;
    for (int i = 0; alive; ++i) {
      if (cleader) {
        int u = -2;
        const int qr = i % kRing;
        if (mbar_wait_cluster_bounded(&sh.ring_full[qr], (i / kRing) & 1, abort_flag)) {
          u = load_volatile(&sh.ring[qr]);
          if (first) mbar_arrive(&sh.ring_empty[qr]);
          else st_async_u32(in_first(&sh.sink), 0u, in_first(&sh.ring_empty[qr]));
          if (u >= 0) {
            const Unit un = decode_unit(p, u);
            shf.cvt_info[i & 1][0] = un.g;
            shf.cvt_info[i & 1][1] = un.f;
          }
        }
        if (u == -2) {
          *abort_flag = 1;
          set_status(p.status, MOE_DEV_WAIT_TIMEOUT);
        }
        shf.cvt_unit[i & 1] = u;
      }
      cvt_sync<kCvtWarps>();
      if (load_volatile(&shf.cvt_unit[i & 1]) < 0) break;
      const int g = load_volatile(&shf.cvt_info[i & 1][0]);
      const int f = load_volatile(&shf.cvt_info[i & 1][1]);
      const bool shared = g == p.N;
      const int K = shared ? p.k_shared : p.k_routed;
      const int nk = K / kBK;                 // K is a multiple of 128 on this path
      const int nkb = K / kFp8Block;          // <= 64
      const int rowA = (shared ? 0 : g * p.a_rows_per_expert) + f * p.tile_cols + rank_rows;
      const int sblocks = shared ? p.sblocks_shared : p.sblocks_routed;
      // this warp's 128-row block: SwiGLU W1 (half 0) or W3 (half 1) rows of
      // the same block; down GEMM two consecutive W2 blocks (a block past the
      // matrix, whose rows load as zeros, takes the last block's scales)
      const int rb = min(rowA / kFp8Block + (MODE == kSwiGLU ? 0 : hsel), sblocks - 1);
      const uint8_t* sc = (MODE == kSwiGLU && hsel ? (shared ? p.s1_shared : p.s1_routed)
                                                   : (shared ? p.s0_shared : p.s0_routed)) +
                          (int64_t)rb * nkb;
      // lane l holds the scale bytes of K blocks l and l + 32
      const int sL = lane < nkb ? __ldg(sc + lane) : 0, sH = lane + 32 < nkb ? __ldg(sc + lane + 32) : 0;
      for (int kc = 0; kc < nk; ++kc, ++j) {
        const uint32_t s = j % kSlots, c = j % kASlots;
        if (cleader) {
          const bool ok = mbar_wait_bounded(&sh.full[s], (j / kSlots) & 1u, abort_flag) &&
                          mbar_wait_cluster_bounded(&shf.conv_empty[c], ((j / kASlots) & 1u) ^ 1u, abort_flag);
          if (ok) shf.seen = j + 1;
          else {
            *abort_flag = 1;
            set_status(p.status, MOE_DEV_WAIT_TIMEOUT);
          }
          shf.cvt_ok = ok;
        }
        cvt_sync<kCvtWarps>();
        if (!load_volatile(&shf.cvt_ok)) {
          alive = false;
          break;
        }
        tc_fence_after();  // the MMAs that read this slot before have completed
        const int kb = kc >> 1;  // 64-wide K block -> 128-wide scale block
        const int sb = __shfl_sync(0xffffffffu, kb < 32 ? sL : sH, kb & 31);
        const uint32_t raw = smem_u32(smem) + *reinterpret_cast<volatile uint32_t*>(&sh.slot_off[s]);
        (void)MOE_IN_BOUNDS(*reinterpret_cast<volatile uint32_t*>(&sh.slot_off[s]) + kA8Bytes <= (uint32_t)kRingBytes,
                            p.status);
        const uint32_t src = raw + row * kBK;
        uint4 wv[4];
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) wv[c4] = ld_shared_v4(src + ((c4 ^ ((row >> 1) & 3)) << 4));
        uint32_t o[32];
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) {
          uint32_t v[8];
          dequant16(wv[c4], sb, v);
#pragma unroll
          for (int e = 0; e < 8; ++e) o[8 * c4 + e] = v[e];
        }
        tmem_st32(tmem_base + ((uint32_t)(32 * q) << 16) + PL::kAccCols + c * kASlotCols + hsel * (kBK / 2), o);
        tmem_wait_st();
        tc_fence_before();
        cvt_sync<kCvtWarps>();
        if (cleader) {
          // CTA 1 signals through an asynchronous store (a blocking
          // cluster-scope arrive costs about 1000 cycles per stage)
          if (first) mbar_arrive_expect_tx(&shf.conv_full[c], 4);
          else st_async_u32(in_first(&shf.peer_word[c]), j, in_first(&shf.conv_full[c]));
        }
      }
    }
  }

  if (warp >= 2 && warp < 2 + kEpiWarps && lane == 0) bulk_wait_group_all();  // epilogue stores complete
  __syncthreads();
  if (warp == 0 && lane == 0 && (first || FP8)) {
    // wait for any stage fill that was issued but never observed complete
    // (bf16: the bytes of both CTAs land on the first CTA's stage barrier;
    // FP8: every CTA's land on its own and its converters observe them)
    for (uint32_t j = FP8 ? shf.seen : sh.consumed; j < fills; ++j) {
      const uint32_t s = j % kSlots, ph = (j / kSlots) & 1u;
      int dummy = 0;
      if (!mbar_wait_cluster_bounded(&sh.full[s], ph, &dummy)) {
        set_status(p.status, MOE_DEV_WAIT_TIMEOUT);
        break;
      }
    }
  }
  tc_fence_before();
  cluster_sync();  // neither CTA leaves while the other may still touch its shared memory
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, kTmemCols);
  }
}

// Token / weight operand: 64 columns x box_rows rows, 128-byte swizzle.
bool make_tmap(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
  return make_tmap_bf16(m, base, rows, cols, kBK, box_rows, true);
}

// Token operand maps with boxes of 32, 64 and 128 rows.
bool make_token_tmaps(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols) {
  for (int i = 0; i < kTokMaps; ++i)
    if (!make_tmap(&m[i], base, rows, cols, (uint32_t)(kTokBox << i))) return false;
  return true;
}

// Destination of the epilogue's 32 x 32 tile stores (64-byte swizzled tile).
bool make_store_tmap(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols) {
  return make_tmap_bf16_swz(m, base, rows, cols, 32, 32, 64);
}

// FP8 weight codes: 64 bytes x box_rows rows, 64-byte swizzle (each
// converter thread reads one row; a warp's 32 rows then cover all banks).
bool make_tmap_codes(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
  return make_tmap_u8(m, base, rows, cols, kBK, box_rows, 64);
}

template <int MODE, bool FP8>
cudaError_t launch_one(const TcParams& prm, int max_units, cudaStream_t s, bool programmatic) {
  // per device: the shared-memory opt-in done and the resident cluster count
  static std::mutex mu;
  static int max_clusters_of[kMaxDevices] = {};
  int dev = 0;
  cudaError_t e0 = cudaGetDevice(&dev);
  if (e0 != cudaSuccess) return e0;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.blockDim = dim3(Plan<FP8>::kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem_bytes<FP8>();
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int clusters = 0;
  {
    std::lock_guard<std::mutex> lock(mu);
    if (max_clusters_of[dev] == 0) {
      cudaError_t e = cudaFuncSetAttribute(expert_gemm_tc_kernel<MODE, FP8>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes<FP8>());
      if (e != cudaSuccess) return e;
      cfg.gridDim = dim3(2 * (device_sm_count() / 2), 1, 1);
      int n = 0;
      e = cudaOccupancyMaxActiveClusters(&n, expert_gemm_tc_kernel<MODE, FP8>, &cfg);
      if (e != cudaSuccess) return e;
      max_clusters_of[dev] = n > 0 ? n : 1;
    }
    clusters = max_clusters_of[dev];
  }
  if (max_units < clusters) clusters = max_units > 0 ? max_units : 1;
  cfg.gridDim = dim3(2 * clusters, 1, 1);
  cfg.numAttrs = programmatic ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, expert_gemm_tc_kernel<MODE, FP8>, prm);
}

}  // namespace

cudaError_t launch_expert_gemms_tc(const Problem& p, const GemmArgs& a, cudaStream_t s,
                                   cudaEvent_t between) {
  const int sms = device_sm_count();
  cudaError_t err0 = cudaMemsetAsync(a.sched, 0, 2 * sizeof(int), s);
  if (err0 != cudaSuccess) return err0;
  const bool fp8 = a.fp8;
  const int cm = fp8 ? Plan<true>::kChunk : Plan<false>::kChunk;  // token rows of a unit at most
  const int64_t chunks_bound = (p.R + cm - 1) / cm + p.N + (p.ns > 0 ? (p.T + cm - 1) / cm : 0);

  // weight maps: bf16 tiles, or the FP8 codes (plus their block scales)
  auto wmap = [&](CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
    return fp8 ? make_tmap_codes(m, base, rows, cols, box_rows) : make_tmap(m, base, rows, cols, box_rows);
  };
  TcParams g1{};
  bool ok = wmap(&g1.a0_routed, a.W1, (uint64_t)p.N * p.F, p.d, 128) &&
            wmap(&g1.a1_routed, a.W3, (uint64_t)p.N * p.F, p.d, 128) &&
            wmap(&g1.a0_shared, a.Ws1, (uint64_t)p.nsF, p.d, 128) &&
            wmap(&g1.a1_shared, a.Ws3, (uint64_t)p.nsF, p.d, 128) &&
            make_token_tmaps(g1.b_routed, a.x_perm, (uint64_t)p.R, p.d) &&
            make_token_tmaps(g1.b_shared, p.ns ? a.x : nullptr, (uint64_t)p.T, p.d) &&
            make_store_tmap(&g1.o_routed, a.h_perm, (uint64_t)p.R, p.F) &&
            make_store_tmap(&g1.o_shared, p.ns ? a.h_sh : nullptr, (uint64_t)p.T, p.nsF);
  if (!ok) return cudaErrorInvalidValue;
  g1.out_row0_shared = 0;
  g1.unit_base = a.unit_base1;
  g1.grp_row0 = a.grp_row0;
  g1.grp_rows = a.grp_rows;
  g1.sched = a.sched;
  g1.N = p.N;
  g1.k_routed = p.d;
  g1.k_shared = p.d;
  g1.cols_routed = p.F;
  g1.cols_shared = p.nsF;
  g1.a_rows_per_expert = p.F;
  g1.tile_cols = kTcBN1;
  g1.out_routed = (__nv_bfloat16*)a.h_perm;
  g1.ld_routed = p.F;
  g1.out_shared = (__nv_bfloat16*)a.h_sh;
  g1.ld_shared = p.nsF;
  g1.gate_perm = nullptr;
  g1.status = a.status;
  g1.s0_routed = a.W1s;
  g1.s1_routed = a.W3s;
  g1.s0_shared = a.Ws1s;
  g1.s1_shared = a.Ws3s;
  g1.sblocks_routed = (int)((int64_t)p.N * p.F / kFp8Block);
  g1.sblocks_shared = p.nsF / kFp8Block;
  g1.chunk_rows = cm;
  g1.tok_rows_routed = p.R;
  g1.tok_rows_shared = p.T;
  g1.a_rows_routed = (int64_t)p.N * p.F;
  g1.a_rows_shared = p.nsF;
  g1.out_rows_routed = p.R;
  g1.out_rows_shared = p.T;
  const int64_t max_cols1 = p.F > p.nsF ? p.F : p.nsF;
  const int64_t units1 = chunks_bound * ((max_cols1 + kTcBN1 - 1) / kTcBN1);
  const int grid1 = (int)(units1 < sms ? units1 : sms);
  cudaError_t err = fp8 ? launch_one<kSwiGLU, true>(g1, grid1, s, false) : launch_one<kSwiGLU, false>(g1, grid1, s, false);
  if (err == cudaSuccess && between) err = cudaEventRecord(between, s);
  if (err != cudaSuccess) return err;

  TcParams g2{};
  ok = wmap(&g2.a0_routed, a.W2, (uint64_t)p.N * p.d, p.F, 256) &&
       wmap(&g2.a0_shared, a.Ws2, (uint64_t)p.d, p.nsF, 256) &&
       make_token_tmaps(g2.b_routed, a.h_perm, (uint64_t)p.R, p.F) &&
       make_token_tmaps(g2.b_shared, p.ns ? a.h_sh : nullptr, (uint64_t)p.T, p.nsF) &&
       make_store_tmap(&g2.o_routed, a.y_rows, (uint64_t)(p.R + p.T), p.d) &&
       make_store_tmap(&g2.o_shared, a.y_rows, (uint64_t)(p.R + p.T), p.d);
  if (!ok) return cudaErrorInvalidValue;
  g2.out_row0_shared = (int)p.R;
  g2.unit_base = a.unit_base2;
  g2.grp_row0 = a.grp_row0;
  g2.grp_rows = a.grp_rows;
  g2.sched = a.sched + 1;
  g2.N = p.N;
  g2.k_routed = p.F;
  g2.k_shared = p.nsF;
  g2.cols_routed = p.d;
  g2.cols_shared = p.d;
  g2.a_rows_per_expert = p.d;
  g2.tile_cols = kTcBN2;
  g2.out_routed = (__nv_bfloat16*)a.y_rows;
  g2.ld_routed = p.d;
  g2.out_shared = (__nv_bfloat16*)a.y_rows + p.R * (int64_t)p.d;
  g2.ld_shared = p.d;
  g2.gate_perm = a.gate_perm;
  g2.status = a.status;
  g2.s0_routed = a.W2s;
  g2.s0_shared = a.Ws2s;
  g2.sblocks_routed = (int)((int64_t)p.N * p.d / kFp8Block);
  g2.sblocks_shared = p.d / kFp8Block;
  g2.chunk_rows = cm;
  g2.tok_rows_routed = p.R;
  g2.tok_rows_shared = p.T;
  g2.a_rows_routed = (int64_t)p.N * p.d;
  g2.a_rows_shared = p.d;
  g2.out_rows_routed = p.R;
  g2.out_rows_shared = p.T;
  const int64_t units2 = chunks_bound * ((p.d + kTcBN2 - 1) / kTcBN2);
  const int grid2 = (int)(units2 < sms ? units2 : sms);
  // the down GEMM overlaps the SwiGLU GEMM's drain unless an event must be
  // recorded between the two
  return fp8 ? launch_one<kGateDown, true>(g2, grid2, s, !between) : launch_one<kGateDown, false>(g2, grid2, s, !between);
}

}  // namespace moe
