// Dispatch: expert histogram, exclusive scan, expert-contiguous permutation
// and the row gather that feeds the grouped GEMMs. The quoted forward of the
// "DeepSeek-V3.2-Exp · Mixture of experts" page counts the tokens per expert
// on the host and searches each expert's rows in a loop; here that is three
// small kernels (one for decode-sized batches) and no host round trip.
//
// Bit-exact by construction: a warp owns 32 consecutive tokens; for each
// expert it forms a ballot of the tokens that chose it, so a pair's rank
// inside the chunk is the popcount of the lower lanes, and chunk bases come
// from a scan in (expert, chunk) order. No atomics decide any position.
#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int kWarpsPerCta = 8;

struct ChunkArgs {
  const int32_t* idx;
  int64_t T;
  int N, k;
  int32_t* chunk_counts;     // [n_chunks, N]
  const int32_t* chunk_base; // [n_chunks, N] (scatter pass)
  const float* gates;        // [T, k]       (scatter pass, may be null)
  int32_t* perm;             // [R]
  int32_t* slot_pos;         // [T, k]: rows of the token's experts, ascending expert
  float* gate_perm;          // [R]
  unsigned* status;
};

// One warp per (chunk of 32 tokens, word of 32 experts): lane l holds token
// 32 c + l and the bits of the experts 32 w .. 32 w + 31 it selected. For each
// expert of the word a ballot gives the tokens that chose it; a pair's rank
// within the chunk is the popcount of the lower lanes. Pass 0 writes the
// per-chunk counts, pass 1 places every pair.
template <bool kScatter>
MOE_DEV void chunk_pass(const ChunkArgs& a, int64_t gw) {
  const int lane = threadIdx.x & 31;
  const int W = (a.N + 31) / 32;
  const int64_t n_chunks = (a.T + 31) / 32;
  if (gw >= n_chunks * W) return;
  const int64_t c = gw / W;
  const int w = (int)(gw % W);
  const int64_t t = c * 32 + lane;
  int32_t my[kMaxTopK];
  uint32_t word = 0;
#pragma unroll
  for (int s = 0; s < kMaxTopK; ++s) {
    my[s] = -1;
    if (s < a.k && t < a.T) {
      const int32_t e = a.idx[t * a.k + s];
      if (e < 0 || e >= a.N) {
        if (!kScatter && w == 0) set_status(a.status, MOE_DEV_BAD_EXPERT);
        continue;
      }
      my[s] = e;
      if ((e >> 5) == w) {
        const uint32_t m = 1u << (e & 31);
        if (word & m) {
          if (!kScatter) set_status(a.status, MOE_DEV_DUP_EXPERT);
          my[s] = -1;
        }
        word |= m;
      }
    }
  }
  const uint32_t lt = (1u << lane) - 1u;
  int my_count = 0;
  for (int b = 0; b < 32; ++b) {
    const bool has = (word >> b) & 1u;
    const uint32_t m = __ballot_sync(0xffffffffu, has);
    if (!kScatter) {
      if (lane == b) my_count = __popc(m);
    } else if (has) {
      const int e = 32 * w + b;
      const int32_t pos = a.chunk_base[c * a.N + e] + __popc(m & lt);
      int slot = 0, below = 0;
#pragma unroll
      for (int s = 0; s < kMaxTopK; ++s) {
        if (my[s] == e) slot = s;
        below += (my[s] >= 0 && my[s] < e) ? 1 : 0;
      }
      const int32_t flat = (int32_t)(t * a.k + slot);
      if (MOE_IN_BOUNDS(pos >= 0 && (int64_t)pos < a.T * a.k && below < a.k, a.status)) {
        a.perm[pos] = flat;
        a.slot_pos[t * a.k + below] = pos;
        if (a.gates) a.gate_perm[pos] = a.gates[flat];
      }
    }
  }
  if (!kScatter) {
    const int e = 32 * w + lane;
    if (e < a.N) a.chunk_counts[c * a.N + e] = my_count;
  }
}

template <bool kScatter>
__global__ void __launch_bounds__(32 * kWarpsPerCta) chunk_kernel(ChunkArgs a) {
  chunk_pass<kScatter>(a, (int64_t)blockIdx.x * kWarpsPerCta + (threadIdx.x >> 5));
}

// Exclusive scan of v over the whole block (blockDim.x a multiple of 32,
// at most 1024); returns the prefix and writes the block total to *total.
MOE_DEV int block_exclusive_scan(int v, int* total) {
  __shared__ int warp_base[32];
  __shared__ int block_total;
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int nw = blockDim.x >> 5;
  int incl = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    int o = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += o;
  }
  if (lane == 31) warp_base[w] = incl;
  __syncthreads();
  if (w == 0) {
    const int x = lane < nw ? warp_base[lane] : 0;
    int xi = x;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      int o = __shfl_up_sync(0xffffffffu, xi, off);
      if (lane >= off) xi += o;
    }
    if (lane < nw) warp_base[lane] = xi - x;
    if (lane == 31) block_total = xi;
  }
  __syncthreads();
  const int res = warp_base[w] + incl - v;
  *total = block_total;
  __syncthreads();  // the shared slots are reused by the next call
  return res;
}

struct ScanArgs {
  int32_t* chunk_counts;  // in: counts per chunk; out (as chunk_base): absolute positions
  int64_t n_chunks, T;
  int N, ns, F, nsF, d;
  int bm, bn1, bn2;
  int32_t* counts;
  int32_t* offsets;
  int32_t* grp_row0;
  int32_t* grp_rows;
  int32_t* unit_base1;
  int32_t* unit_base2;
};

// Run by one CTA of 1024 threads: per-expert totals and chunk bases, offsets,
// and the GEMM unit tables (groups 0..N-1 routed, group N the shared MLP).
MOE_DEV void scan_pass(const ScanArgs& a, int32_t* chunk_base) {
  const int tid = threadIdx.x;
  int cnt = 0;
  if (tid < a.N) {
    // running sum over the chunks; loads are issued 8 at a time so the loop
    // is not one L2 round trip per chunk
    int run = 0;
    int64_t c = 0;
    for (; c + 8 <= a.n_chunks; c += 8) {
      int v[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) v[j] = a.chunk_counts[(c + j) * a.N + tid];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        chunk_base[(c + j) * a.N + tid] = run;
        run += v[j];
      }
    }
    for (; c < a.n_chunks; ++c) {
      int v = a.chunk_counts[c * a.N + tid];
      chunk_base[c * a.N + tid] = run;
      run += v;
    }
    cnt = run;
  }
  int total;
  const int off = block_exclusive_scan(cnt, &total);
  if (tid < a.N) {
    a.counts[tid] = cnt;
    a.offsets[tid] = off;
    int64_t c = 0;
    for (; c + 8 <= a.n_chunks; c += 8) {
      int v[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) v[j] = chunk_base[(c + j) * a.N + tid];
#pragma unroll
      for (int j = 0; j < 8; ++j) chunk_base[(c + j) * a.N + tid] = v[j] + off;
    }
    for (; c < a.n_chunks; ++c) chunk_base[c * a.N + tid] += off;
  }
  if (tid == 0) a.offsets[a.N] = total;

  // unit tables over groups g = 0..N (N = shared MLP)
  int rows = 0, row0 = 0, u1 = 0, u2 = 0;
  if (tid < a.N) {
    rows = cnt;
    row0 = off;
  } else if (tid == a.N && a.ns > 0) {
    rows = (int)a.T;
    row0 = 0;
  }
  if (tid <= a.N) {
    const int mt = (rows + a.bm - 1) / a.bm;
    const int cols1 = tid < a.N ? a.F : a.nsF;
    u1 = mt * ((cols1 + a.bn1 - 1) / a.bn1);
    u2 = mt * ((a.d + a.bn2 - 1) / a.bn2);
    a.grp_rows[tid] = rows;
    a.grp_row0[tid] = row0;
  }
  int tot1, tot2;
  const int b1 = block_exclusive_scan(u1, &tot1);
  const int b2 = block_exclusive_scan(u2, &tot2);
  if (tid <= a.N) {
    a.unit_base1[tid] = b1;
    a.unit_base2[tid] = b2;
  }
  if (tid == 0) {
    a.unit_base1[a.N + 1] = tot1;
    a.unit_base2[a.N + 1] = tot2;
  }
}

__global__ void __launch_bounds__(1024) scan_kernel(ScanArgs a, int32_t* chunk_base) { scan_pass(a, chunk_base); }

// The whole dispatch in one CTA of 1024 threads when every chunk warp fits
// in it (decode-sized batches): slot_pos reset, the counting pass into shared
// memory, the scan, and the placing pass -- the same passes as the three
// kernels above, so the same positions, with one launch instead of three and
// a memset.
__global__ void __launch_bounds__(1024) dispatch_small_kernel(ChunkArgs ca, ScanArgs sa) {
  extern __shared__ int32_t dsm[];  // [n_chunks, N] counts, then [n_chunks, N] bases
  const int64_t n = ((ca.T + 31) / 32) * ca.N;
  for (int64_t i = threadIdx.x; i < ca.T * ca.k; i += blockDim.x) ca.slot_pos[i] = -1;
  ChunkArgs a = ca;
  a.chunk_counts = dsm;
  a.chunk_base = dsm + n;
  const int64_t gw = threadIdx.x >> 5;
  chunk_pass<false>(a, gw);
  __syncthreads();
  ScanArgs s = sa;
  s.chunk_counts = dsm;
  scan_pass(s, dsm + n);
  __syncthreads();
  chunk_pass<true>(a, gw);
}

// x_perm[slot_pos[t, s]] = x[t] for every placed pair: a warp reads its
// part of a token's row once and writes it to each of the token's k permuted
// rows, so x is read from HBM once (a pair left at -1 by an invalid index is
// skipped). A row is split into `parts` column ranges handled by separate
// warps when there are few tokens (decode), so the copy spreads over the GPU.
template <typename TV, int KMAX>
__global__ void __launch_bounds__(256) gather_kernel(const TV* __restrict__ x,
                                                     const int32_t* __restrict__ slot_pos, int64_t T,
                                                     int k, int vecs, int parts, TV* __restrict__ x_perm,
                                                     unsigned* status) {
  const int lane = threadIdx.x & 31;
  const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
  for (int64_t w = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); w < T * parts; w += warps) {
    const int64_t t = w / parts;
    const int part = (int)(w % parts);
    const int v0 = (int)((int64_t)part * vecs / parts), v1 = (int)((int64_t)(part + 1) * vecs / parts);
    int32_t dst[KMAX];
#pragma unroll
    for (int s = 0; s < KMAX; ++s) {
      dst[s] = s < k ? __ldg(slot_pos + t * k + s) : -1;
      if (dst[s] >= 0 && !MOE_IN_BOUNDS((int64_t)dst[s] < T * k, status)) dst[s] = -1;
    }
    const TV* src = x + t * vecs;
    // two loads in flight per lane before their stores
    int v = v0 + lane;
    for (; v + 32 < v1; v += 64) {
      const TV a = __ldg(src + v), b = __ldg(src + v + 32);
#pragma unroll
      for (int s = 0; s < KMAX; ++s)
        if (dst[s] >= 0) {
          x_perm[(int64_t)dst[s] * vecs + v] = a;
          x_perm[(int64_t)dst[s] * vecs + v + 32] = b;
        }
    }
    if (v < v1) {
      const TV a = __ldg(src + v);
#pragma unroll
      for (int s = 0; s < KMAX; ++s)
        if (dst[s] >= 0) x_perm[(int64_t)dst[s] * vecs + v] = a;
    }
  }
}

// Expert-parallel exchange order. counts [W, E]: rows that source rank p
// sends for local expert e. Source-major order holds the blocks (p, e) as
// p-major, e-minor (what an all-to-all delivers); expert-major order holds
// them e-major, p-minor (what the grouped GEMMs read). One CTA per block
// copies its rows, 16 or 4 bytes at a time.
__global__ void __launch_bounds__(256) ep_reorder_kernel(const int32_t* __restrict__ counts, int W, int E,
                                                         int64_t row_bytes, const uint8_t* __restrict__ src,
                                                         uint8_t* __restrict__ dst, int to_expert_major) {
  const int blk = blockIdx.x;
  if (blk >= W * E) return;
  const int p = blk / E, e = blk % E;
  __shared__ int64_t offs[2];
  if (threadIdx.x == 0) {
    int64_t so = 0, eo = 0;
    for (int q = 0; q < W; ++q)
      for (int f = 0; f < E; ++f) {
        const int64_t c = counts[q * E + f];
        if (q < p || (q == p && f < e)) so += c;
        if (f < e || (f == e && q < p)) eo += c;
      }
    offs[0] = so;
    offs[1] = eo;
  }
  __syncthreads();
  const int64_t n = counts[p * E + e];
  const int64_t from = to_expert_major ? offs[0] : offs[1];
  const int64_t to = to_expert_major ? offs[1] : offs[0];
  const uint8_t* s = src + from * row_bytes;
  uint8_t* d = dst + to * row_bytes;
  const int64_t bytes = n * row_bytes;
  if (row_bytes % 16 == 0) {
    for (int64_t i = threadIdx.x; i < bytes / 16; i += blockDim.x)
      reinterpret_cast<uint4*>(d)[i] = reinterpret_cast<const uint4*>(s)[i];
  } else {
    for (int64_t i = threadIdx.x; i < bytes / 4; i += blockDim.x)
      reinterpret_cast<uint32_t*>(d)[i] = reinterpret_cast<const uint32_t*>(s)[i];
  }
}

}  // namespace

cudaError_t launch_ep_reorder(const int32_t* counts, int W, int E, int64_t row_bytes, const void* src, void* dst,
                              bool to_expert_major, cudaStream_t s) {
  if (W <= 0 || E <= 0) return cudaSuccess;
  ep_reorder_kernel<<<W * E, 256, 0, s>>>(counts, W, E, row_bytes, static_cast<const uint8_t*>(src),
                                         static_cast<uint8_t*>(dst), to_expert_major ? 1 : 0);
  return cudaGetLastError();
}

cudaError_t launch_unit_tables(const Problem& p, const int32_t* counts, const DispatchBuffers& db, int bm, int bn1,
                               int bn2, cudaStream_t s) {
  // the scan over a single "chunk" whose counts are the groups' row counts
  ScanArgs sa{const_cast<int32_t*>(counts), 1, p.T, p.N, p.ns, p.F, p.nsF, p.d, bm, bn1, bn2,
              db.counts, db.offsets, db.grp_row0, db.grp_rows, db.unit_base1, db.unit_base2};
  scan_kernel<<<1, 1024, 0, s>>>(sa, db.chunk_base);
  return cudaGetLastError();
}

cudaError_t launch_dispatch(const Problem& p, const DispatchBuffers& db, int bm, int bn1, int bn2,
                            cudaStream_t s) {
  const int64_t n_chunks = (p.T + 31) / 32;
  const int64_t warps = n_chunks * ((p.N + 31) / 32);
  const unsigned blocks = (unsigned)((warps + kWarpsPerCta - 1) / kWarpsPerCta);
  ChunkArgs ca{db.idx, p.T, p.N, p.k, db.chunk_counts, db.chunk_base, db.gates, db.perm,
               db.slot_pos, db.gate_perm, db.status};
  const size_t small_smem = (size_t)2 * n_chunks * p.N * sizeof(int32_t);
  if (warps <= 32 && small_smem <= 48 * 1024) {
    ScanArgs sa{nullptr, n_chunks, p.T, p.N, p.ns, p.F, p.nsF, p.d, bm, bn1, bn2,
                db.counts, db.offsets, db.grp_row0, db.grp_rows, db.unit_base1, db.unit_base2};
    dispatch_small_kernel<<<1, 1024, small_smem, s>>>(ca, sa);
    return cudaGetLastError();
  }
  cudaError_t err = cudaMemsetAsync(db.slot_pos, 0xFF, (size_t)p.R * sizeof(int32_t), s);
  if (err != cudaSuccess) return err;
  chunk_kernel<false><<<blocks, 32 * kWarpsPerCta, 0, s>>>(ca);
  err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  ScanArgs sa{db.chunk_counts, n_chunks, p.T, p.N, p.ns, p.F, p.nsF, p.d, bm, bn1, bn2,
              db.counts, db.offsets, db.grp_row0, db.grp_rows, db.unit_base1, db.unit_base2};
  scan_kernel<<<1, 1024, 0, s>>>(sa, db.chunk_base);
  err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  chunk_kernel<true><<<blocks, 32 * kWarpsPerCta, 0, s>>>(ca);
  return cudaGetLastError();
}

cudaError_t launch_gather(const Problem& p, const void* x, const int32_t* slot_pos, void* x_perm,
                          unsigned* status, cudaStream_t s) {
  if (p.R == 0) return cudaSuccess;
  const int vecs = (int)((int64_t)p.d * p.elem / 16);
  const int sms = device_sm_count();
  // warps per token: enough for about 8 warps per SM, at most 8 and at least
  // 32 vectors (one per lane) per part
  int64_t parts = ((int64_t)sms * 32 + p.T - 1) / p.T;
  if (parts > 8) parts = 8;
  if (parts > vecs / 32) parts = vecs / 32;
  if (parts < 1) parts = 1;
  const int64_t want = (p.T * parts + 7) / 8;
  const int64_t cap = (int64_t)sms * 16;
  const unsigned blocks = (unsigned)(want < cap ? want : cap);
  if (p.k <= 8)
    gather_kernel<uint4, 8><<<blocks, 256, 0, s>>>((const uint4*)x, slot_pos, p.T, p.k, vecs, (int)parts,
                                                   (uint4*)x_perm, status);
  else
    gather_kernel<uint4, kMaxTopK><<<blocks, 256, 0, s>>>((const uint4*)x, slot_pos, p.T, p.k, vecs, (int)parts,
                                                          (uint4*)x_perm, status);
  return cudaGetLastError();
}

}  // namespace moe
