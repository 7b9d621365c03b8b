// C ABI of the layer (declared in include/moe_b200.h): argument checks,
// workspace carving and the launch sequence
//   router -> dispatch -> gather -> SwiGLU GEMM -> gate GEMM -> combine,
// all on the caller's stream with no host synchronisation.
#include <cstring>
#include <mutex>
#include <unordered_map>

#include <nvtx3/nvToolsExt.h>

#include "common.cuh"
#include "internal.h"

namespace moe {

// NVTX ranges for timeline tools: one for a layer forward and, nested in it,
// one per stage (the host-side enqueue of that stage's launches, which a
// timeline tool ties to the kernels). With no tool attached an NVTX call
// costs a check of a function pointer.
class NvtxStages {
 public:
  explicit NvtxStages(const char* call) { nvtxRangePushA(call); }
  void stage(const char* name) {
    if (open_) nvtxRangePop();
    nvtxRangePushA(name);
    open_ = true;
  }
  ~NvtxStages() {
    if (open_) nvtxRangePop();
    nvtxRangePop();
  }
  NvtxStages(const NvtxStages&) = delete;
  NvtxStages& operator=(const NvtxStages&) = delete;

 private:
  bool open_ = false;
};

namespace {
thread_local int32_t g_last_cuda_error = 0;
constexpr int kStageEvents = 7;
thread_local cudaEvent_t g_stage_events[kStageEvents] = {};
thread_local bool g_stage_events_on = false;

cudaError_t mark_stage(int i, cudaStream_t s) {
  return g_stage_events_on ? cudaEventRecord(g_stage_events[i], s) : cudaSuccess;
}

size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

moe_status cuda_fail(cudaError_t e) {
  g_last_cuda_error = (int32_t)e;
  return MOE_ERR_CUDA;
}
}  // namespace

void record_cuda_error(cudaError_t e) { g_last_cuda_error = (int32_t)e; }

int device_sm_count() {
  static int cached_dev = -1, cached_sms = 148;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cached_sms;
  if (dev != cached_dev) {
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && sms > 0) {
      cached_sms = sms;
      cached_dev = dev;
    }
  }
  return cached_sms;
}

moe_status make_problem(const moe_cfg* cfg, int64_t T, Problem* p) {
  if (!cfg || !p || T < 0) return MOE_ERR_INVALID_ARG;
  const moe_cfg& c = *cfg;
  if (c.d <= 0 || c.d_ff <= 0 || c.n_routed <= 0 || c.n_shared < 0 || c.top_k <= 0)
    return MOE_ERR_INVALID_ARG;
  if (c.d % 8 || c.d_ff % 8) return MOE_ERR_INVALID_ARG;
  if (c.top_k > c.n_routed) return MOE_ERR_INVALID_ARG;
  const int G = c.n_groups <= 0 ? 1 : c.n_groups;
  const int TG = G == 1 ? 1 : c.topk_groups;
  if (c.n_routed % G || TG < 1 || TG > G) return MOE_ERR_INVALID_ARG;
  if ((int64_t)c.top_k > (int64_t)TG * (c.n_routed / G)) return MOE_ERR_INVALID_ARG;
  if (c.score_fn != MOE_SOFTMAX && c.score_fn != MOE_SIGMOID) return MOE_ERR_INVALID_ARG;
  if (c.group_score != MOE_GROUP_TOP2_SUM && c.group_score != MOE_GROUP_MAX) return MOE_ERR_INVALID_ARG;
  if (G > 1 && c.group_score == MOE_GROUP_TOP2_SUM && c.n_routed / G < 2) return MOE_ERR_INVALID_ARG;
  if (c.dtype != MOE_F32 && c.dtype != MOE_BF16) return MOE_ERR_INVALID_ARG;
  if (!(c.route_scale == c.route_scale)) return MOE_ERR_INVALID_ARG;  // NaN
  // implemented range
  if (c.n_routed > kMaxRouted || c.top_k > kMaxTopK || G > 32) return MOE_ERR_UNSUPPORTED;
  const int64_t nsF64 = (int64_t)c.n_shared * c.d_ff;
  if (nsF64 > (1 << 30) || (int64_t)c.n_routed * c.d_ff > (1ll << 31) ||
      (int64_t)c.n_routed * c.d > (1ll << 31))
    return MOE_ERR_UNSUPPORTED;
  if (T * (int64_t)c.top_k + T > (1ll << 31) - 1) return MOE_ERR_UNSUPPORTED;
  p->T = T;
  p->d = c.d;
  p->F = c.d_ff;
  p->N = c.n_routed;
  p->ns = c.n_shared;
  p->k = c.top_k;
  p->G = G;
  p->TG = TG;
  p->score_fn = c.score_fn;
  p->normalize = c.normalize != 0;
  p->group_score = c.group_score;
  p->dtype = c.dtype;
  p->route_scale = c.route_scale;
  p->R = T * c.top_k;
  p->nsF = (int)nsF64;
  p->elem = c.dtype == MOE_BF16 ? 2 : 4;
  return MOE_OK;
}

Layout make_layout(const Problem& p) {
  Layout L{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t at = off;
    off = align256(off + bytes);
    return at;
  };
  const int64_t T = p.T, N = p.N, R = p.R;
  L.n_chunks = (T + kChunkTokens - 1) / kChunkTokens;
  L.status = take(256);
  L.sched = take(256);
  L.logits = take(router_scratch_bytes(p));
  L.idx = take((size_t)R * 4);
  L.gates = take((size_t)R * 4);
  L.chunk_counts = take((size_t)L.n_chunks * N * 4);
  L.chunk_base = take((size_t)L.n_chunks * N * 4);
  L.counts = take((size_t)N * 4);
  L.offsets = take((size_t)(N + 1) * 4);
  L.grp_row0 = take((size_t)(N + 1) * 4);
  L.grp_rows = take((size_t)(N + 1) * 4);
  L.unit_base1 = take((size_t)(N + 2) * 4);
  L.unit_base2 = take((size_t)(N + 2) * 4);
  L.perm = take((size_t)R * 4);
  L.slot_pos = take((size_t)R * 4);
  L.gate_perm = take((size_t)R * 4);
  L.x_perm = take((size_t)R * p.d * p.elem);
  L.h_perm = take((size_t)R * p.F * p.elem);
  L.h_sh = take((size_t)T * p.nsF * p.elem);
  L.y_rows = take((size_t)(R + T) * p.d * p.elem);
  L.total = off;
  L.x_stage[0] = take((size_t)T * p.d * p.elem);
  L.x_stage[1] = take((size_t)T * p.d * p.elem);
  L.y_stage[0] = take((size_t)T * p.d * p.elem);
  L.y_stage[1] = take((size_t)T * p.d * p.elem);
  L.total_host = off;
  return L;
}

namespace {

template <typename T>
T* at(void* ws, size_t off) {
  return reinterpret_cast<T*>(static_cast<uint8_t*>(ws) + off);
}

moe_status check_ws(const Layout& L, void* ws, size_t ws_bytes, size_t need) {
  if (!ws || ws_bytes < need || (reinterpret_cast<uintptr_t>(ws) & 255u)) return MOE_ERR_WORKSPACE;
  (void)L;
  return MOE_OK;
}

moe_status run_router(const Problem& p, const Layout& L, const void* x, const void* W_r,
                      const float* b, int32_t* idx, float* gates, void* ws, cudaStream_t s) {
  cudaError_t e = launch_router(p, x, W_r, b, at<float>(ws, L.logits), router_scratch_bytes(p), idx, gates,
                                at<unsigned>(ws, L.status), s);
  return e == cudaSuccess ? MOE_OK : cuda_fail(e);
}

DispatchBuffers dispatch_buffers(const Layout& L, void* ws, const int32_t* idx, const float* gates) {
  DispatchBuffers db;
  db.idx = idx;
  db.chunk_counts = at<int32_t>(ws, L.chunk_counts);
  db.chunk_base = at<int32_t>(ws, L.chunk_base);
  db.counts = at<int32_t>(ws, L.counts);
  db.offsets = at<int32_t>(ws, L.offsets);
  db.grp_row0 = at<int32_t>(ws, L.grp_row0);
  db.grp_rows = at<int32_t>(ws, L.grp_rows);
  db.unit_base1 = at<int32_t>(ws, L.unit_base1);
  db.unit_base2 = at<int32_t>(ws, L.unit_base2);
  db.perm = at<int32_t>(ws, L.perm);
  db.slot_pos = at<int32_t>(ws, L.slot_pos);
  db.gate_perm = at<float>(ws, L.gate_perm);
  db.gates = gates;
  db.status = at<unsigned>(ws, L.status);
  return db;
}

// Scale pointers of FP8 expert weights (W1, W3, W2, Ws1, Ws3, Ws2), or null for bf16 / fp32 weights.
struct Fp8Scales {
  const uint8_t* s[6];
};

moe_status forward_device(const Problem& p, const Layout& L, const void* x, const void* W_r,
                          const float* b, const void* W1, const void* W3, const void* W2,
                          const void* Ws1, const void* Ws3, const void* Ws2, void* y,
                          int32_t* idx_out, float* gates_out, void* ws, cudaStream_t s,
                          const Fp8Scales* fp8 = nullptr) {
  NvtxStages nv(fp8 ? "moe_forward_fp8" : "moe_forward");
  int32_t* idx = at<int32_t>(ws, L.idx);
  float* gates = at<float>(ws, L.gates);
  cudaError_t e0 = cudaMemsetAsync(at<void>(ws, L.status), 0, 4, s);
  if (e0 == cudaSuccess) e0 = mark_stage(0, s);
  if (e0 != cudaSuccess) return cuda_fail(e0);
  nv.stage("moe.router");
  moe_status st = run_router(p, L, x, W_r, b, idx, gates, ws, s);
  if (st != MOE_OK) return st;
  if ((e0 = mark_stage(1, s)) != cudaSuccess) return cuda_fail(e0);
  const bool tc = p.dtype == MOE_BF16;
  DispatchBuffers db = dispatch_buffers(L, ws, idx, gates);
  nv.stage("moe.dispatch");
  // unit tables for the GEMMs: FP8 weights cut groups into chunks of at most kTcBM8 rows
  cudaError_t e = launch_dispatch(p, db, tc ? (fp8 ? kTcBM8 : kTcBM) : kSimtBM, tc ? kTcBN1 : kSimtBN,
                                  tc ? kTcBN2 : kSimtBN, s);
  if (e == cudaSuccess) e = mark_stage(2, s);
  if (e != cudaSuccess) return cuda_fail(e);
  nv.stage("moe.gather");
  e = launch_gather(p, x, db.slot_pos, at<void>(ws, L.x_perm), db.status, s);
  if (e == cudaSuccess) e = mark_stage(3, s);
  if (e != cudaSuccess) return cuda_fail(e);
  GemmArgs ga;
  ga.x = x;
  ga.x_perm = at<void>(ws, L.x_perm);
  ga.W1 = W1;
  ga.W3 = W3;
  ga.W2 = W2;
  ga.Ws1 = p.ns ? Ws1 : nullptr;
  ga.Ws3 = p.ns ? Ws3 : nullptr;
  ga.Ws2 = p.ns ? Ws2 : nullptr;
  ga.h_perm = at<void>(ws, L.h_perm);
  ga.h_sh = at<void>(ws, L.h_sh);
  ga.y_rows = at<void>(ws, L.y_rows);
  ga.grp_row0 = db.grp_row0;
  ga.grp_rows = db.grp_rows;
  ga.unit_base1 = db.unit_base1;
  ga.unit_base2 = db.unit_base2;
  ga.gate_perm = db.gate_perm;
  ga.status = db.status;
  ga.sched = at<int>(ws, L.sched);
  if (fp8) {
    ga.fp8 = true;
    ga.W1s = fp8->s[0];
    ga.W3s = fp8->s[1];
    ga.W2s = fp8->s[2];
    ga.Ws1s = p.ns ? fp8->s[3] : nullptr;
    ga.Ws3s = p.ns ? fp8->s[4] : nullptr;
    ga.Ws2s = p.ns ? fp8->s[5] : nullptr;
  }
  nv.stage("moe.expert_gemms");
  e = tc ? launch_expert_gemms_tc(p, ga, s, g_stage_events_on ? g_stage_events[4] : nullptr)
         : launch_expert_gemms_simt(p, ga, s, g_stage_events_on ? g_stage_events[4] : nullptr);
  if (e == cudaSuccess) e = mark_stage(5, s);
  if (e != cudaSuccess) return cuda_fail(e);
  nv.stage("moe.combine");
  e = launch_combine(p, ga.y_rows, db.slot_pos, y, s);
  if (e == cudaSuccess) e = mark_stage(6, s);
  if (e != cudaSuccess) return cuda_fail(e);
  if (idx_out) {
    e = cudaMemcpyAsync(idx_out, idx, (size_t)p.R * 4, cudaMemcpyDeviceToDevice, s);
    if (e != cudaSuccess) return cuda_fail(e);
  }
  if (gates_out) {
    e = cudaMemcpyAsync(gates_out, gates, (size_t)p.R * 4, cudaMemcpyDeviceToDevice, s);
    if (e != cudaSuccess) return cuda_fail(e);
  }
  return MOE_OK;
}

// Per-workspace state of the host-buffer entry points: two non-blocking
// copy streams (input, output) and a few events (no device memory), created
// on the workspace's first host call and kept until moe_workspace_release(ws)
// or the process exits.
//
// x and y are each staged in two slots that alternate between calls, so the
// input copy of one call overlaps the whole of the previous call: the copy
// into a slot waits only for the end of the call before last (which read
// that slot). The asynchronous calls copy y out on the output stream, so
// that copy overlaps the next call too; a call writes a y slot only after
// the previous copy out of it has finished. That holds while the workspace
// layout stays the same; a call with another T or cfg (other offsets, which
// may overlap regions the previous call still uses), or any device-buffer
// call on the workspace in between, makes the copy wait for the end of the
// previous call (and its output copy) instead, and every device-buffer call
// on the workspace first waits for the output copies still pending.
struct HostPipe {
  int device = -1;
  cudaStream_t copy = nullptr;      // input copies
  cudaStream_t out = nullptr;       // output copies of the asynchronous calls
  cudaEvent_t x_ready = nullptr;    // the staged x of the current call has landed
  cudaEvent_t x_free[2] = {};       // the last call that used x slot i no longer reads it
  cudaEvent_t y_ready = nullptr;    // the current call's y is in its slot
  cudaEvent_t y_free[2] = {};       // the last copy out of y slot i has finished
  cudaEvent_t out_done = nullptr;   // the last asynchronous output copy has finished
  cudaEvent_t done = nullptr;       // end of the last call on this workspace (any entry point)
  bool slot_used[2] = {false, false};
  bool y_used[2] = {false, false};
  bool out_pending = false;         // an asynchronous output copy was issued (out_done recorded)
  bool done_recorded = false;
  bool relayout = true;             // next host call must wait for `done`
  size_t stage_key[5] = {};         // staging offsets and bytes of the last host call
  uint64_t calls = 0;
};
std::mutex g_pipe_mu;
std::unordered_map<const void*, HostPipe> g_pipes;

void destroy_pipe(HostPipe& hp) {
  // copies still in flight read or write the caller's buffers: let them end
  if (hp.copy) cudaStreamSynchronize(hp.copy);
  if (hp.out) cudaStreamSynchronize(hp.out);
  if (hp.copy) cudaStreamDestroy(hp.copy);
  if (hp.out) cudaStreamDestroy(hp.out);
  cudaEvent_t* ev[] = {&hp.x_ready, &hp.x_free[0], &hp.x_free[1], &hp.y_ready, &hp.y_free[0], &hp.y_free[1],
                       &hp.out_done, &hp.done};
  for (cudaEvent_t* e : ev)
    if (*e) cudaEventDestroy(*e);
  hp = HostPipe{};
}

cudaError_t host_pipe_locked(const void* ws, HostPipe** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  HostPipe& hp = g_pipes[ws];
  if (hp.device != dev) {
    if (hp.copy) destroy_pipe(hp);  // a different device reuses this address: start over
    e = cudaStreamCreateWithFlags(&hp.copy, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&hp.out, cudaStreamNonBlocking);
    cudaEvent_t* ev[] = {&hp.x_ready, &hp.x_free[0], &hp.x_free[1], &hp.y_ready, &hp.y_free[0], &hp.y_free[1],
                         &hp.out_done, &hp.done};
    for (cudaEvent_t* ep : ev)
      if (e == cudaSuccess) e = cudaEventCreateWithFlags(ep, cudaEventDisableTiming);
    if (e != cudaSuccess) {
      destroy_pipe(hp);
      return e;
    }
    hp.device = dev;
  }
  *out = &hp;
  return cudaSuccess;
}

// A device-buffer entry point is about to enqueue work on `s` that uses ws:
// if asynchronous host calls on this workspace have output copies that may
// still read it, `s` waits for them first. Copies that have already finished
// need no wait. A stream under graph capture is not made to wait (and the
// event is not queried, which a capture forbids): a capture must start only
// after the outputs have been waited for and their stream synchronised.
cudaError_t wait_host_outputs(const void* ws, cudaStream_t s) {
  std::lock_guard<std::mutex> lock(g_pipe_mu);
  auto it = g_pipes.find(ws);
  if (it == g_pipes.end() || !it->second.out_pending) return cudaSuccess;
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  cudaError_t e = cudaStreamIsCapturing(s, &cs);
  if (e != cudaSuccess || cs != cudaStreamCaptureStatusNone) return e;
  const cudaError_t q = cudaEventQuery(it->second.out_done);
  if (q == cudaSuccess) {
    it->second.out_pending = false;
    return cudaSuccess;
  }
  if (q != cudaErrorNotReady) return q;
  if (cudaPeekAtLastError() == cudaErrorNotReady) (void)cudaGetLastError();  // not an error: drop it
  return cudaStreamWaitEvent(s, it->second.out_done, 0);
}

// A device-buffer entry point (moe_route, moe_dispatch, moe_forward, ...) has
// enqueued work on `s` that uses ws: if the host-buffer calls have state for
// this workspace, mark the end of that work so the next host call's input
// copy waits for it (the copy runs on another stream).
cudaError_t note_device_use(const void* ws, cudaStream_t s) {
  std::lock_guard<std::mutex> lock(g_pipe_mu);
  auto it = g_pipes.find(ws);
  if (it == g_pipes.end() || !it->second.done) return cudaSuccess;
  it->second.relayout = true;
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  cudaError_t e = cudaStreamIsCapturing(s, &cs);
  if (e != cudaSuccess) return e;
  if (cs != cudaStreamCaptureStatusNone) {
    // work captured into a graph runs when the graph is launched: the caller
    // orders its replays with later host-buffer calls on this workspace
    it->second.done_recorded = false;
    return cudaSuccess;
  }
  it->second.done_recorded = true;
  return cudaEventRecord(it->second.done, s);
}

moe_status check_weights(const Problem& p, const void* W_r, const float* b, const void* W1,
                         const void* W3, const void* W2, const void* Ws1, const void* Ws3,
                         const void* Ws2) {
  if (!W_r || !W1 || !W3 || !W2) return MOE_ERR_INVALID_ARG;
  if (!aligned16(W_r) || !aligned16(W1) || !aligned16(W3) || !aligned16(W2)) return MOE_ERR_INVALID_ARG;
  if (b && (reinterpret_cast<uintptr_t>(b) & 3u)) return MOE_ERR_INVALID_ARG;
  if (p.ns > 0) {
    if (!Ws1 || !Ws3 || !Ws2) return MOE_ERR_INVALID_ARG;
    if (!aligned16(Ws1) || !aligned16(Ws3) || !aligned16(Ws2)) return MOE_ERR_INVALID_ARG;
  }
  return MOE_OK;
}

// moe_experts: a problem of E groups over `rows` grouped rows (no routing,
// no shared MLP); workspace regions and a device check of the counts.
moe_status make_group_problem(const moe_cfg* cfg, int64_t rows, Problem* p) {
  if (!cfg || !p || rows < 0) return MOE_ERR_INVALID_ARG;
  const moe_cfg& c = *cfg;
  if (c.d <= 0 || c.d_ff <= 0 || c.n_routed <= 0 || c.d % 8 || c.d_ff % 8) return MOE_ERR_INVALID_ARG;
  if (c.dtype != MOE_F32 && c.dtype != MOE_BF16) return MOE_ERR_INVALID_ARG;
  if (c.n_routed > kMaxRouted || (int64_t)c.n_routed * c.d_ff > (1ll << 31) ||
      (int64_t)c.n_routed * c.d > (1ll << 31) || rows > (1ll << 31) - 1)
    return MOE_ERR_UNSUPPORTED;
  Problem q{};
  q.T = rows;
  q.d = c.d;
  q.F = c.d_ff;
  q.N = c.n_routed;
  q.ns = 0;
  q.k = 1;
  q.G = 1;
  q.TG = 1;
  q.dtype = c.dtype;
  q.R = rows;
  q.nsF = 0;
  q.elem = c.dtype == MOE_BF16 ? 2 : 4;
  *p = q;
  return MOE_OK;
}

struct GroupLayout {
  size_t status, sched, counts_in, chunk_base, counts, offsets, grp_row0, grp_rows, unit_base1, unit_base2, h;
  size_t total;
};

GroupLayout make_group_layout(const Problem& p) {
  GroupLayout L{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t at = off;
    off = align256(off + bytes);
    return at;
  };
  const size_t N = (size_t)p.N;
  L.status = take(256);
  L.sched = take(256);
  L.counts_in = take(N * 4);
  L.chunk_base = take(N * 4);
  L.counts = take(N * 4);
  L.offsets = take((N + 1) * 4);
  L.grp_row0 = take((N + 1) * 4);
  L.grp_rows = take((N + 1) * 4);
  L.unit_base1 = take((N + 2) * 4);
  L.unit_base2 = take((N + 2) * 4);
  L.h = take((size_t)p.R * p.F * p.elem);
  L.total = off;
  return L;
}

// Copies the group counts into the workspace if they are non-negative and
// sum to `rows`; otherwise writes zeros (no group runs) and flags the status.
__global__ void check_counts_kernel(const int32_t* __restrict__ counts, int E, int64_t rows, int32_t* out,
                                    unsigned* status) {
  __shared__ unsigned long long total;
  __shared__ int bad;
  if (threadIdx.x == 0) {
    total = 0;
    bad = 0;
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    const int32_t c = counts[e];
    if (c < 0) atomicExch(&bad, 1);
    atomicAdd(&total, (unsigned long long)(c < 0 ? 0 : c));
  }
  __syncthreads();
  const bool ok = !bad && total == (unsigned long long)rows;
  for (int e = threadIdx.x; e < E; e += blockDim.x) out[e] = ok ? counts[e] : 0;
  if (threadIdx.x == 0 && !ok) set_status(status, MOE_DEV_BAD_EXPERT);
}

}  // namespace
// Configuration checks of the FP8 entry points.
moe_status check_fp8_cfg(const Problem& p) {
  if (p.dtype != MOE_BF16) return MOE_ERR_INVALID_ARG;
  constexpr int kBlock = 128, kMaxK = 8192;  // block size; K / 128 scale blocks per lane pair
  if (p.d % kBlock || p.F % kBlock || p.nsF % kBlock || p.d > kMaxK || p.F > kMaxK || p.nsF > kMaxK)
    return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

// Pointer checks of the FP8 entry points (codes of W1..Ws2 in m; the shared
// ones may be NULL iff n_shared == 0); fills the scale pointers.
moe_status check_fp8_ptrs(const Problem& p, const void* W_r, const float* b, const moe_fp8_matrix* const (&m)[6],
                          Fp8Scales* sc) {
  if (!W_r || !aligned16(W_r)) return MOE_ERR_INVALID_ARG;
  if (b && (reinterpret_cast<uintptr_t>(b) & 3u)) return MOE_ERR_INVALID_ARG;
  for (int i = 0; i < 6; ++i) {
    const bool need = i < 3 || p.ns > 0;
    sc->s[i] = nullptr;
    if (!need) continue;
    if (!m[i] || !m[i]->codes || !m[i]->scales || !aligned16(m[i]->codes)) return MOE_ERR_INVALID_ARG;
    sc->s[i] = m[i]->scales;
  }
  return MOE_OK;
}

const void* fp8_codes(const Problem& p, const moe_fp8_matrix* const (&m)[6], int i) {
  return (i < 3 || p.ns > 0) ? m[i]->codes : nullptr;
}

// The host-buffer pipeline of moe_forward_host(_fp8)(_async) around one
// device forward, run(x_device, y_device) on stream s: x is copied into one
// of the workspace's two input slots on the input stream (overlapping the
// previous call); y, written to one of two output slots, is copied back to
// the host on s, or on the output stream when `async_out` (overlapping the
// next call).
template <class Run>
moe_status forward_host_pipe(const Problem& p, const Layout& L, const void* x_host, void* y_host, void* ws,
                             cudaStream_t s, bool async_out, Run run) {
  const size_t bytes = (size_t)p.T * p.d * p.elem;
  std::lock_guard<std::mutex> lock(g_pipe_mu);
  HostPipe* hp = nullptr;
  cudaError_t e = host_pipe_locked(ws, &hp);
  if (e != cudaSuccess) return cuda_fail(e);
  const size_t key[5] = {L.x_stage[0], L.x_stage[1], L.y_stage[0], L.y_stage[1], bytes};
  if (std::memcmp(key, hp->stage_key, sizeof(key)) != 0) hp->relayout = true;
  if (hp->relayout) {
    // another layout (or device work) since the last host call: the copy may
    // land on regions the previous call still uses, so wait for all of it
    hp->slot_used[0] = hp->slot_used[1] = false;
    hp->y_used[0] = hp->y_used[1] = false;
    if (hp->done_recorded) e = cudaStreamWaitEvent(hp->copy, hp->done, 0);
    // and this call's copy and kernels may write where a pending output copy reads
    if (e == cudaSuccess && hp->out_pending) e = cudaStreamWaitEvent(hp->copy, hp->out_done, 0);
    if (e == cudaSuccess && hp->out_pending) e = cudaStreamWaitEvent(s, hp->out_done, 0);
    hp->calls = 0;
  }
  const int slot = (int)(hp->calls & 1u);
  void* xd = at<void>(ws, L.x_stage[slot]);
  void* yd = at<void>(ws, L.y_stage[slot]);
  if (e == cudaSuccess && hp->slot_used[slot]) e = cudaStreamWaitEvent(hp->copy, hp->x_free[slot], 0);
  if (e == cudaSuccess) e = cudaMemcpyAsync(xd, x_host, bytes, cudaMemcpyHostToDevice, hp->copy);
  if (e == cudaSuccess) e = cudaEventRecord(hp->x_ready, hp->copy);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(s, hp->x_ready, 0);
  // the y slot is written by this call's combine: its last copy out must be over
  if (e == cudaSuccess && hp->y_used[slot]) e = cudaStreamWaitEvent(s, hp->y_free[slot], 0);
  if (e != cudaSuccess) return cuda_fail(e);
  moe_status st = run(xd, yd);
  if (st != MOE_OK) return st;
  // the x slot is free again once this call's kernels are done
  if ((e = cudaEventRecord(hp->x_free[slot], s)) != cudaSuccess) return cuda_fail(e);
  hp->slot_used[slot] = true;
  if (async_out) {
    e = cudaEventRecord(hp->y_ready, s);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(hp->out, hp->y_ready, 0);
    if (e == cudaSuccess) e = cudaMemcpyAsync(y_host, yd, bytes, cudaMemcpyDeviceToHost, hp->out);
    if (e == cudaSuccess) e = cudaEventRecord(hp->y_free[slot], hp->out);
    if (e == cudaSuccess) e = cudaEventRecord(hp->out_done, hp->out);
    // the workspace is in use until the output copy ends
    if (e == cudaSuccess) e = cudaEventRecord(hp->done, hp->out);
    if (e == cudaSuccess) hp->out_pending = true;
  } else {
    e = cudaMemcpyAsync(y_host, yd, bytes, cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaEventRecord(hp->y_free[slot], s);
    if (e == cudaSuccess) e = cudaEventRecord(hp->done, s);
  }
  if (e != cudaSuccess) return cuda_fail(e);
  hp->y_used[slot] = true;
  hp->done_recorded = true;
  hp->relayout = false;
  std::memcpy(hp->stage_key, key, sizeof(key));
  ++hp->calls;
  return MOE_OK;
}

}  // namespace moe

using namespace moe;

extern "C" {

moe_status moe_workspace_size(const moe_cfg* cfg, int64_t T, size_t* bytes) {
  Problem p;
  moe_status st = make_problem(cfg, T, &p);
  if (st != MOE_OK) return st;
  if (!bytes) return MOE_ERR_INVALID_ARG;
  *bytes = make_layout(p).total;
  return MOE_OK;
}

moe_status moe_workspace_size_host(const moe_cfg* cfg, int64_t T, size_t* bytes) {
  Problem p;
  moe_status st = make_problem(cfg, T, &p);
  if (st != MOE_OK) return st;
  if (!bytes) return MOE_ERR_INVALID_ARG;
  *bytes = make_layout(p).total_host;
  return MOE_OK;
}

moe_status moe_route(const moe_cfg* cfg, int64_t T, const void* x, const void* W_r, const float* b,
                     int32_t* topk_idx, float* gates, void* ws, size_t ws_bytes, void* stream) {
  Problem p;
  moe_status st = make_problem(cfg, T, &p);
  if (st != MOE_OK) return st;
  if (T == 0) return MOE_OK;
  if (!x || !W_r || !topk_idx || !gates || !aligned16(x) || !aligned16(W_r)) return MOE_ERR_INVALID_ARG;
  Layout L = make_layout(p);
  if ((st = check_ws(L, ws, ws_bytes, L.total)) != MOE_OK) return st;
  cudaError_t e = wait_host_outputs(ws, (cudaStream_t)stream);
  if (e == cudaSuccess) e = cudaMemsetAsync(at<void>(ws, L.status), 0, 4, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e);
  if ((st = run_router(p, L, x, W_r, b, topk_idx, gates, ws, (cudaStream_t)stream)) != MOE_OK) return st;
  if ((e = note_device_use(ws, (cudaStream_t)stream)) != cudaSuccess) return cuda_fail(e);
  return MOE_OK;
}

moe_status moe_dispatch(const moe_cfg* cfg, int64_t T, const int32_t* topk_idx, int32_t* counts,
                        int32_t* offsets, int32_t* perm, void* ws, size_t ws_bytes, void* stream) {
  Problem p;
  moe_status st = make_problem(cfg, T, &p);
  if (st != MOE_OK) return st;
  if (T == 0) return MOE_OK;
  if (!topk_idx) return MOE_ERR_INVALID_ARG;
  Layout L = make_layout(p);
  if ((st = check_ws(L, ws, ws_bytes, L.total)) != MOE_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;
  DispatchBuffers db = dispatch_buffers(L, ws, topk_idx, nullptr);
  const bool tc = p.dtype == MOE_BF16;
  cudaError_t e = wait_host_outputs(ws, s);
  if (e == cudaSuccess) e = cudaMemsetAsync(db.status, 0, 4, s);
  if (e != cudaSuccess) return cuda_fail(e);
  e = launch_dispatch(p, db, tc ? kTcBM : kSimtBM, tc ? kTcBN1 : kSimtBN,
                                  tc ? kTcBN2 : kSimtBN, s);
  if (e != cudaSuccess) return cuda_fail(e);
  if (counts && (e = cudaMemcpyAsync(counts, db.counts, (size_t)p.N * 4, cudaMemcpyDeviceToDevice, s)))
    return cuda_fail(e);
  if (offsets &&
      (e = cudaMemcpyAsync(offsets, db.offsets, (size_t)(p.N + 1) * 4, cudaMemcpyDeviceToDevice, s)))
    return cuda_fail(e);
  if (perm && (e = cudaMemcpyAsync(perm, db.perm, (size_t)p.R * 4, cudaMemcpyDeviceToDevice, s)))
    return cuda_fail(e);
  if ((e = note_device_use(ws, s)) != cudaSuccess) return cuda_fail(e);
  return MOE_OK;
}

moe_status moe_forward(const moe_cfg* cfg, int64_t T, const void* x, const void* W_r, const float* b,
                       const void* W1, const void* W3, const void* W2, const void* Ws1,
                       const void* Ws3, const void* Ws2, void* y, int32_t* topk_idx_out,
                       float* gates_out, void* ws, size_t ws_bytes, void* stream) {
  Problem p;
  moe_status st = make_problem(cfg, T, &p);
  if (st != MOE_OK) return st;
  if (T == 0) return MOE_OK;
  if (!x || !y || !aligned16(x) || !aligned16(y)) return MOE_ERR_INVALID_ARG;
  if ((st = check_weights(p, W_r, b, W1, W3, W2, Ws1, Ws3, Ws2)) != MOE_OK) return st;
  Layout L = make_layout(p);
  if ((st = check_ws(L, ws, ws_bytes, L.total)) != MOE_OK) return st;
  cudaError_t e0 = wait_host_outputs(ws, (cudaStream_t)stream);
  if (e0 != cudaSuccess) return cuda_fail(e0);
  st = forward_device(p, L, x, W_r, b, W1, W3, W2, Ws1, Ws3, Ws2, y, topk_idx_out, gates_out, ws,
                      (cudaStream_t)stream);
  if (st != MOE_OK) return st;
  cudaError_t e = note_device_use(ws, (cudaStream_t)stream);
  return e == cudaSuccess ? MOE_OK : cuda_fail(e);
}

moe_status moe_forward_fp8(const moe_cfg* cfg, int64_t T, const void* x, const void* W_r, const float* b,
                           const moe_fp8_matrix* W1, const moe_fp8_matrix* W3, const moe_fp8_matrix* W2,
                           const moe_fp8_matrix* Ws1, const moe_fp8_matrix* Ws3, const moe_fp8_matrix* Ws2,
                           void* y, int32_t* topk_idx_out, float* gates_out, void* ws, size_t ws_bytes,
                           void* stream) {
  Problem p;
  moe_status st = make_problem(cfg, T, &p);
  if (st != MOE_OK) return st;
  if ((st = check_fp8_cfg(p)) != MOE_OK) return st;
  if (T == 0) return MOE_OK;
  if (!x || !y || !aligned16(x) || !aligned16(y)) return MOE_ERR_INVALID_ARG;
  const moe_fp8_matrix* m[6] = {W1, W3, W2, Ws1, Ws3, Ws2};
  Fp8Scales sc{};
  if ((st = check_fp8_ptrs(p, W_r, b, m, &sc)) != MOE_OK) return st;
  Layout L = make_layout(p);
  if ((st = check_ws(L, ws, ws_bytes, L.total)) != MOE_OK) return st;
  cudaError_t e0 = wait_host_outputs(ws, (cudaStream_t)stream);
  if (e0 != cudaSuccess) return cuda_fail(e0);
  st = forward_device(p, L, x, W_r, b, fp8_codes(p, m, 0), fp8_codes(p, m, 1), fp8_codes(p, m, 2),
                      fp8_codes(p, m, 3), fp8_codes(p, m, 4), fp8_codes(p, m, 5), y, topk_idx_out, gates_out, ws,
                      (cudaStream_t)stream, &sc);
  if (st != MOE_OK) return st;
  cudaError_t e = note_device_use(ws, (cudaStream_t)stream);
  return e == cudaSuccess ? MOE_OK : cuda_fail(e);
}

}  // extern "C"

namespace moe {
namespace {

moe_status forward_host_bf16(const moe_cfg* cfg, int64_t T, const void* x_host, const void* W_r, const float* b,
                             const void* W1, const void* W3, const void* W2, const void* Ws1, const void* Ws3,
                             const void* Ws2, void* y_host, void* ws, size_t ws_bytes, void* stream,
                             bool async_out) {
  Problem p;
  moe_status st = make_problem(cfg, T, &p);
  if (st != MOE_OK) return st;
  if (T == 0) return MOE_OK;
  if (!x_host || !y_host) return MOE_ERR_INVALID_ARG;
  if ((st = check_weights(p, W_r, b, W1, W3, W2, Ws1, Ws3, Ws2)) != MOE_OK) return st;
  Layout L = make_layout(p);
  if ((st = check_ws(L, ws, ws_bytes, L.total_host)) != MOE_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;
  return forward_host_pipe(p, L, x_host, y_host, ws, s, async_out, [&](const void* xd, void* yd) {
    return forward_device(p, L, xd, W_r, b, W1, W3, W2, Ws1, Ws3, Ws2, yd, nullptr, nullptr, ws, s);
  });
}

moe_status forward_host_fp8(const moe_cfg* cfg, int64_t T, const void* x_host, const void* W_r, const float* b,
                            const moe_fp8_matrix* W1, const moe_fp8_matrix* W3, const moe_fp8_matrix* W2,
                            const moe_fp8_matrix* Ws1, const moe_fp8_matrix* Ws3, const moe_fp8_matrix* Ws2,
                            void* y_host, void* ws, size_t ws_bytes, void* stream, bool async_out) {
  Problem p;
  moe_status st = make_problem(cfg, T, &p);
  if (st != MOE_OK) return st;
  if ((st = check_fp8_cfg(p)) != MOE_OK) return st;
  if (T == 0) return MOE_OK;
  if (!x_host || !y_host) return MOE_ERR_INVALID_ARG;
  const moe_fp8_matrix* m[6] = {W1, W3, W2, Ws1, Ws3, Ws2};
  Fp8Scales sc{};
  if ((st = check_fp8_ptrs(p, W_r, b, m, &sc)) != MOE_OK) return st;
  Layout L = make_layout(p);
  if ((st = check_ws(L, ws, ws_bytes, L.total_host)) != MOE_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;
  return forward_host_pipe(p, L, x_host, y_host, ws, s, async_out, [&](const void* xd, void* yd) {
    return forward_device(p, L, xd, W_r, b, fp8_codes(p, m, 0), fp8_codes(p, m, 1), fp8_codes(p, m, 2),
                          fp8_codes(p, m, 3), fp8_codes(p, m, 4), fp8_codes(p, m, 5), yd, nullptr, nullptr, ws, s,
                          &sc);
  });
}

}  // namespace
}  // namespace moe

extern "C" {

moe_status moe_forward_host(const moe_cfg* cfg, int64_t T, const void* x_host, const void* W_r,
                            const float* b, const void* W1, const void* W3, const void* W2,
                            const void* Ws1, const void* Ws3, const void* Ws2, void* y_host,
                            void* ws, size_t ws_bytes, void* stream) {
  return forward_host_bf16(cfg, T, x_host, W_r, b, W1, W3, W2, Ws1, Ws3, Ws2, y_host, ws, ws_bytes, stream, false);
}

moe_status moe_forward_host_async(const moe_cfg* cfg, int64_t T, const void* x_host, const void* W_r,
                                  const float* b, const void* W1, const void* W3, const void* W2,
                                  const void* Ws1, const void* Ws3, const void* Ws2, void* y_host,
                                  void* ws, size_t ws_bytes, void* stream) {
  return forward_host_bf16(cfg, T, x_host, W_r, b, W1, W3, W2, Ws1, Ws3, Ws2, y_host, ws, ws_bytes, stream, true);
}

moe_status moe_forward_host_fp8(const moe_cfg* cfg, int64_t T, const void* x_host, const void* W_r,
                                const float* b, const moe_fp8_matrix* W1, const moe_fp8_matrix* W3,
                                const moe_fp8_matrix* W2, const moe_fp8_matrix* Ws1, const moe_fp8_matrix* Ws3,
                                const moe_fp8_matrix* Ws2, void* y_host, void* ws, size_t ws_bytes,
                                void* stream) {
  return forward_host_fp8(cfg, T, x_host, W_r, b, W1, W3, W2, Ws1, Ws3, Ws2, y_host, ws, ws_bytes, stream, false);
}

moe_status moe_forward_host_fp8_async(const moe_cfg* cfg, int64_t T, const void* x_host, const void* W_r,
                                      const float* b, const moe_fp8_matrix* W1, const moe_fp8_matrix* W3,
                                      const moe_fp8_matrix* W2, const moe_fp8_matrix* Ws1,
                                      const moe_fp8_matrix* Ws3, const moe_fp8_matrix* Ws2, void* y_host,
                                      void* ws, size_t ws_bytes, void* stream) {
  return forward_host_fp8(cfg, T, x_host, W_r, b, W1, W3, W2, Ws1, Ws3, Ws2, y_host, ws, ws_bytes, stream, true);
}

moe_status moe_host_wait(const void* ws, void* stream) {
  cudaError_t e = wait_host_outputs(ws, (cudaStream_t)stream);
  return e == cudaSuccess ? MOE_OK : cuda_fail(e);
}

moe_status moe_workspace_release(const void* ws) {
  std::lock_guard<std::mutex> lock(g_pipe_mu);
  auto it = g_pipes.find(ws);
  if (it == g_pipes.end()) return MOE_OK;
  int cur = -1;
  cudaError_t e = cudaGetDevice(&cur);
  if (e == cudaSuccess && it->second.device >= 0 && cur != it->second.device) e = cudaSetDevice(it->second.device);
  if (e != cudaSuccess) return cuda_fail(e);
  destroy_pipe(it->second);
  g_pipes.erase(it);
  if (cur >= 0) cudaSetDevice(cur);
  return MOE_OK;
}

moe_status moe_dispatch_rows(const moe_cfg* cfg, int64_t T, const int32_t* topk_idx, const float* gates,
                             const void* x, int32_t* counts, int32_t* offsets, int32_t* slot_pos, void* x_perm,
                             float* gate_perm, void* ws, size_t ws_bytes, void* stream) {
  Problem p;
  moe_status st = make_problem(cfg, T, &p);
  if (st != MOE_OK) return st;
  if (T == 0) return MOE_OK;
  if (!topk_idx || !gates || !x || !counts || !offsets || !slot_pos || !x_perm || !gate_perm) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(x_perm)) return MOE_ERR_INVALID_ARG;
  Layout L = make_layout(p);
  if ((st = check_ws(L, ws, ws_bytes, L.total)) != MOE_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;
  DispatchBuffers db = dispatch_buffers(L, ws, topk_idx, gates);
  db.counts = counts;
  db.offsets = offsets;
  db.slot_pos = slot_pos;
  db.gate_perm = gate_perm;
  const bool tc = p.dtype == MOE_BF16;
  cudaError_t e = wait_host_outputs(ws, s);
  if (e == cudaSuccess) e = cudaMemsetAsync(db.status, 0, 4, s);
  if (e == cudaSuccess)
    e = launch_dispatch(p, db, tc ? kTcBM : kSimtBM, tc ? kTcBN1 : kSimtBN, tc ? kTcBN2 : kSimtBN, s);
  if (e == cudaSuccess) e = launch_gather(p, x, slot_pos, x_perm, db.status, s);
  if (e == cudaSuccess) e = note_device_use(ws, s);
  return e == cudaSuccess ? MOE_OK : cuda_fail(e);
}

moe_status moe_experts_workspace_size(const moe_cfg* cfg, int64_t rows, size_t* bytes) {
  Problem p;
  moe_status st = make_group_problem(cfg, rows, &p);
  if (st != MOE_OK) return st;
  if (!bytes) return MOE_ERR_INVALID_ARG;
  *bytes = make_group_layout(p).total;
  return MOE_OK;
}

moe_status moe_experts(const moe_cfg* cfg, int64_t rows, const int32_t* counts, const void* x_rows,
                       const float* gate_rows, const void* W1, const void* W3, const void* W2, void* y_rows,
                       void* ws, size_t ws_bytes, void* stream) {
  Problem p;
  moe_status st = make_group_problem(cfg, rows, &p);
  if (st != MOE_OK) return st;
  if (rows == 0) return MOE_OK;
  if (!counts || !x_rows || !y_rows || !W1 || !W3 || !W2) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x_rows) || !aligned16(y_rows) || !aligned16(W1) || !aligned16(W3) || !aligned16(W2))
    return MOE_ERR_INVALID_ARG;
  if (gate_rows && (reinterpret_cast<uintptr_t>(gate_rows) & 3u)) return MOE_ERR_INVALID_ARG;
  const GroupLayout L = make_group_layout(p);
  if (!ws || ws_bytes < L.total || (reinterpret_cast<uintptr_t>(ws) & 255u)) return MOE_ERR_WORKSPACE;
  cudaStream_t s = (cudaStream_t)stream;
  unsigned* status = at<unsigned>(ws, L.status);
  cudaError_t e = wait_host_outputs(ws, s);
  if (e == cudaSuccess) e = cudaMemsetAsync(status, 0, 4, s);
  if (e != cudaSuccess) return cuda_fail(e);
  check_counts_kernel<<<1, 256, 0, s>>>(counts, p.N, rows, at<int32_t>(ws, L.counts_in), status);
  if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e);
  DispatchBuffers db{};
  db.chunk_base = at<int32_t>(ws, L.chunk_base);
  db.counts = at<int32_t>(ws, L.counts);
  db.offsets = at<int32_t>(ws, L.offsets);
  db.grp_row0 = at<int32_t>(ws, L.grp_row0);
  db.grp_rows = at<int32_t>(ws, L.grp_rows);
  db.unit_base1 = at<int32_t>(ws, L.unit_base1);
  db.unit_base2 = at<int32_t>(ws, L.unit_base2);
  const bool tc = p.dtype == MOE_BF16;
  e = launch_unit_tables(p, at<int32_t>(ws, L.counts_in), db, tc ? kTcBM : kSimtBM, tc ? kTcBN1 : kSimtBN,
                         tc ? kTcBN2 : kSimtBN, s);
  if (e != cudaSuccess) return cuda_fail(e);
  GemmArgs ga;
  ga.x = nullptr;
  ga.x_perm = x_rows;
  ga.W1 = W1;
  ga.W3 = W3;
  ga.W2 = W2;
  ga.Ws1 = ga.Ws3 = ga.Ws2 = nullptr;
  ga.h_perm = at<void>(ws, L.h);
  ga.h_sh = nullptr;
  ga.y_rows = y_rows;
  ga.grp_row0 = db.grp_row0;
  ga.grp_rows = db.grp_rows;
  ga.unit_base1 = db.unit_base1;
  ga.unit_base2 = db.unit_base2;
  ga.gate_perm = gate_rows;
  ga.status = status;
  ga.sched = at<int>(ws, L.sched);
  e = tc ? launch_expert_gemms_tc(p, ga, s, nullptr) : launch_expert_gemms_simt(p, ga, s, nullptr);
  if (e == cudaSuccess) e = note_device_use(ws, s);
  return e == cudaSuccess ? MOE_OK : cuda_fail(e);
}

moe_status moe_combine(const moe_cfg* cfg, int64_t T, const void* routed_rows, const int32_t* slot_pos,
                       const void* shared_rows, void* y, void* stream) {
  Problem p;
  moe_status st = make_problem(cfg, T, &p);
  if (st != MOE_OK) return st;
  if (T == 0) return MOE_OK;
  if (!routed_rows || !slot_pos || !y || !aligned16(routed_rows) || !aligned16(y)) return MOE_ERR_INVALID_ARG;
  if (shared_rows && !aligned16(shared_rows)) return MOE_ERR_INVALID_ARG;
  cudaError_t e = launch_combine_rows(p, routed_rows, shared_rows, slot_pos, y, (cudaStream_t)stream);
  return e == cudaSuccess ? MOE_OK : cuda_fail(e);
}

moe_status moe_ep_reorder(int32_t world, int32_t local_experts, const int32_t* counts, int64_t row_bytes,
                          const void* src, void* dst, int32_t to_expert_major, void* stream) {
  if (world <= 0 || local_experts <= 0 || (int64_t)world * local_experts > (1 << 20) || row_bytes <= 0 ||
      row_bytes % 4 || !counts || !src || !dst || src == dst || !aligned16(src) || !aligned16(dst))
    return MOE_ERR_INVALID_ARG;
  cudaError_t e = launch_ep_reorder(counts, world, local_experts, row_bytes, src, dst, to_expert_major != 0,
                                    (cudaStream_t)stream);
  return e == cudaSuccess ? MOE_OK : cuda_fail(e);
}

moe_status moe_device_status(const moe_cfg* cfg, int64_t T, void* ws, size_t ws_bytes, int clear,
                             uint32_t* bits, void* stream) {
  Problem p;
  moe_status st = make_problem(cfg, T, &p);
  if (st != MOE_OK) return st;
  if (!bits) return MOE_ERR_INVALID_ARG;
  Layout L = make_layout(p);
  if ((st = check_ws(L, ws, ws_bytes, 256)) != MOE_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;
  uint32_t host = 0;
  cudaError_t e = cudaMemcpyAsync(&host, at<void>(ws, L.status), 4, cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e);
  if (clear) {
    e = cudaMemsetAsync(at<void>(ws, L.status), 0, 4, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return cuda_fail(e);
  }
  *bits = host;
  return host ? MOE_ERR_DEVICE : MOE_OK;
}

const char* moe_status_string(moe_status status) {
  switch (status) {
    case MOE_OK: return "MOE_OK";
    case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG";
    case MOE_ERR_UNSUPPORTED: return "MOE_ERR_UNSUPPORTED";
    case MOE_ERR_WORKSPACE: return "MOE_ERR_WORKSPACE";
    case MOE_ERR_CUDA: return "MOE_ERR_CUDA";
    case MOE_ERR_DEVICE: return "MOE_ERR_DEVICE";
  }
  return "MOE_ERR_UNKNOWN";
}

int32_t moe_last_cuda_error(void) { return g_last_cuda_error; }

moe_status moe_set_stage_events(void* const* events, int32_t n) {
  if (n == 0) {
    g_stage_events_on = false;
    return MOE_OK;
  }
  if (n != kStageEvents || !events) return MOE_ERR_INVALID_ARG;
  for (int i = 0; i < kStageEvents; ++i) {
    if (!events[i]) return MOE_ERR_INVALID_ARG;
    g_stage_events[i] = static_cast<cudaEvent_t>(events[i]);
  }
  g_stage_events_on = true;
  return MOE_OK;
}

}  // extern "C"
