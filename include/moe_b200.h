/*
 * moe_b200.h -- C ABI of the B200 (sm_100a) DeepSeekMoE layer forward.
 *
 * The layer (a DeepSeekMoE feed-forward block, as listed step by step on the
 * "DeepSeek-V3.2-Exp · Mixture of experts" page, section "All 19 steps"):
 *
 *   router    z = x W_r^T            one logit per routed expert
 *             s = softmax(z) | sigmoid(z)
 *             selection: top_k of s + b, restricted to the topk_groups best
 *             of n_groups contiguous expert groups ("top-8 of s+b within the
 *             top 4 groups"); b only steers the selection
 *             gates G = route_scale * s / sum(s over the selection)  (normalize)
 *                   G = route_scale * s                             (otherwise,
 *             the GShard router of the "DeepSeekMoE" walkthrough, Step 2)
 *   experts   E_e(x) = W2_e (silu(W1_e x) * (W3_e x))      fine-grained SwiGLU
 *   shared    y_shared = Ws2 (silu(Ws1 x) * (Ws3 x))       always on, ungated
 *   output    y = sum_e G_e E_e(x) + y_shared              (no residual)
 *
 * Tokens are one flattened axis of T rows (batch and positions folded
 * together, as the page's quoted MoE.forward does). No token is dropped and
 * no expert has a capacity limit.
 *
 * Conventions shared by every entry point
 *   - All tensors are dense row-major in device memory (HBM), element type
 *     cfg->dtype (fp32 or bf16) unless stated; every base pointer must be
 *     16-byte aligned; d and d_ff must be multiples of 8.
 *   - The caller owns every buffer. The library allocates no device memory:
 *     scratch lives in a caller-provided workspace of moe_workspace_size()
 *     bytes (256-byte aligned).
 *   - cfg is read on the host during the call only.
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *     stream) and the call returns without synchronising. Results are ready
 *     when the stream has drained.
 *   - Errors are returned as moe_status values; nothing is thrown across the
 *     ABI. Launch failures return MOE_ERR_CUDA, and the CUDA error code is
 *     kept per host thread for moe_last_cuda_error(). Failures detected on the
 *     device (a pipeline wait that timed out, an out-of-range expert index)
 *     are recorded in a status word inside the workspace; read it with
 *     moe_device_status().
 *   - T == 0 is a valid no-op returning MOE_OK.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum moe_status {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,  /* bad cfg, null or misaligned pointer, negative T */
  MOE_ERR_UNSUPPORTED = 2,  /* valid layer outside what this build implements */
  MOE_ERR_WORKSPACE = 3,    /* workspace null or smaller than moe_workspace_size() */
  MOE_ERR_CUDA = 4,         /* a CUDA runtime call or kernel launch failed */
  MOE_ERR_DEVICE = 5        /* moe_device_status() found a device-side failure */
} moe_status;

enum { MOE_F32 = 0, MOE_BF16 = 1 };                 /* moe_cfg.dtype */
enum { MOE_SOFTMAX = 0, MOE_SIGMOID = 1 };          /* moe_cfg.score_fn */
enum { MOE_GROUP_TOP2_SUM = 0, MOE_GROUP_MAX = 1 }; /* moe_cfg.group_score */

/* Device-status bits (moe_device_status). */
enum {
  MOE_DEV_WAIT_TIMEOUT = 1u << 0,   /* a bounded pipeline wait gave up */
  MOE_DEV_BAD_EXPERT = 1u << 1,     /* an expert index outside [0, n_routed) */
  MOE_DEV_DUP_EXPERT = 1u << 2,     /* a token lists the same expert twice */
  MOE_DEV_TMEM_ALLOC = 1u << 3,     /* tensor-memory allocation returned no columns */
  MOE_DEV_NONFINITE = 1u << 4       /* a token's router logits or keys were NaN or infinite
                                       (non-finite x, W_r or b); it still gets top_k distinct
                                       experts in [0, n_routed), chosen arbitrarily, and the
                                       other tokens are unaffected */,
  MOE_DEV_BOUNDS = 1u << 5          /* a bounds check of the debug build (compiled with
                                       -DMOE_DEBUG_BOUNDS, libmoe_b200_debug.so) failed; the
                                       checked access was skipped. Never set by the release build */
};

/*
 * Layer configuration. Field names follow the page's model arguments
 * (dim, moe_inter_dim, n_routed_experts, n_shared_experts,
 * n_activated_experts) and the router steps.
 *   d            model dimension (dim)
 *   d_ff         width of one routed expert (moe_inter_dim)
 *   n_routed     N, routed experts (1..512)
 *   n_shared     shared experts, fused into one MLP of width n_shared*d_ff
 *   top_k        experts selected per token (1..16, <= topk_groups*N/n_groups)
 *   n_groups     expert groups (1 = no group limit); must divide n_routed
 *   topk_groups  groups kept per token (1..n_groups)
 *   score_fn     MOE_SOFTMAX or MOE_SIGMOID
 *   normalize    nonzero: gates normalised over the selection, then scaled
 *   route_scale  gate multiplier (2.5 for the DeepSeek-V3 layer, 1 for GShard)
 *   group_score  how a group is scored for the group limit: the sum of its
 *                two largest s+b (MOE_GROUP_TOP2_SUM) or its largest (MOE_GROUP_MAX)
 *   dtype        MOE_F32 (SIMT fp32 path) or MOE_BF16 (tensor-core expert GEMMs; the
 *                router runs on the FP32 pipes for both)
 */
typedef struct moe_cfg {
  int32_t d;
  int32_t d_ff;
  int32_t n_routed;
  int32_t n_shared;
  int32_t top_k;
  int32_t n_groups;
  int32_t topk_groups;
  int32_t score_fn;
  int32_t normalize;
  float route_scale;
  int32_t group_score;
  int32_t dtype;
} moe_cfg;

/*
 * Bytes of device workspace that moe_route, moe_dispatch and moe_forward
 * need for T tokens. Returns MOE_ERR_INVALID_ARG for an invalid cfg or
 * T < 0, MOE_ERR_UNSUPPORTED outside the implemented range.
 */
MOE_API moe_status moe_workspace_size(const moe_cfg* cfg, int64_t T, size_t* bytes);

/*
 * Router only (the "Router:" steps of the equation list).
 *   x        [T, d]      tokens, cfg->dtype
 *   W_r      [N, d]      one router row per routed expert, cfg->dtype
 *   b        [N] fp32    selection bias, or NULL for none
 *   topk_idx [T, top_k] int32 out: selected experts, slots in descending s+b
 *   gates    [T, top_k] fp32  out: gate of each slot (from the unbiased s)
 * Logits are accumulated in fp32 with fp64 partial-sum carries; selection
 * breaks exact ties toward the lower group / expert index.
 */
MOE_API moe_status moe_route(const moe_cfg* cfg, int64_t T, const void* x, const void* W_r, const float* b,
                     int32_t* topk_idx, float* gates, void* ws, size_t ws_bytes, void* stream);

/*
 * Expert histogram and expert-contiguous token lists (the quoted forward's
 * bincount over the selected indices and its per-expert token lists).
 *   topk_idx [T, top_k] int32 in (as written by moe_route)
 *   counts   [N] int32 out: (token, slot) pairs per expert
 *   offsets  [N+1] int32 out: exclusive prefix sum of counts
 *   perm     [T*top_k] int32 out: perm[offsets[e] + r] = t*top_k + slot of
 *            the r-th pair that chose e, tokens ascending (bit-exact, no
 *            order-dependent atomics)
 * Any output pointer may be NULL to skip copying it out. An index outside
 * [0, N) or a repeated expert within one token sets a device-status bit.
 */
MOE_API moe_status moe_dispatch(const moe_cfg* cfg, int64_t T, const int32_t* topk_idx, int32_t* counts,
                        int32_t* offsets, int32_t* perm, void* ws, size_t ws_bytes, void* stream);

/*
 * The whole layer forward: y = Delta_ffn.
 *   x            [T, d]
 *   W_r, b       as for moe_route
 *   W1, W3       [N, d_ff, d]        routed experts, stacked (out x in)
 *   W2           [N, d, d_ff]
 *   Ws1, Ws3     [n_shared*d_ff, d]  fused shared MLP; NULL iff n_shared == 0
 *   Ws2          [d, n_shared*d_ff]
 *   y            [T, d] out, cfg->dtype (fp32 accumulation, one rounding)
 *   topk_idx_out, gates_out  optional [T, top_k] copies of the routing (NULL to skip)
 * bf16 path: expert matmuls on tcgen05 tensor cores (bf16 x bf16 -> fp32),
 * SwiGLU output and gated expert rows rounded to bf16, combine in fp32 in
 * ascending expert order. fp32 path: the same steps on CUDA cores in fp32.
 * Deterministic: two calls on the same inputs give the same bits.
 */
MOE_API moe_status moe_forward(const moe_cfg* cfg, int64_t T, const void* x, const void* W_r, const float* b,
                       const void* W1, const void* W3, const void* W2, const void* Ws1,
                       const void* Ws3, const void* Ws2, void* y, int32_t* topk_idx_out,
                       float* gates_out, void* ws, size_t ws_bytes, void* stream);

/*
 * One expert weight matrix in FP8: e4m3 codes with one power-of-two scale
 * per 128 x 128 block, the block-scaled FP8 layout of DeepSeek-V3-style
 * checkpoints (the "DeepSeek-V3.2-Exp · Mixture of experts" page, Parameters:
 * the checkpoint carries FP8 block scales). Element (r, c) has the value
 *   e4m3(codes[r * cols + c]) * 2^(scales[(r / 128) * (cols / 128) + c / 128] - 127)
 * with e4m3 the OCP FP8 E4M3 format (1 sign, 4 exponent bits with bias 7, 3
 * mantissa bits, no infinities, 0x7F / 0xFF NaN, largest finite 448) and the
 * scale byte a UE8M0 exponent.
 *   codes   [rows, cols] uint8, row-major, 16-byte aligned
 *   scales  [rows / 128, cols / 128] uint8
 * For the routed experts the matrices are stacked as in moe_forward (W1, W3:
 * rows = n_routed * d_ff, cols = d; W2: rows = n_routed * d, cols = d_ff).
 */
typedef struct moe_fp8_matrix {
  const void* codes;
  const uint8_t* scales;
} moe_fp8_matrix;

/*
 * moe_forward with FP8 expert weights (routed and shared): the same layer,
 * tokens, router (W_r bf16), outputs and workspace as moe_forward with
 * cfg->dtype == MOE_BF16. Each weight tile is dequantised exactly to bf16 in
 * tensor memory (a power-of-two scale times an e4m3 value is a bf16 value)
 * and multiplied on the tensor cores as in the bf16 path, so the result
 * equals moe_forward run on the dequantised weights (bit for bit, as long as
 * every dequantised weight is a normal bf16 number). Weight bytes streamed
 * from HBM are halved.
 * Requires d, d_ff and n_shared * d_ff to be multiples of 128 and at most
 * 8192 (MOE_ERR_UNSUPPORTED otherwise) and cfg->dtype == MOE_BF16
 * (MOE_ERR_INVALID_ARG otherwise). Ws1 / Ws3 / Ws2 are NULL iff n_shared == 0.
 */
MOE_API moe_status moe_forward_fp8(const moe_cfg* cfg, int64_t T, const void* x, const void* W_r, const float* b,
                                   const moe_fp8_matrix* W1, const moe_fp8_matrix* W3, const moe_fp8_matrix* W2,
                                   const moe_fp8_matrix* Ws1, const moe_fp8_matrix* Ws3,
                                   const moe_fp8_matrix* Ws2, void* y, int32_t* topk_idx_out, float* gates_out,
                                   void* ws, size_t ws_bytes, void* stream);

/*
 * moe_forward with the token rows in host memory: copies x_host [T, d] to
 * the device inside the workspace, runs the layer, and copies y back to
 * y_host [T, d], all enqueued on `stream`. Host buffers should be pinned
 * (cudaHostAlloc / cudaHostRegister) for the copies to be asynchronous; the
 * caller synchronises the stream before reading y_host. Weights stay in
 * device memory. Needs moe_workspace_size_host() bytes of workspace.
 * The host-to-device copy runs on a copy stream the library keeps for the
 * workspace (with a second stream for moe_forward_host_async's output copies
 * and eight events, no device memory; created on the first host call on that
 * workspace, freed by moe_workspace_release or at process exit). x and y are
 * each staged in two slots used by alternate calls, so back-to-back calls
 * with the same T and cfg overlap one call's input copy with the whole of
 * the previous call. A call with another T or cfg, or one that follows a
 * device-buffer call (moe_route, moe_dispatch, moe_forward, ...) on the same
 * workspace, waits for the previous call to finish before copying (its
 * staging area may then overlap buffers that call still uses). The output
 * copy stays on `stream`. All calls on one workspace must be ordered: issue
 * them on one stream, or order the streams yourself.
 */
MOE_API moe_status moe_workspace_size_host(const moe_cfg* cfg, int64_t T, size_t* bytes);
MOE_API moe_status moe_forward_host(const moe_cfg* cfg, int64_t T, const void* x_host, const void* W_r,
                            const float* b, const void* W1, const void* W3, const void* W2,
                            const void* Ws1, const void* Ws3, const void* Ws2, void* y_host,
                            void* ws, size_t ws_bytes, void* stream);

/*
 * moe_forward_host with the output copy off `stream`: the forward is
 * enqueued on `stream` as in moe_forward_host, and y is copied from its
 * staging slot to y_host on the workspace's output stream once the forward
 * has written it. A run of calls then overlaps each call's input copy with
 * the previous call and its output copy with the next call, so it proceeds
 * at the rate of the forward alone. y_host is complete only after a later
 * moe_host_wait(ws, s) has been reached by a stream s (synchronise s, or
 * wait on an event recorded after it, before reading y_host); until then the
 * caller must neither read nor free it. x_host may be reused once `stream`
 * has passed the call, as with moe_forward_host. A slot's y is overwritten
 * two calls later only after its copy out has finished, and every
 * device-buffer entry point on the workspace (and a host call with another
 * T or cfg) first waits for the output copies still pending, so calls of
 * both kinds can be mixed on one workspace. Copies that have finished need
 * no wait. A CUDA graph capture of device-buffer calls on the workspace may
 * start once the outputs have been waited for and their stream synchronised,
 * not while copies are in flight (a capture records no wait on them), and the
 * caller orders the graph's replays with later host-buffer calls on the same
 * workspace. Same arguments, workspace size and errors as moe_forward_host.
 */
MOE_API moe_status moe_forward_host_async(const moe_cfg* cfg, int64_t T, const void* x_host, const void* W_r,
                                          const float* b, const void* W1, const void* W3, const void* W2,
                                          const void* Ws1, const void* Ws3, const void* Ws2, void* y_host,
                                          void* ws, size_t ws_bytes, void* stream);

/*
 * Makes `stream` wait (on the device, without blocking the host) until every
 * output copy that moe_forward_host_async / moe_forward_host_fp8_async have
 * issued on the workspace at `ws` so far has finished. Returns at once (and
 * MOE_OK) when the workspace has no asynchronous output copies or they have
 * already finished, and records nothing while `stream` is being captured
 * into a CUDA graph (wait for the copies before the capture starts).
 * Errors: MOE_ERR_CUDA from the stream query or wait.
 */
MOE_API moe_status moe_host_wait(const void* ws, void* stream);

/*
 * Frees the copy streams and events that the host-buffer calls keep for the
 * workspace at `ws` (nothing happens if it has none). Call it before freeing
 * or reusing that memory for another purpose; it blocks until the copies
 * still queued on those streams (which read or write the caller's host
 * buffers) have finished. The workspace memory itself belongs to the caller.
 * Errors: MOE_ERR_CUDA if the workspace's device cannot be made current.
 */
MOE_API moe_status moe_workspace_release(const void* ws);

/*
 * moe_forward_host with FP8 expert weights: the x and y host buffers,
 * staging, ordering and copy stream of moe_forward_host around the device
 * forward of moe_forward_fp8 (same weights arguments, requirements and
 * results). The workspace is sized by moe_workspace_size_host; the per-
 * workspace state is shared with moe_forward_host and freed by
 * moe_workspace_release. moe_forward_host_fp8_async is the same with the
 * output copy of moe_forward_host_async (y_host complete after a later
 * moe_host_wait).
 */
MOE_API moe_status moe_forward_host_fp8(const moe_cfg* cfg, int64_t T, const void* x_host, const void* W_r,
                                const float* b, const moe_fp8_matrix* W1, const moe_fp8_matrix* W3,
                                const moe_fp8_matrix* W2, const moe_fp8_matrix* Ws1,
                                const moe_fp8_matrix* Ws3, const moe_fp8_matrix* Ws2, void* y_host,
                                void* ws, size_t ws_bytes, void* stream);
MOE_API moe_status moe_forward_host_fp8_async(const moe_cfg* cfg, int64_t T, const void* x_host,
                                              const void* W_r, const float* b, const moe_fp8_matrix* W1,
                                              const moe_fp8_matrix* W3, const moe_fp8_matrix* W2,
                                              const moe_fp8_matrix* Ws1, const moe_fp8_matrix* Ws3,
                                              const moe_fp8_matrix* Ws2, void* y_host, void* ws,
                                              size_t ws_bytes, void* stream);

/*
 * Reads (and optionally clears) the device-status word of a workspace used
 * for T tokens with cfg: synchronises `stream`, writes the MOE_DEV_* bits
 * to *bits, and returns MOE_ERR_DEVICE when any bit is set.
 */
MOE_API moe_status moe_device_status(const moe_cfg* cfg, int64_t T, void* ws, size_t ws_bytes, int clear,
                             uint32_t* bits, void* stream);

/*
 * Stage timing hook for profilers and benchmarks. With n == 7, every later
 * moe_forward / moe_forward_host call on this host thread records
 * events[0..6] (cudaEvent_t handles owned by the caller, created on the
 * stream's device) on its stream at the stage boundaries: before the
 * router, after the router, after dispatch, after the row gather, after
 * the SwiGLU GEMM, after the gate GEMM and after the combine. n == 0
 * detaches. Any other n returns MOE_ERR_INVALID_ARG.
 */
MOE_API moe_status moe_set_stage_events(void* const* events, int32_t n);

/*
 * Router that allocates nothing and takes no workspace. The pages have no
 * counterpart to this call; it exists for callers that cannot allocate
 * device memory for scratch -- a plugin whose host framework owns all device
 * memory and passes it no workspace, or a serving loop with a fixed memory
 * budget that must not call cudaMalloc (which can synchronise the device)
 * once it runs.
 *   Same arguments and outputs as moe_route, without ws/ws_bytes, and the
 *     same results bit for bit: the logits are reduced in the same K ranges
 *     as moe_route's (when moe_route's partial logits for all T tokens do not
 *     fit the array, the router runs over slices of the tokens in turn).
 *   Scratch: the fp32 logits go to a fixed 8 MiB array inside the library,
 *     reserved on every GPU that loads the library until the process exits.
 *     T * n_routed * 4 > 8 MiB (for example T > 8192 at n_routed = 256)
 *     returns MOE_ERR_UNSUPPORTED before any device work; use moe_route
 *     with a workspace for those sizes.
 *   Set-up: the first call on a device (with that device current) looks up
 *     the array's device address and caches it; make that first call before
 *     any stream capture. It never calls cudaMalloc, cudaFree or any other
 *     allocating routine. The cached address belongs to the device's
 *     current primary context: after cudaDeviceReset() on a device, this
 *     call must not be used on that device again in the same process.
 *   Sharing: every call on a device uses the same array and leaves the last
 *     call's logits in it (each call overwrites every value it reads, so
 *     nothing needs clearing). Calls whose work overlaps on the GPU -- on
 *     different streams, or from different host threads -- race on the
 *     array and may return wrong routing: serialise them, e.g. on one stream.
 */
MOE_API moe_status moe_route_noalloc(const moe_cfg* cfg, int64_t T, const void* x, const void* W_r,
                                     const float* b, int32_t* topk_idx, float* gates, void* stream);

/*
 * Auxiliary-loss-free load balancing: the per-batch bias nudge (grasp.study
 * lesson on DeepSeek-V3's MoE design, section "3.2. Auxiliary-Loss-Free Load
 * Balancing"; "The DeepSeekMoE Architecture.", configuration table row
 * "balancing: aux-loss-free bias"). For every routed expert e:
 *   b[e] -= gamma  if counts[e] > T * top_k / N   (overloaded)
 *   b[e] += gamma  if counts[e] < T * top_k / N   (underloaded)
 *   unchanged      otherwise
 * (the comparison is exact, in integers; the update is one fp32 add).
 *   counts [N] int32 in, device: the batch's (token, slot) pairs per expert,
 *          as moe_dispatch writes them for the same T
 *   gamma  the update rate (the pages give none; DeepSeek-V3 style values are
 *          around 1e-3); must be finite
 *   b      [N] fp32 in/out, device: the selection bias that moe_route and
 *          moe_forward read
 * Asynchronous on `stream`; no workspace; b is updated in place.
 * Errors: MOE_ERR_INVALID_ARG for a bad cfg, null or misaligned pointers or a
 * non-finite gamma; MOE_ERR_CUDA for a failed launch.
 */
MOE_API moe_status moe_bias_update(const moe_cfg* cfg, int64_t T, const int32_t* counts, float gamma, float* b,
                                   void* stream);

/*
 * Expert parallelism: the layer spread over W ranks (one process per GPU),
 * rank r holding routed experts [r N / W, (r + 1) N / W) as in the page's
 * quoted MoE.__init__ (experts sliced per rank), the router and the shared
 * MLP on every rank. A rank's step (driven by the caller, who owns the
 * all-to-all exchanges -- NCCL through torch.distributed in the package):
 *   1. moe_route on its own tokens;
 *   2. moe_dispatch_rows: expert histogram, expert-contiguous permutation,
 *      the permuted token rows and their gates (rows for rank q's experts are
 *      the contiguous range offsets[q E] .. offsets[(q + 1) E]);
 *   3. exchange the per-expert counts and the rows (all-to-all);
 *   4. moe_ep_reorder to expert-major order, moe_experts on the local
 *      experts, moe_ep_reorder back;
 *   5. exchange the gated rows back (all-to-all);
 *   6. moe_experts for the shared MLP on its own tokens, then moe_combine.
 * Every row is computed as in moe_forward, so each rank's y equals
 * moe_forward's on the same tokens bit for bit.
 */

/*
 * moe_dispatch plus the permuted rows: counts [N], offsets [N+1] (as
 * moe_dispatch), slot_pos [T, top_k] (the permuted row of each of a token's
 * experts, ascending expert; -1 for an invalid index), x_perm [T*top_k, d]
 * (token rows in permuted order, cfg->dtype) and gate_perm [T*top_k] fp32
 * (the gate of each permuted row, from gates [T, top_k]). All device
 * buffers owned by the caller; workspace as for moe_workspace_size(cfg, T).
 */
MOE_API moe_status moe_dispatch_rows(const moe_cfg* cfg, int64_t T, const int32_t* topk_idx, const float* gates,
                                     const void* x, int32_t* counts, int32_t* offsets, int32_t* slot_pos,
                                     void* x_perm, float* gate_perm, void* ws, size_t ws_bytes, void* stream);

/*
 * Grouped SwiGLU experts over rows already grouped by expert: the two
 * tensor-core GEMMs of moe_forward (fp32 SIMT GEMMs for MOE_F32), without
 * routing or combine. cfg supplies d, d_ff, dtype and n_routed = the number
 * of groups E (1..512); its routing fields are ignored.
 *   counts    [E] int32, device: rows of each group, in order; they must
 *             sum to `rows` (checked on the device: otherwise no group is
 *             computed and moe_device_status reports MOE_DEV_BAD_EXPERT)
 *   x_rows    [rows, d]; gate_rows [rows] fp32 or NULL (gate 1)
 *   W1, W3    [E, d_ff, d]; W2 [E, d, d_ff]
 *   y_rows    [rows, d] out: gate * W2 (silu(W1 x) * W3 x) of each row
 * Workspace: moe_experts_workspace_size(cfg, rows) bytes (the device-status
 * word at its start is read by moe_device_status(cfg, rows, ...)).
 */
MOE_API moe_status moe_experts_workspace_size(const moe_cfg* cfg, int64_t rows, size_t* bytes);
MOE_API moe_status moe_experts(const moe_cfg* cfg, int64_t rows, const int32_t* counts, const void* x_rows,
                               const float* gate_rows, const void* W1, const void* W3, const void* W2, void* y_rows,
                               void* ws, size_t ws_bytes, void* stream);

/*
 * y[t] = sum over the token's permuted rows slot_pos[t, 0..top_k)
 * (ascending expert; -1 skipped) of routed_rows, plus shared_rows[t] (NULL
 * for none), accumulated in fp32 in that order and rounded once.
 *   routed_rows [T*top_k, d] in moe_dispatch_rows' permuted order
 */
MOE_API moe_status moe_combine(const moe_cfg* cfg, int64_t T, const void* routed_rows, const int32_t* slot_pos,
                               const void* shared_rows, void* y, void* stream);

/*
 * Reorders rows between source-major order (blocks (p, e): rank p major,
 * local expert e minor -- what an all-to-all delivers) and expert-major
 * order (e major, p minor -- what moe_experts reads); to_expert_major
 * selects the direction. counts [world, local_experts] int32, device: rows
 * of each block. row_bytes must be a multiple of 4; src and dst 16-byte
 * aligned, distinct buffers.
 */
MOE_API moe_status moe_ep_reorder(int32_t world, int32_t local_experts, const int32_t* counts, int64_t row_bytes,
                                  const void* src, void* dst, int32_t to_expert_major, void* stream);

/*
 * Self-check of the failure path (no counterpart in the pages): launches a
 * one-warp kernel that waits, with the same bounded wait every pipeline in
 * the library uses, on a barrier that nothing ever completes. After the wait
 * limit (1 s) the kernel records MOE_DEV_WAIT_TIMEOUT and returns; the call
 * synchronises `stream` and writes the recorded bits to *bits (expected:
 * MOE_DEV_WAIT_TIMEOUT). The CUDA context stays usable. Takes about 1 s.
 * Calls from different host threads of one process are serialised inside
 * the library (they share one status word per device).
 * Errors: MOE_ERR_INVALID_ARG for a null bits; MOE_ERR_CUDA for a failed
 * launch or copy.
 */
MOE_API moe_status moe_selftest_wait_timeout(uint32_t* bits, void* stream);

/* Human-readable name of a status code (static storage). */
MOE_API const char* moe_status_string(moe_status status);

/* cudaError_t value of the last MOE_ERR_CUDA on this host thread (0 if none). */
MOE_API int32_t moe_last_cuda_error(void);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
