"""B200 (sm_100a) DeepSeekMoE layer forward: thin Python binding of the C ABI
in include/moe_b200.h.

Argument marshalling only: every step of the layer runs in the CUDA kernels of
libmoe_b200.so. PyTorch tensors are accepted for device memory and streams;
their data pointers are handed to the C entry points, which enqueue work on
the given (or current) CUDA stream. There is no fallback: if the library is
missing or the call fails, an exception is raised.
"""
from __future__ import annotations

import contextlib
import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe_b200.so")

MOE_F32, MOE_BF16 = 0, 1
MOE_SOFTMAX, MOE_SIGMOID = 0, 1
MOE_GROUP_TOP2_SUM, MOE_GROUP_MAX = 0, 1
MOE_DEV_WAIT_TIMEOUT, MOE_DEV_BAD_EXPERT, MOE_DEV_DUP_EXPERT, MOE_DEV_TMEM_ALLOC, MOE_DEV_NONFINITE = 1, 2, 4, 8, 16
STATUS_NAMES = {0: "MOE_OK", 1: "MOE_ERR_INVALID_ARG", 2: "MOE_ERR_UNSUPPORTED", 3: "MOE_ERR_WORKSPACE",
                4: "MOE_ERR_CUDA", 5: "MOE_ERR_DEVICE"}
EXPORTS = ["moe_workspace_size", "moe_workspace_size_host", "moe_route", "moe_dispatch", "moe_forward",
           "moe_forward_fp8", "moe_dispatch_rows", "moe_experts_workspace_size", "moe_experts", "moe_combine",
           "moe_ep_reorder",
           "moe_forward_host", "moe_forward_host_fp8", "moe_forward_host_async", "moe_forward_host_fp8_async",
           "moe_host_wait", "moe_workspace_release", "moe_device_status", "moe_set_stage_events", "moe_route_noalloc", "moe_bias_update", "moe_selftest_wait_timeout",
           "moe_status_string", "moe_last_cuda_error"]
STAGES = ["router", "dispatch", "gather", "gemm_swiglu", "gemm_gate", "combine"]


class MoeCfg(ctypes.Structure):
    """moe_cfg of the C ABI (field order and types must match the header)."""

    _fields_ = [("d", ctypes.c_int32), ("d_ff", ctypes.c_int32), ("n_routed", ctypes.c_int32),
                ("n_shared", ctypes.c_int32), ("top_k", ctypes.c_int32), ("n_groups", ctypes.c_int32),
                ("topk_groups", ctypes.c_int32), ("score_fn", ctypes.c_int32),
                ("normalize", ctypes.c_int32), ("route_scale", ctypes.c_float),
                ("group_score", ctypes.c_int32), ("dtype", ctypes.c_int32)]


class Fp8Matrix(ctypes.Structure):
    """moe_fp8_matrix of the C ABI: e4m3 codes and UE8M0 scales per 128 x 128 block."""

    _fields_ = [("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p)]


class MoeError(RuntimeError):
    def __init__(self, call: str, status: int, cuda_error: int = 0):
        self.status = status
        self.cuda_error = cuda_error
        msg = f"{call} failed: {STATUS_NAMES.get(status, status)}"
        if cuda_error:
            msg += f" (cudaError {cuda_error})"
        super().__init__(msg)


_lib = None
DEBUG_LIB_PATH = os.path.join(_HERE, "libmoe_b200_debug.so")


@contextlib.contextmanager
def using_library(path: str):
    """Route every call of the binding through the library at `path` (e.g.
    DEBUG_LIB_PATH, the bounds-checked build) inside the with-block."""
    global _lib, LIB_PATH
    saved = (_lib, LIB_PATH)
    _lib, LIB_PATH = None, path
    try:
        yield lib()
    finally:
        _lib, LIB_PATH = saved


def lib() -> ctypes.CDLL:
    """The loaded CUDA library; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} not found: build it with "
                               "`python -m mixture_experts_layer_group_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, I64, SZ = ctypes.c_void_p, ctypes.c_int64, ctypes.c_size_t
        CFG = ctypes.POINTER(MoeCfg)
        L.moe_workspace_size.argtypes = [CFG, I64, ctypes.POINTER(SZ)]
        L.moe_workspace_size_host.argtypes = [CFG, I64, ctypes.POINTER(SZ)]
        L.moe_route.argtypes = [CFG, I64, P, P, P, P, P, P, SZ, P]
        L.moe_dispatch.argtypes = [CFG, I64, P, P, P, P, P, SZ, P]
        L.moe_forward.argtypes = [CFG, I64, P, P, P, P, P, P, P, P, P, P, P, P, P, SZ, P]
        L.moe_dispatch_rows.argtypes = [CFG, I64, P, P, P, P, P, P, P, P, P, SZ, P]
        L.moe_experts_workspace_size.argtypes = [CFG, I64, ctypes.POINTER(SZ)]
        L.moe_experts.argtypes = [CFG, I64, P, P, P, P, P, P, P, P, SZ, P]
        L.moe_combine.argtypes = [CFG, I64, P, P, P, P, P]
        L.moe_ep_reorder.argtypes = [ctypes.c_int32, ctypes.c_int32, P, I64, P, P, ctypes.c_int32, P]
        FP8P = ctypes.POINTER(Fp8Matrix)
        L.moe_forward_fp8.argtypes = [CFG, I64, P, P, P, FP8P, FP8P, FP8P, FP8P, FP8P, FP8P, P, P, P, P, SZ, P]
        L.moe_forward_host.argtypes = [CFG, I64, P, P, P, P, P, P, P, P, P, P, P, SZ, P]
        L.moe_forward_host_fp8.argtypes = [CFG, I64, P, P, P, FP8P, FP8P, FP8P, FP8P, FP8P, FP8P, P, P, SZ, P]
        L.moe_forward_host_async.argtypes = L.moe_forward_host.argtypes
        L.moe_forward_host_fp8_async.argtypes = L.moe_forward_host_fp8.argtypes
        L.moe_host_wait.argtypes = [P, P]
        L.moe_workspace_release.argtypes = [P]
        L.moe_device_status.argtypes = [CFG, I64, P, SZ, ctypes.c_int, ctypes.POINTER(ctypes.c_uint32), P]
        L.moe_set_stage_events.argtypes = [ctypes.POINTER(ctypes.c_void_p), ctypes.c_int32]
        L.moe_route_noalloc.argtypes = [CFG, I64, P, P, P, P, P, P]
        L.moe_bias_update.argtypes = [CFG, I64, P, ctypes.c_float, P, P]
        L.moe_selftest_wait_timeout.argtypes = [ctypes.POINTER(ctypes.c_uint32), P]
        L.moe_status_string.argtypes = [ctypes.c_int]
        L.moe_status_string.restype = ctypes.c_char_p
        L.moe_last_cuda_error.argtypes = []
        L.moe_last_cuda_error.restype = ctypes.c_int32
        for name in EXPORTS:
            if name not in ("moe_status_string", "moe_last_cuda_error"):
                getattr(L, name).restype = ctypes.c_int
        _lib = L
    return _lib


_SCORES = {"softmax": MOE_SOFTMAX, "sigmoid": MOE_SIGMOID}
_GROUP_SCORES = {"top2_sum": MOE_GROUP_TOP2_SUM, "max": MOE_GROUP_MAX}
_DTYPES = {"bf16": MOE_BF16, "f32": MOE_F32}


def _lookup(table: dict, what: str, value: str) -> int:
    try:
        return table[value]
    except KeyError:
        raise ValueError(f"unknown {what} {value!r}; expected one of {sorted(table)}") from None


def make_cfg(d, d_ff, n_routed, n_shared, top_k, n_groups=1, topk_groups=1, score="softmax",
             normalize=False, route_scale=1.0, group_score="top2_sum", dtype="bf16") -> MoeCfg:
    """moe_cfg from Python values; an unknown score, group_score or dtype
    string raises ValueError instead of falling back to a default."""
    return MoeCfg(d, d_ff, n_routed, n_shared, top_k, n_groups, topk_groups, _lookup(_SCORES, "score", score),
                  int(bool(normalize)), float(route_scale), _lookup(_GROUP_SCORES, "group_score", group_score),
                  _lookup(_DTYPES, "dtype", dtype))


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(call: str, rc: int):
    if rc != 0:
        raise MoeError(call, rc, lib().moe_last_cuda_error() if rc == 4 else 0)


def workspace_size(cfg: MoeCfg, T: int) -> int:
    n = ctypes.c_size_t(0)
    _check("moe_workspace_size", lib().moe_workspace_size(ctypes.byref(cfg), T, ctypes.byref(n)))
    return n.value


def workspace_size_host(cfg: MoeCfg, T: int) -> int:
    n = ctypes.c_size_t(0)
    _check("moe_workspace_size_host", lib().moe_workspace_size_host(ctypes.byref(cfg), T, ctypes.byref(n)))
    return n.value


def route(cfg, T, x, W_r, b, topk_idx, gates, ws, ws_bytes=None, stream=None):
    ws_bytes = ws.numel() * ws.element_size() if ws_bytes is None else ws_bytes
    _check("moe_route", lib().moe_route(ctypes.byref(cfg), T, _ptr(x), _ptr(W_r), _ptr(b), _ptr(topk_idx),
                                        _ptr(gates), _ptr(ws), ws_bytes, _stream(stream)))


def route_noalloc(cfg, T, x, W_r, b, topk_idx, gates, stream=None):
    """moe_route without a workspace: for callers that cannot allocate device
    scratch. Uses a fixed 8 MiB array inside the library (T * n_routed * 4
    bytes at most); calls that overlap on the GPU race on it."""
    _check("moe_route_noalloc", lib().moe_route_noalloc(ctypes.byref(cfg), T, _ptr(x), _ptr(W_r), _ptr(b),
                                                        _ptr(topk_idx), _ptr(gates), _stream(stream)))


def bias_update(cfg, T, counts, gamma, b, stream=None):
    """Auxiliary-loss-free balancing step: b[e] -= gamma where counts[e] exceeds
    the mean load T * top_k / N, += gamma where it falls short (in place)."""
    _check("moe_bias_update", lib().moe_bias_update(ctypes.byref(cfg), T, _ptr(counts), float(gamma), _ptr(b),
                                                    _stream(stream)))


def selftest_wait_timeout(stream=None) -> int:
    """Runs the bounded-wait self-check (about 1 s) and returns the device
    status bits it recorded (MOE_DEV_WAIT_TIMEOUT when the wait gave up)."""
    bits = ctypes.c_uint32(0)
    _check("moe_selftest_wait_timeout", lib().moe_selftest_wait_timeout(ctypes.byref(bits), _stream(stream)))
    return bits.value


def dispatch(cfg, T, topk_idx, counts, offsets, perm, ws, ws_bytes=None, stream=None):
    ws_bytes = ws.numel() * ws.element_size() if ws_bytes is None else ws_bytes
    _check("moe_dispatch", lib().moe_dispatch(ctypes.byref(cfg), T, _ptr(topk_idx), _ptr(counts),
                                              _ptr(offsets), _ptr(perm), _ptr(ws), ws_bytes,
                                              _stream(stream)))


def forward(cfg, T, x, W_r, b, W1, W3, W2, Ws1, Ws3, Ws2, y, ws, topk_idx_out=None, gates_out=None,
            ws_bytes=None, stream=None):
    ws_bytes = ws.numel() * ws.element_size() if ws_bytes is None else ws_bytes
    _check("moe_forward", lib().moe_forward(ctypes.byref(cfg), T, _ptr(x), _ptr(W_r), _ptr(b), _ptr(W1),
                                            _ptr(W3), _ptr(W2), _ptr(Ws1), _ptr(Ws3), _ptr(Ws2), _ptr(y),
                                            _ptr(topk_idx_out), _ptr(gates_out), _ptr(ws), ws_bytes,
                                            _stream(stream)))


def _fp8(m):
    """(codes, scales) tensors -> a moe_fp8_matrix pointer (None stays NULL)."""
    if m is None:
        return None
    codes, scales = m
    return ctypes.pointer(Fp8Matrix(_ptr(codes), _ptr(scales)))


def forward_fp8(cfg, T, x, W_r, b, W1, W3, W2, Ws1, Ws3, Ws2, y, ws, topk_idx_out=None, gates_out=None,
                ws_bytes=None, stream=None):
    """moe_forward with FP8 expert weights; each of W1 .. Ws2 is a (codes, scales)
    pair of uint8 tensors (e4m3 codes [rows, cols], UE8M0 scales [rows/128, cols/128])."""
    ws_bytes = ws.numel() * ws.element_size() if ws_bytes is None else ws_bytes
    _check("moe_forward_fp8", lib().moe_forward_fp8(ctypes.byref(cfg), T, _ptr(x), _ptr(W_r), _ptr(b), _fp8(W1),
                                                    _fp8(W3), _fp8(W2), _fp8(Ws1), _fp8(Ws3), _fp8(Ws2), _ptr(y),
                                                    _ptr(topk_idx_out), _ptr(gates_out), _ptr(ws), ws_bytes,
                                                    _stream(stream)))


def dispatch_rows(cfg, T, topk_idx, gates, x, counts, offsets, slot_pos, x_perm, gate_perm, ws, ws_bytes=None,
                  stream=None):
    """moe_dispatch plus the permuted token rows and their gates (expert parallelism, step 2)."""
    ws_bytes = ws.numel() * ws.element_size() if ws_bytes is None else ws_bytes
    _check("moe_dispatch_rows", lib().moe_dispatch_rows(ctypes.byref(cfg), T, _ptr(topk_idx), _ptr(gates), _ptr(x),
                                                        _ptr(counts), _ptr(offsets), _ptr(slot_pos), _ptr(x_perm),
                                                        _ptr(gate_perm), _ptr(ws), ws_bytes, _stream(stream)))


def experts_workspace_size(cfg: MoeCfg, rows: int) -> int:
    n = ctypes.c_size_t(0)
    _check("moe_experts_workspace_size", lib().moe_experts_workspace_size(ctypes.byref(cfg), rows, ctypes.byref(n)))
    return n.value


def experts(cfg, rows, counts, x_rows, gate_rows, W1, W3, W2, y_rows, ws, ws_bytes=None, stream=None):
    """Grouped SwiGLU experts over rows grouped by expert (counts[e] rows each, in order)."""
    ws_bytes = ws.numel() * ws.element_size() if ws_bytes is None else ws_bytes
    _check("moe_experts", lib().moe_experts(ctypes.byref(cfg), rows, _ptr(counts), _ptr(x_rows), _ptr(gate_rows),
                                            _ptr(W1), _ptr(W3), _ptr(W2), _ptr(y_rows), _ptr(ws), ws_bytes,
                                            _stream(stream)))


def combine(cfg, T, routed_rows, slot_pos, shared_rows, y, stream=None):
    """y[t] = sum of the token's permuted rows (ascending expert) + shared_rows[t] (None for none)."""
    _check("moe_combine", lib().moe_combine(ctypes.byref(cfg), T, _ptr(routed_rows), _ptr(slot_pos),
                                            _ptr(shared_rows), _ptr(y), _stream(stream)))


def ep_reorder(world, local_experts, counts, row_bytes, src, dst, to_expert_major, stream=None):
    """Rows between source-major and expert-major order of the blocks counts[world, local_experts]."""
    _check("moe_ep_reorder", lib().moe_ep_reorder(world, local_experts, _ptr(counts), row_bytes, _ptr(src), _ptr(dst),
                                                  int(bool(to_expert_major)), _stream(stream)))


def forward_host(cfg, T, x_host, W_r, b, W1, W3, W2, Ws1, Ws3, Ws2, y_host, ws, ws_bytes=None,
                 stream=None):
    ws_bytes = ws.numel() * ws.element_size() if ws_bytes is None else ws_bytes
    _check("moe_forward_host", lib().moe_forward_host(ctypes.byref(cfg), T, _ptr(x_host), _ptr(W_r), _ptr(b),
                                                      _ptr(W1), _ptr(W3), _ptr(W2), _ptr(Ws1), _ptr(Ws3),
                                                      _ptr(Ws2), _ptr(y_host), _ptr(ws), ws_bytes,
                                                      _stream(stream)))


def forward_host_fp8(cfg, T, x_host, W_r, b, W1, W3, W2, Ws1, Ws3, Ws2, y_host, ws, ws_bytes=None,
                     stream=None):
    """moe_forward_host with FP8 expert weights ((codes, scales) pairs as in forward_fp8)."""
    ws_bytes = ws.numel() * ws.element_size() if ws_bytes is None else ws_bytes
    _check("moe_forward_host_fp8", lib().moe_forward_host_fp8(ctypes.byref(cfg), T, _ptr(x_host), _ptr(W_r),
                                                              _ptr(b), _fp8(W1), _fp8(W3), _fp8(W2), _fp8(Ws1),
                                                              _fp8(Ws3), _fp8(Ws2), _ptr(y_host), _ptr(ws),
                                                              ws_bytes, _stream(stream)))


def forward_host_async(cfg, T, x_host, W_r, b, W1, W3, W2, Ws1, Ws3, Ws2, y_host, ws, ws_bytes=None,
                       stream=None):
    """moe_forward_host with the output copy on the workspace's own stream:
    y_host is complete after a later host_wait(ws, stream) has been reached."""
    ws_bytes = ws.numel() * ws.element_size() if ws_bytes is None else ws_bytes
    _check("moe_forward_host_async",
           lib().moe_forward_host_async(ctypes.byref(cfg), T, _ptr(x_host), _ptr(W_r), _ptr(b), _ptr(W1), _ptr(W3),
                                        _ptr(W2), _ptr(Ws1), _ptr(Ws3), _ptr(Ws2), _ptr(y_host), _ptr(ws), ws_bytes,
                                        _stream(stream)))


def forward_host_fp8_async(cfg, T, x_host, W_r, b, W1, W3, W2, Ws1, Ws3, Ws2, y_host, ws, ws_bytes=None,
                           stream=None):
    """forward_host_async with FP8 expert weights."""
    ws_bytes = ws.numel() * ws.element_size() if ws_bytes is None else ws_bytes
    _check("moe_forward_host_fp8_async",
           lib().moe_forward_host_fp8_async(ctypes.byref(cfg), T, _ptr(x_host), _ptr(W_r), _ptr(b), _fp8(W1),
                                            _fp8(W3), _fp8(W2), _fp8(Ws1), _fp8(Ws3), _fp8(Ws2), _ptr(y_host),
                                            _ptr(ws), ws_bytes, _stream(stream)))


def host_wait(ws, stream=None) -> None:
    """Order `stream` after every output copy the asynchronous host calls issued on ws."""
    _check("moe_host_wait", lib().moe_host_wait(_ptr(ws), _stream(stream)))


def workspace_release(ws) -> None:
    """Free the copy streams and events the host-buffer calls keep for this
    workspace (blocks until their copies in flight have finished)."""
    _check("moe_workspace_release", lib().moe_workspace_release(_ptr(ws)))


def device_status(cfg, T, ws, clear=True, ws_bytes=None, stream=None) -> int:
    """MOE_DEV_* bits recorded by the kernels of the last call on this workspace (synchronises)."""
    ws_bytes = ws.numel() * ws.element_size() if ws_bytes is None else ws_bytes
    bits = ctypes.c_uint32(0)
    rc = lib().moe_device_status(ctypes.byref(cfg), T, _ptr(ws), ws_bytes, int(clear), ctypes.byref(bits),
                                 _stream(stream))
    if rc not in (0, 5):
        _check("moe_device_status", rc)
    return bits.value


def set_stage_events(events) -> None:
    """Attach 7 CUDA events (torch.cuda.Event(enable_timing=True), already
    recorded once so their handles exist) to be recorded at the stage
    boundaries of later forward calls on this thread; None detaches."""
    if events is None:
        _check("moe_set_stage_events", lib().moe_set_stage_events(None, 0))
        return
    arr = (ctypes.c_void_p * len(events))(*[e.cuda_event if hasattr(e, "cuda_event") else e for e in events])
    _check("moe_set_stage_events", lib().moe_set_stage_events(arr, len(events)))


def status_string(status: int) -> str:
    return lib().moe_status_string(status).decode()


class MoELayer:
    """A DeepSeekMoE layer bound to device-resident weights and a workspace.

    weights: dict with W_r, b (or None), W1, W3, W2 and, when n_shared > 0,
    Ws1, Ws3, Ws2 -- torch CUDA tensors in the layouts of the C ABI. Expert
    weights given as (codes, scales) pairs of uint8 tensors are FP8 (e4m3 with
    a power-of-two scale per 128 x 128 block) and run through
    moe_forward_fp8 / moe_forward_host_fp8.
    """

    def __init__(self, cfg: MoeCfg, weights: dict, max_tokens: int, device="cuda", host_io=False):
        import torch
        self.cfg = cfg
        self.w = weights
        self.max_tokens = max_tokens
        nbytes = (workspace_size_host if host_io else workspace_size)(cfg, max_tokens)
        self.ws = torch.empty(nbytes, dtype=torch.uint8, device=device)

    def _wargs(self):
        w = self.w
        return (w["W_r"], w.get("b"), w["W1"], w["W3"], w["W2"], w.get("Ws1"), w.get("Ws3"), w.get("Ws2"))

    @property
    def fp8(self) -> bool:
        return isinstance(self.w["W1"], (tuple, list))

    def __call__(self, x, y=None, topk_idx_out=None, gates_out=None, stream=None):
        import torch
        T = x.shape[0]
        assert T <= self.max_tokens
        if y is None:
            y = torch.empty_like(x)
        fwd = forward_fp8 if self.fp8 else forward
        fwd(self.cfg, T, x, *self._wargs(), y, self.ws, topk_idx_out, gates_out, stream=stream)
        return y

    def forward_host(self, x_host, y_host, stream=None, wait=True):
        """x_host in, y_host out (pinned host tensors). With wait=False the
        output copy runs on the workspace's own stream and overlaps the next
        call; y_host is then complete after a later host_wait()."""
        T = x_host.shape[0]
        assert T <= self.max_tokens
        if wait:
            fwd = forward_host_fp8 if self.fp8 else forward_host
        else:
            fwd = forward_host_fp8_async if self.fp8 else forward_host_async
        fwd(self.cfg, T, x_host, *self._wargs(), y_host, self.ws, stream=stream)
        return y_host

    def host_wait(self, stream=None) -> None:
        host_wait(self.ws, stream)

    def device_status(self, T=None, stream=None) -> int:
        return device_status(self.cfg, self.max_tokens if T is None else T, self.ws, stream=stream)
