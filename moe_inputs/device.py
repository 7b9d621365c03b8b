"""Device-side fill of the seeded inputs (same bits as the host generator).

Uses torch only to own the HBM buffers and the stream; the values are written
by the generator kernel in ``gen_device.cu``.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np
import torch

from . import (DEVICE_LIB, FP8_BLOCK, TID, TID_SCALE, LayerShape, dims_of, f32_to_bf16, factor_of, fp8_e0,
               mat_dims, zipf_offsets)

_dev = None


def _device_lib():
    global _dev
    if _dev is None:
        if not os.path.exists(DEVICE_LIB):
            raise RuntimeError(f"{DEVICE_LIB} is missing: run moe_inputs.build.build_device()")
        lib = ctypes.CDLL(DEVICE_LIB)
        lib.gen_normal_device.argtypes = [ctypes.c_uint32, ctypes.c_uint32, ctypes.c_uint64,
                                          ctypes.c_uint64, ctypes.c_double, ctypes.c_int,
                                          ctypes.c_void_p, ctypes.c_void_p]
        lib.gen_uniform_device.argtypes = [ctypes.c_uint32, ctypes.c_uint32, ctypes.c_uint64,
                                           ctypes.c_uint64, ctypes.c_double, ctypes.c_double,
                                           ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p]
        lib.gen_fp8_device.argtypes = [ctypes.c_uint32, ctypes.c_uint32, ctypes.c_uint32, ctypes.c_int,
                                       ctypes.c_uint64, ctypes.c_uint64, ctypes.c_uint64, ctypes.c_double,
                                       ctypes.c_void_p, ctypes.c_void_p]
        lib.gen_fp8_scales_device.argtypes = [ctypes.c_uint32, ctypes.c_uint32, ctypes.c_int, ctypes.c_uint64,
                                              ctypes.c_uint64, ctypes.c_void_p, ctypes.c_void_p]
        _dev = lib
    return _dev


def storage_dtype(shape: LayerShape) -> torch.dtype:
    return torch.bfloat16 if shape.dtype == "bf16" else torch.float32


def device_tensor(shape: LayerShape, name: str, device="cuda") -> torch.Tensor:
    """Allocate and fill one tensor of the layer on the device (current stream)."""
    dims = dims_of(shape, name)
    stream = torch.cuda.current_stream(device).cuda_stream
    if name == "b":
        out = torch.empty(dims, dtype=torch.float32, device=device)
        rc = _device_lib().gen_uniform_device(shape.seed, TID["b"], 0, out.numel(), -0.1, 0.1, 0,
                                              out.data_ptr(), stream)
    else:
        out = torch.empty(dims, dtype=storage_dtype(shape), device=device)
        rc = _device_lib().gen_normal_device(shape.seed, TID[name], 0, out.numel(),
                                             factor_of(shape, name), int(shape.dtype == "bf16"),
                                             out.data_ptr(), stream)
    if rc != 0:
        raise RuntimeError(f"device generator failed for {name}: cudaError {rc}")
    if shape.zipf_s is not None and name in ("x", "W_r"):
        if name == "x":
            out[:, 0] = 1.0
        else:
            o = zipf_offsets(shape).astype(np.float32)
            if shape.dtype == "bf16":
                col = torch.from_numpy(f32_to_bf16(o).view(np.int16)).view(torch.bfloat16)
            else:
                col = torch.from_numpy(o)
            out[:, 0] = col.to(device)
    return out


def device_fp8(shape: LayerShape, name: str, device="cuda"):
    """(codes uint8 [rows, cols], scales uint8 [rows/128, cols/128]) of an FP8 expert matrix."""
    rows, cols = mat_dims(shape, name)
    stream = torch.cuda.current_stream(device).cuda_stream
    q = torch.empty((rows, cols), dtype=torch.uint8, device=device)
    sc = torch.empty((rows // FP8_BLOCK, cols // FP8_BLOCK), dtype=torch.uint8, device=device)
    lib = _device_lib()
    rc = lib.gen_fp8_device(shape.seed, TID[name], TID_SCALE[name], fp8_e0(shape, name), cols, 0, q.numel(),
                            factor_of(shape, name), q.data_ptr(), stream)
    if rc == 0:
        rc = lib.gen_fp8_scales_device(shape.seed, TID_SCALE[name], fp8_e0(shape, name), 0, sc.numel(),
                                       sc.data_ptr(), stream)
    if rc != 0:
        raise RuntimeError(f"device FP8 generator failed for {name}: cudaError {rc}")
    return q, sc


def device_all(shape: LayerShape, device="cuda") -> dict:
    """Every tensor of the layer on the device; with FP8 expert weights each
    of W1, W3, W2, Ws1, Ws3, Ws2 is a (codes, scales) pair."""
    experts = ["W1", "W3", "W2"] + (["Ws1", "Ws3", "Ws2"] if shape.n_shared else [])
    out = {nm: device_tensor(shape, nm, device) for nm in ("x", "W_r")}
    for nm in experts:
        out[nm] = device_fp8(shape, nm, device) if shape.wdtype == "fp8" else device_tensor(shape, nm, device)
    out["b"] = device_tensor(shape, "b", device) if shape.bias else None
    if shape.n_shared == 0:
        out.update(Ws1=None, Ws3=None, Ws2=None)
    return out
