"""Seeded synthetic inputs for the DeepSeekMoE layer forward.

Shared infrastructure for the tests, the oracle's callers and the bench. It
holds the layer shapes and the recipe that fills every tensor, and none of
the layer's arithmetic. Values come from a counter-based generator (see
``gen_host.c``): each element is a pure function of (seed, tensor id, flat
index), so any slice (one expert, a few token rows) can be regenerated on the
host without materialising the rest, and the device generator
(``gen_device.cu``) writes the identical bits straight into HBM.

Recipe (the shapes and distributions of the five layer configurations):
  x   ~ approx. N(0, 1)                      [T, d]
  W_r ~ approx. N(0, 1/d)                    [N, d]   router rows ("centroids")
  b   ~ U(-0.1, 0.1), fp32                   [N]      only where the layer has a bias
  W1, W3 ~ approx. N(0, 1/d)                 [N, d_ff, d]
  W2  ~ approx. N(0, 1/d_ff)                 [N, d, d_ff]
  Ws1, Ws3 ~ approx. N(0, 1/d)               [n_s*d_ff, d]   fused shared MLP
  Ws2 ~ approx. N(0, 1/(n_s*d_ff))           [d, n_s*d_ff]
  "approx. N" is the Irwin-Hall sum of four uniforms rescaled to the stated
  standard deviation (same mean and variance, support +-3.46 sd).
  FP8 expert weights (wdtype "fp8"): each expert matrix, viewed as
  [rows, cols], is stored as e4m3 codes with one power-of-two scale per
  128 x 128 block: block b gets the exponent e_b = e0 + (hash & 3), e0 the
  smallest with 2^e0 * 448 >= the largest generated |value|, and each code is
  the e4m3 value nearest (ties to even) to v * 2^-e_b for the same
  approximately normal v as above; the scale byte is e_b + 127 (UE8M0).
  So the dequantised weights keep the N(0, 1/fan_in) shape while the block
  scales differ from block to block by up to 8x.
  Skewed routing (decode shape): a seeded permutation gives each expert a
  rank r_e in 1..N; column 0 of x is set to 1 and column 0 of W_r to
  o_e = -s * ln(r_e), so the router logits carry an offset whose exponential
  falls off as r_e^-s (Zipf exponent s = 1.2).
"""
from __future__ import annotations

import ctypes
import math
import os
from dataclasses import dataclass, replace

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
HOST_LIB = os.path.join(_HERE, "libmoe_gen_host.so")
DEVICE_LIB = os.path.join(_HERE, "libmoe_gen_device.so")

# tensor ids of the counter-based generator
TID = {"x": 0, "W_r": 1, "b": 2, "W1": 3, "W3": 4, "W2": 5, "Ws1": 6, "Ws3": 7, "Ws2": 8, "zipf": 9}
# tensor ids of the FP8 block exponents of each expert matrix
TID_SCALE = {"W1": 10, "W3": 11, "W2": 12, "Ws1": 13, "Ws3": 14, "Ws2": 15}
FP8_BLOCK = 128
IRWIN_HALL4_SD = math.sqrt(1431655765.0)  # sd of the sum of four 16-bit uniforms


@dataclass(frozen=True)
class LayerShape:
    """One MoE layer configuration: shapes, routing rule, dtype and seed."""

    name: str
    T: int
    d: int
    n_routed: int
    n_shared: int
    d_ff: int
    top_k: int
    score: str = "softmax"  # "softmax" | "sigmoid"
    n_groups: int = 1
    topk_groups: int = 1
    normalize: bool = False
    route_scale: float = 1.0
    group_score: str = "top2_sum"  # "top2_sum" | "max"
    dtype: str = "bf16"  # "bf16" | "f32"
    seed: int = 0
    bias: bool = False
    zipf_s: float | None = None
    wdtype: str = "bf16"  # expert weights: "bf16" (as dtype) or "fp8" (e4m3 + 128 x 128 block scales)

    def with_(self, **kw) -> "LayerShape":
        return replace(self, **kw)

    @property
    def N(self) -> int:
        return self.n_routed


# The five layer configurations (GShard toy, 2B-scale, V2-, V3-prefill- and
# V3-decode-shaped layers) plus small variants used by the parity tests.
SHAPES = {
    "gshard_tiny_f32": LayerShape("gshard_tiny_f32", T=256, d=256, n_routed=16, n_shared=0,
                                  d_ff=512, top_k=2, score="softmax", dtype="f32", seed=0),
    "dsmoe_2b_bf16": LayerShape("dsmoe_2b_bf16", T=8192, d=1280, n_routed=63, n_shared=1,
                                d_ff=896, top_k=7, score="softmax", seed=1),
    "v2_layer_bf16": LayerShape("v2_layer_bf16", T=4096, d=5120, n_routed=160, n_shared=2,
                                d_ff=1536, top_k=6, score="softmax", seed=2),
    "v3_prefill_bf16": LayerShape("v3_prefill_bf16", T=4096, d=7168, n_routed=256, n_shared=1,
                                  d_ff=2048, top_k=8, score="sigmoid", n_groups=8, topk_groups=4,
                                  normalize=True, route_scale=2.5, seed=3, bias=True),
    "v3_decode_bf16": LayerShape("v3_decode_bf16", T=128, d=7168, n_routed=256, n_shared=1,
                                 d_ff=2048, top_k=8, score="sigmoid", n_groups=8, topk_groups=4,
                                 normalize=True, route_scale=2.5, seed=4, bias=True, zipf_s=1.2),
}
# A V3-shaped layer cut to 32 routed experts (2.9 GB of weights, still far
# beyond L2) for full-metric profiler captures of the same kernels.
SHAPES["v3_profile_32e"] = LayerShape("v3_profile_32e", T=1024, d=7168, n_routed=32, n_shared=1, d_ff=2048,
                                      top_k=8, score="sigmoid", n_groups=8, topk_groups=4, normalize=True,
                                      route_scale=2.5, seed=5, bias=True)
# Supplementary V3 prefill at T = 16384 (512 tokens per routed expert on
# average): the same layer and seed with four times the tokens, which moves
# the expert GEMMs from the HBM roofline to the tensor-core roofline.
SHAPES["v3_prefill_t16k_bf16"] = SHAPES["v3_prefill_bf16"].with_(name="v3_prefill_t16k_bf16", T=16384)
# V2-shaped layer with device-limited routing: the 160 routed experts spread
# over 8 devices of 20, each token's experts drawn from the 3 devices holding
# its highest affinities (group score = the device's best expert score).
SHAPES["v2_device_limited_bf16"] = SHAPES["v2_layer_bf16"].with_(name="v2_device_limited_bf16", n_groups=8,
                                                                   topk_groups=3, group_score="max")
# The V3 prefill layer with FP8 expert weights (e4m3 codes, one power-of-two
# scale per 128 x 128 block); tokens, router and bias as in the bf16 layer.
SHAPES["v3_prefill_fp8"] = SHAPES["v3_prefill_bf16"].with_(name="v3_prefill_fp8", wdtype="fp8")
SHAPES["v3_decode_fp8"] = SHAPES["v3_decode_bf16"].with_(name="v3_decode_fp8", wdtype="fp8")
# The small profiling layer with FP8 weights (1.5 GB of codes: ncu full-section captures)
SHAPES["v3_profile_32e_fp8"] = SHAPES["v3_profile_32e"].with_(name="v3_profile_32e_fp8", wdtype="fp8")
# Variants of the V3 prefill layer for DRAM-traffic captures of the expert
# GEMMs: without the shared expert; without it and without the selection bias
# (near-uniform routing, no expert over 256 rows); and at half the tokens
# (no expert over 256 rows either). Same seed, so the same weights and the
# same leading token rows.
SHAPES["v3_prefill_noshared_bf16"] = SHAPES["v3_prefill_bf16"].with_(name="v3_prefill_noshared_bf16", n_shared=0)
SHAPES["v3_prefill_noshared_nobias_bf16"] = SHAPES["v3_prefill_bf16"].with_(
    name="v3_prefill_noshared_nobias_bf16", n_shared=0, bias=False)
SHAPES["v3_prefill_t2048_noshared_bf16"] = SHAPES["v3_prefill_bf16"].with_(
    name="v3_prefill_t2048_noshared_bf16", T=2048, n_shared=0)
ORDER = ["gshard_tiny_f32", "dsmoe_2b_bf16", "v2_layer_bf16", "v3_prefill_bf16", "v3_decode_bf16"]


def std_of(shape: LayerShape, name: str) -> float:
    d, F, ns = shape.d, shape.d_ff, shape.n_shared
    return {"x": 1.0, "W_r": 1.0 / math.sqrt(d), "W1": 1.0 / math.sqrt(d), "W3": 1.0 / math.sqrt(d),
            "W2": 1.0 / math.sqrt(F), "Ws1": 1.0 / math.sqrt(d), "Ws3": 1.0 / math.sqrt(d),
            "Ws2": 1.0 / math.sqrt(max(ns * F, 1))}[name]


def dims_of(shape: LayerShape, name: str) -> tuple:
    d, F, N, ns, T = shape.d, shape.d_ff, shape.n_routed, shape.n_shared, shape.T
    return {"x": (T, d), "W_r": (N, d), "b": (N,), "W1": (N, F, d), "W3": (N, F, d),
            "W2": (N, d, F), "Ws1": (ns * F, d), "Ws3": (ns * F, d), "Ws2": (d, ns * F)}[name]


def factor_of(shape: LayerShape, name: str) -> float:
    return std_of(shape, name) / IRWIN_HALL4_SD


_host = None


def _host_lib():
    global _host
    if _host is None:
        if not os.path.exists(HOST_LIB):
            raise RuntimeError(f"{HOST_LIB} is missing: run moe_inputs.build.build_host()")
        lib = ctypes.CDLL(HOST_LIB)
        lib.gen_normal.argtypes = [ctypes.c_uint32, ctypes.c_uint32, ctypes.c_uint64, ctypes.c_uint64,
                                   ctypes.c_double, ctypes.c_int, ctypes.c_void_p, ctypes.c_int]
        lib.gen_uniform.argtypes = [ctypes.c_uint32, ctypes.c_uint32, ctypes.c_uint64, ctypes.c_uint64,
                                    ctypes.c_double, ctypes.c_double, ctypes.c_int, ctypes.c_void_p,
                                    ctypes.c_int]
        lib.gen_hash.argtypes = [ctypes.c_uint32, ctypes.c_uint32, ctypes.c_uint64, ctypes.c_uint64,
                                 ctypes.c_void_p]
        lib.gen_fp8.argtypes = [ctypes.c_uint32, ctypes.c_uint32, ctypes.c_uint32, ctypes.c_int, ctypes.c_uint64,
                                ctypes.c_uint64, ctypes.c_uint64, ctypes.c_double, ctypes.c_void_p, ctypes.c_int]
        lib.gen_fp8_scales.argtypes = [ctypes.c_uint32, ctypes.c_uint32, ctypes.c_int, ctypes.c_uint64,
                                       ctypes.c_uint64, ctypes.c_void_p]
        _host = lib
    return _host


def _nthreads() -> int:
    return max(1, min(64, os.cpu_count() or 1))


def host_normal(seed: int, tid: int, offset: int, n: int, factor: float, bf16: bool) -> np.ndarray:
    out = np.empty(n, dtype=np.uint16 if bf16 else np.float32)
    _host_lib().gen_normal(seed, tid, offset, n, factor, int(bf16), out.ctypes.data, _nthreads())
    return out


def host_uniform(seed: int, tid: int, offset: int, n: int, lo: float, hi: float, bf16: bool) -> np.ndarray:
    out = np.empty(n, dtype=np.uint16 if bf16 else np.float32)
    _host_lib().gen_uniform(seed, tid, offset, n, lo, hi, int(bf16), out.ctypes.data, _nthreads())
    return out


def host_hash(seed: int, tid: int, offset: int, n: int) -> np.ndarray:
    out = np.empty(n, dtype=np.uint64)
    _host_lib().gen_hash(seed, tid, offset, n, out.ctypes.data)
    return out


def mat_dims(shape: LayerShape, name: str) -> tuple:
    """2-D view [rows, cols] of an expert weight tensor (routed experts stacked along rows)."""
    d, F, N, ns = shape.d, shape.d_ff, shape.n_routed, shape.n_shared
    return {"W1": (N * F, d), "W3": (N * F, d), "W2": (N * d, F), "Ws1": (ns * F, d), "Ws3": (ns * F, d),
            "Ws2": (d, ns * F)}[name]


def fp8_e0(shape: LayerShape, name: str) -> int:
    """Smallest block exponent: 2^e0 * 448 covers the largest value the
    generator can produce (131070 * factor, about 3.46 standard deviations)."""
    return int(math.ceil(math.log2(131070.0 * factor_of(shape, name) / 448.0)))


def host_fp8(shape: LayerShape, name: str, offset: int = 0, n: int | None = None) -> np.ndarray:
    """e4m3 codes (uint8) of elements [offset, offset + n) of an expert matrix."""
    rows, cols = mat_dims(shape, name)
    n = rows * cols - offset if n is None else n
    out = np.empty(n, dtype=np.uint8)
    _host_lib().gen_fp8(shape.seed, TID[name], TID_SCALE[name], fp8_e0(shape, name), cols, offset, n,
                        factor_of(shape, name), out.ctypes.data, _nthreads())
    return out


def host_fp8_scales(shape: LayerShape, name: str, offset: int = 0, n: int | None = None) -> np.ndarray:
    """UE8M0 scale bytes of blocks [offset, offset + n) (row-major over [rows/128, cols/128])."""
    rows, cols = mat_dims(shape, name)
    n = (rows // FP8_BLOCK) * (cols // FP8_BLOCK) - offset if n is None else n
    out = np.empty(n, dtype=np.uint8)
    _host_lib().gen_fp8_scales(shape.seed, TID_SCALE[name], fp8_e0(shape, name), offset, n, out.ctypes.data)
    return out


def host_expert_fp8(shape: LayerShape, e: int):
    """((q, s) of W1_e, W3_e, W2_e): codes [F, d] / [d, F] and block scales [F/128, d/128] / [d/128, F/128]."""
    d, F = shape.d, shape.d_ff
    n, nb = F * d, (F // FP8_BLOCK) * (d // FP8_BLOCK)
    out = []
    for nm, shp in (("W1", (F, d)), ("W3", (F, d)), ("W2", (d, F))):
        q = host_fp8(shape, nm, e * n, n).reshape(shp)
        sc = host_fp8_scales(shape, nm, e * nb, nb).reshape(shp[0] // FP8_BLOCK, shp[1] // FP8_BLOCK)
        out.append((q, sc))
    return tuple(out)


def host_shared_fp8(shape: LayerShape):
    """((q, s) of Ws1, Ws3, Ws2), or None without a shared expert."""
    if shape.n_shared == 0:
        return None
    out = []
    for nm in ("Ws1", "Ws3", "Ws2"):
        rows, cols = mat_dims(shape, nm)
        out.append((host_fp8(shape, nm).reshape(rows, cols),
                    host_fp8_scales(shape, nm).reshape(rows // FP8_BLOCK, cols // FP8_BLOCK)))
    return tuple(out)


def bf16_to_f32(u16: np.ndarray) -> np.ndarray:
    return (u16.astype(np.uint32) << 16).view(np.float32)


def f32_to_bf16(f: np.ndarray) -> np.ndarray:
    """Round-to-nearest-even fp32 -> bf16 bit patterns (finite inputs)."""
    u = np.ascontiguousarray(f, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = u + 0x7FFF + ((u >> 16) & 1)
    return (u >> 16).astype(np.uint16)


def zipf_offsets(shape: LayerShape) -> np.ndarray:
    """Per-expert router offsets o_e = -s ln r_e for a seeded rank permutation r_e (fp64)."""
    h = host_hash(shape.seed, TID["zipf"], 0, shape.n_routed)
    order = np.argsort(h, kind="stable")
    rank = np.empty(shape.n_routed, dtype=np.int64)
    rank[order] = np.arange(1, shape.n_routed + 1)
    return -float(shape.zipf_s) * np.log(rank.astype(np.float64))


def _bits(shape: LayerShape) -> bool:
    return shape.dtype == "bf16"


def host_tensor(shape: LayerShape, name: str, offset: int = 0, n: int | None = None,
                ) -> np.ndarray:
    """A flat slice [offset, offset+n) of one tensor, in its storage dtype
    (uint16 bf16 bit patterns or float32). The decode shape's column-0 edits of
    x and W_r are applied here too."""
    total = int(np.prod(dims_of(shape, name)))
    n = total - offset if n is None else n
    if name == "b":
        return host_uniform(shape.seed, TID["b"], offset, n, -0.1, 0.1, False)
    out = host_normal(shape.seed, TID[name], offset, n, factor_of(shape, name), _bits(shape))
    if shape.zipf_s is not None and name in ("x", "W_r"):
        d = shape.d
        idx = np.arange(offset, offset + n)
        col0 = idx % d == 0
        if name == "x":
            one = np.array([1.0], dtype=np.float32)
            out[col0] = f32_to_bf16(one)[0] if _bits(shape) else one[0]
        else:
            o = zipf_offsets(shape).astype(np.float32)[idx[col0] // d]
            out[col0] = f32_to_bf16(o) if _bits(shape) else o
    return out


def host_rows(shape: LayerShape, name: str, rows) -> np.ndarray:
    """Selected rows of a 2-D tensor (x: token rows), storage dtype, shape [len(rows), cols]."""
    dims = dims_of(shape, name)
    cols = dims[-1]
    out = [host_tensor(shape, name, int(r) * cols, cols) for r in rows]
    return np.stack(out) if out else np.zeros((0, cols), dtype=np.uint16 if _bits(shape) else np.float32)


def host_expert(shape: LayerShape, e: int):
    """(W1_e [F,d], W3_e [F,d], W2_e [d,F]) of routed expert e, storage dtype."""
    d, F = shape.d, shape.d_ff
    n = F * d
    w1 = host_tensor(shape, "W1", e * n, n).reshape(F, d)
    w3 = host_tensor(shape, "W3", e * n, n).reshape(F, d)
    w2 = host_tensor(shape, "W2", e * n, n).reshape(d, F)
    return w1, w3, w2


def host_shared(shape: LayerShape):
    """(Ws1 [n_s F, d], Ws3, Ws2 [d, n_s F]) or None when the layer has no shared expert."""
    if shape.n_shared == 0:
        return None
    return tuple(host_tensor(shape, nm).reshape(dims_of(shape, nm)) for nm in ("Ws1", "Ws3", "Ws2"))


def host_all(shape: LayerShape) -> dict:
    """Every tensor of a (small) layer, storage dtype, reshaped."""
    names = ["x", "W_r", "W1", "W3", "W2"] + (["Ws1", "Ws3", "Ws2"] if shape.n_shared else [])
    out = {nm: host_tensor(shape, nm).reshape(dims_of(shape, nm)) for nm in names}
    out["b"] = host_tensor(shape, "b") if shape.bias else None
    return out


def to_f64(a: np.ndarray | None, shape: LayerShape) -> np.ndarray | None:
    if a is None:
        return None
    if a.dtype == np.uint16:
        return bf16_to_f32(a).astype(np.float64)
    return a.astype(np.float64)
