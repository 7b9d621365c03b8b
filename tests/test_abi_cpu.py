"""Host-side checks of the C ABI that need no GPU: the library builds and
loads, exports every function the header declares, the ctypes struct
matches the header, and argument validation / workspace sizing behave."""
import ctypes
import os
import re
import subprocess

import pytest

import mixture_experts_layer_group_b200 as moe
from mixture_experts_layer_group_b200 import build as moe_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe_b200.h")


@pytest.fixture(scope="module")
def L():
    moe_build.build()
    return moe.lib()


def header_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return re.findall(r"^\s*MOE_API\s+(?:const\s+)?[a-z_0-9]+\s*\*?\s*(moe_[a-z_0-9]+)\s*\(", src, flags=re.M)


def test_header_declares_the_abi():
    fns = header_functions()
    assert set(fns) == set(moe.EXPORTS), fns


def test_library_exports_every_header_function(L):
    out = subprocess.run(["nm", "-D", "--defined-only", moe.LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    syms = {line.split()[-1] for line in out.splitlines() if line.strip()}
    for fn in header_functions():
        assert fn in syms, fn
        assert getattr(L, fn) is not None
    # nothing else with C linkage leaks out of the library
    assert {s for s in syms if s.startswith("moe_")} == set(header_functions())


def test_binding_declares_argument_types(L):
    """Every function the binding calls has ctypes argument types: without
    them a 64-bit argument (T, a byte count) is passed as a 32-bit int."""
    for name in moe.EXPORTS:
        assert getattr(L, name).argtypes is not None, name


def test_debug_build_exports_the_same_abi():
    """The bounds-checked debug build (-DMOE_DEBUG_BOUNDS) compiles, loads and
    exports exactly the header's functions, like the release build."""
    path = moe_build.build(debug=True)
    assert path == moe.DEBUG_LIB_PATH
    out = subprocess.run(["nm", "-D", "--defined-only", path], capture_output=True, text=True, check=True).stdout
    syms = {line.split()[-1] for line in out.splitlines() if line.strip()}
    assert {s for s in syms if s.startswith("moe_")} == set(header_functions())
    with moe.using_library(path) as D:
        assert D.moe_status_string(0).decode() == moe.lib().moe_status_string(0).decode()
    assert moe.LIB_PATH != path


def test_cfg_struct_matches_header():
    src = open(HEADER).read()
    body = re.search(r"typedef struct moe_cfg \{(.*?)\} moe_cfg;", src, flags=re.S).group(1)
    fields = re.findall(r"(int32_t|float)\s+(\w+);", body)
    assert [n for _, n in fields] == [n for n, _ in moe.MoeCfg._fields_]
    for (ctype, name), (pname, ptype) in zip(fields, moe.MoeCfg._fields_):
        assert (ctype == "float") == (ptype is ctypes.c_float), name
    assert ctypes.sizeof(moe.MoeCfg) == 4 * len(fields)


def v3_cfg(**kw):
    base = dict(d=7168, d_ff=2048, n_routed=256, n_shared=1, top_k=8, n_groups=8, topk_groups=4,
                score="sigmoid", normalize=True, route_scale=2.5)
    base.update(kw)
    return moe.make_cfg(**base)


def test_status_strings(L):
    for code, name in moe.STATUS_NAMES.items():
        assert moe.status_string(code) == name
    assert moe.status_string(99) == "MOE_ERR_UNKNOWN"


def test_workspace_size_grows_and_covers_intermediates(L):
    cfg = v3_cfg()
    sizes = [moe.workspace_size(cfg, T) for T in (1, 128, 4096)]
    assert sizes[0] < sizes[1] < sizes[2]
    T, k, d, F = 4096, 8, 7168, 2048
    # permuted token rows, SwiGLU rows, expert output rows (+ shared) in bf16
    assert sizes[2] >= 2 * (T * k * d + T * k * F + T * 2048 + (T * k + T) * d)
    assert moe.workspace_size_host(cfg, 4096) >= sizes[2] + 2 * 2 * T * d
    assert moe.workspace_size(cfg, 0) >= 0


@pytest.mark.parametrize("bad", [dict(d=7164), dict(d_ff=2044), dict(top_k=300), dict(n_groups=7),
                                 dict(topk_groups=9), dict(top_k=17, topk_groups=1),
                                 dict(n_routed=-1), dict(score="x", n_groups=1, topk_groups=1)])
def test_invalid_cfg_rejected(L, bad):
    if bad.get("score") == "x":
        cfg = v3_cfg(n_groups=1, topk_groups=1)
        cfg.score_fn = 7
    else:
        cfg = v3_cfg(**bad)
    n = ctypes.c_size_t(0)
    rc = L.moe_workspace_size(ctypes.byref(cfg), 16, ctypes.byref(n))
    assert rc in (1, 2)


def test_unsupported_and_limits(L):
    n = ctypes.c_size_t(0)
    assert L.moe_workspace_size(ctypes.byref(v3_cfg(n_routed=1024, n_groups=8)), 4, ctypes.byref(n)) == 2
    assert L.moe_workspace_size(ctypes.byref(v3_cfg()), -1, ctypes.byref(n)) == 1
    assert L.moe_workspace_size(None, 4, ctypes.byref(n)) == 1


def test_argument_errors_need_no_device(L):
    cfg = v3_cfg()
    # T == 0 is a no-op
    assert L.moe_forward(ctypes.byref(cfg), 0, None, None, None, None, None, None, None, None, None, None,
                         None, None, None, 0, None) == 0
    assert L.moe_route(ctypes.byref(cfg), 0, None, None, None, None, None, None, 0, None) == 0
    # null tensors
    assert L.moe_forward(ctypes.byref(cfg), 4, None, None, None, None, None, None, None, None, None, None,
                         None, None, None, 0, None) == 1
    assert L.moe_route(ctypes.byref(cfg), 4, None, None, None, None, None, None, 0, None) == 1
    # misaligned token pointer
    assert L.moe_route(ctypes.byref(cfg), 4, 8, 16, None, 16, 16, 256, 1 << 30, None) == 1
    # workspace too small / misaligned (checked before any device work)
    fake = 1 << 20
    assert L.moe_route(ctypes.byref(cfg), 4, fake, fake, None, fake, fake, fake, 16, None) == 3
    assert L.moe_route(ctypes.byref(cfg), 4, fake, fake, None, fake, fake, fake + 16, 1 << 30, None) == 3
    # shared weights required when n_shared > 0
    assert L.moe_forward(ctypes.byref(cfg), 4, fake, fake, None, fake, fake, fake, None, None, None, fake,
                         None, None, fake, 1 << 40, None) == 1
    # host-buffer calls: T == 0 is a no-op, null buffers are rejected; waiting on
    # (or releasing) a workspace without host-call state does nothing
    for fn in (L.moe_forward_host, L.moe_forward_host_async):
        assert fn(ctypes.byref(cfg), 0, None, None, None, None, None, None, None, None, None, None, None, 0,
                  None) == 0
        assert fn(ctypes.byref(cfg), 4, None, fake, None, fake, fake, fake, fake, fake, fake, fake, fake,
                  1 << 40, None) == 1
    assert L.moe_host_wait(None, None) == 0
    assert L.moe_host_wait(fake, None) == 0
    assert L.moe_workspace_release(fake) == 0
    # bias update: null / misaligned pointers, non-finite rate
    assert L.moe_bias_update(ctypes.byref(cfg), 4, None, ctypes.c_float(1e-3), fake, None) == 1
    assert L.moe_bias_update(ctypes.byref(cfg), 4, fake, ctypes.c_float(1e-3), fake + 2, None) == 1
    assert L.moe_bias_update(ctypes.byref(cfg), 4, fake, ctypes.c_float(float("nan")), fake, None) == 1
    assert L.moe_bias_update(None, 4, fake, ctypes.c_float(1e-3), fake, None) == 1
    assert L.moe_last_cuda_error() == 0


def test_make_cfg_rejects_unknown_strings():
    # a misspelt score, group score or dtype is an error, not a silent default
    for kw in ({"score": "sigmoidd"}, {"group_score": "top2"}, {"dtype": "fp16"}):
        with pytest.raises(ValueError):
            moe.make_cfg(64, 64, 8, 0, 2, **kw)
    c = moe.make_cfg(64, 64, 8, 0, 2, score="sigmoid", group_score="max", dtype="f32")
    assert (c.score_fn, c.group_score, c.dtype) == (moe.MOE_SIGMOID, moe.MOE_GROUP_MAX, moe.MOE_F32)
