"""moe_route_noalloc: the router for callers that cannot allocate device
scratch (a plugin given no workspace by its host framework, or a serving
loop that must not call cudaMalloc once running). Its output must match
moe_route, which uses a caller-provided workspace, on consecutive calls."""
import numpy as np
import pytest
import torch

import moe_inputs as mi
from moe_inputs import device as mdev
import mixture_experts_layer_group_b200 as moe

pytestmark = pytest.mark.gpu

GATE_RTOL = 2e-5  # the gate tolerance of the routing parity tests


def _cfg(s):
    return moe.make_cfg(s.d, s.d_ff, s.n_routed, s.n_shared, s.top_k, s.n_groups, s.topk_groups, s.score,
                        s.normalize, s.route_scale, s.group_score, s.dtype)


def _route_with_workspace(s, cfg, x, w):
    ws = torch.empty(moe.workspace_size(cfg, s.T), dtype=torch.uint8, device="cuda")
    idx = torch.empty((s.T, s.top_k), dtype=torch.int32, device="cuda")
    gates = torch.empty((s.T, s.top_k), dtype=torch.float32, device="cuda")
    moe.route(cfg, s.T, x, w["W_r"], w["b"], idx, gates, ws)
    return idx, gates


def _route_noalloc(s, cfg, x, w):
    idx = torch.full((s.T, s.top_k), -1, dtype=torch.int32, device="cuda")
    gates = torch.full((s.T, s.top_k), -1.0, dtype=torch.float32, device="cuda")
    moe.route_noalloc(cfg, s.T, x, w["W_r"], w["b"], idx, gates)
    return idx, gates


def test_route_noalloc_matches_route_on_consecutive_calls():
    from mixture_experts_layer_group_b200 import build
    from moe_inputs import build as gen_build
    gen_build.build()
    build.build()
    torch.cuda.set_device(0)
    base = mi.SHAPES["v3_prefill_bf16"]
    # two calls in a row with different batches (the second smaller, so any
    # stale logits of the first call would show up if they were read)
    for T, seed in [(1000, 41), (300, 42)]:
        s = base.with_(T=T, seed=seed)
        cfg = _cfg(s)
        w = {"W_r": mdev.device_tensor(s, "W_r"), "b": mdev.device_tensor(s, "b")}
        x = mdev.device_tensor(s, "x")
        ref_idx, ref_gates = _route_with_workspace(s, cfg, x, w)
        idx, gates = _route_noalloc(s, cfg, x, w)
        torch.cuda.synchronize()
        assert torch.equal(idx.cpu(), ref_idx.cpu()), T
        np.testing.assert_allclose(gates.cpu().numpy(), ref_gates.cpu().numpy(), rtol=GATE_RTOL, atol=1e-7)


def test_route_noalloc_matches_route_bitwise_at_v3_prefill_size():
    # T = 4096 at the V3 shape: moe_route's partial logits for the whole batch
    # (8 K ranges x 4 MiB) do not fit the fixed 8 MiB array, so the call runs
    # the router over token slices with moe_route's K ranges; indices and
    # gates must be moe_route's bit for bit, on two calls in a row
    from mixture_experts_layer_group_b200 import build
    from moe_inputs import build as gen_build
    gen_build.build()
    build.build()
    torch.cuda.set_device(0)
    s = mi.SHAPES["v3_prefill_bf16"]
    cfg = _cfg(s)
    w = {"W_r": mdev.device_tensor(s, "W_r"), "b": mdev.device_tensor(s, "b")}
    x = mdev.device_tensor(s, "x")
    ref_idx, ref_gates = _route_with_workspace(s, cfg, x, w)
    for _ in range(2):
        idx, gates = _route_noalloc(s, cfg, x, w)
        torch.cuda.synchronize()
        assert torch.equal(idx, ref_idx)
        assert torch.equal(gates, ref_gates)


def test_route_noalloc_rejects_sizes_beyond_its_scratch():
    torch.cuda.set_device(0)
    s = mi.SHAPES["v3_prefill_bf16"].with_(T=8193)  # 8193 * 256 * 4 bytes > 8 MiB
    cfg = _cfg(s)
    with pytest.raises(moe.MoeError) as ei:
        moe.route_noalloc(cfg, s.T, 16, 16, None, 16, 16)
    assert ei.value.status == 2  # MOE_ERR_UNSUPPORTED, before any device work
