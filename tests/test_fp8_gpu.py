"""GPU parity of the FP8-weight layer forward (moe_forward_fp8): e4m3 expert
weights with one power-of-two scale per 128 x 128 block, dequantised exactly
to bf16 on the device. Checked bit for bit against moe_forward run on the
same weights dequantised on the host, and against the fp64 oracle (on the
exactly dequantised weights) on every token."""
import numpy as np
import pytest
import torch

import moe_inputs as mi
import oracle
from moe_inputs import device as mdev
import mixture_experts_layer_group_b200 as moe

from gpu_helpers import (PrefetchedExperts, cfg_of, check_outputs, check_routing, f64, oracle_forward, router_cfg_of,
                         t2np64, workspace)

pytestmark = pytest.mark.gpu

LS = mi.LayerShape
SMALL = {
    # several SwiGLU and down tiles, a ragged token tail, the shared expert
    "fp8_v3_like": LS("fp8_v3_like", T=300, d=512, n_routed=32, n_shared=1, d_ff=256, top_k=4, score="sigmoid",
                      n_groups=4, topk_groups=2, normalize=True, route_scale=2.5, seed=31, bias=True, wdtype="fp8"),
    # d = 384: the down GEMM's 512-column tiles end inside a 128-row scale
    # block past the matrix; two shared experts; softmax gates
    "fp8_ragged": LS("fp8_ragged", T=517, d=384, n_routed=20, n_shared=2, d_ff=384, top_k=3, score="softmax",
                     seed=32, wdtype="fp8"),
    "fp8_no_shared": LS("fp8_no_shared", T=129, d=256, n_routed=16, n_shared=0, d_ff=128, top_k=2,
                        score="softmax", seed=33, wdtype="fp8"),
}


@pytest.fixture(autouse=True)
def _lib():
    from mixture_experts_layer_group_b200 import build
    from moe_inputs import build as gb
    build.build()
    gb.build_device()
    torch.cuda.set_device(0)
    yield
    torch.cuda.empty_cache()


def _dequant(q, sc):
    return oracle.dequant_fp8(q, sc)


def expert_fn_fp8(s):
    def fn(e):
        return tuple(_dequant(q, sc) for q, sc in mi.host_expert_fp8(s, e))
    return fn


def shared_fp8(s):
    sh = mi.host_shared_fp8(s)
    return None if sh is None else tuple(_dequant(q, sc) for q, sc in sh)


def bf16_device(a64):
    """Exactly representable fp64 values -> a bf16 CUDA tensor (asserting exactness)."""
    f = a64.astype(np.float32)
    assert np.array_equal(f.astype(np.float64), a64)
    bits = mi.f32_to_bf16(f)
    assert np.array_equal(mi.bf16_to_f32(bits), f)
    return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).cuda()


def run_fp8(s, w, x):
    cfg = cfg_of(s)
    T = x.shape[0]
    ws = workspace(cfg, T)
    y = torch.empty_like(x)
    idx = torch.empty((T, s.top_k), dtype=torch.int32, device="cuda")
    gates = torch.empty((T, s.top_k), dtype=torch.float32, device="cuda")
    moe.forward_fp8(cfg, T, x, w["W_r"], w["b"], w["W1"], w["W3"], w["W2"], w["Ws1"], w["Ws3"], w["Ws2"], y, ws,
                    idx, gates)
    torch.cuda.synchronize()
    assert moe.device_status(cfg, T, ws) == 0
    return y, idx.cpu().numpy().astype(np.int64), gates.cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("name", list(SMALL))
def test_fp8_equals_bf16_path_on_dequantised_weights(name):
    s = SMALL[name]
    w = mdev.device_all(s)
    x = mdev.device_tensor(s, "x")
    y8, i8, g8 = run_fp8(s, w, x)
    # the same layer through moe_forward with the weights dequantised on the host
    wb = dict(w)
    for nm in ("W1", "W3", "W2") + (("Ws1", "Ws3", "Ws2") if s.n_shared else ()):
        q, sc = w[nm]
        wb[nm] = bf16_device(oracle.dequant_fp8(q.cpu().numpy(), sc.cpu().numpy()))
    cfg = cfg_of(s)
    ws = workspace(cfg, s.T)
    yb = torch.empty_like(x)
    ib = torch.empty((s.T, s.top_k), dtype=torch.int32, device="cuda")
    gb_ = torch.empty((s.T, s.top_k), dtype=torch.float32, device="cuda")
    moe.forward(cfg, s.T, x, wb["W_r"], wb["b"], wb["W1"], wb["W3"], wb["W2"], wb["Ws1"], wb["Ws3"], wb["Ws2"], yb,
                ws, ib, gb_)
    torch.cuda.synchronize()
    assert np.array_equal(ib.cpu().numpy(), i8) and np.array_equal(gb_.cpu().numpy(), g8.astype(np.float32))
    assert torch.equal(yb, y8)


@pytest.mark.parametrize("name", list(SMALL))
def test_fp8_small_layer_against_oracle(name):
    s = SMALL[name]
    w = mdev.device_all(s)
    x = mdev.device_tensor(s, "x")
    y, gidx, ggates = run_fp8(s, w, x)
    h = mi.host_all(s.with_(wdtype="bf16"))
    x64, W_r64 = f64(h["x"]), f64(h["W_r"])
    b = None if h["b"] is None else h["b"].astype(np.float64)
    ref, r = oracle_forward(s, x64, W_r64, b, expert_fn_fp8(s), shared_fp8(s), gidx)
    check_routing(gidx, ggates, r, router_cfg_of(s))
    check_outputs(t2np64(y), ref, "bf16", name)


def test_fp8_skewed_routing_many_chunks():
    """Every token drawn to the same four experts by a large selection bias:
    each gets T = 1000 rows, seven chunks of equal size on the FP8 path.
    Bit for bit equal to moe_forward on the dequantised weights (whose
    chunks are larger) and within tolerance of the oracle."""
    s = LS("fp8_skewed", T=1000, d=256, n_routed=32, n_shared=1, d_ff=256, top_k=4, score="sigmoid",
           n_groups=4, topk_groups=2, normalize=True, route_scale=2.5, seed=34, bias=True, wdtype="fp8")
    hot = [3, 5, 17, 22]
    bias = np.zeros(s.n_routed, np.float32)
    bias[hot] = 4.0
    w = mdev.device_all(s)
    w["b"] = torch.from_numpy(bias).cuda()
    x = mdev.device_tensor(s, "x")
    y, gidx, ggates = run_fp8(s, w, x)
    assert (np.sort(gidx, axis=1) == hot).all()
    wb = dict(w)
    for nm in ("W1", "W3", "W2", "Ws1", "Ws3", "Ws2"):
        q, sc = w[nm]
        wb[nm] = bf16_device(oracle.dequant_fp8(q.cpu().numpy(), sc.cpu().numpy()))
    cfg = cfg_of(s)
    yb = torch.empty_like(x)
    moe.forward(cfg, s.T, x, wb["W_r"], wb["b"], wb["W1"], wb["W3"], wb["W2"], wb["Ws1"], wb["Ws3"], wb["Ws2"], yb,
                workspace(cfg, s.T))
    torch.cuda.synchronize()
    assert torch.equal(yb, y)
    h = mi.host_all(s.with_(wdtype="bf16"))
    ref, r = oracle_forward(s, f64(h["x"]), f64(h["W_r"]), bias.astype(np.float64), expert_fn_fp8(s), shared_fp8(s),
                            gidx)
    check_routing(gidx, ggates, r, router_cfg_of(s))
    check_outputs(t2np64(y), ref, "bf16", s.name)


@pytest.mark.parametrize("name", ["v3_decode_fp8", "v3_prefill_fp8"])
def test_fp8_full_size_every_token(name):
    s = mi.SHAPES[name]
    w = mdev.device_all(s)
    x = mdev.device_tensor(s, "x")
    y, gidx, ggates = run_fp8(s, w, x)
    del w
    torch.cuda.empty_cache()
    x64 = f64(mi.host_tensor(s, "x").reshape(s.T, s.d))
    W_r64 = f64(mi.host_tensor(s, "W_r").reshape(s.n_routed, s.d))
    b = mi.host_tensor(s, "b").astype(np.float64) if s.bias else None
    rcfg = router_cfg_of(s)
    r = oracle.route(x64, W_r64, b, rcfg)
    check_routing(gidx, ggates, r, rcfg)
    experts = PrefetchedExperts(s, sorted(set(gidx.reshape(-1).tolist())), fn=expert_fn_fp8(s))
    try:
        ref, _ = oracle_forward(s, x64, W_r64, b, experts, shared_fp8(s), gidx)
    finally:
        experts.close()
    check_outputs(t2np64(y), ref, "bf16", name)


def test_fp8_rejects_unsupported_shapes():
    cfg = moe.make_cfg(200, 256, 8, 0, 2)  # d = 200 is not a multiple of 128
    with pytest.raises(moe.MoeError) as ei:
        moe.forward_fp8(cfg, 4, 16, 16, None, (16, 16), (16, 16), (16, 16), None, None, None, 16, 256, ws_bytes=0)
    assert ei.value.status == 2
    cfg32 = moe.make_cfg(256, 256, 8, 0, 2, dtype="f32")
    with pytest.raises(moe.MoeError) as ei:
        moe.forward_fp8(cfg32, 4, 16, 16, None, (16, 16), (16, 16), (16, 16), None, None, None, 16, 256,
                        ws_bytes=0)
    assert ei.value.status == 1


def test_fp8_host_entry_matches_device_entry():
    """moe_forward_host_fp8 (pinned host x in, y out) gives moe_forward_fp8's
    bits, on back-to-back calls that alternate the two staging slots and on a
    smaller batch on the same workspace afterwards; so does
    moe_forward_host_fp8_async once host_wait has been reached."""
    s = SMALL["fp8_ragged"]
    w = mdev.device_all(s)
    x = mdev.device_tensor(s, "x")
    cfg = cfg_of(s)
    wargs = (w["W_r"], w["b"], w["W1"], w["W3"], w["W2"], w["Ws1"], w["Ws3"], w["Ws2"])
    y_dev, _, _ = run_fp8(s, w, x)
    ws = workspace(cfg, s.T, host=True)
    xh = x.cpu().pin_memory()
    yh = [torch.empty_like(xh).pin_memory() for _ in range(3)]
    for i in range(3):
        moe.forward_host_fp8(cfg, s.T, xh, *wargs, yh[i], ws)
    torch.cuda.synchronize()
    for i in range(3):
        assert torch.equal(yh[i], y_dev.cpu())
    T2 = 200
    y2_dev, _, _ = run_fp8(s, w, x[:T2].contiguous())
    y2h = torch.empty((T2, s.d), dtype=xh.dtype).pin_memory()
    moe.forward_host_fp8(cfg, T2, xh[:T2].contiguous().pin_memory(), *wargs, y2h, ws)
    torch.cuda.synchronize()
    assert torch.equal(y2h, y2_dev.cpu())
    assert moe.device_status(cfg, T2, ws) == 0
    # the asynchronous output copies: y_host complete after host_wait
    for y in yh:
        y.zero_()
    for i in range(3):
        moe.forward_host_fp8_async(cfg, s.T, xh, *wargs, yh[i], ws)
    moe.host_wait(ws)
    torch.cuda.synchronize()
    for i in range(3):
        assert torch.equal(yh[i], y_dev.cpu())
    moe.workspace_release(ws)


def test_moelayer_runs_fp8_weights():
    """MoELayer takes (codes, scales) expert weights and runs the FP8 entry
    points, device and host-buffer, with the same bits as moe_forward_fp8."""
    s = SMALL["fp8_v3_like"]
    w = mdev.device_all(s)
    x = mdev.device_tensor(s, "x")
    y_dev, _, _ = run_fp8(s, w, x)
    layer = moe.MoELayer(cfg_of(s), w, max_tokens=s.T, host_io=True)
    assert layer.fp8
    y = layer(x)
    torch.cuda.synchronize()
    assert torch.equal(y, y_dev)
    xh = x.cpu().pin_memory()
    yh = torch.empty_like(xh).pin_memory()
    layer.forward_host(xh, yh)
    torch.cuda.synchronize()
    assert torch.equal(yh, y_dev.cpu())
    assert layer.device_status() == 0
    moe.workspace_release(layer.ws)


def test_fp8_token_permutation_equivariance_bitwise():
    """Permuting the tokens permutes the FP8 path's outputs bit for bit."""
    s = SMALL["fp8_ragged"]
    w = mdev.device_all(s)
    x = mdev.device_tensor(s, "x")
    y, idx, _ = run_fp8(s, w, x)
    perm = torch.randperm(s.T, generator=torch.Generator().manual_seed(9))
    yp, idxp, _ = run_fp8(s, w, x[perm.cuda()].contiguous())
    assert np.array_equal(idxp, idx[perm.numpy()])
    assert torch.equal(yp, y[perm.cuda()])
