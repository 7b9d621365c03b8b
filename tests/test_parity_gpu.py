"""GPU parity of the CUDA path against the fp64 oracle, through the C ABI.

Small layers (full oracle, several tiles and ragged tails) and the five
layer configurations at full size (oracle on sampled tokens; routing on all
tokens). Inputs come from the seeded generator on both sides."""
import time

import numpy as np
import pytest
import torch

import moe_inputs as mi
import oracle
from moe_inputs import device as mdev
import mixture_experts_layer_group_b200 as moe

from gpu_helpers import (TOL, PrefetchedExperts, cfg_of, check_outputs, check_routing, chunk_probe_rows, f64,
                         host_shared64, oracle_forward, rel_fro, router_cfg_of, run_forward, t2np64, workspace)

pytestmark = pytest.mark.gpu

LS = mi.LayerShape
# small layers whose oracle runs in seconds; each spans several tiles and has ragged tails
SMALL = {
    "v3_like_small": LS("v3_like_small", T=300, d=512, n_routed=32, n_shared=1, d_ff=256, top_k=4,
                        score="sigmoid", n_groups=4, topk_groups=2, normalize=True, route_scale=2.5, seed=11,
                        bias=True),
    "softmax_ragged": LS("softmax_ragged", T=517, d=384, n_routed=20, n_shared=2, d_ff=384, top_k=3,
                         score="softmax", seed=12),
    "group_max_odd": LS("group_max_odd", T=129, d=256, n_routed=63, n_shared=0, d_ff=128, top_k=6,
                        score="sigmoid", n_groups=9, topk_groups=3, normalize=True, route_scale=1.0,
                        group_score="max", seed=13, bias=True),
    "single_token": LS("single_token", T=1, d=512, n_routed=16, n_shared=1, d_ff=256, top_k=2,
                       score="softmax", seed=14),
    "tiny_f32": LS("tiny_f32", T=77, d=136, n_routed=12, n_shared=1, d_ff=200, top_k=3, score="sigmoid",
                   normalize=True, route_scale=2.5, dtype="f32", seed=15, bias=True),
    "gshard_tiny_f32": mi.SHAPES["gshard_tiny_f32"],
    # the library's limits: 512 routed experts, top-16, 32 groups
    "max_limits": LS("max_limits", T=300, d=256, n_routed=512, n_shared=1, d_ff=128, top_k=16,
                     score="sigmoid", n_groups=32, topk_groups=8, normalize=True, route_scale=2.5, seed=16,
                     bias=True),
    # bf16 with reduction lengths that are not multiples of the 64-wide K block
    "bf16_ragged_k": LS("bf16_ragged_k", T=97, d=200, n_routed=10, n_shared=1, d_ff=136, top_k=3,
                        score="softmax", seed=17),
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


def full_oracle_check(s, w=None, x=None):
    w = mdev.device_all(s) if w is None else w
    x = mdev.device_tensor(s, "x") if x is None else x
    y, gidx, ggates = run_forward(s, w, x)
    h = mi.host_all(s)
    x64 = f64(h["x"])
    W_r64 = f64(h["W_r"])
    b = None if h["b"] is None else h["b"].astype(np.float64)
    expert = lambda e: (f64(h["W1"][e]), f64(h["W3"][e]), f64(h["W2"][e]))  # noqa: E731
    shared = None if s.n_shared == 0 else (f64(h["Ws1"]), f64(h["Ws3"]), f64(h["Ws2"]))
    ref, r = oracle_forward(s, x64, W_r64, b, expert, shared, gidx)
    n_flag, n_diff = check_routing(gidx, ggates, r, router_cfg_of(s))
    err, _, _ = check_outputs(t2np64(y), ref, s.dtype, s.name)
    return err, gidx, y


@pytest.mark.parametrize("name", list(SMALL))
def test_small_layer_full_parity(name):
    full_oracle_check(SMALL[name])


@pytest.mark.parametrize("dtype,strength", [("bf16", 4.0), ("bf16", 0.3), ("f32", 4.0)])
def test_skewed_routing_many_chunks(dtype, strength):
    """A selection bias that draws (nearly) every token to the same four
    experts: each of them gets up to T = 1000 rows, so its units split into
    several chunks of equal size with a ragged last one (the bias moves the
    selection only, the gates still come from the unbiased scores)."""
    s = LS("skewed_" + dtype, T=1000, d=256, n_routed=32, n_shared=1, d_ff=192, top_k=4, score="sigmoid",
           n_groups=4, topk_groups=2, normalize=True, route_scale=2.5, dtype=dtype, seed=21, bias=True)
    hot = [3, 5, 17, 22]  # two experts in each of groups 0 and 2
    bias = np.zeros(s.n_routed, np.float32)
    bias[hot] = strength
    w = mdev.device_all(s)
    w["b"] = torch.from_numpy(bias).cuda()
    x = mdev.device_tensor(s, "x")
    y, gidx, ggates = run_forward(s, w, x)
    h = mi.host_all(s)
    expert = lambda e: (f64(h["W1"][e]), f64(h["W3"][e]), f64(h["W2"][e]))  # noqa: E731
    shared = (f64(h["Ws1"]), f64(h["Ws3"]), f64(h["Ws2"]))
    x64, W_r64 = f64(h["x"]), f64(h["W_r"])
    ref, r = oracle_forward(s, x64, W_r64, bias.astype(np.float64), expert, shared, gidx)
    check_routing(gidx, ggates, r, router_cfg_of(s))
    counts = np.bincount(gidx.ravel(), minlength=s.n_routed)
    if strength >= 1.0:
        assert (np.sort(gidx, axis=1) == hot).all()
    else:
        assert counts[hot].min() > 256 and counts[hot].max() < s.T, counts[hot]
    check_outputs(t2np64(y), ref, s.dtype, s.name)


def test_dispatch_bit_exact_and_edge_cases():
    s = SMALL["v3_like_small"]
    cfg = cfg_of(s)
    for T, idx in [(300, None), (1, None), (33, None), (257, "hot"), (64, "reverse")]:
        if idx is None:
            x = mdev.device_tensor(s.with_(T=T), "x")
            w = mdev.device_all(s)
            ws = workspace(cfg, T)
            gi = torch.empty((T, s.top_k), dtype=torch.int32, device="cuda")
            gg = torch.empty((T, s.top_k), dtype=torch.float32, device="cuda")
            moe.route(cfg, T, x, w["W_r"], w["b"], gi, gg, ws)
            torch.cuda.synchronize()
            idx_np = gi.cpu().numpy()
        elif idx == "hot":  # every token picks the same experts
            idx_np = np.tile(np.array([[5, 2, 31, 0]], dtype=np.int32), (T, 1))
        else:  # experts in descending order per token
            idx_np = np.stack([np.random.default_rng(t).choice(32, 4, replace=False) for t in range(T)])
            idx_np = -np.sort(-idx_np, axis=1).astype(np.int32)
        ws = workspace(cfg, T)
        counts = torch.empty(s.n_routed, dtype=torch.int32, device="cuda")
        offsets = torch.empty(s.n_routed + 1, dtype=torch.int32, device="cuda")
        perm = torch.empty(T * s.top_k, dtype=torch.int32, device="cuda")
        moe.dispatch(cfg, T, torch.from_numpy(idx_np).cuda(), counts, offsets, perm, ws)
        torch.cuda.synchronize()
        assert moe.device_status(cfg, T, ws) == 0
        c_ref, o_ref, p_ref = oracle.permutation(idx_np.astype(np.int64), s.n_routed)
        assert (counts.cpu().numpy() == c_ref).all()
        assert (offsets.cpu().numpy() == o_ref).all()
        assert (perm.cpu().numpy() == p_ref).all()


def test_dispatch_flags_invalid_indices():
    s = SMALL["v3_like_small"]
    cfg = cfg_of(s)
    T = 40
    idx = torch.zeros((T, s.top_k), dtype=torch.int32)
    idx[:] = torch.tensor([1, 2, 3, 4], dtype=torch.int32)
    idx[7, 2] = 99       # out of range
    idx[9, 3] = 1        # duplicate of slot 0
    ws = workspace(cfg, T)
    moe.dispatch(cfg, T, idx.cuda(), None, None, None, ws)
    torch.cuda.synchronize()
    bits = moe.device_status(cfg, T, ws)
    assert bits & moe.MOE_DEV_BAD_EXPERT and bits & moe.MOE_DEV_DUP_EXPERT


def test_route_matches_forward_routing_and_is_deterministic():
    s = SMALL["v3_like_small"]
    w = mdev.device_all(s)
    x = mdev.device_tensor(s, "x")
    y1, i1, g1 = run_forward(s, w, x)
    y2, i2, g2 = run_forward(s, w, x)
    assert torch.equal(y1, y2) and (i1 == i2).all() and (g1 == g2).all()
    cfg = cfg_of(s)
    ws = workspace(cfg, s.T)
    gi = torch.empty((s.T, s.top_k), dtype=torch.int32, device="cuda")
    gg = torch.empty((s.T, s.top_k), dtype=torch.float32, device="cuda")
    moe.route(cfg, s.T, x, w["W_r"], w["b"], gi, gg, ws)
    torch.cuda.synchronize()
    assert (gi.cpu().numpy() == i1).all() and (gg.cpu().numpy() == g1).all()


def test_bias_update_bit_exact():
    # counts straight from the GPU's own routing and dispatch, plus a crafted
    # vector with loads at, above and below the mean
    s = SMALL["v3_like_small"]
    cfg = cfg_of(s)
    w = mdev.device_all(s)
    x = mdev.device_tensor(s, "x")
    _, gidx, _ = run_forward(s, w, x)
    ws = workspace(cfg, s.T)
    counts = torch.zeros(s.n_routed, dtype=torch.int32, device="cuda")
    moe.dispatch(cfg, s.T, torch.from_numpy(gidx).cuda(), counts, None, None, ws)
    crafted = np.zeros(s.n_routed, dtype=np.int32)
    mean = s.T * s.top_k // s.n_routed
    crafted[: s.n_routed // 2] = mean
    crafted[s.n_routed // 2:] = mean + np.arange(s.n_routed - s.n_routed // 2) % 3 - 1
    for c in (counts, torch.from_numpy(crafted).cuda()):
        b0 = torch.from_numpy(np.random.default_rng(3).normal(size=s.n_routed).astype(np.float32)).cuda()
        b = b0.clone()
        moe.bias_update(cfg, s.T, c, 1e-3, b)
        torch.cuda.synchronize()
        ref = oracle.bias_update(b0.cpu().numpy(), c.cpu().numpy(), s.T, s.top_k, np.float64(np.float32(1e-3)))
        assert np.array_equal(b.cpu().numpy(), ref.astype(np.float32))


def test_forward_replays_from_a_cuda_graph():
    # moe_forward issues only stream-ordered work (memsets, kernel launches),
    # so a captured step replays to the same bits as an eager one
    s = SMALL["v3_like_small"]
    w = mdev.device_all(s)
    x = mdev.device_tensor(s, "x")
    y_eager, _, _ = run_forward(s, w, x)
    cfg = cfg_of(s)
    ws = workspace(cfg, s.T)
    y = torch.empty_like(x)
    wargs = (w["W_r"], w["b"], w["W1"], w["W3"], w["W2"], w["Ws1"], w["Ws3"], w["Ws2"])
    side = torch.cuda.Stream()
    with torch.cuda.stream(side):
        moe.forward(cfg, s.T, x, *wargs, y, ws, stream=side)  # per-device setup outside the capture
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=side):
        moe.forward(cfg, s.T, x, *wargs, y, ws, stream=side)
    y.zero_()
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    assert torch.equal(y, y_eager)


def test_bounded_wait_gives_up_and_context_survives():
    # a wait that nothing completes runs out after the limit and is reported
    # as a device-status bit; the same process then runs a layer correctly
    t0 = time.perf_counter()
    bits = moe.selftest_wait_timeout()
    dt = time.perf_counter() - t0
    assert bits == moe.MOE_DEV_WAIT_TIMEOUT and 0.9 < dt < 30.0, (bits, dt)
    full_oracle_check(SMALL["single_token"])


def test_identical_experts_invariant():
    # every routed expert identical, normalised gates: y = 2.5 FFN(x) + shared(x) whatever the routing
    s = SMALL["v3_like_small"]
    w = mdev.device_all(s)
    for nm in ("W1", "W3", "W2"):
        w[nm] = w[nm][:1].expand_as(w[nm]).contiguous()
    x = mdev.device_tensor(s, "x")
    y, gidx, _ = run_forward(s, w, x)
    h = mi.host_all(s)
    x64 = f64(h["x"])
    e0 = (f64(h["W1"][0]), f64(h["W3"][0]), f64(h["W2"][0]))
    ref = 2.5 * oracle.expert_ffn(x64, *e0) + oracle.expert_ffn(x64, f64(h["Ws1"]), f64(h["Ws3"]), f64(h["Ws2"]))
    check_outputs(t2np64(y), ref, "bf16", "identical experts")


def test_forward_host_matches_device_forward():
    s = SMALL["softmax_ragged"]
    w = mdev.device_all(s)
    x = mdev.device_tensor(s, "x")
    y_dev, _, _ = run_forward(s, w, x)
    cfg = cfg_of(s)
    ws = workspace(cfg, s.T, host=True)
    xh = x.cpu().pin_memory()
    yh = torch.empty_like(xh).pin_memory()
    moe.forward_host(cfg, s.T, xh, w["W_r"], w["b"], w["W1"], w["W3"], w["W2"], w["Ws1"], w["Ws3"], w["Ws2"],
                     yh, ws)
    torch.cuda.synchronize()
    assert torch.equal(yh, y_dev.cpu())


def test_forward_host_back_to_back_calls():
    # consecutive calls on one workspace overlap the next input copy with the
    # previous call's tail: every call must still see its own tokens
    s = SMALL["v3_like_small"]
    w = mdev.device_all(s)
    cfg = cfg_of(s)
    ws = workspace(cfg, s.T, host=True)
    wargs = (w["W_r"], w["b"], w["W1"], w["W3"], w["W2"], w["Ws1"], w["Ws3"], w["Ws2"])
    xs = [mdev.device_tensor(s.with_(seed=s.seed + i), "x") for i in range(4)]
    refs = [run_forward(s, w, x)[0].cpu() for x in xs]
    xh = [x.cpu().pin_memory() for x in xs]
    yh = [torch.empty_like(h).pin_memory() for h in xh]
    for _ in range(2):
        for i in range(4):  # no synchronisation between calls
            moe.forward_host(cfg, s.T, xh[i], *wargs, yh[i], ws)
        torch.cuda.synchronize()
        for i in range(4):
            assert torch.equal(yh[i], refs[i]), i


def test_forward_host_alternating_sizes_and_device_calls():
    # one workspace, no synchronisation: host calls alternate a large and a
    # small batch (whose staging areas sit at other offsets, over buffers the
    # previous call still uses), with a device-buffer forward in between;
    # every call must still produce its own batch's output
    s = SMALL["v3_like_small"]
    w = mdev.device_all(s)
    cfg = cfg_of(s)
    wargs = (w["W_r"], w["b"], w["W1"], w["W3"], w["W2"], w["Ws1"], w["Ws3"], w["Ws2"])
    sizes = [300, 37, 300, 129, 37, 300]
    ws = workspace(cfg, max(sizes), host=True)
    xs = [mdev.device_tensor(s.with_(T=T, seed=s.seed + 10 + i), "x") for i, T in enumerate(sizes)]
    refs = [run_forward(s.with_(T=x.shape[0]), w, x)[0].cpu() for x in xs]
    xh = [x.cpu().pin_memory() for x in xs]
    yh = [torch.empty_like(h).pin_memory() for h in xh]
    xd = mdev.device_tensor(s.with_(T=200, seed=99), "x")
    yd_ref = run_forward(s.with_(T=200), w, xd)[0]
    yd = torch.empty_like(xd)
    for rep in range(2):
        for i, x in enumerate(xh):
            moe.forward_host(cfg, x.shape[0], x, *wargs, yh[i], ws)
            if i == 2:
                moe.forward(cfg, 200, xd, *wargs, yd, ws)
        torch.cuda.synchronize()
        for i in range(len(sizes)):
            assert torch.equal(yh[i], refs[i]), (rep, i)
        assert torch.equal(yd, yd_ref)
    moe.workspace_release(ws)
    moe.workspace_release(ws)  # nothing left: a no-op
    moe.forward_host(cfg, 300, xh[0], *wargs, yh[0], ws)  # state is rebuilt on the next call
    torch.cuda.synchronize()
    assert torch.equal(yh[0], refs[0])
    moe.workspace_release(ws)


def test_forward_host_async_back_to_back_and_mixed_calls():
    # asynchronous output copies: successive calls on one workspace with no
    # synchronisation, their y copied out on the workspace's output stream
    # while the next call runs; mixed with synchronous host calls, other
    # batch sizes (staging at other offsets) and device-buffer calls (a
    # moe_forward and a moe_route over a larger batch, whose buffers cover
    # the staging slots a pending output copy reads). Every y_host must hold
    # its own batch's output once host_wait has been reached.
    s = SMALL["v3_like_small"]
    w = mdev.device_all(s)
    cfg = cfg_of(s)
    wargs = (w["W_r"], w["b"], w["W1"], w["W3"], w["W2"], w["Ws1"], w["Ws3"], w["Ws2"])
    sizes = [300, 300, 300, 37, 300, 300, 129, 300]
    big = 600
    ws = workspace(cfg, big, host=True)
    xs = [mdev.device_tensor(s.with_(T=T, seed=s.seed + 20 + i), "x") for i, T in enumerate(sizes)]
    refs = [run_forward(s.with_(T=x.shape[0]), w, x)[0].cpu() for x in xs]
    xh = [x.cpu().pin_memory() for x in xs]
    yh = [torch.full_like(h, float("nan")).pin_memory() for h in xh]
    xd = mdev.device_tensor(s.with_(T=big, seed=98), "x")
    yd_ref, idx_ref, _ = run_forward(s.with_(T=big), w, xd)
    yd = torch.empty_like(xd)
    idx = torch.empty((big, s.top_k), dtype=torch.int32, device="cuda")
    gates = torch.empty((big, s.top_k), dtype=torch.float32, device="cuda")
    for rep in range(2):
        for i, x in enumerate(xh):
            if i == 5:
                moe.forward_host(cfg, x.shape[0], x, *wargs, yh[i], ws)  # a synchronous call in between
            else:
                moe.forward_host_async(cfg, x.shape[0], x, *wargs, yh[i], ws)
            if i == 2:
                moe.forward(cfg, big, xd, *wargs, yd, ws)
            if i == 6:
                moe.route(cfg, big, xd, w["W_r"], w["b"], idx, gates, ws)
        moe.host_wait(ws)
        torch.cuda.synchronize()
        for i in range(len(sizes)):
            assert torch.equal(yh[i], refs[i]), (rep, i)
            yh[i].fill_(float("nan"))
        assert torch.equal(yd, yd_ref)
        assert np.array_equal(idx.cpu().numpy(), idx_ref)
    # a long run of asynchronous calls of one size, then the wait
    for rep in range(3):
        for i in (0, 1, 2, 4):
            moe.forward_host_async(cfg, 300, xh[i], *wargs, yh[i], ws)
    moe.host_wait(ws)
    torch.cuda.synchronize()
    for i in (0, 1, 2, 4):
        assert torch.equal(yh[i], refs[i]), i
    moe.workspace_release(ws)


def test_graph_capture_after_async_host_calls():
    # once the asynchronous output copies have finished, a device-buffer
    # forward on the same workspace captures and replays like on a fresh one
    s = SMALL["v3_like_small"]
    w = mdev.device_all(s)
    x = mdev.device_tensor(s, "x")
    y_eager, _, _ = run_forward(s, w, x)
    cfg = cfg_of(s)
    wargs = (w["W_r"], w["b"], w["W1"], w["W3"], w["W2"], w["Ws1"], w["Ws3"], w["Ws2"])
    ws = workspace(cfg, s.T, host=True)
    xh = x.cpu().pin_memory()
    yh = [torch.empty_like(xh).pin_memory() for _ in range(2)]
    side = torch.cuda.Stream()
    for y_h in yh:
        moe.forward_host_async(cfg, s.T, xh, *wargs, y_h, ws, stream=side)
    moe.host_wait(ws, side)
    side.synchronize()
    for y_h in yh:
        assert torch.equal(y_h, y_eager.cpu())
    y = torch.empty_like(x)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=side):
        moe.forward(cfg, s.T, x, *wargs, y, ws, stream=side)
    for _ in range(2):
        g.replay()
    torch.cuda.synchronize()
    assert torch.equal(y, y_eager)
    del g
    moe.workspace_release(ws)


def test_moelayer_async_host_output():
    s = SMALL["softmax_ragged"]
    w = mdev.device_all(s)
    x = mdev.device_tensor(s, "x")
    y_dev, _, _ = run_forward(s, w, x)
    layer = moe.MoELayer(cfg_of(s), w, s.T, host_io=True)
    xh = x.cpu().pin_memory()
    yh = [torch.empty_like(xh).pin_memory() for _ in range(3)]
    for y in yh:
        layer.forward_host(xh, y, wait=False)
    layer.host_wait()
    torch.cuda.synchronize()
    for y in yh:
        assert torch.equal(y, y_dev.cpu())
    moe.workspace_release(layer.ws)


def test_abi_errors_on_device_buffers():
    s = SMALL["v3_like_small"]
    cfg = cfg_of(s)
    w = mdev.device_all(s)
    x = mdev.device_tensor(s, "x")
    y = torch.empty_like(x)
    small = torch.empty(1024, dtype=torch.uint8, device="cuda")
    with pytest.raises(moe.MoeError) as ei:
        moe.forward(cfg, s.T, x, w["W_r"], w["b"], w["W1"], w["W3"], w["W2"], w["Ws1"], w["Ws3"], w["Ws2"], y,
                    small)
    assert ei.value.status == 3
    ws = workspace(cfg, s.T)
    with pytest.raises(moe.MoeError):
        moe.forward(cfg, s.T, x, w["W_r"], w["b"], w["W1"], w["W3"], w["W2"], None, None, None, y, ws)
    moe.forward(cfg, 0, x, w["W_r"], w["b"], w["W1"], w["W3"], w["W2"], w["Ws1"], w["Ws3"], w["Ws2"], y, ws)


# ------------------------------------------------------------- full size ----

# Token rows whose outputs are compared with the oracle at full size: every
# token, except for the T = 16384 layer, where the tokens at every chunk edge
# of every expert (the first token of each chunk the GEMMs cut an expert's
# rows into, and its last token) plus 128 seeded random ones are checked.
ALL_TOKENS = {"gshard_tiny_f32", "dsmoe_2b_bf16", "v2_layer_bf16", "v3_prefill_bf16", "v3_decode_bf16",
              "v2_device_limited_bf16"}


def _dispatch_bit_exact(s, gidx):
    """moe_dispatch on the GPU's own routing of the whole batch against the
    oracle's permutation, bit for bit."""
    cfg = cfg_of(s)
    ws = workspace(cfg, s.T)
    counts = torch.empty(s.n_routed, dtype=torch.int32, device="cuda")
    offsets = torch.empty(s.n_routed + 1, dtype=torch.int32, device="cuda")
    perm = torch.empty(s.T * s.top_k, dtype=torch.int32, device="cuda")
    moe.dispatch(cfg, s.T, torch.from_numpy(gidx.astype(np.int32)).cuda(), counts, offsets, perm, ws)
    torch.cuda.synchronize()
    assert moe.device_status(cfg, s.T, ws) == 0
    c_ref, o_ref, p_ref = oracle.permutation(gidx, s.n_routed)
    assert np.array_equal(counts.cpu().numpy(), c_ref)
    assert np.array_equal(offsets.cpu().numpy(), o_ref)
    assert np.array_equal(perm.cpu().numpy(), p_ref)


@pytest.mark.parametrize("name", mi.ORDER + ["v3_prefill_t16k_bf16", "v2_device_limited_bf16"])
def test_full_size_config(name):
    s = mi.SHAPES[name]
    w = mdev.device_all(s)
    x = mdev.device_tensor(s, "x")
    y, gidx, ggates = run_forward(s, w, x)
    del w
    torch.cuda.empty_cache()
    _dispatch_bit_exact(s, gidx)
    # routing of every token
    x64 = f64(mi.host_tensor(s, "x").reshape(s.T, s.d))
    W_r64 = f64(mi.host_tensor(s, "W_r").reshape(s.n_routed, s.d))
    b = mi.host_tensor(s, "b").astype(np.float64) if s.bias else None
    rcfg = router_cfg_of(s)
    r = oracle.route(x64, W_r64, b, rcfg)
    check_routing(gidx, ggates, r, rcfg)
    # outputs of every token, or of every chunk edge plus a random sample
    if name in ALL_TOKENS:
        rows = np.arange(s.T)
    else:
        rnd = np.random.default_rng(s.seed).choice(s.T, 128, replace=False)
        rows = np.union1d(chunk_probe_rows(gidx, s.n_routed), rnd)
    experts = PrefetchedExperts(s, sorted(set(gidx[rows].reshape(-1).tolist())))
    try:
        ref, _ = oracle_forward(s, x64[rows], W_r64, b, experts, host_shared64(s), gidx[rows])
    finally:
        experts.close()
    check_outputs(t2np64(y[torch.from_numpy(rows).cuda()]), ref, s.dtype, name)


def test_full_size_identical_experts_v3_prefill():
    # The V3 prefill layer (T = 4096, d = 7168, 256 routed of d_ff = 2048 + 1
    # shared) with every routed expert a copy of expert 0: with normalised
    # gates scaled by 2.5, y = 2.5 FFN_0(x) + shared(x) for every token
    # whatever the routing, so all 4096 outputs are checked in fp64 with no
    # dependence on ties.
    s = mi.SHAPES["v3_prefill_bf16"]
    w = mdev.device_all(s)
    for nm in ("W1", "W3", "W2"):
        w[nm] = w[nm][:1].expand_as(w[nm]).contiguous()
    x = mdev.device_tensor(s, "x")
    y, _, _ = run_forward(s, w, x)
    del w
    torch.cuda.empty_cache()
    x64 = f64(mi.host_tensor(s, "x").reshape(s.T, s.d))
    e0 = tuple(f64(a) for a in mi.host_expert(s, 0))
    ref = 2.5 * oracle.expert_ffn(x64, *e0) + oracle.expert_ffn(x64, *host_shared64(s))
    check_outputs(t2np64(y), ref, "bf16", "identical experts, V3 prefill")


def test_nonfinite_token_is_flagged_and_isolated():
    # one token of NaNs: the router records MOE_DEV_NONFINITE, still gives it
    # top_k distinct experts in range, and every other token's routing and
    # output are those of the clean batch
    s = SMALL["v3_like_small"]
    w = mdev.device_all(s)
    x = mdev.device_tensor(s, "x")
    y0, i0, g0 = run_forward(s, w, x)
    xb = x.clone()
    xb[7] = float("nan")
    cfg = cfg_of(s)
    ws = workspace(cfg, s.T)
    for use_forward in (False, True):
        idx = torch.empty((s.T, s.top_k), dtype=torch.int32, device="cuda")
        gates = torch.empty((s.T, s.top_k), dtype=torch.float32, device="cuda")
        y = torch.empty_like(x)
        if use_forward:
            moe.forward(cfg, s.T, xb, w["W_r"], w["b"], w["W1"], w["W3"], w["W2"], w["Ws1"], w["Ws3"], w["Ws2"],
                        y, ws, idx, gates)
        else:
            moe.route(cfg, s.T, xb, w["W_r"], w["b"], idx, gates, ws)
        torch.cuda.synchronize()
        bits = moe.device_status(cfg, s.T, ws)
        assert bits & moe.MOE_DEV_NONFINITE and not bits & (moe.MOE_DEV_BAD_EXPERT | moe.MOE_DEV_DUP_EXPERT)
        gi = idx.cpu().numpy()
        assert ((gi >= 0) & (gi < s.n_routed)).all()
        assert len(set(gi[7].tolist())) == s.top_k
        keep = np.arange(s.T) != 7
        assert np.array_equal(gi[keep], i0[keep])
        assert np.array_equal(gates.cpu().numpy()[keep], g0[keep].astype(np.float32))
        if use_forward:
            yk, y0k = t2np64(y)[keep], t2np64(y0)[keep]
            check_outputs(yk, y0k, "bf16", "clean tokens next to a NaN token")


@pytest.mark.parametrize("name", ["softmax_ragged", "v3_prefill_bf16"])
def test_token_permutation_equivariance_bitwise(name):
    """Each token's output is computed in an order fixed by its own row alone
    (router K order, the per-element MMA reduction over K, the combine's
    ascending expert order), so permuting the tokens permutes the outputs,
    the routing and the gates bit for bit -- although every expert's token
    rows, MMA tiles and chunks change."""
    s = SMALL[name] if name in SMALL else mi.SHAPES[name]
    w = mdev.device_all(s)
    x = mdev.device_tensor(s, "x")
    y, idx, gates = run_forward(s, w, x)
    perm = torch.randperm(s.T, generator=torch.Generator().manual_seed(7))
    yp, idxp, gatesp = run_forward(s, w, x[perm.cuda()].contiguous())
    p = perm.numpy()
    assert np.array_equal(idxp, idx[p])
    assert np.array_equal(gatesp, gates[p])
    assert torch.equal(yp, y[perm.cuda()])
