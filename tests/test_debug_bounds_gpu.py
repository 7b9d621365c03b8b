"""The bounds-checked debug build (libmoe_b200_debug.so, compiled with
-DMOE_DEBUG_BOUNDS): before its indexed accesses every kernel checks the
index -- destination rows of the scatter and the gather, unit rows and
weight rows of the expert GEMMs, ring and tensor-memory placement, the
epilogue's row stores and gate reads, the FP8 converters' ring reads -- and
records MOE_DEV_BOUNDS instead of making a bad access. On small layers that
span several tiles, ragged tails, the library's limits, fp32, FP8 and the
expert-parallel steps, no check fires and every output equals the release
build's bit for bit: the release build's indices stay in bounds on the same
inputs."""
import numpy as np
import pytest
import torch

import moe_inputs as mi
from moe_inputs import device as mdev
import mixture_experts_layer_group_b200 as moe

from gpu_helpers import cfg_of, workspace

pytestmark = pytest.mark.gpu

LS = mi.LayerShape
CASES = {
    "v3_like_small": LS("v3_like_small", T=300, d=512, n_routed=32, n_shared=1, d_ff=256, top_k=4,
                        score="sigmoid", n_groups=4, topk_groups=2, normalize=True, route_scale=2.5, seed=11,
                        bias=True),
    "softmax_ragged": LS("softmax_ragged", T=517, d=384, n_routed=20, n_shared=2, d_ff=384, top_k=3,
                         score="softmax", seed=12),
    "bf16_ragged_k": LS("bf16_ragged_k", T=97, d=200, n_routed=10, n_shared=1, d_ff=136, top_k=3,
                        score="softmax", seed=17),
    "max_limits": LS("max_limits", T=300, d=256, n_routed=512, n_shared=1, d_ff=128, top_k=16,
                     score="sigmoid", n_groups=32, topk_groups=8, normalize=True, route_scale=2.5, seed=16,
                     bias=True),
    "single_token": LS("single_token", T=1, d=512, n_routed=16, n_shared=1, d_ff=256, top_k=2,
                       score="softmax", seed=14),
    "tiny_f32": LS("tiny_f32", T=77, d=136, n_routed=12, n_shared=1, d_ff=200, top_k=3, score="sigmoid",
                   normalize=True, route_scale=2.5, dtype="f32", seed=15, bias=True),
    "fp8_ragged": LS("fp8_ragged", T=517, d=384, n_routed=20, n_shared=2, d_ff=384, top_k=3, score="softmax",
                     seed=32, wdtype="fp8"),
    # a skewed layer: experts with several chunks of the largest unit
    "skewed_chunks": LS("skewed_chunks", T=1024, d=256, n_routed=16, n_shared=1, d_ff=256, top_k=2,
                        score="softmax", seed=41, zipf_s=1.5),
    # the same on the FP8 path (chunks of its smaller unit)
    "fp8_skewed_chunks": LS("fp8_skewed_chunks", T=1024, d=256, n_routed=16, n_shared=1, d_ff=256, top_k=2,
                            score="softmax", seed=42, zipf_s=1.5, wdtype="fp8"),
}


@pytest.fixture(autouse=True)
def _lib():
    from mixture_experts_layer_group_b200 import build
    from moe_inputs import build as gb
    build.build()
    build.build(debug=True)
    gb.build_device()
    torch.cuda.set_device(0)
    yield
    torch.cuda.empty_cache()


def _forward(s, w, x):
    cfg = cfg_of(s)
    ws = workspace(cfg, s.T)
    y = torch.empty_like(x)
    idx = torch.empty((s.T, s.top_k), dtype=torch.int32, device="cuda")
    gates = torch.empty((s.T, s.top_k), dtype=torch.float32, device="cuda")
    fwd = moe.forward_fp8 if s.wdtype == "fp8" else moe.forward
    fwd(cfg, s.T, x, w["W_r"], w["b"], w["W1"], w["W3"], w["W2"], w["Ws1"], w["Ws3"], w["Ws2"], y, ws, idx, gates)
    torch.cuda.synchronize()
    return y, idx, gates, moe.device_status(cfg, s.T, ws)


@pytest.mark.parametrize("name", list(CASES))
def test_debug_build_flags_nothing_and_matches_release(name):
    s = CASES[name]
    w = mdev.device_all(s)
    x = mdev.device_tensor(s, "x")
    y, idx, gates, status = _forward(s, w, x)
    assert status == 0
    with moe.using_library(moe.DEBUG_LIB_PATH):
        yd, idxd, gatesd, statusd = _forward(s, w, x)
    assert statusd == 0, f"debug build status {statusd:#x}"
    assert torch.equal(idxd, idx) and torch.equal(gatesd, gates)
    assert torch.equal(yd, y)


def test_debug_build_expert_parallel_steps():
    """The expert-parallel steps (dispatch_rows, expert-major reorder,
    experts, combine) of two ranks emulated on one GPU through the debug build
    give the release build's rows bit for bit, with no check firing."""
    from mixture_experts_layer_group_b200 import ep
    s = CASES["v3_like_small"]
    lc = ep.LayerCfg(d=s.d, d_ff=s.d_ff, n_routed=s.n_routed, n_shared=s.n_shared, top_k=s.top_k,
                     n_groups=s.n_groups, topk_groups=s.topk_groups, score=s.score, normalize=s.normalize,
                     route_scale=s.route_scale, group_score=s.group_score, dtype=s.dtype)
    w = mdev.device_all(s)
    x = mdev.device_tensor(s, "x")
    W = 2
    E = s.n_routed // W

    def run():
        ranks = []
        for r in range(W):
            wr = {"W_r": w["W_r"], "b": w["b"], "Ws1": w["Ws1"], "Ws3": w["Ws3"], "Ws2": w["Ws2"]}
            for nm in ("W1", "W3", "W2"):
                wr[nm] = w[nm][r * E:(r + 1) * E].contiguous()
            ranks.append(ep.ExpertParallelMoE(lc, r, W, wr))
        halves = [x[: s.T // 2].contiguous(), x[s.T // 2:].contiguous()]
        sents = [m.prepare(h) for m, h in zip(ranks, halves)]
        recv = ep.exchange_in_process(sents)
        backs = [m.compute(*rv) for m, rv in zip(ranks, recv)]
        outs = ep.return_in_process(sents, backs)
        ys = [m.finish(sn, o) for m, sn, o in zip(ranks, sents, outs)]
        torch.cuda.synchronize()
        return torch.cat(ys)

    y = run()
    with moe.using_library(moe.DEBUG_LIB_PATH):
        yd = run()
    assert torch.equal(yd, y)
