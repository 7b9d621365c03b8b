"""Expert parallelism on the GPU: ranks holding contiguous expert blocks
exchange permuted rows; each rank's output must equal moe_forward on the
whole layer for its tokens, bit for bit. Several ranks are driven from one
process, one phase at a time (no kernel waits on another rank), and a
single-rank NCCL group runs forward() with the real collectives."""
import os
import socket

import pytest
import torch

import moe_inputs as mi
from moe_inputs import device as mdev
import mixture_experts_layer_group_b200 as moe
from mixture_experts_layer_group_b200 import ep

from gpu_helpers import cfg_of, run_forward

pytestmark = pytest.mark.gpu

LS = mi.LayerShape
LAYERS = {
    "v3_like": LS("ep_v3_like", T=300, d=512, n_routed=32, n_shared=1, d_ff=256, top_k=4, score="sigmoid",
                  n_groups=4, topk_groups=2, normalize=True, route_scale=2.5, seed=41, bias=True),
    "softmax_2shared": LS("ep_softmax", T=173, d=384, n_routed=24, n_shared=2, d_ff=384, top_k=3, score="softmax",
                          seed=42),
    "f32": LS("ep_f32", T=77, d=136, n_routed=12, n_shared=1, d_ff=200, top_k=3, score="sigmoid", normalize=True,
              route_scale=2.5, dtype="f32", seed=43, bias=True),
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


def layer_cfg(s):
    return ep.LayerCfg(s.d, s.d_ff, s.n_routed, s.n_shared, s.top_k, s.n_groups, s.topk_groups, s.score,
                       s.normalize, s.route_scale, s.group_score, s.dtype)


def shard(w, rank, world, N):
    E = N // world
    out = {"W_r": w["W_r"], "b": w["b"], "Ws1": w["Ws1"], "Ws3": w["Ws3"], "Ws2": w["Ws2"]}
    for nm in ("W1", "W3", "W2"):
        out[nm] = w[nm][rank * E:(rank + 1) * E].contiguous()
    return out


@pytest.mark.parametrize("name,world", [("v3_like", 2), ("v3_like", 4), ("softmax_2shared", 3), ("f32", 2)])
def test_ep_ranks_equal_single_gpu_forward(name, world):
    s = LAYERS[name]
    w = mdev.device_all(s)
    lc = layer_cfg(s)
    # every rank has its own batch (its own seed and size)
    toks = [mdev.device_tensor(s.with_(T=s.T - 17 * r, seed=s.seed + 100 + r), "x") for r in range(world)]
    refs = [run_forward(s.with_(T=x.shape[0]), w, x)[0] for x in toks]
    ranks = [ep.ExpertParallelMoE(lc, r, world, shard(w, r, world, s.n_routed)) for r in range(world)]
    sents = [rk.prepare(x) for rk, x in zip(ranks, toks)]
    recvs = ep.exchange_in_process(sents)
    backs = [rk.compute(*rv) for rk, rv in zip(ranks, recvs)]
    outs = ep.return_in_process(sents, backs)
    ys = [rk.finish(st, o) for rk, st, o in zip(ranks, sents, outs)]
    torch.cuda.synchronize()
    for r in range(world):
        assert torch.equal(ys[r], refs[r]), (name, world, r)


def test_ep_reorder_round_trip_and_block_order():
    # blocks (p, e) of a 3 x 4 count matrix (zeros included): expert-major
    # order is e-major, p-minor, and reordering back restores the input
    W, E, d = 3, 4, 8
    counts = torch.tensor([[2, 0, 1, 3], [0, 0, 2, 1], [4, 1, 0, 0]], dtype=torch.int32, device="cuda")
    M = int(counts.sum())
    rows = torch.arange(M * d, dtype=torch.float32, device="cuda").view(M, d)
    em = torch.empty_like(rows)
    moe.ep_reorder(W, E, counts, d * 4, rows, em, True)
    back = torch.empty_like(rows)
    moe.ep_reorder(W, E, counts, d * 4, em, back, False)
    torch.cuda.synchronize()
    assert torch.equal(back, rows)
    c = counts.cpu().tolist()
    src_off = {}
    o = 0
    for p in range(W):
        for e in range(E):
            src_off[(p, e)] = o
            o += c[p][e]
    want = []
    for e in range(E):
        for p in range(W):
            want += list(range(src_off[(p, e)], src_off[(p, e)] + c[p][e]))
    assert torch.equal(em, rows[torch.tensor(want, device="cuda")])


def test_experts_rejects_counts_that_do_not_sum_to_rows():
    s = LAYERS["v3_like"]
    w = mdev.device_all(s)
    cfg = moe.make_cfg(s.d, s.d_ff, 4, 0, 1)
    rows = 64
    x = mdev.device_tensor(s.with_(T=rows), "x")
    y = torch.full_like(x, 7.0)
    ws = torch.empty(moe.experts_workspace_size(cfg, rows), dtype=torch.uint8, device="cuda")
    counts = torch.tensor([10, 20, 30, 40], dtype=torch.int32, device="cuda")  # sums to 100, not 64
    moe.experts(cfg, rows, counts, x, None, w["W1"][:4].contiguous(), w["W3"][:4].contiguous(),
                w["W2"][:4].contiguous(), y, ws)
    torch.cuda.synchronize()
    assert moe.device_status(cfg, rows, ws) & moe.MOE_DEV_BAD_EXPERT
    assert (y == 7.0).all()  # nothing was computed or written


def _free_port():
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        return sk.getsockname()[1]


def test_ep_forward_through_nccl_single_rank():
    # forward() with torch.distributed over NCCL, one rank holding all experts
    import datetime
    import torch.distributed as dist
    s = LAYERS["v3_like"]
    w = mdev.device_all(s)
    x = mdev.device_tensor(s, "x")
    ref = run_forward(s, w, x)[0]
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()))
    dist.init_process_group("nccl", rank=0, world_size=1, timeout=datetime.timedelta(seconds=60),
                            device_id=torch.device("cuda", 0))
    try:
        y = ep.ExpertParallelMoE(layer_cfg(s), 0, 1, shard(w, 0, 1, s.n_routed)).forward(x)
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    assert torch.equal(y, ref)
