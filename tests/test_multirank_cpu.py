"""Host logic of the multi-process bench on CPU: world-size 2 over gloo.

The layer shards by tokens (independent replicas, no collective on the data
path); what needs checking without GPUs is the rank plumbing: distinct token
batches per rank on identical weights, the max-over-ranks timing reduction,
and that only rank 0 reports."""
import os
import socket

import pytest
import torch.multiprocessing as mp

import moe_inputs as mi


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import datetime
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world), RANK=str(rank),
                      LOCAL_RANK=str(rank))
    import bench
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    try:
        w, r, lr = bench.rank_env()
        s = mi.SHAPES["v3_decode_bf16"]
        sx = bench.token_shape_for_rank(s, r)
        x_head = mi.host_tensor(sx, "x", 0, 64).tolist()
        wr_head = mi.host_tensor(s, "W_r", 0, 64).tolist()
        # rank r "took" 1 + r ms and 10 - r ms on its two timers
        mx = bench.max_over_ranks([1.0 + r, 10.0 - r])
        out.put((r, w, lr, sx.seed, x_head, wr_head, mx))
    finally:
        dist.destroy_process_group()


def test_two_rank_plumbing():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(2):
        r, w, lr, seed, x_head, wr_head, mx = q.get(timeout=120)
        res[r] = (w, lr, seed, x_head, wr_head, mx)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert res[0][0] == res[1][0] == 2 and res[0][1] == 0 and res[1][1] == 1
    assert res[0][2] != res[1][2]                 # different token seeds
    assert res[0][3] != res[1][3]                 # so different token batches
    assert res[0][4] == res[1][4]                 # identical weights
    assert res[0][5] == res[1][5] == [2.0, 10.0]  # max over ranks of each timer


def test_single_process_defaults(monkeypatch):
    import bench
    for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    assert bench.rank_env() == (1, 0, 0)
    assert bench.max_over_ranks([3.0, 4.0]) == [3.0, 4.0]
    s = mi.SHAPES["v3_prefill_bf16"]
    assert bench.token_shape_for_rank(s, 0) == s


def _ref_worker(rank, world, port, out):
    os.environ.update(WORLD_SIZE=str(world), RANK=str(rank), LOCAL_RANK=str(rank))
    import contextlib
    import io
    import bench
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        rc = bench.main(["--impl", "reference", "--config", "gshard_tiny_f32", "--steps", "1", "--warmup", "3",
                         "--cpu-tokens", "2"])
    out.put((rank, rc, buf.getvalue()))


def test_reference_arm_reports_on_rank0_only():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_ref_worker, args=(r, 2, 0, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = {}
    for _ in range(2):
        r, rc, text = q.get(timeout=180)
        got[r] = (rc, text)
    for p in procs:
        p.join(timeout=60)
    assert got[0][0] == 0 and got[1][0] == 0
    assert '"impl": "reference"' in got[0][1] and got[1][1].strip() == ""


def test_bench_gpus_2_starts_two_ranks():
    # `bench.py --gpus 2` outside torchrun re-launches itself as two local
    # ranks; --check-launch stops after the ranks have joined a gloo group
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = {k: v for k, v in os.environ.items() if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK")}
    out = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--gpus", "2", "--check-launch"],
                         capture_output=True, text=True, timeout=240, env=env, cwd=root)
    assert out.returncode == 0, out.stderr[-2000:]
    rep = json.loads([ln for ln in out.stdout.splitlines() if ln.startswith("{")][-1])
    assert rep["n_gpus"] == 2
    assert sorted(r["rank"] for r in rep["ranks"]) == [0, 1]
    assert len({r["pid"] for r in rep["ranks"]}) == 2


class _OracleOps:
    """CPU stand-ins for the device steps of an expert-parallel rank (fp64,
    from the oracle's definitions), so the exchange logic of the product's
    ExpertParallelMoE can run over gloo without a GPU."""

    def __init__(self, lc, E):
        import oracle
        self.o = oracle
        self.lc, self.E = lc, E
        self.rcfg = oracle.RouterCfg(n_routed=lc.n_routed, top_k=lc.top_k, score=lc.score, n_groups=lc.n_groups,
                                     topk_groups=lc.topk_groups, normalize=lc.normalize,
                                     route_scale=lc.route_scale, group_score=lc.group_score)

    def route_dispatch(self, x, W_r, b):
        import numpy as np
        import torch
        r = self.o.route(x.numpy(), W_r.numpy(), None if b is None else b.numpy(), self.rcfg)
        counts, offsets, perm = self.o.permutation(r.idx, self.lc.n_routed)
        k = self.lc.top_k
        T = x.shape[0]
        pos = np.empty(T * k, dtype=np.int64)
        pos[perm] = np.arange(T * k)
        slot_pos = np.empty((T, k), dtype=np.int64)
        for t in range(T):  # the token's rows in ascending expert order
            order = np.argsort(r.idx[t], kind="stable")
            slot_pos[t] = pos[t * k + order]
        x_perm = x[torch.from_numpy(perm // k)]
        gate_perm = torch.from_numpy(r.gates.reshape(-1)[perm])
        return (torch.from_numpy(counts.astype(np.int32)), torch.from_numpy(slot_pos), x_perm, gate_perm)

    def reorder(self, W, block_counts, rows, to_expert_major):
        import torch
        c = block_counts.tolist()
        src, o = {}, 0
        for p in range(W):
            for e in range(self.E):
                src[(p, e)] = o
                o += c[p][e]
        em = [i for e in range(self.E) for p in range(W) for i in range(src[(p, e)], src[(p, e)] + c[p][e])]
        idx = torch.tensor(em, dtype=torch.int64)
        if to_expert_major:
            return rows[idx]
        out = torch.empty_like(rows)
        out[idx] = rows
        return out

    def experts(self, counts, rows, gates, W1, W3, W2):
        import torch
        out = torch.empty_like(rows)
        o = 0
        for e, n in enumerate(counts.tolist()):
            if n:
                y = self.o.expert_ffn(rows[o:o + n].numpy(), W1[e].numpy(), W3[e].numpy(), W2[e].numpy())
                out[o:o + n] = torch.from_numpy(y * gates[o:o + n].numpy()[:, None])
            o += n
        return out

    def shared(self, x, Ws1, Ws3, Ws2):
        import torch
        return torch.from_numpy(self.o.expert_ffn(x.numpy(), Ws1.numpy(), Ws3.numpy(), Ws2.numpy()))

    def combine(self, routed_rows, slot_pos, shared_rows):
        y = routed_rows[slot_pos].sum(dim=1)
        return y if shared_rows is None else y + shared_rows


def _ep_worker(rank, world, port, out):
    import datetime
    import numpy as np
    import torch
    import torch.distributed as dist
    import oracle
    from mixture_experts_layer_group_b200 import ep
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world), RANK=str(rank))
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    try:
        rng = np.random.default_rng(7)  # the same layer on every rank
        N, d, F, k, ns = 12, 10, 8, 3, 1
        W_r = rng.standard_normal((N, d)) / np.sqrt(d)
        b = rng.uniform(-0.1, 0.1, N)
        W1, W3 = rng.standard_normal((N, F, d)) / np.sqrt(d), rng.standard_normal((N, F, d)) / np.sqrt(d)
        W2 = rng.standard_normal((N, d, F)) / np.sqrt(F)
        Ws = (rng.standard_normal((ns * F, d)), rng.standard_normal((ns * F, d)), rng.standard_normal((d, ns * F)))
        x = np.random.default_rng(100 + rank).standard_normal((20 + 5 * rank, d))  # own tokens per rank
        lc = ep.LayerCfg(d, F, N, ns, k, n_groups=4, topk_groups=2, score="sigmoid", normalize=True,
                         route_scale=2.5, dtype="f32")
        E = N // world
        t = torch.from_numpy
        w = {"W_r": t(W_r), "b": t(b), "W1": t(W1[rank * E:(rank + 1) * E]), "W3": t(W3[rank * E:(rank + 1) * E]),
             "W2": t(W2[rank * E:(rank + 1) * E]), "Ws1": t(Ws[0]), "Ws3": t(Ws[1]), "Ws2": t(Ws[2])}
        layer = ep.ExpertParallelMoE(lc, rank, world, w, ops=_OracleOps(lc, E))
        y = layer.forward(t(x)).numpy()
        rcfg = _OracleOps(lc, E).rcfg
        ref, *_ = oracle.forward(x, W_r, b, rcfg, lambda e: (W1[e], W3[e], W2[e]), Ws)
        out.put((rank, float(np.abs(y - ref).max()), float(np.abs(ref).max())))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_expert_parallel_exchange_over_gloo(world):
    # each rank routes its own tokens, sends rows to the ranks holding their
    # experts, computes its expert block, returns the rows and combines: the
    # result is the oracle's whole-layer forward on that rank's tokens
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_ep_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=180) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, err, scale in res:
        assert err <= 1e-12 * max(scale, 1.0), (rank, err)
