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
