"""Throughput of the DeepSeekMoE layer forward on B200.

python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl ours|reference]

One step = one moe_forward over one batch of T synthetic tokens (router,
dispatch, row gather, SwiGLU GEMM, gate GEMM, combine), weights resident in
HBM. With N > 1 (torchrun, one process per GPU) every rank runs its own batch
on a full replica of the weights: data-parallel, no collective on the data
path (weak scaling); timing is the max over ranks. Rank 0 prints one JSON line.

The reference arm (--impl reference) times the fp64 CPU oracle on a bounded
sample of the same workload on the host cores.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import moe_inputs as mi  # noqa: E402

METRIC = "MoE-layer fwd tokens/s at V3 shape on 1 B200; % of bf16 TC / HBM roofline"
DEFAULT_CONFIG = "v3_prefill_bf16"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
KERNEL_SOURCES = ["mixture_experts_layer_group_b200/csrc/expert_tc.cu",
                  "mixture_experts_layer_group_b200/csrc/common.cuh"]
LAUNCHES_PER_STEP = 9  # router logits, router select, count, scan, scatter, gather, 2 GEMMs, combine


def describe(s: mi.LayerShape) -> str:
    route = f"{s.score} top-{s.top_k}"
    if s.n_groups > 1:
        route += f" in top-{s.topk_groups} of {s.n_groups} groups"
    if s.bias:
        route += " with selection bias"
    if s.normalize:
        route += f", gates normalised x{s.route_scale}"
    if s.zipf_s:
        route += f", Zipf {s.zipf_s} expert skew"
    return (f"{s.name}: DeepSeekMoE layer forward, T={s.T} tokens, d={s.d}, {s.n_shared} shared + "
            f"{s.n_routed} routed SwiGLU experts d_ff={s.d_ff}, {route}, {s.dtype}")


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            return json.load(f), "measured (MEASURED_PEAKS.json)"
    return dict(FALLBACK_PEAKS), "fallback (6.65 TB/s, 1.59 PFLOP/s)"


def kernel_sha() -> str:
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def ncu_traffic(config: str):
    """DRAM bytes per launch of the SwiGLU GEMM from a committed ncu capture,
    or None when absent or when the kernel source changed since."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f).get(config)
    if not rec or rec.get("kernel_sha") != kernel_sha():
        return None
    return rec.get("bytes_per_launch")


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id):
        self.gpu = gpu_id
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            sel = [f"--id={self.gpu}"] if self.gpu else []
            self.proc = subprocess.Popen(["nvidia-smi", *sel, f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        rows = []
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((float(parts[1]), float(parts[2]), parts[5:9]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for _, _, fl in rows for i, v in enumerate(fl) if v.lower() == "active"})
        return {"sm_mhz": float(np.median([r[0] for r in rows])), "sm_max_mhz": rows[0][1],
                "reasons": reasons, "samples": len(rows)}


def rank_env():
    """(world, rank, local_rank) from the torchrun environment (1, 0, 0 without it)."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def token_shape_for_rank(s: mi.LayerShape, rank: int) -> mi.LayerShape:
    """Every rank holds the same weights; its token batch comes from its own seed."""
    return s.with_(seed=(s.seed + 17 * rank) & 0xFF)


def max_over_ranks(values, device=None):
    """Element-wise max of a list of floats over all ranks (identity without a process group)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return list(values)
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def algorithmic(s: mi.LayerShape, counts: np.ndarray):
    """FLOPs and HBM bytes the layer must move (touched expert weights, router
    weights, x read, y written), and the SwiGLU GEMM's own bytes."""
    U = int((counts > 0).sum())
    e = 2 if s.dtype == "bf16" else 4
    flops = s.T * (s.top_k + s.n_shared) * 6 * s.d * s.d_ff
    layer_bytes = (U + s.n_shared) * 3 * s.d * s.d_ff * e + s.n_routed * s.d * e + 2 * s.T * s.d * e
    R = s.T * s.top_k
    swiglu_bytes = ((U + s.n_shared) * 2 * s.d * s.d_ff * e          # W1, W3 of touched experts
                    + (R + (s.T if s.n_shared else 0)) * s.d * e       # token rows read
                    + (R * s.d_ff + s.T * s.n_shared * s.d_ff) * e)    # SwiGLU rows written
    return U, flops, layer_bytes, swiglu_bytes


def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    import mixture_experts_layer_group_b200 as moe
    from mixture_experts_layer_group_b200 import build as lib_build
    from moe_inputs import build as gen_build
    from moe_inputs import device as mdev

    if rank == 0 or world == 1:
        lib_build.build()
        gen_build.build()
    if world > 1:
        dist.barrier()
    torch.cuda.set_device(local_rank)
    s = mi.SHAPES[args.config]
    # weights are the same replica everywhere; each rank draws its own token batch
    sx = token_shape_for_rank(s, rank)
    w = mdev.device_all(s)
    x = mdev.device_tensor(sx, "x")
    cfg = moe.make_cfg(s.d, s.d_ff, s.n_routed, s.n_shared, s.top_k, s.n_groups, s.topk_groups, s.score,
                       s.normalize, s.route_scale, s.group_score, s.dtype)
    ws = torch.empty(moe.workspace_size_host(cfg, s.T), dtype=torch.uint8, device="cuda")
    y = torch.empty_like(x)
    idx = torch.empty((s.T, s.top_k), dtype=torch.int32, device="cuda")
    gates = torch.empty((s.T, s.top_k), dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream()
    wargs = (w["W_r"], w["b"], w["W1"], w["W3"], w["W2"], w["Ws1"], w["Ws3"], w["Ws2"])

    def step():
        moe.forward(cfg, s.T, x, *wargs, y, ws, stream=stream)

    for _ in range(args.warmup):
        step()
    moe.forward(cfg, s.T, x, *wargs, y, ws, idx, gates, stream=stream)
    torch.cuda.synchronize()
    status = moe.device_status(cfg, s.T, ws)
    counts = np.bincount(idx.cpu().numpy().reshape(-1), minlength=s.n_routed)

    # --- device-timed region: K steps, stage events on the launching stream
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(7)] for _ in range(args.steps)]
    for row in ev:
        for e in row:
            e.record(stream)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    try:
        gpu_id = "GPU-" + str(torch.cuda.get_device_properties(local_rank).uuid)
    except Exception:
        gpu_id = None
    with ClockSampler(gpu_id) as clk:
        wall0 = time.perf_counter()
        t0.record(stream)
        for k in range(args.steps):
            moe.set_stage_events(ev[k])
            step()
        t1.record(stream)
        moe.set_stage_events(None)
        torch.cuda.synchronize()
        wall = time.perf_counter() - wall0
    if world > 1:
        dist.barrier()
    ms = t0.elapsed_time(t1) / args.steps
    stage_ms = {name: float(np.mean([ev[k][i].elapsed_time(ev[k][i + 1]) for k in range(args.steps)]))
                for i, name in enumerate(moe.STAGES)}

    # --- end to end: host tokens in, host output back, every step
    xh = x.cpu().pin_memory()
    yh = torch.empty_like(xh).pin_memory()
    for _ in range(max(1, args.warmup // 2)):
        moe.forward_host(cfg, s.T, xh, *wargs, yh, ws, stream=stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        moe.forward_host(cfg, s.T, xh, *wargs, yh, ws, stream=stream)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1) / args.steps

    ms, e2e_ms = max_over_ranks([ms, e2e_ms], device="cuda")
    if rank != 0:
        return None

    peaks, peak_src = load_peaks()
    U, flops, layer_bytes, swiglu_bytes = algorithmic(s, counts)
    t_sec = ms / 1e3
    tok_s = world * s.T / t_sec
    tflops = flops / t_sec / 1e12
    gbs = layer_bytes / t_sec / 1e9
    t_tc = flops / (peaks["bf16_tflops_sustained"] * 1e12)
    t_hbm = layer_bytes / (peaks["hbm_gbs"] * 1e9)
    sw_ms = stage_ms["gemm_swiglu"]
    achieved = swiglu_bytes / (sw_ms / 1e3) / 1e9
    clocks = clk.summary()
    out = {
        "metric": METRIC,
        "value": round(tok_s, 1),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": s.dtype,
        "data": "synthetic (seeded counter-based generator; random-init weights of the layer's shapes)",
        "config": {"workload": describe(s), "T": s.T, "d": s.d, "n_routed": s.n_routed,
                   "n_shared": s.n_shared, "d_ff": s.d_ff, "top_k": s.top_k, "global_batch": world * s.T,
                   "parallelism": f"dp{world} (independent replicas, no collective)",
                   "l2": "inputs larger than L2: every step streams "
                         f"{(U + s.n_shared) * 3 * s.d * s.d_ff * 2 / 1e9:.1f} GB of expert weights"},
        "e2e": {"value": round(world * s.T / (e2e_ms / 1e3), 1), "unit": "tokens/s",
                "h2d_bytes_per_step": s.T * s.d * (2 if s.dtype == "bf16" else 4),
                "d2h_bytes_per_step": s.T * s.d * (2 if s.dtype == "bf16" else 4)},
        "gpu_launches": LAUNCHES_PER_STEP * args.steps,
        "roofline": {"bound": "hbm", "kernel": "expert_gemm_tc_kernel<SwiGLU>",
                     "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": round(achieved / peaks["hbm_gbs"], 4), "traffic": ncu_traffic(args.config),
                     "peak_source": f"hbm_gbs, {peak_src}", "launch_ms": round(sw_ms, 4),
                     "algorithmic_bytes": swiglu_bytes},
        "layer": {"tflops": round(tflops, 1), "tc_frac_of_sustained": round(tflops * 1e12 / (peaks["bf16_tflops_sustained"] * 1e12), 4),
                  "hbm_gbs": round(gbs, 1), "hbm_frac": round(gbs / peaks["hbm_gbs"], 4),
                  "binding_roofline_ms": round(max(t_tc, t_hbm) * 1e3, 4),
                  "binding_frac": round(max(t_tc, t_hbm) / t_sec, 4),
                  "bound": "hbm" if t_hbm > t_tc else "tensor",
                  "touched_routed_experts": U, "stage_ms": {k: round(v, 4) for k, v in stage_ms.items()}},
        "clocks": clocks,
        "device_status": status,
        "wall_s_timed": round(wall, 3),
    }
    if world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(s, args.cpu_tokens)
    return out


def cpu_baseline(s: mi.LayerShape, n_tok: int):
    """The oracle, as it stands, on the host cores: the layer forward for a
    resident sample of n_tok tokens, repeated for about 10 s of CPU work."""
    sample = reference_sample(s, sample_token_cap(s, n_tok), 1234)
    n = sample[0].shape[0]
    times = [oracle_step(sample)]
    while sum(times) < 10.0 and len(times) < 200:
        times.append(oracle_step(sample))
    dt = float(np.mean(times))
    return {"value": round(n / dt, 3), "unit": "tokens/s", "cores": os.cpu_count(), "kind": "oracle",
            "sample": f"{n} seeded tokens of {s.name} (router, their experts, shared MLP, combine), fp64 numpy "
                      f"oracle with resident fp64 weights, {len(times)} repetitions, {sum(times):.1f} s"}


def reference_sample(s: mi.LayerShape, n_tok: int, seed: int):
    """The reference arm's resident inputs: n_tok seeded tokens of the
    workload with the router and the weights of every expert they use,
    widened to the oracle's fp64 once (as the GPU arm's weights sit in HBM
    before its timed region)."""
    import oracle
    rows = np.sort(np.random.default_rng(seed).choice(s.T, n_tok, replace=False))
    widen = (lambda a: mi.bf16_to_f32(a).astype(np.float64)) if s.dtype == "bf16" else \
        (lambda a: a.astype(np.float64))
    x64 = widen(mi.host_rows(s, "x", rows))
    W_r = widen(mi.host_tensor(s, "W_r").reshape(s.n_routed, s.d))
    b = mi.host_tensor(s, "b").astype(np.float64) if s.bias else None
    rcfg = oracle.RouterCfg(n_routed=s.n_routed, top_k=s.top_k, score=s.score, n_groups=s.n_groups,
                            topk_groups=s.topk_groups, normalize=s.normalize, route_scale=s.route_scale,
                            group_score=s.group_score)
    need = sorted(set(oracle.route(x64, W_r, b, rcfg).idx.reshape(-1).tolist()))
    experts = {e: tuple(widen(a) for a in mi.host_expert(s, e)) for e in need}
    shared = mi.host_shared(s)
    shared = None if shared is None else tuple(widen(a) for a in shared)
    return x64, W_r, b, rcfg, experts, shared


def oracle_step(sample) -> float:
    """Seconds for one oracle layer forward over a resident sample."""
    import oracle
    x64, W_r, b, rcfg, experts, shared = sample
    t0 = time.perf_counter()
    oracle.forward(x64, W_r, b, rcfg, lambda e: experts[e], shared)
    return time.perf_counter() - t0


def sample_token_cap(s: mi.LayerShape, want: int) -> int:
    """At most `want` tokens, fewer if their fp64 expert weights would take
    more than a quarter of the host's available memory."""
    try:
        import psutil
        avail = psutil.virtual_memory().available
    except Exception:  # no psutil: trust the request
        return want
    per_expert = 3 * s.d * s.d_ff * 8
    n = want
    while n > 1 and (n * s.top_k + s.n_shared) * per_expert > avail // 4:
        n -= 1
    return n


def run_reference(args, rank, world):
    """The reference arm of this tier: the fp64 oracle, as it stands, on the
    host cores. Each step runs the whole layer forward (router, every chosen
    expert, shared MLP, combine) for the same sample of tokens; the sample
    (1 to 4 tokens) is sized from a first timing so the run stays within
    about two minutes."""
    if rank != 0:
        return None
    s = mi.SHAPES[args.config]
    from moe_inputs import build as gen_build
    gen_build.build_host()

    step = oracle_step
    probe = reference_sample(s, 1, 99)
    t1 = min(step(probe) for _ in range(2))
    n_tok = int(max(1, min(sample_token_cap(s, args.cpu_tokens),
                           120.0 / max(1e-9, (args.steps + args.warmup) * t1))))
    sample = probe if n_tok == 1 else reference_sample(s, n_tok, 99)
    for _ in range(args.warmup):
        step(sample)
    times = [step(sample) for _ in range(args.steps)]
    ms = 1e3 * float(np.mean(times))
    v = n_tok / (ms / 1e3)
    desc = (f"{n_tok} seeded token(s) of {s.name} per step, the layer forward for them (router, their "
            f"experts, shared MLP, combine) in the fp64 numpy oracle, weights resident in fp64")
    return {"metric": METRIC, "value": round(v, 3), "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms, 1), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": {"workload": describe(s), "global_batch": n_tok},
            "cpu_baseline": {"value": round(v, 3), "unit": "tokens/s", "cores": os.cpu_count(), "kind": "oracle",
                             "sample": desc},
            "e2e": {"value": round(v, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def run_router_only(args):
    """moe_route alone (router logits + selection) on the config's x, W_r, b:
    for profiling the router without the expert weights on the device."""
    import torch
    import mixture_experts_layer_group_b200 as moe
    from mixture_experts_layer_group_b200 import build as lib_build
    from moe_inputs import build as gen_build
    from moe_inputs import device as mdev

    lib_build.build()
    gen_build.build()
    s = mi.SHAPES[args.config]
    x = mdev.device_tensor(s, "x")
    W_r = mdev.device_tensor(s, "W_r")
    b = mdev.device_tensor(s, "b") if s.bias else None
    cfg = moe.make_cfg(s.d, s.d_ff, s.n_routed, s.n_shared, s.top_k, s.n_groups, s.topk_groups, s.score,
                       s.normalize, s.route_scale, s.group_score, s.dtype)
    ws = torch.empty(moe.workspace_size(cfg, s.T), dtype=torch.uint8, device="cuda")
    idx = torch.empty((s.T, s.top_k), dtype=torch.int32, device="cuda")
    gates = torch.empty((s.T, s.top_k), dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream()
    for _ in range(args.warmup):
        moe.route(cfg, s.T, x, W_r, b, idx, gates, ws, stream=stream)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(args.steps):
        moe.route(cfg, s.T, x, W_r, b, idx, gates, ws, stream=stream)
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / args.steps
    if args.stage == "bias":
        # the balancing step on this batch's counts: route once, dispatch, then
        # time moe_bias_update alone (N fp32 updates; launch-bound)
        counts = torch.zeros(s.n_routed, dtype=torch.int32, device="cuda")
        moe.dispatch(cfg, s.T, idx, counts, None, None, ws, stream=stream)
        bias = b.clone() if b is not None else torch.zeros(s.n_routed, dtype=torch.float32, device="cuda")
        for _ in range(args.warmup):
            moe.bias_update(cfg, s.T, counts, 1e-3, bias, stream=stream)
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(args.steps):
            moe.bias_update(cfg, s.T, counts, 1e-3, bias, stream=stream)
        e1.record(stream)
        torch.cuda.synchronize()
        us = e0.elapsed_time(e1) / args.steps * 1e3
        return {"metric": "moe_bias_update time", "value": round(us, 2), "unit": "us", "steps": args.steps,
                "warmup": args.warmup, "higher_is_better": False, "config": {"workload": s.name, "N": s.n_routed}}
    flops = 2.0 * s.T * s.n_routed * s.d
    return {"metric": "router tokens/s (moe_route alone)", "value": round(s.T / (ms * 1e-3), 1),
            "unit": "tokens/s", "ms_per_step": round(ms, 4), "steps": args.steps, "warmup": args.warmup,
            "router_tflops": round(flops / (ms * 1e-3) / 1e12, 2), "config": {"workload": s.name, "T": s.T}}


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--config", default=DEFAULT_CONFIG, choices=list(mi.SHAPES))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-tokens", type=int, default=4)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--stage", default="layer", choices=["layer", "router", "bias"],
                    help="router: time moe_route alone; bias: time moe_bias_update (profiling aids; 1 GPU)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        args.warmup = 3
    world, rank, local_rank = rank_env()
    if args.stage in ("router", "bias"):
        print(json.dumps(run_router_only(args)), flush=True)
        return 0
    if args.impl == "reference":
        out = run_reference(args, rank, world)
        if out:
            print(json.dumps(out), flush=True)
        return 0
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local_rank))
    try:
        out = run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
    if out:
        print(json.dumps(out), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
