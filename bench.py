"""Throughput of the DeepSeekMoE layer forward on B200.

python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl ours|reference]

One step = one moe_forward over one batch of T synthetic tokens (router,
dispatch, row gather, SwiGLU GEMM, gate GEMM, combine), weights resident in
HBM. The timed loop calls moe_forward exactly as a user does (no per-stage
events, so the two GEMMs overlap through programmatic dependent launch); a
second, shorter pass with stage events gives the per-kernel times. With
--gpus N > 1 the script starts N local ranks itself (torch.distributed.run)
unless it already runs under torchrun; every rank runs its own batch on a full
replica of the weights: data-parallel, no collective on the data path (weak
scaling); timing is the max over ranks. Rank 0 prints one JSON line, with the
V3 decode layer timed the same way in its "decode" object.

The reference arm (--impl reference) times the fp64 CPU oracle on a bounded
sample of the same workload on the host cores.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import socket
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


def wait_event(ev, poll_s=0.0005):
    """Waits for a CUDA event by polling it with short sleeps, which release
    the interpreter lock, so the clock sampler's thread keeps running while
    the device works through the timed region."""
    while not ev.query():
        time.sleep(poll_s)


class ClockSampler:
    """SM clock and clock-event reasons of one GPU, polled through NVML every
    few milliseconds while the timed region runs (nvidia-smi's 200 ms period
    gives a single sample over a 0.1 s region)."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, uuid, period_s=0.003):
        self.uuid = uuid
        self.period = period_s
        self.samples = []
        self.handle = None
        self.max_mhz = None
        self._stop = threading.Event()
        self.t = None

    def __enter__(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nvml = pynvml
            self.handle = (pynvml.nvmlDeviceGetHandleByUUID(self.uuid) if self.uuid
                           else pynvml.nvmlDeviceGetHandleByIndex(0))
            self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(self.handle, pynvml.NVML_CLOCK_SM))
            self.t = threading.Thread(target=self._poll, daemon=True)
            self.t.start()
        except Exception:  # no NVML: the line reports the clocks as unsampled
            self.handle = None
        return self

    def _poll(self):
        nv = self.nvml
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self.handle, nv.NVML_CLOCK_SM)
                why = nv.nvmlDeviceGetCurrentClocksEventReasons(self.handle)
                self.samples.append((float(mhz), int(why)))
            except Exception:
                break
            self._stop.wait(self.period)

    def __exit__(self, *a):
        self._stop.set()
        if self.t is not None:
            self.t.join(timeout=5)

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unsampled"], "samples": 0}
        mhz = [m for m, _ in self.samples]
        seen = {}
        for _, why in self.samples:
            for bit, name in self.REASONS.items():
                if why & bit:
                    seen[name] = seen.get(name, 0) + 1
        return {"sm_mhz": float(np.median(mhz)), "sm_min_mhz": float(min(mhz)), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(seen), "reason_samples": seen, "samples": len(self.samples),
                "source": "NVML, every ~3 ms over the timed region"}


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


def weight_bytes_per_element(s: mi.LayerShape) -> float:
    """HBM bytes per expert-weight element: 2 (bf16), 4 (fp32), or 1 + 1/128^2 (e4m3 + block scale)."""
    if s.wdtype == "fp8":
        return 1.0 + 1.0 / (128 * 128)
    return 2.0 if s.dtype == "bf16" else 4.0


def algorithmic(s: mi.LayerShape, counts: np.ndarray):
    """What the layer must do, independent of how: FLOPs of the expert
    matmuls, HBM bytes of the layer (touched expert weights, router weights,
    x read, y written), and the SwiGLU GEMM's bytes counted two ways --
    touched W1/W3 weights plus x read once (the algorithmic count), and that
    plus the implementation's own token-row reads and SwiGLU-row writes."""
    U = int((counts > 0).sum())
    e = 2 if s.dtype == "bf16" else 4
    we = weight_bytes_per_element(s)
    flops = s.T * (s.top_k + s.n_shared) * 6 * s.d * s.d_ff
    layer_bytes = int((U + s.n_shared) * 3 * s.d * s.d_ff * we) + s.n_routed * s.d * e + 2 * s.T * s.d * e
    R = s.T * s.top_k
    w13 = int((U + s.n_shared) * 2 * s.d * s.d_ff * we)
    swiglu_alg = w13 + s.T * s.d * e
    swiglu_impl = (w13 + (R + (s.T if s.n_shared else 0)) * s.d * e
                   + (R * s.d_ff + s.T * s.n_shared * s.d_ff) * e)
    return {"U": U, "flops": flops, "layer_bytes": layer_bytes, "swiglu_alg": swiglu_alg,
            "swiglu_impl": swiglu_impl}


class Layer:
    """One layer configuration on the device: weights, a token batch, a
    workspace, and the moe_forward / moe_forward_host calls a user makes."""

    def __init__(self, s: mi.LayerShape, rank: int):
        import torch
        import mixture_experts_layer_group_b200 as moe
        from moe_inputs import device as mdev
        self.moe = moe
        self.s = s
        self.w = mdev.device_all(s)  # the same replica on every rank
        self.x = mdev.device_tensor(token_shape_for_rank(s, rank), "x")
        self.cfg = moe.make_cfg(s.d, s.d_ff, s.n_routed, s.n_shared, s.top_k, s.n_groups, s.topk_groups, s.score,
                                s.normalize, s.route_scale, s.group_score, s.dtype)
        self.ws = torch.empty(moe.workspace_size_host(self.cfg, s.T), dtype=torch.uint8, device="cuda")
        self.y = torch.empty_like(self.x)
        self.stream = torch.cuda.current_stream()
        w = self.w
        self.wargs = (w["W_r"], w["b"], w["W1"], w["W3"], w["W2"], w["Ws1"], w["Ws3"], w["Ws2"])

    def _forward(self, *extra):
        fwd = self.moe.forward_fp8 if self.s.wdtype == "fp8" else self.moe.forward
        fwd(self.cfg, self.s.T, self.x, *self.wargs, self.y, self.ws, *extra, stream=self.stream)

    def step(self):
        self._forward()

    def routing_counts(self):
        import torch
        s = self.s
        idx = torch.empty((s.T, s.top_k), dtype=torch.int32, device="cuda")
        gates = torch.empty((s.T, s.top_k), dtype=torch.float32, device="cuda")
        self._forward(idx, gates)
        torch.cuda.synchronize()
        status = self.moe.device_status(self.cfg, s.T, self.ws)
        return np.bincount(idx.cpu().numpy().reshape(-1), minlength=s.n_routed), status

    def timed(self, steps, clk=None):
        """ms per step of `steps` back-to-back moe_forward calls, CUDA events on the launching stream."""
        import torch
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        t0.record(self.stream)
        for _ in range(steps):
            self.step()
        t1.record(self.stream)
        wait_event(t1)
        torch.cuda.synchronize()
        return t0.elapsed_time(t1) / steps

    def graph_timed(self, steps):
        """ms per step of `steps` replays of one moe_forward captured in a CUDA
        graph (the serving pattern for small batches: no host launch work and
        shorter gaps between the layer's kernels), CUDA events on the replaying
        stream."""
        import torch
        side = torch.cuda.Stream()
        side.wait_stream(self.stream)
        fwd = self.moe.forward_fp8 if self.s.wdtype == "fp8" else self.moe.forward
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=side):
            fwd(self.cfg, self.s.T, self.x, *self.wargs, self.y, self.ws, stream=side)
        for _ in range(3):
            g.replay()
        torch.cuda.synchronize()
        cur = torch.cuda.current_stream()
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(cur)
        for _ in range(steps):
            g.replay()
        t1.record(cur)
        wait_event(t1)
        torch.cuda.synchronize()
        del g
        return t0.elapsed_time(t1) / steps

    def stage_pass(self, steps):
        """Per-stage ms (mean over `steps` calls) from the library's stage
        events; with events between the GEMMs the down GEMM starts after the
        SwiGLU GEMM instead of overlapping its drain."""
        import torch
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(7)] for _ in range(steps)]
        for row in ev:
            for e in row:
                e.record(self.stream)
        torch.cuda.synchronize()
        for k in range(steps):
            self.moe.set_stage_events(ev[k])
            self.step()
        self.moe.set_stage_events(None)
        torch.cuda.synchronize()
        return {name: float(np.mean([ev[k][i].elapsed_time(ev[k][i + 1]) for k in range(steps)]))
                for i, name in enumerate(self.moe.STAGES)}

    def e2e(self, steps, warmup, async_out=True):
        """ms per step through the host-buffer calls: x copied in from pinned
        host memory and y copied back to it on every step. async_out: the
        moe_forward_host(_fp8)_async calls (each step's output copy overlaps
        the next step; the wait for the last one is inside the timed region),
        else moe_forward_host(_fp8) (output copy on the caller's stream)."""
        import torch
        xh = self.x.cpu().pin_memory()
        yh = [torch.empty_like(xh).pin_memory() for _ in range(2)]
        fp8 = self.s.wdtype == "fp8"
        if async_out:
            fwd = self.moe.forward_host_fp8_async if fp8 else self.moe.forward_host_async
        else:
            fwd = self.moe.forward_host_fp8 if fp8 else self.moe.forward_host
        for i in range(warmup):
            fwd(self.cfg, self.s.T, xh, *self.wargs, yh[i & 1], self.ws, stream=self.stream)
        self.moe.host_wait(self.ws, self.stream)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(self.stream)
        for i in range(steps):
            fwd(self.cfg, self.s.T, xh, *self.wargs, yh[i & 1], self.ws, stream=self.stream)
        self.moe.host_wait(self.ws, self.stream)
        e1.record(self.stream)
        torch.cuda.synchronize()
        self.moe.workspace_release(self.ws)
        return e0.elapsed_time(e1) / steps, xh.numel() * xh.element_size(), yh[0].numel() * yh[0].element_size()

    def free(self):
        import torch
        self.w = self.x = self.ws = self.y = self.wargs = None
        torch.cuda.empty_cache()


def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    from mixture_experts_layer_group_b200 import build as lib_build
    from moe_inputs import build as gen_build

    if rank == 0 or world == 1:
        lib_build.build()
        gen_build.build()
    if world > 1:
        dist.barrier()
    torch.cuda.set_device(local_rank)
    s = mi.SHAPES[args.config]
    L = Layer(s, rank)
    for _ in range(args.warmup):
        L.step()
    counts, status = L.routing_counts()
    try:
        uuid = "GPU-" + str(torch.cuda.get_device_properties(local_rank).uuid)
    except Exception:
        uuid = None

    # --- device-timed region: K product-path steps (no stage events)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    with ClockSampler(uuid) as clk:
        wall0 = time.perf_counter()
        ms = L.timed(args.steps)
        wall = time.perf_counter() - wall0
    if world > 1:
        dist.barrier()
    # --- per-kernel times (separate pass with stage events)
    stage_ms = L.stage_pass(min(args.steps, 20))
    # --- end to end through the host-buffer entry point
    e2e_ms, h2d, d2h = L.e2e(args.steps, max(1, args.warmup // 2))
    e2e_sync_ms = L.e2e(args.steps, max(1, args.warmup // 2), async_out=False)[0]
    L.free()

    # --- the V3 decode layer, timed the same way
    dec = None
    if not args.no_decode and args.config != "v3_decode_bf16":
        ds = mi.SHAPES["v3_decode_bf16"]
        D = Layer(ds, rank)
        for _ in range(args.warmup):
            D.step()
        dcounts, dstatus = D.routing_counts()
        if world > 1:
            dist.barrier()
        with ClockSampler(uuid) as dclk:
            dms = D.timed(args.steps)
        dstage = D.stage_pass(min(args.steps, 20))
        dgraph = D.graph_timed(args.steps)
        D.free()
        dec = (ds, dms, dcounts, dstatus, dstage, dclk.summary(), dgraph)

    # --- the V3 prefill layer with FP8 expert weights, timed the same way
    f8 = None
    if not args.no_fp8 and s.name == "v3_prefill_bf16":
        fs = mi.SHAPES["v3_prefill_fp8"]
        Fl = Layer(fs, rank)
        for _ in range(args.warmup):
            Fl.step()
        fcounts, fstatus = Fl.routing_counts()
        if world > 1:
            dist.barrier()
        with ClockSampler(uuid) as fclk:
            fms = Fl.timed(args.steps)
        fstage = Fl.stage_pass(min(args.steps, 20))
        Fl.free()
        f8 = (fs, fms, fcounts, fstatus, fstage, fclk.summary())

    vals = [ms, e2e_ms, e2e_sync_ms] + ([dec[1], dec[6]] if dec else []) + ([f8[1]] if f8 else [])
    vals = max_over_ranks(vals, device="cuda")
    ms, e2e_ms, e2e_sync_ms = vals[0], vals[1], vals[2]
    if rank != 0:
        return None

    peaks, peak_src = load_peaks()
    A = algorithmic(s, counts)
    t_sec = ms / 1e3
    tflops = A["flops"] / t_sec / 1e12
    gbs = A["layer_bytes"] / t_sec / 1e9
    t_tc = A["flops"] / (peaks["bf16_tflops_sustained"] * 1e12)
    t_hbm = A["layer_bytes"] / (peaks["hbm_gbs"] * 1e9)
    sw_ms = stage_ms["gemm_swiglu"]
    achieved = A["swiglu_alg"] / (sw_ms / 1e3) / 1e9
    achieved_impl = A["swiglu_impl"] / (sw_ms / 1e3) / 1e9
    out = {
        "metric": METRIC,
        "value": round(world * s.T / t_sec, 1),
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
                         f"{(A['U'] + s.n_shared) * 3 * s.d * s.d_ff * weight_bytes_per_element(s) / 1e9:.1f} "
                         "GB of expert weights"},
        "e2e": {"value": round(world * s.T / (e2e_ms / 1e3), 1), "unit": "tokens/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": round(e2e_ms, 4),
                "api": ("moe_forward_host_fp8_async" if s.wdtype == "fp8" else "moe_forward_host_async")
                       + " (pinned host x in, y out, every step; each step's output copy overlaps the next "
                         "step, moe_host_wait for the last one inside the timed region)",
                "sync_ms_per_step": round(e2e_sync_ms, 4),
                "sync_api": ("moe_forward_host_fp8" if s.wdtype == "fp8" else "moe_forward_host")
                            + " (output copy on the caller's stream after each step)"},
        "gpu_launches": LAUNCHES_PER_STEP * args.steps,
        "roofline": {"bound": "hbm", "kernel": "expert_gemm_tc_kernel<SwiGLU>",
                     "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": round(achieved / peaks["hbm_gbs"], 4), "traffic": ncu_traffic(args.config),
                     "peak_source": f"hbm_gbs, {peak_src}", "launch_ms": round(sw_ms, 4),
                     "algorithmic_bytes": A["swiglu_alg"],
                     "counting": "touched W1/W3 weights + x read once; launch_ms from the stage pass",
                     "impl_bytes": A["swiglu_impl"], "impl_frac": round(achieved_impl / peaks["hbm_gbs"], 4)},
        "layer": {"tflops": round(tflops, 1),
                  "tc_frac_of_sustained": round(tflops * 1e12 / (peaks["bf16_tflops_sustained"] * 1e12), 4),
                  "hbm_gbs": round(gbs, 1), "hbm_frac": round(gbs / peaks["hbm_gbs"], 4),
                  "binding_roofline_ms": round(max(t_tc, t_hbm) * 1e3, 4),
                  "binding_frac": round(max(t_tc, t_hbm) / t_sec, 4),
                  "bound": "hbm" if t_hbm > t_tc else "tensor",
                  "touched_routed_experts": A["U"], "stage_ms": {k: round(v, 4) for k, v in stage_ms.items()},
                  "stage_pass": "separate pass with stage events (down GEMM not overlapped)"},
        "clocks": clk.summary(),
        "device_status": status,
        "wall_s_timed": round(wall, 3),
    }
    if dec:
        ds, dms, dcounts, dstatus, dstage, dclocks, dgraph = dec
        dms, dgraph = vals[3], vals[4]
        DA = algorithmic(ds, dcounts)
        dt = dms / 1e3
        d_t_hbm = DA["layer_bytes"] / (peaks["hbm_gbs"] * 1e9)
        d_t_tc = DA["flops"] / (peaks["bf16_tflops_sustained"] * 1e12)
        out["decode"] = {"workload": describe(ds), "ms_per_step": round(dms, 4),
                         "tokens_per_s": round(world * ds.T / dt, 1), "touched_routed_experts": DA["U"],
                         "hbm_gbs": round(DA["layer_bytes"] / dt / 1e9, 1),
                         "hbm_frac": round(DA["layer_bytes"] / dt / 1e9 / peaks["hbm_gbs"], 4),
                         "binding_frac": round(max(d_t_hbm, d_t_tc) / dt, 4),
                         "bound": "hbm" if d_t_hbm > d_t_tc else "tensor",
                         "bytes": DA["layer_bytes"], "stage_ms": {k: round(v, 4) for k, v in dstage.items()},
                         "clocks": dclocks, "device_status": dstatus,
                         "graph_ms_per_step": round(dgraph, 4),
                         "graph": "the same forward captured once in a CUDA graph and replayed (not the headline)"}
    if f8:
        fs, fms, fcounts, fstatus, fstage, fclocks = f8
        fms = vals[-1]
        FA = algorithmic(fs, fcounts)
        ft = fms / 1e3
        f_t_hbm = FA["layer_bytes"] / (peaks["hbm_gbs"] * 1e9)
        f_t_tc = FA["flops"] / (peaks["bf16_tflops_sustained"] * 1e12)
        out["fp8"] = {"workload": describe(fs) + ", expert weights e4m3 with one power-of-two scale per 128x128 block",
                      "ms_per_step": round(fms, 4), "tokens_per_s": round(world * fs.T / ft, 1),
                      "hbm_gbs": round(FA["layer_bytes"] / ft / 1e9, 1),
                      "hbm_frac": round(FA["layer_bytes"] / ft / 1e9 / peaks["hbm_gbs"], 4),
                      "tflops": round(FA["flops"] / ft / 1e12, 1),
                      "binding_frac": round(max(f_t_hbm, f_t_tc) / ft, 4),
                      "bound": "hbm" if f_t_hbm > f_t_tc else "tensor (bf16 MMA after dequantisation)",
                      "bytes": FA["layer_bytes"], "stage_ms": {k: round(v, 4) for k, v in fstage.items()},
                      "clocks": fclocks, "device_status": fstatus}
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


def free_port() -> int:
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        return sk.getsockname()[1]


def launch_ranks(n: int, argv) -> int:
    """Re-run this script as n local ranks, one process per GPU, through
    torch.distributed.run on 127.0.0.1; returns the launcher's exit code."""
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
           "--master-addr", "127.0.0.1", f"--master-port={free_port()}", os.path.abspath(__file__), *argv]
    return subprocess.call(cmd)


def check_launch(world: int, rank: int) -> int:
    """The rank plumbing alone: every rank joins a gloo group, rank 0 prints
    the ranks it saw."""
    import datetime
    import torch.distributed as dist
    if world > 1:
        dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
        seen = [None] * world
        dist.all_gather_object(seen, {"rank": rank, "pid": os.getpid()})
        dist.destroy_process_group()
    else:
        seen = [{"rank": 0, "pid": os.getpid()}]
    if rank == 0:
        print(json.dumps({"n_gpus": world, "ranks": seen}), flush=True)
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--config", default=DEFAULT_CONFIG, choices=list(mi.SHAPES))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-tokens", type=int, default=4)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-decode", action="store_true", help="skip the V3 decode sub-measurement")
    ap.add_argument("--no-fp8", action="store_true", help="skip the FP8-weight V3 prefill sub-measurement")
    ap.add_argument("--check-launch", action="store_true",
                    help="start the ranks, join a gloo process group, report them and exit (no GPU work)")
    ap.add_argument("--stage", default="layer", choices=["layer", "router", "bias"],
                    help="router: time moe_route alone; bias: time moe_bias_update (profiling aids; 1 GPU)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        args.warmup = 3
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        return launch_ranks(args.gpus, sys.argv[1:] if argv is None else list(argv))
    world, rank, local_rank = rank_env()
    if args.check_launch:
        return check_launch(world, rank)
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
