"""Shared helpers of the GPU parity tests: inputs on the device, the oracle
on the host (fp64), and the comparison rules.

Comparison rules:
  * routing: expert indices must equal the oracle's for every token the
    oracle does not flag; a flagged token (selection margin < 1e-6) may pick
    any selection that is optimal within the margin. Slot order may differ
    only where the oracle flags an order tie.
  * outputs: the relative Frobenius error ||y - y_ref|| / ||y_ref|| over the
    checked rows within 2e-2 for bf16 layers and 1e-5 for fp32 layers, and
    the same error of every single token row, max_t ||y_t - ref_t|| /
    ||ref_t||, within 1e-2 (bf16) and 1e-5 (fp32), where y_ref is the oracle
    evaluated with the GPU's selection for flagged tokens. The bf16 bound per
    token: the path rounds h, each gated expert row and y to bf16 (relative
    RMS 2^-9 / sqrt(3) ~ 1.1e-3 each), so a token's row error is ~2-3e-3
    with d in the hundreds or more; 1e-2 leaves a factor of 3 or more, while
    a token row that is wrong in a quarter of its columns shows ~0.5.
"""
from __future__ import annotations

import concurrent.futures
import threading

import numpy as np
import torch

import moe_inputs as mi
import oracle
from moe_inputs import device as mdev
import mixture_experts_layer_group_b200 as moe

TOL = {"bf16": 2e-2, "f32": 1e-5}
TOKEN_TOL = {"bf16": 1e-2, "f32": 1e-5}


def cfg_of(s: mi.LayerShape) -> moe.MoeCfg:
    return moe.make_cfg(s.d, s.d_ff, s.n_routed, s.n_shared, s.top_k, s.n_groups, s.topk_groups, s.score,
                        s.normalize, s.route_scale, s.group_score, s.dtype)


def router_cfg_of(s: mi.LayerShape) -> oracle.RouterCfg:
    return oracle.RouterCfg(n_routed=s.n_routed, top_k=s.top_k, score=s.score, n_groups=s.n_groups,
                            topk_groups=s.topk_groups, normalize=s.normalize, route_scale=s.route_scale,
                            group_score=s.group_score)


def f64(a):
    return a.astype(np.float64) if a.dtype != np.uint16 else mi.bf16_to_f32(a).astype(np.float64)


def t2np64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def device_layer(s: mi.LayerShape) -> dict:
    return mdev.device_all(s)


def workspace(cfg, T, host=False):
    n = (moe.workspace_size_host if host else moe.workspace_size)(cfg, T)
    return torch.empty(max(n, 256), dtype=torch.uint8, device="cuda")


def run_forward(s: mi.LayerShape, w: dict, x: torch.Tensor, ws=None):
    cfg = cfg_of(s)
    T = x.shape[0]
    ws = workspace(cfg, T) if ws is None else ws
    y = torch.empty_like(x)
    idx = torch.empty((T, s.top_k), dtype=torch.int32, device="cuda")
    gates = torch.empty((T, s.top_k), dtype=torch.float32, device="cuda")
    moe.forward(cfg, T, x, w["W_r"], w["b"], w["W1"], w["W3"], w["W2"], w["Ws1"], w["Ws3"], w["Ws2"], y, ws,
                idx, gates)
    torch.cuda.synchronize()
    status = moe.device_status(cfg, T, ws)
    assert status == 0, f"device status bits {status:#x}"
    return y, idx.cpu().numpy().astype(np.int64), gates.cpu().numpy().astype(np.float64)


def check_routing(gidx: np.ndarray, ggates: np.ndarray, r: oracle.Routing, rcfg: oracle.RouterCfg,
                  gate_rtol=2e-5):
    T, k = gidx.shape
    same_order = (gidx == r.idx).all(axis=1)
    same_set = np.array([set(gidx[t]) == set(r.idx[t]) for t in range(T)])
    flagged = r.flagged
    bad_unflagged = ~same_set & ~flagged
    assert not bad_unflagged.any(), f"routing differs on unflagged tokens {np.where(bad_unflagged)[0][:10]}"
    bad_order = same_set & ~same_order & ~(r.order_tie | flagged)
    assert not bad_order.any(), f"slot order differs without an order tie: {np.where(bad_order)[0][:10]}"
    # flagged tokens: the GPU's selection must be optimal within the tie margin
    for t in np.where(flagged & ~same_set)[0]:
        sel = gidx[t]
        keys = r.keys[t]
        assert len(set(sel.tolist())) == k, t
        if r.group_tie[t]:
            S = rcfg.n_routed // rcfg.n_groups
            gs = oracle.moe_oracle._group_scores(keys[None, :], rcfg)[0]
            thr = np.sort(gs)[::-1][rcfg.topk_groups - 1] - 2 * oracle.TIE_EPS
            groups = set((sel // S).tolist())
            assert len(groups) <= rcfg.topk_groups and all(gs[g] >= thr for g in groups), t
        else:
            assert r.allowed[t][sel].all(), t
            best = np.sort(np.where(r.allowed[t], keys, -np.inf))[::-1][:k].sum()
            assert keys[sel].sum() >= best - 2 * k * oracle.TIE_EPS, t
    # gates of the GPU's own selection, from the oracle's unbiased scores
    want = oracle.gates_for(r.scores, gidx, rcfg)
    np.testing.assert_allclose(ggates, want, rtol=gate_rtol, atol=1e-7)
    return int(flagged.sum()), int((~same_set).sum())


def rel_fro(y, ref):
    return float(np.linalg.norm(y - ref) / max(np.linalg.norm(ref), 1e-300))


def token_rel_max(y, ref):
    """max over token rows of ||y_t - ref_t|| / ||ref_t||, and the worst row."""
    num = np.linalg.norm(y - ref, axis=1)
    den = np.maximum(np.linalg.norm(ref, axis=1), 1e-300)
    r = num / den
    t = int(np.argmax(r)) if r.size else -1
    return (float(r[t]) if r.size else 0.0), t


def check_outputs(y, ref, dtype, what=""):
    """Whole-block relative Frobenius error and the worst token row, each
    within its bound; returns (whole, worst_token, worst_row)."""
    err = rel_fro(y, ref)
    tok, t = token_rel_max(y, ref)
    assert err <= TOL[dtype], (what, "rel_fro", err)
    assert tok <= TOKEN_TOL[dtype], (what, "token", t, tok)
    return err, tok, t


def oracle_forward(s: mi.LayerShape, x64, W_r64, b, expert_fn, shared, gidx=None):
    """fp64 oracle output for token rows x64; tokens the oracle flags are
    re-evaluated with the GPU's selection gidx (when given)."""
    rcfg = router_cfg_of(s)
    y, r, idx, gates = oracle.forward(x64, W_r64, b, rcfg, expert_fn, shared)
    if gidx is not None:
        redo = r.flagged & ~(gidx == r.idx).all(axis=1)
        if redo.any():
            rows = np.where(redo)[0]
            r2 = oracle.route(x64[rows], W_r64, b, rcfg)
            y2, *_ = oracle.forward(x64[rows], W_r64, b, rcfg, expert_fn, shared, routing=r2,
                                    idx_override=gidx[rows])
            y[rows] = y2
    return y, r


def host_expert_fn(s: mi.LayerShape):
    def fn(e):
        w1, w3, w2 = mi.host_expert(s, e)
        return f64(w1), f64(w3), f64(w2)
    return fn


class PrefetchedExperts:
    """expert(e) for the oracle, with the fp64 weights of the next experts in
    `order` generated and widened on worker threads (at most `depth` ahead,
    so only a few experts are resident). Experts outside the order, or asked
    for again, are built on the spot."""

    def __init__(self, s: mi.LayerShape, order, depth: int = 6, fn=None):
        self.fn = host_expert_fn(s) if fn is None else fn
        self.order = list(order)
        self.pos = {e: i for i, e in enumerate(self.order)}
        self.pool = concurrent.futures.ThreadPoolExecutor(max_workers=depth)
        self.depth = depth
        self.futs = {}
        self.next = 0
        self.lock = threading.Lock()
        self._fill(0)

    def _fill(self, i):
        with self.lock:
            self.next = max(self.next, i)
            while self.next < len(self.order) and self.next < i + self.depth:
                e = self.order[self.next]
                self.futs[e] = self.pool.submit(self.fn, e)
                self.next += 1

    def __call__(self, e):
        fut = self.futs.pop(e, None)
        if e in self.pos:
            self._fill(self.pos[e] + 1)
        return fut.result() if fut is not None else self.fn(e)

    def close(self):
        self.pool.shutdown(wait=True, cancel_futures=True)


def chunk_probe_rows(idx: np.ndarray, n_routed: int, max_tok: int = 256):
    """Token rows that reach the expert GEMMs' chunk edges: for every routed
    expert, the first token of each chunk the kernels cut its rows into
    (ceil(rows / max_tok) chunks of equal size) and its last token (the end
    of its last, ragged 32-token block)."""
    T, k = idx.shape
    picks = set()
    for e in range(n_routed):
        toks = np.nonzero((idx == e).any(axis=1))[0]
        n = toks.size
        if n == 0:
            continue
        nc = (n + max_tok - 1) // max_tok
        cs = (n + nc - 1) // nc
        for c in range(nc):
            picks.add(int(toks[c * cs]))
        picks.add(int(toks[-1]))
    return np.array(sorted(picks), dtype=np.int64)


def host_shared64(s: mi.LayerShape):
    sh = mi.host_shared(s)
    return None if sh is None else tuple(f64(a) for a in sh)
