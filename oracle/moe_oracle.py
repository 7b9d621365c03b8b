"""Plain fp64 CPU definition of the DeepSeekMoE layer forward.

TEST INFRASTRUCTURE ONLY. Only the tests, the smoke check and the bench's CPU
baseline may import this module; the library never does, and it shares no
code with the CUDA path.

Everything here is written from the pages' statement of the layer:
  * "DeepSeek-V3.2-Exp · Mixture of experts", section "All 19 steps": the
    router (z = x W_r, s = sigma(z), top-8 of s+b within the top 4 groups,
    G_i = 2.5 s_i E_i / sum_j s_j E_j), the routed SwiGLU expert
    (g = x W1, u = x W3, a = g sigma(g), h = a * u, E = h W2), the shared
    expert, and Delta_ffn = y_routed + y_shared.
  * the same page's quoted MoE module: tokens flattened to one axis, the
    shared MLP of width n_shared * moe_inter_dim applied to every token.
  * "DeepSeekMoE" walkthrough, Step 2: the GShard router (dot product with
    every centroid, softmax over all of them, keep the top 2 values as gates,
    the rest are 0 -- no renormalisation).
  * "The DeepSeekMoE Architecture.", Idea 1 / Idea 2: fine-grained
    segmentation and shared-expert isolation.

Readings where the pages are silent (each is listed in the design notes):
  * group score: sum of the two largest s+b in the group ("top2_sum"); the
    page names the top-4-groups step but not the score. "max" is offered too.
  * groups are contiguous index ranges of N / n_groups experts.
  * ties: larger value first, then lower index (groups and experts).
  * tie flags: a token is flagged when a selection boundary margin is below
    TIE_EPS = 1e-6 (the k-th vs (k+1)-th allowed key, or the TG-th vs
    (TG+1)-th group score); slot-order ties are flagged separately.
  * the residual is not part of Delta_ffn.
No value is rounded: inputs are widened exactly to fp64 and stay there.

Pins (tests/test_oracle_pins.py), by function:
  * softmax / sigmoid / silu: closed forms and value pins (sigma(ln 3) = 3/4,
    silu(ln 3) = 3/4 ln 3).
  * router_logits: the product with each router row written out.
  * route: top-k against brute force over all subsets, with and without the
    group limit; tie flags; normalised gates summing to route_scale; the bias
    steering the selection but not the gates.
  * gates_for: a hand-computed example; equal to route's gates.
  * permutation: the sorted (expert, token) pairs.
  * bias_update: a hand example and its sign / magnitude properties.
  * expert_ffn / forward / gate_matrix: the SwiGLU bilinear identity, the
    segmentation and shared-fusion identities, the dense ceiling, identical
    experts (route_scale x FFN + shared), the GShard two-expert closed form,
    expert and token permutation equivariance, the idx_override path on the
    routing's own selection and on a hand-built exact tie.
  * e4m3_value / dequant_fp8: every code against the OCP E4M3 definition; a
    hand-computed 128 x 128 block example.
  * expert_params / router_params / block_params / routing_combinations /
    flops_per_token: the pages' printed counts.
The pages print no worked layer output, so output values are pinned only
through those identities and closed forms: beyond them, parity unpinned.
"""
from __future__ import annotations

from dataclasses import dataclass
from math import comb

import numpy as np

TIE_EPS = 1e-6


@dataclass
class RouterCfg:
    n_routed: int
    top_k: int
    score: str = "softmax"  # "softmax" | "sigmoid"
    n_groups: int = 1
    topk_groups: int = 1
    normalize: bool = False
    route_scale: float = 1.0
    group_score: str = "top2_sum"  # "top2_sum" | "max"


@dataclass
class Routing:
    idx: np.ndarray  # [T, k] int64, slots in descending key order
    gates: np.ndarray  # [T, k] fp64
    scores: np.ndarray  # [T, N] fp64 (s, before the bias)
    keys: np.ndarray  # [T, N] fp64 (s + b)
    allowed: np.ndarray  # [T, N] bool (experts inside the chosen groups)
    sel_tie: np.ndarray  # [T] bool: selection boundary margin < TIE_EPS
    group_tie: np.ndarray  # [T] bool: group boundary margin < TIE_EPS
    order_tie: np.ndarray  # [T] bool: two selected keys closer than TIE_EPS

    @property
    def flagged(self) -> np.ndarray:
        return self.sel_tie | self.group_tie


# ---------------------------------------------------------------- scores ----

def softmax(z: np.ndarray) -> np.ndarray:
    """exp(z_e - max z) / sum_j exp(z_j - max z) over the last axis
    ("DeepSeekMoE" walkthrough, Step 2: exponentiate and normalise)."""
    m = z.max(axis=-1, keepdims=True)
    e = np.exp(z - m)
    return e / e.sum(axis=-1, keepdims=True)


def sigmoid(z: np.ndarray) -> np.ndarray:
    """1 / (1 + exp(-z)), the per-expert affinity s = sigma(z) of the router
    ("DeepSeek-V3.2-Exp · Mixture of experts", All 19 steps)."""
    return 1.0 / (1.0 + np.exp(-z))


def silu(g: np.ndarray) -> np.ndarray:
    """a = g sigma(g) (same page, routed-expert steps)."""
    return g * sigmoid(g)


# ---------------------------------------------------------------- router ----

def router_logits(x: np.ndarray, W_r: np.ndarray) -> np.ndarray:
    """z = x W_r, one logit per routed expert; W_r is stored [N, d] (one row
    per expert "centroid"), so z = x @ W_r^T."""
    return x @ W_r.T


def _group_scores(keys: np.ndarray, cfg: RouterCfg) -> np.ndarray:
    T, N = keys.shape
    G = cfg.n_groups
    grouped = keys.reshape(T, G, N // G)
    if cfg.group_score == "max":
        return grouped.max(axis=-1)
    top2 = -np.sort(-grouped, axis=-1)[:, :, :2]
    return top2.sum(axis=-1)


def _descending(values: np.ndarray) -> np.ndarray:
    """Indices ordered by larger value first, lower index first among equals."""
    return np.argsort(-values, axis=-1, kind="stable")


def route(x: np.ndarray, W_r: np.ndarray, b: np.ndarray | None, cfg: RouterCfg) -> Routing:
    """Router of the "All 19 steps" list, in the page's order:
    z = x W_r; s = score(z); selection on s + b restricted to the top
    groups; gates from the unbiased s (normalised and scaled, or the raw
    score values for the GShard-style softmax router)."""
    N, k = cfg.n_routed, cfg.top_k
    z = router_logits(x, W_r)
    s = softmax(z) if cfg.score == "softmax" else sigmoid(z)
    keys = s + (0.0 if b is None else b[None, :].astype(np.float64))
    T = keys.shape[0]

    allowed = np.ones((T, N), dtype=bool)
    group_tie = np.zeros(T, dtype=bool)
    if cfg.n_groups > 1:
        gs = _group_scores(keys, cfg)
        gorder = _descending(gs)
        keep = gorder[:, : cfg.topk_groups]
        gmask = np.zeros_like(gs, dtype=bool)
        np.put_along_axis(gmask, keep, True, axis=1)
        allowed = np.repeat(gmask, N // cfg.n_groups, axis=1)
        if cfg.topk_groups < cfg.n_groups:
            gsorted = np.take_along_axis(gs, gorder, axis=1)
            group_tie = (gsorted[:, cfg.topk_groups - 1] - gsorted[:, cfg.topk_groups]) < TIE_EPS

    masked = np.where(allowed, keys, -np.inf)
    order = _descending(masked)
    idx = order[:, :k].astype(np.int64)
    ksorted = np.take_along_axis(masked, order, axis=1)
    n_allowed = allowed.sum(axis=1)
    sel_tie = np.zeros(T, dtype=bool)
    has_next = n_allowed > k
    if k < N:
        margin = ksorted[:, k - 1] - np.where(has_next, ksorted[:, min(k, N - 1)], -np.inf)
        sel_tie = margin < TIE_EPS
    order_tie = np.zeros(T, dtype=bool)
    if k > 1:
        order_tie = (np.diff(-ksorted[:, :k], axis=1) < TIE_EPS).any(axis=1)

    s_sel = np.take_along_axis(s, idx, axis=1)
    if cfg.normalize:
        gates = cfg.route_scale * s_sel / s_sel.sum(axis=1, keepdims=True)
    else:
        gates = cfg.route_scale * s_sel
    return Routing(idx, gates, s, keys, allowed, sel_tie, group_tie, order_tie)


def gates_for(routing_scores: np.ndarray, idx: np.ndarray, cfg: RouterCfg) -> np.ndarray:
    """Gates of a given selection, from the unbiased scores (used when a
    tied token is re-evaluated with another valid selection)."""
    s_sel = np.take_along_axis(routing_scores, idx, axis=1)
    if cfg.normalize:
        return cfg.route_scale * s_sel / s_sel.sum(axis=1, keepdims=True)
    return cfg.route_scale * s_sel


# ------------------------------------------------------------ permutation ----

def permutation(idx: np.ndarray, n_routed: int):
    """Expert histogram and expert-contiguous token lists, as the quoted
    forward counts the selections per expert and finds each expert's rows:
    counts[e] = number of (token, slot) pairs that chose e; offsets is their
    exclusive prefix sum; perm[offsets[e] + r] is the r-th such pair in
    ascending token order, stored as token * k + slot."""
    T, k = idx.shape
    flat = idx.reshape(-1)
    counts = np.bincount(flat, minlength=n_routed).astype(np.int64)
    offsets = np.zeros(n_routed + 1, dtype=np.int64)
    offsets[1:] = np.cumsum(counts)
    perm = np.empty(T * k, dtype=np.int64)
    for e in range(n_routed):
        tok, slot = np.where(idx == e)  # row-major: ascending token
        perm[offsets[e]: offsets[e + 1]] = tok * k + slot
    return counts, offsets, perm


# ------------------------------------------------------------ balancing ----

def bias_update(b: np.ndarray, counts: np.ndarray, T: int, k: int, gamma: float) -> np.ndarray:
    """Auxiliary-loss-free load balancing, the per-batch bias nudge (grasp.study
    lesson on DeepSeek-V3's MoE design, "3.2. Auxiliary-Loss-Free Load
    Balancing": each expert's bias is adjusted by whether it was overloaded or
    underloaded in the batch; "The DeepSeekMoE Architecture.", configuration
    table: "aux-loss-free bias"). Reading (the pages give the direction only):
    overloaded = more than the mean load T*k/N pairs, which lowers b_e by
    gamma; underloaded raises it by gamma; exactly the mean leaves it.
    Returns fp64; the caller's bias is fp32, so compare after rounding."""
    counts = np.asarray(counts, dtype=np.int64)
    N = counts.shape[0]
    mean = T * k / N  # exact comparison below uses integers
    direction = np.sign(T * k - N * counts)  # +1 under, -1 over, 0 at the mean
    assert np.all((counts > mean) == (direction < 0))
    return np.asarray(b, dtype=np.float64) + gamma * direction


# ---------------------------------------------------------------- experts ----

def expert_ffn(x: np.ndarray, W1: np.ndarray, W3: np.ndarray, W2: np.ndarray) -> np.ndarray:
    """One SwiGLU expert on token rows x [n, d]: g = x W1, u = x W3,
    h = silu(g) * u, E = h W2, with W1, W3 stored [d_ff, d] and W2 [d, d_ff]
    (out x in), so the products are x @ W1^T and h @ W2^T."""
    g = x @ W1.T
    u = x @ W3.T
    h = silu(g) * u
    return h @ W2.T


def gate_matrix(idx: np.ndarray, gates: np.ndarray, n_routed: int) -> np.ndarray:
    """G [T, N]: G[t, i] is the gate of expert i for token t, zero for every
    expert outside the token's selection (the equation list's G_i carries the
    selection indicator E_sel_i, so unselected experts contribute nothing)."""
    T, k = idx.shape
    G = np.zeros((T, n_routed), dtype=np.float64)
    rows = np.repeat(np.arange(T), k)
    G[rows, idx.reshape(-1)] = gates.reshape(-1)
    return G


def forward(x: np.ndarray, W_r: np.ndarray, b, cfg: RouterCfg, expert, shared=None,
            routing: Routing | None = None, idx_override: np.ndarray | None = None):
    """Delta_ffn = y_routed + y_shared for token rows x [T, d] (fp64), the
    last steps of the "All 19 steps" list ("DeepSeek-V3.2-Exp · Mixture of
    experts"): y_routed = sum_i G_i E_i(x) over the routed experts, with
    E_i the SwiGLU expert and G_i zero outside the selection, and y_shared
    the always-on shared MLP, ungated.

    expert(i) returns (W1_i, W3_i, W2_i) as fp64 arrays; shared is None or
    (Ws1, Ws3, Ws2), the fused shared MLP of width n_shared * d_ff. The sum
    over i runs in ascending expert index; E_i is evaluated only on the rows
    where G_i is nonzero (a zero gate adds nothing). idx_override replaces
    the selection (gates recomputed from the unbiased scores) to evaluate an
    alternative valid routing of tied tokens. Returns (y, routing, idx,
    gates)."""
    if routing is None:
        routing = route(x, W_r, b, cfg)
    idx, gates = routing.idx, routing.gates
    if idx_override is not None:
        idx = idx_override.astype(np.int64)
        gates = gates_for(routing.scores, idx, cfg)
    G = gate_matrix(idx, gates, cfg.n_routed)
    y_routed = np.zeros_like(x, dtype=np.float64)
    for i in range(cfg.n_routed):
        rows = np.nonzero(G[:, i])[0]
        if rows.size == 0:
            continue
        y_routed[rows] += G[rows, i][:, None] * expert_ffn(x[rows], *expert(i))
    y_shared = 0.0 if shared is None else expert_ffn(x, *shared)
    return y_routed + y_shared, routing, idx, gates


# ---------------------------------------------------- FP8 expert weights ----

def e4m3_value(codes: np.ndarray) -> np.ndarray:
    """Value of OCP FP8 E4M3 codes (the element format of the FP8 checkpoint
    the "DeepSeek-V3.2-Exp · Mixture of experts" page's Parameters section
    mentions; format from the OCP 8-bit floating point specification):
    1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits; exponent field 0
    holds subnormals m 2^-9; no infinities; 0x7F and 0xFF are NaN."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    mag = np.where(e == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    mag = np.where((c & 0x7F) == 0x7F, np.nan, mag)
    return sign * mag


def dequant_fp8(codes: np.ndarray, scales: np.ndarray, block: int = 128) -> np.ndarray:
    """w[r, c] = e4m3(codes[r, c]) * 2^(scales[r // block, c // block] - 127),
    exactly, in fp64: one UE8M0 (power-of-two) scale per block x block tile.
    The pages say only that the checkpoint carries FP8 block scales; the block
    size (128 x 128) and the scale format are DeepSeek-V3's."""
    codes = np.asarray(codes, dtype=np.uint8)
    R, C = codes.shape
    assert R % block == 0 and C % block == 0 and scales.shape == (R // block, C // block)
    values = e4m3_value(np.arange(256, dtype=np.uint8))[codes]        # the code table, indexed
    factors = np.exp2(np.asarray(scales, dtype=np.float64) - 127.0)   # exact powers of two
    return (values.reshape(R // block, block, C // block, block) * factors[:, None, :, None]).reshape(R, C)


# ------------------------------------------------- counts the pages print ----

def expert_params(d: int, d_ff: int) -> int:
    """W1, W3 (d -> d_ff) and W2 (d_ff -> d), no biases ("Parameters" table,
    routed/shared expert rows)."""
    return 3 * d * d_ff


def router_params(d: int, n_routed: int) -> int:
    """Router rows plus one bias value per routed expert ("Parameters" table,
    router row)."""
    return n_routed * d + n_routed


def block_params(d: int, d_ff: int, n_routed: int, n_shared: int) -> int:
    return router_params(d, n_routed) + (n_routed + n_shared) * expert_params(d, d_ff)


def routing_combinations(n_experts: int, k: int) -> int:
    """Number of distinct expert teams a token can be served by: C(n, k)
    ("DeepSeekMoE" walkthrough, Step 5)."""
    return comb(n_experts, k)


def segment_expert(W1, W3, W2, m: int):
    """Fine-grained segmentation ("The DeepSeekMoE Architecture.", Idea 1):
    split one expert of width d_ff into m experts of width d_ff/m, slicing
    the rows of W1, W3 and the columns of W2."""
    F = W1.shape[0]
    assert F % m == 0
    w = F // m
    return [(W1[i * w:(i + 1) * w], W3[i * w:(i + 1) * w], W2[:, i * w:(i + 1) * w]) for i in range(m)]


def flops_per_token(d: int, d_ff: int, top_k: int, n_shared: int) -> int:
    """Expert-matmul FLOPs per token: (k + n_shared) experts x 3 matmuls x 2 d d_ff."""
    return (top_k + n_shared) * 6 * d * d_ff
