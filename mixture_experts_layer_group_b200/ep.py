"""Expert parallelism for the DeepSeekMoE layer forward.

The routed experts are split over W ranks (one process per GPU): rank r holds
the contiguous block of E = N / W experts [r E, (r + 1) E), as the quoted
MoE.__init__ on the "DeepSeek-V3.2-Exp · Mixture of experts" page slices them
per rank. The router and the shared MLP are on every rank, and every rank
routes its own tokens. Where that excerpt all-reduces the dense output, this
path moves only the routed rows: an all-to-all sends each permuted token row
to the rank holding its expert, and a second one returns the gated expert
rows; the combine stays local.

Every compute step runs in the library's CUDA kernels through its C ABI
(moe_route, moe_dispatch_rows, moe_ep_reorder, moe_experts, moe_combine).
This module only orders the calls, sizes the buffers and owns the two
exchanges (torch.distributed all_to_all_single; NCCL on GPUs). Each row is
computed exactly as moe_forward computes it, so a rank's output equals
moe_forward's on the same tokens bit for bit.

The step is split into phases around the exchanges (prepare, compute,
finish) so that a caller can drive them itself; forward() runs them with
torch.distributed.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch

from . import (MoeCfg, combine, dispatch_rows, ep_reorder, experts, experts_workspace_size, make_cfg, route,
               workspace_size)


@dataclass
class LayerCfg:
    """The whole layer's configuration (the fields of moe_cfg)."""

    d: int
    d_ff: int
    n_routed: int
    n_shared: int
    top_k: int
    n_groups: int = 1
    topk_groups: int = 1
    score: str = "softmax"
    normalize: bool = False
    route_scale: float = 1.0
    group_score: str = "top2_sum"
    dtype: str = "bf16"

    def moe_cfg(self) -> MoeCfg:
        return make_cfg(self.d, self.d_ff, self.n_routed, self.n_shared, self.top_k, self.n_groups,
                        self.topk_groups, self.score, self.normalize, self.route_scale, self.group_score, self.dtype)


class CudaOps:
    """The device steps of an expert-parallel rank, each one C-ABI call."""

    def __init__(self, lc: LayerCfg, local_experts: int, device="cuda"):
        self.lc = lc
        self.cfg = lc.moe_cfg()
        self.E = local_experts
        self.device = device
        self.dtype = torch.bfloat16 if lc.dtype == "bf16" else torch.float32
        # grouped-expert problems: the local experts, and the shared MLP as one group
        self.cfg_local = make_cfg(lc.d, lc.d_ff, local_experts, 0, 1, dtype=lc.dtype)
        self.cfg_shared = make_cfg(lc.d, max(lc.n_shared, 1) * lc.d_ff, 1, 0, 1, dtype=lc.dtype)

    def _ws(self, nbytes):
        return torch.empty(max(nbytes, 256), dtype=torch.uint8, device=self.device)

    def route_dispatch(self, x, W_r, b):
        lc, T = self.lc, x.shape[0]
        ws = self._ws(workspace_size(self.cfg, T))
        idx = torch.empty((T, lc.top_k), dtype=torch.int32, device=self.device)
        gates = torch.empty((T, lc.top_k), dtype=torch.float32, device=self.device)
        route(self.cfg, T, x, W_r, b, idx, gates, ws)
        counts = torch.empty(lc.n_routed, dtype=torch.int32, device=self.device)
        offsets = torch.empty(lc.n_routed + 1, dtype=torch.int32, device=self.device)
        slot_pos = torch.empty((T, lc.top_k), dtype=torch.int32, device=self.device)
        x_perm = torch.empty((T * lc.top_k, lc.d), dtype=self.dtype, device=self.device)
        gate_perm = torch.empty(T * lc.top_k, dtype=torch.float32, device=self.device)
        dispatch_rows(self.cfg, T, idx, gates, x, counts, offsets, slot_pos, x_perm, gate_perm, ws)
        return counts, slot_pos, x_perm, gate_perm

    def reorder(self, W, block_counts, rows, to_expert_major):
        out = torch.empty_like(rows)
        if rows.numel():
            ep_reorder(W, self.E, block_counts, rows[0].numel() * rows.element_size(), rows, out, to_expert_major)
        return out

    def experts(self, counts, rows, gates, W1, W3, W2):
        M = rows.shape[0]
        y = torch.empty_like(rows)
        if M:
            ws = self._ws(experts_workspace_size(self.cfg_local, M))
            experts(self.cfg_local, M, counts, rows, gates, W1, W3, W2, y, ws)
        return y

    def shared(self, x, Ws1, Ws3, Ws2):
        T = x.shape[0]
        y = torch.empty_like(x)
        ws = self._ws(experts_workspace_size(self.cfg_shared, T))
        counts = torch.tensor([T], dtype=torch.int32, device=self.device)
        experts(self.cfg_shared, T, counts, x, None, Ws1, Ws3, Ws2, y, ws)
        return y

    def combine(self, routed_rows, slot_pos, shared_rows):
        T = slot_pos.shape[0]
        y = torch.empty((T, self.lc.d), dtype=self.dtype, device=self.device)
        combine(self.cfg, T, routed_rows, slot_pos, shared_rows, y)
        return y


@dataclass
class Sent:
    """What a rank sends in the first exchange, and what it keeps for finish()."""

    block_counts: torch.Tensor  # [W, E] int32: rows for each destination rank's local experts
    rows: torch.Tensor          # [R, d] permuted token rows, destination-major
    gates: torch.Tensor         # [R] fp32
    splits: list                # rows per destination rank
    slot_pos: torch.Tensor      # [T, k]
    x: torch.Tensor             # [T, d]


class ExpertParallelMoE:
    """One rank of the expert-parallel layer.

    weights: W_r [N, d], b [N] or None, this rank's W1, W3 [E, d_ff, d] and
    W2 [E, d, d_ff], and the shared Ws1, Ws3, Ws2 (or None). ops: the device
    steps (CudaOps by default, the CUDA library; there is no other backend in
    the package)."""

    def __init__(self, lc: LayerCfg, rank: int, world: int, weights: dict, ops=None, group=None):
        if lc.n_routed % world:
            raise ValueError(f"n_routed {lc.n_routed} does not split over {world} ranks")
        self.lc, self.rank, self.world = lc, rank, world
        self.E = lc.n_routed // world
        self.w = weights
        self.ops = CudaOps(lc, self.E) if ops is None else ops
        self.group = group

    # ------------------------------------------------------------ phases --
    def prepare(self, x) -> Sent:
        """Route this rank's tokens and lay out the rows to send."""
        counts, slot_pos, x_perm, gate_perm = self.ops.route_dispatch(x, self.w["W_r"], self.w.get("b"))
        block_counts = counts.view(self.world, self.E)
        splits = [int(v) for v in block_counts.sum(dim=1).tolist()]
        return Sent(block_counts, x_perm, gate_perm, splits, slot_pos, x)

    def compute(self, recv_counts, recv_rows, recv_gates):
        """The local experts on the rows received from every rank.
        recv_counts [W, E]: rows from source rank p for local expert e;
        recv_rows / recv_gates: source-major, as an all-to-all delivers them.
        Returns the gated rows in the same source-major order."""
        W = self.world
        rows_em = self.ops.reorder(W, recv_counts, recv_rows, True)
        gates_em = self.ops.reorder(W, recv_counts, recv_gates.view(-1, 1), True).view(-1)
        per_expert = recv_counts.sum(dim=0).to(torch.int32)
        y_em = self.ops.experts(per_expert, rows_em, gates_em, self.w["W1"], self.w["W3"], self.w["W2"])
        return self.ops.reorder(W, recv_counts, y_em, False)

    def finish(self, sent: Sent, back_rows):
        """Shared MLP on this rank's tokens and the combine."""
        shared = None
        if self.lc.n_shared:
            shared = self.ops.shared(sent.x, self.w["Ws1"], self.w["Ws3"], self.w["Ws2"])
        return self.ops.combine(back_rows, sent.slot_pos, shared)

    # ----------------------------------------------------------- forward --
    def forward(self, x):
        """The layer forward on this rank's tokens, with the two exchanges
        done by torch.distributed (every rank of the group calls it)."""
        import torch.distributed as dist
        g = self.group
        sent = self.prepare(x)
        recv_counts = torch.empty_like(sent.block_counts)
        dist.all_to_all_single(recv_counts, sent.block_counts.contiguous(), group=g)
        recv_splits = [int(v) for v in recv_counts.sum(dim=1).tolist()]
        M = sum(recv_splits)
        recv_rows = sent.rows.new_empty((M,) + tuple(sent.rows.shape[1:]))
        recv_gates = sent.gates.new_empty(M)
        dist.all_to_all_single(recv_rows, sent.rows, recv_splits, sent.splits, group=g)
        dist.all_to_all_single(recv_gates, sent.gates, recv_splits, sent.splits, group=g)
        back = self.compute(recv_counts, recv_rows, recv_gates)
        out_rows = sent.rows.new_empty(sent.rows.shape)
        dist.all_to_all_single(out_rows, back, sent.splits, recv_splits, group=g)
        return self.finish(sent, out_rows)


def exchange_in_process(sents):
    """The two exchanges for ranks driven from one process (no collective):
    given every rank's Sent, returns each rank's (recv_counts, recv_rows,
    recv_gates) in source-major order. Used to run several ranks' kernels on
    one device, one phase at a time; nothing waits on another rank."""
    W = len(sents)
    out = []
    for q in range(W):
        counts = torch.stack([s.block_counts[q] for s in sents])
        rows, gates = [], []
        for s in sents:
            start = sum(s.splits[:q])
            rows.append(s.rows[start:start + s.splits[q]])
            gates.append(s.gates[start:start + s.splits[q]])
        out.append((counts.contiguous(), torch.cat(rows), torch.cat(gates)))
    return out


def return_in_process(sents, backs):
    """The second exchange for ranks driven from one process: rank p gets,
    for each destination q, the block q computed for it, in destination order."""
    W = len(sents)
    outs = []
    for p in range(W):
        parts = []
        for q in range(W):
            recv_splits_q = [s.splits[q] for s in sents]
            start = sum(recv_splits_q[:p])
            parts.append(backs[q][start:start + recv_splits_q[p]])
        outs.append(torch.cat(parts))
    return outs
