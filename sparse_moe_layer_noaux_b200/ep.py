"""Expert parallelism of the DeepSeekMoE layer over torch.distributed ranks.

The routed experts are spread over the `world` ranks of a process group, rank r
holding experts [r * E/world, (r + 1) * E/world); the router and the shared
experts are replicated, and every rank brings its own tokens ("DeepSeek-V3
notes" (knlb.dev), § infrastructure: expert parallelism with all-to-all dispatch
and combine; § architecture: a token goes to a limited number of nodes — with
contiguous expert blocks per rank and groups that do not straddle ranks, to at
most topk_group ranks).

A token crosses to a rank once, however many of its experts live there: the
source sends one row per (token, destination rank) carrying the token's values
and routing, the destination runs all of the token's experts it was sent and
sends back one row, their weighted sum.  So each direction moves at most
min(k, topk_group ranks) rows per token instead of k.

Redundant experts (same notes, § infrastructure, prefilling: copies of the
experts with the most load, placed from live statistics, to balance the ranks):
an EPPlacement lists the ranks holding each expert; the rows of an expert with
n copies are split over them by token index mod n.  EPPlacement.from_load builds
one from per-expert row counts (libmoe's moe_ep_place).

Every step of the layer runs in libmoe (include/moe.h lists the sequence); this
module only allocates the buffers and moves them between ranks with the process
group's all-to-all (NCCL on GPUs): the per-rank row counts, the send rows, and
after the experts the return rows.  The split sizes of an all-to-all are host
integers, so the counts are read back to the host once per forward.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import List, Optional

import torch

from . import abi
from .workloads import MoEShape


@dataclass
class EPStep:
    """One rank's buffers for one batch, filled phase by phase."""

    T: int
    idx: torch.Tensor            # [T, k] int32
    w: torch.Tensor              # [T, k] fp32
    send_counts: torch.Tensor    # [world] int32: rows for each rank
    send_rows: torch.Tensor      # [T * min(k, world), send_row_bytes] uint8, sorted by rank
    send_row_of: torch.Tensor    # [T, k] int32: send row of a token's first slot on a rank, else -1
    send_splits: Optional[List[int]] = None   # rows to each rank
    recv_splits: Optional[List[int]] = None   # rows from each rank
    recv_rows: Optional[torch.Tensor] = None    # [R, send_row_bytes] uint8
    return_rows: Optional[torch.Tensor] = None  # [R, return_row_bytes] uint8
    back_rows: Optional[torch.Tensor] = None    # [sum(send_splits), return_row_bytes] uint8, send order
    y_shared: Optional[torch.Tensor] = None     # [T, H] fp16 (block-scaled)
    y_shared_scale: Optional[torch.Tensor] = None


class EPPlacement:
    """Which ranks hold a copy of each routed expert.

    expert_ranks: int32 [E, max_rep] (host): the ranks holding expert e in its first
    entries, then -1; None means contiguous blocks of E/world experts per rank and no
    copies.  A rank holds its experts in ascending id order.
    """

    def __init__(self, E: int, world: int, expert_ranks: Optional[torch.Tensor] = None):
        if world < 1 or E % world:
            raise ValueError(f"world {world} must divide n_routed_experts {E}")
        self.E, self.world, self.expert_ranks = E, world, expert_ranks

    @classmethod
    def from_load(cls, E: int, world: int, load, n_redundant: int, max_rep: int = 2) -> "EPPlacement":
        """Copies of the most loaded experts, from rows per expert [E] (moe_ep_place)."""
        return cls(E, world, abi.ep_place(E, world, load, n_redundant, max_rep))

    def local_experts(self, rank: int):
        """(local_of int32 [E] or None, n_local, the rank's expert ids in local order)."""
        if self.expert_ranks is None:
            El = self.E // self.world
            return None, El, list(range(rank * El, (rank + 1) * El))
        local_of, n = abi.ep_local_experts(self.E, self.world, rank, self.expert_ranks)
        return local_of, n, [e for e in range(self.E) if int(local_of[e]) >= 0]

    def rank_weights(self, t: torch.Tensor, rank: int) -> torch.Tensor:
        """Rank `rank`'s experts of a per-expert tensor [E, ...], in local order."""
        ids = self.local_experts(rank)[2]
        return t[torch.as_tensor(ids, device=t.device)].contiguous()


class MoELayerEP:
    """One rank's part of an expert-parallel layer.

    shape: the whole layer's configuration (E = all routed experts).
    world, rank: the ranks of `group` (default: the default process group).
    placement: an EPPlacement (default: blocks of E/world experts, no copies).
    w_gate / w_up [n_local, I, H], w_down [n_local, H, I]: this rank's experts in the
    placement's local order (placement.rank_weights; expert_block for blocks).
    router_w, e_bias and the shared experts: the full (replicated) tensors.
    """

    def __init__(self, shape: MoEShape, world: int, rank: int, router_w, e_bias, w_gate, w_up, w_down,
                 ws_gate=None, ws_up=None, ws_down=None, group=None, placement: Optional[EPPlacement] = None,
                 _kernels=None):
        if world < 1 or shape.E % world:
            raise ValueError(f"world {world} must divide n_routed_experts {shape.E}")
        if not 0 <= rank < world:
            raise ValueError(f"rank {rank} outside [0, {world})")
        self.shape, self.world, self.rank, self.group = shape, world, rank, group
        self.cfg = abi.MoEConfig.from_shape(shape)
        self.router_w, self.e_bias = router_w, e_bias
        self.w_gate, self.w_up, self.w_down = w_gate, w_up, w_down
        self.ws_gate, self.ws_up, self.ws_down = ws_gate, ws_up, ws_down
        self.device = router_w.device
        self.placement = placement if placement is not None else EPPlacement(shape.E, world)
        if self.placement.E != shape.E or self.placement.world != world:
            raise ValueError("placement was made for another E or world")
        local_of, self.n_local, self.local_ids = self.placement.local_experts(rank)
        if w_gate.shape[0] != self.n_local:
            raise ValueError(f"w_gate holds {w_gate.shape[0]} experts, rank {rank} holds {self.n_local}")
        ranks = self.placement.expert_ranks
        self.expert_ranks = None if ranks is None else ranks.to(self.device)
        self.local_of = None if local_of is None else local_of.to(self.device)
        # The library binding; the CPU tests of the exchange pass a stand-in.
        self.lib = _kernels if _kernels is not None else abi
        self.send_row_bytes, self.return_row_bytes = self.lib.ep_row_bytes(self.cfg)
        self._ws: Optional[torch.Tensor] = None

    def _empty(self, shape, dtype):
        return torch.empty(shape, dtype=dtype, device=self.device)

    def _workspace(self, need: int) -> torch.Tensor:
        need = max(need, 256)
        if self._ws is None or self._ws.numel() < need:
            self._ws = self._empty(need, torch.uint8)
        return self._ws

    # ---- phases (each a libmoe call; the collectives sit between them) ----
    def send(self, x: torch.Tensor) -> EPStep:
        """Route the rank's tokens and build their send rows, one per (token, rank)."""
        s, L = self.shape, self.lib
        T, k = x.shape[0], s.k
        n_max = L.ep_send_rows_max(self.cfg, T, self.world)
        st = EPStep(T=T, idx=self._empty((T, k), torch.int32), w=self._empty((T, k), torch.float32),
                    send_counts=self._empty(self.world, torch.int32),
                    send_rows=self._empty((n_max, self.send_row_bytes), torch.uint8),
                    send_row_of=self._empty((T, k), torch.int32))
        ws = self._workspace(max(L.workspace_size(self.cfg, T),
                                 L.ep_workspace_size(self.cfg, self.world, T, 0, n_local=self.n_local)))
        if T:
            L.moe_route(self.cfg, x, self.router_w, self.e_bias, st.idx, st.w, ws)
        L.moe_ep_send(self.cfg, self.world, x, st.idx, st.w, st.send_counts, st.send_rows, st.send_row_of, ws,
                      expert_ranks=self.expert_ranks)
        return st

    def plan(self, st: EPStep, recv_counts: torch.Tensor) -> None:
        """From the row counts this rank received ([world], one per source): the split
        sizes of the exchanges and the receive, return and back buffers."""
        s = self.shape
        both = torch.stack([st.send_counts, recv_counts]).cpu()
        st.send_splits = [int(v) for v in both[0]]
        st.recv_splits = [int(v) for v in both[1]]
        R = sum(st.recv_splits)
        st.recv_rows = self._empty((R, self.send_row_bytes), torch.uint8)
        st.return_rows = self._empty((R, self.return_row_bytes), torch.uint8)
        st.back_rows = self._empty((sum(st.send_splits), self.return_row_bytes), torch.uint8)
        st.y_shared = self._empty((st.T, s.H), torch.float16)
        st.y_shared_scale = self._empty((st.T, self.lib.y_perm_scale_cols(s.H)), torch.uint8)

    def experts(self, st: EPStep, x: torch.Tensor) -> None:
        """The rank's experts over the received rows; the shared experts over its own tokens."""
        L = self.lib
        R = st.recv_rows.shape[0]
        ws = self._workspace(L.ep_workspace_size(self.cfg, self.world, st.T, R, n_local=self.n_local))
        L.moe_ep_experts(self.cfg, self.world, self.rank, x, st.recv_rows, self.w_gate, self.w_up, self.w_down,
                         self.ws_gate, self.ws_up, self.ws_down, st.return_rows, st.y_shared, st.y_shared_scale, ws,
                         local_of=self.local_of, n_local=self.n_local)

    def combine(self, st: EPStep, out_dtype=torch.float32) -> torch.Tensor:
        y = self._empty((st.T, self.shape.H), out_dtype)
        self.lib.moe_ep_combine(self.cfg, self.world, st.back_rows, st.send_row_of, st.y_shared, st.y_shared_scale, y)
        return y

    # ---- live load statistics and re-placement of the copies ----
    def count_load(self, st: EPStep, load: Optional[torch.Tensor] = None) -> torch.Tensor:
        """Rows this step's tokens routed to each expert (int32 [E] on the device), added
        into `load` when given.  The count is libmoe's balancing step with gamma = 0,
        which leaves the bias unchanged."""
        cnt = self._empty(self.shape.E, torch.int32)
        if st.T:
            self.lib.moe_bias_update(self.cfg, st.idx, self.e_bias, 0.0, cnt)
        else:
            cnt.zero_()
        return cnt if load is None else load.add_(cnt)

    def replan(self, load, n_redundant: int, max_rep: Optional[int] = None) -> EPPlacement:
        """Re-place the copies from a global per-expert load [E] that every rank passes
        unchanged (e.g. count_load over recent steps, summed over the ranks): the new
        placement from moe_ep_place, each copy's weights sent by the rank whose block
        holds the expert (one all-to-all per weight tensor), and the layer switched to
        it.  Every rank of the group calls it with the same arguments."""
        import torch.distributed as dist
        E, W, r = self.shape.E, self.world, self.rank
        El = E // W
        new = EPPlacement.from_load(E, W, torch.as_tensor(load).cpu(), n_redundant, max_rep or W)
        held = [new.local_experts(d)[2] for d in range(W)]
        cur = {e: i for i, e in enumerate(self.local_ids)}
        send_ids = [[e for e in held[d] if e // El == r] if d != r else [] for d in range(W)]
        recv_ids = [[e for e in held[r] if e // El == s] if s != r else [] for s in range(W)]
        stacks = []
        for t in (self.w_gate, self.w_up, self.w_down):
            per = t[0].numel() * t.element_size()
            rows = lambda ids: t[torch.as_tensor([cur[e] for e in ids], device=t.device, dtype=torch.long)]  # noqa: E731
            flat = [e for ids in send_ids for e in ids]
            send = rows(flat).reshape(len(flat), -1).view(torch.uint8) if flat else \
                self._empty((0, per), torch.uint8)
            n_recv = sum(len(ids) for ids in recv_ids)
            recv = self._empty((n_recv, per), torch.uint8)
            dist.all_to_all_single(recv, send.contiguous(), [len(i) for i in recv_ids], [len(i) for i in send_ids],
                                   group=self.group)
            got = recv.view(t.dtype).view((n_recv,) + tuple(t.shape[1:]))
            from_peer = {e: got[i] for i, e in enumerate(e for ids in recv_ids for e in ids)}
            stacks.append(torch.stack([t[cur[e]] if e // El == r else from_peer[e] for e in held[r]]).contiguous())
        self.w_gate, self.w_up, self.w_down = stacks
        self.placement = new
        local_of, self.n_local, self.local_ids = new.local_experts(r)
        self.expert_ranks = new.expert_ranks.to(self.device)
        self.local_of = local_of.to(self.device)
        return new

    # ---- the forward with the process group's all-to-all ----
    def forward(self, x: torch.Tensor, out_dtype=torch.float32) -> torch.Tensor:
        """y [T, H] = layer(x [T, H] bf16) for this rank's tokens; every rank of the
        group must call it (each with its own batch) in the same order."""
        import torch.distributed as dist
        g = self.group
        st = self.send(x)
        recv_counts = torch.empty_like(st.send_counts)
        dist.all_to_all_single(recv_counts, st.send_counts, group=g)  # one count to each rank
        self.plan(st, recv_counts)
        n_send = sum(st.send_splits)
        dist.all_to_all_single(st.recv_rows, st.send_rows[:n_send], st.recv_splits, st.send_splits, group=g)
        self.experts(st, x)
        dist.all_to_all_single(st.back_rows, st.return_rows, st.send_splits, st.recv_splits, group=g)
        return self.combine(st, out_dtype)

    __call__ = forward


def expert_block(t: torch.Tensor, world: int, rank: int) -> torch.Tensor:
    """Rank `rank`'s contiguous block of a per-expert tensor [E, ...]."""
    El = t.shape[0] // world
    return t[rank * El:(rank + 1) * El].contiguous()
