"""Expert parallelism of the DeepSeekMoE layer over torch.distributed ranks.

The routed experts are spread over the `world` ranks of a process group, rank r
holding experts [r * E/world, (r + 1) * E/world); the router and the shared
experts are replicated, and every rank brings its own tokens ("DeepSeek-V3
notes" (knlb.dev), § infrastructure: expert parallelism with all-to-all dispatch
and combine; § architecture: a token's rows go to a limited number of nodes —
with contiguous expert blocks per rank and groups that do not straddle ranks, to
at most topk_group ranks).

Every step of the layer runs in libmoe (include/moe.h lists the sequence); this
module only allocates the buffers and moves them between ranks with the process
group's all-to-all (NCCL on GPUs): the per-expert counts, then the rows and their
routing weights, and, after the experts, their outputs back to the ranks the
rows came from.  The split sizes of an all-to-all are host integers, so the
counts are read back to the host once per forward.
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
    offsets: torch.Tensor        # [E + 1] int32
    x_perm: torch.Tensor         # [T*k, H] bf16, expert order
    perm_src: torch.Tensor       # [T*k] int32
    row_of: torch.Tensor         # [T, k] int32
    counts: torch.Tensor         # [E] int32: rows per expert (sent to the experts' ranks)
    w_perm: torch.Tensor         # [T*k] fp32: routing weight of each row
    send_splits: Optional[List[int]] = None   # rows to each rank
    recv_splits: Optional[List[int]] = None   # rows from each rank
    recv_counts: Optional[torch.Tensor] = None  # [world, E/world] int32
    recv_offsets: Optional[torch.Tensor] = None  # [E + 1] int32
    x_recv: Optional[torch.Tensor] = None       # [R, H] bf16
    w_recv: Optional[torch.Tensor] = None       # [R] fp32
    y_recv: Optional[torch.Tensor] = None       # [R, H] fp16 (block-scaled)
    y_recv_scale: Optional[torch.Tensor] = None
    y_back: Optional[torch.Tensor] = None       # [T*k + T, H] fp16: returned rows, then shared rows
    y_back_scale: Optional[torch.Tensor] = None


def _wire(t: torch.Tensor) -> torch.Tensor:
    """The tensor as a collective moves it: bf16 bits travel as fp16 (same size;
    the collective copies, it never computes on them)."""
    return t.view(torch.float16) if t.dtype == torch.bfloat16 else t


class MoELayerEP:
    """One rank's part of an expert-parallel layer.

    shape: the whole layer's configuration (E = all routed experts).
    world, rank: the ranks of `group` (default: the default process group).
    w_gate / w_up [E/world, I, H], w_down [E/world, H, I]: this rank's experts.
    router_w, e_bias and the shared experts: the full (replicated) tensors.
    """

    def __init__(self, shape: MoEShape, world: int, rank: int, router_w, e_bias, w_gate, w_up, w_down,
                 ws_gate=None, ws_up=None, ws_down=None, group=None, _kernels=None):
        if world < 1 or shape.E % world:
            raise ValueError(f"world {world} must divide n_routed_experts {shape.E}")
        self.shape, self.world, self.rank, self.group = shape, world, rank, group
        self.cfg = abi.MoEConfig.from_shape(shape)
        self.router_w, self.e_bias = router_w, e_bias
        self.w_gate, self.w_up, self.w_down = w_gate, w_up, w_down
        self.ws_gate, self.ws_up, self.ws_down = ws_gate, ws_up, ws_down
        self.device = router_w.device
        # The library binding; the CPU tests of the exchange pass a stand-in.
        self.lib = _kernels if _kernels is not None else abi
        self._ws: Optional[torch.Tensor] = None

    @property
    def experts_per_rank(self) -> int:
        return self.shape.E // self.world

    def _empty(self, shape, dtype):
        return torch.empty(shape, dtype=dtype, device=self.device)

    def _workspace(self, T: int) -> torch.Tensor:
        need = max(self.lib.workspace_size(self.cfg, T), 256)
        if self._ws is None or self._ws.numel() < need:
            self._ws = self._empty(need, torch.uint8)
        return self._ws

    # ---- phases (each a libmoe call; the collectives sit between them) ----
    def route_and_pack(self, x: torch.Tensor) -> EPStep:
        """Route the rank's tokens, sort their rows into expert order, count them."""
        s, L = self.shape, self.lib
        T, k, E, H = x.shape[0], s.k, s.E, s.H
        st = EPStep(T=T, idx=self._empty((T, k), torch.int32), w=self._empty((T, k), torch.float32),
                    offsets=self._empty(E + 1, torch.int32), x_perm=self._empty((T * k, H), torch.bfloat16),
                    perm_src=self._empty(T * k, torch.int32), row_of=self._empty((T, k), torch.int32),
                    counts=self._empty(E, torch.int32), w_perm=self._empty(T * k, torch.float32))
        ws = self._workspace(T)
        if T:
            L.moe_route(self.cfg, x, self.router_w, self.e_bias, st.idx, st.w, ws)
        L.moe_dispatch(self.cfg, x, st.idx, st.offsets, st.x_perm, st.perm_src, st.row_of, ws)
        L.moe_ep_pack(self.cfg, T, st.offsets, st.perm_src, st.w, st.counts, st.w_perm)
        return st

    def plan(self, st: EPStep, recv_counts: torch.Tensor) -> None:
        """From the counts this rank received ([world, E/world], source-major): the
        split sizes of the row exchange, the received segments' offsets, and the
        receive and return buffers."""
        s, L = self.shape, self.lib
        El = self.experts_per_rank
        st.recv_counts = recv_counts
        sent = st.counts.cpu().view(self.world, El).sum(1)
        got = recv_counts.cpu().view(self.world, El).sum(1)
        st.send_splits = [int(v) for v in sent]
        st.recv_splits = [int(v) for v in got]
        R = sum(st.recv_splits)
        st.recv_offsets = self._empty(s.E + 1, torch.int32)
        L.moe_ep_recv_offsets(self.cfg, self.world, recv_counts, st.recv_offsets)
        H = s.H
        st.x_recv = self._empty((R, H), torch.bfloat16)
        st.w_recv = self._empty(R, torch.float32)
        st.y_recv = self._empty((R, H), torch.float16)
        st.y_recv_scale = self._empty((R, L.y_perm_scale_cols(H)), torch.uint8)
        n_back = st.T * s.k + (st.T if s.S else 0)
        st.y_back = self._empty((n_back, H), torch.float16)
        st.y_back_scale = self._empty((n_back, L.y_perm_scale_cols(H)), torch.uint8)

    def experts(self, st: EPStep, x: torch.Tensor) -> None:
        """The rank's expert GEMMs over the received rows; the shared experts over its own tokens."""
        s, L = self.shape, self.lib
        R, H, I = st.x_recv.shape[0], s.H, s.I
        tk = st.T * s.k
        h_recv = self._empty((R, I), torch.bfloat16)
        shared = s.S > 0 and st.T > 0
        h_shared = self._empty((st.T, s.S * I), torch.bfloat16) if shared else None
        L.moe_ep_experts(self.cfg, self.world, st.T, x if shared else None, st.x_recv, st.recv_offsets, st.w_recv,
                         self.w_gate, self.w_up, self.w_down, self.ws_gate, self.ws_up, self.ws_down, h_recv,
                         h_shared, st.y_recv, st.y_recv_scale, st.y_back[tk:] if shared else None,
                         st.y_back_scale[tk:] if shared else None)

    def combine(self, st: EPStep, out_dtype=torch.float32) -> torch.Tensor:
        y = self._empty((st.T, self.shape.H), out_dtype)
        self.lib.moe_combine(self.cfg, st.T, st.y_back, st.y_back_scale, st.row_of, y)
        return y

    # ---- the forward with the process group's all-to-all ----
    def forward(self, x: torch.Tensor, out_dtype=torch.float32) -> torch.Tensor:
        """y [T, H] = layer(x [T, H] bf16) for this rank's tokens; every rank of the
        group must call it (each with its own batch) in the same order."""
        import torch.distributed as dist
        g = self.group
        st = self.route_and_pack(x)
        recv_counts = torch.empty_like(st.counts)
        dist.all_to_all_single(recv_counts, st.counts, group=g)  # E/world counts to each rank
        self.plan(st, recv_counts)
        tk = st.T * self.shape.k
        dist.all_to_all_single(_wire(st.x_recv), _wire(st.x_perm[:tk]), st.recv_splits, st.send_splits, group=g)
        dist.all_to_all_single(st.w_recv, st.w_perm[:tk], st.recv_splits, st.send_splits, group=g)
        self.experts(st, x)
        dist.all_to_all_single(st.y_back[:tk], st.y_recv, st.send_splits, st.recv_splits, group=g)
        dist.all_to_all_single(st.y_back_scale[:tk], st.y_recv_scale, st.send_splits, st.recv_splits, group=g)
        return self.combine(st, out_dtype)

    __call__ = forward


def expert_block(t: torch.Tensor, world: int, rank: int) -> torch.Tensor:
    """Rank `rank`'s contiguous block of a per-expert tensor [E, ...]."""
    El = t.shape[0] // world
    return t[rank * El:(rank + 1) * El].contiguous()
