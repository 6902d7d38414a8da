"""B200-native DeepSeekMoE layer forward (noaux_tc routing) behind a C ABI.

The compute path is libmoe.so (hand-written CUDA for sm_100a; see
include/moe.h).  This package only marshals arguments: `abi` mirrors the C
entry points one to one, and `MoELayer` is the user-facing call that owns the
weights and a reusable workspace.  PyTorch supplies device memory and streams.
"""
from __future__ import annotations

from typing import Optional

import torch

from . import abi
from .abi import (MoEConfig, MoEError, moe_combine, moe_dispatch, moe_experts, moe_forward,
                  moe_route, workspace_size)
from .workloads import MoEShape

__all__ = ["MoELayer", "MoELayerMX", "MoEConfig", "MoEError", "MoEShape", "abi", "moe_route", "moe_dispatch",
           "moe_experts", "moe_combine", "moe_forward", "workspace_size"]


class MoELayer:
    """One DeepSeekMoE feed-forward layer with caller-provided weights.

    Weights (device tensors, nn.Linear (out, in) layout):
      router_w fp32 [E,H], e_bias fp32 [E], w_gate/w_up bf16 [E,I,H],
      w_down bf16 [E,H,I], ws_gate/ws_up bf16 [S*I,H], ws_down bf16 [H,S*I].
    """

    def __init__(self, shape: MoEShape, router_w, e_bias, w_gate, w_up, w_down,
                 ws_gate=None, ws_up=None, ws_down=None):
        self.shape = shape
        self.cfg = MoEConfig.from_shape(shape)
        self.router_w, self.e_bias = router_w, e_bias
        self.w_gate, self.w_up, self.w_down = w_gate, w_up, w_down
        self.ws_gate, self.ws_up, self.ws_down = ws_gate, ws_up, ws_down
        self._ws: Optional[torch.Tensor] = None

    @classmethod
    def from_inputs(cls, shape: MoEShape, inputs: dict) -> "MoELayer":
        return cls(shape, inputs["router_w"], inputs["e_bias"], inputs["w_gate"], inputs["w_up"],
                   inputs["w_down"], inputs.get("ws_gate"), inputs.get("ws_up"), inputs.get("ws_down"))

    def workspace(self, T: int) -> torch.Tensor:
        need = workspace_size(self.cfg, T)
        if self._ws is None or self._ws.numel() < need:
            self._ws = torch.empty(max(need, 256), dtype=torch.uint8, device=self.w_gate.device)
        return self._ws

    def forward(self, x: torch.Tensor, y: Optional[torch.Tensor] = None,
                topk_idx: Optional[torch.Tensor] = None, topk_w: Optional[torch.Tensor] = None,
                stream=None, out_dtype: torch.dtype = torch.float32) -> torch.Tensor:
        """y [T,H] = layer(x [T,H] bf16).  y is fp32 (the unrounded fp32 sum) unless a
        bf16 `y` or out_dtype is given; topk_idx / topk_w optionally receive the routing."""
        T = x.shape[0]
        if y is None:
            y = torch.empty(x.shape, dtype=out_dtype, device=x.device)
        moe_forward(self.cfg, x, self.router_w, self.e_bias, self.w_gate, self.w_up, self.w_down,
                    self.ws_gate, self.ws_up, self.ws_down, y, topk_idx, topk_w,
                    self.workspace(T), stream)
        return y

    __call__ = forward

    def forward_host(self, x_host: torch.Tensor, y_host: Optional[torch.Tensor] = None, chunk_tokens: int = 0,
                     stream=None, out_dtype: torch.dtype = torch.float32) -> torch.Tensor:
        """y_host = layer(x_host) for host tensors (pinned for overlap): the batch goes
        through in chunks of chunk_tokens rows (0: one chunk) with the copies to and
        from the GPU overlapping the layer.  Returns once the work is enqueued on
        `stream`; synchronise it before reading y_host."""
        T = x_host.shape[0]
        if y_host is None:
            y_host = torch.empty(x_host.shape, dtype=out_dtype, pin_memory=True)
        need = abi.workspace_size_host(self.cfg, T, chunk_tokens, abi.out_dtype_code(y_host))
        if getattr(self, "_ws_host", None) is None or self._ws_host.numel() < need:
            self._ws_host = torch.empty(max(need, 256), dtype=torch.uint8, device=self.w_gate.device)
        abi.moe_forward_host(self.cfg, x_host, self.router_w, self.e_bias, self.w_gate, self.w_up, self.w_down,
                             self.ws_gate, self.ws_up, self.ws_down, y_host, chunk_tokens, self._ws_host, stream)
        return y_host

    def _grads_like(self, x):
        dev = x.device
        g = {"x": torch.empty(x.shape, dtype=torch.float32, device=dev),
             "router_w": torch.empty_like(self.router_w, dtype=torch.float32),
             "w_gate": torch.empty_like(self.w_gate), "w_up": torch.empty_like(self.w_up),
             "w_down": torch.empty_like(self.w_down)}
        if self.shape.n_shared_experts > 0:
            g.update(ws_gate=torch.empty_like(self.ws_gate), ws_up=torch.empty_like(self.ws_up),
                     ws_down=torch.empty_like(self.ws_down))
        return g

    def forward_train(self, x: torch.Tensor, y: Optional[torch.Tensor] = None, stream=None,
                      out_dtype: torch.dtype = torch.float32) -> torch.Tensor:
        """The forward, keeping routing, rows and g / u for backward_train (on this layer)."""
        T = x.shape[0]
        if y is None:
            y = torch.empty(x.shape, dtype=out_dtype, device=x.device)
        need = abi.workspace_size_bwd(self.cfg, T)
        if getattr(self, "_ctx", None) is None or self._ctx.numel() < need:
            self._ctx = torch.empty(max(need, 256), dtype=torch.uint8, device=x.device)
        abi.moe_forward_train(self.cfg, x, self.router_w, self.e_bias, self.w_gate, self.w_up, self.w_down,
                              self.ws_gate, self.ws_up, self.ws_down, y, self._ctx, stream)
        return y

    def backward_train(self, x: torch.Tensor, dy: torch.Tensor, grads: Optional[dict] = None, stream=None) -> dict:
        """Gradients as backward(), from the context of the last forward_train(x)."""
        g = grads if grads is not None else self._grads_like(x)
        abi.moe_backward_train(self.cfg, x, self.router_w, self.w_gate, self.w_up, self.w_down, self.ws_gate,
                               self.ws_up, self.ws_down, dy, g["x"], g["router_w"], g["w_gate"], g["w_up"],
                               g["w_down"], g.get("ws_gate"), g.get("ws_up"), g.get("ws_down"), self._ctx, stream)
        return g

    def backward(self, x: torch.Tensor, dy: torch.Tensor, stream=None) -> dict:
        """Gradients of sum(layer(x) * dy) (dy bf16 [T,H]), expert selection held fixed:
        dx fp32, router_w fp32, expert / shared weights bf16 (same shapes as the weights)."""
        T = x.shape[0]
        dev = x.device
        g = {"x": torch.empty(x.shape, dtype=torch.float32, device=dev),
             "router_w": torch.empty_like(self.router_w, dtype=torch.float32),
             "w_gate": torch.empty_like(self.w_gate), "w_up": torch.empty_like(self.w_up),
             "w_down": torch.empty_like(self.w_down)}
        if self.shape.n_shared_experts > 0:
            g.update(ws_gate=torch.empty_like(self.ws_gate), ws_up=torch.empty_like(self.ws_up),
                     ws_down=torch.empty_like(self.ws_down))
        need = abi.workspace_size_bwd(self.cfg, T)
        if getattr(self, "_ws_bwd", None) is None or self._ws_bwd.numel() < need:
            self._ws_bwd = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
        abi.moe_backward(self.cfg, x, self.router_w, self.e_bias, self.w_gate, self.w_up, self.w_down,
                         self.ws_gate, self.ws_up, self.ws_down, dy, g["x"], g["router_w"], g["w_gate"],
                         g["w_up"], g["w_down"], g.get("ws_gate"), g.get("ws_up"), g.get("ws_down"),
                         self._ws_bwd, stream)
        return g


class MoELayerMX:
    """The layer with MXFP8 expert FFNs (E4M3 with power-of-two scales per 32
    elements, include/moe.h).  The bf16 weights are quantised once, here, through
    the library (moe_mx_quantize); the router keeps its fp32 weights."""

    def __init__(self, shape: MoEShape, router_w, e_bias, w_gate, w_up, w_down,
                 ws_gate=None, ws_up=None, ws_down=None, stream=None):
        self.shape = shape
        self.cfg = MoEConfig.from_shape(shape)
        self.router_w, self.e_bias = router_w, e_bias
        q = lambda w: None if w is None else abi.mx_quantize(w.reshape(-1, w.shape[-1]), stream)
        self.gate, self.up, self.down = q(w_gate), q(w_up), q(w_down)
        self.shared = tuple(q(w) for w in (ws_gate, ws_up, ws_down)) if shape.n_shared_experts > 0 \
            else (None, None, None)
        self.weights = abi.mx_weights(self.gate, self.up, self.down, *self.shared)
        self._ws: Optional[torch.Tensor] = None

    @classmethod
    def from_inputs(cls, shape: MoEShape, inputs: dict) -> "MoELayerMX":
        return cls(shape, inputs["router_w"], inputs["e_bias"], inputs["w_gate"], inputs["w_up"],
                   inputs["w_down"], inputs.get("ws_gate"), inputs.get("ws_up"), inputs.get("ws_down"))

    def workspace(self, T: int) -> torch.Tensor:
        need = abi.workspace_size_mx(self.cfg, T)
        if self._ws is None or self._ws.numel() < need:
            self._ws = torch.empty(max(need, 256), dtype=torch.uint8, device=self.router_w.device)
        return self._ws

    def forward(self, x: torch.Tensor, y: Optional[torch.Tensor] = None,
                topk_idx: Optional[torch.Tensor] = None, topk_w: Optional[torch.Tensor] = None,
                stream=None, out_dtype: torch.dtype = torch.float32) -> torch.Tensor:
        T = x.shape[0]
        if y is None:
            y = torch.empty(x.shape, dtype=out_dtype, device=x.device)
        abi.moe_forward_mx(self.cfg, x, self.router_w, self.e_bias, self.weights, y, topk_idx, topk_w,
                           self.workspace(T), stream)
        return y

    __call__ = forward
