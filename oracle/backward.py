"""Float64 backward of the DeepSeekMoE layer — TEST INFRASTRUCTURE ONLY.

Gradients of L = sum(y * dy) for an upstream gradient dy, with respect to the
token rows x, the router weight and every expert weight, written out by the
chain rule from the forward's definition (the layer of ``oracle.moe_layer``:
"The Evolving Transformer · 07 — DeepSeek V2 & V3", § 02 DeepSeekMoE and § 03
Shared Expert; routing as in the "DeepSeekV3.2-Tiered-Implementations" README,
§ Architecture).  The checking method follows the "dsv3-native-reference"
page, § NumPy Oracle: float64 finite differences of the forward, full on micro
shapes and sampled on larger ones (tests/test_oracle_backward.py).

Readings where the pages say nothing:
  * the expert selection (group keep, top-k) is piecewise constant in the
    inputs: gradients flow through the routing weights w only, with the chosen
    experts held fixed; the correction bias gets no gradient (it only steers
    the selection and is updated by the load rule instead);
  * w_j = c s_j / sum(s_sel) when norm_topk_prob, else c s_j (c the routed
    scaling factor), s = sigmoid(logits).

Everything here is float64 numpy; nothing is shared with the CUDA path.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Callable, Dict, Optional, Tuple

import numpy as np

from . import route, widen_bf16


def _sigmoid(z):
    return 1.0 / (1.0 + np.exp(-z))


def _f64(a):
    a = np.asarray(a)
    return widen_bf16(a) if a.dtype == np.uint16 else np.asarray(a, np.float64)


@dataclass
class Grads:
    dx: np.ndarray                                   # [n, H]
    d_router_w: np.ndarray                           # [E, H]
    d_experts: Dict[int, Tuple[np.ndarray, np.ndarray, np.ndarray]]   # e -> (dWg [I,H], dWu [I,H], dWd [H,I])
    d_shared: Optional[Tuple[np.ndarray, np.ndarray, np.ndarray]]     # (dWsg, dWsu, dWsd)
    d_topk_w: np.ndarray                             # [n, k] gradient w.r.t. the routing weights


def swiglu_f64(x, wg, wu, wd):
    """down(silu(gate x) * up x), float64, weights in (out, in) layout."""
    g, u = x @ wg.T, x @ wu.T
    return (g * _sigmoid(g) * u) @ wd.T


def _swiglu_backward(x, wg, wu, wd, do):
    """Gradients of sum(do * down(silu(gate x) * up x)) w.r.t. x, Wg, Wu, Wd,
    and the forward output o (for the routing-weight gradient)."""
    g, u = x @ wg.T, x @ wu.T
    sg = _sigmoid(g)
    a = g * sg                      # silu(g)
    h = a * u
    o = h @ wd.T
    dh = do @ wd                    # [n, I]
    d_wd = do.T @ h                 # [H, I]
    dg = dh * u * (sg * (1.0 + g * (1.0 - sg)))   # silu'(g) = s (1 + g (1 - s))
    du = dh * a
    d_wg = dg.T @ x
    d_wu = du.T @ x
    dx = dg @ wg + du @ wu
    return dx, d_wg, d_wu, d_wd, o


def moe_forward_f64(shape, x, router_w, e_bias, experts, shared, routing=None):
    """The layer's forward with float64 inputs (for finite differences).
    experts: e -> (Wg, Wu, Wd) float64; shared: (Wsg, Wsu, Wsd) or None.
    routing (idx, held fixed) optional: then only the weights are recomputed."""
    x = np.asarray(x, np.float64)
    n, H = x.shape
    k = shape.num_experts_per_tok
    s = _sigmoid(x @ np.asarray(router_w, np.float64).T)           # [n, E]
    if routing is None:
        raise ValueError("pass the expert selection (it is held fixed)")
    idx = np.asarray(routing, np.int64)
    s_sel = np.take_along_axis(s, idx, axis=1)
    w = s_sel / s_sel.sum(axis=1, keepdims=True) if shape.norm_topk_prob else s_sel
    w = w * shape.routed_scaling_factor
    y = np.zeros((n, H))
    if shared is not None and shape.n_shared_experts > 0:
        y += swiglu_f64(x, *shared)
    for e in np.unique(idx):
        rows, slots = np.nonzero(idx == e)
        y[rows] += w[rows, slots][:, None] * swiglu_f64(x[rows], *experts(int(e)))
    return y


def moe_layer_backward(shape, x_bits, router_w, e_bias, expert: Callable, shared, dy,
                       routing=None) -> Grads:
    """Gradients of sum(y * dy) for the rows of x (bf16 bits or float64).

    ``expert(e)`` returns (Wg, Wu, Wd) as bf16 bits or float64; ``shared`` the
    concatenated shared expert or None; ``routing`` optionally the expert
    selection idx [n, k] to hold fixed (default: the oracle router's)."""
    x = _f64(x_bits)
    dy = _f64(dy)
    n, H = x.shape
    E, k = shape.n_routed_experts, shape.num_experts_per_tok
    rw = np.asarray(router_w, np.float64)
    if routing is None:
        xb = np.asarray(x_bits)
        if xb.dtype != np.uint16:
            raise ValueError("float64 rows need an explicit routing")
        idx, _, _ = route(shape, xb, router_w, e_bias)
    else:
        idx = np.asarray(routing, np.int64)
    s = _sigmoid(x @ rw.T)
    s_sel = np.take_along_axis(s, idx, axis=1)
    c = shape.routed_scaling_factor
    S = s_sel.sum(axis=1, keepdims=True)
    w = c * s_sel / S if shape.norm_topk_prob else c * s_sel

    dx = np.zeros((n, H))
    d_shared = None
    if shared is not None and shape.n_shared_experts > 0:
        wsg, wsu, wsd = (_f64(a) for a in shared)
        ddx, dg, du, dd, _ = _swiglu_backward(x, wsg, wsu, wsd, dy)
        dx += ddx
        d_shared = (dg, du, dd)

    d_experts = {}
    dw = np.zeros((n, k))
    for e in np.unique(idx):
        rows, slots = np.nonzero(idx == e)
        wg, wu, wd = (_f64(a) for a in expert(int(e)))
        do = w[rows, slots][:, None] * dy[rows]
        ddx, dg, du, dd, o = _swiglu_backward(x[rows], wg, wu, wd, do)
        np.add.at(dx, rows, ddx)
        dw[rows, slots] = np.sum(dy[rows] * o, axis=1)   # o: the unweighted expert output
        d_experts[int(e)] = (dg, du, dd)

    # Routing weights -> selected scores -> logits -> router weight and x.
    if shape.norm_topk_prob:
        ds_sel = c / S * (dw - np.sum(dw * s_sel, axis=1, keepdims=True) / S)
    else:
        ds_sel = c * dw
    dl = np.zeros((n, E))
    np.add.at(dl, (np.repeat(np.arange(n), k), idx.reshape(-1)), (ds_sel * s_sel * (1.0 - s_sel)).reshape(-1))
    d_rw = dl.T @ x
    dx += dl @ rw
    return Grads(dx=dx, d_router_w=d_rw, d_experts=d_experts, d_shared=d_shared, d_topk_w=dw)
