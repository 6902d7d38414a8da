"""A CPU stand-in for the libmoe calls that MoELayerEP makes, built on the float64
oracle (test infrastructure: it lets the expert-parallel exchange — counts,
split sizes, segment offsets, the return of the outputs and their reassembly —
run over gloo ranks on a machine without a GPU).

Each function keeps the contract include/moe.h states for the library call of
the same name, on CPU tensors:
  moe_route           oracle routing (float64), weights stored as fp32
  moe_dispatch        stable counting sort of the (token, slot) entries by expert
  moe_ep_pack         per-expert counts, routing weight per row
  moe_ep_recv_offsets exclusive prefix sum of the received counts
  moe_ep_experts      oracle SwiGLU per segment (local expert = segment % E/world),
                      outputs in the block-scaled fp16 format with scale code 141
                      (factor 1), i.e. plain fp16 values
  moe_combine         shared row + the token's k rows, decoded, summed in fp32
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from sparse_moe_layer_noaux_b200.workloads import bf16_bits

_UNIT_CODE = 141  # block-scale code whose factor is 2^(141 - 141) = 1


def workspace_size(cfg, T):
    return 256


def y_perm_scale_cols(H):
    return (H // 32 + 7) // 8 * 8


def _shape(cfg):
    return cfg  # the MoEConfig fields are all the oracle reads


def moe_route(cfg, x, router_w, e_bias, topk_idx, topk_w, workspace=None):
    idx, w, _ = oracle.route(_shape(cfg), bf16_bits(x), router_w.numpy(), e_bias.numpy())
    topk_idx.copy_(torch.from_numpy(idx))
    topk_w.copy_(torch.from_numpy(w.astype(np.float32)))


def moe_dispatch(cfg, x, topk_idx, expert_offsets, x_perm, perm_src, row_of, workspace=None):
    k, E = cfg.num_experts_per_tok, cfg.n_routed_experts
    flat = topk_idx.numpy().reshape(-1).astype(np.int64)
    order = np.argsort(flat, kind="stable")
    counts = np.bincount(flat, minlength=E)
    expert_offsets.copy_(torch.from_numpy(np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)))
    perm_src.copy_(torch.from_numpy(order.astype(np.int32)))
    inv = np.empty_like(order)
    inv[order] = np.arange(order.size)
    row_of.copy_(torch.from_numpy(inv.reshape(row_of.shape).astype(np.int32)))
    if order.size:
        x_perm.copy_(x[torch.from_numpy(order // k)])


def moe_ep_pack(cfg, T, expert_offsets, perm_src, topk_w, expert_counts, w_perm):
    off = expert_offsets.numpy().astype(np.int64)
    expert_counts.copy_(torch.from_numpy((off[1:] - off[:-1]).astype(np.int32)))
    if perm_src.numel():
        w_perm.copy_(topk_w.reshape(-1)[perm_src.long()])


def moe_ep_recv_offsets(cfg, world, recv_counts, recv_offsets):
    c = recv_counts.numpy().reshape(-1).astype(np.int64)
    recv_offsets.copy_(torch.from_numpy(np.concatenate([[0], np.cumsum(c)]).astype(np.int32)))


def _store_unit_scale(values, scales, rows_f64):
    values.copy_(torch.from_numpy(rows_f64).to(torch.float16))
    scales.fill_(_UNIT_CODE)


def moe_ep_experts(cfg, world, T, x, x_recv, recv_offsets, w_recv, w_gate, w_up, w_down, ws_gate, ws_up, ws_down,
                   h_recv, h_shared, y_recv, y_recv_scale, y_shared, y_shared_scale):
    El = cfg.n_routed_experts // world
    off = recv_offsets.numpy().astype(np.int64)
    xb = bf16_bits(x_recv)
    out = np.zeros((x_recv.shape[0], cfg.hidden_size), np.float64)
    for s in range(cfg.n_routed_experts):
        a, b = off[s], off[s + 1]
        if b > a:
            e = s % El
            o = oracle.swiglu(xb[a:b], bf16_bits(w_gate[e]), bf16_bits(w_up[e]), bf16_bits(w_down[e]))
            out[a:b] = w_recv[a:b].numpy().astype(np.float64)[:, None] * o
    _store_unit_scale(y_recv, y_recv_scale, out)
    if cfg.n_shared_experts > 0 and T > 0:
        o = oracle.swiglu(bf16_bits(x), bf16_bits(ws_gate), bf16_bits(ws_up), bf16_bits(ws_down))
        _store_unit_scale(y_shared, y_shared_scale, o)


def moe_combine(cfg, T, y_perm, y_perm_scale, row_of, y):
    k, H = cfg.num_experts_per_tok, cfg.hidden_size
    codes = y_perm_scale[:, : H // 32].to(torch.int32)
    f = torch.ldexp(torch.ones_like(codes, dtype=torch.float32), codes - 141)
    v = (y_perm.float().view(-1, H // 32, 32) * f[:, :, None]).view(-1, H)
    acc = v[T * k:T * k + T].clone() if cfg.n_shared_experts > 0 else torch.zeros((T, H))
    for j in range(k):
        acc += v[row_of[:, j].long()]
    y.copy_(acc)
