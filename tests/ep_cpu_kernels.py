"""A CPU stand-in for the libmoe calls that MoELayerEP makes, built on the float64
oracle (test infrastructure: it lets the expert-parallel exchange — the send rows,
their counts and split sizes, the return of the sums and their reassembly — run
over gloo ranks on a machine without a GPU).

Each function keeps the contract include/moe.h states for the library call of
the same name, on CPU tensors, wire formats included:
  send row    H bf16 values, k int32 expert ids (-1 for slots bound for another
              rank), k fp32 weights, zeros to 16 bytes
  return row  H fp16 values, H/32 scale codes, zeros to 16 bytes; this stand-in
              always writes code 141 (factor 2^0), i.e. plain fp16 values
  moe_route       oracle routing (float64), weights stored as fp32
  moe_ep_send     slot (t, j) of expert e goes to e's block rank, or with a
                  placement table to replica t mod n_e of e's ranks; one row per
                  (token, destination), sorted by rank and token; send_row_of marks
                  the token's first slot bound for the rank
  moe_ep_experts  per received row, the float64 sum over its slots with an id of
                  w * SwiGLU_e(x), e's weights at its local index; the shared
                  experts over the rank's own tokens
  moe_ep_combine  shared row + the token's returned rows, decoded, summed in fp32
  moe_bias_update loads per expert (and the bias step, unused here with gamma 0)
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from sparse_moe_layer_noaux_b200.workloads import bf16_bits

_UNIT_CODE = 141  # block-scale code whose factor is 2^(141 - 141) = 1


def _pad16(n):
    return (n + 15) // 16 * 16


def ep_row_bytes(cfg):
    H, k = cfg.hidden_size, cfg.num_experts_per_tok
    return 2 * H + _pad16(8 * k), 2 * H + _pad16(H // 32)


def ep_send_rows_max(cfg, T, world):
    return T * min(cfg.num_experts_per_tok, world)


def workspace_size(cfg, T):
    return 256


def ep_workspace_size(cfg, world, T, R, n_local=None):
    return 256


def y_perm_scale_cols(H):
    return (H // 32 + 7) // 8 * 8


def moe_route(cfg, x, router_w, e_bias, topk_idx, topk_w, workspace=None):
    idx, w, _ = oracle.route(cfg, bf16_bits(x), router_w.numpy(), e_bias.numpy())
    topk_idx.copy_(torch.from_numpy(idx))
    topk_w.copy_(torch.from_numpy(w.astype(np.float32)))


def _dest(e, t, El, ranks):
    if ranks is None:
        return e // El
    reps = [int(r) for r in ranks[e] if r >= 0]
    return reps[t % len(reps)]


def moe_ep_send(cfg, world, x, topk_idx, topk_w, send_counts, send_rows, send_row_of, workspace=None,
                expert_ranks=None):
    T, H, k = x.shape[0], cfg.hidden_size, cfg.num_experts_per_tok
    El = cfg.n_routed_experts // world
    ranks = None if expert_ranks is None else expert_ranks.numpy()
    idx, w = topk_idx.numpy(), topk_w.numpy()
    dest = np.array([[_dest(int(idx[t, j]), t, El, ranks) for j in range(k)] for t in range(T)],
                    dtype=np.int64).reshape(T, k)
    entries = []                                   # (rank, token, slot), the token's first slot bound there
    for t in range(T):
        for j in range(k):
            if dest[t, j] not in dest[t, :j]:
                entries.append((int(dest[t, j]), t, j))
    entries.sort(key=lambda e: (e[0], e[1]))
    send_counts.copy_(torch.from_numpy(np.bincount([e[0] for e in entries], minlength=world).astype(np.int32)))
    row_of = np.full((T, k), -1, np.int32)
    rows = send_rows.numpy()
    xb = bf16_bits(x)
    for r, (d, t, j) in enumerate(entries):
        row_of[t, j] = r
        rows[r] = 0
        rows[r, :2 * H] = xb[t].view(np.uint8)
        ids = np.where(dest[t] == d, idx[t], -1).astype("<i4")
        rows[r, 2 * H:2 * H + 4 * k] = ids.view(np.uint8)
        rows[r, 2 * H + 4 * k:2 * H + 8 * k] = w[t].astype("<f4").view(np.uint8)
    send_row_of.copy_(torch.from_numpy(row_of))


def moe_bias_update(cfg, topk_idx, e_bias, gamma, expert_load=None):
    """The balancing step (include/moe.h): loads per expert, bias moved by gamma."""
    E, k = cfg.n_routed_experts, cfg.num_experts_per_tok
    load = np.bincount(topk_idx.numpy().reshape(-1), minlength=E).astype(np.int64)
    T = topk_idx.shape[0]
    b = e_bias.numpy()
    b[load * E > T * k] -= np.float32(gamma)
    b[load * E < T * k] += np.float32(gamma)
    if expert_load is not None:
        expert_load.copy_(torch.from_numpy(load.astype(np.int32)))


def _store_unit_scale(values, scales, rows_f64):
    values.copy_(torch.from_numpy(rows_f64).to(torch.float16))
    scales.fill_(_UNIT_CODE)


def moe_ep_experts(cfg, world, rank, x, recv_rows, w_gate, w_up, w_down, ws_gate, ws_up, ws_down, return_rows,
                   y_shared, y_shared_scale, workspace=None, local_of=None, n_local=None):
    H, k, E = cfg.hidden_size, cfg.num_experts_per_tok, cfg.n_routed_experts
    El = E // world
    local = (np.arange(E) - rank * El) if local_of is None else local_of.numpy().astype(np.int64)
    rows = recv_rows.numpy()
    R = rows.shape[0]
    xb = np.ascontiguousarray(rows[:, :2 * H]).view(np.uint16)
    ids = np.ascontiguousarray(rows[:, 2 * H:2 * H + 4 * k]).view("<i4")
    wts = np.ascontiguousarray(rows[:, 2 * H + 4 * k:2 * H + 8 * k]).view("<f4")
    out = np.zeros((R, H), np.float64)
    for e in range(E):
        r_sel, j_sel = np.nonzero(ids == e)
        if r_sel.size:
            li = int(local[e])
            assert 0 <= li < w_gate.shape[0], (rank, e, li)   # the sender only sends this rank's experts
            o = oracle.swiglu(xb[r_sel], bf16_bits(w_gate[li]), bf16_bits(w_up[li]), bf16_bits(w_down[li]))
            np.add.at(out, r_sel, wts[r_sel, j_sel].astype(np.float64)[:, None] * o)
    ret = return_rows.numpy()
    ret[:] = 0
    if R:
        ret[:, :2 * H] = out.astype(np.float16).view(np.uint8)
        ret[:, 2 * H:2 * H + H // 32] = _UNIT_CODE
    if cfg.n_shared_experts > 0 and x.shape[0] > 0:
        o = oracle.swiglu(bf16_bits(x), bf16_bits(ws_gate), bf16_bits(ws_up), bf16_bits(ws_down))
        _store_unit_scale(y_shared, y_shared_scale, o)


def _decode(values_f16, codes):
    n, H = values_f16.shape
    f = np.ldexp(1.0, codes.astype(np.int64) - 141)
    return (values_f16.astype(np.float32).reshape(n, H // 32, 32) * f[:, :, None]).reshape(n, H)


def moe_ep_combine(cfg, world, back_rows, send_row_of, y_shared, y_shared_scale, y):
    T, H, k = y.shape[0], cfg.hidden_size, cfg.num_experts_per_tok
    rows = back_rows.numpy()
    vals = _decode(np.ascontiguousarray(rows[:, :2 * H]).view(np.float16), rows[:, 2 * H:2 * H + H // 32])
    acc = np.zeros((T, H), np.float32)
    if cfg.n_shared_experts > 0 and T:
        acc += _decode(y_shared.numpy(), y_shared_scale.numpy()[:, :H // 32])
    row_of = send_row_of.numpy()
    for j in range(k):
        live = row_of[:, j] >= 0
        acc[live] += vals[row_of[live, j]]
    y.copy_(torch.from_numpy(acc))
