"""Parity helpers shared by the GPU tests, smoke() and bench's CPU baseline.

They compare the CUDA path's results with the float64 oracle on the same bits.
Tolerances (bf16 storage, fp32 accumulation):
  max |y - y_ref| <= 2e-2 * RMS(y_ref)
  sum |y - y_ref| / sum |y_ref| <= 5e-3
Routing: expert sets must match exactly, except on tokens whose oracle margin
(the gap at the group-keep or top-k boundary) is below 1e-4; such a token is
counted, its GPU set must be optimal within that margin, and its output is
compared with the oracle recomputed on the GPU's set.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import List

import numpy as np
import torch

import oracle
from sparse_moe_layer_noaux_b200.workloads import MoEShape, bf16_bits

MAX_ABS_REL_RMS = 2e-2
MEAN_REL = 5e-3
NEAR_TIE = 1e-4


def oracle_route_all(shape: MoEShape, x_bits, rw, bias, workers: int = 0):
    """Oracle routing of every row (row blocks in spawned processes when large)."""
    from oracle.pool import route_rows
    return route_rows(shape, x_bits, rw, bias, workers)


@dataclass
class RoutingReport:
    tokens: int = 0
    near_ties: int = 0
    mismatched_near_ties: int = 0
    order_mismatches: int = 0
    mismatched_tokens: List[int] = field(default_factory=list)


def compare_routing(shape, gpu_idx, gpu_w, ref_idx, ref_w, margin, scores, bias) -> RoutingReport:
    """Sets must agree unless the oracle margin is a near tie; weights within 1e-4 relative."""
    rep = RoutingReport(tokens=len(ref_idx))
    b = scores + np.asarray(bias, np.float64)[None, :]
    gsz = shape.E // shape.n_group
    for t in range(len(ref_idx)):
        g_set, r_set = set(gpu_idx[t].tolist()), set(ref_idx[t].tolist())
        near = margin[t] < NEAR_TIE
        rep.near_ties += int(near)
        if g_set != r_set:
            if not near:
                rep.mismatched_tokens.append(t)
                continue
            rep.mismatched_near_ties += 1
            # The GPU's choice must be valid and optimal within the margin.
            assert len(g_set) == shape.k
            assert len({e // gsz for e in g_set}) <= shape.topk_group
            assert abs(sum(b[t, list(g_set)]) - sum(b[t, list(r_set)])) <= 2 * shape.k * NEAR_TIE
            continue
        if gpu_idx[t].tolist() != ref_idx[t].tolist():
            rep.order_mismatches += 1
        order = {e: j for j, e in enumerate(ref_idx[t].tolist())}
        w_ref = np.array([ref_w[t, order[e]] for e in gpu_idx[t].tolist()])
        np.testing.assert_allclose(gpu_w[t], w_ref, rtol=1e-4, atol=1e-5,
                                   err_msg=f"routing weights of token {t}")
    return rep


def weights_for_set(shape, scores_row, idx_row):
    """Routing weights (float64) of a given expert set, from the oracle's unbiased scores."""
    s = scores_row[np.asarray(idx_row)]
    w = s / s.sum() if shape.norm_topk_prob else s
    return w * shape.routed_scaling_factor


def output_errors(y, y_ref):
    y = np.asarray(y, np.float64)
    y_ref = np.asarray(y_ref, np.float64)
    rms = float(np.sqrt(np.mean(y_ref ** 2)))
    max_abs = float(np.max(np.abs(y - y_ref))) if y.size else 0.0
    rel_l1 = float(np.sum(np.abs(y - y_ref)) / max(np.sum(np.abs(y_ref)), 1e-300))
    return {"rms": rms, "max_abs": max_abs, "max_abs_over_rms": max_abs / max(rms, 1e-300),
            "rel_l1": rel_l1}


def assert_output_close(y, y_ref, what=""):
    e = output_errors(y, y_ref)
    assert e["max_abs_over_rms"] <= MAX_ABS_REL_RMS, (what, e)
    assert e["rel_l1"] <= MEAN_REL, (what, e)
    return e


# Gradients (backward pass): every element is an fp32 sum of products of three
# bf16-rounded factors (dO = w dy, g / u or h, x or the weights), each rounded
# once to bf16 (2^-9 relative), so an element can be off by ~3 * 2^-9 of its own
# size and, with few rows per expert, that does not average out.  Bar:
# max |err| <= 2e-2 * max |ref| (per tensor) and relative L1 <= 1e-2.
GRAD_MAX_ABS_REL_MAX = 2e-2
GRAD_REL_L1 = 1e-2


def assert_gradient_close(got, ref, what=""):
    e = output_errors(np.asarray(got, np.float64), ref)
    e["max_abs_over_max"] = e["max_abs"] / max(float(np.abs(ref).max()), 1e-300)
    assert e["max_abs_over_max"] <= GRAD_MAX_ABS_REL_MAX and e["rel_l1"] <= GRAD_REL_L1, (what, e)
    return e


def compare_gradients(shape, grads, ref, tag=""):
    """Every gradient of the layer (dict from MoELayer.backward) against the
    float64 backward oracle's Grads; experts no token chose must get zero."""
    out = {"dx": assert_gradient_close(grads["x"].cpu().numpy(), ref.dx, f"{tag} dx"),
           "router_w": assert_gradient_close(grads["router_w"].cpu().numpy(), ref.d_router_w,
                                             f"{tag} d_router_w")}
    for j, name in enumerate(("w_gate", "w_up", "w_down")):
        got = grads[name].float().cpu().numpy()
        want = np.zeros_like(got, dtype=np.float64)
        for e, gr in ref.d_experts.items():
            want[e] = gr[j]
        out[name] = assert_gradient_close(got, want, f"{tag} d_{name}")
        unused = sorted(set(range(shape.E)) - set(ref.d_experts))
        assert all((got[e] == 0).all() for e in unused), (tag, name, "unused experts")
    if shape.S > 0:
        for j, name in enumerate(("ws_gate", "ws_up", "ws_down")):
            out[name] = assert_gradient_close(grads[name].float().cpu().numpy(), ref.d_shared[j],
                                              f"{tag} d_{name}")
    return out


def assert_bf16_rounded(t, ref, what=""):
    """A bf16-stored intermediate: within one bf16 rounding (2^-8 relative) of the
    float64 reference, plus a small fp32-accumulation allowance."""
    t = t.double()
    ref = ref.double().to(t.device)
    rms = ref.pow(2).mean().sqrt()
    bad = (t - ref).abs() > 2.0 ** -8 * ref.abs() + 2e-3 * rms
    assert not bool(bad.any()), (what, int(bad.sum()), float((t - ref).abs().max()), float(rms))


def targeted_rows(shape, idx, n_min: int = 256, seed: int = 0, swap_max_rows: int = 112,
                  n_partial_experts: int = 16, n_small_segments: int = 4):
    """Token rows for a sampled full-size check, aimed at the tiles most likely to
    hide an indexing mistake in the expert GEMMs (rows of an expert segment are
    the expert's (token, slot) entries in ascending (t, j) order, 128 per tile):
      * two rows from the last, partial 128-row tile of each of the
        `n_partial_experts` largest segments whose length is not a multiple of 128;
      * every row of the `n_small_segments` smallest non-empty segments of at
        most `swap_max_rows` rows (those tiles run transposed);
      * 16 rows of the most loaded expert, its last rows included;
      * the first and last token, then seeded random rows up to `n_min`.
    Returns (sorted token array, dict of what was targeted)."""
    idx = np.asarray(idx)
    T, k = idx.shape
    flat = idx.reshape(-1)
    order = np.argsort(flat, kind="stable")          # slot indices, expert-major
    counts = np.bincount(flat, minlength=shape.E)
    starts = np.concatenate([[0], np.cumsum(counts)])
    tokens_of = lambda e: order[starts[e]:starts[e + 1]] // k  # noqa: E731
    rows = {0, T - 1}
    partial = [e for e in np.argsort(-counts, kind="stable") if counts[e] % 128 and counts[e] > 0]
    partial = [int(e) for e in partial[:n_partial_experts]]
    for e in partial:
        toks = tokens_of(e)
        last_tile = toks[(len(toks) - 1) // 128 * 128:]
        rows |= {int(last_tile[0]), int(last_tile[-1])}
    small = [int(e) for e in np.argsort(counts, kind="stable") if 0 < counts[e] <= swap_max_rows]
    small = small[:n_small_segments]
    for e in small:
        rows |= set(tokens_of(e).tolist())
    hot = int(counts.argmax())
    toks = tokens_of(hot)
    rows |= set(toks[:8].tolist()) | set(toks[-8:].tolist())
    rng = np.random.default_rng(seed)
    free = np.setdiff1d(np.arange(T), np.fromiter(rows, dtype=np.int64))
    extra = max(0, n_min - len(rows))
    if extra and len(free):
        rows |= set(rng.choice(free, min(extra, len(free)), replace=False).tolist())
    info = {"partial_tile_experts": partial, "small_segments": {e: int(counts[e]) for e in small},
            "hot_expert": hot, "hot_rows": int(counts[hot])}
    return np.array(sorted(rows)), info


def decode_y_perm(y_perm: torch.Tensor, y_perm_scale: torch.Tensor) -> torch.Tensor:
    """fp32 values of a block-scaled y_perm (the library's expert-output format,
    include/moe.h): fp16 * 2^(code - 141), one code per 32 columns."""
    rows, H = y_perm.shape
    codes = y_perm_scale[:, : H // 32].to(torch.int32)
    f = torch.ldexp(torch.ones_like(codes, dtype=torch.float32), codes - 141)
    return (y_perm.float().view(rows, H // 32, 32) * f[:, :, None]).view(rows, H)


def device_expert_fetch(inp):
    """Oracle expert fetcher copying one expert's bf16 bits from the device at a time."""
    def fetch(e):
        return (bf16_bits(inp["w_gate"][e]), bf16_bits(inp["w_up"][e]), bf16_bits(inp["w_down"][e]))
    return fetch


def shared_bits(inp, shape):
    if shape.n_shared_experts == 0:
        return None
    return tuple(bf16_bits(inp[n]) for n in ("ws_gate", "ws_up", "ws_down"))


def oracle_layer_rows(shape, inp, rows, gpu_idx=None, scores=None, ref_idx=None, ref_w=None,
                      margin=None, layer=None, parallel: bool = False):
    """Oracle output for the given token rows.  Where the GPU picked a different
    (near-tie) expert set, that row is computed on the GPU's set.  ``layer`` is the
    oracle layer function (default: the bf16 one; oracle.moe_layer_mx for MXFP8).
    ``parallel`` runs the per-expert calls in spawned processes (same arithmetic)."""
    x_bits = bf16_bits(inp["x"][torch.as_tensor(rows, device=inp["x"].device)])
    rw = inp["router_w"].cpu().numpy()
    bias = inp["e_bias"].cpu().numpy()
    routing = None
    if gpu_idx is not None and ref_idx is not None:
        use_idx = ref_idx[rows].copy()
        use_w = ref_w[rows].copy()
        for i, t in enumerate(rows):
            if set(gpu_idx[t].tolist()) != set(ref_idx[t].tolist()):
                assert margin[t] < NEAR_TIE
                use_idx[i] = gpu_idx[t]
                use_w[i] = weights_for_set(shape, scores[t], gpu_idx[t])
        routing = (use_idx, use_w)
    run = None
    if parallel:
        from oracle.pool import ExpertRunner
        run = ExpertRunner()
    y, *_ = (layer or oracle.moe_layer)(shape, x_bits, rw, bias, device_expert_fetch(inp),
                                        shared_bits(inp, shape), routing=routing, run_experts=run)
    return y
