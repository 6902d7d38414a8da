"""Pins of the float64 oracle to facts other than itself (CPU only).

Each test ties one oracle function to something independent of its code:
hand-worked values (tests/golden), brute-force subset enumeration, a closed
form that reduces to a dense SwiGLU MLP, library routines (torch.topk,
torch float64 linear algebra) on special cases, and invariants of the method.
A plausible mistake — a dropped term, a wrong sign or index, a transposed
weight, zeroing instead of excluding dropped groups, biased instead of unbiased
weights — fails at least one of them.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from sparse_moe_layer_noaux_b200.workloads import MoEShape, TINY, MID, bf16_bits, make_inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _bits(a):
    return bf16_bits(torch.as_tensor(a, dtype=torch.float32).to(torch.bfloat16))


def _toy_shape(cfg):
    return MoEShape("toy", T=1, hidden_size=cfg["hidden_size"],
                    n_routed_experts=cfg["n_routed_experts"], n_group=cfg["n_group"],
                    topk_group=cfg["topk_group"], num_experts_per_tok=cfg["num_experts_per_tok"],
                    moe_intermediate_size=cfg["moe_intermediate_size"],
                    n_shared_experts=cfg["n_shared_experts"],
                    routed_scaling_factor=cfg["routed_scaling_factor"],
                    norm_topk_prob=cfg["norm_topk_prob"])


# --------------------------------------------------------------------------
# 1. Hand-worked golden toy (tests/golden/toy_groups.json)
# --------------------------------------------------------------------------
def test_golden_toy_layer(oracle_lib):
    g = json.load(open(os.path.join(GOLDEN, "toy_groups.json")))
    shape = _toy_shape(g["config"])
    x = _bits(g["x"])
    rw = np.array(g["router_w"], np.float32)
    E = shape.E
    wg = np.stack([_bits([[1.0, 0.0]]) for _ in range(E)])
    wu = np.stack([_bits([[1.0, 0.0]]) for _ in range(E)])
    wd = np.stack([_bits([[e + 1.0], [-(e + 1.0)]]) for e in range(E)])
    shared = (_bits(g["shared"]["ws_gate"]), _bits(g["shared"]["ws_up"]),
              _bits(g["shared"]["ws_down"]))
    for case in g["cases"]:
        bias = np.array(case["e_bias"], np.float32)
        y, idx, w, margin = oracle_lib.moe_layer(
            shape, x, rw, bias, oracle_lib.in_memory_experts(wg, wu, wd), shared)
        assert idx[0].tolist() == case["idx"], case["name"]
        np.testing.assert_allclose(w[0], case["w"], rtol=0, atol=1e-6, err_msg=case["name"])
        np.testing.assert_allclose(margin[0], case["margin"], rtol=0, atol=1e-6)
        np.testing.assert_allclose(y[0], case["y"], rtol=0, atol=1e-5, err_msg=case["name"])


# --------------------------------------------------------------------------
# 2. Brute force: enumerate every group subset and every expert subset.
# --------------------------------------------------------------------------
def _brute_force_choice(shape, b):
    """Best TG-group subset by total group score, where a group's score is the
    best pair sum inside it (enumerated over pairs), then the best k-subset of
    the surviving experts by total biased score."""
    E, G, TG, k = shape.E, shape.n_group, shape.topk_group, shape.k
    gsz = E // G
    members = [list(range(g * gsz, (g + 1) * gsz)) for g in range(G)]

    def group_score(g):
        m = members[g]
        if len(m) == 1:
            return b[m[0]]
        return max(b[i] + b[j] for i, j in itertools.combinations(m, 2))

    gsc = [group_score(g) for g in range(G)]
    best_groups = max(itertools.combinations(range(G), TG), key=lambda c: sum(gsc[g] for g in c))
    cand = [e for g in best_groups for e in members[g]]
    best_set = max(itertools.combinations(cand, k), key=lambda c: sum(b[e] for e in c))
    return set(best_set)


@pytest.mark.parametrize("E,G,TG,k,seed", [
    (16, 4, 2, 4, 0), (16, 4, 2, 4, 1), (8, 2, 1, 2, 2), (8, 4, 3, 5, 3), (12, 3, 2, 3, 4),
    (16, 1, 1, 3, 5), (16, 16, 4, 4, 6), (16, 8, 8, 6, 7)])
def test_brute_force_selection(oracle_lib, E, G, TG, k, seed):
    H, T = 32, 24
    shape = MoEShape("bf", T=T, hidden_size=H, n_routed_experts=E, n_group=G, topk_group=TG,
                     num_experts_per_tok=k, moe_intermediate_size=8, n_shared_experts=0,
                     routed_scaling_factor=1.0, norm_topk_prob=True)
    rng = np.random.default_rng(seed)
    x = _bits(rng.standard_normal((T, H)))
    rw = (rng.standard_normal((E, H)) * 0.3).astype(np.float32)
    bias = rng.uniform(-0.3, 0.3, E).astype(np.float32)
    idx, w, margin, scores = oracle_lib.route(shape, x, rw, bias, want_scores=True)
    b = scores + bias.astype(np.float64)[None, :]
    checked = 0
    for t in range(T):
        if margin[t] < 1e-9:
            continue
        assert set(idx[t].tolist()) == _brute_force_choice(shape, b[t].tolist()), t
        checked += 1
    assert checked >= T - 2


# --------------------------------------------------------------------------
# 3. Special case: one flat group, zero bias -> plain top-k of sigmoid scores.
# --------------------------------------------------------------------------
def test_flat_group_is_torch_topk(oracle_lib):
    T, H, E, k = 40, 64, 32, 6
    shape = MoEShape("flat", T=T, hidden_size=H, n_routed_experts=E, n_group=1, topk_group=1,
                     num_experts_per_tok=k, moe_intermediate_size=8, n_shared_experts=0,
                     routed_scaling_factor=1.7, norm_topk_prob=True)
    g = torch.Generator().manual_seed(11)
    xb = torch.randn(T, H, generator=g).to(torch.bfloat16)
    rw = torch.randn(E, H, generator=g) * 0.1
    idx, w, margin = oracle_lib.route(shape, bf16_bits(xb), rw.numpy(), np.zeros(E, np.float32))
    probs = torch.sigmoid(xb.double() @ rw.double().T)
    top_v, top_i = torch.topk(probs, k, dim=-1)
    for t in range(T):
        assert idx[t].tolist() == top_i[t].tolist()
    ref_w = top_v / top_v.sum(-1, keepdim=True) * 1.7
    np.testing.assert_allclose(w, ref_w.numpy(), rtol=1e-12, atol=1e-14)


def test_ties_go_to_lower_index(oracle_lib):
    # All router weights zero -> every score is sigmoid(0) = 1/2 and with zero bias
    # every biased score ties; the lower index wins every comparison, so groups
    # 0..TG-1 survive and their first k experts are chosen in index order.
    shape = TINY.with_(T=3)
    x = _bits(np.ones((3, shape.H)))
    idx, w, margin = oracle_lib.route(shape, x, np.zeros((shape.E, shape.H), np.float32),
                                      np.zeros(shape.E, np.float32))
    assert (idx == np.arange(shape.k)[None, :]).all()
    np.testing.assert_allclose(w, shape.routed_scaling_factor / shape.k)
    assert (margin == 0).all()


# --------------------------------------------------------------------------
# 4. Closed form: E=1, top_k=1, no shared expert, normalised -> scaled dense SwiGLU.
# --------------------------------------------------------------------------
def _torch_swiglu(x, wg, wu, wd):
    x, wg, wu, wd = (torch.from_numpy(a.astype(np.uint16).view(np.int16)).view(torch.bfloat16)
                     .double() for a in (x, wg, wu, wd))
    return F.linear(F.silu(F.linear(x, wg)) * F.linear(x, wu), wd).numpy()


def test_single_expert_is_scaled_dense_swiglu(oracle_lib):
    shape = MoEShape("one", T=9, hidden_size=48, n_routed_experts=1, n_group=1, topk_group=1,
                     num_experts_per_tok=1, moe_intermediate_size=20, n_shared_experts=0,
                     routed_scaling_factor=2.5, norm_topk_prob=True)
    inp = make_inputs(shape, "cpu", seed=5, weight_std=0.2)
    x = bf16_bits(inp["x"])
    wg, wu, wd = (bf16_bits(inp[n]) for n in ("w_gate", "w_up", "w_down"))
    y, idx, w, _ = oracle_lib.moe_layer(shape, x, inp["router_w"].numpy(),
                                        inp["e_bias"].numpy(),
                                        oracle_lib.in_memory_experts(wg, wu, wd), None)
    assert (idx == 0).all() and np.allclose(w, 2.5)
    ref = 2.5 * _torch_swiglu(x, wg[0], wu[0], wd[0])
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-12)


def test_swiglu_matches_torch_float64(oracle_lib):
    rng = np.random.default_rng(3)
    n, H, I = 7, 40, 24
    x = _bits(rng.standard_normal((n, H)))
    wg, wu = _bits(rng.standard_normal((I, H)) * 0.2), _bits(rng.standard_normal((I, H)) * 0.2)
    wd = _bits(rng.standard_normal((H, I)) * 0.2)
    np.testing.assert_allclose(oracle_lib.swiglu(x, wg, wu, wd), _torch_swiglu(x, wg, wu, wd),
                               rtol=1e-12, atol=1e-13)


# --------------------------------------------------------------------------
# 5. Shared-only: zero routed experts -> y is the shared SwiGLU MLP.
# --------------------------------------------------------------------------
def test_zero_routed_experts_leave_shared_mlp(oracle_lib):
    shape = TINY.with_(T=12, n_shared_experts=2)
    inp = make_inputs(shape, "cpu", seed=9)
    x = bf16_bits(inp["x"])
    zeros = np.zeros((shape.E, shape.I, shape.H), np.uint16)
    zeros_d = np.zeros((shape.E, shape.H, shape.I), np.uint16)
    shared = tuple(bf16_bits(inp[n]) for n in ("ws_gate", "ws_up", "ws_down"))
    y, *_ = oracle_lib.moe_layer(shape, x, inp["router_w"].numpy(), inp["e_bias"].numpy(),
                                 oracle_lib.in_memory_experts(zeros, zeros, zeros_d), shared)
    np.testing.assert_allclose(y, _torch_swiglu(x, *shared), rtol=1e-12, atol=1e-13)


def test_two_shared_experts_equal_their_sum(oracle_lib):
    # S shared experts stored concatenated along the intermediate axis equal the
    # sum of S separate SwiGLU experts.
    shape = TINY.with_(T=5, n_shared_experts=2)
    inp = make_inputs(shape, "cpu", seed=10)
    x = bf16_bits(inp["x"])
    sg, su, sd = (bf16_bits(inp[n]) for n in ("ws_gate", "ws_up", "ws_down"))
    I = shape.I
    whole = oracle_lib.swiglu(x, sg, su, sd)
    parts = sum(oracle_lib.swiglu(x, sg[i * I:(i + 1) * I], su[i * I:(i + 1) * I],
                                  np.ascontiguousarray(sd[:, i * I:(i + 1) * I]))
                for i in range(2))
    np.testing.assert_allclose(whole, parts, rtol=1e-12, atol=1e-13)


# --------------------------------------------------------------------------
# 6. Invariants on the workload shapes.
# --------------------------------------------------------------------------
@pytest.mark.parametrize("shape,rows", [(TINY, 64), (MID, 48)])
def test_routing_invariants(oracle_lib, shape, rows):
    inp = make_inputs(shape.with_(T=rows), "cpu")
    idx, w, margin, scores = oracle_lib.route(shape, bf16_bits(inp["x"]),
                                              inp["router_w"].numpy(), inp["e_bias"].numpy(),
                                              want_scores=True)
    gsz = shape.E // shape.n_group
    b = scores + inp["e_bias"].numpy().astype(np.float64)[None]
    for t in range(rows):
        chosen = idx[t].tolist()
        assert len(set(chosen)) == shape.k
        assert all(0 <= e < shape.E for e in chosen)
        assert len({e // gsz for e in chosen}) <= shape.topk_group
        assert all(b[t, chosen[j]] >= b[t, chosen[j + 1]] for j in range(shape.k - 1))
        assert (w[t] > 0).all()
        if shape.norm_topk_prob:
            assert math.isclose(w[t].sum(), shape.routed_scaling_factor, rel_tol=1e-12)
        else:
            np.testing.assert_allclose(w[t], scores[t, chosen] * shape.routed_scaling_factor,
                                       rtol=1e-15)
        assert margin[t] >= 0


def test_layer_rows_are_independent(oracle_lib):
    # Computing a subset of tokens gives exactly the rows of the full computation
    # (the property the sampled full-size parity checks rely on).
    shape = TINY
    inp = make_inputs(shape, "cpu")
    args = (bf16_bits(inp["x"]), inp["router_w"].numpy(), inp["e_bias"].numpy())
    fetch = oracle_lib.in_memory_experts(*(bf16_bits(inp[n]) for n in ("w_gate", "w_up",
                                                                         "w_down")))
    shared = tuple(bf16_bits(inp[n]) for n in ("ws_gate", "ws_up", "ws_down"))
    y_all, *_ = oracle_lib.moe_layer(shape, *args, fetch, shared)
    rows = np.array([3, 17, 40, 63])
    y_sub, *_ = oracle_lib.moe_layer(shape, args[0][rows], args[1], args[2], fetch, shared)
    np.testing.assert_array_equal(y_sub, y_all[rows])


def test_parallel_expert_runner_is_exact(oracle_lib):
    """The process-pool runner used for large sampled checks only moves where each
    expert's call runs: its layer output equals the serial oracle's bit for bit,
    for the bf16 and the MXFP8 layer."""
    from oracle.pool import ExpertRunner
    shape = MoEShape("pool", T=40, hidden_size=256, n_routed_experts=16, n_group=4, topk_group=2,
                     num_experts_per_tok=4, moe_intermediate_size=128, n_shared_experts=1,
                     routed_scaling_factor=2.5, norm_topk_prob=True, seed=31)
    inp = make_inputs(shape)
    x = bf16_bits(inp["x"])
    rw, bias = inp["router_w"].numpy(), inp["e_bias"].numpy()
    fetch = oracle_lib.in_memory_experts(bf16_bits(inp["w_gate"]), bf16_bits(inp["w_up"]),
                                         bf16_bits(inp["w_down"]))
    shared = tuple(bf16_bits(inp[n]) for n in ("ws_gate", "ws_up", "ws_down"))
    runner = ExpertRunner(workers=2)
    for layer in (oracle_lib.moe_layer, oracle_lib.moe_layer_mx):
        y_serial, idx, w, _ = layer(shape, x, rw, bias, fetch, shared)
        y_pool, idx2, w2, _ = layer(shape, x, rw, bias, fetch, shared, run_experts=runner)
        assert np.array_equal(idx, idx2) and np.array_equal(w, w2)
        assert np.array_equal(y_serial, y_pool), layer.__name__
