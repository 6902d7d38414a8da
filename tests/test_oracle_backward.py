"""Pins of the float64 backward ("dsv3-native-reference", § NumPy Oracle: float64
finite-difference gradients, full-parameter on micro shapes, sampled on larger
ones).  The float64 forward that is differenced is itself pinned to the C oracle
on bf16 inputs; the one-expert dense case is checked against torch autograd."""
import numpy as np
import torch

import oracle
from oracle import backward as B
from sparse_moe_layer_noaux_b200.workloads import TINY, MoEShape, bf16_bits, make_inputs

MICRO = MoEShape("micro", T=3, hidden_size=32, n_routed_experts=4, n_group=2, topk_group=1,
                 num_experts_per_tok=2, moe_intermediate_size=16, n_shared_experts=1,
                 routed_scaling_factor=2.5, norm_topk_prob=True, seed=31)


def _setup(shape, weight_std=0.2):
    inp = make_inputs(shape, "cpu", weight_std=weight_std)
    xb = bf16_bits(inp["x"])
    rw, eb = inp["router_w"].numpy().astype(np.float64), inp["e_bias"].numpy()
    W = {n: oracle.widen_bf16(bf16_bits(inp[n])) for n in ("w_gate", "w_up", "w_down", "ws_gate", "ws_up", "ws_down")}
    idx, _, margin = oracle.route(shape, xb, inp["router_w"].numpy(), eb)
    dy = np.random.default_rng(shape.seed).standard_normal((shape.T, shape.H))
    return inp, xb, rw, eb, W, idx, margin, dy


def _fwd(shape, x, rw, eb, W, idx):
    shared = (W["ws_gate"], W["ws_up"], W["ws_down"]) if shape.n_shared_experts else None
    return B.moe_forward_f64(shape, x, rw, eb, lambda e: (W["w_gate"][e], W["w_up"][e], W["w_down"][e]),
                             shared, routing=idx)


def _grads(shape, xb, rw, eb, W, idx, dy):
    shared = (W["ws_gate"], W["ws_up"], W["ws_down"]) if shape.n_shared_experts else None
    return B.moe_layer_backward(shape, xb, rw, eb, lambda e: (W["w_gate"][e], W["w_up"][e], W["w_down"][e]),
                                shared, dy, routing=idx)


def test_f64_forward_matches_the_c_oracle():
    inp, xb, rw, eb, W, idx, _, _ = _setup(TINY, weight_std=0.02)
    y = _fwd(TINY, oracle.widen_bf16(xb), rw, eb, W, idx)
    fetch = oracle.in_memory_experts(*(bf16_bits(inp[n]) for n in ("w_gate", "w_up", "w_down")))
    shared = tuple(bf16_bits(inp[n]) for n in ("ws_gate", "ws_up", "ws_down"))
    y_ref, *_ = oracle.moe_layer(TINY, xb, inp["router_w"].numpy(), eb, fetch, shared)
    np.testing.assert_allclose(y, y_ref, rtol=1e-10, atol=1e-13)


def _fd_check(shape, xb, rw, eb, W, idx, dy, g, coords, eps=1e-6, tol=1e-5):
    """Central differences of L = sum(y * dy) at the given (tensor, index) coordinates."""
    x = oracle.widen_bf16(xb)
    tensors = {"x": x, "rw": rw, **W}
    analytic = {"x": g.dx, "rw": g.d_router_w,
                "ws_gate": g.d_shared[0] if g.d_shared else None, "ws_up": g.d_shared[1] if g.d_shared else None,
                "ws_down": g.d_shared[2] if g.d_shared else None}
    worst = 0.0
    for name, ix in coords:
        t = tensors[name]
        old = t[ix]
        t[ix] = old + eps
        lp = np.sum(_fwd(shape, tensors["x"], tensors["rw"], eb, W, idx) * dy)
        t[ix] = old - eps
        lm = np.sum(_fwd(shape, tensors["x"], tensors["rw"], eb, W, idx) * dy)
        t[ix] = old
        fd = (lp - lm) / (2 * eps)
        if name in ("w_gate", "w_up", "w_down"):
            e = ix[0]
            j = {"w_gate": 0, "w_up": 1, "w_down": 2}[name]
            a = g.d_experts[e][j][ix[1:]] if e in g.d_experts else 0.0
        else:
            a = analytic[name][ix]
        scale = max(abs(fd), abs(a), 1e-3)
        worst = max(worst, abs(fd - a) / scale)
    assert worst < tol, worst
    return worst


def test_full_finite_differences_on_a_micro_layer():
    shape = MICRO
    inp, xb, rw, eb, W, idx, margin, dy = _setup(shape)
    g = _grads(shape, xb, rw, eb, W, idx, dy)
    coords = []
    for name in ("x", "rw", "w_gate", "w_up", "w_down", "ws_gate", "ws_up", "ws_down"):
        shape_t = {"x": (shape.T, shape.H), "rw": rw.shape}.get(name, W.get(name, np.zeros(0)).shape)
        coords += [(name, ix) for ix in np.ndindex(*shape_t)]
    assert len(coords) > 7000
    _fd_check(shape, xb, rw, eb, W, idx, dy, g, coords)


def test_sampled_finite_differences_on_tiny():
    shape = TINY
    inp, xb, rw, eb, W, idx, margin, dy = _setup(shape, weight_std=0.05)
    g = _grads(shape, xb, rw, eb, W, idx, dy)
    rng = np.random.default_rng(5)
    coords = []
    for name, shp in (("x", (shape.T, shape.H)), ("rw", rw.shape), ("w_gate", W["w_gate"].shape),
                      ("w_up", W["w_up"].shape), ("w_down", W["w_down"].shape), ("ws_gate", W["ws_gate"].shape),
                      ("ws_down", W["ws_down"].shape)):
        for _ in range(30):
            coords.append((name, tuple(int(rng.integers(0, d)) for d in shp)))
    # routed weight entries of experts that some token actually uses
    used = np.unique(idx)
    for _ in range(60):
        e = int(rng.choice(used))
        coords.append(("w_down", (e, int(rng.integers(0, shape.H)), int(rng.integers(0, shape.I)))))
        coords.append(("w_gate", (e, int(rng.integers(0, shape.I)), int(rng.integers(0, shape.H)))))
    _fd_check(shape, xb, rw, eb, W, idx, dy, g, coords, tol=1e-5)


def test_one_expert_dense_layer_against_torch_autograd():
    # E = 1, top-1, one group, no shared expert, normalised: y = c * SwiGLU(x), the
    # routing weight is the constant c, so the router gets no gradient.
    shape = MICRO.with_(n_routed_experts=1, n_group=1, topk_group=1, num_experts_per_tok=1, n_shared_experts=0)
    inp, xb, rw, eb, W, idx, _, dy = _setup(shape)
    g = _grads(shape, xb, rw, eb, W, idx, dy)
    x = torch.tensor(oracle.widen_bf16(xb), requires_grad=True)
    wg, wu, wd = (torch.tensor(W[n][0], requires_grad=True) for n in ("w_gate", "w_up", "w_down"))
    y = shape.routed_scaling_factor * torch.nn.functional.linear(
        torch.nn.functional.silu(torch.nn.functional.linear(x, wg)) * torch.nn.functional.linear(x, wu), wd)
    (y * torch.tensor(dy)).sum().backward()
    np.testing.assert_allclose(g.dx, x.grad.numpy(), rtol=1e-10, atol=1e-12)
    for got, t in zip(g.d_experts[0], (wg, wu, wd)):
        np.testing.assert_allclose(got, t.grad.numpy(), rtol=1e-10, atol=1e-12)
    assert np.abs(g.d_router_w).max() < 1e-12
