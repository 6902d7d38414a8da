"""Backward pass on B200 against the float64 backward oracle (oracle/backward.py,
pinned by finite differences).  Every gradient — dx, the router weight, each
expert's gate / up / down weights and the shared expert's — is compared with
the oracle on the same bits, with the expert selection the GPU's router made
(the backward holds it fixed).  Full-size shapes: sampled token rows of dx and
the weight gradients of a sampled expert."""
import numpy as np
import pytest
import torch

import oracle
from oracle import backward as B
from sparse_moe_layer_noaux_b200 import MoELayer, abi
from sparse_moe_layer_noaux_b200.workloads import MID, TINY, V3_PREFILL, V3_SKEWED, MoEShape, bf16_bits, make_inputs
from tests import parity

pytestmark = pytest.mark.gpu

# Tolerance (derived beside parity.assert_gradient_close): max |err| <= 2e-2 *
# max |ref| per tensor and relative L1 <= 1e-2.


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from sparse_moe_layer_noaux_b200 import build
    build.build()
    oracle.build()
    yield
    torch.cuda.empty_cache()


def close(got, ref, what):
    e = parity.assert_gradient_close(got, ref, what)
    print(what, e)
    return e


def gpu_backward(shape, inp, seed=0):
    g = torch.Generator(device="cuda").manual_seed(1000 + seed)
    dy = torch.randn((shape.T, shape.H), device="cuda", generator=g).bfloat16()
    layer = MoELayer.from_inputs(shape, inp)
    grads = layer.backward(inp["x"], dy)
    cfg = abi.MoEConfig.from_shape(shape)
    ws = torch.empty(max(abi.workspace_size(cfg, shape.T), 256), dtype=torch.uint8, device="cuda")
    idx = torch.empty((shape.T, shape.k), dtype=torch.int32, device="cuda")
    w = torch.empty((shape.T, shape.k), dtype=torch.float32, device="cuda")
    abi.moe_route(cfg, inp["x"], inp["router_w"], inp["e_bias"], idx, w, ws)
    torch.cuda.synchronize()
    assert abi.device_status() == 0
    return grads, dy, idx.cpu().numpy()


SMALL = [
    TINY,
    MoEShape("ragged", T=300, hidden_size=512, n_routed_experts=32, n_group=4, topk_group=2,
             num_experts_per_tok=4, moe_intermediate_size=256, n_shared_experts=1,
             routed_scaling_factor=2.5, norm_topk_prob=True, seed=7),
    MoEShape("tiles", T=2200, hidden_size=512, n_routed_experts=8, n_group=2, topk_group=1,
             num_experts_per_tok=4, moe_intermediate_size=384, n_shared_experts=2,
             routed_scaling_factor=1.3, norm_topk_prob=False, seed=8),
    MoEShape("noshared", T=500, hidden_size=256, n_routed_experts=16, n_group=1, topk_group=1,
             num_experts_per_tok=3, moe_intermediate_size=128, n_shared_experts=0,
             routed_scaling_factor=1.0, norm_topk_prob=True, seed=9),
]


@pytest.mark.parametrize("shape", SMALL, ids=lambda s: s.name)
def test_backward_small_every_gradient(shape):
    inp = make_inputs(shape, "cuda")
    grads, dy, idx = gpu_backward(shape, inp)
    fetch = parity.device_expert_fetch(inp)
    shared = parity.shared_bits(inp, shape)
    ref = B.moe_layer_backward(shape, bf16_bits(inp["x"]), inp["router_w"].cpu().numpy(),
                               inp["e_bias"].cpu().numpy(), fetch, shared, bf16_bits(dy), routing=idx)
    print(parity.compare_gradients(shape, grads, ref, shape.name))


def test_backward_deterministic():
    shape = SMALL[1]
    inp = make_inputs(shape, "cuda")
    g1, *_ = gpu_backward(shape, inp)
    g2, *_ = gpu_backward(shape, inp)
    for k in g1:
        assert torch.equal(g1[k], g2[k]), k


@pytest.mark.parametrize("shape,n_rows", [(MID, 64), (V3_PREFILL, 64), (V3_SKEWED, 64)],
                         ids=lambda v: getattr(v, "name", str(v)))
def test_backward_full_size_sampled(shape, n_rows):
    """dx of sampled rows, and the weight gradients of two experts (all of their
    rows: a sampled one and the least loaded one) against the oracle's expert
    backward on the same operands."""
    inp = make_inputs(shape, "cuda")
    grads, dy, idx = gpu_backward(shape, inp)
    rng = np.random.default_rng(shape.seed)
    rows = np.sort(rng.choice(shape.T, n_rows, replace=False))
    x_rows = bf16_bits(inp["x"][torch.as_tensor(rows, device="cuda")])
    ref = B.moe_layer_backward(shape, x_rows, inp["router_w"].cpu().numpy(), inp["e_bias"].cpu().numpy(),
                               parity.device_expert_fetch(inp), parity.shared_bits(inp, shape),
                               bf16_bits(dy[torch.as_tensor(rows, device="cuda")]), routing=idx[rows])
    close(grads["x"].cpu().numpy()[rows], ref.dx, f"{shape.name} dx rows")
    # One expert's weight gradients over all of its rows (for the skewed workload, where
    # a few experts take most rows and many take none: the one closest to 1024 rows).
    used, n_used = np.unique(idx, return_counts=True)
    e1 = int(used[np.argmin(np.abs(n_used - 1024))]) if shape.name == "v3_skewed" else int(rng.choice(used))
    e2 = int(used[np.argmin(n_used)])
    if shape.name == "v3_skewed":
        unused = sorted(set(range(shape.E)) - set(used.tolist()))
        assert unused and all(not grads["w_down"][u].float().abs().sum().item() for u in unused[:8])
    for e in dict.fromkeys((e1, e2)):
        check_expert_weight_grads(shape, inp, grads, dy, idx, e)


def check_expert_weight_grads(shape, inp, grads, dy, idx, e):
    toks, slots = np.nonzero(idx == e)
    xt = oracle.widen_bf16(bf16_bits(inp["x"]))[toks]
    rw = inp["router_w"].cpu().numpy().astype(np.float64)
    s = 1.0 / (1.0 + np.exp(-(xt @ rw.T)))
    s_sel = np.take_along_axis(s, idx[toks].astype(np.int64), axis=1)
    w = s_sel / s_sel.sum(1, keepdims=True) if shape.norm_topk_prob else s_sel
    w = shape.routed_scaling_factor * w[np.arange(len(toks)), slots]
    do = w[:, None] * oracle.widen_bf16(bf16_bits(dy))[toks]
    wg, wu, wd = (oracle.widen_bf16(a) for a in parity.device_expert_fetch(inp)(e))
    _, dwg, dwu, dwd, _ = B._swiglu_backward(xt, wg, wu, wd, do)
    close(grads["w_gate"][e].float().cpu().numpy(), dwg, f"{shape.name} d_w_gate[{e}]")
    close(grads["w_up"][e].float().cpu().numpy(), dwu, f"{shape.name} d_w_up[{e}]")
    close(grads["w_down"][e].float().cpu().numpy(), dwd, f"{shape.name} d_w_down[{e}] ({len(toks)} rows)")


def test_backward_empty_batch_gives_zero_weight_gradients():
    shape = TINY.with_(T=0)
    inp = make_inputs(shape, "cuda")
    dy = torch.empty((0, shape.H), dtype=torch.bfloat16, device="cuda")
    layer = MoELayer.from_inputs(shape, inp)
    grads = layer.backward(inp["x"], dy)
    torch.cuda.synchronize()
    for k in ("router_w", "w_gate", "w_up", "w_down", "ws_gate", "ws_up", "ws_down"):
        assert not grads[k].float().abs().sum().item(), k


def test_backward_replays_from_a_cuda_graph():
    shape = SMALL[1]
    inp = make_inputs(shape, "cuda")
    g = torch.Generator(device="cuda").manual_seed(7)
    dy = torch.randn((shape.T, shape.H), device="cuda", generator=g).bfloat16()
    layer = MoELayer.from_inputs(shape, inp)
    eager = {k: v.clone() for k, v in layer.backward(inp["x"], dy).items()}
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        out = layer.backward(inp["x"], dy)  # allocates the outputs and workspace before capture
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    for v in out.values():
        v.zero_()
    cfg = layer.cfg
    with torch.cuda.graph(graph):
        abi.moe_backward(cfg, inp["x"], layer.router_w, layer.e_bias, layer.w_gate, layer.w_up, layer.w_down,
                         layer.ws_gate, layer.ws_up, layer.ws_down, dy, out["x"], out["router_w"], out["w_gate"],
                         out["w_up"], out["w_down"], out["ws_gate"], out["ws_up"], out["ws_down"], layer._ws_bwd)
    graph.replay()
    torch.cuda.synchronize()
    assert abi.device_status() == 0
    for k in eager:
        assert torch.equal(out[k], eager[k]), k
    del graph


@pytest.mark.parametrize("shape", [SMALL[0], SMALL[1], SMALL[2], SMALL[3]], ids=lambda s: s.name)
def test_training_pair(shape):
    """moe_forward_train gives moe_forward's output — bit for bit when every expert
    segment has more than 112 rows (moe_forward computes smaller segments transposed),
    else to within fp16 rounding of the expert outputs — and the oracle's at the
    forward's tolerances; moe_backward_train, from its context, gives exactly
    moe_backward's gradients."""
    inp = make_inputs(shape, "cuda")
    layer = MoELayer.from_inputs(shape, inp)
    g = torch.Generator(device="cuda").manual_seed(1000)
    dy = torch.randn((shape.T, shape.H), device="cuda", generator=g).bfloat16()
    y = layer.forward_train(inp["x"])
    y_fwd = layer(inp["x"])
    grads_t = layer.backward_train(inp["x"], dy)
    grads = layer.backward(inp["x"], dy)
    torch.cuda.synchronize()
    assert abi.device_status() == 0
    for k in grads:
        assert torch.equal(grads_t[k], grads[k]), k
    x_bits = bf16_bits(inp["x"])
    rw, bias = inp["router_w"].cpu().numpy(), inp["e_bias"].cpu().numpy()
    ref_idx, ref_w, margin, scores = parity.oracle_route_all(shape, x_bits, rw, bias)
    cfg = abi.MoEConfig.from_shape(shape)
    ws = torch.empty(max(abi.workspace_size(cfg, shape.T), 256), dtype=torch.uint8, device="cuda")
    idx = torch.empty((shape.T, shape.k), dtype=torch.int32, device="cuda")
    w = torch.empty((shape.T, shape.k), dtype=torch.float32, device="cuda")
    abi.moe_route(cfg, inp["x"], inp["router_w"], inp["e_bias"], idx, w, ws)
    counts = np.bincount(idx.cpu().numpy().reshape(-1), minlength=shape.E)
    if counts[counts > 0].min() > 112:
        assert torch.equal(y, y_fwd)
    else:
        assert float((y - y_fwd).abs().max()) <= 2.0 ** -9 * float(y_fwd.abs().max())
    y_ref = parity.oracle_layer_rows(shape, inp, np.arange(shape.T), idx.cpu().numpy(), scores, ref_idx, ref_w,
                                     margin)
    parity.assert_output_close(y.cpu().numpy(), y_ref, f"{shape.name} forward_train")
