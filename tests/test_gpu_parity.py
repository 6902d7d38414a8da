"""Parity of the CUDA path (through the C ABI) with the float64 oracle on B200.

Small and ragged shapes are checked on every token; the five workload shapes
at full size are checked on every token's routing and dispatch, and on a
seeded sample of tokens for the layer output (rows are independent, so a
sample is an exact subset check).
"""
import numpy as np
import pytest
import torch

import oracle
from sparse_moe_layer_noaux_b200 import abi
from sparse_moe_layer_noaux_b200.workloads import (MID, TINY, V3_DECODE, V3_E32, V3_PREFILL, V3_SKEWED,
                                                   MoEShape, bf16_bits, make_inputs)
from tests import parity

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from sparse_moe_layer_noaux_b200 import build
    build.build()
    oracle.build()
    yield
    torch.cuda.empty_cache()


def run_forward(shape, inp, out_dtype=torch.float32):
    T, k = shape.T, shape.k
    cfg = abi.MoEConfig.from_shape(shape)
    dev = inp["x"].device
    y = torch.empty((T, shape.H), dtype=out_dtype, device=dev)
    idx = torch.empty((T, k), dtype=torch.int32, device=dev)
    w = torch.empty((T, k), dtype=torch.float32, device=dev)
    ws = torch.empty(max(abi.workspace_size(cfg, T), 256), dtype=torch.uint8, device=dev)
    abi.moe_forward(cfg, inp["x"], inp["router_w"], inp["e_bias"], inp["w_gate"], inp["w_up"],
                    inp["w_down"], inp["ws_gate"], inp["ws_up"], inp["ws_down"], y, idx, w, ws)
    torch.cuda.synchronize()
    assert abi.device_status() == 0
    return y, idx, w


def check_dispatch(shape, x, topk_idx, offsets, x_perm, perm_src, row_of):
    """Bit-exact: offsets = counts' exclusive scan; rows in stable (t, j) order."""
    T, k, E = shape.T, shape.k, shape.E
    flat = topk_idx.cpu().numpy().reshape(-1)
    counts = np.bincount(flat, minlength=E)
    np.testing.assert_array_equal(offsets.cpu().numpy(), np.concatenate([[0], np.cumsum(counts)]))
    order = np.argsort(flat, kind="stable")
    np.testing.assert_array_equal(perm_src.cpu().numpy(), order)
    inv = np.empty(T * k, np.int64)
    inv[order] = np.arange(T * k)
    np.testing.assert_array_equal(row_of.cpu().numpy().reshape(-1), inv)
    src_tok = perm_src.long() // k
    assert torch.equal(x_perm.view(torch.int16), x[src_tok].view(torch.int16))


SMALL = [
    TINY,
    TINY.with_(name="tiny_T1", T=1, seed=21),
    TINY.with_(name="tiny_T3", T=3, seed=22),
    MoEShape("ragged", T=300, hidden_size=512, n_routed_experts=32, n_group=4, topk_group=2,
             num_experts_per_tok=4, moe_intermediate_size=256, n_shared_experts=1,
             routed_scaling_factor=2.5, norm_topk_prob=True, seed=7),
    # I = 192: the gate/up column tile is cut at 64 of 128; ~550 rows per expert;
    # T >= 2048 puts the router logits on the tensor cores.
    MoEShape("tiles", T=2200, hidden_size=256, n_routed_experts=8, n_group=2, topk_group=1,
             num_experts_per_tok=2, moe_intermediate_size=192, n_shared_experts=2,
             routed_scaling_factor=1.3, norm_topk_prob=False, seed=8),
    # No shared expert, flat routing, H = 320: the down-projection tile is cut at 64 of 256.
    MoEShape("noshared", T=500, hidden_size=320, n_routed_experts=16, n_group=1, topk_group=1,
             num_experts_per_tok=3, moe_intermediate_size=128, n_shared_experts=0,
             routed_scaling_factor=1.0, norm_topk_prob=True, seed=9),
    # k = 12 at T >= 2048: tensor-core logits, a wider top-k in the warp-per-token select.
    MoEShape("k12", T=2100, hidden_size=256, n_routed_experts=64, n_group=4, topk_group=2,
             num_experts_per_tok=12, moe_intermediate_size=128, n_shared_experts=1,
             routed_scaling_factor=2.5, norm_topk_prob=True, seed=10),
    # DeepSeek-V2's expert counts (160 routed, top-6, 2 shared) under the noaux_tc
    # router: 8 groups of 20 (groups straddle the 32-expert lane blocks of the select
    # kernel), keep 3, scale 16, no normalisation; CUDA-core logits (T = 700) and
    # tensor-core logits (T = 2300).
    MoEShape("v2_groups", T=700, hidden_size=256, n_routed_experts=160, n_group=8, topk_group=3,
             num_experts_per_tok=6, moe_intermediate_size=128, n_shared_experts=2,
             routed_scaling_factor=16.0, norm_topk_prob=False, seed=11),
    MoEShape("v2_groups_tc", T=2300, hidden_size=256, n_routed_experts=160, n_group=8, topk_group=3,
             num_experts_per_tok=6, moe_intermediate_size=128, n_shared_experts=2,
             routed_scaling_factor=16.0, norm_topk_prob=False, seed=12),
]


@pytest.mark.parametrize("shape", SMALL, ids=lambda s: s.name)
def test_small_layer_every_token(shape):
    inp = make_inputs(shape, "cuda")
    y, idx, w = run_forward(shape, inp)
    x_bits = bf16_bits(inp["x"])
    rw, bias = inp["router_w"].cpu().numpy(), inp["e_bias"].cpu().numpy()
    ref_idx, ref_w, margin, scores = parity.oracle_route_all(shape, x_bits, rw, bias)
    rep = parity.compare_routing(shape, idx.cpu().numpy(), w.cpu().numpy(), ref_idx, ref_w, margin,
                                 scores, bias)
    assert not rep.mismatched_tokens, rep
    rows = np.arange(shape.T)
    y_ref = parity.oracle_layer_rows(shape, inp, rows, idx.cpu().numpy(), scores, ref_idx, ref_w, margin)
    err = parity.output_errors(y.float().cpu().numpy(), y_ref)
    print(f"{shape.name}: {err}, near ties {rep.near_ties}")
    parity.assert_output_close(y.float().cpu().numpy(), y_ref, shape.name)


def test_stages_compose_to_forward():
    """route -> dispatch -> experts -> combine through the C ABI equals moe_forward,
    and each stage matches its own definition."""
    shape = SMALL[4]
    inp = make_inputs(shape, "cuda")
    T, k, E, H, I, S = shape.T, shape.k, shape.E, shape.H, shape.I, shape.S
    cfg = abi.MoEConfig.from_shape(shape)
    dev = "cuda"
    ws = torch.empty(abi.workspace_size(cfg, T), dtype=torch.uint8, device=dev)
    idx = torch.empty((T, k), dtype=torch.int32, device=dev)
    w = torch.empty((T, k), dtype=torch.float32, device=dev)
    abi.moe_route(cfg, inp["x"], inp["router_w"], inp["e_bias"], idx, w, ws)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    x_perm = torch.empty((T * k, H), dtype=torch.bfloat16, device=dev)
    perm_src = torch.empty(T * k, dtype=torch.int32, device=dev)
    row_of = torch.empty((T, k), dtype=torch.int32, device=dev)
    abi.moe_dispatch(cfg, inp["x"], idx, offsets, x_perm, perm_src, row_of, ws)
    torch.cuda.synchronize()
    check_dispatch(shape, inp["x"], idx, offsets, x_perm, perm_src, row_of)

    h_r = torch.empty((T * k, I), dtype=torch.bfloat16, device=dev)
    h_s = torch.empty((T, S * I), dtype=torch.bfloat16, device=dev)
    y_perm = torch.empty((T * k + T, H), dtype=torch.float16, device=dev)
    y_sc = torch.empty((T * k + T, abi.y_perm_scale_cols(H)), dtype=torch.uint8, device=dev)
    abi.moe_experts(cfg, T, inp["x"], x_perm, offsets, perm_src, w, inp["w_gate"], inp["w_up"],
                    inp["w_down"], inp["ws_gate"], inp["ws_up"], inp["ws_down"], h_r, h_s, y_perm, y_sc)
    y = torch.empty((T, H), dtype=torch.float32, device=dev)
    abi.moe_combine(cfg, T, y_perm, y_sc, row_of, y)
    y16 = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
    abi.moe_combine(cfg, T, y_perm, y_sc, row_of, y16)
    torch.cuda.synchronize()
    assert abi.device_status() == 0

    # Expert stage against float64 matrix products of the same bf16 operands.
    yp = parity.decode_y_perm(y_perm, y_sc)
    # Block scaling: every 32-column block's largest magnitude sits in [2^14, 2^15] as fp16.
    blk = y_perm.float().abs().view(y_perm.shape[0], -1, 32).amax(-1)
    nz = blk > 0
    assert bool(((blk[nz] >= 2.0 ** 14) & (blk[nz] <= 2.0 ** 15)).all())
    off = offsets.cpu().tolist()
    for e in range(E):
        a, b = off[e], off[e + 1]
        if a == b:
            continue
        xe = x_perm[a:b].double()
        g = xe @ inp["w_gate"][e].double().T
        u = xe @ inp["w_up"][e].double().T
        h_ref = torch.nn.functional.silu(g) * u
        parity.assert_bf16_rounded(h_r[a:b], h_ref, f"h expert {e}")
        y_ref = (h_r[a:b].double() @ inp["w_down"][e].double().T) * w.view(-1)[perm_src[a:b].long()].double()[:, None]
        parity.assert_output_close(yp[a:b].double().cpu(), y_ref.cpu(), f"y_perm expert {e}")
    gs = inp["x"].double() @ inp["ws_gate"].double().T
    us = inp["x"].double() @ inp["ws_up"].double().T
    parity.assert_bf16_rounded(h_s, torch.nn.functional.silu(gs) * us, "h shared")
    ys_ref = h_s.double() @ inp["ws_down"].double().T
    parity.assert_output_close(yp[T * k:].double().cpu(), ys_ref.cpu(), "y shared")
    # Combine: fp32 gather-sum of the decoded rows in the order shared, slot 0..k-1;
    # the bf16 output is that sum rounded once to nearest.
    ref = yp[T * k:].clone()
    for j in range(k):
        ref += yp[row_of[:, j].long()]
    assert torch.equal(y.view(torch.int32), ref.view(torch.int32))
    assert torch.equal(y16.view(torch.int16), ref.to(torch.bfloat16).view(torch.int16))

    y_fwd, idx_fwd, w_fwd = run_forward(shape, inp)
    assert torch.equal(idx_fwd, idx) and torch.equal(w_fwd, w)
    assert torch.equal(y_fwd.view(torch.int32), y.view(torch.int32))
    y_fwd16, _, _ = run_forward(shape, inp, torch.bfloat16)
    assert torch.equal(y_fwd16.view(torch.int16), y16.view(torch.int16))


def test_zero_tokens_is_noop():
    shape = TINY.with_(T=0)
    cfg = abi.MoEConfig.from_shape(shape)
    inp = make_inputs(TINY, "cuda")
    empty = torch.empty((0, shape.H), dtype=torch.bfloat16, device="cuda")
    y = torch.empty_like(empty)
    ws = torch.empty(256, dtype=torch.uint8, device="cuda")
    n0 = abi.launch_count()
    abi.moe_forward(cfg, empty, inp["router_w"], inp["e_bias"], inp["w_gate"], inp["w_up"],
                    inp["w_down"], inp["ws_gate"], inp["ws_up"], inp["ws_down"], y, workspace=ws)
    assert abi.launch_count() == n0


def test_bounded_wait_gives_up_cleanly():
    """A wait on a barrier nothing arrives on returns an error status; the context survives."""
    assert abi.device_status() == 0
    abi.selftest_wait_timeout(20_000_000)  # 20 ms
    assert abi.device_status() == 0x901
    assert abi.device_status() == 0
    run_forward(TINY, make_inputs(TINY, "cuda"))  # the GPU still computes


def test_deterministic_and_launch_count():
    shape = SMALL[3]
    inp = make_inputs(shape, "cuda")
    n0 = abi.launch_count()
    y1, i1, w1 = run_forward(shape, inp)
    per_call = abi.launch_count() - n0
    assert per_call == 9  # router 2, dispatch 4, experts 2, combine 1
    y2, i2, w2 = run_forward(shape, inp)
    assert torch.equal(y1.view(torch.int32), y2.view(torch.int32)) and torch.equal(i1, i2)


# ---------------------------------------------------------------------------
# The five workload shapes at full size.
# ---------------------------------------------------------------------------
FULL = [(TINY, None), (MID, 256), (V3_DECODE, 256), (V3_PREFILL, 256), (V3_SKEWED, 256), (V3_E32, 64)]


@pytest.mark.parametrize("shape,n_sample", FULL, ids=lambda v: getattr(v, "name", str(v)))
def test_workload_full_size(shape, n_sample):
    inp = make_inputs(shape, "cuda")
    T, k, E = shape.T, shape.k, shape.E
    y, idx, w = run_forward(shape, inp)
    idx_h, w_h = idx.cpu().numpy(), w.cpu().numpy()

    # Routing of every token.
    x_bits = bf16_bits(inp["x"])
    rw, bias = inp["router_w"].cpu().numpy(), inp["e_bias"].cpu().numpy()
    ref_idx, ref_w, margin, scores = parity.oracle_route_all(shape, x_bits, rw, bias)
    rep = parity.compare_routing(shape, idx_h, w_h, ref_idx, ref_w, margin, scores, bias)
    assert not rep.mismatched_tokens, rep
    print(f"{shape.name}: near-ties {rep.near_ties}, differing near-tie sets "
          f"{rep.mismatched_near_ties}, order differences {rep.order_mismatches}")

    # Dispatch of every slot, in the launch configuration of moe_forward.
    cfg = abi.MoEConfig.from_shape(shape)
    ws = torch.empty(abi.workspace_size(cfg, T), dtype=torch.uint8, device="cuda")
    offsets = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    x_perm = torch.empty((T * k, shape.H), dtype=torch.bfloat16, device="cuda")
    perm_src = torch.empty(T * k, dtype=torch.int32, device="cuda")
    row_of = torch.empty((T, k), dtype=torch.int32, device="cuda")
    abi.moe_dispatch(cfg, inp["x"], idx, offsets, x_perm, perm_src, row_of, ws)
    torch.cuda.synchronize()
    check_dispatch(shape, inp["x"], idx, offsets, x_perm, perm_src, row_of)
    del x_perm, ws

    # Layer output: every token when small, else a seeded sample aimed at the risky
    # tiles (the last partial tile of 16 experts, every row of the 4 smallest segments
    # of <= 112 rows, which run transposed, rows of the most loaded expert), topped
    # up with random rows; rows are independent, so this is an exact subset check.
    if n_sample is None:
        rows, info = np.arange(T), {}
    else:
        rows, info = parity.targeted_rows(shape, idx_h, n_min=n_sample, seed=1234 + shape.seed)
    y_ref = parity.oracle_layer_rows(shape, inp, rows, idx_h, scores, ref_idx, ref_w, margin,
                                     parallel=n_sample is not None)
    err = parity.assert_output_close(y[torch.as_tensor(rows, device="cuda")].float().cpu().numpy(),
                                     y_ref, shape.name)
    print(f"{shape.name}: {len(rows)} rows ({info}), max|err|/RMS {err['max_abs_over_rms']:.2e}, "
          f"rel L1 {err['rel_l1']:.2e}")
    # Properties at any size: finite output, every token routed to k distinct experts.
    assert torch.isfinite(y.float()).all()
    srt = torch.sort(idx, dim=1).values
    assert (srt[:, 1:] != srt[:, :-1]).all()


def test_forward_replays_from_a_cuda_graph():
    """moe_forward captured into a CUDA graph and replayed gives the eager bits."""
    shape = SMALL[3]
    inp = make_inputs(shape, "cuda")
    from sparse_moe_layer_noaux_b200 import MoELayer
    layer = MoELayer.from_inputs(shape, inp)
    y_eager = layer(inp["x"])
    y = torch.empty_like(y_eager)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        layer(inp["x"], y)  # warm-up on the capture stream
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    y.zero_()
    with torch.cuda.graph(g):
        layer(inp["x"], y)
    g.replay()
    torch.cuda.synchronize()
    assert abi.device_status() == 0
    assert torch.equal(y, y_eager)
    del g


@pytest.mark.parametrize("shape,chunk", [(SMALL[3], 128), (SMALL[3], 0), (SMALL[4], 1000), (SMALL[0], 7)],
                         ids=["ragged-3chunks", "ragged-1chunk", "tiles-3chunks", "tiny-10chunks"])
def test_host_buffer_forward_matches_device_forward(shape, chunk):
    """moe_forward_host (pinned host x and y, the batch in chunks with copies overlapping
    the layer) gives moe_forward's output: rows are independent.  Bit for bit when the
    chunks and the whole batch take the same router-logit path (both >= 2048 rows, on
    the tensor cores, or both fewer); across that switch the logits' fp32 summation
    order differs, and the outputs agree to the fp16 rounding of the expert outputs."""
    inp = make_inputs(shape, "cuda")
    from sparse_moe_layer_noaux_b200 import MoELayer
    layer = MoELayer.from_inputs(shape, inp)
    y_dev = layer(inp["x"])
    x_host = inp["x"].cpu().pin_memory()
    y_host = layer.forward_host(x_host, chunk_tokens=chunk)
    y16 = layer.forward_host(x_host, chunk_tokens=chunk, out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    assert abi.device_status() == 0
    c = chunk if 0 < chunk < shape.T else shape.T
    last = shape.T - ((shape.T + c - 1) // c - 1) * c
    same_path = all((n >= 2048) == (shape.T >= 2048) for n in (c, last))
    if same_path:
        assert torch.equal(y_host, y_dev.cpu())
        assert torch.equal(y16, y_dev.cpu().bfloat16())
    else:
        # a last-bit change of a routing weight can move an expert output's block-scaled
        # fp16 storage by one step (2^-11 of its block maximum)
        ref = y_dev.cpu()
        assert float((y_host - ref).abs().max()) <= 2.0 ** -9 * float(ref.abs().max())
