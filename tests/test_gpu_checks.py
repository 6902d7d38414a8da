"""Robustness of the CUDA path to values and indices it cannot trust.

  * The router gives every token k distinct expert indices in [0, E) from at
    most topk_group groups even when scores are NaN or infinite (a NaN in x or
    an infinite bias), so the dispatch that follows never sees a bad index.
  * Index arrays passed in by a caller are checked on the device before they
    are used: an out-of-range entry is skipped (nothing is read or written
    through it), the rest of the call is exact, and moe_device_status reports
    MOE_ERR_DEVICE_CHECK with the kernel's code.

Every bad index here is caught by the kernel's own check before any access."""
import numpy as np
import pytest
import torch

from sparse_moe_layer_noaux_b200 import abi
from sparse_moe_layer_noaux_b200.workloads import TINY, MoEShape, make_inputs

pytestmark = pytest.mark.gpu

RAGGED = MoEShape("ragged", T=300, hidden_size=512, n_routed_experts=32, n_group=4, topk_group=2,
                  num_experts_per_tok=4, moe_intermediate_size=256, n_shared_experts=1,
                  routed_scaling_factor=2.5, norm_topk_prob=True, seed=7)
ERR_EXPERT_ID, ERR_ROW_INDEX, ERR_SEGMENT, ERR_SLOT = 0x401, 0x402, 0x403, 0x404


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from sparse_moe_layer_noaux_b200 import build
    build.build()
    assert abi.device_status() == 0
    yield
    abi.device_status()


def _route(shape, x, router_w, e_bias):
    cfg = abi.MoEConfig.from_shape(shape)
    idx = torch.full((x.shape[0], shape.k), -7, dtype=torch.int32, device="cuda")
    w = torch.empty((x.shape[0], shape.k), dtype=torch.float32, device="cuda")
    ws = torch.empty(abi.workspace_size(cfg, x.shape[0]), dtype=torch.uint8, device="cuda")
    abi.moe_route(cfg, x, router_w, e_bias, idx, w, ws)
    torch.cuda.synchronize()
    return idx.cpu().numpy()


def _valid_routing(shape, idx):
    gsz = shape.E // shape.n_group
    for row in idx:
        assert ((row >= 0) & (row < shape.E)).all(), row
        assert len(set(row.tolist())) == shape.k, row
        assert len({int(e) // gsz for e in row}) <= shape.topk_group, row


@pytest.mark.parametrize("T", [40, 2100], ids=["cuda-core-logits", "tensor-core-logits"])
def test_router_nan_and_infinite_scores_give_valid_ids(T):
    shape = RAGGED.with_(T=T)
    inp = make_inputs(shape, "cuda")
    x = inp["x"].clone()
    x[1] = float("nan")                 # every logit of token 1 is NaN
    x[2, :7] = float("nan")
    x[3] = float("inf")                 # logits +-inf or NaN
    bias = inp["e_bias"].clone()
    bias[0] = float("inf")              # group 0: +inf + (-inf) is NaN for its group score
    bias[1] = float("-inf")
    bias[9] = float("nan")
    idx = _route(shape, x, inp["router_w"], bias)
    _valid_routing(shape, idx)
    # A fully NaN token ranks every score as -inf: the lowest groups and indices win.
    assert sorted(idx[1].tolist()) == list(range(shape.k))
    assert abi.device_status() == 0


def test_out_of_range_expert_ids_are_skipped_by_dispatch_and_bias_update():
    shape = RAGGED
    T, k, E, H = shape.T, shape.k, shape.E, shape.H
    inp = make_inputs(shape, "cuda")
    cfg = abi.MoEConfig.from_shape(shape)
    g = torch.Generator(device="cuda").manual_seed(5)
    idx = torch.rand((T, E), generator=g, device="cuda").argsort(dim=1)[:, :k].to(torch.int32).contiguous()
    bad = [(3, 0, -1), (3, 2, E), (17, 1, E + 1000), (299, 3, 2 ** 31 - 1), (150, 0, -(2 ** 31))]
    for t, j, v in bad:
        idx[t, j] = v
    ws = torch.empty(abi.workspace_size(cfg, T), dtype=torch.uint8, device="cuda")
    offsets = torch.full((E + 1,), -5, dtype=torch.int32, device="cuda")
    x_perm = torch.zeros((T * k, H), dtype=torch.bfloat16, device="cuda")
    perm_src = torch.full((T * k,), -5, dtype=torch.int32, device="cuda")
    row_of = torch.full((T, k), -5, dtype=torch.int32, device="cuda")
    abi.moe_dispatch(cfg, inp["x"], idx, offsets, x_perm, perm_src, row_of, ws)
    assert abi.device_status() == ERR_EXPERT_ID
    assert abi.device_status() == 0  # read and cleared

    flat = idx.cpu().numpy().reshape(-1).astype(np.int64)
    ok = (flat >= 0) & (flat < E)
    counts = np.bincount(flat[ok], minlength=E)
    np.testing.assert_array_equal(offsets.cpu().numpy(), np.concatenate([[0], np.cumsum(counts)]))
    n_rows = int(ok.sum())
    order = np.nonzero(ok)[0][np.argsort(flat[ok], kind="stable")]
    np.testing.assert_array_equal(perm_src[:n_rows].cpu().numpy(), order)
    assert (perm_src[n_rows:].cpu().numpy() == -5).all()  # rows past the valid ones untouched
    ro = row_of.cpu().numpy().reshape(-1)
    assert (ro[~ok] == -1).all()
    np.testing.assert_array_equal(ro[order], np.arange(n_rows))
    src_tok = perm_src[:n_rows].long() // k
    assert torch.equal(x_perm[:n_rows].view(torch.int16), inp["x"][src_tok].view(torch.int16))
    assert not x_perm[n_rows:].view(torch.int16).any()  # nothing written past them

    bias = inp["e_bias"].clone()
    load = torch.empty(E, dtype=torch.int32, device="cuda")
    abi.moe_bias_update(cfg, idx, bias, 0.01, load)
    assert abi.device_status() == ERR_EXPERT_ID
    np.testing.assert_array_equal(load.cpu().numpy(), counts)


def test_out_of_range_rows_slots_and_segments_are_skipped():
    """combine with a bad row_of entry, the down GEMM with a bad perm_src entry and the
    gate/up GEMM with a segment past the row space: the bad entry is skipped, the
    rest matches the unmodified call exactly."""
    shape = RAGGED
    T, k, E, H, I, S = shape.T, shape.k, shape.E, shape.H, shape.I, shape.S
    inp = make_inputs(shape, "cuda")
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
    h_r = torch.zeros((T * k, I), dtype=torch.bfloat16, device=dev)
    h_s = torch.zeros((T, S * I), dtype=torch.bfloat16, device=dev)
    abi.moe_experts_gate_up(cfg, T, inp["x"], x_perm, offsets, inp["w_gate"], inp["w_up"], inp["ws_gate"],
                            inp["ws_up"], h_r, h_s)
    y_perm = torch.empty((T * k + T, H), dtype=torch.float16, device=dev)
    y_sc = torch.empty((T * k + T, abi.y_perm_scale_cols(H)), dtype=torch.uint8, device=dev)
    abi.moe_experts_down(cfg, T, h_r, h_s, offsets, perm_src, w, inp["w_down"], inp["ws_down"], y_perm, y_sc)
    y = torch.empty((T, H), dtype=torch.float32, device=dev)
    abi.moe_combine(cfg, T, y_perm, y_sc, row_of, y)
    assert abi.device_status() == 0

    # combine: token 5's slot 1 row index beyond the routed rows
    bad_row_of = row_of.clone()
    bad_row_of[5, 1] = T * k + 3
    bad_row_of[9, 0] = -2
    y2 = torch.empty_like(y)
    abi.moe_combine(cfg, T, y_perm, y_sc, bad_row_of, y2)
    assert abi.device_status() == ERR_ROW_INDEX
    keep = torch.ones(T, dtype=torch.bool, device=dev)
    keep[5] = keep[9] = False
    assert torch.equal(y2[keep], y[keep])
    from tests.parity import decode_y_perm
    yp = decode_y_perm(y_perm, y_sc)
    ref5 = yp[T * k + 5] + sum(yp[row_of[5, j].long()] for j in range(k) if j != 1)
    assert torch.allclose(y2[5], ref5, rtol=0, atol=1e-5 * float(ref5.abs().max()))

    # down GEMM: one routed row's slot index out of range -> weight 0 for that row
    bad_perm = perm_src.clone()
    r_bad = int(offsets[3].item())
    bad_perm[r_bad] = T * k + 11
    y_perm2, y_sc2 = torch.empty_like(y_perm), torch.empty_like(y_sc)
    abi.moe_experts_down(cfg, T, h_r, h_s, offsets, bad_perm, w, inp["w_down"], inp["ws_down"], y_perm2, y_sc2)
    assert abi.device_status() == ERR_SLOT
    yp2 = decode_y_perm(y_perm2, y_sc2)
    others = torch.ones(T * k + T, dtype=torch.bool, device=dev)
    others[r_bad] = False
    assert torch.equal(yp2[others], yp[others])
    assert not yp2[r_bad].any()

    # gate/up GEMM: the last expert's segment made to run past the T*k routed rows
    bad_off = offsets.clone()
    bad_off[E] = T * k + 500
    h_r2 = torch.zeros_like(h_r)
    h_s2 = torch.zeros_like(h_s)
    abi.moe_experts_gate_up(cfg, T, inp["x"], x_perm, bad_off, inp["w_gate"], inp["w_up"], inp["ws_gate"],
                            inp["ws_up"], h_r2, h_s2)
    assert abi.device_status() == ERR_SEGMENT
    last = int(offsets[E - 1].item())
    assert torch.equal(h_r2[:last], h_r[:last])
    assert not h_r2[last:].any()  # the rejected segment computed nothing
    assert torch.equal(h_s2, h_s)


def test_expert_parallel_ids_and_placement_entries_are_checked():
    """moe_ep_experts: a received expert id outside [-1, E), or one this rank does not
    hold, is skipped and recorded; the other received rows come back byte for byte.
    moe_ep_send: a placement entry outside [0, world) gives no row and is recorded."""
    from sparse_moe_layer_noaux_b200.ep import MoELayerEP, expert_block
    shape, world = RAGGED, 2
    cfg = abi.MoEConfig.from_shape(shape)
    inp = make_inputs(shape, "cuda")
    layers = [MoELayerEP(shape, world, r, inp["router_w"], inp["e_bias"], expert_block(inp["w_gate"], world, r),
                         expert_block(inp["w_up"], world, r), expert_block(inp["w_down"], world, r),
                         inp["ws_gate"], inp["ws_up"], inp["ws_down"]) for r in range(world)]
    st = layers[0].send(inp["x"])
    torch.cuda.synchronize()
    assert abi.device_status() == 0
    c0, c1 = st.send_counts.cpu().tolist()
    rows = st.send_rows[c0:c0 + c1].clone()       # rank 0's rows for rank 1
    H, k, El = shape.H, shape.k, shape.E // world
    L = layers[1]
    none = torch.empty((0, H), dtype=torch.bfloat16, device="cuda")

    def run(recv):
        ret = torch.zeros((recv.shape[0], L.return_row_bytes), dtype=torch.uint8, device="cuda")
        ws = torch.empty(abi.ep_workspace_size(cfg, world, 0, recv.shape[0]), dtype=torch.uint8, device="cuda")
        abi.moe_ep_experts(cfg, world, 1, none, recv, L.w_gate, L.w_up, L.w_down, None, None, None, ret,
                           None, None, ws)
        return ret, abi.device_status()

    clean, status = run(rows)
    assert status == 0
    bad = rows.clone()
    ids = bad[:, 2 * H:2 * H + 4 * k].view(torch.int32)   # a view into `bad`
    j0 = int(torch.nonzero(ids[0] >= 0)[0])
    j1 = int(torch.nonzero(ids[1] >= 0)[0])
    ids[0, j0] = 10 ** 6                                 # outside [-1, E)
    ids[1, j1] = 0                                       # an expert of rank 0, not held here
    got, status = run(bad)
    assert status == ERR_EXPERT_ID
    assert torch.equal(got[2:], clean[2:])

    # A placement entry outside [0, world): the slots sent to it get no row.
    table = torch.full((shape.E, 2), -1, dtype=torch.int32)
    table[:, 0] = torch.arange(shape.E, dtype=torch.int32) // El
    torch.cuda.synchronize()
    e_hot = int(torch.bincount(st.idx.reshape(-1).long(), minlength=shape.E).argmax())
    table[e_hot, 1] = 5
    n_max = abi.ep_send_rows_max(cfg, shape.T, world)
    counts = torch.empty(world, dtype=torch.int32, device="cuda")
    srows = torch.empty((n_max, L.send_row_bytes), dtype=torch.uint8, device="cuda")
    row_of = torch.empty((shape.T, k), dtype=torch.int32, device="cuda")
    ws = torch.empty(abi.ep_workspace_size(cfg, world, shape.T, 0), dtype=torch.uint8, device="cuda")
    abi.moe_ep_send(cfg, world, inp["x"], st.idx, st.w, counts, srows, row_of, ws, expert_ranks=table.cuda())
    assert abi.device_status() == ERR_EXPERT_ID
    table[e_hot, 1] = 1 - e_hot // El                    # the other rank: a valid copy
    abi.moe_ep_send(cfg, world, inp["x"], st.idx, st.w, counts, srows, row_of, ws, expert_ranks=table.cuda())
    assert abi.device_status() == 0
