"""The expert-parallel layer on the GPU (libmoe's moe_ep_* calls).

  * world = 1 over a real NCCL process group: MoELayerEP.forward through the
    same code path as on many GPUs matches moe_forward (up to the fp16 rounding
    of the returned sums) and repeats bit for bit.
  * world = 2, 4 and 8 on one GPU: every rank's phases run on this GPU and the
    all-to-alls are done by copying each rank's row blocks into the others'
    receive buffers (no kernel waits on another, so nothing can deadlock); each
    rank's output is checked against moe_forward on its tokens and, on a sample,
    against the float64 oracle.
  * the send rows, counts and slot map of moe_ep_send byte for byte against a
    host restatement of the contract, and the block encoding of the return rows."""
import datetime
import os
import socket

import numpy as np
import pytest
import torch

from sparse_moe_layer_noaux_b200 import MoELayer, abi
from sparse_moe_layer_noaux_b200.ep import EPPlacement, MoELayerEP, expert_block
from sparse_moe_layer_noaux_b200.workloads import MID, V3_DECODE, V3_SKEWED, MoEShape, bf16_bits, make_inputs
from tests import parity

pytestmark = pytest.mark.gpu

SMALL = MoEShape("ep_small", T=300, hidden_size=512, n_routed_experts=32, n_group=4, topk_group=2,
                 num_experts_per_tok=4, moe_intermediate_size=256, n_shared_experts=1,
                 routed_scaling_factor=2.5, norm_topk_prob=True, seed=13)


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from sparse_moe_layer_noaux_b200 import build
    build.build()
    yield
    torch.cuda.empty_cache()


def _layers(shape, inp, world, placement=None):
    if placement is None:
        return [MoELayerEP(shape, world, r, inp["router_w"], inp["e_bias"], expert_block(inp["w_gate"], world, r),
                           expert_block(inp["w_up"], world, r), expert_block(inp["w_down"], world, r),
                           inp["ws_gate"], inp["ws_up"], inp["ws_down"]) for r in range(world)]
    return [MoELayerEP(shape, world, r, inp["router_w"], inp["e_bias"], placement.rank_weights(inp["w_gate"], r),
                       placement.rank_weights(inp["w_up"], r), placement.rank_weights(inp["w_down"], r),
                       inp["ws_gate"], inp["ws_up"], inp["ws_down"], placement=placement) for r in range(world)]


def loopback_forward(layers, xs):
    """All ranks' phases on this GPU, the all-to-alls done as copies of row blocks."""
    W = len(layers)
    steps = [L.send(x) for L, x in zip(layers, xs)]
    counts = [st.send_counts.cpu().tolist() for st in steps]      # counts[s][d]: rows of s for d
    for d in range(W):
        layers[d].plan(steps[d], torch.tensor([counts[s][d] for s in range(W)], dtype=torch.int32, device="cuda"))
    off = [np.concatenate([[0], np.cumsum(c)]).astype(int) for c in counts]
    for d in range(W):
        if steps[d].recv_rows.shape[0]:
            steps[d].recv_rows.copy_(torch.cat([steps[s].send_rows[off[s][d]:off[s][d + 1]] for s in range(W)]))
    for d in range(W):
        layers[d].experts(steps[d], xs[d])
    for s in range(W):
        for d in range(W):
            a, b = off[s][d], off[s][d + 1]
            r0 = sum(steps[d].recv_splits[:s])
            steps[s].back_rows[a:b].copy_(steps[d].return_rows[r0:r0 + b - a])
    ys = [L.combine(st) for L, st in zip(layers, steps)]
    torch.cuda.synchronize()
    assert abi.device_status() == 0
    return ys, steps


def host_send(idx, w, x_bits, world, E, row_bytes, table=None):
    """moe_ep_send's outputs restated on the host: slot (t, j) of expert e goes to e's
    block rank (or replica t mod n_e of its copies); one row per (token, destination)
    at the token's first slot bound there, rows by rank then token; a row carries the
    ids of the slots bound for its rank and -1 for the others."""
    T, k = idx.shape
    H = x_bits.shape[1]
    El = E // world

    def dest(e, t):
        if table is None:
            return e // El
        reps = [int(r) for r in table[e] if r >= 0]
        return reps[t % len(reps)]
    d = np.array([[dest(int(idx[t, j]), t) for j in range(k)] for t in range(T)], dtype=np.int64).reshape(T, k)
    entries = sorted(((int(d[t, j]), t, j) for t in range(T) for j in range(k) if d[t, j] not in d[t, :j]),
                     key=lambda e: (e[0], e[1]))
    counts = np.bincount([e[0] for e in entries], minlength=world).astype(np.int32)
    row_of = np.full((T, k), -1, np.int32)
    rows = np.zeros((len(entries), row_bytes), np.uint8)
    for r, (rank, t, j) in enumerate(entries):
        row_of[t, j] = r
        rows[r, :2 * H] = x_bits[t].view(np.uint8)
        rows[r, 2 * H:2 * H + 4 * k] = np.where(d[t] == rank, idx[t], -1).astype("<i4").view(np.uint8)
        rows[r, 2 * H + 4 * k:2 * H + 8 * k] = w[t].astype("<f4").view(np.uint8)
    return counts, row_of, rows


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_world_one_over_nccl_matches_moe_forward():
    import torch.distributed as dist
    shape = SMALL
    inp = make_inputs(shape, "cuda")
    store = dist.TCPStore("127.0.0.1", _free_port(), 1, True, timeout=datetime.timedelta(seconds=60))
    dist.init_process_group("nccl", store=store, rank=0, world_size=1, timeout=datetime.timedelta(seconds=60),
                            device_id=torch.device("cuda", torch.cuda.current_device()))
    try:
        layer = _layers(shape, inp, 1)[0]
        y = layer(inp["x"])
        y2 = layer(inp["x"])
        # Load statistics and a re-plan through the same collectives (one rank: no
        # copy is possible, the weight exchange is empty); the bias must not move.
        bias0 = inp["e_bias"].clone()
        st = layer.send(inp["x"])
        load = layer.count_load(st)
        layer.replan(load, n_redundant=4)
        y3 = layer(inp["x"])
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    assert abi.device_status() == 0
    assert torch.equal(inp["e_bias"], bias0)
    assert torch.equal(load.cpu(), torch.bincount(st.idx.reshape(-1).long().cpu(), minlength=shape.E).int())
    assert torch.equal(y3, y)
    y_ref = MoELayer.from_inputs(shape, inp)(inp["x"])
    # One row per token each way: the returned row is the token's k weighted expert
    # outputs summed in fp32 and stored once more as block-scaled fp16.
    parity.assert_output_close(y.cpu().numpy(), y_ref.cpu().numpy(), "world 1 vs moe_forward")
    assert torch.equal(y2, y)


@pytest.mark.parametrize("world,copies", [(1, 0), (4, 0), (8, 0), (8, 24)])
def test_send_rows_match_the_contract(world, copies):
    shape = V3_DECODE
    inp = make_inputs(shape, "cuda")
    placement = None
    if copies:
        load = torch.arange(shape.E, dtype=torch.int64) % 7   # any loads: the rule is what is checked
        placement = EPPlacement.from_load(shape.E, world, load, copies, max_rep=3)
    layer = _layers(shape, inp, world, placement)[0]
    st = layer.send(inp["x"])
    torch.cuda.synchronize()
    assert abi.device_status() == 0
    idx, w = st.idx.cpu().numpy(), st.w.cpu().numpy()
    table = None if placement is None else placement.expert_ranks.numpy()
    counts, row_of, rows = host_send(idx, w, bf16_bits(inp["x"]), world, shape.E, layer.send_row_bytes, table)
    np.testing.assert_array_equal(st.send_counts.cpu().numpy(), counts)
    np.testing.assert_array_equal(st.send_row_of.cpu().numpy(), row_of)
    np.testing.assert_array_equal(st.send_rows[:rows.shape[0]].cpu().numpy(), rows)
    if world == 8 and not copies:   # 32 experts per rank = one expert group per rank
        assert (row_of >= 0).sum(1).max() <= shape.topk_group
        print(f"world 8: {rows.shape[0]} send rows for {idx.shape[0]} tokens "
              f"({rows.shape[0] / idx.shape[0]:.2f} per token; k = {shape.k} without the per-rank merge)")


V2_GROUPS = MoEShape("v2_groups", T=700, hidden_size=256, n_routed_experts=160, n_group=8, topk_group=3,
                     num_experts_per_tok=6, moe_intermediate_size=128, n_shared_experts=2,
                     routed_scaling_factor=16.0, norm_topk_prob=False, seed=11)


@pytest.mark.parametrize("shape,world,T_rank", [(SMALL, 2, 300), (SMALL, 4, 150), (MID, 4, 1024),
                                                (V3_DECODE, 8, 128), (V2_GROUPS, 8, 200)],
                         ids=["small-w2", "small-w4", "mid-w4", "v3_decode-w8", "v2_groups-w8"])
def test_loopback_ranks_match_single_gpu_layer(shape, world, T_rank):
    inp = make_inputs(shape, "cuda")
    layers = _layers(shape, inp, world)
    g = torch.Generator(device="cuda").manual_seed(77)
    xs = [torch.randn((T_rank + 3 * r, shape.H), generator=g, device="cuda").to(torch.bfloat16)
          for r in range(world)]
    ys, steps = loopback_forward(layers, xs)
    # The return rows are block-scaled fp16: every 32-value block's largest
    # magnitude sits in [2^14, 2^15] unless the block is tiny (code 15) or zero.
    H = shape.H
    for st in steps:
        ret = st.return_rows.cpu().numpy()
        if ret.shape[0]:
            vals = np.abs(np.ascontiguousarray(ret[:, :2 * H]).view(np.float16).astype(np.float32))
            bmax = vals.reshape(ret.shape[0], H // 32, 32).max(2)
            codes = ret[:, 2 * H:2 * H + H // 32]
            assert (((bmax >= 2.0 ** 14) & (bmax <= 2.0 ** 15)) | (codes == 15)).all()
    full = MoELayer.from_inputs(shape, inp)
    gsz = shape.E // shape.n_group
    El = shape.E // world
    worst = 0.0
    for r in range(world):
        y_ref = full(xs[r])
        torch.cuda.synchronize()
        srt = torch.sort(steps[r].idx, dim=1).values
        assert bool((srt[:, 1:] != srt[:, :-1]).all())  # k distinct experts per token
        # The same rows through the same expert GEMM code: equal up to the fp16
        # storage of the expert outputs (a segment that runs transposed in one layout
        # and not the other can round differently in the last place).
        e = parity.assert_output_close(ys[r].cpu().numpy(), y_ref.cpu().numpy(), f"{shape.name} rank {r}")
        worst = max(worst, e["max_abs_over_rms"])
        if El % gsz == 0:
            ranks = (steps[r].idx.long() // El).cpu().numpy()
            assert max(len(set(row.tolist())) for row in ranks) <= shape.topk_group
            assert sum(steps[r].send_splits) <= shape.topk_group * xs[r].shape[0]
    print(f"{shape.name} world {world}: worst max|err|/RMS vs single GPU {worst:.2e}, "
          f"rows received per rank {[sum(s.recv_splits) for s in steps]}, "
          f"rows sent per token {[round(sum(s.send_splits) / max(s.T, 1), 2) for s in steps]}")
    # One rank against the float64 oracle on a sample of its tokens (near ties
    # scored on the GPU's expert set, as in the single-GPU parity tests).
    r = world - 1
    inp_r = dict(inp, x=xs[r])
    x_bits = bf16_bits(xs[r])
    rw, bias = inp["router_w"].cpu().numpy(), inp["e_bias"].cpu().numpy()
    ref_idx, ref_w, margin, scores = parity.oracle_route_all(shape, x_bits, rw, bias)
    idx_r = steps[r].idx.cpu().numpy()
    rep = parity.compare_routing(shape, idx_r, steps[r].w.cpu().numpy(), ref_idx, ref_w, margin, scores, bias)
    assert not rep.mismatched_tokens, rep
    rows = np.sort(np.random.default_rng(5).choice(xs[r].shape[0], min(48, xs[r].shape[0]), replace=False))
    y_or = parity.oracle_layer_rows(shape, inp_r, rows, idx_r, scores, ref_idx, ref_w, margin)
    parity.assert_output_close(ys[r][torch.as_tensor(rows, device="cuda")].cpu().numpy(), y_or,
                               f"{shape.name} rank {r} vs oracle")


def test_loopback_rank_without_tokens_and_rank_without_rows():
    """World 2 with every token's experts on rank 0 (a bias of +10 on rank 0's expert
    block): rank 0 brings no tokens but receives all rows (routed experts only, no
    shared rows), rank 1 brings tokens but receives no rows (shared experts only,
    empty expert segments)."""
    shape = SMALL
    inp = make_inputs(shape, "cuda")
    El = shape.E // 2
    bias = inp["e_bias"].clone()
    bias[:El] += 10.0
    inp = dict(inp, e_bias=bias)
    layers = _layers(shape, inp, 2)
    g = torch.Generator(device="cuda").manual_seed(78)
    xs = [torch.empty((0, shape.H), device="cuda", dtype=torch.bfloat16),
          torch.randn((200, shape.H), generator=g, device="cuda").to(torch.bfloat16)]
    ys, steps = loopback_forward(layers, xs)
    assert steps[0].recv_rows.shape[0] == 200 and steps[1].recv_rows.shape[0] == 0
    assert ys[0].shape == (0, shape.H)
    assert int(steps[1].idx.max()) < El
    y_ref = MoELayer.from_inputs(shape, inp)(xs[1])
    torch.cuda.synchronize()
    parity.assert_output_close(ys[1].cpu().numpy(), y_ref.cpu().numpy(), "rank 1 vs single GPU")


def _expert_rows(steps, H, k):
    """Per rank: slots it computes (received ids other than -1)."""
    out = []
    for st in steps:
        ids = st.recv_rows[:, 2 * H:2 * H + 4 * k].contiguous().view(torch.int32)
        out.append(int((ids != -1).sum()))
    return out


def test_redundant_experts_balance_the_skewed_load():
    """V3 skewed routing (zipf bias: a few experts take most rows) over 8 ranks: copies
    of the most loaded experts, placed from the routing of the batch itself, cut the
    most loaded rank's expert rows, and every rank's output still matches the
    single-GPU layer."""
    shape, world, T_rank = V3_SKEWED, 8, 1024
    inp = make_inputs(shape, "cuda")
    xs = [inp["x"][r * T_rank:(r + 1) * T_rank].contiguous() for r in range(world)]
    plain = _layers(shape, inp, world)
    _, steps0 = loopback_forward(plain, xs)
    load = torch.bincount(torch.cat([st.idx.reshape(-1) for st in steps0]).long(), minlength=shape.E).cpu()
    rows_plain = _expert_rows(steps0, shape.H, shape.k)
    del plain, steps0
    placement = EPPlacement.from_load(shape.E, world, load, n_redundant=32, max_rep=world)
    layers = _layers(shape, inp, world, placement)
    ys, steps = loopback_forward(layers, xs)
    rows_copies = _expert_rows(steps, shape.H, shape.k)
    assert sum(rows_copies) == sum(rows_plain) == world * T_rank * shape.k
    mean = sum(rows_plain) / world
    print(f"v3_skewed world 8: expert rows per rank without copies {rows_plain} (max/mean "
          f"{max(rows_plain) / mean:.2f}), with 32 copies {rows_copies} (max/mean {max(rows_copies) / mean:.2f})")
    assert max(rows_copies) < 0.7 * max(rows_plain)
    full = MoELayer.from_inputs(shape, inp)
    for r in (0, world - 1):
        y_ref = full(xs[r])
        torch.cuda.synchronize()
        parity.assert_output_close(ys[r].cpu().numpy(), y_ref.cpu().numpy(), f"skewed copies rank {r}")

