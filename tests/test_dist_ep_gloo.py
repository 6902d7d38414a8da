"""The expert-parallel layer's exchange on CPU ranks (gloo): MoELayerEP.forward with
its all-to-alls over a real process group, the library calls replaced by the
oracle-backed stand-in of tests/ep_cpu_kernels.py.  Each rank holds E/world of
the routed experts and its own tokens; every rank's output must equal the float64
oracle's single-device layer on its tokens; a token must cross to each rank that
holds one of its experts exactly once; and the rows a rank receives must be
exactly the other ranks' send rows for it, in rank order."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from sparse_moe_layer_noaux_b200.workloads import MoEShape, bf16_bits, make_inputs

SHAPE = MoEShape("ep", T=24, hidden_size=256, n_routed_experts=16, n_group=4, topk_group=2,
                 num_experts_per_tok=4, moe_intermediate_size=128, n_shared_experts=1,
                 routed_scaling_factor=2.5, norm_topk_prob=True, seed=41)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_tokens(shape, rank):
    T = shape.T + 5 * rank  # ranks bring different batch sizes (one may be empty)
    if rank == 3:
        T = 0
    g = torch.Generator().manual_seed(1000 + rank)
    return torch.randn((T, shape.H), generator=g).to(torch.bfloat16)


def _placement(shape, world, n_redundant):
    """Every rank builds the same placement: copies of the experts that the oracle's
    routing of all ranks' batches loads most (the live statistics of the pages)."""
    import oracle
    from sparse_moe_layer_noaux_b200.ep import EPPlacement
    if n_redundant == 0:
        return EPPlacement(shape.E, world)
    inp = make_inputs(shape, "cpu")
    load = np.zeros(shape.E, np.int64)
    for r in range(world):
        x = _rank_tokens(shape, r)
        if x.shape[0]:
            idx, _, _ = oracle.route(shape, bf16_bits(x), inp["router_w"].numpy(), inp["e_bias"].numpy())
            load += np.bincount(idx.reshape(-1), minlength=shape.E)
    return EPPlacement.from_load(shape.E, world, load, n_redundant, max_rep=world)


def _worker(rank, world, n_redundant, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    from sparse_moe_layer_noaux_b200.ep import MoELayerEP
    from tests import ep_cpu_kernels
    import oracle
    shape = SHAPE
    inp = make_inputs(shape, "cpu")            # same seed: the same weights on every rank
    pl = _placement(shape, world, n_redundant)
    layer = MoELayerEP(shape, world, rank, inp["router_w"], inp["e_bias"], pl.rank_weights(inp["w_gate"], rank),
                       pl.rank_weights(inp["w_up"], rank), pl.rank_weights(inp["w_down"], rank),
                       inp["ws_gate"], inp["ws_up"], inp["ws_down"], placement=pl, _kernels=ep_cpu_kernels)
    x = _rank_tokens(shape, rank)
    y = layer(x)
    # The same batch through the exchange phases by hand, to look at what moved.
    st = layer.send(x)
    recv = torch.empty_like(st.send_counts)
    dist.all_to_all_single(recv, st.send_counts)
    layer.plan(st, recv)
    n_send = sum(st.send_splits)
    dist.all_to_all_single(st.recv_rows, st.send_rows[:n_send], st.recv_splits, st.send_splits)
    # The oracle's single-device layer on this rank's tokens (all experts).
    fetch = oracle.in_memory_experts(bf16_bits(inp["w_gate"]), bf16_bits(inp["w_up"]), bf16_bits(inp["w_down"]))
    shared = tuple(bf16_bits(inp[n]) for n in ("ws_gate", "ws_up", "ws_down"))
    y_ref, idx_ref, _, _ = oracle.moe_layer(shape, bf16_bits(x), inp["router_w"].numpy(), inp["e_bias"].numpy(),
                                            fetch, shared)
    out[rank] = {"y": y.numpy(), "y_ref": y_ref, "idx": st.idx.numpy(), "idx_ref": idx_ref,
                 "recv_counts": recv.numpy(), "send_splits": st.send_splits, "recv_splits": st.recv_splits,
                 "send_rows": st.send_rows[:n_send].numpy(), "recv_rows": st.recv_rows.numpy(),
                 "send_row_of": st.send_row_of.numpy(),
                 "expert_ranks": None if pl.expert_ranks is None else pl.expert_ranks.numpy()}
    dist.barrier()
    dist.destroy_process_group()


def _dest(e, t, El, table):
    """The rank slot (t, ., e) is sent to: e's block, or replica t mod n_e of its copies."""
    if table is None:
        return e // El
    reps = [int(r) for r in table[e] if r >= 0]
    return reps[t % len(reps)]


@pytest.mark.parametrize("world,n_redundant", [(2, 0), (4, 0), (2, 3), (4, 6)],
                         ids=["w2", "w4", "w2-3copies", "w4-6copies"])
def test_expert_parallel_exchange_matches_the_single_device_layer(world, n_redundant, oracle_lib):
    port = _free_port()
    with mp.get_context("spawn").Manager() as m:   # no fork of a multi-threaded process
        out = m.dict()
        mp.spawn(_worker, args=(world, n_redundant, port, out), nprocs=world, join=True)
        res = dict(out)
    El = SHAPE.E // world
    gsz = SHAPE.E // SHAPE.n_group
    H, k = SHAPE.H, SHAPE.k
    table = res[0]["expert_ranks"]
    if n_redundant:
        assert int((table >= 0).sum()) == SHAPE.E + n_redundant
    to_copies = 0
    for r in range(world):
        d = res[r]
        assert (d["idx"] == d["idx_ref"]).all()
        if d["y"].size:
            rms = np.sqrt(np.mean(d["y_ref"] ** 2))
            err = np.abs(d["y"] - d["y_ref"]).max() / rms
            assert err <= 2e-2, (r, err)   # fp16 storage of the expert outputs
        # One row per (token, destination rank), at the token's first slot bound there;
        # rows sorted by rank, tokens ascending within a rank.
        T = d["idx"].shape[0]
        dest = np.array([[_dest(int(d["idx"][t, j]), t, El, table) for j in range(k)] for t in range(T)],
                        dtype=np.int64).reshape(T, k)
        to_copies += int((dest != d["idx"] // El).sum())
        off = np.concatenate([[0], np.cumsum(d["send_splits"])])
        for t in range(T):
            first = [j for j in range(k) if dest[t, j] not in dest[t, :j]]
            assert sorted(np.nonzero(d["send_row_of"][t] >= 0)[0].tolist()) == first
            for j in first:
                row = d["send_row_of"][t, j]
                assert off[dest[t, j]] <= row < off[dest[t, j] + 1]
                # The row carries the ids of the token's slots bound for that rank, -1 elsewhere.
                np.testing.assert_array_equal(d["send_rows"][row, 2 * H:2 * H + 4 * k].view("<i4"),
                                              np.where(dest[t] == dest[t, j], d["idx"][t], -1))
        for dst in range(world):
            # Tokens with a slot bound for dst, ascending, hold rows off[dst], off[dst] + 1, ...
            rows_dst = [int(d["send_row_of"][t][(dest[t] == dst) & (d["send_row_of"][t] >= 0)][0])
                        for t in range(T) if (dest[t] == dst).any()]
            assert rows_dst == list(range(off[dst], off[dst + 1]))
            assert res[dst]["recv_counts"][r] == d["send_splits"][dst] == res[dst]["recv_splits"][r]
            # What dst received from r is r's send rows for dst, byte for byte.
            r0 = sum(res[dst]["recv_splits"][:r])
            np.testing.assert_array_equal(res[dst]["recv_rows"][r0:r0 + d["send_splits"][dst]],
                                          d["send_rows"][off[dst]:off[dst + 1]])
        # Groups do not straddle ranks here, so without copies a token reaches at most
        # topk_group ranks.
        if table is None and El % gsz == 0 and T:
            assert (d["send_row_of"] >= 0).sum(1).max() <= SHAPE.topk_group
    if n_redundant:
        assert to_copies > 0   # some slots went to a copy on another rank than the expert's block


def _replan_worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    from sparse_moe_layer_noaux_b200.ep import MoELayerEP, expert_block
    from tests import ep_cpu_kernels
    import oracle
    shape = SHAPE
    inp = make_inputs(shape, "cpu")
    layer = MoELayerEP(shape, world, rank, inp["router_w"], inp["e_bias"], expert_block(inp["w_gate"], world, rank),
                       expert_block(inp["w_up"], world, rank), expert_block(inp["w_down"], world, rank),
                       inp["ws_gate"], inp["ws_up"], inp["ws_down"], _kernels=ep_cpu_kernels)
    x = _rank_tokens(shape, rank)
    y0 = layer(x)
    # Live statistics: this batch's loads, summed over the ranks, then new copies.
    load = layer.count_load(layer.send(x))
    dist.all_reduce(load)
    pl = layer.replan(load, n_redundant=4)
    y1 = layer(x)
    fetch = oracle.in_memory_experts(bf16_bits(inp["w_gate"]), bf16_bits(inp["w_up"]), bf16_bits(inp["w_down"]))
    shared = tuple(bf16_bits(inp[n]) for n in ("ws_gate", "ws_up", "ws_down"))
    y_ref = oracle.moe_layer(shape, bf16_bits(x), inp["router_w"].numpy(), inp["e_bias"].numpy(), fetch, shared)[0]
    ids = layer.local_ids
    out[rank] = {"y0": y0.numpy(), "y1": y1.numpy(), "y_ref": y_ref, "load": load.numpy(),
                 "table": pl.expert_ranks.numpy(), "ids": ids,
                 "weights_ok": all(torch.equal(getattr(layer, n), inp[n][torch.as_tensor(ids)])
                                   for n in ("w_gate", "w_up", "w_down"))}
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_replan_moves_the_copies_and_keeps_the_output(world, oracle_lib):
    """count_load + replan: the copies' weights arrive from their block ranks (each
    rank then holds exactly the weights of the experts its new table gives it), and
    the layer's output is unchanged against the oracle."""
    from sparse_moe_layer_noaux_b200 import abi
    port = _free_port()
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.spawn(_replan_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    load = res[0]["load"]
    # The summed load is every rank's routing counted once.
    total = sum(_rank_tokens(SHAPE, r).shape[0] for r in range(world)) * SHAPE.k
    assert int(load.sum()) == total
    want = abi.ep_place(SHAPE.E, world, torch.as_tensor(load, dtype=torch.int64), 4, world).numpy()
    for r in range(world):
        d = res[r]
        np.testing.assert_array_equal(d["table"], want)
        assert d["ids"] == [e for e in range(SHAPE.E) if r in want[e].tolist()]
        assert d["weights_ok"]
        if d["y1"].size:
            rms = np.sqrt(np.mean(d["y_ref"] ** 2))
            for y in (d["y0"], d["y1"]):
                assert np.abs(y - d["y_ref"]).max() / rms <= 2e-2
    assert int((want >= 0).sum()) == SHAPE.E + 4
