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


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    from sparse_moe_layer_noaux_b200.ep import MoELayerEP, expert_block
    from tests import ep_cpu_kernels
    import oracle
    shape = SHAPE
    inp = make_inputs(shape, "cpu")            # same seed: the same weights on every rank
    layer = MoELayerEP(shape, world, rank, inp["router_w"], inp["e_bias"],
                       expert_block(inp["w_gate"], world, rank), expert_block(inp["w_up"], world, rank),
                       expert_block(inp["w_down"], world, rank), inp["ws_gate"], inp["ws_up"], inp["ws_down"],
                       _kernels=ep_cpu_kernels)
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
                 "send_row_of": st.send_row_of.numpy()}
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_expert_parallel_exchange_matches_the_single_device_layer(world, oracle_lib):
    port = _free_port()
    with mp.get_context("spawn").Manager() as m:   # no fork of a multi-threaded process
        out = m.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    El = SHAPE.E // world
    gsz = SHAPE.E // SHAPE.n_group
    H, k = SHAPE.H, SHAPE.k
    for r in range(world):
        d = res[r]
        assert (d["idx"] == d["idx_ref"]).all()
        if d["y"].size:
            rms = np.sqrt(np.mean(d["y_ref"] ** 2))
            err = np.abs(d["y"] - d["y_ref"]).max() / rms
            assert err <= 2e-2, (r, err)   # fp16 storage of the expert outputs
        # One row per (token, rank holding one of its experts), at the token's first
        # slot on that rank; rows sorted by rank, tokens ascending within a rank.
        ranks = d["idx"] // El
        off = np.concatenate([[0], np.cumsum(d["send_splits"])])
        for t in range(d["idx"].shape[0]):
            first = [j for j in range(k) if ranks[t, j] not in ranks[t, :j]]
            assert sorted(np.nonzero(d["send_row_of"][t] >= 0)[0].tolist()) == first
            for j in first:
                row = d["send_row_of"][t, j]
                assert off[ranks[t, j]] <= row < off[ranks[t, j] + 1]
                # The row carries x[t]'s routing: the token's k expert ids.
                np.testing.assert_array_equal(d["send_rows"][row, 2 * H:2 * H + 4 * k].view("<i4"), d["idx"][t])
        for dst in range(world):
            # Tokens with an expert on dst, ascending, hold rows off[dst], off[dst] + 1, ...
            rows_dst = [int(d["send_row_of"][t][(ranks[t] == dst) & (d["send_row_of"][t] >= 0)][0])
                        for t in range(d["idx"].shape[0]) if (ranks[t] == dst).any()]
            assert rows_dst == list(range(off[dst], off[dst + 1]))
            assert res[dst]["recv_counts"][r] == d["send_splits"][dst] == res[dst]["recv_splits"][r]
            # What dst received from r is r's send rows for dst, byte for byte.
            r0 = sum(res[dst]["recv_splits"][:r])
            np.testing.assert_array_equal(res[dst]["recv_rows"][r0:r0 + d["send_splits"][dst]],
                                          d["send_rows"][off[dst]:off[dst + 1]])
        # Groups do not straddle ranks here, so a token reaches at most topk_group ranks.
        if El % gsz == 0 and d["idx"].size:
            assert max(len(set(row.tolist())) for row in ranks) <= SHAPE.topk_group
            assert (d["send_row_of"] >= 0).sum(1).max() <= SHAPE.topk_group
