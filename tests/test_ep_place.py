"""The redundant-expert placement of the expert-parallel layer (libmoe's host-only
moe_ep_place and moe_ep_local_experts), on the CPU.

moe_ep_place: every expert starts on its block rank e // (E/world); then, once per
extra copy, the expert whose copies carry the most rows each gets a copy on the
least loaded rank that does not hold it, its rows split evenly over its copies
("DeepSeek-V3 notes" (knlb.dev), § infrastructure, prefilling: redundant experts
for load balance, from live statistics).  Pinned by hand-worked placements and by
the properties that define a placement table."""
import numpy as np
import pytest
import torch

from sparse_moe_layer_noaux_b200 import abi
from sparse_moe_layer_noaux_b200.abi import MoEError


def table(E, world, load, n_redundant, max_rep):
    return abi.ep_place(E, world, torch.tensor(load, dtype=torch.int64), n_redundant, max_rep).numpy()


def rank_loads(t, load, world):
    """Rows per rank when each expert's rows split evenly over its copies."""
    out = np.zeros(world)
    for e, reps in enumerate(t):
        reps = [int(r) for r in reps if r >= 0]
        for r in reps:
            out[r] += load[e] / len(reps)
    return out


def test_no_copies_is_the_block_placement():
    t = table(8, 4, [5, 1, 0, 9, 2, 2, 7, 3], 0, 3)
    np.testing.assert_array_equal(t[:, 0], np.arange(8) // 2)
    assert (t[:, 1:] == -1).all()


def test_hand_worked_single_hot_expert():
    # E = 4 on 2 ranks, all rows on expert 0: one copy goes to rank 1 and halves it;
    # a second copy is refused (two ranks, two copies at most), and no other expert
    # carries rows, so the planner stops.
    t1 = table(4, 2, [10, 0, 0, 0], 1, 2)
    np.testing.assert_array_equal(t1, [[0, 1], [0, -1], [1, -1], [1, -1]])
    t2 = table(4, 2, [10, 0, 0, 0], 2, 2)
    np.testing.assert_array_equal(t2, t1)


def test_hand_worked_two_copies_of_one_expert():
    # E = 8 on 4 ranks (2 each), load [40, 10, 0, 0, 0, 0, 0, 10]: rank loads 50, 0,
    # 0, 10.  Copy 1: expert 0 (40 per copy) to rank 1 (0, lowest rank of the tie
    # with rank 2) -> 30, 20, 0, 10.  Copy 2: expert 0 still carries the most per
    # copy (20 > 10) -> rank 2 -> 23.3, 13.3, 13.3, 10.
    t = table(8, 4, [40, 10, 0, 0, 0, 0, 0, 10], 2, 3)
    want = np.full((8, 3), -1)
    want[:, 0] = np.arange(8) // 2
    want[0] = [0, 1, 2]
    np.testing.assert_array_equal(t, want)
    np.testing.assert_allclose(rank_loads(t, [40, 10, 0, 0, 0, 0, 0, 10], 4), [70 / 3, 40 / 3, 40 / 3, 10])


@pytest.mark.parametrize("seed", range(6))
def test_placement_properties(seed):
    rng = np.random.default_rng(seed)
    E, world, max_rep = 32, 8, 3
    load = (rng.zipf(1.3, E) * 10).astype(np.int64)
    before = rank_loads(table(E, world, load, 0, max_rep), load, world).max()
    for n_red in (1, 4, 16):
        t = table(E, world, load, n_red, max_rep)
        np.testing.assert_array_equal(t[:, 0], np.arange(E) // (E // world))   # blocks stay put
        for reps in t:
            live = [int(r) for r in reps if r >= 0]
            n = len(live)
            assert 1 <= n <= max_rep and (reps[n:] == -1).all()                 # a prefix, then -1
            assert len(set(live)) == n and all(0 <= r < world for r in live)   # distinct ranks
        assert int((t >= 0).sum()) == E + n_red                                 # every copy placed
        after = rank_loads(t, load, world).max()
        assert after <= before + 1e-9                                           # the hottest rank never gains
        before = after


def test_local_experts_are_the_held_ids_in_ascending_order():
    t = torch.tensor([[0, 1], [0, -1], [1, 0], [1, -1]], dtype=torch.int32)
    local0, n0 = abi.ep_local_experts(4, 2, 0, t)
    local1, n1 = abi.ep_local_experts(4, 2, 1, t)
    assert (n0, n1) == (3, 3)
    np.testing.assert_array_equal(local0.numpy(), [0, 1, 2, -1])
    np.testing.assert_array_equal(local1.numpy(), [0, -1, 1, 2])


@pytest.mark.parametrize("bad", [
    [[0, 0], [0, -1], [1, -1], [1, -1]],     # a rank listed twice
    [[0, 2], [0, -1], [1, -1], [1, -1]],     # a rank outside [0, world)
    [[-1, 0], [0, -1], [1, -1], [1, -1]],    # a copy after a -1
    [[-1, -1], [0, -1], [1, -1], [1, -1]],   # no copy at all
])
def test_malformed_tables_are_rejected(bad):
    with pytest.raises(MoEError):
        abi.ep_local_experts(4, 2, 0, torch.tensor(bad, dtype=torch.int32))


def test_bad_planner_arguments():
    with pytest.raises(MoEError):
        table(6, 4, [1] * 6, 1, 2)            # world does not divide E
    with pytest.raises(MoEError):
        table(4, 2, [1] * 4, 1, 0)            # max_rep < 1
    with pytest.raises(MoEError):
        table(4, 2, [1, -1, 1, 1], 1, 2)      # negative load
    with pytest.raises(MoEError):
        table(4, 2, [1] * 4, -1, 2)           # negative number of copies


def test_edges_of_the_planner():
    # All loads zero: no copy carries rows, so none is placed.
    t = table(8, 4, [0] * 8, 5, 3)
    assert (t[:, 1:] == -1).all()
    # max_rep above world: copies stop at one per rank.
    t = table(4, 2, [100, 1, 1, 1], 10, 5)
    assert sorted(int(r) for r in t[0] if r >= 0) == [0, 1]
    assert int((t >= 0).sum(1).max()) <= 2
    # One expert per rank (E = world): the hottest expert spreads over every rank first.
    t = table(4, 4, [400, 1, 1, 1], 3, 4)
    assert sorted(int(r) for r in t[0] if r >= 0) == [0, 1, 2, 3]
    # More copies asked than there is room for: every expert ends on every rank.
    t = table(4, 2, [5, 4, 3, 2], 100, 2)
    assert int((t >= 0).sum()) == 8


def test_workspace_sizes_cover_the_local_experts():
    from sparse_moe_layer_noaux_b200.workloads import V3_DECODE
    cfg = abi.MoEConfig.from_shape(V3_DECODE)
    base = abi.ep_workspace_size(cfg, 8, 128, 500)               # 32 local experts
    more = abi.ep_workspace_size(cfg, 8, 128, 500, n_local=40)   # 8 copies more
    assert more >= base > 0
    with pytest.raises(MoEError):
        abi.ep_workspace_size(cfg, 8, 128, 500, n_local=0)
    with pytest.raises(MoEError):
        abi.ep_workspace_size(cfg, 8, 128, -1)
    with pytest.raises(MoEError):
        abi.ep_workspace_size(cfg, 3, 128, 10)                   # 3 does not divide 256
