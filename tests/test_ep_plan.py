"""Host logic of expert parallelism (forward_moe_route_b200/ep.py): expert
placement, redundant copies, the dispatch plan and the receive plan.  Pure
integer work, checked exactly on the CPU against the permutation it serves."""
import numpy as np
import pytest

from forward_moe_route_b200 import ep
from oracle import moe_oracle as mo


def routing(T, N, K, seed, skew=0.0):
    rng = np.random.default_rng(seed)
    logits = rng.normal(size=(T, N)) + skew * np.log1p(np.arange(N))[None, ::-1]
    idx = np.argsort(-logits, axis=1, kind="stable")[:, :K]
    return mo.permutation(idx, N)


def test_placement_slots_and_holders():
    pl = ep.Placement(8, 4, {3: (0,), 6: (1, 2)})
    assert pl.per_rank == 2
    assert pl.slots(0) == [0, 1, 3] and pl.slots(1) == [2, 3, 6] and pl.slots(2) == [4, 5, 6]
    assert pl.slots(3) == [6, 7]
    assert pl.holders(3) == [1, 0] and pl.holders(6) == [3, 1, 2] and pl.holders(0) == [0]
    assert pl.max_slots == 3
    with pytest.raises(ValueError):
        ep.Placement(10, 4)
    with pytest.raises(ValueError):
        ep.Placement(8, 4, {3: (1,)})          # a copy on the expert's home rank
    with pytest.raises(ValueError):
        ep.Placement(8, 4, {3: (0, 0)})


@pytest.mark.parametrize("world,replicas", [(1, {}), (2, {}), (4, {}), (4, {0: (3,), 5: (0, 1)})])
def test_dispatch_plan_sends_every_row_once(world, replicas):
    T, N, K = 97, 8, 3
    counts, offsets, perm_src, slot_of = routing(T, N, K, seed=world)
    pl = ep.Placement(N, world, replicas)
    plan = ep.dispatch_plan(pl, counts, offsets, slot_of)
    R = T * K
    assert sum(plan.send_splits) == R
    # the send buffer holds every permuted row once, and row_of finds each pair's row
    assert np.array_equal(np.sort(plan.send_perm), np.arange(R))
    assert np.array_equal(plan.send_perm[plan.row_of], slot_of)
    # rows sent to q belong to the experts q holds, in q's slot order, each expert's
    # rows split between its holders in contiguous chunks that differ by at most one row
    base = 0
    for q in range(world):
        rows = plan.send_perm[base:base + plan.send_splits[q]]
        experts = np.searchsorted(offsets, rows, side="right") - 1
        want = []
        for s, j in enumerate(pl.slots(q)):
            want += [j] * int(plan.send_counts[q, s])
        assert np.array_equal(experts, want)
        base += plan.send_splits[q]
    for j in range(N):
        h = pl.holders(j)
        got = [int(plan.send_counts[q, pl.slots(q).index(j)]) for q in h]
        assert sum(got) == counts[j] and max(got) - min(got) <= 1


def test_receive_plan_groups_follow_sources_and_slots():
    pl = ep.Placement(8, 2, {1: (1,)})
    recv = np.array([[3, 0, 2, 1, 4], [0, 5, 1, 0, 2]])   # [source, slot], rank 1 has 5 slots
    rp = ep.receive_plan(pl, 1, recv)
    assert rp.recv_splits == [10, 8]
    assert rp.groups.tolist() == [[0, 3, 0, 0], [3, 2, 2, 3], [5, 1, 3, 5], [6, 4, 4, 6],
                                  [10, 5, 1, 10], [15, 1, 2, 15], [16, 2, 4, 16]]
    assert rp.slot_rows.tolist() == [3, 5, 3, 1, 6]


def received_rows(pl, plans):
    """Rows each rank's experts process, summed over the sources' plans."""
    return [sum(int(p.send_counts[q].sum()) for p in plans) for q in range(pl.world)]


def test_redundant_experts_lower_the_busiest_rank():
    # strongly skewed loads: a few experts take most rows
    world, N, K = 4, 16, 2
    shards = [routing(64, N, K, seed=10 + r, skew=3.0) for r in range(world)]
    loads = sum(s[0] for s in shards)
    plain = ep.Placement(N, world)
    before = received_rows(plain, [ep.dispatch_plan(plain, *s[:2], s[3]) for s in shards])
    rep = ep.Placement(N, world, ep.choose_replicas(loads, world, n_redundant=4))
    after = received_rows(rep, [ep.dispatch_plan(rep, *s[:2], s[3]) for s in shards])
    assert sum(before) == sum(after) == world * 64 * K
    assert max(after) < max(before)
    # the copies went to the hottest experts, never to the expert's home rank
    hot = sorted(range(N), key=lambda j: (-loads[j], j))[:4]
    assert sorted(rep.replicas) == sorted(hot)


def test_choose_replicas_ties_and_empty():
    assert ep.choose_replicas([0, 0, 0, 0], 2, 2) == {}
    assert ep.choose_replicas([5, 5, 1, 1], 2, 1) == {0: (1,)}
    assert ep.chunk_bounds(7, 3) == [0, 2, 4, 7] and ep.chunk_bounds(0, 2) == [0, 0, 0]
