"""Host side of the peer-memory exchange (forward_moe_route_b200/ep.py):
peer_offsets and peer_return_rows must place every row where the uneven
all-to-all of the collective path puts it, and send every expert output back
to the send-order row it came from.  Checked against a direct simulation of
the all-to-all (concatenation by source rank) on random send matrices,
including empty blocks and ranks that send or receive nothing."""
import numpy as np
import pytest

from forward_moe_route_b200 import ep


def random_matrix(rng, W, S, slots_of, p_zero):
    M = rng.integers(0, 6, size=(W, W, S))
    M[rng.random((W, W, S)) < p_zero] = 0
    for q in range(W):
        M[:, q, slots_of[q]:] = 0     # rank q has slots_of[q] local slots
    return M


def simulate_all_to_all(M):
    """recv[q] = list of (source, send-order row) in arrival order."""
    W = M.shape[0]
    recv = [[] for _ in range(W)]
    for q in range(W):
        for s in range(W):
            first = int(M[s, :q].sum())
            recv[q] += [(s, first + i) for i in range(int(M[s, q].sum()))]
    return recv


@pytest.mark.parametrize("W,seed,p_zero", [(1, 0, 0.0), (2, 1, 0.2), (4, 2, 0.5), (8, 3, 0.3),
                                           (3, 4, 0.9)])
def test_peer_offsets_match_the_all_to_all(W, seed, p_zero):
    rng = np.random.default_rng(seed)
    S = 3
    slots_of = [int(v) for v in rng.integers(1, S + 1, size=W)]
    M = random_matrix(rng, W, S, slots_of, p_zero)
    recv = simulate_all_to_all(M)
    placed = [dict() for _ in range(W)]
    for s in range(W):
        start, base = ep.peer_offsets(M, s)
        assert start[0] == 0 and start[-1] == int(M[s].sum())
        for q in range(W):
            for p in range(start[q], start[q + 1]):
                row = base[q] + p - start[q]
                assert row not in placed[q], "two rows land on one receive row"
                placed[q][row] = (s, p)
    for q in range(W):
        assert [placed[q][i] for i in range(len(recv[q]))] == recv[q]
        assert len(placed[q]) == len(recv[q])


class _Pl:
    """The slots of a placement, for receive_plan."""
    def __init__(self, slots_of):
        self.world = len(slots_of)
        self._n = slots_of

    def slots(self, r):
        return list(range(self._n[r]))


@pytest.mark.parametrize("W,seed,p_zero", [(2, 5, 0.2), (4, 6, 0.5), (8, 7, 0.3), (3, 8, 0.9)])
def test_peer_return_rows_go_back_to_their_source_rows(W, seed, p_zero):
    rng = np.random.default_rng(seed)
    S = 4
    slots_of = [int(v) for v in rng.integers(1, S + 1, size=W)]
    M = random_matrix(rng, W, S, slots_of, p_zero)
    recv = simulate_all_to_all(M)
    pl = _Pl(slots_of)
    for r in range(W):
        plan = ep.receive_plan(pl, r, M[:, r, :])
        back = ep.peer_return_rows(M, r, plan)
        assert len(back) == len(plan.groups)
        covered = 0
        for (row0, rows, slot, out0), (s, row) in zip(plan.groups, back):
            for i in range(rows):
                assert recv[r][row0 + i] == (s, row + i)
            covered += rows
        assert covered == len(recv[r])
