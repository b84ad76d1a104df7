"""Pins for the oracle's policy and round scheduler (CPU only).

What fixes the expected values here (not the oracle itself):
* hand-written phi values (tests/golden/phi_table.txt) from the design-space
  paper's Table 1 / Figure 1;
* hand-derived tiny schedules (tests/golden/schedule_tiny.txt);
* the closed forms of the design-space paper's Figure 2: B+K-1 pipelined
  rounds, B*K serial rounds, B*K updates either way;
* an independent legality checker plus an exhaustive minimum-makespan search on
  tiny cases.
"""
import itertools
import os

import pytest

from oracle import policy, schedule

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden_lines(name):
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                yield line


def test_phi_golden():
    n = 0
    for line in _golden_lines("phi_table.txt"):
        pol, j, r, want = line.split()
        assert policy.phi(pol, int(j), int(r)) == int(want), line
        n += 1
    assert n >= 20


def test_phi_rejects_own_chunk_and_unknown_policy():
    with pytest.raises(ValueError):
        policy.phi("progressive", 2, 0)
    with pytest.raises(ValueError):
        policy.phi("bogus", 1, 1)


def test_schedule_tiny_golden():
    want = {}
    for line in _golden_lines("schedule_tiny.txt"):
        head, rest = line.split(":")
        pol, rnd = head.split()
        nodes = [tuple(int(x) for x in tok.split(",")) for tok in rest.split()]
        want.setdefault(pol, {})[int(rnd)] = nodes
    for pol, rounds in want.items():
        got = schedule.schedule(3, 2, pol)
        assert len(got) == len(rounds), pol
        for t, nodes in rounds.items():
            assert got[t] == nodes, (pol, t)


@pytest.mark.parametrize("B", [1, 2, 3, 5, 7, 9])
@pytest.mark.parametrize("K", [1, 2, 3, 4, 5])
def test_round_counts_closed_form(B, K):
    # design-space paper, Figure 2: pipelined B+K-1 rounds, serial B*K rounds,
    # the same B*K chunk-level updates in both.
    for pol, want in (("progressive", B + K - 1), ("same", B + K - 1), ("clean", B * K)):
        rounds = schedule.schedule(B, K, pol)
        assert len(rounds) == want, (pol, B, K)
        updates = [n for r in rounds for n in r if n[1] > 0]
        assert sorted(updates) == sorted((c, j) for c in range(B) for j in range(1, K + 1))
        for r in rounds:
            assert sum(1 for n in r if n[1] > 0) <= K
            assert len({n[0] for n in r}) == len(r), "one node per chunk per round"


@pytest.mark.parametrize("pol", ["progressive", "same", "clean"])
def test_updates_of_a_chunk_are_consecutive(pol):
    rnd = schedule.node_rounds(6, 4, pol)
    for c in range(6):
        rs = [rnd[(c, j)] for j in range(4, 0, -1)]
        assert rs == list(range(rs[0], rs[0] + 4))


def test_pipelined_rounds_closed_form_per_node():
    # progressive and same-level: chunk c at level j runs in round c + K - j.
    for pol in ("progressive", "same"):
        rnd = schedule.node_rounds(7, 4, pol)
        for (c, l), t in rnd.items():
            if l > 0:
                assert t == c + 4 - l
    # clean: chunk c starts in the round of the refresh of chunk c - 1.
    rnd = schedule.node_rounds(7, 4, "clean")
    for c in range(1, 7):
        assert rnd[(c, 4)] == rnd[(c - 1, 0)]


def test_one_output_chunk_per_round_after_fill():
    # Wave Forcing page, "Key Findings": one output chunk per concurrent round
    # after the pipeline fills (K=1 included).
    for K in (1, 2, 4):
        rounds = schedule.schedule(8, K, "progressive")
        finished = [sum(1 for n in r if n[1] == 1) for r in rounds]
        assert finished[K - 1:] == [1] * (len(rounds) - K + 1)


def test_workload_node_counts():
    r = schedule.schedule(7, 4, "progressive")
    assert len(r) == 10
    assert r[6] == [(2, 0), (3, 1), (4, 2), (5, 3), (6, 4)]
    assert sum(1 for x in r for n in x if n[1] == 0) == 6
    r = schedule.schedule(40, 5, "progressive", 6)
    assert len(r) == 44
    assert sum(1 for x in r for n in x if n[1] > 0) == 200
    assert sum(1 for x in r for n in x if n[1] == 0) == 39


# ---------------------------------------------------------------- brute force

def _reads(node, pol, W):
    """History entries read by node, as a predicate over all earlier chunks."""
    c, l = node
    out = []
    for cc in range(c):
        r = c - cc
        if W > 0 and r > W:
            continue
        out.append((cc, policy.phi(pol, l, r)))
    return out


def _node_set(B, K, pol, W):
    nodes = {(c, j) for c in range(B) for j in range(1, K + 1)}
    while True:
        extra = {e for n in nodes for e in _reads(n, pol, W) if e[1] == 0} - nodes
        if not extra:
            return nodes
        nodes |= extra


def _legal(assign, B, K, pol, W):
    for (c, l), t in assign.items():
        if l == K and t < c:
            return False
        if l < K and t < assign[(c, l + 1)] + 1:
            return False
        for e in _reads((c, l), pol, W):
            if e not in assign or assign[e] > t:
                return False
    return True


def _min_makespan(B, K, pol, W):
    nodes = sorted(_node_set(B, K, pol, W), key=lambda n: (n[0], -n[1]))
    for M in range(1, B * (K + 1) + 1):
        assign = {}

        def dfs(i):
            if i == len(nodes):
                return True
            c, l = nodes[i]
            for t in range(M):
                assign[(c, l)] = t
                ok = (l != K or t >= c) and (l == K or t >= assign[(c, l + 1)] + 1)
                ok = ok and all(e in assign and assign[e] <= t for e in _reads((c, l), pol, W))
                if ok and dfs(i + 1):
                    return True
                del assign[(c, l)]
            return False

        if dfs(0):
            return M
    raise AssertionError("no legal schedule")


@pytest.mark.parametrize("B,K", list(itertools.product([1, 2, 3], [1, 2, 3])))
@pytest.mark.parametrize("pol", ["progressive", "same", "clean"])
@pytest.mark.parametrize("W", [0, 1])
def test_schedule_is_legal_and_minimal(B, K, pol, W):
    rnd = schedule.node_rounds(B, K, pol, W)
    assert set(rnd) == _node_set(B, K, pol, W)
    assert _legal(rnd, B, K, pol, W)
    assert max(rnd.values()) + 1 == _min_makespan(B, K, pol, W)


def test_legality_checker_catches_a_planted_error():
    rnd = dict(schedule.node_rounds(3, 2, "progressive"))
    rnd[(1, 2)] = 0  # before its history (0, 1) is produced
    assert not _legal(rnd, 3, 2, "progressive", 0)
