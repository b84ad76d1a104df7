"""Pins of oracle.parallel (Wave Parallelism placement, one-way pushes, per-rank
page tables) against what fixes them independently: one rank reproduces the
single-GPU rollout tables page for page; the same-level policy needs no pushes
when every level has its own rank; the progressive policy pushes only from a
cleaner level's rank to a noisier one (the pages' one-way K/V); the clean
policy pushes only from rank 0; a brute-force check that every cross-rank read
is served by exactly one push no later than the reader's round."""
import itertools

import pytest

from oracle import cache, parallel, schedule
from oracle.schedule import history_reads, node_rounds

SHAPES = [(3, 2, 0), (5, 3, 0), (6, 4, 2), (4, 1, 0), (7, 4, 0)]


@pytest.mark.parametrize("B,K,W", SHAPES)
@pytest.mark.parametrize("policy", ["clean", "same", "progressive"])
def test_one_rank_is_the_single_gpu_rollout(B, K, W, policy):
    T, pre, pages = 300, 77, 400
    want = cache.rollout_tables(B, K, policy, W, T, pre, pages)
    got = parallel.rank_tables(B, K, policy, W, 1, 0, T, pre, pages)
    assert got == want
    assert all(not r for r in parallel.transfers(B, K, policy, W, 1))


@pytest.mark.parametrize("B,K,W", SHAPES)
def test_same_level_needs_no_pushes_with_a_rank_per_level(B, K, W):
    assert all(not r for r in parallel.transfers(B, K, "same", W, K + 1))


@pytest.mark.parametrize("B,K,W", SHAPES)
def test_progressive_pushes_one_way(B, K, W):
    pushes = [p for r in parallel.transfers(B, K, "progressive", W, K + 1) for p in r]
    assert pushes, "progressive history crosses levels"
    for (c, l), src, dst in pushes:
        assert src == l and dst > src  # from a cleaner level's rank to a noisier one


@pytest.mark.parametrize("B,K,W", SHAPES)
def test_clean_pushes_only_from_rank_zero(B, K, W):
    for r in parallel.transfers(B, K, "clean", W, K + 1):
        for e, src, dst in r:
            assert src == 0 and e[1] == 0


@pytest.mark.parametrize("B,K,W,N", [(5, 3, 0, 2), (6, 4, 2, 3), (7, 4, 0, 5), (4, 2, 1, 3)])
@pytest.mark.parametrize("policy", ["clean", "same", "progressive"])
def test_every_cross_rank_read_is_served_once_in_time(B, K, W, N, policy):
    rnd = node_rounds(B, K, policy, W)
    pushes = parallel.transfers(B, K, policy, W, N)
    when = {}
    for t, r in enumerate(pushes):
        for e, src, dst in r:
            assert (e, dst) not in when, "pushed twice"
            assert src == e[1] % N and rnd[e] == t  # pushed by its producer, in its round
            when[(e, dst)] = t
    needed = set()
    for node, t in rnd.items():
        for e in history_reads(node, policy, W):
            if e[1] % N != node[1] % N:
                needed.add((e, node[1] % N))
                assert when[(e, node[1] % N)] <= t
    assert needed == set(when)  # nothing pushed that nobody reads


@pytest.mark.parametrize("B,K,W,N", [(5, 3, 0, 4), (6, 2, 2, 3), (7, 4, 0, 2)])
@pytest.mark.parametrize("policy", ["clean", "same", "progressive"])
def test_rank_tables_cover_every_node_once_with_its_key_entries(B, K, W, N, policy):
    T, pages = 200, 600
    rounds = schedule.schedule(B, K, policy, W)
    seen = {}
    for rank in range(N):
        for t, (mine, table) in enumerate(parallel.rank_tables(B, K, policy, W, N, rank, T, 0,
                                                               pages)):
            for node, rows in zip(mine, table):
                assert node not in seen
                seen[node] = (t, rows)
                # each entry of the key list contributes its 2 pages (200 tokens)
                assert len(rows) == 2 * len(cache.key_entries(node, policy, W, False))
                assert [v for _, v in rows] == [128, 72] * (len(rows) // 2)
    assert sorted(seen) == sorted(itertools.chain.from_iterable(rounds))
    for t, active in enumerate(rounds):
        for node in active:
            assert seen[node][0] == t
