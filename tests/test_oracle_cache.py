"""Pins for the oracle's key lists and paged-pool tables (CPU only).

Expected values: closed forms for page counts and tail lengths; the allocator
rule (lowest free id first) checked on hand cases; the table's meaning checked
by writing entries page by page into a simulated pool and reading the key
sequence back through the table.
"""
import numpy as np
import pytest

from oracle import cache, schedule


@pytest.mark.parametrize("n,pages,last", [(4680, 37, 72), (984, 8, 88), (512, 4, 128),
                                          (32, 1, 32), (128, 1, 128), (129, 2, 1)])
def test_page_counts_closed_form(n, pages, last):
    pool = cache.PagePoolModel(64)
    pool.alloc((0, 1), n)
    rows = pool.rows((0, 1))
    assert len(rows) == pages
    assert rows[-1][1] == last
    assert sum(v for _, v in rows) == n


def test_lowest_free_page_first():
    pool = cache.PagePoolModel(10)
    assert pool.alloc((0, 2), 300) == [0, 1, 2]
    assert pool.alloc((1, 2), 200) == [3, 4]
    pool.release((0, 2))
    assert pool.alloc((2, 2), 129) == [0, 1]
    assert pool.alloc((3, 2), 256) == [2, 5]
    with pytest.raises(MemoryError):
        pool.alloc((4, 2), 5 * 128)
    with pytest.raises(KeyError):
        pool.alloc((1, 2), 1)


def test_missing_entry_is_an_error():
    pool = cache.PagePoolModel(10)
    pool.alloc((1, 1), 32)
    with pytest.raises(KeyError):
        pool.gather([(1, 1)], "progressive", 0, False)


@pytest.mark.parametrize("pol", ["clean", "same", "progressive"])
@pytest.mark.parametrize("W,prefix", [(0, 0), (2, 40)])
def test_table_reads_back_the_key_sequence(pol, W, prefix):
    B, K, T, P = 4, 3, 150, cache.PAGE_TOKENS
    rng = np.random.default_rng(7)
    rounds = schedule.schedule(B, K, pol, W)
    last = schedule.last_read_round(B, K, pol, W)
    pool = cache.PagePoolModel(200)
    pages = np.full((200, P), -1.0)
    data = {}

    def put(e, n):
        data[e] = rng.standard_normal(n)
        for i, p in enumerate(pool.alloc(e, n)):
            chunk = data[e][i * P:(i + 1) * P]
            pages[p, :len(chunk)] = chunk

    if prefix:
        put(cache.PREFIX, prefix)
    for t, active in enumerate(rounds):
        for n in active:
            put(n, T)
        table = pool.gather(active, pol, W, prefix > 0)
        for node, rows in zip(active, table):
            seq = np.concatenate([pages[p, :v] for p, v in rows])
            want = np.concatenate([data[e] for e in cache.key_entries(node, pol, W, prefix > 0)])
            np.testing.assert_array_equal(seq, want)
        for e in sorted(e for e, lr in last.items() if lr == t):
            pool.release(e)


def test_rollout_tables_progressive_tiny():
    # B=3, K=2, T=32: one page per entry; entries die after their last reader.
    t = cache.rollout_tables(3, 2, "progressive", 0, 32, 0, 16)
    assert [a for a, _ in t] == schedule.schedule(3, 2, "progressive")
    assert t[0][1] == [[(0, 32)]]
    assert t[1][1] == [[(0, 32)], [(0, 32), (1, 32)]]
    assert t[3][1] == [[(0, 32), (1, 32)], [(0, 32), (1, 32), (2, 32)]]


def test_window_bounds_live_pages():
    # 40 chunks, window 6, 5 levels: live level-0 entries never exceed 7.
    T = 128
    rounds = schedule.schedule(40, 5, "progressive", 6)
    last = schedule.last_read_round(40, 5, "progressive", 6)
    pool = cache.PagePoolModel(64)
    peak = 0
    for t, active in enumerate(rounds):
        for n in active:
            pool.alloc(n, T)
        pool.gather(active, "progressive", 6, False)
        peak = max(peak, len(pool.entries))
        for e in [e for e, lr in last.items() if lr == t]:
            pool.release(e)
    assert peak <= 6 + 6 + 1
