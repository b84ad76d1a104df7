"""Key lists and the paged (chunk, level) K/V pool -- oracle side.

Sources: Wave Forcing page ("Key Findings": chunk-wise causal attention reads
earlier, cleaner chunks; early K/V delivery); Wan-Streamer v0.2 page (glossary
"K/V cache", "pre-sharded": incoming K/V is written into a local cache) for the
cache itself. The pages fix neither a page size nor an allocation rule; the
reading used here (and by the library) is:

* Key order of node (c, l): the conditioning prefix (if any), then the history
  entries E(c - r, phi(l, r)) by ascending chunk, then the node's own E(c, l).
* Pages hold P = 128 tokens. An entry of n tokens takes ceil(n / P) pages; the
  last one holds n - P * (ceil(n / P) - 1) valid tokens.
* Pages are taken one at a time, lowest free id first, in the order entries are
  appended. A released entry returns its pages to the free set.
* Rollout driver: the prefix is appended first; in each round the active nodes'
  entries are appended in list order, attention runs, then every entry whose
  last reading round is this one is released (the prefix never is).
"""
from __future__ import annotations

import heapq

from .schedule import history_reads, last_read_round, schedule

PAGE_TOKENS = 128
PREFIX = (-1, 0)


def key_entries(node, policy: str, window: int, has_prefix: bool):
    """Ordered cache entries whose tokens form node's key set."""
    out = [PREFIX] if has_prefix else []
    out += history_reads(node, policy, window)
    out.append(tuple(node))
    return out


def pages_for(ntokens: int) -> int:
    return (ntokens + PAGE_TOKENS - 1) // PAGE_TOKENS


class PagePoolModel:
    """Lowest-free-id-first page allocator over ``max_pages`` pages."""

    def __init__(self, max_pages: int):
        self.free = list(range(max_pages))
        heapq.heapify(self.free)
        self.entries = {}

    def alloc(self, entry, ntokens: int):
        if entry in self.entries:
            raise KeyError(f"entry {entry} already present")
        n = pages_for(ntokens)
        if n < 1 or n > len(self.free):
            raise MemoryError("out of pages")
        pages = [heapq.heappop(self.free) for _ in range(n)]
        self.entries[entry] = (pages, ntokens)
        return pages

    def release(self, entry):
        pages, _ = self.entries.pop(entry)
        for p in pages:
            heapq.heappush(self.free, p)

    def rows(self, entry):
        """(page id, valid tokens) for each page of ``entry``."""
        pages, ntok = self.entries[entry]
        out = []
        for i, p in enumerate(pages):
            valid = min(PAGE_TOKENS, ntok - i * PAGE_TOKENS)
            out.append((p, valid))
        return out

    def gather(self, active, policy: str, window: int, has_prefix: bool):
        """Per active node, the (page, valid) rows of its key list in key order."""
        table = []
        for node in active:
            rows = []
            for e in key_entries(node, policy, window, has_prefix):
                if e not in self.entries:
                    raise KeyError(f"missing K/V for entry {e} read by node {node}")
                rows += self.rows(e)
            table.append(rows)
        return table


def rollout_tables(B, K, policy, window, tokens, prefix_tokens, max_pages):
    """Simulate the rollout driver; returns [(active nodes, gather table), ...] per round."""
    rounds = schedule(B, K, policy, window)
    last = last_read_round(B, K, policy, window)
    pool = PagePoolModel(max_pages)
    if prefix_tokens > 0:
        pool.alloc(PREFIX, prefix_tokens)
    out = []
    for t, active in enumerate(rounds):
        for node in active:
            pool.alloc(tuple(node), tokens)
        out.append((list(active), pool.gather(active, policy, window, prefix_tokens > 0)))
        for e in sorted(e for e, lr in last.items() if lr == t):
            pool.release(e)
    return out
