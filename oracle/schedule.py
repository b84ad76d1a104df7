"""Round schedule -- oracle side.

Sources: design-space paper (arXiv 2609.22283 summary page), Figure 2: serial
execution finishes all K updates of a chunk before the next (B*K rounds);
pipelined execution staggers chunks across levels (B+K-1 rounds) while keeping
the same B*K chunk-level updates. Wave Forcing page, "Key Findings": one output
chunk per concurrent forward round after the pipeline fills; history K/V comes
from a cache refresh (a forward pass over the clean chunk).

Reading used where the pages leave steps open:

* Nodes. Update (c, j) for chunk c = 0..B-1 and level j = K..1 turns the state
  at level j into level j-1. Refresh (c, 0) runs the clean chunk once to make
  its level-0 K/V; it exists only if some node reads E(c, 0).
* Reads. Node (c, l) reads its own entry E(c, l) and the history entries
  E(c - r, phi(l, r)) for r = 1..min(c, W) (W = 0 means unbounded).
* Delivery. E(c, l) is written by node (c, l) in its own round, before that
  round's attention, so a reader may share the producer's round.
* Constraints. round(c, l) >= round(c, l + 1) + 1 (the state chain);
  round(reader) >= round(producer); admission round(c, K) >= c (one new chunk
  enters per round -- streaming).
* Each node takes the least round meeting these (as soon as possible); within a
  round nodes are listed by ascending chunk.
"""
from __future__ import annotations

from .policy import phi


def history_reads(node, policy: str, window: int):
    """Entries (chunk, level) of earlier chunks that ``node`` reads, ascending chunk."""
    c, l = node
    span = c if window <= 0 else min(c, window)
    return [(c - r, phi(policy, l, r)) for r in range(span, 0, -1)]


def _needed_refreshes(B: int, K: int, policy: str, window: int):
    """Chunks whose level-0 entry is read by some node (fixpoint over refreshes)."""
    needed = set()
    for c in range(B):
        for j in range(K, 0, -1):
            for (cc, ll) in history_reads((c, j), policy, window):
                if ll == 0:
                    needed.add(cc)
    changed = True
    while changed:
        changed = False
        for c in sorted(needed):
            for (cc, ll) in history_reads((c, 0), policy, window):
                if ll == 0 and cc not in needed:
                    needed.add(cc)
                    changed = True
    return needed


def node_rounds(B: int, K: int, policy: str, window: int = 0):
    """Dict node -> round index under the as-soon-as-possible rule."""
    if B < 1 or K < 1:
        raise ValueError("need B >= 1 and K >= 1")
    refresh = _needed_refreshes(B, K, policy, window)
    rnd = {}
    for c in range(B):
        levels = list(range(K, 0, -1)) + ([0] if c in refresh else [])
        for l in levels:
            lo = c if l == K else rnd[(c, l + 1)] + 1
            for e in history_reads((c, l), policy, window):
                if e not in rnd:
                    raise AssertionError(f"entry {e} read by {(c, l)} has no producer")
                lo = max(lo, rnd[e])
            rnd[(c, l)] = lo
    return rnd


def schedule(B: int, K: int, policy: str, window: int = 0):
    """List of rounds; each round is a list of (chunk, level) in ascending chunk."""
    rnd = node_rounds(B, K, policy, window)
    n_rounds = max(rnd.values()) + 1
    rounds = [[] for _ in range(n_rounds)]
    for node, t in rnd.items():
        rounds[t].append(node)
    for r in rounds:
        r.sort()
    return rounds


def last_read_round(B: int, K: int, policy: str, window: int = 0):
    """Dict entry (chunk, level) -> last round in which any node reads it.

    A node reads its own entry in its own round, so every entry appears.
    """
    rnd = node_rounds(B, K, policy, window)
    last = dict(rnd)
    for node, t in rnd.items():
        for e in history_reads(node, policy, window):
            last[e] = max(last[e], t)
    return last
