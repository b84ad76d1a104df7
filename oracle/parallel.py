"""Wave Parallelism on several GPUs: node placement, one-way K/V pushes and each
rank's page tables -- oracle side (host logic only, no arithmetic on data).

TEST INFRASTRUCTURE ONLY (see the package docstring).

Sources: Wave Forcing page, "Key Findings" (full-model replicas, each running
nodes of the concurrent round; early K/V delivery) and "Wave Forcing Targets
Near-Light-Speed Video Streaming Generation" (aipulsen.com): Wave Parallelism
with one-way key-value communication. The pages give no placement rule or
protocol; readings used here:

* Placement: node (c, l) runs on rank l mod N (N ranks). With N = K + 1 every
  rank owns one denoising level, the stages of the wave: a chunk's state moves
  down the ranks and, under the progressive policy, K/V only ever moves from a
  cleaner level's rank to a noisier level's rank (one-way).
* Delivery: entry E(c, l), produced by node (c, l) in its round, is pushed in
  that same round (before the round's attention, the in-round delivery of the
  schedule) from its producer's rank to every other rank that runs a node
  reading it.
* Each rank holds the conditioning prefix and the entries its own nodes read.
  Per round its pool takes pages (lowest free id first) for the entries its
  own nodes produce, in node order, then for the entries it receives, in
  ascending (chunk, level); it releases an entry after the last round in which
  one of its own nodes reads it.
"""
from __future__ import annotations

from .cache import PREFIX, PagePoolModel
from .schedule import history_reads, node_rounds, schedule


def owner(node, n_ranks: int) -> int:
    """Rank that runs ``node``."""
    return node[1] % n_ranks


def readers(B: int, K: int, policy: str, window: int = 0):
    """Dict entry -> sorted list of the nodes that read it (its producer included)."""
    rnd = node_rounds(B, K, policy, window)
    out = {e: {e} for e in rnd}
    for node in rnd:
        for e in history_reads(node, policy, window):
            out[e].add(node)
    return {e: sorted(v) for e, v in out.items()}


def transfers(B: int, K: int, policy: str, window: int, n_ranks: int):
    """Per round, the sorted list of pushes (entry, src rank, dst rank)."""
    rounds = schedule(B, K, policy, window)
    rd = readers(B, K, policy, window)
    out = []
    for active in rounds:
        push = []
        for e in active:
            src = owner(e, n_ranks)
            for dst in sorted({owner(n, n_ranks) for n in rd[e]} - {src}):
                push.append((e, src, dst))
        out.append(sorted(push))
    return out


def rank_last_read(B: int, K: int, policy: str, window: int, n_ranks: int, rank: int):
    """Dict entry -> last round in which a node of ``rank`` reads it (entries
    the rank holds only)."""
    rnd = node_rounds(B, K, policy, window)
    last = {}
    for node, t in rnd.items():
        if owner(node, n_ranks) != rank:
            continue
        for e in [node] + history_reads(node, policy, window):
            last[e] = max(last.get(e, -1), t)
    return last


def rank_tables(B, K, policy, window, n_ranks, rank, tokens, prefix_tokens, max_pages):
    """Simulate one rank's pool through the rollout: per round, (its nodes,
    their gather tables) after that round's own appends and received pushes."""
    rounds = schedule(B, K, policy, window)
    pushes = transfers(B, K, policy, window, n_ranks)
    last = rank_last_read(B, K, policy, window, n_ranks, rank)
    pool = PagePoolModel(max_pages)
    if prefix_tokens > 0:
        pool.alloc(PREFIX, prefix_tokens)
    out = []
    for t, active in enumerate(rounds):
        mine = [n for n in active if owner(n, n_ranks) == rank]
        for n in mine:
            pool.alloc(tuple(n), tokens)
        for e in sorted(e for e, _, dst in pushes[t] if dst == rank):
            pool.alloc(tuple(e), tokens)
        out.append((mine, pool.gather(mine, policy, window, prefix_tokens > 0)))
        for e in sorted(e for e, lr in last.items() if lr == t):
            pool.release(e)
    return out
