"""Wave Parallelism driver: one node per rank, one-way K/V page pushes.

Argument marshalling and message passing only. The placement (node (c, l) on
rank l mod N), each round's pushes and each rank's release rounds come from
libwave (wave_wp_transfers, wave_wp_rank_last_read); the pages move with
torch.distributed point-to-point operations -- NCCL over NVLink between GPUs,
gloo between CPU processes -- straight from the producer's pool pages into the
pages the receiver has just taken for the entry, so no append kernel runs on
the receiving side (Wave Forcing page, "Key Findings": early K/V delivery;
"Wave Forcing Targets Near-Light-Speed Video Streaming Generation": one-way
key-value communication between replicas).
"""
from __future__ import annotations

from ._binding import schedule, wp_rank_last_read, wp_transfers


class WaveParallel:
    """One rank's view of a Wave-Parallel rollout.

    ``kv`` is this rank's KVCache; ``pool`` the byte tensor holding its pages
    (the device pool, or for a host-only handle a host tensor laid out the
    same way). Per round the caller appends the entries of ``own_nodes(t)``
    (wave_kv_append, wave_qkv_append or wave_qkv_append_round), then calls
    ``exchange(t)``, runs the attention of its nodes, and calls ``release(t)``.
    """

    def __init__(self, kv, pool, B, K, policy, window, rank, world, group=None):
        self.kv, self.pool = kv, pool
        self.B, self.K, self.policy, self.window = B, K, policy, window
        self.rank, self.world, self.group = rank, world, group
        self.rounds = schedule(B, K, policy, window)
        mine = sorted({e for t in range(len(self.rounds)) for e in self._held(t)})
        self.last = wp_rank_last_read(B, K, policy, window, world, rank, mine)

    def _held(self, t):
        own = self.own_nodes(t)
        got = [e for e, _, dst in wp_transfers(self.B, self.K, self.policy, self.window,
                                                self.world, t) if dst == self.rank]
        return [tuple(n) for n in own] + got

    def own_nodes(self, t):
        """The nodes of round t that run on this rank, ascending chunk."""
        return [n for n in self.rounds[t] if n[1] % self.world == self.rank]

    def _page(self, page):
        page_bytes, off, _ = self.kv.layout()
        return self.pool[off + page * page_bytes:off + (page + 1) * page_bytes]

    def exchange(self, t):
        """Push this rank's new entries of round t to the ranks that read them
        and take in the entries pushed to it (pages taken in ascending
        (chunk, level)); returns the received entries."""
        import torch.distributed as dist
        pushes = wp_transfers(self.B, self.K, self.policy, self.window, self.world, t)
        incoming = sorted({e for e, _, dst in pushes if dst == self.rank})
        for e in incoming:
            self.kv.alloc(*e)
        # NCCL moves device pages directly; a backend without device support
        # (gloo) gets host copies of them.
        staged = self.pool.is_cuda and dist.get_backend(self.group) != "nccl"
        reqs, landing = [], []
        if staged:
            import torch
            torch.cuda.current_stream().synchronize()  # the appends wrote the pages
        for e, src, dst in pushes:  # the same order on every rank
            if src == self.rank:
                for p in self.kv.entry_pages(*e):
                    buf = self._page(p).cpu() if staged else self._page(p)
                    reqs.append((dist.isend(buf, dst, group=self.group), buf))
            elif dst == self.rank:
                for p in self.kv.entry_pages(*e):
                    if staged:
                        buf = self._page(p).new_empty(self._page(p).shape, device="cpu")
                        landing.append((p, buf))
                    else:
                        buf = self._page(p)
                    reqs.append((dist.irecv(buf, src, group=self.group), buf))
        for r, _ in reqs:
            r.wait()
        for p, buf in landing:
            self._page(p).copy_(buf)
        return incoming

    def release(self, t):
        """Release the entries whose last reader on this rank ran in round t."""
        for e in sorted(e for e, lr in self.last.items() if lr == t):
            self.kv.release(*e)
