"""Policy and level sweep: rounds, attention FLOPs per chunk and peak cache bytes.

For each context policy (design-space paper, Table 1 / Figure 1) and each
number of levels K, runs the library's scheduler and page allocator on a
host-only handle (no GPU) through a whole rollout and reports:

* rounds (design-space paper, Figure 2: B+K-1 pipelined, B*K serial);
* update and refresh nodes;
* attention FLOPs per chunk, 4 * T * N_keys * H * d summed over the chunk's
  nodes (updates and, separately, its refresh);
* the peak number of cached entries and pages held at once, and their bytes
  per layer.

Usage: ``python -m block_causal_attention_wave_b200.sweep`` (Wan2.1-shaped:
7 chunks of 4680 tokens, 12 heads, d = 128).
"""
from __future__ import annotations

import json
import sys

from ._binding import PAGE_TOKENS, KVCache, last_read_rounds, schedule

POLICY_NAMES = ("clean", "same", "progressive")


def sweep_one(B, K, policy, tokens, heads, head_dim, window=0):
    rounds = schedule(B, K, policy, window)
    last = last_read_rounds(B, K, policy, window)
    pages_per_entry = (tokens + PAGE_TOKENS - 1) // PAGE_TOKENS
    n_entries_max = B * (K + 1)
    pool_pages = n_entries_max * pages_per_entry
    kv = KVCache(heads, head_dim, tokens, K, window, 0, pool=None,
                 pool_bytes=4096 + pool_pages * KVCache.page_bytes(heads, head_dim))
    upd_flops = [0] * B
    ref_flops = [0] * B
    live, peak_entries, peak_pages = set(), 0, 0
    for t, active in enumerate(rounds):
        for n in active:
            kv.alloc(*n)
            live.add(n)
        table = kv.gather_table(active, policy)
        for (c, l), rows in zip(active, table):
            n_keys = sum(v for _, v in rows)
            f = 4 * tokens * n_keys * heads * head_dim
            if l > 0:
                upd_flops[c] += f
            else:
                ref_flops[c] += f
        peak_entries = max(peak_entries, len(live))
        peak_pages = max(peak_pages, len(live) * pages_per_entry)
        for e in sorted(e for e, lr in last.items() if lr == t):
            kv.release(*e)
            live.discard(e)
    page_bytes = KVCache.page_bytes(heads, head_dim)
    return {
        "policy": policy, "K": K, "rounds": len(rounds),
        "updates": sum(1 for r in rounds for n in r if n[1] > 0),
        "refreshes": sum(1 for r in rounds for n in r if n[1] == 0),
        "update_tflop_per_chunk": [round(f / 1e12, 4) for f in upd_flops],
        "refresh_tflop_per_chunk": [round(f / 1e12, 4) for f in ref_flops],
        "peak_entries": peak_entries,
        "peak_cache_bytes_per_layer": peak_pages * page_bytes,
    }


def sweep(B=7, levels=(1, 2, 3, 4, 5), tokens=4680, heads=12, head_dim=128, window=0):
    return [sweep_one(B, K, pol, tokens, heads, head_dim, window)
            for pol in POLICY_NAMES for K in levels]


def main(argv=None):
    rows = sweep()
    for r in rows:
        print(json.dumps(r))
    return 0


if __name__ == "__main__":
    sys.exit(main())
