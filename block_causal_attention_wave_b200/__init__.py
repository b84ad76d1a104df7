"""Wave-round block-causal attention for B200 (sm_100a).

The library (``libwave.so``, C ABI in ``include/wave.h``) holds the round
scheduler, the paged (chunk, level) K/V cache with its append kernel, and the
tcgen05/TMA attention kernel that runs every active node of a round in one
launch. This package is its thin ctypes binding.
"""
from ._binding import (  # noqa: F401
    KVCache, Node, WaveError, load, schedule, last_read_rounds, exported_symbols,
    wp_transfers, wp_rank_last_read,
    POLICIES, PAGE_TOKENS, ACT_NONE, ACT_GELU_TANH, KV_BF16, KV_FP8_E4M3, PREFIX_CHUNK, MAX_NODES, MAX_PAGES_PER_ROUND, LIB_PATH,
)
