"""Float64 CPU oracle for wave-round block-causal attention.

TEST INFRASTRUCTURE ONLY. Nothing in the product path may import this package:
only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` use it. It shares no code with the CUDA library
(``block_causal_attention_wave_b200``); the only module both sides read is
``wave_inputs`` (seeded data, no method arithmetic).

What it computes, each part written as the plain definition from the pages:

* ``policy.phi``            -- the context policy phi(j, r) (design-space paper,
                               Table 1 and Figure 1).
* ``schedule.schedule``     -- serial / pipelined rounds (design-space paper,
                               Figure 2) under the as-soon-as-possible reading.
* ``cache``                 -- key lists per (chunk, level) node and the paged
                               pool's page/valid-length tables.
* ``attention``             -- softmax(Q K^T / sqrt(d)) V over each node's key
                               list, in float64 (Wave Forcing page, "Key
                               Findings": chunk-wise causal attention over
                               earlier, cleaner chunks).
* ``projection``            -- a node's Q, K, V = X W^T split by (Q/K/V, head),
                               in float64 (the K/V of in-round delivery).
* ``block``                 -- the rest of one transformer block of a round:
                               rotary position embedding of Q and K over
                               (frame, row, column), out-projection and
                               tanh-GELU MLP with residuals, bf16 storage
                               between kernels (readings stated there).
* ``quant``                 -- FP8 (E4M3) K/V pages with per-(page, head)
                               scales and their bf16 read-back.
* ``parallel``              -- Wave Parallelism host logic: node placement on
                               ranks, one-way K/V pushes per round, and each
                               rank's page tables.

Parity pins: every function here is checked by ``tests/test_oracle_*.py``
against something other than itself (brute-force dense masks, closed forms,
torch's CPU attention, exhaustive search). Absolute attention values printed by
the pages: none exist, so that part is "parity unpinned" against the pages and
pinned only by the mathematics.
"""
from . import policy, schedule, cache, attention, projection, block, parallel, quant  # noqa: F401
