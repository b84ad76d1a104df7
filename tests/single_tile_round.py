"""One attention round whose work items are half single-tile.

Chunks of 384 tokens give three 128-row query tiles per node and head, so the
second pair of every (node, head) holds one tile. With 64 heads and the
Wan2.1 schedule (B = 7, K = 4, progressive), round 6 has 5 nodes and 640
items, about four per CTA, and single-tile items alternate with two-tile ones.

Run as a script, it writes the round's output (bf16 bits as int16) to the path
given; the library is the one WAVE_LIBRARY names, else the in-tree build.
"""
from __future__ import annotations

import math
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
for p in (HERE, os.path.dirname(HERE)):
    if p not in sys.path:
        sys.path.insert(0, p)

import numpy as np  # noqa: E402

import wave_inputs as wi  # noqa: E402
from wave_testlib import Inputs, append, make_cache, queries  # noqa: E402

WL = wi.Workload("single-tile-items", chunks=7, levels=4, heads=64, head_dim=128, tokens=384,
                 scale=1.0 / math.sqrt(128.0))
POLICY = "progressive"
ROUND = 6
PAGES = 256  # live entries x 3 pages stay well below this


def run(wave):
    """Append rounds 0..ROUND, run ROUND's attention; returns (active, inputs, O)."""
    import torch
    inp = Inputs(WL)
    kv = make_cache(wave, WL, PAGES)
    rounds = wave.schedule(WL.chunks, WL.levels, POLICY, WL.window)
    last = wave.last_read_rounds(WL.chunks, WL.levels, POLICY, WL.window)
    keep = []
    for t in range(ROUND + 1):
        keep += [append(kv, inp, n) for n in rounds[t]]
        if t < ROUND:
            for e in sorted(e for e, lr in last.items() if lr == t):
                kv.release(*e)
    active = rounds[ROUND]
    q = queries(inp, active)
    o = torch.full_like(q, float("nan"))
    kv.round_attn(active, POLICY, q, o)
    kv.status()
    torch.cuda.synchronize()
    return active, inp, o


def output_bits(o) -> np.ndarray:
    import torch
    return o.view(torch.int16).cpu().numpy()


if __name__ == "__main__":
    import block_causal_attention_wave_b200 as wave
    wave.load()
    _, _, out = run(wave)
    np.save(sys.argv[1], output_bits(out))
