"""GPU parity of the split-KV attention (wave_round_attn_split): each node's
key list cut into page ranges whose partial results a second kernel combines.

Every element against the float64 oracle on small cases that split key lists
into 2, 3 and 7 ranges (ranges of unequal length, a node with fewer pages than
ranges, prefix, window, d 64 and 128, ragged query and key tails); sampled rows
of a Wan-Streamer steady round with the automatic range count; one range gives
exactly wave_round_attn's bytes; a missing or small workspace is refused. Bar
as elsewhere: max-abs <= 1e-2, rel-L2 <= 5e-3 per node.
"""
import pytest

import wave_inputs as wi
from oracle import cache as ocache
from oracle import schedule as osched

from wave_testlib import (Inputs, append, assert_close, make_cache, oracle_outputs, queries,
                          torch_to_f64)

pytestmark = pytest.mark.gpu

CASES = [
    wi.Workload("split-d128-prefix", chunks=5, levels=2, heads=3, head_dim=128, tokens=300,
                prefix=77),
    wi.Workload("split-d64-window", chunks=6, levels=3, heads=2, head_dim=64, tokens=200,
                window=2),
    wi.Workload("split-d128-k1", chunks=4, levels=1, heads=2, head_dim=128, tokens=129),
]


def _round(wave, wl, pages=200):
    pol = "progressive"
    inp = Inputs(wl)
    rounds = osched.schedule(wl.chunks, wl.levels, pol, wl.window)
    active = max(rounds, key=lambda r: (len(r), r[-1][0]))
    entries = set()
    for n in active:
        entries.update(e for e in ocache.key_entries(n, pol, wl.window, wl.prefix > 0))
    kv = make_cache(wave, wl, pages)
    keep = [append(kv, inp, e) for e in sorted(entries)]
    return kv, inp, active, pol, keep


@pytest.mark.parametrize("splits", [2, 3, 7])
@pytest.mark.parametrize("wl", CASES, ids=lambda w: w.name)
def test_split_every_element(cuda_lib, wl, splits):
    import torch
    kv, inp, active, pol, keep = _round(cuda_lib, wl)
    nbytes, used = kv.split_workspace(active, pol, splits)
    assert used == splits and nbytes > 0
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    q = queries(inp, active)
    o = torch.full_like(q, float("nan"))
    kv.round_attn_split(active, pol, q, o, ws, splits)
    kv.status()
    ref = oracle_outputs(inp, active, pol)
    got = torch_to_f64(o).reshape(len(active), wl.tokens, wl.heads, wl.head_dim)
    for i, n in enumerate(active):
        assert_close(got[i], ref[n], f"{wl.name} splits {splits} node {n}")
    del keep


def test_one_range_is_wave_round_attn(cuda_lib):
    import torch
    wl = CASES[0]
    kv, inp, active, pol, keep = _round(cuda_lib, wl)
    assert kv.split_workspace(active, pol, 1) == (0, 1)
    q = queries(inp, active)
    o1, o2 = torch.empty_like(q), torch.empty_like(q)
    kv.round_attn(active, pol, q, o1)
    kv.round_attn_split(active, pol, q, o2, None, 1)
    kv.status()
    assert torch.equal(o1, o2)
    del keep


def test_workspace_is_checked(cuda_lib):
    import torch
    wave = cuda_lib
    wl = CASES[0]
    kv, inp, active, pol, keep = _round(wave, wl)
    nbytes, _ = kv.split_workspace(active, pol, 3)
    q = queries(inp, active)
    o = torch.empty_like(q)
    with pytest.raises(wave.WaveError):
        kv.round_attn_split(active, pol, q, o, None, 3)
    small = torch.empty(nbytes - 16, dtype=torch.uint8, device="cuda")
    with pytest.raises(wave.WaveError):
        kv.round_attn_split(active, pol, q, o, small, 3)
    del keep


def test_wan_streamer_round_auto_splits_sampled_rows(cuda_lib):
    """A Wan-Streamer-shaped round with one update node (984-token unit, 24
    heads, 512-token prefix, 32-unit window): 96 work items, so the automatic
    count splits the 268-page key list; sampled rows of every head."""
    import numpy as np
    import torch
    wl = wi.WAN_STREAMER
    pol = "progressive"
    inp = Inputs(wl)
    node = (35, 2)
    entries = [e for e in ocache.key_entries(node, pol, wl.window, True)]
    kv = make_cache(cuda_lib, wl, 300)
    keep = [append(kv, inp, e) for e in entries]
    active = [node]
    nbytes, used = kv.split_workspace(active, pol, 0)
    assert used > 1
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    q = queries(inp, active)
    o = torch.empty_like(q)
    kv.round_attn_split(active, pol, q, o, ws, 0)
    kv.status()
    rows = np.unique(np.concatenate([np.linspace(0, wl.tokens - 1, 40).astype(int),
                                     [127, 128, 895, 896, wl.tokens - 1]]))
    ref = oracle_outputs(inp, active, pol, {node: rows})
    got = torch_to_f64(o).reshape(wl.tokens, wl.heads, wl.head_dim)[rows]
    assert_close(got, ref[node], f"wan-streamer split {used}")
    del keep
