"""Edge cases of the attention launch on the GPU, against the float64 oracle:
an empty round, chunks of a single token (one-key pages, one-row query
tiles), a single chunk (no history at all), and the limits of one launch used
in full -- WAVE_MAX_NODES (64) nodes, and a key list of exactly
WAVE_MAX_PAGES_PER_ROUND (7168) pages. Every element is compared (max-abs
1e-2, rel-L2 5e-3 per node)."""
import numpy as np
import pytest

import wave_inputs as wi

from wave_testlib import (Inputs, append, assert_close, make_cache, oracle_outputs, queries,
                          torch_to_f64)

pytestmark = pytest.mark.gpu


def test_empty_round_launches_nothing(cuda_lib):
    import torch
    wl = wi.TINY
    kv = make_cache(cuda_lib, wl, 4)
    q = torch.zeros(wl.tokens, wl.heads, wl.head_dim, dtype=torch.bfloat16, device="cuda")
    o = torch.full_like(q, 7.0)
    kv.round_attn([], "progressive", q, o)
    kv.status()
    assert torch.equal(o, torch.full_like(q, 7.0))


def _rollout_all_elements(wave, wl, pol, pages=64):
    import torch
    inp = Inputs(wl)
    kv = make_cache(wave, wl, pages)
    rounds = wave.schedule(wl.chunks, wl.levels, pol, wl.window)
    last = wave.last_read_rounds(wl.chunks, wl.levels, pol, wl.window)
    keep = []
    for t, active in enumerate(rounds):
        keep += [append(kv, inp, n) for n in active]
        q = queries(inp, active)
        o = torch.full_like(q, float("nan"))
        kv.round_attn(active, pol, q, o)
        kv.status()
        ref = oracle_outputs(inp, active, pol)
        got = torch_to_f64(o).reshape(len(active), wl.tokens, wl.heads, wl.head_dim)
        for i, n in enumerate(active):
            assert_close(got[i], ref[n], f"{wl.name} {pol} round {t} node {n}")
        for e in sorted(e for e, lr in last.items() if lr == t):
            kv.release(*e)


@pytest.mark.parametrize("pol", wi.POLICIES)
def test_one_token_chunks(cuda_lib, pol):
    """T = 1: every page holds one valid key, every query tile one row."""
    wl = wi.Workload("one-token", chunks=4, levels=2, heads=3, head_dim=64, tokens=1)
    _rollout_all_elements(cuda_lib, wl, pol)


def test_single_chunk_has_no_history(cuda_lib):
    wl = wi.Workload("one-chunk", chunks=1, levels=3, heads=2, head_dim=128, tokens=200)
    _rollout_all_elements(cuda_lib, wl, "progressive")


def test_max_nodes_in_one_launch(cuda_lib):
    """64 nodes (the limit) in one launch: chunks 0..63 at level 1 under the
    clean policy, each reading every earlier chunk's level-0 entry."""
    import torch
    wl = wi.Workload("max-nodes", chunks=64, levels=1, heads=1, head_dim=64, tokens=96)
    inp = Inputs(wl)
    kv = make_cache(cuda_lib, wl, 200)
    keep = [append(kv, inp, (c, 0)) for c in range(63)]
    active = [(c, 1) for c in range(64)]
    keep += [append(kv, inp, n) for n in active]
    q = queries(inp, active)
    o = torch.full_like(q, float("nan"))
    kv.round_attn(active, "clean", q, o)
    kv.status()
    ref = oracle_outputs(inp, active, "clean")
    got = torch_to_f64(o).reshape(64, wl.tokens, wl.heads, wl.head_dim)
    for i, n in enumerate(active):
        assert_close(got[i], ref[n], f"max-nodes node {n}")
    del keep


def test_max_pages_in_one_launch(cuda_lib):
    """One node whose key list is exactly 7168 pages (the limit): 7167 one-page
    level-0 history entries plus its own entry, 128 tokens each."""
    import torch
    n_hist = cuda_lib.MAX_PAGES_PER_ROUND - 1
    wl = wi.Workload("max-pages", chunks=n_hist + 1, levels=1, heads=1, head_dim=64, tokens=128)
    inp = Inputs(wl)
    kv = make_cache(cuda_lib, wl, n_hist + 4)
    hist = [(c, 0) for c in range(n_hist)]
    ks = [None] * n_hist
    # one batched append per 64 entries (the batch limit)
    for i in range(0, n_hist, 64):
        chunk = hist[i:i + 64]
        from wave_testlib import bits_to_torch
        kk = [bits_to_torch(inp.bits("k", *e)) for e in chunk]
        vv = [bits_to_torch(inp.bits("v", *e)) for e in chunk]
        kv.append_batch(chunk, kk, vv)
        ks[i] = (kk, vv)
    node = (n_hist, 1)
    keep = [append(kv, inp, node)]
    assert sum(len(r) for r in kv.gather_table([node], "clean")) == cuda_lib.MAX_PAGES_PER_ROUND
    q = queries(inp, [node])
    o = torch.full_like(q, float("nan"))
    kv.round_attn([node], "clean", q, o)
    kv.status()
    ref = oracle_outputs(inp, [node], "clean")
    got = torch_to_f64(o).reshape(wl.tokens, wl.heads, wl.head_dim)
    assert_close(got, ref[node], "max-pages node")
    del keep, ks
