"""GPU parity: libwave.so's append and attention kernels vs the float64 oracle.

Every test here runs the CUDA path through the C ABI and compares with the
oracle on the same seeded bf16 inputs: element by element on small cases that
span several query tiles, several pages and ragged tails; on sampled query rows
at the full workload sizes (Wan2.1 round, Wan-Streamer unit, long rollout).
Bar: max-abs <= 1e-2 and relative L2 <= 5e-3 per node; gather tables and the
appended page bytes bit-exact.
"""
import dataclasses

import numpy as np
import pytest

import wave_inputs as wi
from oracle import cache as ocache
from oracle import schedule as osched

from wave_testlib import (Inputs, append, assert_close, bits_to_torch, make_cache, oracle_outputs,
                          queries, torch_to_f64)

pytestmark = pytest.mark.gpu


def _rollout_and_check(wave, wl, pol, check_rounds=None, rows_per_node=None, pages=4000,
                       batch=False):
    """Drive a full rollout through the library; check outputs and tables.
    With batch=True each round's entries go through one batched append."""
    import torch
    inp = Inputs(wl)
    kv = make_cache(wave, wl, pages)
    rounds = wave.schedule(wl.chunks, wl.levels, pol, wl.window)
    last = wave.last_read_rounds(wl.chunks, wl.levels, pol, wl.window)
    want_tables = ocache.rollout_tables(wl.chunks, wl.levels, pol, wl.window, wl.tokens,
                                        wl.prefix, kv.layout()[2])
    if wl.prefix:
        append(kv, inp, (-1, 0))
    keep = []
    results = []
    for t, active in enumerate(rounds):
        if batch:
            ks = [bits_to_torch(inp.bits("k", *n)) for n in active]
            vs = [bits_to_torch(inp.bits("v", *n)) for n in active]
            kv.append_batch(active, ks, vs)
            keep.append((ks, vs))
        for n in ([] if batch else active):
            keep.append(append(kv, inp, n))
        assert kv.gather_table(active, pol) == want_tables[t][1], f"round {t} table"
        if check_rounds is None or t in check_rounds:
            q = queries(inp, active)
            o = torch.empty_like(q)
            kv.round_attn(active, pol, q, o)
            kv.status()
            rows = None
            if rows_per_node is not None:
                rows = {n: rows_per_node for n in active}
            ref = oracle_outputs(inp, active, pol, rows)
            got = torch_to_f64(o).reshape(len(active), wl.tokens, wl.heads, wl.head_dim)
            for i, n in enumerate(active):
                g = got[i] if rows is None else got[i][rows[n]]
                results.append(assert_close(g, ref[n], f"{wl.name} {pol} round {t} node {n}"))
        for e in sorted(e for e, lr in last.items() if lr == t):
            kv.release(*e)
    torch.cuda.synchronize()
    return results


@pytest.mark.parametrize("pol", wi.POLICIES)
def test_tiny_all_rounds(cuda_lib, pol):
    """Tiny case: 3 chunks, 2 levels, 2 heads, d 64, 32 tokens; every round."""
    _rollout_and_check(cuda_lib, wi.TINY, pol)


SMALL = [
    wi.Workload("small-d128", chunks=4, levels=3, heads=3, head_dim=128, tokens=300),
    wi.Workload("small-d64-prefix-window", chunks=5, levels=2, heads=2, head_dim=64, tokens=260,
                window=2, prefix=200),
    wi.Workload("small-d128-prefix", chunks=3, levels=2, heads=2, head_dim=128, tokens=128,
                prefix=77),
    wi.Workload("small-k1", chunks=4, levels=1, heads=2, head_dim=128, tokens=129),
]


@pytest.mark.parametrize("wl", SMALL, ids=lambda w: w.name)
@pytest.mark.parametrize("pol", wi.POLICIES)
def test_small_multi_tile_ragged(cuda_lib, wl, pol):
    """Several query tiles and pages with ragged tails; every round, every element."""
    _rollout_and_check(cuda_lib, wl, pol)


def test_append_bytes_exact(cuda_lib):
    """Pages hold exactly the appended K/V in [H][128][d] order, tail zero."""
    import torch
    wl = wi.Workload("append", chunks=2, levels=1, heads=3, head_dim=128, tokens=300)
    inp = Inputs(wl)
    kv = make_cache(cuda_lib, wl, 16)
    kv.alloc(0, 1)  # occupy pages 0..2 so the appended entry starts at page 3
    append(kv, inp, (1, 1))
    (rows,) = kv.gather_table([(1, 1)], "same")
    torch.cuda.synchronize()
    page_bytes, off, _ = kv.layout()
    pool = kv.pool.cpu().numpy()
    tail = 1
    for kind, kvi in (("k", 0), ("v", 1)):
        src = inp.bits(kind, 1, 1)  # [T][H][d]
        for pi, (page, valid) in enumerate(rows[-3:]):
            base = off + page * page_bytes + kvi * wl.heads * 128 * wl.head_dim * 2
            blk = pool[base:base + wl.heads * 128 * wl.head_dim * 2].view(np.uint16)
            blk = blk.reshape(wl.heads, 128, wl.head_dim)
            want = np.zeros_like(blk)
            n = min(128, wl.tokens - pi * 128)
            want[:, :n, :] = src[pi * 128:pi * 128 + n].transpose(1, 0, 2)
            np.testing.assert_array_equal(blk, want)
            tail = valid
    assert tail == 300 - 256


@pytest.mark.parametrize("pol", ["progressive", "clean"])
def test_wan21_round6_sampled_rows(cuda_lib, pol):
    """Full Wan2.1-shaped round (12 heads, d 128, 4680 tokens), sampled query rows."""
    wl = wi.WAN21
    rounds = osched.schedule(wl.chunks, wl.levels, pol)
    t_check = 6 if pol == "progressive" else 10
    rows = np.array([0, 1, 127, 128, 1000, 2047, 2048, 3333, 4607, 4608, 4650, 4679])
    res = _rollout_and_check(cuda_lib, wl, pol, check_rounds={t_check}, rows_per_node=rows,
                             pages=1200)
    assert len(res) == len(rounds[t_check])


def _one_round(wave, wl, pol, t, rows):
    """Append just what round t reads, run it, compare sampled rows."""
    import torch
    inp = Inputs(wl)
    rounds = osched.schedule(wl.chunks, wl.levels, pol, wl.window)
    active = rounds[t]
    needed = set()
    for n in active:
        needed.update(ocache.key_entries(n, pol, wl.window, wl.prefix > 0))
    per_entry = ocache.pages_for(max(wl.tokens, wl.prefix))
    kv = make_cache(wave, wl, len(needed) * per_entry + 8)
    keep = [append(kv, inp, e) for e in sorted(needed)]
    q = queries(inp, active)
    o = torch.empty_like(q)
    kv.round_attn(active, pol, q, o)
    kv.status()
    ref = oracle_outputs(inp, active, pol, {n: rows for n in active})
    got = torch_to_f64(o).reshape(len(active), wl.tokens, wl.heads, wl.head_dim)
    del keep
    return [assert_close(got[i][rows], ref[n], f"{wl.name} round {t} node {n}")
            for i, n in enumerate(active)]


def test_wan_streamer_steady_round(cuda_lib):
    """Wan-Streamer-shaped unit: 24 heads, 984 tokens, 512 prefix, 32-unit window."""
    rows = np.array([0, 5, 127, 128, 500, 895, 896, 983])
    res = _one_round(cuda_lib, wi.WAN_STREAMER, "progressive", 35, rows)
    assert len(res) == 3


def test_long_rollout_steady_round(cuda_lib):
    """40 chunks x 4680 tokens, window 6, 5 levels: a steady-state round."""
    rows = np.array([0, 77, 128, 2500, 4608, 4679])
    res = _one_round(cuda_lib, wi.LONG_ROLLOUT, "progressive", 20, rows)
    assert len(res) == 6


def test_same_level_max_growth_rescales(cuda_lib):
    """Scores that grow along the key list force the O rescale path."""
    import torch
    wl = wi.Workload("growth", chunks=3, levels=1, heads=2, head_dim=128, tokens=256)
    inp = Inputs(wl)
    # Scale each entry's K by a growing factor so later pages carry larger scores.
    for c, f in ((0, 0.25), (1, 1.0), (2, 4.0)):
        kb = inp.bits("k", c, 1)
        kf = wi.bf16_bits_to_f64(kb) * f
        inp._bits[("k", c, 1)] = wi.f32_to_bf16_bits(kf.astype(np.float32))
    kv = make_cache(cuda_lib, wl, 32)
    keep = [append(kv, inp, (c, 1)) for c in range(3)]
    active = [(2, 1)]
    q = queries(inp, active)
    o = torch.empty_like(q)
    kv.round_attn(active, "same", q, o)
    kv.status()
    ref = oracle_outputs(inp, active, "same")
    assert float(np.abs(ref[(2, 1)]).max()) > 1.0  # outputs well above 1: bf16 ulp matters
    assert_close(torch_to_f64(o), ref[(2, 1)], "growth", scale_with_output=True)
    del keep


def test_missing_kv_is_reported_before_launch(cuda_lib):
    import torch
    wl = wi.TINY
    kv = make_cache(cuda_lib, wl, 8)
    inp = Inputs(wl)
    keep = append(kv, inp, (1, 2))
    q = queries(inp, [(1, 2)])
    with pytest.raises(cuda_lib.WaveError) as e:
        kv.round_attn([(1, 2)], "progressive", q, torch.empty_like(q))
    assert e.value.code == -2
    kv.status()
    del keep


def test_duplicate_and_single_nodes(cuda_lib):
    """The same node twice in one launch gives the same rows twice."""
    import torch
    wl = dataclasses.replace(wi.TINY, tokens=200, head_dim=128)
    inp = Inputs(wl)
    kv = make_cache(cuda_lib, wl, 16)
    keep = [append(kv, inp, e) for e in ((0, 0), (1, 1))]
    active = [(1, 1), (1, 1)]
    q = queries(inp, active)
    o = torch.empty_like(q)
    kv.round_attn(active, "progressive", q, o)
    kv.status()
    assert torch.equal(o[:200], o[200:])
    ref = oracle_outputs(inp, [(1, 1)], "progressive")
    assert_close(torch_to_f64(o[:200]), ref[(1, 1)], "dup")
    del keep


def test_wan21_same_level_round_sampled_rows(cuda_lib):
    """Same-level policy at the Wan2.1 shapes: history read at the node's own level."""
    rows = np.array([0, 129, 2222, 4607, 4679])
    res = _one_round(cuda_lib, wi.WAN21, "same", 6, rows)
    assert len(res) == 4  # (3,4)...: same-level round 6 has no refresh


def test_long_rollout_clean_round_sampled_rows(cuda_lib):
    """Clean policy, 40 chunks x 4680 tokens, window 6, 5 levels: a late round."""
    rows = np.array([0, 4000, 4679])
    rounds = osched.schedule(wi.LONG_ROLLOUT.chunks, wi.LONG_ROLLOUT.levels, "clean", 6)
    res = _one_round(cuda_lib, wi.LONG_ROLLOUT, "clean", len(rounds) - 5, rows)
    assert len(res) == len(rounds[len(rounds) - 5])


def test_capacity_and_alignment_errors_before_launch(cuda_lib):
    """Rounds beyond one launch's tables, and misaligned Q, fail cleanly."""
    import torch
    wl = wi.Workload("cap", chunks=8000, levels=1, heads=1, head_dim=64, tokens=128)
    kv = make_cache(cuda_lib, wl, 7300)
    # 7200 cached level-0 history entries (reserved, not written) + the node's own:
    # chunk 7200 at level 1 reads 7201 one-page entries > 7168 pages per launch.
    for c in range(7200):
        kv.alloc(c, 0)
    kv.alloc(7200, 1)
    q = torch.zeros(128, 1, 64, dtype=torch.bfloat16, device="cuda")
    o = torch.empty_like(q)
    with pytest.raises(cuda_lib.WaveError) as e:
        kv.round_attn([(7200, 1)], "clean", q, o)
    assert e.value.code == -7
    nodes = [(c, 0) for c in range(65)]
    q65 = torch.zeros(65 * 128, 1, 64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(cuda_lib.WaveError) as e:
        kv.round_attn(nodes, "clean", q65, torch.empty_like(q65))
    assert e.value.code == -7
    raw = torch.zeros(128 * 64 + 8, dtype=torch.bfloat16, device="cuda")
    q_mis = raw[1:1 + 128 * 64].view(128, 1, 64)  # 2-byte offset
    with pytest.raises(cuda_lib.WaveError) as e:
        kv.round_attn([(1, 0)], "clean", q_mis, o)
    assert e.value.code == -1
    kv.status()


def test_launch_clock_words(cuda_lib):
    """The attention launch records its first CTA's SM cycles and nanoseconds;
    before any launch both words are zero."""
    import torch
    wl = dataclasses.replace(wi.TINY, tokens=200, head_dim=128)
    inp = Inputs(wl)
    kv = make_cache(cuda_lib, wl, 16)
    assert kv.last_launch_clock() == (0, 0)
    keep = [append(kv, inp, e) for e in ((0, 0), (1, 1))]
    q = queries(inp, [(1, 1)])
    kv.round_attn([(1, 1)], "progressive", q, torch.empty_like(q))
    kv.status()
    cyc, ns = kv.last_launch_clock()
    assert cyc > 0 and ns > 0
    assert 0.2 < cyc / ns < 2.5, (cyc, ns)  # GHz
    del keep


@pytest.mark.parametrize("pol", wi.POLICIES)
def test_tiny_all_rounds_batched_append(cuda_lib, pol):
    """The same rollout with each round's appends in one batched launch."""
    _rollout_and_check(cuda_lib, dataclasses.replace(wi.TINY, tokens=300, prefix=200), pol,
                       batch=True)


@pytest.mark.parametrize("d", [64, 128])
def test_append_batch_bytes_exact(cuda_lib, d):
    """A batched append (prefix + ragged entries) takes the pages that the same
    appends one by one take and writes the same bytes: each page [H][128][d]
    of K then V, rows past the entry's tokens zero."""
    import torch
    wl = wi.Workload("batch", chunks=3, levels=2, heads=3, head_dim=d, tokens=300, prefix=130)
    inp = Inputs(wl)
    entries = [(-1, 0), (0, 2), (1, 1), (0, 0)]
    kb = make_cache(cuda_lib, wl, 32)
    ks = [bits_to_torch(inp.bits("k", *e)) for e in entries]
    vs = [bits_to_torch(inp.bits("v", *e)) for e in entries]
    kb.alloc(2, 1)  # pages 0..2 taken first
    kb.append_batch(entries, ks, vs)
    ks1 = make_cache(cuda_lib, wl, 32)
    ks1.alloc(2, 1)
    keep = [append(ks1, inp, e) for e in entries]
    torch.cuda.synchronize()
    page_bytes, off, _ = kb.layout()
    pool, pool1 = kb.pool.cpu().numpy(), ks1.pool.cpu().numpy()
    n_pre, n_own = (wl.prefix + 127) // 128, (wl.tokens + 127) // 128
    for e in entries[1:]:
        (rows,) = kb.gather_table([e], "clean")
        assert [rows] == ks1.gather_table([e], "clean")
        spans = [((-1, 0), rows[:n_pre], wl.prefix), (e, rows[-n_own:], wl.tokens)]
        for ent, own, ntok in spans:
            for kind, kvi in (("k", 0), ("v", 1)):
                src = inp.bits(kind, *ent)
                for pi, (page, valid) in enumerate(own):
                    base = off + page * page_bytes + kvi * wl.heads * 128 * d * 2
                    blk = pool[base:base + wl.heads * 128 * d * 2].view(np.uint16)
                    blk1 = pool1[base:base + wl.heads * 128 * d * 2].view(np.uint16)
                    np.testing.assert_array_equal(blk, blk1)
                    blk = blk.reshape(wl.heads, 128, d)
                    want = np.zeros_like(blk)
                    n = min(128, ntok - pi * 128)
                    want[:, :n, :] = src[pi * 128:pi * 128 + n].transpose(1, 0, 2)
                    np.testing.assert_array_equal(blk, want)
                    assert valid == n
    del keep


def test_append_batch_errors_take_nothing(cuda_lib):
    import torch
    wl = wi.Workload("batch-err", chunks=4, levels=1, heads=1, head_dim=64, tokens=128)
    kv = make_cache(cuda_lib, wl, 3)
    k = torch.zeros(128, 1, 64, dtype=torch.bfloat16, device="cuda")
    free0 = kv.free_pages()
    cases = [([(0, 1), (0, 1)], -1),                  # named twice
             ([(0, 1), (1, 1), (2, 1), (3, 1)], -3),  # 4 pages, 3 free
             ([(c, 0) for c in range(65)], -7)]       # more entries than one call takes
    for entries, code in cases:
        with pytest.raises(cuda_lib.WaveError) as e:
            kv.append_batch(entries, [k] * len(entries), [k] * len(entries))
        assert e.value.code == code, entries
        assert kv.free_pages() == free0
    kv.append_batch([(0, 1)], [k], [k])
    with pytest.raises(cuda_lib.WaveError) as e:
        kv.append_batch([(1, 1), (0, 1)], [k, k], [k, k])
    assert e.value.code == -6 and kv.free_pages() == free0 - 1
    kv.status()


def _qkv_case(wave, heads, head_dim, tokens, dim, rows=None):
    """Fused projection + append of entry (1, 1) vs the oracle's X W^T."""
    import torch
    from oracle import projection
    wl = wi.Workload("qkv", chunks=2, levels=1, heads=heads, head_dim=head_dim, tokens=tokens)
    kv = make_cache(wave, wl, 2 * ((tokens + 127) // 128) + 4)
    kv.alloc(0, 0)  # the entry's pages do not start at page 0
    xb = wi.hidden_states(1, 1, tokens, dim)
    wb = wi.qkv_weight(heads, head_dim, dim)
    x, w = bits_to_torch(xb), bits_to_torch(wb)
    q = torch.empty(tokens, heads, head_dim, dtype=torch.bfloat16, device="cuda")
    kv.qkv_append(1, 1, x, w, q)
    kv.status()
    sel = np.arange(tokens) if rows is None else np.asarray(rows)
    rq, rk, rv = projection.qkv(wi.bf16_bits_to_f64(xb[sel]), wi.bf16_bits_to_f64(wb), heads,
                                head_dim)
    assert_close(torch_to_f64(q)[sel], rq, "qkv Q", scale_with_output=True)
    (table,) = kv.gather_table([(1, 1)], "clean")
    own = table[-((tokens + 127) // 128):]
    page_bytes, off, _ = kv.layout()
    pool = kv.pool.cpu().numpy()
    for kvi, ref in ((0, rk), (1, rv)):
        got = np.zeros(((tokens + 127) // 128 * 128, heads, head_dim), dtype=np.uint16)
        for pi, (page, valid) in enumerate(own):
            base = off + page * page_bytes + kvi * heads * 128 * head_dim * 2
            blk = pool[base:base + heads * 128 * head_dim * 2].view(np.uint16)
            got[pi * 128:(pi + 1) * 128] = blk.reshape(heads, 128, head_dim).transpose(1, 0, 2)
            assert valid == min(128, tokens - pi * 128)
        assert not got[tokens:].any(), "page tail must be zero"
        assert_close(wi.bf16_bits_to_f64(got[sel]), ref, f"qkv {'KV'[kvi]}",
                     scale_with_output=True)


@pytest.mark.parametrize("heads,d", [(3, 64), (3, 128), (2, 128)])
def test_qkv_append_small_ragged(cuda_lib, heads, d):
    """Three pages (300 tokens, ragged tail), three 64-wide slices of C. With d
    128 and 3 H even the 256-feature persistent kernel runs (H = 2), else the
    128-feature one."""
    _qkv_case(cuda_lib, heads=heads, head_dim=d, tokens=300, dim=192)


def test_qkv_append_wan21_sampled_rows(cuda_lib):
    """Wan2.1-1.3B shapes: 4680 tokens, C = 1536, 12 heads of 128; sampled rows
    across every page, including the last (partial) one."""
    rows = list(range(0, 4680, 37)) + [4607, 4608, 4679]
    _qkv_case(cuda_lib, heads=12, head_dim=128, tokens=4680, dim=1536, rows=rows)


def test_qkv_append_errors_take_nothing(cuda_lib):
    import torch
    wl = wi.Workload("qkv-err", chunks=2, levels=1, heads=2, head_dim=64, tokens=128)
    kv = make_cache(cuda_lib, wl, 4)
    free0 = kv.free_pages()
    x = torch.zeros(128, 96, dtype=torch.bfloat16, device="cuda")  # C not a multiple of 64
    w = torch.zeros(3 * 2 * 64, 96, dtype=torch.bfloat16, device="cuda")
    q = torch.empty(128, 2, 64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(cuda_lib.WaveError) as e:
        kv.qkv_append(0, 1, x, w, q)
    assert e.value.code == -1 and kv.free_pages() == free0
    x = torch.zeros(100, 64, dtype=torch.bfloat16, device="cuda")  # not tokens_per_chunk
    w = torch.zeros(3 * 2 * 64, 64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(cuda_lib.WaveError) as e:
        kv.qkv_append(0, 1, x, w, q)
    assert e.value.code == -1 and kv.free_pages() == free0
    kv.status()
