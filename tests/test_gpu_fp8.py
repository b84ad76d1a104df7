"""GPU parity of FP8 (E4M3) K/V pages: the quantising append and the attention
over an FP8 pool (pages expanded to bf16 staging, then the attention kernel).

The append's codes and scales are compared bit for bit with the oracle's
quantisation of the same bf16 K/V (single and batched appends, ragged tails,
d 64 and 128). The attention is compared element by element with the float64
oracle over the oracle's own read-back of those codes, bf16(code * scale), on
small rollouts (every round) and on sampled rows of the Wan2.1-1.3B round;
bar as elsewhere (max-abs 1e-2, rel-L2 5e-3) -- the quantisation itself is in
the oracle, so only the attention's rounding remains. Calls that cannot work
on an FP8 pool are refused.
"""
import numpy as np
import pytest

import wave_inputs as wi
from oracle import attention as oatt
from oracle import cache as ocache
from oracle import quant as oquant
from oracle import schedule as osched

from wave_testlib import Inputs, assert_close, bits_to_torch, queries, torch_to_f64

pytestmark = pytest.mark.gpu


def _fp8_cache(wave, wl, pages):
    import torch
    pb = wave.KVCache.page_bytes(wl.heads, wl.head_dim, wave.KV_FP8_E4M3)
    nbytes = 4096 + 256 + pages * (pb + 2 * wl.heads * 4)
    pool = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
    kv = wave.KVCache(wl.heads, wl.head_dim, wl.tokens, wl.levels, wl.window, wl.prefix,
                      pool=pool, kv_format=wave.KV_FP8_E4M3)
    return kv, pool


def _read_fp8_entry(kv, pool, entry):
    """Codes [pages][2][H][128][d] and scales [pages][2][H] of one entry."""
    page_bytes, off, maxp = kv.layout()
    H, d = kv.heads, kv.head_dim
    soff = kv.scale_offset()
    host = pool.cpu().numpy()
    scales = host[soff:soff + maxp * 2 * H * 4].view(np.float32).reshape(maxp, 2, H)
    pages = kv.entry_pages(*entry)
    codes = np.stack([host[off + p * page_bytes:off + (p + 1) * page_bytes].reshape(2, H, 128, d)
                      for p in pages])
    return codes, scales[pages]


class _Oracle:
    """The oracle's view of an FP8 pool: quantised entries and their read-back."""

    def __init__(self, inp):
        self.inp = inp
        self.q = {}

    def entry(self, e):
        if e not in self.q:
            k, v = self.inp.f64("k", *e), self.inp.f64("v", *e)
            self.q[e] = (oquant.quantize_entry(k), oquant.quantize_entry(v))
        return self.q[e]

    def readback(self, e):
        (kc, ks), (vc, vs) = self.entry(e)
        n = self.inp.wl.prefix if e[0] == -1 else self.inp.wl.tokens
        return oquant.dequantize_entry(kc, ks, n), oquant.dequantize_entry(vc, vs, n)


def _append(kv, inp, e):
    k, v = bits_to_torch(inp.bits("k", *e)), bits_to_torch(inp.bits("v", *e))
    kv.append(e[0], e[1], k, v)
    return k, v


@pytest.mark.parametrize("wl", [
    wi.Workload("fp8-d128", chunks=3, levels=2, heads=3, head_dim=128, tokens=300, prefix=77),
    wi.Workload("fp8-d64", chunks=3, levels=2, heads=2, head_dim=64, tokens=129),
], ids=lambda w: w.name)
def test_fp8_append_bytes_and_scales_exact(cuda_lib, wl):
    wave = cuda_lib
    inp = Inputs(wl)
    orc = _Oracle(inp)
    kv, pool = _fp8_cache(wave, wl, 32)
    ents = [(0, 2), (1, 1)] + ([(-1, 0)] if wl.prefix else [])
    keep = [_append(kv, inp, e) for e in ents]
    # the rest in one batched launch
    batch = [(2, 2), (0, 1)]
    ks = [bits_to_torch(inp.bits("k", *e)) for e in batch]
    vs = [bits_to_torch(inp.bits("v", *e)) for e in batch]
    kv.append_batch(batch, ks, vs)
    kv.status()
    for e in ents + batch:
        codes, scales = _read_fp8_entry(kv, pool, e)
        (kc, kscale), (vc, vscale) = orc.entry(e)
        np.testing.assert_array_equal(codes[:, 0], kc, err_msg=f"K codes of {e}")
        np.testing.assert_array_equal(codes[:, 1], vc, err_msg=f"V codes of {e}")
        np.testing.assert_array_equal(scales[:, 0], kscale, err_msg=f"K scales of {e}")
        np.testing.assert_array_equal(scales[:, 1], vscale, err_msg=f"V scales of {e}")
    del keep, ks, vs


def _attn_round(wave, kv, inp, orc, active, pol, rows=None):
    import torch
    wl = inp.wl
    q = queries(inp, active)
    o = torch.full_like(q, float("nan"))
    nbytes, _ = kv.split_workspace(active, pol, 1)
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    kv.round_attn_split(active, pol, q, o, ws, 1)
    kv.status()
    needed = set()
    for n in active:
        needed.update(e for e in ocache.key_entries(n, pol, wl.window, wl.prefix > 0)
                      if e != ocache.PREFIX)
    ents = {e: orc.readback(e) for e in needed}
    pre = orc.readback((-1, 0)) if wl.prefix else None
    qs = {n: inp.f64("q", *n) for n in active}
    ref = oatt.round_attention(active, pol, wl.window, qs, ents, pre,
                               {n: rows for n in active} if rows is not None else None)
    got = torch_to_f64(o).reshape(len(active), wl.tokens, wl.heads, wl.head_dim)
    for i, n in enumerate(active):
        g = got[i] if rows is None else got[i][rows]
        assert_close(g, ref[n], f"{wl.name} fp8 node {n}")


@pytest.mark.parametrize("wl", [
    wi.Workload("fp8-roll-d128", chunks=4, levels=2, heads=2, head_dim=128, tokens=300,
                prefix=77),
    wi.Workload("fp8-roll-d64-window", chunks=5, levels=2, heads=2, head_dim=64, tokens=200,
                window=2),
], ids=lambda w: w.name)
def test_fp8_rollout_every_round(cuda_lib, wl):
    wave = cuda_lib
    pol = "progressive"
    inp = Inputs(wl)
    orc = _Oracle(inp)
    kv, _ = _fp8_cache(wave, wl, 80)
    rounds = wave.schedule(wl.chunks, wl.levels, pol, wl.window)
    last = wave.last_read_rounds(wl.chunks, wl.levels, pol, wl.window)
    keep = []
    if wl.prefix:
        keep.append(_append(kv, inp, (-1, 0)))
    for t, active in enumerate(rounds):
        keep += [_append(kv, inp, n) for n in active]
        _attn_round(wave, kv, inp, orc, active, pol)
        for e in sorted(e for e, lr in last.items() if lr == t):
            kv.release(*e)


def test_fp8_wan21_round_sampled_rows(cuda_lib):
    wave = cuda_lib
    wl = wi.WAN21
    pol = "progressive"
    inp = Inputs(wl)
    orc = _Oracle(inp)
    active = osched.schedule(wl.chunks, wl.levels, pol, wl.window)[6]
    ents = set()
    for n in active:
        ents.update(ocache.key_entries(n, pol, wl.window, False))
    kv, _ = _fp8_cache(wave, wl, len(ents) * 37 + 8)
    keep = [_append(kv, inp, e) for e in sorted(ents)]
    rows = np.unique(np.concatenate([np.linspace(0, wl.tokens - 1, 12).astype(int),
                                     [4607, 4608, wl.tokens - 1]]))
    _attn_round(wave, kv, inp, orc, active, pol, rows)
    del keep


def test_fp8_pool_refuses_what_needs_bf16_pages(cuda_lib):
    import torch
    wave = cuda_lib
    wl = wi.Workload("fp8-err", chunks=2, levels=1, heads=2, head_dim=128, tokens=128)
    inp = Inputs(wl)
    kv, _ = _fp8_cache(wave, wl, 8)
    keep = [_append(kv, inp, (0, 1))]
    q = queries(inp, [(0, 1)])
    o = torch.empty_like(q)
    with pytest.raises(wave.WaveError):
        kv.round_attn([(0, 1)], "progressive", q, o)
    with pytest.raises(wave.WaveError):
        kv.round_attn_static_scratch([(0, 1)], "progressive", q, o)
    x = torch.zeros((128, 128), dtype=torch.bfloat16, device="cuda")
    w = torch.zeros((3 * 2 * 128, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(wave.WaveError):
        kv.qkv_append(1, 1, x, w, torch.empty((128, 2, 128), dtype=torch.bfloat16, device="cuda"))
    assert kv.split_workspace([(0, 1)], "progressive", 1)[0] > 0
    del keep


def test_fp8_pool_with_split_key_ranges(cuda_lib):
    """FP8 pages and split key ranges together: the workspace holds the bf16
    staging pages first and the ranges' partial results after them."""
    wave = cuda_lib
    wl = wi.Workload("fp8-split", chunks=5, levels=2, heads=2, head_dim=128, tokens=300,
                     prefix=77)
    pol = "progressive"
    inp = Inputs(wl)
    orc = _Oracle(inp)
    kv, _ = _fp8_cache(wave, wl, 80)
    active = max(osched.schedule(wl.chunks, wl.levels, pol, wl.window),
                 key=lambda r: (len(r), r[-1][0]))
    ents = set()
    for n in active:
        ents.update(ocache.key_entries(n, pol, wl.window, True))
    keep = [_append(kv, inp, e) for e in sorted(ents)]
    import torch
    q = queries(inp, active)
    o = torch.full_like(q, float("nan"))
    nbytes, used = kv.split_workspace(active, pol, 3)
    assert used == 3 and nbytes > kv.split_workspace(active, pol, 1)[0]
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    kv.round_attn_split(active, pol, q, o, ws, 3)
    kv.status()
    needed = set(e for n in active for e in ocache.key_entries(n, pol, wl.window, True)
                 if e != ocache.PREFIX)
    ref = oatt.round_attention(active, pol, wl.window, {n: inp.f64("q", *n) for n in active},
                               {e: orc.readback(e) for e in needed}, orc.readback((-1, 0)))
    got = torch_to_f64(o).reshape(len(active), wl.tokens, wl.heads, wl.head_dim)
    for i, n in enumerate(active):
        assert_close(got[i], ref[n], f"fp8 + 3 ranges, node {n}")
    del keep
