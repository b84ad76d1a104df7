"""Library host logic vs the oracle, bit for bit (CPU only; no kernel runs).

The scheduler, the last-read table and the page/valid tables of libwave.so are
compared with the oracle's on every workload shape and policy, and the C ABI is
checked to export every function include/wave.h declares.
"""
import os
import re
import subprocess

import pytest

import wave_inputs as wi
from oracle import cache as ocache
from oracle import schedule as osched

wave = pytest.importorskip("block_causal_attention_wave_b200")

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    return wave.load()


def _declared_functions():
    with open(os.path.join(ROOT, "include", "wave.h")) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(wave_[a-z_]+)\s*\(", text)))


def test_header_symbols_are_exported(lib):
    declared = _declared_functions()
    assert len(declared) >= 14
    out = subprocess.run(["nm", "-D", "--defined-only", wave.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (wave_[a-z_]+)\b", out))
    missing = [f for f in declared if f not in exported]
    assert not missing, missing
    assert sorted(wave.exported_symbols()) == declared


@pytest.mark.parametrize("pol", wi.POLICIES)
def test_schedules_match_oracle(lib, pol):
    for B in (1, 2, 3, 5, 7, 12, 40):
        for K in (1, 2, 3, 4, 5):
            for W in (0, 1, 2, 6, 32):
                assert wave.schedule(B, K, pol, W) == osched.schedule(B, K, pol, W), (B, K, W)


@pytest.mark.parametrize("pol", wi.POLICIES)
def test_last_read_rounds_match_oracle(lib, pol):
    for B, K, W in ((3, 2, 0), (7, 4, 0), (40, 5, 6), (40, 2, 32), (9, 3, 2)):
        assert wave.last_read_rounds(B, K, pol, W) == osched.last_read_round(B, K, pol, W)


def _library_rollout(wl, pol, max_pages):
    kv = wave.KVCache(wl.heads, wl.head_dim, wl.tokens, wl.levels, wl.window, wl.prefix,
                      pool=None, pool_bytes=4096 + max_pages * wave.KVCache.page_bytes(
                          wl.heads, wl.head_dim))
    rounds = wave.schedule(wl.chunks, wl.levels, pol, wl.window)
    last = wave.last_read_rounds(wl.chunks, wl.levels, pol, wl.window)
    if wl.prefix:
        kv.alloc(wave.PREFIX_CHUNK, 0, wl.prefix)
    out = []
    for t, active in enumerate(rounds):
        for n in active:
            kv.alloc(*n)
        out.append((active, kv.gather_table(active, pol)))
        for e in sorted(e for e, lr in last.items() if lr == t):
            kv.release(*e)
    assert kv.free_pages() == max_pages - (ocache.pages_for(wl.prefix) if wl.prefix else 0)
    return out


@pytest.mark.parametrize("wl", [wi.TINY, wi.WAN21, wi.WAN_STREAMER, wi.LONG_ROLLOUT],
                         ids=lambda w: w.name)
@pytest.mark.parametrize("pol", wi.POLICIES)
def test_gather_tables_match_oracle_bit_exact(lib, wl, pol):
    max_pages = 6000
    got = _library_rollout(wl, pol, max_pages)
    want = ocache.rollout_tables(wl.chunks, wl.levels, pol, wl.window, wl.tokens, wl.prefix,
                                 max_pages)
    assert len(got) == len(want)
    for (ga, gt), (wa, wt) in zip(got, want):
        assert ga == wa
        assert gt == wt


def test_error_paths(lib):
    kv = wave.KVCache(2, 64, 200, 2, pool=None, pool_bytes=4096 + 5 * 65536)
    assert kv.free_pages() == 5
    kv.alloc(0, 2)
    with pytest.raises(wave.WaveError) as e:
        kv.alloc(0, 2)
    assert e.value.code == -6
    with pytest.raises(wave.WaveError) as e:
        kv.alloc(1, 2, 199)  # wrong token count
    assert e.value.code == -1
    kv.alloc(1, 2)
    with pytest.raises(wave.WaveError) as e:
        kv.alloc(2, 2)  # needs 2 pages, 1 free
    assert e.value.code == -3
    assert kv.free_pages() == 1
    with pytest.raises(wave.WaveError) as e:
        kv.gather_table([(1, 1)], "progressive")
    assert e.value.code == -2
    with pytest.raises(wave.WaveError) as e:
        kv.gather_table([(0, 3)], "progressive")  # level above num_levels
    assert e.value.code == -1
    with pytest.raises(wave.WaveError) as e:
        kv.release(3, 1)
    assert e.value.code == -2
    with pytest.raises(wave.WaveError) as e:
        kv.alloc(-1, 0, 10)  # no prefix configured
    assert e.value.code == -1
    import torch
    k = torch.zeros(200, 2, 64, dtype=torch.bfloat16)
    free = kv.free_pages()
    with pytest.raises(wave.WaveError) as e:  # a host-only handle has no device to copy to
        kv.append_batch([(3, 1)], [k], [k], stream=0)
    assert e.value.code == -1 and kv.free_pages() == free
    x = torch.zeros(200, 64, dtype=torch.bfloat16)
    w = torch.zeros(3 * 2 * 64, 64, dtype=torch.bfloat16)
    with pytest.raises(wave.WaveError) as e:  # nor one to project on
        kv.qkv_append(3, 1, x, w, k, stream=0)
    assert e.value.code == -1 and kv.free_pages() == free
    with pytest.raises(wave.WaveError) as e:
        wave.KVCache(2, 96, 32, 2, pool=None, pool_bytes=1 << 20)
    assert e.value.code == -8
    with pytest.raises(wave.WaveError) as e:
        wave.schedule(0, 2)
    assert e.value.code == -1
    # Kernels refuse a host-only handle without touching a device.
    import torch
    q = torch.zeros(200, 2, 64, dtype=torch.bfloat16)
    with pytest.raises(wave.WaveError) as e:
        kv.round_attn([(0, 2)], "progressive", q, q, stream=0)
    assert e.value.code == -1


def test_random_rollouts_match_oracle_bit_exact(lib):
    """Seeded random shapes (chunks, levels, window, tokens incl. ragged and
    exact multiples of 128, prefix, policy): schedules, last-read tables and
    every round's gather table equal the oracle's."""
    import numpy as np
    rng = np.random.default_rng(20261202)
    for case in range(150):
        B = int(rng.integers(1, 10))
        K = int(rng.integers(1, 6))
        W = int(rng.choice([0, 1, 2, 3, 5]))
        T = int(rng.choice([1, 64, 127, 128, 129, 300, 1000]))
        prefix = int(rng.choice([0, 0, 1, 128, 200]))
        pol = str(rng.choice(wi.POLICIES))
        wl = wi.Workload(f"rand{case}", chunks=B, levels=K, heads=1, head_dim=64, tokens=T,
                         window=W, prefix=prefix)
        assert wave.schedule(B, K, pol, W) == osched.schedule(B, K, pol, W), (B, K, W, pol)
        assert wave.last_read_rounds(B, K, pol, W) == osched.last_read_round(B, K, pol, W)
        max_pages = 2000
        got = _library_rollout(wl, pol, max_pages)
        want = ocache.rollout_tables(B, K, pol, W, T, prefix, max_pages)
        assert got == [(a, t) for a, t in want], (B, K, W, T, prefix, pol)


def test_host_only_handle_refuses_device_calls_of_the_block_and_split(lib):
    """Calls that launch kernels refuse a host-only handle before any work."""
    import ctypes
    import block_causal_attention_wave_b200 as wave
    from block_causal_attention_wave_b200 import _binding as b
    kv = wave.KVCache(2, 128, 256, 2, pool=None, pool_bytes=4096 + 16 * wave.KVCache.page_bytes(2, 128))
    node = (b.Node * 1)(b.Node(0, 1))
    nbytes, used = ctypes.c_uint64(), ctypes.c_int32()
    assert lib.wave_round_attn_split_workspace(kv.h, node, 1, 2, 0, ctypes.byref(nbytes),
                                               ctypes.byref(used)) == b.ERR_ARG
    assert lib.wave_round_attn_split(kv.h, node, 1, 2, 0, None, None, None, 0, None) == b.ERR_ARG
    assert lib.wave_qkv_append_round(kv.h, node, 1, None, 128, None, None, None, None) == b.ERR_ARG
    assert lib.wave_linear(kv.h, None, 128, 128, None, 256, None, 0, None, None) == b.ERR_ARG
    off = ctypes.c_int64()
    assert lib.wave_kv_scale_offset(kv.h, ctypes.byref(off)) == b.ERR_ARG  # not an FP8 pool
    assert lib.wave_kv_set_wait_limit(kv.h, 1000) == b.OK
    assert kv.free_pages() == 16  # nothing was taken


def test_fp8_host_only_layout(lib):
    """An FP8 pool's pages hold one-byte codes, and its scale table sits after
    the last page, 256-byte aligned, with 2 H float32 per page."""
    import block_causal_attention_wave_b200 as wave
    H, d = 3, 128
    pb8 = wave.KVCache.page_bytes(H, d, wave.KV_FP8_E4M3)
    assert pb8 == 2 * H * 128 * d
    pool_bytes = 4096 + 256 + 10 * (pb8 + 2 * H * 4)
    kv = wave.KVCache(H, d, 300, 2, pool=None, pool_bytes=pool_bytes, kv_format=wave.KV_FP8_E4M3)
    page_bytes, off, maxp = kv.layout()
    assert page_bytes == pb8 and maxp == 10
    soff = kv.scale_offset()
    assert soff % 256 == 0 and soff >= off + maxp * pb8
    assert soff + maxp * 2 * H * 4 <= pool_bytes
    kv.alloc(0, 1)
    assert kv.entry_pages(0, 1) == [0, 1, 2]
