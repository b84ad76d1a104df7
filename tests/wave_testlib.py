"""Helpers shared by the GPU parity tests: build seeded inputs, drive the
library through a rollout, and compare with the oracle.

Tolerances (stated for the GPU path vs the float64 oracle on the same bf16
inputs): max-abs error <= 1e-2 and relative L2 error <= 5e-3 per node.
"""
from __future__ import annotations

import numpy as np

import wave_inputs as wi
from oracle import attention as oatt

MAX_ABS = 1e-2
REL_L2 = 5e-3


def bits_to_torch(bits, device="cuda"):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)
    return t.to(device)


def torch_to_f64(t):
    return t.float().cpu().numpy().astype(np.float64)


class Inputs:
    """Seeded bf16 Q/K/V per (chunk, level), memoised, as bits and as float64."""

    def __init__(self, wl: wi.Workload):
        self.wl = wl
        self._bits = {}

    def bits(self, kind, chunk, level):
        key = (kind, chunk, level)
        if key not in self._bits:
            n = self.wl.prefix if chunk == -1 else self.wl.tokens
            self._bits[key] = wi.node_tensor(kind, chunk, level, n, self.wl.heads,
                                             self.wl.head_dim, self.wl.scale)
        return self._bits[key]

    def f64(self, kind, chunk, level):
        return wi.bf16_bits_to_f64(self.bits(kind, chunk, level))

    def entries_f64(self, entries):
        return {e: (self.f64("k", *e), self.f64("v", *e)) for e in entries}


def make_cache(wave, wl: wi.Workload, pages: int):
    import torch
    page_bytes = wave.KVCache.page_bytes(wl.heads, wl.head_dim)
    pool = torch.empty(4096 + pages * page_bytes, dtype=torch.uint8, device="cuda")
    return wave.KVCache(wl.heads, wl.head_dim, wl.tokens, wl.levels, wl.window, wl.prefix,
                        pool=pool)


def append(kv, inp: Inputs, entry):
    k = bits_to_torch(inp.bits("k", *entry))
    v = bits_to_torch(inp.bits("v", *entry))
    kv.append(entry[0], entry[1], k, v)
    return k, v


def queries(inp: Inputs, active):
    import torch
    return torch.cat([bits_to_torch(inp.bits("q", *n)) for n in active], dim=0)


def oracle_outputs(inp: Inputs, active, pol, rows=None):
    """Oracle O for each node (optionally only at the given query rows)."""
    wl = inp.wl
    from oracle import cache as ocache
    needed = set()
    for n in active:
        needed.update(e for e in ocache.key_entries(n, pol, wl.window, wl.prefix > 0)
                      if e != ocache.PREFIX)
    ents = inp.entries_f64(needed)
    pre = (inp.f64("k", -1, 0), inp.f64("v", -1, 0)) if wl.prefix else None
    qs = {n: inp.f64("q", *n) for n in active}
    return oatt.round_attention(active, pol, wl.window, qs, ents, pre, rows)


def compare(got: np.ndarray, want: np.ndarray):
    err = got - want
    max_abs = float(np.abs(err).max()) if err.size else 0.0
    denom = float(np.linalg.norm(want))
    rel = float(np.linalg.norm(err)) / denom if denom > 0 else float(np.linalg.norm(err))
    return max_abs, rel


def assert_close(got, want, what="", scale_with_output=False):
    """Max-abs <= 1e-2 and rel-L2 <= 5e-3.

    With ``scale_with_output`` the max-abs bound is 1e-2 * max(1, max|want|):
    the output is stored in bf16, whose rounding alone is up to 2^-8 of |O|
    (0.0078 at |O| = 2), so an absolute 1e-2 cannot hold for outputs well above
    1. The workload cases (|O| < 1) use the plain absolute bound.
    """
    max_abs, rel = compare(got, want)
    bound = MAX_ABS * max(1.0, float(np.abs(want).max())) if scale_with_output else MAX_ABS
    assert max_abs <= bound and rel <= REL_L2, f"{what}: max_abs={max_abs:.3e} rel_l2={rel:.3e}"
    return max_abs, rel


def read_entry(kv, pool, entry, tokens):
    """K and V of one cache entry read back from the pool: ([T][H][d] float64
    each, bf16 values) and whether the rows past the tokens are all zero."""
    page_bytes, off, _ = kv.layout()
    H, d = kv.heads, kv.head_dim
    host = pool.cpu().numpy()
    pages = kv.entry_pages(*entry)
    out, tail_zero = [], True
    for kvi in range(2):
        rows = np.zeros((len(pages) * 128, H, d), dtype=np.uint16)
        for pi, page in enumerate(pages):
            base = off + page * page_bytes + kvi * H * 128 * d * 2
            blk = host[base:base + H * 128 * d * 2].view(np.uint16)
            rows[pi * 128:(pi + 1) * 128] = blk.reshape(H, 128, d).transpose(1, 0, 2)
        tail_zero = tail_zero and not rows[tokens:].any()
        out.append(wi.bf16_bits_to_f64(rows[:tokens]))
    return out[0], out[1], tail_zero
