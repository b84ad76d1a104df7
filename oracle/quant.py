"""FP8 (E4M3) K/V pages with per-(page, head) scales -- oracle side.

TEST INFRASTRUCTURE ONLY (see the package docstring).

The Wan-Streamer v0.2 page leaves the growth of the K/V cache open (its
limitations discussion); the design-space paper's same-level policy keeps K
levels of history alive (Table 1 / Figure 1). Storing cache pages in 8-bit
floats halves their bytes. The pages give no format; the reading used here:

* Format E4M3 (1 sign, 4 exponent bits with bias 7, 3 mantissa bits): finite
  values (1 + m/8) 2^(e-7) for e = 1..15 (e = 15, m = 7 is not a number, so the
  largest is 448) and subnormals (m/8) 2^-6; conversion rounds to nearest,
  ties to even, and saturates to +-448.
* One scale per (page, head) for K and one for V: with amax the largest |x|
  over the page's 128 token rows of that head (tail rows are zero),
  s = amax / 448 computed in float32 (s = 1 when amax = 0); q = E4M3(x / s)
  with x / s computed in float32.
* Read-back for attention: bf16(q * s), the product in float32 then rounded to
  bfloat16 (to nearest, ties to even) -- the values the attention consumes.
"""
from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0


def e4m3_values() -> np.ndarray:
    """Value of each of the 256 E4M3 codes (NaN for the two NaN codes)."""
    vals = np.empty(256)
    for code in range(256):
        s = -1.0 if code & 0x80 else 1.0
        e = (code >> 3) & 0xF
        m = code & 0x7
        if e == 15 and m == 7:
            vals[code] = np.nan
        elif e == 0:
            vals[code] = s * (m / 8.0) * 2.0 ** -6
        else:
            vals[code] = s * (1.0 + m / 8.0) * 2.0 ** (e - 7)
    return vals


_VALUES = e4m3_values()
# Non-negative finite codes in increasing value order (0x00 .. 0x7E).
_POS_CODES = np.arange(0x7F)
_POS_VALUES = _VALUES[_POS_CODES]


def e4m3_encode(x: np.ndarray) -> np.ndarray:
    """Round each value to the nearest E4M3 value (ties to the even code),
    saturating at +-448; returns the uint8 codes. -0 encodes as 0x80."""
    x = np.asarray(x, dtype=np.float64)
    a = np.minimum(np.abs(x), E4M3_MAX)
    # index of the largest representable value <= a, and the next one up
    lo = np.searchsorted(_POS_VALUES, a, side="right") - 1
    hi = np.minimum(lo + 1, len(_POS_VALUES) - 1)
    v_lo, v_hi = _POS_VALUES[lo], _POS_VALUES[hi]
    d_lo, d_hi = a - v_lo, v_hi - a
    take_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi != lo) & (_POS_CODES[lo] % 2 == 1))
    code = np.where(take_hi, _POS_CODES[hi], _POS_CODES[lo]).astype(np.uint8)
    return np.where(np.signbit(x), code | 0x80, code).astype(np.uint8)


def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    return _VALUES[np.asarray(codes, dtype=np.uint8)]


def quantize_tile(x: np.ndarray):
    """(codes, scale) of one page-head tile x (any shape, bf16 values as
    float64), per the reading above."""
    x32 = np.asarray(x, dtype=np.float64).astype(np.float32)
    amax = np.float32(np.abs(x32).max()) if x32.size else np.float32(0)
    s = np.float32(amax / np.float32(E4M3_MAX)) if amax > 0 else np.float32(1.0)
    q = e4m3_encode((x32 / s).astype(np.float32).astype(np.float64))
    return q, s


def dequantize_tile(codes: np.ndarray, scale) -> np.ndarray:
    """bf16(q * s) as float64: the product in float32, then bf16 rounding."""
    from .block import bf16_round
    p = (e4m3_decode(codes).astype(np.float32) * np.float32(scale)).astype(np.float32)
    return bf16_round(p.astype(np.float64))


def quantize_entry(x: np.ndarray, tokens_per_page: int = 128):
    """An entry's K (or V) [T][H][d] as stored: per page p and head h the
    codes [128][d] (tail rows zero before quantising) and the scale."""
    T, H, d = x.shape
    n_pages = (T + tokens_per_page - 1) // tokens_per_page
    padded = np.zeros((n_pages * tokens_per_page, H, d))
    padded[:T] = x
    codes = np.zeros((n_pages, H, tokens_per_page, d), dtype=np.uint8)
    scales = np.zeros((n_pages, H), dtype=np.float32)
    for p in range(n_pages):
        for h in range(H):
            tile = padded[p * tokens_per_page:(p + 1) * tokens_per_page, h, :]
            codes[p, h], scales[p, h] = quantize_tile(tile)
    return codes, scales


def dequantize_entry(codes: np.ndarray, scales: np.ndarray, tokens: int) -> np.ndarray:
    """[T][H][d] float64 values the attention reads from a quantised entry."""
    n_pages, H, P, d = codes.shape
    out = np.zeros((n_pages * P, H, d))
    for p in range(n_pages):
        for h in range(H):
            out[p * P:(p + 1) * P, h, :] = dequantize_tile(codes[p, h], scales[p, h])
    return out[:tokens]
