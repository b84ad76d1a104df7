"""The attention kernel's FMA-pipe exp2 (minimax cubic + exponent scaling).

A share of the softmax's 2^x runs as: clamp x to >= -126, j = round(x) via
adding 1.5 * 2^23, f = x - j in [-1/2, 1/2], 2^f ~ c0 + c1 f + c2 f^2 + c3 f^3
(coefficients from csrc/exp2_poly.h, fitted by csrc/fit_exp2_poly.py), then
2^j by adding j to the exponent field. This replays those float32 steps with
numpy and checks the result against 2^x in float64: relative error well under
bf16's 2^-9 (the precision P is stored in), over the whole input range the
kernel feeds it (x <= 8).
"""
import os
import re

import numpy as np

HDR = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "block_causal_attention_wave_b200", "csrc", "exp2_poly.h")


def _coeffs():
    text = open(HDR).read()
    c = [float(re.search(rf"WAVE_EXP2_C{i} ([-0-9.e]+)f", text).group(1)) for i in range(4)]
    return [np.float32(v) for v in c]


def _exp2_fma_pipe(x):
    c0, c1, c2, c3 = _coeffs()
    x = np.maximum(x.astype(np.float32), np.float32(-126.0))
    rnd = np.float32(12582912.0)
    t = (x + rnd).astype(np.float32)
    jf = (t - rnd).astype(np.float32)
    f = (x - jf).astype(np.float32)
    p = (c3 * f + c2).astype(np.float32)
    p = (p * f + c1).astype(np.float32)
    p = (p * f + c0).astype(np.float32)
    bits = p.view(np.uint32).astype(np.uint64) + ((t.view(np.uint32).astype(np.uint64) << 23))
    return (bits & 0xFFFFFFFF).astype(np.uint32).view(np.float32)


def test_relative_error_over_the_kernel_range():
    x = np.concatenate([np.linspace(-126.0, 8.0, 2_000_001), np.arange(-126, 9, 0.5),
                        np.random.default_rng(0).uniform(-30, 8, 100_000)]).astype(np.float32)
    y = _exp2_fma_pipe(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(y - ref) / ref
    assert rel.max() < 1.5e-4, rel.max()
    assert rel.max() < 2.0 ** -9 / 10


def test_fit_error_is_the_one_recorded():
    text = open(HDR).read()
    recorded = float(re.search(r"([0-9.]+e-0\d) \(float32 coefficients\)", text).group(1))
    f = np.linspace(-0.5, 0.5, 200_001)
    c = [float(v) for v in _coeffs()]
    p = c[0] + f * (c[1] + f * (c[2] + f * c[3]))
    err = np.abs(p - 2.0 ** f) / 2.0 ** f
    assert abs(err.max() - recorded) / recorded < 0.05


def test_very_negative_and_minus_infinity_give_negligible_values():
    x = np.array([-np.inf, -1e30, -500.0, -127.0, -126.0], dtype=np.float32)
    y = _exp2_fma_pipe(x)
    assert np.all(np.isfinite(y)) and np.all(y >= 0)
    assert np.all(y <= np.float32(2.0 ** -125))
