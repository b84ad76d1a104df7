"""Pins of oracle.quant (E4M3 encoding, per-(page, head) scales, read-back):
hand-worked codes, ties to even, saturation, every finite code round-trips,
agreement with torch's own float8_e4m3fn conversion (an independent
implementation) inside the finite range, and the amax element landing on 448."""
import numpy as np
import pytest
import torch

from oracle import quant


@pytest.mark.parametrize("x,code", [
    (0.0, 0x00), (1.0, 0x38), (0.5, 0x30), (448.0, 0x7E), (240.0, 0x77), (-1.0, 0xB8),
    (2.0 ** -9, 0x01), (2.0 ** -6, 0x08), (1.125, 0x39), (-448.0, 0xFE), (3.5, 0x46),
])
def test_hand_codes(x, code):
    assert int(quant.e4m3_encode(np.array([x]))[0]) == code
    assert quant.e4m3_decode(np.array([code]))[0] == x


def test_ties_to_even_and_saturation():
    enc = lambda v: int(quant.e4m3_encode(np.array([v]))[0])  # noqa: E731
    assert enc(1 + 1 / 16) == 0x38        # halfway 1 .. 1.125 -> even (1.0)
    assert enc(1 + 3 / 16) == 0x3A        # halfway 1.125 .. 1.25 -> even (1.25)
    assert enc(2.0 ** -10) == 0x00        # halfway 0 .. 2^-9 -> even (0)
    assert enc(3 * 2.0 ** -10) == 0x02    # halfway 2^-9 .. 2^-8 -> even
    assert enc(15.5) == 0x58              # halfway 15 (0x57) .. 16 (0x58) -> even 0x58
    assert enc(1000.0) == 0x7E and enc(-500.0) == 0xFE and enc(460.0) == 0x7E


def test_every_finite_code_round_trips():
    vals = quant.e4m3_values()
    codes = np.array([c for c in range(256) if not np.isnan(vals[c])], dtype=np.uint8)
    back = quant.e4m3_encode(vals[codes])
    # +0 and -0 both decode to 0; -0 encodes as 0x80 only for a negative zero
    np.testing.assert_array_equal(back[codes != 0x80], codes[codes != 0x80])


def test_matches_torch_float8_e4m3fn_in_range():
    rng = np.random.default_rng(3)
    x = np.concatenate([rng.standard_normal(20000) * 40, rng.uniform(-448, 448, 20000),
                        rng.standard_normal(5000) * 1e-2]).astype(np.float32)
    want = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = quant.e4m3_encode(x.astype(np.float64))
    np.testing.assert_array_equal(got, want)


def test_tile_scale_puts_amax_on_448_and_zero_tile():
    rng = np.random.default_rng(4)
    x = rng.standard_normal((128, 64))
    x[17, 5] = -7.25  # the largest magnitude
    codes, s = quant.quantize_tile(x)
    assert s == np.float32(np.float32(7.25) / np.float32(448))
    assert codes[17, 5] == 0xFE
    back = quant.dequantize_tile(codes, s)
    rel = np.abs(back - x) / np.maximum(np.abs(x), 2.0 ** -6 * s)
    assert rel.max() <= 2.0 ** -4 + 2.0 ** -8  # half an E4M3 step plus bf16 rounding
    z, sz = quant.quantize_tile(np.zeros((128, 64)))
    assert sz == 1.0 and not z.any()


def test_entry_pages_and_zero_tail():
    rng = np.random.default_rng(5)
    x = rng.standard_normal((200, 2, 64))
    codes, scales = quant.quantize_entry(x)
    assert codes.shape == (2, 2, 128, 64) and scales.shape == (2, 2)
    assert not codes[1, :, 72:, :].any()  # rows past the 200 tokens stay zero
    back = quant.dequantize_entry(codes, scales, 200)
    assert back.shape == x.shape
    for p in range(2):
        for h in range(2):
            amax = np.abs(x[p * 128:(p + 1) * 128, h]).max()
            assert scales[p, h] == np.float32(np.float32(amax) / np.float32(448))
