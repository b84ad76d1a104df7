"""Pins of oracle.block (rotary embedding, out-projection, tanh-GELU MLP, bf16
storage) against what fixes them independently of their code: hand-worked
angles on a tiny grid, rotation direction and norm, the relative-position
property of rotary embeddings, the exact odd-part identity of GELU and its
distance to the erf form, selection/one-hot weights, brute-force loops, and an
independent bf16 rounding."""
import math

import numpy as np
import pytest

import wave_inputs as wi
from oracle import block


def test_rope_groups_split_the_pairs():
    assert block.rope_groups(128) == (22, 21, 21)
    assert block.rope_groups(64) == (12, 10, 10)
    assert block.rope_groups(6) == (1, 1, 1)
    for d in (6, 8, 64, 96, 128):
        assert sum(block.rope_groups(d)) == d // 2


def test_rope_angles_tiny_grid_by_hand():
    # d = 6: one pair per axis, each turning at 1 rad per position step.
    # Grid 2 frames x 2 rows x 3 columns; chunk 1 starts at frame 2.
    ang = block.rope_angles(chunk=1, frames=2, rows=2, cols=3, head_dim=6)
    assert ang.shape == (12, 3)
    want = {0: (2, 0, 0), 1: (2, 0, 1), 4: (2, 1, 1), 5: (2, 1, 2), 6: (3, 0, 0), 11: (3, 1, 2)}
    for t, w in want.items():
        np.testing.assert_array_equal(ang[t], w)


def test_rope_frequencies_per_group():
    ang = block.rope_angles(chunk=0, frames=2, rows=2, cols=2, head_dim=128)
    # token 4 sits at frame 1, row 0, column 0: only the frame group (pairs
    # 0..21) turns, pair 0 by exactly 1 rad and pair 11 by 10000^(-1/2) = 0.01;
    # consecutive pairs of the group turn 10000^(1/22) times slower.
    assert ang[4, 0] == 1.0
    assert abs(ang[4, 11] - 0.01) < 1e-15
    np.testing.assert_allclose(ang[4, 1:22] / ang[4, :21], 10000 ** (-1 / 22), rtol=1e-12)
    np.testing.assert_array_equal(ang[4, 22:], 0.0)
    # token 2: row 1 -> pairs 22..42 (row group, 21 pairs) turn, pair 22 by 1 rad.
    assert ang[2, 22] == 1.0 and ang[2, 21] == 0.0 and ang[2, 43] == 0.0
    # token 1: column 1 -> pairs 43..63.
    assert ang[1, 43] == 1.0 and ang[1, 42] == 0.0
    np.testing.assert_array_equal(ang[0], 0.0)


def test_rope_identity_at_origin_and_rotation_direction():
    x = np.random.default_rng(1).standard_normal((1, 2, 8))
    np.testing.assert_array_equal(block.apply_rope(x, np.zeros((1, 4))), x)
    e = np.zeros((1, 1, 2))
    e[0, 0, 0] = 1.0
    r = block.apply_rope(e, np.array([[math.pi / 2]]))
    np.testing.assert_allclose(r[0, 0], [0.0, 1.0], atol=1e-15)  # (1, 0) -> (0, 1)
    e[0, 0] = [0.0, 1.0]
    r = block.apply_rope(e, np.array([[math.pi / 2]]))
    np.testing.assert_allclose(r[0, 0], [-1.0, 0.0], atol=1e-15)


def test_rope_keeps_pair_norms():
    rng = np.random.default_rng(2)
    x = rng.standard_normal((40, 3, 128))
    ang = block.rope_angles(chunk=3, frames=2, rows=4, cols=5, head_dim=128)
    y = block.apply_rope(x, ang)
    nx = x[..., 0::2] ** 2 + x[..., 1::2] ** 2
    ny = y[..., 0::2] ** 2 + y[..., 1::2] ** 2
    np.testing.assert_allclose(ny, nx, rtol=1e-12)


def test_rope_scores_depend_on_position_differences_only():
    # Rotated q.k for two tokens equals that of the same two tokens one chunk
    # later (every frame position moves by F): only differences matter.
    rng = np.random.default_rng(3)
    F, R, W, d = 2, 3, 4, 64
    q = rng.standard_normal((F * R * W, 1, d))
    k = rng.standard_normal((F * R * W, 1, d))
    s = []
    for c in (0, 5):
        ang = block.rope_angles(chunk=c, frames=F, rows=R, cols=W, head_dim=d)
        qr, kr = block.apply_rope(q, ang), block.apply_rope(k, ang)
        s.append(qr[:, 0] @ kr[:, 0].T)
    np.testing.assert_allclose(s[0], s[1], rtol=1e-10, atol=1e-10)
    # ... and differs from the unrotated scores (the rotation does act).
    assert np.abs(s[0] - q[:, 0] @ k[:, 0].T).max() > 1e-3


def test_qkv_rope_rotates_q_and_k_not_v():
    rng = np.random.default_rng(4)
    H, d, C = 2, 8, 6
    x = rng.standard_normal((12, C))
    w = rng.standard_normal((3 * H * d, C))
    q, k, v = block.qkv_rope(x, w, H, d, chunk=1, grid=(1, 3, 4))
    q0, k0, v0 = block.qkv_rope(x, w, H, d, chunk=1, grid=None)
    np.testing.assert_array_equal(v, v0)
    assert np.abs(q - q0).max() > 1e-3 and np.abs(k - k0).max() > 1e-3
    np.testing.assert_allclose(np.linalg.norm(q, axis=-1), np.linalg.norm(q0, axis=-1), rtol=1e-12)


def test_gelu_odd_part_and_limits():
    x = np.linspace(-9, 9, 181)
    np.testing.assert_allclose(block.gelu_tanh(x) - block.gelu_tanh(-x), x, atol=1e-13)
    assert block.gelu_tanh(np.array(0.0)) == 0.0
    assert abs(block.gelu_tanh(np.array(12.0)) - 12.0) < 1e-12
    assert abs(block.gelu_tanh(np.array(-12.0))) < 1e-12


def test_gelu_tanh_close_to_erf_form():
    x = np.linspace(-6, 6, 1201)
    erf_form = np.array([0.5 * v * (1 + math.erf(v / math.sqrt(2))) for v in x])
    err = np.abs(block.gelu_tanh(x) - erf_form).max()
    assert 1e-5 < err < 1e-3  # the tanh form is an approximation, within 1e-3


def test_linear_brute_force_and_residual():
    rng = np.random.default_rng(5)
    M, K, N = 3, 4, 5
    x, w, r = rng.standard_normal((M, K)), rng.standard_normal((N, K)), rng.standard_normal((M, N))
    y = block.linear(x, w, residual=r)
    for i in range(M):
        for j in range(N):
            acc = r[i, j]
            for kk in range(K):
                acc += x[i, kk] * w[j, kk]
            assert abs(y[i, j] - acc) < 1e-12
    g = block.linear(x, w, act="gelu_tanh")
    np.testing.assert_allclose(g, block.gelu_tanh(x @ w.T), rtol=1e-14)


def test_out_proj_selection_weights():
    rng = np.random.default_rng(6)
    T, H, d = 4, 2, 3
    C = 5
    x = rng.standard_normal((T, C))
    a = rng.standard_normal((T, H, d))
    np.testing.assert_array_equal(block.out_proj(x, a, np.zeros((C, H * d))), x)
    wo = np.zeros((C, H * d))
    wo[2, 1 * d + 0] = 1.0  # output feature 2 copies head 1, component 0
    y = block.out_proj(x, a, wo)
    np.testing.assert_allclose(y[:, 2], x[:, 2] + a[:, 1, 0], rtol=1e-14)
    np.testing.assert_array_equal(np.delete(y, 2, axis=1), np.delete(x, 2, axis=1))


def test_mlp_zero_and_selection():
    rng = np.random.default_rng(7)
    T, C, F = 3, 4, 6
    y = rng.standard_normal((T, C))
    w1 = rng.standard_normal((F, C))
    np.testing.assert_array_equal(block.mlp(y, w1, np.zeros((C, F))), y)
    w1 = np.zeros((F, C))
    w1[0, 1] = 1.0
    w2 = np.zeros((C, F))
    w2[3, 0] = 1.0  # Z[:, 3] = Y[:, 3] + GELU(Y[:, 1])
    z = block.mlp(y, w1, w2, stored=False)
    np.testing.assert_allclose(z[:, 3], y[:, 3] + block.gelu_tanh(y[:, 1]), rtol=1e-14)


def test_bf16_round_matches_the_input_generator_and_ties_to_even():
    rng = np.random.default_rng(8)
    x = rng.standard_normal(10000).astype(np.float32)
    want = wi.bf16_bits_to_f64(wi.f32_to_bf16_bits(x))
    np.testing.assert_array_equal(block.bf16_round(x.astype(np.float64)), want)
    one = 1.0
    assert block.bf16_round(np.array(one + 2 ** -8)) == 1.0           # tie -> even
    assert block.bf16_round(np.array(one + 3 * 2 ** -8)) == one + 2 ** -6  # tie -> even
    assert block.bf16_round(np.array(one + 2 ** -8 + 2 ** -20)) == one + 2 ** -7
