"""Pins of oracle.projection against what fixes it independently of its code:
selection matrices (each output feature copies one input column), one-hot
inputs (each output row is a column of W), a brute-force triple loop on a tiny
case, and the Q/K/V and head order of the output features."""
import numpy as np

from oracle import projection


def test_selection_matrix_copies_columns():
    rng = np.random.default_rng(7)
    T, H, d = 5, 2, 4
    C = 3 * H * d
    x = rng.standard_normal((T, C))
    perm = rng.permutation(C)
    w = np.zeros((3 * H * d, C))
    w[np.arange(3 * H * d), perm] = 1.0  # feature f copies input column perm[f]
    q, k, v = projection.qkv(x, w, H, d)
    for s, out in enumerate((q, k, v)):
        for h in range(H):
            for j in range(d):
                f = (s * H + h) * d + j
                np.testing.assert_array_equal(out[:, h, j], x[:, perm[f]])


def test_one_hot_rows_give_weight_columns():
    rng = np.random.default_rng(8)
    T, H, d, C = 6, 3, 2, 6
    w = rng.standard_normal((3 * H * d, C))
    x = np.eye(C)[:T]
    q, k, v = projection.qkv(x, w, H, d)
    y = np.concatenate([q.reshape(T, -1), k.reshape(T, -1), v.reshape(T, -1)], axis=1)
    np.testing.assert_array_equal(y, w.T[:T])


def test_brute_force_loops():
    rng = np.random.default_rng(9)
    T, H, d, C = 3, 2, 3, 5
    x = rng.standard_normal((T, C))
    w = rng.standard_normal((3 * H * d, C))
    q, k, v = projection.qkv(x, w, H, d)
    outs = (q, k, v)
    for t in range(T):
        for s in range(3):
            for h in range(H):
                for j in range(d):
                    acc = 0.0
                    for c in range(C):
                        acc += x[t, c] * w[(s * H + h) * d + j, c]
                    assert abs(outs[s][t, h, j] - acc) < 1e-12
