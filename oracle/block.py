"""One transformer block of a concurrent forward round, in float64 -- oracle side.

TEST INFRASTRUCTURE ONLY (see the package docstring): nothing on the product
path imports this module.

In one concurrent forward round every active (chunk, level) node runs the same
block of the denoiser: its hidden states are projected to Q, K and V, its K and
V join the cache (in-round delivery), the wave-round attention runs over each
node's key list, and the attention output goes through the out-projection and
the MLP (Wave Forcing page, "Key Findings": one output chunk per concurrent
forward round after pipeline fill, early K/V delivery; design-space paper,
abstract: multiple denoising nodes processed together). The pages give no
formula for the block itself. Readings used here, each the plainest one the
rest of the pages supports:

* Projection: [Q | K | V] = X Wqkv^T (``projection.qkv``), no bias.
* Rotary position embedding on Q and K, per head, with three position axes of
  a video latent: frame, row, column. A token t of chunk c, on a grid of F
  frames x R rows x W columns (T = F R W tokens per chunk), sits at frame
  c F + t // (R W), row (t // W) mod R, column t mod W. The d/2 rotation pairs
  of a head (elements 2p, 2p+1) are split into three consecutive groups: the
  frame axis takes the first P - 2 (P // 3) pairs, then rows and columns
  P // 3 each (P = d/2). Pair i of a group of n pairs turns by
  position * base^(-i / n) radians (base 10000):
  (a, b) -> (a cos - b sin, a sin + b cos).
  K is stored in the cache after the rotation.
* Out-projection with the residual: Y = X + A Wo^T, A the attention output
  [T][H d], Wo [C][H d].
* MLP with the residual: Z = Y + GELU(Y W1^T) W2^T, W1 [F][C], W2 [C][F],
  GELU in its tanh form 0.5 x (1 + tanh(sqrt(2/pi) (x + 0.044715 x^3))).
* No normalisation, modulation or bias terms: they are elementwise steps off
  the attention path, left out of this block.
* Storage precision: every tensor that the block hands from one kernel to the
  next (Q, K, V, the attention output, Y, the MLP hidden U and Z) is stored in
  bfloat16 (round to nearest even); arithmetic in between is exact here.
"""
from __future__ import annotations

import math

import numpy as np

from . import projection

ROPE_BASE = 10000.0


def bf16_round(x: np.ndarray) -> np.ndarray:
    """Round float64 values to bfloat16 (nearest, ties to even), as float64.

    Rounds to float32 first (numpy's cast is round-to-nearest-even), then keeps
    the top 16 bits with round-to-nearest-even on the dropped 16.
    """
    f = np.ascontiguousarray(x, dtype=np.float64).astype(np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    u = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16) << 16
    return u.astype(np.uint32).view(np.float32).astype(np.float64)


def rope_groups(head_dim: int):
    """Pairs per axis (frame, row, column) for a head of ``head_dim``."""
    p = head_dim // 2
    n_hw = p // 3
    return p - 2 * n_hw, n_hw, n_hw


def rope_angles(chunk: int, frames: int, rows: int, cols: int, head_dim: int,
                base: float = ROPE_BASE) -> np.ndarray:
    """Rotation angle of every (token, pair) of one chunk: [T][d/2] float64."""
    n_t, n_h, n_w = rope_groups(head_dim)
    T = frames * rows * cols
    tok = np.arange(T)
    pos = [chunk * frames + tok // (rows * cols), (tok // cols) % rows, tok % cols]
    ang = np.zeros((T, head_dim // 2))
    p0 = 0
    for axis, n in enumerate((n_t, n_h, n_w)):
        for i in range(n):
            ang[:, p0 + i] = pos[axis] * base ** (-i / n)
        p0 += n
    return ang


def apply_rope(x: np.ndarray, angles: np.ndarray) -> np.ndarray:
    """Rotate the pairs of x [T][H][d] by angles [T][d/2] (same for every head)."""
    a = x[..., 0::2]
    b = x[..., 1::2]
    c = np.cos(angles)[:, None, :]
    s = np.sin(angles)[:, None, :]
    out = np.empty_like(x, dtype=np.float64)
    out[..., 0::2] = a * c - b * s
    out[..., 1::2] = a * s + b * c
    return out


def qkv_rope(x, w, heads, head_dim, chunk, grid, base=ROPE_BASE):
    """Q, K, V [T][H][d] of one node: projection, then rotation of Q and K.
    ``grid`` = (frames, rows, cols) with frames * rows * cols = T, or None for
    no rotation."""
    q, k, v = projection.qkv(x, w, heads, head_dim)
    if grid is not None:
        ang = rope_angles(chunk, *grid, head_dim, base)
        q, k = apply_rope(q, ang), apply_rope(k, ang)
    return q, k, v


def gelu_tanh(x: np.ndarray) -> np.ndarray:
    """GELU, tanh form."""
    x = np.asarray(x, dtype=np.float64)
    return 0.5 * x * (1.0 + np.tanh(math.sqrt(2.0 / math.pi) * (x + 0.044715 * x ** 3)))


def linear(x, w, residual=None, act=None):
    """y = act(x W^T) (+ residual): x [M][K], w [N][K], residual [M][N]."""
    y = np.asarray(x, dtype=np.float64) @ np.asarray(w, dtype=np.float64).T
    if act == "gelu_tanh":
        y = gelu_tanh(y)
    elif act is not None:
        raise ValueError(f"unknown activation {act!r}")
    if residual is not None:
        y = y + np.asarray(residual, dtype=np.float64)
    return y


def out_proj(x, a, wo):
    """Y = X + A Wo^T for x [T][C], a [T][H][d] (or [T][H d]), wo [C][H d]."""
    return linear(a.reshape(a.shape[0], -1), wo, residual=x)


def mlp(y, w1, w2, stored=True):
    """Z = Y + GELU(Y W1^T) W2^T; with ``stored`` the hidden U is rounded to
    bfloat16 between the two matrices, as the block stores it."""
    u = linear(y, w1, act="gelu_tanh")
    if stored:
        u = bf16_round(u)
    return linear(u, w2, residual=y)
