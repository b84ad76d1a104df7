"""QKV projection of one node's tokens in float64 -- oracle side.

A node's forward pass produces its Q, K and V from its hidden states; its K and
V are what in-round delivery hands to the other nodes of the round (Wave
Forcing page, "Key Findings": early K/V delivery; Wan-Streamer v0.2 page,
glossary "pre-sharded": incoming K/V written into a local cache). The pages
give no formula for the projection itself. Reading used: the plain linear map
of a multi-head attention layer, no bias, no positional or normalisation term:

    Y = X W^T,  X [T][C], W [3 H d][C]  (the [out][in] layout of a linear layer)

with output feature f = (s * H + h) * d + j giving Q (s = 0), K (s = 1) or
V (s = 2) of head h, component j.
"""
from __future__ import annotations

import numpy as np


def qkv(x: np.ndarray, w: np.ndarray, heads: int, head_dim: int):
    """(Q, K, V), each [T][H][d] float64, from x [T][C] and w [3 H d][C]."""
    t = x.shape[0]
    y = x.astype(np.float64) @ w.astype(np.float64).T
    y = y.reshape(t, 3, heads, head_dim)
    return y[:, 0], y[:, 1], y[:, 2]
