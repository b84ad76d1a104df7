"""Wave-round attention in float64 -- oracle side.

Definition (Wave Forcing page, "Key Findings": chunk-wise causal attention over
earlier, cleaner chunks; Wan-Streamer v0.2 page, Figure 1 and glossary
"block-causal attention": full attention inside a block, causal across blocks;
design-space paper, Table 1 / Figure 1 for which level each history chunk is
read at). For an active node (c, l) and head h, with its key list
KL(c, l) = prefix + history E(c - r, phi(l, r)) + own E(c, l):

    O[q, h] = sum_k softmax_k(Q[q, h] . K[k, h] / sqrt(d)) V[k, h]

with every token of every listed entry visible (no mask inside a chunk). The
pages give no scale, bias or positional term; 1/sqrt(d) and none are used.
Computed with max subtraction in float64; inputs are the bf16 values widened.
"""
from __future__ import annotations

import math

import numpy as np

from .cache import key_entries


def attend(q: np.ndarray, k: np.ndarray, v: np.ndarray) -> np.ndarray:
    """softmax(q k^T / sqrt(d)) v per head. q [n, H, d], k/v [N, H, d], float64."""
    n, H, d = q.shape
    out = np.empty((n, H, v.shape[2]), dtype=np.float64)
    for h in range(H):
        s = q[:, h, :] @ k[:, h, :].T / math.sqrt(d)
        s = s - s.max(axis=1, keepdims=True)
        p = np.exp(s)
        out[:, h, :] = (p @ v[:, h, :]) / p.sum(axis=1, keepdims=True)
    return out


def node_keys(node, policy: str, window: int, entries: dict, prefix=None):
    """Concatenate the K and V of node's key list. ``entries`` maps (c, l) -> (K, V)."""
    ks, vs = [], []
    for e in key_entries(node, policy, window, prefix is not None):
        kv = prefix if e == (-1, 0) else entries[e]
        ks.append(kv[0])
        vs.append(kv[1])
    return np.concatenate(ks, axis=0), np.concatenate(vs, axis=0)


def round_attention(active, policy: str, window: int, q_by_node: dict,
                    entries: dict, prefix=None, rows=None):
    """O for every active node. ``rows`` optionally maps node -> query row indices."""
    out = {}
    for node in active:
        k, v = node_keys(node, policy, window, entries, prefix)
        q = q_by_node[node]
        if rows is not None and node in rows:
            q = q[rows[node]]
        out[node] = attend(q, k, v)
    return out


def flops(n_queries: int, n_keys: int, heads: int, head_dim: int) -> int:
    """Algorithmic FLOPs of one node: QK^T and PV, 2 flops per multiply-add each."""
    return 4 * n_queries * n_keys * heads * head_dim
