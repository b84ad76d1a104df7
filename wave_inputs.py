"""Seeded synthetic inputs shared by the CUDA path's tests/bench and the oracle.

This module holds data generation only: random draws, the float32 -> bfloat16
storage conversion, and the workload shapes. None of the attention, policy or
scheduling arithmetic lives here, so neither side can borrow the other's maths
through it.

Recipe (one stream per tensor): ``numpy.random.Generator(PCG64(seed))``,
``standard_normal(float32)``, optionally multiplied by ``scale``, then rounded
to bfloat16 with round-to-nearest-even. The seed is ``1234 + tensor_id`` where
the id encodes (kind, chunk, level); chunk -1 is the conditioning prefix.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

SEED_BASE = 1234
_KINDS = {"q": 0, "k": 1, "v": 2}


def tensor_id(kind: str, chunk: int, level: int) -> int:
    """Stable id of one synthetic tensor: the Q, K or V of (chunk, level)."""
    if kind not in _KINDS:
        raise ValueError(f"kind must be q/k/v, got {kind!r}")
    if chunk < -1 or not (0 <= level < 64):
        raise ValueError(f"bad (chunk, level) = ({chunk}, {level})")
    return ((chunk + 1) * 64 + level) * 3 + _KINDS[kind]


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> bfloat16 bit patterns (uint16), round to nearest, ties to even."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    r = (u + 0x7FFF + lsb) >> 16
    return r.astype(np.uint16)


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """bfloat16 bit patterns -> exact float64 values."""
    u = bits.astype(np.uint32) << 16
    return u.view(np.float32).astype(np.float64)


def normal_bf16(seed: int, shape, scale: float = 1.0) -> np.ndarray:
    """bf16 bit patterns of ``scale * N(0, 1)`` drawn from one PCG64 stream."""
    g = np.random.Generator(np.random.PCG64(seed))
    x = g.standard_normal(size=shape, dtype=np.float32)
    if scale != 1.0:
        x = x * np.float32(scale)
    return f32_to_bf16_bits(x)


PROJ_SEED_BASE = SEED_BASE + 1_000_000  # projection inputs: disjoint from the ids above


def hidden_states(chunk: int, level: int, tokens: int, dim: int) -> np.ndarray:
    """``[tokens][dim]`` bf16 bits of N(0, 1): a node's hidden states (projection input)."""
    return normal_bf16(PROJ_SEED_BASE + tensor_id("q", chunk, level), (tokens, dim))


def qkv_weight(heads: int, head_dim: int, dim: int) -> np.ndarray:
    """``[3 * heads * head_dim][dim]`` bf16 bits of N(0, 1) / sqrt(dim): a random
    QKV projection weight in a linear layer's [out][in] layout."""
    return normal_bf16(PROJ_SEED_BASE - 1, (3 * heads * head_dim, dim), 1.0 / math.sqrt(dim))


_BLOCK_WEIGHTS = {"wo": 2, "w1": 3, "w2": 4}


def block_weight(name: str, out_dim: int, in_dim: int) -> np.ndarray:
    """``[out_dim][in_dim]`` bf16 bits of N(0, 1) / sqrt(in_dim): a random weight
    of the block's out-projection ("wo") or MLP ("w1", "w2"), [out][in] layout."""
    return normal_bf16(PROJ_SEED_BASE - _BLOCK_WEIGHTS[name], (out_dim, in_dim),
                       1.0 / math.sqrt(in_dim))


# Wan2.1-1.3B block: hidden size 1536 (12 heads x 128), MLP width 8960; a chunk
# is 3 latent frames of 30 x 52 patch tokens.
WAN21_DIM, WAN21_MLP = 1536, 8960
WAN21_GRID = (3, 30, 52)


def node_tensor(kind: str, chunk: int, level: int, tokens: int, heads: int,
                head_dim: int, scale: float = 1.0) -> np.ndarray:
    """Token-major ``[tokens][heads][head_dim]`` bf16 bits for one (chunk, level)."""
    seed = SEED_BASE + tensor_id(kind, chunk, level)
    return normal_bf16(seed, (tokens, heads, head_dim), scale)


@dataclasses.dataclass(frozen=True)
class Workload:
    """Shape of one workload. ``window`` 0 means unbounded history."""
    name: str
    chunks: int            # B
    levels: int            # K (update levels K..1, level 0 = clean)
    heads: int             # H
    head_dim: int          # d
    tokens: int            # T, tokens per chunk (or per streaming unit)
    window: int = 0        # W, history window in chunks; 0 = unbounded
    prefix: int = 0        # conditioning K/V prefix tokens (always visible)
    policy: str = "progressive"
    scale: float = 1.0     # multiplier on N(0,1) before bf16 rounding


# Tiny case: 3 chunks, 2 levels, 2 heads, d=64, 2 latent frames of 4x4 = 32 tokens.
TINY = Workload("tiny", chunks=3, levels=2, heads=2, head_dim=64, tokens=32)

# Wan2.1-1.3B-shaped round: 832x480 -> 104x60 latent -> 52x30 patches = 1560
# tokens per latent frame, 3 frames per chunk, 7 chunks, 4 levels, 12 heads, d=128.
WAN21 = Workload("wan2.1-1.3b", chunks=7, levels=4, heads=12, head_dim=128,
                 tokens=3 * 1560, policy="progressive", scale=1.0 / math.sqrt(128.0))

# Wan-Streamer-shaped unit: 640x368 /16 = 40x23 = 920 video tokens + 64 audio
# tokens per 160 ms unit, 512-token conditioning prefix, 24 heads, 32-unit window.
WAN_STREAMER = Workload("wan-streamer", chunks=40, levels=2, heads=24, head_dim=128,
                        tokens=920 + 64, window=32, prefix=512, policy="progressive")

# Long rollout: 40 chunks of 3 latent frames, 6-chunk window, 5 levels.
LONG_ROLLOUT = Workload("long-rollout", chunks=40, levels=5, heads=12, head_dim=128,
                        tokens=3 * 1560, window=6, policy="progressive")

POLICIES = ("clean", "same", "progressive")
