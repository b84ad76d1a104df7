"""GPU parity of one transformer block of a wave round: the round's QKV
projection with the rotary embedding and the K/V append fused in
(wave_qkv_append_round), the dense layers (wave_linear: out-projection with
residual, tanh-GELU MLP up, MLP down with residual), and a whole block rollout
(projection -> attention -> out-projection -> MLP) against the float64
oracle chain with bf16 storage between kernels.

Each kernel is compared with the oracle on the kernel's own bf16 inputs:
every element on small cases spanning several 128 x 256 tiles with ragged
row tails, sampled rows at the Wan2.1-1.3B shapes. Bar: max-abs <= 1e-2 x
max(1, max|ref|) (outputs are bf16, whose rounding is 2^-9 of |value|) and
relative L2 <= 5e-3; page tails exactly zero.
"""
import numpy as np
import pytest

import wave_inputs as wi
from oracle import attention as oatt
from oracle import block as oblock
from oracle import cache as ocache
from oracle import schedule as osched

from wave_testlib import assert_close, bits_to_torch, read_entry, torch_to_f64

pytestmark = pytest.mark.gpu


def _cache(wave, heads, head_dim, tokens, levels, pages, window=0):
    import torch
    pb = wave.KVCache.page_bytes(heads, head_dim)
    pool = torch.empty(4096 + pages * pb, dtype=torch.uint8, device="cuda")
    return wave.KVCache(heads, head_dim, tokens, levels, window, 0, pool=pool), pool


@pytest.mark.parametrize("M,K,N,act,resid", [
    (300, 192, 512, "none", False),
    (300, 192, 512, "none", True),
    (257, 128, 768, "gelu", False),
    (129, 320, 256, "gelu", True),
    (128, 64, 256, "none", True),
])
def test_linear_small_every_element(cuda_lib, M, K, N, act, resid):
    import torch
    wave = cuda_lib
    kv, _ = _cache(wave, 2, 128, 128, 1, 1)
    a_b = wi.normal_bf16(77, (M, K))
    w_b = wi.normal_bf16(78, (N, K), 1.0 / np.sqrt(K))
    r_b = wi.normal_bf16(79, (M, N)) if resid else None
    A, W = bits_to_torch(a_b), bits_to_torch(w_b)
    R = bits_to_torch(r_b) if resid else None
    Y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    kv.linear(A, W, Y, R=R, act=wave.ACT_GELU_TANH if act == "gelu" else wave.ACT_NONE)
    kv.status()
    ref = oblock.linear(wi.bf16_bits_to_f64(a_b), wi.bf16_bits_to_f64(w_b),
                        residual=wi.bf16_bits_to_f64(r_b) if resid else None,
                        act="gelu_tanh" if act == "gelu" else None)
    assert_close(torch_to_f64(Y), ref, f"linear M{M} K{K} N{N} {act} resid={resid}",
                 scale_with_output=True)


def test_linear_in_place_residual(cuda_lib):
    """Y may be the residual buffer itself (Z = Y + U W2^T in place)."""
    wave = cuda_lib
    kv, _ = _cache(wave, 2, 128, 128, 1, 1)
    M, K, N = 200, 128, 512
    a_b, w_b, r_b = (wi.normal_bf16(81, (M, K)), wi.normal_bf16(82, (N, K), 1 / np.sqrt(K)),
                     wi.normal_bf16(83, (M, N)))
    R = bits_to_torch(r_b)
    kv.linear(bits_to_torch(a_b), bits_to_torch(w_b), R, R=R)
    kv.status()
    ref = oblock.linear(wi.bf16_bits_to_f64(a_b), wi.bf16_bits_to_f64(w_b),
                        residual=wi.bf16_bits_to_f64(r_b))
    assert_close(torch_to_f64(R), ref, "in-place residual", scale_with_output=True)


def _sample_rows(M, n=48):
    rows = np.unique(np.concatenate([np.linspace(0, M - 1, n).astype(int), [M - 1, M - 2]]))
    return rows


@pytest.mark.parametrize("which", ["out_proj", "mlp_up", "mlp_down"])
def test_linear_wan21_round_sampled_rows(cuda_lib, which):
    """The block's dense layers at the Wan2.1-1.3B shapes over a whole round
    (5 nodes x 4680 tokens = 23400 rows; C 1536, MLP 8960), sampled rows."""
    import torch
    wave = cuda_lib
    kv, _ = _cache(wave, 12, 128, 4680, 4, 1)
    M = 5 * 4680
    C, F = wi.WAN21_DIM, wi.WAN21_MLP
    K, N, act, resid, wname = {
        "out_proj": (C, C, None, True, "wo"),
        "mlp_up": (C, F, "gelu_tanh", False, "w1"),
        "mlp_down": (F, C, None, True, "w2"),
    }[which]
    a_b = wi.normal_bf16(90, (M, K))
    w_b = wi.block_weight(wname, N, K)
    r_b = wi.normal_bf16(91, (M, N)) if resid else None
    Y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    kv.linear(bits_to_torch(a_b), bits_to_torch(w_b), Y,
              R=bits_to_torch(r_b) if resid else None,
              act=wave.ACT_GELU_TANH if act else wave.ACT_NONE)
    kv.status()
    rows = _sample_rows(M)
    ref = oblock.linear(wi.bf16_bits_to_f64(a_b[rows]), wi.bf16_bits_to_f64(w_b),
                        residual=wi.bf16_bits_to_f64(r_b[rows]) if resid else None, act=act)
    assert_close(torch_to_f64(Y[torch.as_tensor(rows, device="cuda")]), ref, which,
                 scale_with_output=True)


def _check_qkv_round(wave, kv, pool, nodes, xs_b, w_b, grid, heads, d, T, Q, rows=None):
    for i, n in enumerate(nodes):
        x = wi.bf16_bits_to_f64(xs_b[i] if rows is None else xs_b[i][rows])
        q, k, v = oblock.qkv_rope(x, wi.bf16_bits_to_f64(w_b), heads, d, n[0], None)
        if grid is not None:
            ang = oblock.rope_angles(n[0], *grid, d)
            if rows is not None:
                ang = ang[rows]
            q, k = oblock.apply_rope(q, ang), oblock.apply_rope(k, ang)
        got_q = torch_to_f64(Q[i * T:(i + 1) * T]).reshape(T, heads, d)
        gk, gv, tail0 = read_entry(kv, pool, n, T)
        if rows is not None:
            got_q, gk, gv = got_q[rows], gk[rows], gv[rows]
        assert tail0, f"node {n}: page tail not zero"
        assert_close(got_q, q, f"Q of {n}", scale_with_output=True)
        assert_close(gk, k, f"K of {n}", scale_with_output=True)
        assert_close(gv, v, f"V of {n}", scale_with_output=True)


@pytest.mark.parametrize("grid", [(3, 10, 10), None], ids=["rope", "no-rope"])
def test_qkv_round_small_every_element(cuda_lib, grid):
    """Three nodes of 300 tokens (3 pages each, ragged tail), H 2, d 128,
    C 256: Q, K and V of every node, every element, against the oracle's
    projection and rotary embedding; pages as wave_kv_alloc would take them."""
    import torch
    wave = cuda_lib
    H, d, T, C = 2, 128, 300, 256
    kv, pool = _cache(wave, H, d, T, 3, 16)
    nodes = [(2, 1), (1, 2), (0, 3)]
    xs_b = [wi.hidden_states(c, l, T, C) for c, l in nodes]
    w_b = wi.qkv_weight(H, d, C)
    X = torch.cat([bits_to_torch(x) for x in xs_b])
    Q = torch.full((3 * T, H, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    kv.qkv_append_round(nodes, X, bits_to_torch(w_b), Q, rope=grid)
    kv.status()
    assert [kv.entry_pages(*n) for n in nodes] == [[0, 1, 2], [3, 4, 5], [6, 7, 8]]
    _check_qkv_round(wave, kv, pool, nodes, xs_b, w_b, grid, H, d, T, Q)


def test_qkv_round_errors_leave_no_pages(cuda_lib):
    import torch
    wave = cuda_lib
    H, d, T, C = 2, 128, 300, 256
    kv, _ = _cache(wave, H, d, T, 3, 16)
    X = torch.zeros((2 * T, C), dtype=torch.bfloat16, device="cuda")
    W = torch.zeros((3 * H * d, C), dtype=torch.bfloat16, device="cuda")
    Q = torch.empty((2 * T, H, d), dtype=torch.bfloat16, device="cuda")
    free0 = kv.free_pages()
    with pytest.raises(wave.WaveError):  # grid does not cover T
        kv.qkv_append_round([(0, 1), (1, 1)], X, W, Q, rope=(3, 10, 11))
    kv.alloc(1, 1)
    with pytest.raises(wave.WaveError):  # (1, 1) exists: nothing else stays taken
        kv.qkv_append_round([(0, 1), (1, 1)], X, W, Q, rope=(3, 10, 10))
    kv.release(1, 1)
    assert kv.free_pages() == free0


def test_qkv_round_wan21_sampled_rows(cuda_lib):
    """Round 6 of the Wan2.1-1.3B schedule: 5 nodes x 4680 tokens, C 1536,
    12 heads, rotary grid 3 x 30 x 52, one launch; sampled token rows."""
    import torch
    wave = cuda_lib
    H, d, T, C = 12, 128, 4680, wi.WAN21_DIM
    kv, pool = _cache(wave, H, d, T, 4, 5 * 37 + 4)
    nodes = osched.schedule(7, 4, "progressive", 0)[6]
    xs_b = [wi.hidden_states(c, l, T, C) for c, l in nodes]
    w_b = wi.qkv_weight(H, d, C)
    X = torch.cat([bits_to_torch(x) for x in xs_b])
    Q = torch.empty((len(nodes) * T, H, d), dtype=torch.bfloat16, device="cuda")
    kv.qkv_append_round(nodes, X, bits_to_torch(w_b), Q, rope=wi.WAN21_GRID)
    kv.status()
    rows = _sample_rows(T, 24)
    _check_qkv_round(wave, kv, pool, nodes, xs_b, w_b, wi.WAN21_GRID, H, d, T, Q, rows)


def test_block_rollout_small_every_round(cuda_lib):
    """A whole rollout of one transformer block through the library: per
    round, the nodes' projection (rotary, K/V into the cache, one launch), the
    wave-round attention, the out-projection with the residual and the MLP,
    checked every element against the oracle chain (bf16 storage between the
    kernels) in every round. 3 chunks, 2 levels, progressive; H 2, d 128,
    160 tokens (2 frames of 8 x 10), C 256, MLP 512."""
    import torch
    wave = cuda_lib
    B, Kl, H, d, C, Fm = 3, 2, 2, 128, 256, 512
    grid = (2, 8, 10)
    T = grid[0] * grid[1] * grid[2]
    pol = "progressive"
    kv, _ = _cache(wave, H, d, T, Kl, 40)
    wq_b, wo_b = wi.qkv_weight(H, d, C), wi.block_weight("wo", C, H * d)
    w1_b, w2_b = wi.block_weight("w1", Fm, C), wi.block_weight("w2", C, Fm)
    Wq, Wo, W1, W2 = (bits_to_torch(b) for b in (wq_b, wo_b, w1_b, w2_b))
    wq, wo, w1, w2 = (wi.bf16_bits_to_f64(b) for b in (wq_b, wo_b, w1_b, w2_b))
    rounds = wave.schedule(B, Kl, pol)
    last = wave.last_read_rounds(B, Kl, pol)
    ents = {}  # oracle cache: (chunk, level) -> (K, V) as stored (bf16)
    rb = oblock.bf16_round
    for t, active in enumerate(rounds):
        xs_b = [wi.hidden_states(c, l, T, C) for c, l in active]
        X = torch.cat([bits_to_torch(x) for x in xs_b])
        n = len(active)
        Q = torch.empty((n * T, H, d), dtype=torch.bfloat16, device="cuda")
        A = torch.empty_like(Q)
        Y = torch.empty((n * T, C), dtype=torch.bfloat16, device="cuda")
        U = torch.empty((n * T, Fm), dtype=torch.bfloat16, device="cuda")
        kv.qkv_append_round(active, X, Wq, Q, rope=grid)
        kv.round_attn(active, pol, Q, A)
        kv.linear(A.view(n * T, H * d), Wo, Y, R=X)
        kv.linear(Y, W1, U, act=wave.ACT_GELU_TANH)
        kv.linear(U, W2, Y, R=Y)  # Z in place of Y
        kv.status()
        got = torch_to_f64(Y)
        # oracle chain
        qs = {}
        for i, node in enumerate(active):
            q, k, v = oblock.qkv_rope(wi.bf16_bits_to_f64(xs_b[i]), wq, H, d, node[0], grid)
            qs[node] = rb(q)
            ents[node] = (rb(k), rb(v))
        outs = oatt.round_attention(active, pol, 0, qs, ents)
        for i, node in enumerate(active):
            x = wi.bf16_bits_to_f64(xs_b[i])
            a = rb(outs[node])
            y = rb(oblock.out_proj(x, a, wo))
            z = oblock.mlp(y, w1, w2, stored=True)
            assert_close(got[i * T:(i + 1) * T], z, f"round {t} node {node} block output",
                         scale_with_output=True)
        for e in sorted(e for e, lr in last.items() if lr == t):
            kv.release(*e)
    torch.cuda.synchronize()
