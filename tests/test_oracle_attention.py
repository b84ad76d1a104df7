"""Pins for the oracle's float64 attention (CPU only).

Expected values come from outside the oracle:
* brute force: the whole timeline of cached (chunk, level) states as one key
  sequence with an explicit 0 / -inf mask, plain softmax;
* torch's CPU scaled_dot_product_attention (float64) with a block-causal mask,
  which the clean policy's refresh nodes must reproduce;
* closed-form invariants: one key returns V, identical keys return mean(V),
  V = 1 returns 1, history order does not matter, progressive = clean at K = 1,
  same-level = clean when every level holds the same tensor.
"""
import math

import numpy as np
import pytest
import torch

import wave_inputs as wi
from oracle import attention, policy, schedule


def _entry(kind, c, l, T, H, d, scale=1.0):
    return wi.bf16_bits_to_f64(wi.node_tensor(kind, c, l, T, H, d, scale))


def _make_entries(B, K, pol, W, T, H, d, prefix_tokens=0):
    rounds = schedule.schedule(B, K, pol, W)
    ents = {}
    qs = {}
    for r in rounds:
        for n in r:
            ents[n] = (_entry("k", *n, T, H, d), _entry("v", *n, T, H, d))
            qs[n] = _entry("q", *n, T, H, d)
    pre = None
    if prefix_tokens:
        pre = (_entry("k", -1, 0, prefix_tokens, H, d), _entry("v", -1, 0, prefix_tokens, H, d))
    return rounds, ents, qs, pre


def _brute(node, pol, W, ents, q, pre):
    """Dense masked softmax over every cached state; visibility as a predicate."""
    labels, ks, vs = [], [], []
    if pre is not None:
        labels += [("prefix",)] * pre[0].shape[0]
        ks.append(pre[0])
        vs.append(pre[1])
    for e in sorted(ents):
        labels += [e] * ents[e][0].shape[0]
        ks.append(ents[e][0])
        vs.append(ents[e][1])
    k = np.concatenate(ks)
    v = np.concatenate(vs)
    c, l = node

    def visible(lab):
        if lab == ("prefix",):
            return True
        cc, ll = lab
        if (cc, ll) == (c, l):
            return True
        if cc >= c:
            return False
        r = c - cc
        if W > 0 and r > W:
            return False
        return ll == policy.phi(pol, l, r)

    mask = np.array([0.0 if visible(lab) else -np.inf for lab in labels])
    d = q.shape[2]
    out = np.empty_like(q)
    for h in range(q.shape[1]):
        s = q[:, h, :] @ k[:, h, :].T / math.sqrt(d) + mask[None, :]
        w = np.exp(s - s.max(axis=1, keepdims=True))
        w /= w.sum(axis=1, keepdims=True)
        out[:, h, :] = w @ v[:, h, :]
    return out


@pytest.mark.parametrize("pol", ["clean", "same", "progressive"])
@pytest.mark.parametrize("W,prefix", [(0, 0), (1, 0), (0, 8), (2, 8)])
def test_oracle_matches_dense_mask_brute_force(pol, W, prefix):
    B, K, T, H, d = 4, 3, 8, 2, 16
    rounds, ents, qs, pre = _make_entries(B, K, pol, W, T, H, d, prefix)
    for r in rounds:
        got = attention.round_attention(r, pol, W, qs, ents, pre)
        for n in r:
            want = _brute(n, pol, W, ents, qs[n], pre)
            np.testing.assert_allclose(got[n], want, rtol=0, atol=1e-12)


def test_brute_force_detects_a_dropped_history_chunk():
    # A plausible oracle mistake (own chunk only, history dropped) must fail.
    B, K, T, H, d = 3, 2, 8, 2, 16
    rounds, ents, qs, pre = _make_entries(B, K, "progressive", 0, T, H, d)
    n = (2, 2)
    wrong = attention.attend(qs[n], *ents[n])
    assert np.abs(wrong - _brute(n, "progressive", 0, ents, qs[n], pre)).max() > 1e-3


@pytest.mark.parametrize("W", [0, 2])
def test_clean_refresh_nodes_equal_block_causal_sdpa(W):
    # Clean history with one level: the refresh of chunk c attends to the clean
    # chunks c-W..c in full -- plain block-causal attention over the clean video.
    B, K, T, H, d = 5, 1, 6, 3, 32
    rounds, ents, qs, pre = _make_entries(B, K, "clean", W, T, H, d)
    seq_k = np.concatenate([ents[(c, 0)][0] for c in range(B - 1)])
    seq_v = np.concatenate([ents[(c, 0)][1] for c in range(B - 1)])
    seq_q = np.concatenate([qs[(c, 0)] for c in range(B - 1)])
    blk = np.arange((B - 1) * T) // T
    allowed = blk[None, :] <= blk[:, None]
    if W > 0:
        allowed &= blk[None, :] >= blk[:, None] - W
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(seq_q).permute(1, 0, 2), torch.from_numpy(seq_k).permute(1, 0, 2),
        torch.from_numpy(seq_v).permute(1, 0, 2), attn_mask=torch.from_numpy(allowed)
    ).permute(1, 0, 2).numpy()
    for r in rounds:
        got = attention.round_attention(r, "clean", W, qs, ents)
        for (c, l) in r:
            if l == 0:
                np.testing.assert_allclose(got[(c, l)], ref[c * T:(c + 1) * T], atol=1e-12)


def test_single_key_returns_v():
    q = np.random.default_rng(0).standard_normal((5, 2, 8))
    k = np.random.default_rng(1).standard_normal((1, 2, 8))
    v = np.random.default_rng(2).standard_normal((1, 2, 8))
    out = attention.attend(q, k, v)
    np.testing.assert_allclose(out, np.broadcast_to(v, out.shape), atol=1e-15)


def test_identical_keys_return_mean_v():
    rng = np.random.default_rng(3)
    q = rng.standard_normal((7, 2, 8))
    k = np.broadcast_to(rng.standard_normal((1, 2, 8)), (11, 2, 8)).copy()
    v = rng.standard_normal((11, 2, 8))
    out = attention.attend(q, k, v)
    np.testing.assert_allclose(out, np.broadcast_to(v.mean(axis=0), out.shape), atol=1e-13)


def test_unit_values_give_unit_output():
    rng = np.random.default_rng(4)
    out = attention.attend(rng.standard_normal((9, 3, 16)) * 5, rng.standard_normal((40, 3, 16)) * 5,
                           np.ones((40, 3, 16)))
    np.testing.assert_allclose(out, 1.0, atol=1e-13)


def test_scale_is_inverse_sqrt_head_dim():
    # two keys, scores differ by exactly sqrt(d) * 1 -> weights e/(1+e), 1/(1+e)
    d = 16
    q = np.zeros((1, 1, d)); q[0, 0, 0] = math.sqrt(d)
    k = np.zeros((2, 1, d)); k[0, 0, 0] = 1.0
    v = np.array([[[1.0] + [0.0] * (d - 1)], [[0.0] * d]])
    out = attention.attend(q, k, v)
    assert abs(out[0, 0, 0] - math.e / (1 + math.e)) < 1e-15


def test_history_order_does_not_matter():
    B, K, T, H, d = 4, 2, 8, 2, 16
    rounds, ents, qs, pre = _make_entries(B, K, "progressive", 0, T, H, d)
    n = (3, 2)
    k, v = attention.node_keys(n, "progressive", 0, ents)
    perm = np.random.default_rng(5).permutation(k.shape[0])
    np.testing.assert_allclose(attention.attend(qs[n], k[perm], v[perm]),
                               attention.attend(qs[n], k, v), atol=1e-12)


def test_progressive_equals_clean_with_one_level():
    B, K, T, H, d = 4, 1, 8, 2, 16
    rounds, ents, qs, pre = _make_entries(B, K, "progressive", 0, T, H, d)
    for r in rounds:
        a = attention.round_attention(r, "progressive", 0, qs, ents)
        b = attention.round_attention(r, "clean", 0, qs, ents)
        for n in r:
            np.testing.assert_array_equal(a[n], b[n])


def test_same_level_equals_clean_when_levels_hold_the_same_tensor():
    B, K, T, H, d = 4, 3, 8, 2, 16
    rounds, ents, qs, pre = _make_entries(B, K, "same", 0, T, H, d)
    for c in range(B):
        for l in range(0, K + 1):
            ents[(c, l)] = (_entry("k", c, 0, T, H, d), _entry("v", c, 0, T, H, d))
    for r in rounds:
        a = attention.round_attention(r, "same", 0, qs, ents)
        b = attention.round_attention(r, "clean", 0, qs, ents)
        for n in r:
            np.testing.assert_allclose(a[n], b[n], atol=1e-13)


def test_flops_closed_form():
    # Wan2.1-shaped round 6: nodes (2,0),(3,1),(4,2),(5,3),(6,4) read 3..7 chunks.
    T, H, d = 4680, 12, 128
    upd = sum(attention.flops(T, n * T, H, d) for n in (4, 5, 6, 7))
    ref = attention.flops(T, 3 * T, H, d)
    assert abs(upd / 1e12 - 2.9605) < 1e-4 and abs(ref / 1e12 - 0.4037) < 1e-4
