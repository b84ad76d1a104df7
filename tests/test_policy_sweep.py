"""Policy and level sweep (Wan2.1 shapes, K = 1..5): library report vs oracle
and closed forms (CPU only, host-only handle).

Closed forms (design-space paper, Figure 2): B+K-1 rounds for same-level and
progressive, B*K for clean, B*K updates in every case. With an unbounded
window a node of chunk c reads c history chunks plus its own, so an update of
chunk c costs 4*T*(c+1)*T*H*d FLOPs at every level and its refresh the same
once. Peak live entries come from the oracle's allocator simulation.
"""
import pytest

from oracle import cache as ocache
from oracle import schedule as osched

wave = pytest.importorskip("block_causal_attention_wave_b200")
from block_causal_attention_wave_b200 import sweep  # noqa: E402

B, T, H, D = 7, 4680, 12, 128


def _oracle_peak_entries(K, pol):
    rounds = osched.schedule(B, K, pol)
    last = osched.last_read_round(B, K, pol)
    pool = ocache.PagePoolModel(10_000)
    peak = 0
    for t, active in enumerate(rounds):
        for n in active:
            pool.alloc(n, T)
        peak = max(peak, len(pool.entries))
        for e in [e for e, lr in last.items() if lr == t]:
            pool.release(e)
    return peak


@pytest.mark.parametrize("pol", ["clean", "same", "progressive"])
@pytest.mark.parametrize("K", [1, 2, 3, 4, 5])
def test_sweep_row(pol, K):
    wave.load()
    r = sweep.sweep_one(B, K, pol, T, H, D)
    assert r["rounds"] == (B * K if pol == "clean" else B + K - 1)
    assert r["updates"] == B * K
    unit = 4 * T * T * H * D / 1e12
    for c in range(B):
        assert abs(r["update_tflop_per_chunk"][c] - round(K * (c + 1) * unit, 4)) < 1e-3
        has_refresh = pol != "same" and c < B - 1
        want = round((c + 1) * unit, 4) if has_refresh else 0.0
        assert abs(r["refresh_tflop_per_chunk"][c] - want) < 1e-3
    assert r["refreshes"] == (0 if pol == "same" else B - 1)
    assert r["peak_entries"] == _oracle_peak_entries(K, pol)
    pages = (T + 127) // 128
    assert r["peak_cache_bytes_per_layer"] == r["peak_entries"] * pages * 2 * H * 128 * D * 2
