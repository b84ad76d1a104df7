"""The attention kernel's barrier protocol, checked on an executable model.

tests/attn_protocol_model.py restates the roles of round_attn_kernel (TMA
producer, the two MMA issuing threads, the ring watcher, eight softmax warps)
with the kernel's counters, waits, arrivals and commits, and runs them under a
seeded random interleaving against a model of mbarrier phases, an in-order
tensor pipe and delayed copies. These tests run many interleavings:
- the protocol as built finishes every random item mix, single-tile items
  included, with no early parity pass, no stall and no data hazard, and so
  does a watcher that joins each phase without waiting for the previous one;
- the protocol before the single-tile fix is caught: with single-tile items in
  the mix, runs end in data hazards (an S MMA reading a K slot that does not
  hold its page, a copy into a slot an MMA still has to read); with two-tile
  items only it stays clean. So the model is not vacuous, and the hazard is the
  one of single-tile items.
"""
import random

import attn_protocol_model as m

SEEDS = 300


def _violations(protocol, p_single, count=10, max_pages=4, early_fatal=True, seeds=SEEDS,
                slots=m.RING_SLOTS):
    bad = []
    for seed in range(seeds):
        items = m.random_items(random.Random(seed), count, max_pages=max_pages, p_single=p_single)
        try:
            m.run(items, seed, protocol=protocol, early_fatal=early_fatal, slots=slots)
        except m.Violation as e:
            bad.append((seed, str(e)))
    return bad


def test_current_protocol_is_clean():
    bad = _violations("current", p_single=0.4)
    assert not bad, bad[:3]


def test_current_protocol_single_tile_heavy_and_long():
    assert not _violations("current", p_single=0.8), "single-tile heavy"
    assert not _violations("current", p_single=0.4, count=30, max_pages=7, seeds=60), "long"


def test_current_protocol_with_the_d64_ring():
    """The d = 64 kernel streams K/V through 10 ring slots instead of 5."""
    assert not _violations("current", p_single=0.4, max_pages=8, slots=10)


def test_watcher_previous_phase_waits_are_implied():
    """Joining S_FREE / P_FULL without waiting for the previous phase stays clean:
    the watcher's other waits already imply those phases are complete."""
    bad = _violations("lean-watcher", p_single=0.4)
    assert not bad, bad[:3]


def test_original_protocol_is_caught_on_single_tile_items():
    bad = _violations("original", p_single=0.4, early_fatal=False)
    assert len(bad) >= SEEDS // 10, f"only {len(bad)} of {SEEDS} runs hit a hazard"
    assert any("reads K slot" in msg or "MMAs to read it" in msg for _, msg in bad), bad[:3]


def test_original_protocol_is_clean_without_single_tile_items():
    assert not _violations("original", p_single=0.0)


def test_parity_wait_semantics():
    """The model's barrier answers like an mbarrier parity wait: right only for the phase
    after the last completed one, wrong both ways two phases away."""
    b = m.Bar("b", 2)
    assert not b.parity_passes(0)
    b.arrive()
    assert not b.parity_passes(0)           # one of two arrivals
    b.arrive()                              # phase 0 complete
    assert b.parity_passes(0) and not b.parity_passes(1)
    b.arrive(2)                             # phase 1 complete, phase 2 pending
    assert b.parity_passes(1) and not b.parity_passes(2)
    assert b.parity_passes(3)               # phase 3 is not complete, yet the wait passes
    assert not b.parity_passes(0)           # phase 0 is long complete, yet the wait blocks
