"""Wave Parallelism host logic across processes (gloo on CPU, world size 2-3).

Each rank runs its share of a rollout through the library's placement, push
list and release rounds (wave_wp_transfers, wave_wp_rank_last_read) and the
driver's page pushes (torch.distributed point-to-point, straight between the
ranks' pool pages). Host-only cache handles stand in for the device pools, with
a host byte tensor per rank laid out as the pool. Checked every round, on every
rank, against the oracle (oracle/parallel.py): the rank's nodes, their gather
tables page for page, and the bytes of every entry its nodes read -- equal to
what the producer wrote, wherever it ran. The library's push lists and release
rounds are also compared with the oracle's for many shapes in this process.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from oracle import cache as ocache
from oracle import parallel as opar


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _entry_bytes(entry, nbytes):
    seed = 977 + (entry[0] + 1) * 64 + entry[1]
    return np.random.Generator(np.random.PCG64(seed)).integers(0, 256, nbytes, dtype=np.uint8)


def _worker(rank, world, port, cfg, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime

    import torch.distributed as dist

    import block_causal_attention_wave_b200 as wave
    from block_causal_attention_wave_b200.wave_parallel import WaveParallel
    B, K, pol, W, T, H, d = cfg
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        pb = wave.KVCache.page_bytes(H, d)
        kv = wave.KVCache(H, d, T, K, W, 0, pool=None, pool_bytes=4096 + 64 * pb)
        page_bytes, off, maxp = kv.layout()
        pool = torch.zeros(off + maxp * page_bytes, dtype=torch.uint8)
        wp = WaveParallel(kv, pool, B, K, pol, W, rank, world)
        want = opar.rank_tables(B, K, pol, W, world, rank, T, 0, maxp)
        assert len(want) == len(wp.rounds)
        npages = (T + 127) // 128
        for t in range(len(wp.rounds)):
            own = wp.own_nodes(t)
            for n in own:  # this rank's nodes produce their entries
                kv.alloc(*n)
                data = torch.from_numpy(_entry_bytes(n, npages * page_bytes))
                for i, p in enumerate(kv.entry_pages(*n)):
                    pool[off + p * page_bytes:off + (p + 1) * page_bytes] = \
                        data[i * page_bytes:(i + 1) * page_bytes]
            wp.exchange(t)
            table = kv.gather_table(own, pol) if own else []
            assert (own, table) == (want[t][0], want[t][1]), f"rank {rank} round {t}"
            for node in own:
                for e in ocache.key_entries(node, pol, W, False):
                    got = np.concatenate([
                        pool[off + p * page_bytes:off + (p + 1) * page_bytes].numpy()
                        for p in kv.entry_pages(*e)])
                    assert np.array_equal(got, _entry_bytes(e, npages * page_bytes)), \
                        f"rank {rank} round {t}: bytes of {e}"
            wp.release(t)
        assert kv.free_pages() == maxp  # everything released at the end
        out[rank] = "ok"
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(240)
@pytest.mark.parametrize("cfg,world", [
    ((5, 2, "progressive", 0, 200, 2, 64), 3),
    ((6, 3, "progressive", 2, 130, 1, 64), 2),
    ((4, 2, "clean", 0, 200, 2, 64), 3),
    ((4, 2, "same", 0, 200, 2, 64), 3),
])
def test_wave_parallel_rollout_over_gloo(cfg, world):
    port = _free_port()
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, port, cfg, out), nprocs=world, join=True)
        assert dict(out) == {r: "ok" for r in range(world)}


@pytest.mark.parametrize("B,K,W", [(3, 2, 0), (6, 4, 2), (7, 4, 0), (5, 1, 0), (9, 3, 3)])
@pytest.mark.parametrize("policy", ["clean", "same", "progressive"])
@pytest.mark.parametrize("N", [1, 2, 3, 5])
def test_library_push_lists_and_release_rounds_match_the_oracle(B, K, W, policy, N):
    import block_causal_attention_wave_b200 as wave
    want = opar.transfers(B, K, policy, W, N)
    for t in range(len(want)):
        assert wave.wp_transfers(B, K, policy, W, N, t) == want[t]
    for r in range(N):
        last = opar.rank_last_read(B, K, policy, W, N, r)
        if last:
            assert wave.wp_rank_last_read(B, K, policy, W, N, r, sorted(last)) == last
