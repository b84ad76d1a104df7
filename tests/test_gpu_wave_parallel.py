"""Wave Parallelism's data path on the GPU: three ranks as three processes sharing
the one GPU of this machine, each with its own device pool, exchanging page
bytes through host memory (gloo). No kernel of one rank waits on the other's:
each rank appends its own nodes' K/V with the append kernel, receives the
entries it needs into pages it has just taken, and runs the attention kernel
over its nodes' key lists -- every round, every element checked against the
float64 oracle. (On several GPUs the same driver moves device pages with NCCL.)
"""
import os
import socket

import pytest
import torch.multiprocessing as mp

pytestmark = pytest.mark.gpu


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime

    import torch
    import torch.distributed as dist

    import block_causal_attention_wave_b200 as wave
    import wave_inputs as wi
    from block_causal_attention_wave_b200.wave_parallel import WaveParallel
    from wave_testlib import Inputs, assert_close, bits_to_torch, oracle_outputs, queries, torch_to_f64
    torch.cuda.set_device(0)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=120))
    try:
        wl = wi.Workload("wp-gpu", chunks=4, levels=2, heads=2, head_dim=128, tokens=300)
        pol = "progressive"
        inp = Inputs(wl)
        pb = wave.KVCache.page_bytes(wl.heads, wl.head_dim)
        pool = torch.zeros(4096 + 40 * pb, dtype=torch.uint8, device="cuda")
        kv = wave.KVCache(wl.heads, wl.head_dim, wl.tokens, wl.levels, wl.window, 0, pool=pool)
        wp = WaveParallel(kv, pool, wl.chunks, wl.levels, pol, wl.window, rank, world)
        keep, checked = [], 0
        for t in range(len(wp.rounds)):
            own = wp.own_nodes(t)
            if own:
                ks = [bits_to_torch(inp.bits("k", *n)) for n in own]
                vs = [bits_to_torch(inp.bits("v", *n)) for n in own]
                kv.append_batch(own, ks, vs)
                keep.append((ks, vs))
            wp.exchange(t)
            if own:
                q = queries(inp, own)
                o = torch.full_like(q, float("nan"))
                kv.round_attn(own, pol, q, o)
                kv.status()
                ref = oracle_outputs(inp, own, pol)
                got = torch_to_f64(o).reshape(len(own), wl.tokens, wl.heads, wl.head_dim)
                for i, n in enumerate(own):
                    assert_close(got[i], ref[n], f"rank {rank} round {t} node {n}")
                    checked += 1
            wp.release(t)
        torch.cuda.synchronize()
        out[rank] = checked
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(300)
def test_wave_parallel_three_ranks_on_one_gpu(cuda_lib):
    world = 3  # K + 1 ranks: one per level of the 2-level schedule
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        # every node of the schedule was checked on exactly one rank
        import block_causal_attention_wave_b200 as wave
        total = sum(len(r) for r in wave.schedule(4, 2, "progressive", 0))
        assert sum(out.values()) == total
