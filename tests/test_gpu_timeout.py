"""Failure detection on the GPU without a fault: a bounded wait that runs out.

Every barrier wait inside the attention and fused-projection kernels is
bounded (2 s by default). Here the handle's bound is set to 100 ns on rounds
whose TMA copies and MMAs take microseconds, so some wait is bound to run out.
The kernel must then stop every role, let the copies and MMAs it issued
finish, free its tensor memory and return: wave_kv_status reports
WAVE_ERR_TIMEOUT and the context stays usable. With the default bound restored
the same pool must give oracle-correct results. Nothing faults, traps or hangs
on the device: the kernel simply gives up and returns.
"""
import numpy as np
import pytest

import wave_inputs as wi
from oracle import cache as ocache
from oracle import projection as oproj
from oracle import schedule as osched

from wave_testlib import (Inputs, append, assert_close, bits_to_torch, make_cache, oracle_outputs,
                          queries, torch_to_f64)

pytestmark = pytest.mark.gpu

WL = wi.Workload("timeout-d128", chunks=4, levels=3, heads=3, head_dim=128, tokens=300,
                 prefix=77)


def _expect_timeout(wave, kv):
    with pytest.raises(wave.WaveError) as ei:
        kv.status()
    assert ei.value.code == wave._binding.ERR_TIMEOUT, str(ei.value)


def test_attention_wait_runs_out_then_recovers(cuda_lib):
    import torch
    wave = cuda_lib
    pol = "progressive"
    inp = Inputs(WL)
    active = max(osched.schedule(WL.chunks, WL.levels, pol, WL.window), key=len)
    entries = set()
    for n in active:
        entries.update(ocache.key_entries(n, pol, WL.window, True))
    kv = make_cache(wave, WL, 64)
    keep = [append(kv, inp, e) for e in sorted(entries)]
    q = queries(inp, active)
    o = torch.empty_like(q)
    kv.status()
    kv.set_wait_limit(100)  # 100 ns: shorter than any TMA copy
    kv.round_attn(active, pol, q, o)
    _expect_timeout(wave, kv)
    kv.status()  # the status word was cleared by the read above
    kv.set_wait_limit(0)    # back to the default bound
    o.fill_(float("nan"))
    kv.round_attn(active, pol, q, o)
    kv.status()
    ref = oracle_outputs(inp, active, pol)
    got = torch_to_f64(o).reshape(len(active), WL.tokens, WL.heads, WL.head_dim)
    for i, n in enumerate(active):
        assert_close(got[i], ref[n], f"after a timed-out launch, node {n}")
    del keep


def test_projection_wait_runs_out_then_recovers(cuda_lib):
    import torch
    wave = cuda_lib
    dim = 256
    kv = make_cache(wave, WL, 16)
    xb = wi.hidden_states(0, 3, WL.tokens, dim)
    wb = wi.qkv_weight(WL.heads, WL.head_dim, dim)
    x, w = bits_to_torch(xb), bits_to_torch(wb)
    qp = torch.empty(WL.tokens, WL.heads, WL.head_dim, dtype=torch.bfloat16, device="cuda")
    kv.set_wait_limit(100)
    kv.qkv_append(0, 3, x, w, qp)
    _expect_timeout(wave, kv)
    kv.release(0, 3)
    kv.set_wait_limit(0)
    qp.fill_(float("nan"))
    kv.qkv_append(0, 3, x, w, qp)
    kv.status()
    rq, _, _ = oproj.qkv(wi.bf16_bits_to_f64(xb), wi.bf16_bits_to_f64(wb), WL.heads, WL.head_dim)
    got = torch_to_f64(qp)
    assert np.isfinite(got).all()
    assert_close(got, rq, "projection Q after a timed-out launch", scale_with_output=True)
