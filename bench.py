"""Benchmark: wave-round attention on the Wan2.1-1.3B-shaped round.

One step = one pass of the whole hot path over one wave round: the round's
schedule and key tables (host), the K/V append of every active node (one
batched kernel launch for the round), and the attention of all active nodes in one kernel launch. The
workload is round 6 of the 7-chunk, 4-level progressive schedule: nodes (2,0)
[refresh], (3,1), (4,2), (5,3), (6,4); 12 heads, head_dim 128, 4680 tokens per
chunk; its history K/V (rounds 0..5) is appended once before timing, and each
step appends the round's own K/V again (released after the step, so every step
does identical work on identical pages).

Output: one JSON line (rank 0). ``value`` is attention TFLOP/s over the whole
job (all ranks; algorithmic FLOPs 4*Nq*Nk*d per head, valid tokens only,
divided by the step time, so append time counts against it). Inputs (K/V cache
of the round ~0.7 GB, Q 72 MB) exceed the 126 MB L2, so no flush is needed.

``e2e`` repeats the step through the same public API with the step's inputs
copied from pinned host memory and O copied back every step; copies of one
step overlap the previous step's compute.

``--impl reference`` times the float64 CPU oracle instead (rank 0 only) on a
bounded sample of the same round.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import wave_inputs as wi  # noqa: E402

METRIC = "wave-round attention TFLOP/s and chunk-updates/s at 1 B200; % of BF16 dense peak"
UNIT = "TFLOP/s"
POLICY = "progressive"


class Spec:
    """A timed wave round: the workload's shapes and which round of its schedule."""

    def __init__(self, key, wl, round_index, label, pool_pages):
        self.key, self.wl, self.round, self.label, self.pool_pages = (
            key, wl, round_index, label, pool_pages)


WORKLOADS = {
    # Wan2.1-1.3B-shaped round (the headline): nodes (2,0) refresh, (3,1), (4,2),
    # (5,3), (6,4); the live cache peaks near 900 pages.
    "wan21": Spec("wan21", wi.WAN21, 6, "wan2.1-1.3b round 6 (B=7, K=4, progressive)", 2400),
    # Wan-Streamer-shaped steady round: (33,0) refresh, (34,1), (35,2); 984-token
    # units, 512-token prefix, 32-unit window, 24 heads.
    "wan-streamer": Spec("wan-streamer", wi.WAN_STREAMER, 35,
                         "wan-streamer unit round 35 (K=2, W=32, prefix 512, progressive)", 1000),
    # Long rollout steady round: (15,0) refresh, (16,1) .. (20,5); window 6.
    "long-rollout": Spec("long-rollout", wi.LONG_ROLLOUT, 20,
                         "long rollout round 20 (40 chunks, K=5, W=6, progressive)", 1400),
}
DEFAULT_WORKLOAD = "wan21"
# Headline constants (the CPU-baseline and reference legs time this round).
ROUND = WORKLOADS[DEFAULT_WORKLOAD].round
WORKLOAD = WORKLOADS[DEFAULT_WORKLOAD].label


def _config(extra=None, spec=None):
    spec = spec or WORKLOADS[DEFAULT_WORKLOAD]
    wl = spec.wl
    cfg = {"workload": spec.label, "heads": wl.heads, "head_dim": wl.head_dim,
           "tokens_per_chunk": wl.tokens, "chunks": wl.chunks, "levels": wl.levels,
           "window": wl.window, "prefix_tokens": wl.prefix, "policy": POLICY, "round": spec.round,
           "l2": "inputs larger than L2 (the round's K/V and Q); no flush"}
    if extra:
        cfg.update(extra)
    return cfg


def _kernel_source_hash():
    import hashlib
    h = hashlib.sha256()
    for name in ("wave_attn.cu", "ptx.cuh", "exp2_poly.h", "wave_sync.cuh"):
        with open(os.path.join(ROOT, "block_causal_attention_wave_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def _measured_traffic(workload):
    """DRAM bytes per attention launch from the committed ncu capture, if it was
    taken on the current kernel source and on this workload (else None)."""
    path = os.path.join(ROOT, "profiles", "round_attn_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f)
    if rec.get("kernel_source_sha256") != _kernel_source_hash() or rec.get("workload_key") != workload:
        return None
    return rec.get("dram_bytes_per_launch")


def _source_hash(names):
    import hashlib
    h = hashlib.sha256()
    for name in names:
        with open(os.path.join(ROOT, "block_causal_attention_wave_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def _measured_append_traffic(workload):
    """DRAM bytes of the batched append launch from the committed ncu record, if
    it was taken on the current append source and on this workload (else None)."""
    path = os.path.join(ROOT, "profiles", "kv_append_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f)
    if rec.get("kernel_source_sha256") != _source_hash(["wave_device.cu"]) or rec.get("workload_key") != workload:
        return None
    return {k: rec.get(k) for k in ("dram_read_bytes", "dram_write_bytes", "duration_ns")}


def _measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            return json.load(f), "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


# ------------------------------------------------------------------ distributed

def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def reduce_max(x: float, backend_device=None) -> float:
    """Max of a float over all ranks (identity without a process group)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return x
    t = torch.tensor([x], dtype=torch.float64, device=backend_device or "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier():
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dist.barrier()


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during a region."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int, path: str | None = None):
        self.idx = device_index
        self.proc = None
        self.f = None
        self.temporary = path is None
        if path is None:
            import tempfile
            fd, path = tempfile.mkstemp(prefix=f"wave_clocks_rank{device_index}_", suffix=".csv")
            os.close(fd)
        self.path = path

    def start(self):
        try:
            os.makedirs(os.path.dirname(os.path.abspath(self.path)), exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"], stdout=self.f,
                stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        out = None
        if self.proc is not None:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.f.close()
            out = self.summary()
        elif getattr(self, "f", None) is not None:
            self.f.close()
        if self.temporary and os.path.exists(self.path):
            os.remove(self.path)
        return out

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    mx = float(parts[2])
                except ValueError:
                    continue
                for n, v in zip(names, parts[5:9]):
                    if v.lower().startswith("active"):
                        reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------------ workload

class Round:
    """Host-side description of the timed round, from the library's scheduler."""

    def __init__(self, wave, spec=None):
        spec = spec or WORKLOADS[DEFAULT_WORKLOAD]
        wl = spec.wl
        self.spec, self.wl = spec, wl
        self.rounds = wave.schedule(wl.chunks, wl.levels, POLICY, wl.window)
        self.last = wave.last_read_rounds(wl.chunks, wl.levels, POLICY, wl.window)
        self.active = self.rounds[spec.round]


def _bits_to_dev(bits, pin=False):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)
    return t.pin_memory() if pin else t.cuda()


def run_gpu(args):
    import torch
    import block_causal_attention_wave_b200 as wave

    ws, rank, local = dist_env()
    torch.cuda.set_device(local)
    if ws > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    wave.load()
    spec = WORKLOADS[args.workload]
    rd = Round(wave, spec)
    wl = rd.wl
    page_bytes = wave.KVCache.page_bytes(wl.heads, wl.head_dim)
    pool = torch.empty(4096 + spec.pool_pages * page_bytes, dtype=torch.uint8, device="cuda")
    kv = wave.KVCache(wl.heads, wl.head_dim, wl.tokens, wl.levels, wl.window, wl.prefix,
                      pool=pool)
    stream = torch.cuda.current_stream()

    def kvbits(kind, e):
        n = wl.prefix if e[0] == -1 else wl.tokens
        return wi.node_tensor(kind, e[0], e[1], n, wl.heads, wl.head_dim, wl.scale)

    # Bring the cache to the start of the timed round (untimed).
    if wl.prefix:
        kv.append(-1, 0, _bits_to_dev(kvbits("k", (-1, 0))), _bits_to_dev(kvbits("v", (-1, 0))))
    for t in range(spec.round):
        for n in rd.rounds[t]:
            kv.append(n[0], n[1], _bits_to_dev(kvbits("k", n)), _bits_to_dev(kvbits("v", n)))
        for e in sorted(e for e, lr in rd.last.items() if lr == t):
            kv.release(*e)
    torch.cuda.synchronize()
    active = rd.active
    host_k = [kvbits("k", n) for n in active]
    host_v = [kvbits("v", n) for n in active]
    host_q = np.concatenate([kvbits("q", n) for n in active])
    dk = [_bits_to_dev(b) for b in host_k]
    dv = [_bits_to_dev(b) for b in host_v]
    dq = _bits_to_dev(host_q)
    do = torch.empty_like(dq)

    def append_round():
        kv.append_batch(active, dk, dv, stream)

    # FLOPs from the library's own key tables (valid tokens only).
    append_round()
    table = kv.gather_table(active, POLICY)
    for n in active:
        kv.release(*n)
    n_keys = [sum(v for _, v in rows) for rows in table]
    flops = sum(4 * wl.tokens * nk * wl.heads * wl.head_dim for nk in n_keys)
    upd_nodes = sum(1 for n in active if n[1] > 0)
    per_node_read = 2 * wl.tokens * wl.heads * wl.head_dim * 2
    per_node_write = 2 * math.ceil(wl.tokens / 128) * 128 * wl.heads * wl.head_dim * 2
    append_bytes = len(active) * (per_node_read + per_node_write)

    def step(ev_a=None, ev_b=None, ev_c=None):
        if ev_c is not None:
            ev_c.record(stream)
        append_round()
        if ev_a is not None:
            ev_a.record(stream)
        kv.round_attn(active, POLICY, dq, do, stream)
        if ev_b is not None:
            ev_b.record(stream)
        for n in active:
            kv.release(*n)

    for _ in range(args.warmup):
        step()
    kv.status(stream)

    # ---- device-timed region
    K = args.steps
    ev_a = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    ev_b = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    ev_c = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clk = ClockSampler(local, args.clocks_csv.format(rank=rank) if args.clocks_csv else None)
    clk.start()
    barrier()
    torch.cuda.synchronize()
    t0.record(stream)
    for i in range(K):
        step(ev_a[i], ev_b[i], ev_c[i])
    t1.record(stream)
    torch.cuda.synchronize()
    barrier()
    clocks = clk.stop()
    kv.status(stream)
    # SM clock the last timed attention launch ran at (its CTA 0's cycles / ns).
    cyc, ns = kv.last_launch_clock(stream)
    eff_mhz = cyc / ns * 1e3 if ns > 0 else None
    sms = torch.cuda.get_device_properties(local).multi_processor_count
    ms_local = t0.elapsed_time(t1)
    attn_ms = [a.elapsed_time(b) for a, b in zip(ev_a, ev_b)]
    ms = reduce_max(ms_local, "cuda" if ws > 1 else None)
    ms_step = ms / K
    value = ws * flops * K / (ms * 1e-3) / 1e12
    attn_avg = sum(attn_ms) / len(attn_ms)

    # ---- the round's 4 update nodes alone (the refresh node's queries left out):
    # the 2.9605-TFLOP headline of the round, beside the 5-node figure above.
    upd_only = [n for n in active if n[1] > 0]
    updates = None
    if len(upd_only) < len(active):
        idx = [active.index(n) for n in upd_only]
        T = wl.tokens
        q_u = torch.cat([dq[i * T:(i + 1) * T] for i in idx])
        o_u = torch.empty_like(q_u)
        kv.append_batch(active, dk, dv, stream)
        u_table = kv.gather_table(upd_only, POLICY)
        u_flops = sum(4 * T * sum(v for _, v in rows) * wl.heads * wl.head_dim for rows in u_table)
        for _ in range(3):
            kv.round_attn(upd_only, POLICY, q_u, o_u, stream)
        ua, ub = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda._sleep(int(2e6))
        ua.record(stream)
        for _ in range(10):
            kv.round_attn(upd_only, POLICY, q_u, o_u, stream)
        ub.record(stream)
        torch.cuda.synchronize()
        for n in active:
            kv.release(*n)
        u_ms = ua.elapsed_time(ub) / 10
        updates = {"nodes": [list(n) for n in upd_only], "flops_per_launch": u_flops,
                   "avg_launch_ms": round(u_ms, 4),
                   "achieved": round(u_flops / (u_ms * 1e-3) / 1e12, 2), "unit": UNIT,
                   "chunk_updates_per_s": round(len(upd_only) / (u_ms * 1e-3), 2)}

    # ---- the batched append launch (HBM roofline context): events around it in
    # every timed step. The host runs ahead of the GPU during each attention
    # launch, so these events see the kernel, not the host's enqueue time; the
    # median drops the first step, which starts from an idle GPU.
    append_ms = statistics.median(c.elapsed_time(a) for c, a in zip(ev_c, ev_a))

    # ---- fused QKV projection + K/V append of the round's nodes (the step
    # that produces the K/V the round appends), random Wan2.1-shaped weights:
    # X [5 T][C] for the round's nodes, W [3 H d][C]; ONE launch for the round
    # (wave_qkv_append_round, no rotary here: the block line below has it). A
    # sleep kernel keeps the GPU busy while the host enqueues, so the events see
    # only the launches.
    proj = None
    if wl.head_dim == 128 and (3 * wl.heads) % 2 == 0 and spec.key == DEFAULT_WORKLOAD:
        dim = wi.WAN21_DIM
        X = torch.cat([_bits_to_dev(wi.hidden_states(n[0], n[1], wl.tokens, dim)) for n in active])
        wqkv = _bits_to_dev(wi.qkv_weight(wl.heads, wl.head_dim, dim))
        qp = torch.empty(len(active) * wl.tokens, wl.heads, wl.head_dim, dtype=torch.bfloat16,
                         device="cuda")

        def proj_round():
            kv.qkv_append_round(active, X, wqkv, qp, stream=stream)
            for n in active:
                kv.release(*n)

        proj_round()
        torch.cuda.synchronize()
        reps = 10
        pa, pb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda._sleep(int(3e6))
        pa.record(stream)
        for _ in range(reps):
            proj_round()
        pb.record(stream)
        torch.cuda.synchronize()
        kv.status(stream)
        p_ms = pa.elapsed_time(pb) / reps
        p_flops = 2 * len(active) * wl.tokens * 3 * wl.heads * wl.head_dim * dim
        proj = {"kernel": "gemm_wide_kernel (QKV epilogue)",
                "what": "Q,K,V = X W^T for the round's 5 nodes in one launch, K/V written "
                "into each node's new pages in the epilogue", "dim": dim,
                "flops_per_launch": p_flops, "avg_launch_ms": round(p_ms, 4),
                "achieved": round(p_flops / (p_ms * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
                "frac": round(p_flops / (p_ms * 1e-3) / 1e12 / _measured_peaks()[0]["bf16_tflops"],
                              4)}

    # ---- one whole transformer block of the round (Wan2.1-1.3B shapes, random
    # weights): the round's QKV projection with the rotary embedding and the K/V
    # append fused in (one launch for all nodes), the wave-round attention, the
    # out-projection with the residual, the tanh-GELU MLP up and the MLP down
    # with the residual. Events around every launch; a sleep kernel keeps the
    # GPU busy while the host enqueues the first launches.
    block = None
    if spec.key == DEFAULT_WORKLOAD and not args.no_block:
        block = block_round(wave, kv, wl, active, stream, args)

    # ---- FP8 (E4M3) pages: the same round over an FP8 pool holding the round's
    # key lists (history appended once, quantised); per step the round's pages
    # are expanded to bf16 staging in the workspace, then the attention runs.
    fp8 = None
    if spec.key == DEFAULT_WORKLOAD and not args.no_block:
        fp8 = fp8_round(wave, wl, rd, active, dq, stream, flops)

    # ---- split-KV attention (key lists cut into ranges, partials combined):
    # the same round with the automatic range count, and a round of a single
    # update node (few work items: the case the ranges are for).
    split = None
    if spec.key == "wan-streamer":
        split = split_rounds(wave, kv, wl, active, dq, do, stream, flops)

    # ---- end to end through the public API with host buffers. Every step copies
    # its Q and the round's K/V from pinned host memory and reads O back; the
    # copies of step i+1 run on their own streams while step i computes (device
    # input and output buffers are double-buffered), so PCIe and compute overlap.
    hq = _bits_to_dev(host_q, pin=True)
    hk = [_bits_to_dev(b, pin=True) for b in host_k]
    hv = [_bits_to_dev(b, pin=True) for b in host_v]
    ho = [torch.empty(dq.shape, dtype=torch.bfloat16, pin_memory=True) for _ in range(2)]
    h2d = hq.numel() * 2 + sum(x.numel() * 2 for x in hk + hv)
    d2h = ho[0].numel() * 2
    bq = [dq, torch.empty_like(dq)]
    bk = [dk, [torch.empty_like(x) for x in dk]]
    bv = [dv, [torch.empty_like(x) for x in dv]]
    bo = [do, torch.empty_like(do)]
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_done = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    for b in range(2):  # buffers start free
        ev_done[b].record(stream)
        ev_out[b].record(stream)

    def e2e_step(i):
        b = i % 2
        with torch.cuda.stream(s_in):
            s_in.wait_event(ev_done[b])  # step i-2 finished reading buffer b
            bq[b].copy_(hq, non_blocking=True)
            for d, h in zip(bk[b], hk):
                d.copy_(h, non_blocking=True)
            for d, h in zip(bv[b], hv):
                d.copy_(h, non_blocking=True)
            ev_in[b].record(s_in)
        stream.wait_event(ev_in[b])
        stream.wait_event(ev_out[b])  # O buffer b read back by step i-2
        kv.append_batch(active, bk[b], bv[b], stream)
        kv.round_attn(active, POLICY, bq[b], bo[b], stream)
        for n in active:
            kv.release(*n)
        ev_done[b].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_done[b])
            ho[b].copy_(bo[b], non_blocking=True)
            ev_out[b].record(s_out)

    for i in range(2):
        e2e_step(i)
    torch.cuda.synchronize()
    E = max(3, min(K, 20))
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    for i in range(E):
        e2e_step(i)
    s_in.wait_stream(s_out)
    s_in.wait_stream(stream)
    e1.record(s_in)
    torch.cuda.synchronize()
    barrier()
    e2e_ms = reduce_max(e0.elapsed_time(e1), "cuda" if ws > 1 else None) / E
    kv.status(stream)

    peaks, src = _measured_peaks()
    achieved = flops / (attn_avg * 1e-3) / 1e12
    peak = peaks["bf16_tflops"]
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": ws, "steps": K,
        "warmup": args.warmup, "ms_per_step": round(ms_step, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": _config({"replicas": ws}, spec),
        "chunk_updates_per_s": round(ws * upd_nodes * K / (ms * 1e-3), 2),
        "pct_bf16_dense_peak": round(100 * value / ws / peak, 2),
        "e2e": {"value": round(ws * flops / (e2e_ms * 1e-3) / 1e12, 2), "unit": UNIT,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": round(e2e_ms, 4),
                "note": "pinned H2D of Q and K/V and D2H of O every step, overlapped with the "
                        "previous step's compute (double-buffered device buffers)"},
        "roofline": {"bound": "tensor", "kernel": "round_attn_kernel<128>",
                     "achieved": round(achieved, 2), "peak": peak, "unit": "TFLOP/s",
                     "frac": round(achieved / peak, 4), "traffic": _measured_traffic(spec.key),
                     "peak_source": f"{src} bf16_tflops (burst, cuBLAS 8192^3)",
                     "flops_per_launch": flops, "avg_launch_ms": round(attn_avg, 4),
                     "effective_sm_mhz": round(eff_mhz, 1) if eff_mhz else None,
                     "per_clock_frac": (round(achieved / (sms * 8192 * eff_mhz * 1e-6), 4)
                                        if eff_mhz else None),
                     "per_clock_note": "achieved / (SMs x 8192 dense bf16 FLOP/clk x the "
                                       "effective SM clock of the last timed launch)"},
        "append": {"kernel": "kv_append_kernel", "nodes_per_launch": len(active),
                   "bytes_per_launch": append_bytes, "median_launch_ms": round(append_ms, 4),
                   "achieved_gbs": round(append_bytes / (append_ms * 1e-3) / 1e9, 1),
                   "peak_gbs": peaks["hbm_gbs"],
                   "frac": round(append_bytes / (append_ms * 1e-3) / 1e9 /
                                 peaks["hbm_gbs"], 4),
                   "ncu": _measured_append_traffic(spec.key),
                   "ncu_note": "DRAM bytes of one batched append launch (ncu): writes that are "
                               "still in L2 when the kernel ends reach DRAM later"},
        "gpu_launches": K * 2,
        "updates_only": updates,
        "projection": proj,
        "block": block,
        "split_kv": split,
        "fp8_pages": fp8,
        "clocks": clocks,
    }
    if rank == 0 and ws == 1 and not args.no_cpu_baseline and spec.key == DEFAULT_WORKLOAD:
        line["cpu_baseline"] = cpu_baseline(target_s=args.cpu_seconds)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if ws > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def fp8_round(wave, wl, rd, active, dq, stream, flops):
    """Attention of the round over an FP8 pool: expand + attention per step."""
    import torch
    ents = set()
    table_nodes = active
    pb8 = wave.KVCache.page_bytes(wl.heads, wl.head_dim, wave.KV_FP8_E4M3)
    pb16 = wave.KVCache.page_bytes(wl.heads, wl.head_dim)
    pages = 1000
    pool = torch.zeros(4096 + 256 + pages * (pb8 + 2 * wl.heads * 4), dtype=torch.uint8,
                       device="cuda")
    kv8 = wave.KVCache(wl.heads, wl.head_dim, wl.tokens, wl.levels, wl.window, wl.prefix,
                       pool=pool, kv_format=wave.KV_FP8_E4M3)
    # every entry the round's nodes read: history from earlier rounds, then the round's own
    last = rd.last
    for t in range(rd.spec.round + 1):
        for n in rd.rounds[t]:
            if last[tuple(n)] >= rd.spec.round:
                ents.add(tuple(n))
    for e in sorted(ents):
        kv8.append(e[0], e[1],
                   _bits_to_dev(wi.node_tensor("k", e[0], e[1], wl.tokens, wl.heads, wl.head_dim,
                                               wl.scale)),
                   _bits_to_dev(wi.node_tensor("v", e[0], e[1], wl.tokens, wl.heads, wl.head_dim,
                                               wl.scale)), stream)
    nbytes, _ = kv8.split_workspace(table_nodes, POLICY, 1)
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    o = torch.empty_like(dq)
    for _ in range(3):
        kv8.round_attn_split(table_nodes, POLICY, dq, o, ws, 1, stream)
    torch.cuda.synchronize()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    torch.cuda._sleep(int(2e6))
    ev[0].record(stream)
    for _ in range(10):
        kv8.round_attn_split(table_nodes, POLICY, dq, o, ws, 1, stream)
    ev[1].record(stream)
    torch.cuda.synchronize()
    kv8.status(stream)
    ms = ev[0].elapsed_time(ev[1]) / 10
    n_pages = len({p for rows in kv8.gather_table(table_nodes, POLICY) for p, _ in rows})
    return {"what": "attention of the round over an FP8 (E4M3, per-(page, head) scale) pool: "
                    "the round's pages expanded to bf16 staging, then the attention kernel",
            "entry_bytes_bf16": (wl.tokens + 127) // 128 * pb16,
            "entry_bytes_fp8": (wl.tokens + 127) // 128 * (pb8 + 2 * wl.heads * 4),
            "round_pages": n_pages, "staging_bytes": nbytes,
            "ms": round(ms, 4), "tflops": round(flops / (ms * 1e-3) / 1e12, 2)}


def split_rounds(wave, kv, wl, active, dq, do, stream, flops):
    """Time wave_round_attn_split (automatic ranges) against wave_round_attn
    on the timed round and on its last update node alone."""
    import torch
    out = {}
    T = wl.tokens
    upd = [n for n in active if n[1] > 0][-1:]
    kv.append_batch(active, *_round_kv(wl, active), stream)
    one_flops = None
    for name, nodes in (("round", active), ("one_node", upd)):
        idx = [active.index(n) for n in nodes]
        q = torch.cat([dq[i * T:(i + 1) * T] for i in idx])
        o = torch.empty_like(q)
        nbytes, used = kv.split_workspace(nodes, POLICY, 0)
        wsb = torch.empty(max(nbytes, 16), dtype=torch.uint8, device="cuda")
        if name == "one_node":
            table = kv.gather_table(nodes, POLICY)
            f = sum(4 * T * sum(v for _, v in rows) * wl.heads * wl.head_dim for rows in table)
        else:
            f = flops
        res = {"nodes": [list(n) for n in nodes], "flops": f, "splits": used}
        for key, call in (("plain", lambda: kv.round_attn(nodes, POLICY, q, o, stream)),
                          ("split", lambda: kv.round_attn_split(nodes, POLICY, q, o, wsb, 0,
                                                                stream))):
            for _ in range(3):
                call()
            torch.cuda.synchronize()
            ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
            torch.cuda._sleep(int(2e6))
            ev[0].record(stream)
            for _ in range(10):
                call()
            ev[1].record(stream)
            torch.cuda.synchronize()
            ms = ev[0].elapsed_time(ev[1]) / 10
            res[key] = {"ms": round(ms, 4), "tflops": round(f / (ms * 1e-3) / 1e12, 2)}
        out[name] = res
    kv.status(stream)
    for n in active:
        kv.release(*n)
    return out


def _round_kv(wl, active):
    ks = [_bits_to_dev(wi.node_tensor("k", c, l, wl.tokens, wl.heads, wl.head_dim, wl.scale))
          for c, l in active]
    vs = [_bits_to_dev(wi.node_tensor("v", c, l, wl.tokens, wl.heads, wl.head_dim, wl.scale))
          for c, l in active]
    return ks, vs


def block_round(wave, kv, wl, active, stream, args):
    """Time one transformer block of the round; per-kernel ms and TFLOP/s."""
    import torch
    C, F = wi.WAN21_DIM, wi.WAN21_MLP
    n, T, H, d = len(active), wl.tokens, wl.heads, wl.head_dim
    M = n * T
    X = torch.cat([_bits_to_dev(wi.hidden_states(c, l, T, C)) for c, l in active])
    Wq = _bits_to_dev(wi.qkv_weight(H, d, C))
    Wo = _bits_to_dev(wi.block_weight("wo", C, H * d))
    W1 = _bits_to_dev(wi.block_weight("w1", F, C))
    W2 = _bits_to_dev(wi.block_weight("w2", C, F))
    Q = torch.empty((M, H, d), dtype=torch.bfloat16, device="cuda")
    A = torch.empty_like(Q)
    Y = torch.empty((M, C), dtype=torch.bfloat16, device="cuda")
    U = torch.empty((M, F), dtype=torch.bfloat16, device="cuda")
    Z = torch.empty((M, C), dtype=torch.bfloat16, device="cuda")
    names = ["qkv_rope_append", "attention", "out_proj", "mlp_up", "mlp_down"]
    flops = [2 * M * 3 * H * d * C, None, 2 * M * C * H * d, 2 * M * F * C, 2 * M * C * F]

    def one(ev=None):
        steps = [
            lambda: kv.qkv_append_round(active, X, Wq, Q, rope=wi.WAN21_GRID, stream=stream),
            lambda: kv.round_attn(active, POLICY, Q, A, stream),
            lambda: kv.linear(A.view(M, H * d), Wo, Y, R=X, stream=stream),
            lambda: kv.linear(Y, W1, U, act=wave.ACT_GELU_TANH, stream=stream),
            lambda: kv.linear(U, W2, Z, R=Y, stream=stream),
        ]
        for i, f in enumerate(steps):
            if ev is not None:
                ev[i].record(stream)
            f()
        if ev is not None:
            ev[len(steps)].record(stream)
        for nd in active:
            kv.release(*nd)

    one()  # the attention FLOPs come from the library's own key tables
    kv.qkv_append_round(active, X, Wq, Q, rope=wi.WAN21_GRID, stream=stream)
    table = kv.gather_table(active, POLICY)
    for nd in active:
        kv.release(*nd)
    flops[1] = sum(4 * T * sum(v for _, v in rows) * H * d for rows in table)
    for _ in range(2):
        one()
    torch.cuda.synchronize()
    reps = max(3, min(args.steps, 10))
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(reps)]
    torch.cuda._sleep(int(3e6))
    for r in range(reps):
        one(evs[r])
    torch.cuda.synchronize()
    kv.status(stream)
    per = [[evs[r][i].elapsed_time(evs[r][i + 1]) for r in range(reps)] for i in range(5)]
    total = [evs[r][0].elapsed_time(evs[r][5]) for r in range(reps)]
    ms_round = statistics.median(total)
    peak = _measured_peaks()[0]["bf16_tflops"]
    kernels = {}
    for i, name in enumerate(names):
        ms = statistics.median(per[i])
        tf = flops[i] / (ms * 1e-3) / 1e12
        kernels[name] = {"ms": round(ms, 4), "flops": flops[i], "tflops": round(tf, 2),
                         "frac": round(tf / peak, 4)}
    upd = sum(1 for nd in active if nd[1] > 0)
    return {"what": "one transformer block per round: QKV projection + rotary + K/V append "
                    "(one launch for the round's nodes), wave attention, out-projection + "
                    "residual, tanh-GELU MLP up, MLP down + residual; Wan2.1-1.3B shapes "
                    f"(C {C}, MLP {F}, grid {wi.WAN21_GRID}), random weights",
            "ms_per_round": round(ms_round, 4), "flops_per_round": sum(flops),
            "tflops": round(sum(flops) / (ms_round * 1e-3) / 1e12, 2),
            "chunk_updates_per_s": round(upd / (ms_round * 1e-3), 2),
            "gemm_kernel": "gemm_wide_kernel", "kernels": kernels,
            "peak_tflops": peak, "reps": reps}


# ------------------------------------------------------------------ CPU oracle

def _oracle_round():
    """Float64 inputs of the timed round for the oracle (rank 0 only)."""
    from oracle import cache as ocache
    from oracle import schedule as osched
    wl = wi.WAN21
    active = osched.schedule(wl.chunks, wl.levels, POLICY, wl.window)[ROUND]
    ents = set()
    for n in active:
        ents.update(ocache.key_entries(n, POLICY, wl.window, False))

    def f64(kind, e):
        return wi.bf16_bits_to_f64(
            wi.node_tensor(kind, e[0], e[1], wl.tokens, wl.heads, wl.head_dim, wl.scale))

    entries = {e: (f64("k", e), f64("v", e)) for e in sorted(ents)}
    qs = {n: f64("q", n) for n in active}
    return active, entries, qs


def _sample_rows(n_rows, T):
    return np.unique(np.linspace(0, T - 1, n_rows).astype(np.int64))


def _oracle_sample(active, entries, qs, n_rows):
    from oracle import attention as oatt
    wl = wi.WAN21
    rows = _sample_rows(n_rows, wl.tokens)
    t = time.perf_counter()
    oatt.round_attention(active, POLICY, wl.window, qs, entries, None,
                         {n: rows for n in active})
    dt = time.perf_counter() - t
    from oracle import cache as ocache
    flops = 0
    for n in active:
        nk = len(ocache.key_entries(n, POLICY, wl.window, False)) * wl.tokens
        flops += 4 * len(rows) * nk * wl.heads * wl.head_dim
    return dt, flops, len(rows)


def _cores():
    try:
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
        return max(i.get("num_threads", 1) for i in info) if info else os.cpu_count()
    except Exception:
        return os.cpu_count()


# Query rows per node in one oracle sample: the same sample for the CPU-baseline
# leg (repeated for about --cpu-seconds) and for each step of the reference arm.
ORACLE_SAMPLE_ROWS = 32


def cpu_baseline(target_s=10.0):
    active, entries, qs = _oracle_round()
    _oracle_sample(active, entries, qs, 4)  # first touch of the float64 inputs
    total, flops, reps, nr = 0.0, 0, 0, 0
    while total < target_s or reps < 1:
        dt, f, nr = _oracle_sample(active, entries, qs, ORACLE_SAMPLE_ROWS)
        total += dt
        flops += f
        reps += 1
    out = {"value": round(flops / total / 1e12, 6), "unit": UNIT, "cores": _cores(),
           "kind": "oracle",
           "sample": f"{reps} x {nr} of 4680 query rows of each of the 5 nodes, all 12 heads, "
                     f"full key lists ({flops / 1e9:.1f} GFLOP in {total:.2f} s, float64 numpy); "
                     "the reference arm times the same sample per step"}
    try:  # the same sample on one core
        import threadpoolctl
        with threadpoolctl.threadpool_limits(limits=1):
            dt1, f1, _ = _oracle_sample(active, entries, qs, ORACLE_SAMPLE_ROWS)
        out["value_1core"] = round(f1 / dt1 / 1e12, 6)
        out["sample_1core"] = f"one sample ({f1 / 1e9:.1f} GFLOP in {dt1:.2f} s) on 1 thread"
    except Exception as e:  # threadpoolctl missing: no 1-core figure
        out["value_1core"] = None
        out["sample_1core"] = f"not measured: {type(e).__name__}"
    return out


def run_reference(args):
    ws, rank, _ = dist_env()
    if rank != 0:
        return
    active, entries, qs = _oracle_round()
    n_rows = ORACLE_SAMPLE_ROWS
    for _ in range(args.warmup):
        _oracle_sample(active, entries, qs, n_rows)
    times, flops = [], 0
    for _ in range(args.steps):
        dt, flops, nr = _oracle_sample(active, entries, qs, n_rows)
        times.append(dt)
    total = sum(times)
    value = flops * len(times) / total / 1e12
    line = {
        "metric": METRIC, "value": round(value, 6), "unit": UNIT, "n_gpus": ws,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1e3 * total / len(times), 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "impl": "reference", "config": _config(),
        "cpu_baseline": {"value": round(value, 6), "unit": UNIT, "cores": _cores(),
                         "kind": "oracle",
                         "sample": f"{nr} of 4680 query rows per node per step, all heads, "
                                   "full key lists"},
        "e2e": {"value": round(value, 6), "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["wave", "reference"], default="wave")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-block", action="store_true",
                    help="skip the whole-block round (projection, attention, MLP)")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--clocks-csv", default=None,
                    help="keep the raw nvidia-smi samples here ({rank} is replaced); "
                         "default: a temporary file")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default=DEFAULT_WORKLOAD,
                    help="timed round; the default is the headline Wan2.1-shaped round")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
