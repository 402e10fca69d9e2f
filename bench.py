#!/usr/bin/env python
"""Benchmark of block-sparse 3D-RoPE attention (one attention layer per step).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload i2v_480p] [--no-extra] [--no-cpu-baseline]

One step = one lc_bsa_forward call over one layer: B=1 per GPU, 32 heads x 64,
the 480x832 93-frame image-to-video latent (24x30x52 = 37,440 tokens, first
frame = condition, local=2, stride=4) unless --workload says otherwise.  The
metric is attended TFLOP/s (4 * head_dim * heads * attended token pairs per
second) with ms per layer and the fraction of the measured bf16 dense tensor
peak.  Inputs (q, k, v: 153 MB each) are larger than the 126 MB L2, so no
flush is needed between steps.  With N > 1 (torchrun) every rank runs its own
batch element (weak scaling, no collective on the data path); the time is the
max over ranks.

--impl reference times the fp64 CPU oracle (the reference arm of this
project) on the host cores, on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import re
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "block-sparse attn ms/layer, attended TFLOP/s, % bf16 tensor peak @37k/86k tok"
UNIT = "attended TFLOP/s"
KERNEL_SRC = os.path.join(ROOT, "block_sparse_attention_rope_b200", "csrc", "attn_sm100.cu")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.json")
FALLBACK_PEAK_TFLOPS = 1590.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="i2v_480p")
    ap.add_argument("--no-extra", action="store_true",
                    help="time only --workload (skip the other workloads, backward and ring)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--backward-only", action="store_true",
                    help="time only the backward pass of --workload (one JSON line; for profiling)")
    ap.add_argument("--plan-only", action="store_true",
                    help="time only the planner and the RoPE tables of --workload (one JSON "
                         "line; for profiling)")
    ap.add_argument("--ring-only", type=int, default=0, metavar="RANKS",
                    help="time only the ring over RANKS ranks (all in this process) on "
                         "--workload (one JSON line; for profiling)")
    return ap.parse_args()


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["bf16_tflops"]), "measured (MEASURED_PEAKS.json bf16_tflops, burst)"
    return FALLBACK_PEAK_TFLOPS, "fallback 1.59 PFLOP/s"


def kernel_hash() -> str:
    """sha256[:16] of the kernel source's code: comments and whitespace are
    removed first, so a comment edit does not orphan the committed counters."""
    src = open(KERNEL_SRC).read()
    src = re.sub(r"/\*.*?\*/", " ", src, flags=re.S)
    src = re.sub(r"//[^\n]*", " ", src)
    src = re.sub(r"\s+", " ", src).strip()
    return hashlib.sha256(src.encode()).hexdigest()[:16]


def traffic_for(workload: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on the current kernel source; else None."""
    if not os.path.exists(TRAFFIC_FILE):
        return None
    d = json.load(open(TRAFFIC_FILE))
    e = d.get(workload)
    if not e or e.get("kernel_sha") != kernel_hash():
        return None
    return e.get("dram_bytes_per_launch")


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML every 10 ms."""

    def __init__(self, device_index: int):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # pragma: no cover
            self.nv, self.err = None, str(e)

    def _run(self):
        nv = self.nv
        names = {
            "gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4,
            "hw_slowdown": 0x8, "sync_boost": 0x10, "sw_thermal_slowdown": 0x20,
            "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80,
        }
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for n, bit in names.items():
                    if r & bit:
                        self.reasons.add(n)
            except Exception:
                pass
            time.sleep(0.01)

    def __enter__(self):
        if self.nv:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self.nv:
            self.t.join()

    def summary(self):
        if not self.nv:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"]}
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons - {"gpu_idle"}),
                "samples": len(self.samples)}


def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def max_over_ranks(value: float, dist, device: str = "cuda") -> float:
    """Max of a per-rank time over all ranks (one all-reduce, outside the data
    path); identity without a process group."""
    if dist is None:
        return value
    import torch
    t = torch.tensor([value], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_seed_offset(rank: int) -> int:
    """Each rank draws its own batch element (weak scaling: fixed work per GPU)."""
    return rank


# ----------------------------------------------------------------------------- ours
def time_forward(api, torch, w, d, plan, rope, steps, warmup, dist, stream):
    """Device time of `steps` back-to-back forward calls, bracketed by a
    barrier and synchronisations; per-launch CUDA events on the launching
    stream.  Returns (max-over-ranks total ms, mean per-launch ms)."""
    out = torch.empty_like(d["q"])
    call = (lambda: api.forward_cached(d["q"], d["k"], d["v"], d["cond_k"], d["cond_v"], plan,
                                       rope, out=out, stream=stream)) if w.cached else \
        (lambda: api.forward(d["q"], d["k"], d["v"], plan, rope, out=out, stream=stream))
    with torch.cuda.stream(stream):
        for _ in range(warmup):
            call()
    torch.cuda.synchronize()
    if api.last_device_status() != 0:
        raise RuntimeError("device status set during warm-up")
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(steps + 1)]
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        evs[0].record(stream)
        for i in range(steps):
            call()
            evs[i + 1].record(stream)
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    per = [evs[i].elapsed_time(evs[i + 1]) for i in range(steps)]
    total = evs[0].elapsed_time(evs[-1])
    total = max_over_ranks(total, dist)
    st = api.last_device_status()
    if st != 0:
        raise RuntimeError("device status %d after the timed region" % st)
    time_forward.last_spread = (min(per), statistics.median(per), max(per))
    return total, sum(per) / len(per), out


def time_backward(api, synthetic, torch, name, steps, warmup, stream):
    """Device time of the backward pass (lc_bsa_backward) on one workload:
    the forward's out and lse are produced first, outside the timed region.
    Algorithmic work 10 * 64 FLOP per attended pair and head (recomputed S,
    dP, dQ, dK, dV)."""
    w = synthetic.get(name)
    x = synthetic.make_inputs(w, device="cuda")
    g = synthetic.make_dout(w, device="cuda")
    plan = api.Plan(w.T, w.H, w.W, local=w.local, stride=w.stride, n_cond=w.n_cond)
    rope = api.Rope3D(w.T, w.H, w.W)
    with torch.cuda.stream(stream):
        out, lse = api.forward(x["q"], x["k"], x["v"], plan, rope, return_lse=True, stream=stream)
        for _ in range(warmup):
            api.backward(x["q"], x["k"], x["v"], out, lse, g, plan, rope, stream=stream)
    torch.cuda.synchronize()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    with torch.cuda.stream(stream):
        ev[0].record(stream)
        for _ in range(steps):
            api.backward(x["q"], x["k"], x["v"], out, lse, g, plan, rope, stream=stream)
        ev[1].record(stream)
    torch.cuda.synchronize()
    if api.last_device_status() != 0:
        raise RuntimeError("device status set by the backward pass")
    ms = ev[0].elapsed_time(ev[1]) / steps
    pairs = plan.info().attended_token_pairs
    flops = 10.0 * w.head_dim * w.heads * w.batch * pairs
    return {"workload": name, "ms_per_layer": round(ms, 3),
            "attended_tflops": round(flops / (ms * 1e-3) / 1e12, 3),
            "work": "10*64 FLOP per attended pair and head",
            "kernels": "rope_k_kernel (Q', K'), bwd_delta, bsa_bwd_sm100_kernel (tcgen05), "
                       "bwd_grad_finalize"}


def time_ring(api, synthetic, torch, name, world, stream, reps=3):
    """Ring context parallelism over `world` ranks, every rank run in turn on
    this GPU with the K/V shards it receives already resident (the NCCL
    exchange is left out: on NVLink it overlaps the compute).  Per rank: device
    time of its own q / k rotation, its shard forwards and the final merge;
    the slowest rank bounds a real ring's step.  Compared with one
    whole-sequence launch divided by `world`."""
    import numpy as np
    from block_sparse_attention_rope_b200 import ring
    w = synthetic.get(name)
    x = synthetic.make_inputs(w, device="cuda")
    plan = api.Plan(w.T, w.H, w.W, local=w.local, stride=w.stride, n_cond=w.n_cond)
    rope = api.Rope3D(w.T, w.H, w.W)
    rp, ci = plan.csr()
    cb = plan.info().num_cond_blocks
    shards = ring.planned_shards(rp.tolist(), ci.tolist(), cb, world, heads=w.heads,
                                 batch=w.batch)
    ranks = [ring.GpuRingRank(api, w.T, w.H, w.W, local=w.local, stride=w.stride,
                              n_cond=w.n_cond, shards=shards, rank=r, rope=rope, batch=w.batch,
                              heads=w.heads) for r in range(world)]
    toks = ranks[0].sched.tokens
    own = [{n: x[n][:, a:b].contiguous() for n in ("q", "k", "v")} for a, b in toks]
    k_rot = [ranks[s].rotate(own[s]["k"], s, None) for s in range(world)]  # as received

    def run_rank(r):
        return ranks[r].forward(own[r]["q"], own[r]["k"], own[r]["v"],
                                fetch=lambda src: (k_rot[src], own[src]["v"]))
    per = []
    with torch.cuda.stream(stream):
        for r in range(world):
            run_rank(r)  # warm-up
        torch.cuda.synchronize()
        for r in range(world):
            ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
            ev[0].record(stream)
            for _ in range(reps):
                run_rank(r)
            ev[1].record(stream)
            torch.cuda.synchronize()
            per.append(ev[0].elapsed_time(ev[1]) / reps)
        out = torch.empty_like(x["q"])
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
        api.forward(x["q"], x["k"], x["v"], plan, rope, out=out, stream=stream)
        ev[0].record(stream)
        for _ in range(reps):
            api.forward(x["q"], x["k"], x["v"], plan, rope, out=out, stream=stream)
        ev[1].record(stream)
    torch.cuda.synchronize()
    if api.last_device_status() != 0:
        raise RuntimeError("device status set by the ring")
    full = ev[0].elapsed_time(ev[1]) / reps
    steps = sum(sum(rr.sched.computes) for rr in ranks)
    return {"workload": name, "ranks": world, "shards_blocks": shards,
            "computing_steps": steps, "skipped_steps": world * world - steps,
            "ms_per_rank_max": round(max(per), 3), "ms_per_rank_mean": round(sum(per) / world, 3),
            "whole_sequence_ms": round(full, 3), "ideal_ms": round(full / world, 3),
            "compute_efficiency": round(full / world / max(per), 3),
            "kernels": "per rank: rope_apply (q, k once); per step: bsa_sm100_kernel (steps "
                       "after the first by programmatic dependent launch); lse_merge_parts once"}


def time_e2e(api, torch, w, host, plan, rope, steps, stream):
    """End to end through the public API: every step copies its inputs from
    pinned host memory to the device, runs the forward, and reads the result
    back into pinned host memory.  Timed two ways: serial (copy in, compute,
    copy out, one after another on one stream) and pipelined as a serving loop
    runs it (two device buffer sets; the host-to-device copy of step i+1 and
    the device-to-host copy of step i-1 run on their own streams while step i
    computes).  Returns (pipelined ms / step, serial ms / step, bytes in,
    bytes out)."""
    names = list(host.keys())
    dev = [{k: torch.empty_like(host[k], device="cuda") for k in names} for _ in range(2)]
    out_d = [torch.empty_like(dev[0]["q"]) for _ in range(2)]
    out_h = [torch.empty_like(host["q"]).pin_memory() for _ in range(2)]
    h2d = sum(v.numel() * v.element_size() for v in host.values())
    d2h = out_h[0].numel() * out_h[0].element_size()

    def forward(b):
        d = dev[b]
        if w.cached:
            api.forward_cached(d["q"], d["k"], d["v"], d["cond_k"], d["cond_v"], plan, rope,
                               out=out_d[b], stream=stream)
        else:
            api.forward(d["q"], d["k"], d["v"], plan, rope, out=out_d[b], stream=stream)

    def serial_step():
        with torch.cuda.stream(stream):
            for k in names:
                dev[0][k].copy_(host[k], non_blocking=True)
            forward(0)
            out_h[0].copy_(out_d[0], non_blocking=True)

    ev = lambda: torch.cuda.Event(enable_timing=True)
    serial_step()
    torch.cuda.synchronize()
    e0, e1 = ev(), ev()
    e0.record(stream)
    for _ in range(steps):
        serial_step()
    e1.record(stream)
    torch.cuda.synchronize()
    serial_ms = e0.elapsed_time(e1) / steps

    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    in_done = [torch.cuda.Event() for _ in range(2)]
    comp_done = [torch.cuda.Event() for _ in range(2)]
    out_done = [torch.cuda.Event() for _ in range(2)]
    t0, t1 = ev(), ev()
    t0.record(s_in)
    for i in range(steps + 1):  # one extra step: the first fills the pipeline untimed
        b = i % 2
        if i == 1:
            torch.cuda.synchronize()
            t0.record(s_in)
        if i >= 2:
            s_in.wait_event(comp_done[b])      # step i-2 has read dev[b]
        with torch.cuda.stream(s_in):
            for k in names:
                dev[b][k].copy_(host[k], non_blocking=True)
            in_done[b].record(s_in)
        stream.wait_event(in_done[b])
        if i >= 2:
            stream.wait_event(out_done[b])     # step i-2's result has left out_d[b]
        forward(b)
        comp_done[b].record(stream)
        s_out.wait_event(comp_done[b])
        with torch.cuda.stream(s_out):
            out_h[b].copy_(out_d[b], non_blocking=True)
            out_done[b].record(s_out)
    t1.record(s_out)
    torch.cuda.synchronize()
    return t0.elapsed_time(t1) / steps, serial_ms, h2d, d2h


def measure_workload(api, synthetic, torch, name, steps, warmup, dist, rank, stream, e2e_steps=0):
    w = synthetic.get(name)
    plan = api.Plan(w.T, w.H, w.W, local=w.local, stride=w.stride, n_cond=w.n_cond)
    rope = api.Rope3D(w.T, w.H, w.W)
    info = plan.info()
    pairs = info.attended_token_pairs_noisy if w.cached else info.attended_token_pairs
    flops = 4.0 * w.head_dim * w.heads * w.batch * pairs
    host = synthetic.make_inputs(w, seed_offset=rank_seed_offset(rank))
    host = {k: v.pin_memory() for k, v in host.items()}
    d = {k: v.cuda() for k, v in host.items()}
    total_ms, launch_ms, out = time_forward(api, torch, w, d, plan, rope, steps, warmup, dist,
                                            stream)
    res = {"w": w, "flops": flops, "pairs": pairs, "total_ms": total_ms, "launch_ms": launch_ms,
           "scores": kernel_scores_per_head(plan, w.cached) * w.heads * w.batch,
           "spread": [round(x, 4) for x in time_forward.last_spread],
           "nnz": info.nnz}
    if e2e_steps:
        del d, out
        torch.cuda.empty_cache()
        res["e2e_ms"], res["e2e_serial_ms"], res["h2d"], res["d2h"] = time_e2e(
            api, torch, w, host, plan, rope, e2e_steps, stream)
    return res


def kernel_scores_per_head(plan, cached: bool) -> int:
    """Score elements the bf16 kernel forms (one exp2 each) per head: work
    items are groups of 4 consecutive query blocks of one segment (two
    128-row tiles), walking the union of their key lists 128 keys at a time.
    Counted on the host from the plan's block CSR."""
    import numpy as np
    rp, ci = (t.numpy() for t in plan.csr())
    inf = plan.info()
    Cb, Nb = inf.num_cond_blocks, inf.num_noisy_blocks
    total = 0
    for seg0, nb in ((0, Cb), (Cb, Nb)):
        if cached and seg0 == 0:
            continue
        for g in range(0, nb, 4):
            r0, r1 = seg0 + g, seg0 + min(g + 4, nb)
            n = len(np.unique(ci[rp[r0]:rp[r1]]))
            total += 256 * 128 * ((n + 1) // 2)
    return total


def oracle_sample(w, x, heads, row_stride):
    """Time the fp64 oracle, as it stands, on `heads` (one at a time: a head
    is an independent unit of the layer) x every `row_stride`-th query row.
    The oracle's own RoPE of that head's q and k is inside the timed region.
    Returns (attended TFLOP/s, seconds, threads, attended pairs)."""
    import numpy as np

    import oracle
    Nc, Nn, Cb, Nb = oracle.segment_sizes(w.T, w.H, w.W, w.n_cond)
    if w.cached:
        k = np.concatenate([oracle._f64(x["cond_k"]), oracle._f64(x["k"])], axis=1)
        v = np.concatenate([oracle._f64(x["cond_v"]), oracle._f64(x["v"])], axis=1)
        q, q_off, nq = oracle._f64(x["q"]), Nc, Nn
    else:
        q, k, v = oracle._f64(x["q"]), oracle._f64(x["k"]), oracle._f64(x["v"])
        q_off, nq = 0, w.n_tokens
    rows = np.arange(0, nq, row_stride)
    trip = np.stack([np.zeros_like(rows), np.zeros_like(rows), rows], axis=1)
    # attended keys of the sampled rows, from the oracle's block CSR
    rp, ci = oracle.block_csr(w.T, w.H, w.W, w.block, w.local, w.stride, w.n_cond)
    bsize = np.array([min(64, Nc - 64 * b) for b in range(Cb)] +
                     [min(64, Nn - 64 * j) for j in range(Nb)], dtype=np.int64)
    keys = np.array([bsize[ci[rp[i]:rp[i + 1]]].sum() for i in range(Cb + Nb)])
    tok = rows + q_off
    qb = np.where(tok < Nc, tok // 64, Cb + (tok - Nc) // 64)
    pairs = int(keys[qb].sum()) * len(heads)
    sec = 0.0
    for h in heads:
        qh, kh, vh = (np.ascontiguousarray(a[:, :, h:h + 1]) for a in (q, k, v))
        t0 = time.perf_counter()
        oracle.attention_rows(qh, kh, vh, H=w.H, W=w.W, Nc=Nc, block=w.block, local=w.local,
                              stride=w.stride, rows=trip, q_offset=q_off)
        sec += time.perf_counter() - t0
    return 4.0 * w.head_dim * pairs / sec / 1e12, sec, oracle.max_threads(), pairs


def cpu_baseline(name: str):
    """The oracle on a bounded sample of the workload (about 10-30 s of CPU
    work on the benchmark host): 8 heads x every 6th query row."""
    from block_sparse_attention_rope_b200 import synthetic
    w = synthetic.get(name)
    x = synthetic.make_inputs(w)
    heads, stride = list(range(8)), 3
    tf, sec, threads, pairs = oracle_sample(w, x, heads, stride)
    sample = ("fp64 oracle (C, OpenMP) on heads 0-7 x every %dth query row of %s "
              "(%.3g attended token pairs, RoPE of those heads included), %.1f s" %
              (stride, name, pairs, sec))
    return tf, sec, threads, sample


def exp_roofline(res, clocks):
    """The softmax's exp2 runs on the MUFU unit: 16 results per clock per SM
    on B200, 148 SMs.  At head dim 64 that unit, not the tensor pipe, sets the
    ceiling (4*64 attended FLOP per exp2 against ~16 x 256 per clock)."""
    mhz = (clocks or {}).get("sm_mhz") or 1965.0
    peak = 148 * 16 * mhz * 1e6 / 1e9
    achieved = res["scores"] / (res["launch_ms"] * 1e-3) / 1e9
    return {"bound": "alu", "unit": "Gexp2/s", "achieved": round(achieved, 1),
            "peak": round(peak, 1), "frac": round(achieved / peak, 4),
            "peak_derivation": "148 SM x 16 MUFU ex2/clk x median SM clock under load (%.0f MHz)"
                               % mhz,
            "work": "%d score elements per launch (kernel tiles, masked padding included)"
                    % res["scores"]}


def workload_config(w, world: int) -> dict:
    """The `config` object of a bench line (both arms name the workload the
    same way)."""
    return {"workload": w.name, "T": w.T, "H": w.H, "W": w.W, "n_cond_frames": w.n_cond,
            "tokens": w.n_tokens, "heads": w.heads, "head_dim": w.head_dim, "block": w.block,
            "local": w.local, "stride": w.stride, "batch_per_gpu": w.batch,
            "global_batch": w.batch * world,
            "parallelism": "replicas: one batch element per GPU, no data-path collective",
            "l2": "inputs larger than L2 (q, k, v 153 MB each); no flush"}


def run_ours(a):
    import torch
    world, rank, local = dist_env()
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    from block_sparse_attention_rope_b200 import api, synthetic
    stream = torch.cuda.Stream()
    peak, peak_src = peaks()
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    nvml_index = int(vis.split(",")[local]) if vis else local
    with ClockSampler(nvml_index) as clk:
        main = measure_workload(api, synthetic, torch, a.workload, a.steps, a.warmup, dist, rank,
                                stream)
    clocks = clk.summary()
    e2e = None
    if a.e2e_steps > 0:
        w = main["w"]
        res = measure_workload(api, synthetic, torch, a.workload, 1, 1, dist, rank, stream,
                               e2e_steps=a.e2e_steps)
        e2e_ms = res["e2e_ms"]
        e2e_ms = max_over_ranks(e2e_ms, dist)
        serial_ms = max_over_ranks(res["e2e_serial_ms"], dist)
        e2e = {"value": round(world * res["flops"] / (e2e_ms * 1e-3) / 1e12, 3), "unit": UNIT,
               "ms_per_step": round(e2e_ms, 3), "h2d_bytes_per_step": res["h2d"],
               "d2h_bytes_per_step": res["d2h"],
               "path": "pinned host q/k/v -> device, lc_bsa_forward, out -> pinned host; "
                       "pipelined: the copy in of step i+1 and the copy out of step i-1 run "
                       "on their own streams while step i computes",
               "serial": {"value": round(world * res["flops"] / (serial_ms * 1e-3) / 1e12, 3),
                          "ms_per_step": round(serial_ms, 3),
                          "path": "copy in, forward, copy out one after another"}}
    extra = {}
    # every other named workload: the 86,400-token refine pass, the cached
    # continuation and the five masks of the sparsity sweep at 37,440 tokens
    names = [] if a.no_extra else (["refine_720p", "continuation_cached"] +
                                   ["sweep_" + s for s in
                                    ("dense", "l2s4", "l2s8", "l1s16", "l1s32")])
    for n in names:
        if n == a.workload:
            continue
        r = measure_workload(api, synthetic, torch, n, max(10, a.steps // 2), a.warmup, dist, rank,
                             stream)
        ms = r["total_ms"] / max(10, a.steps // 2)
        extra[n] = {"tokens": r["w"].n_tokens, "ms_per_layer": round(ms, 4),
                    "attended_tflops": round(r["flops"] / (ms * 1e-3) / 1e12, 2),
                    "pct_bf16_peak": round(100.0 * r["flops"] / (r["launch_ms"] * 1e-3) / 1e12 / peak, 2),
                    "attended_pairs_per_head": r["pairs"],
                    "launch_ms_min_median_max": r["spread"]}
    if not a.no_extra and a.workload == "i2v_480p":
        extra["backward_i2v_480p"] = time_backward(api, synthetic, torch, "i2v_480p", 2, 1,
                                                   stream)
        extra["ring_8_ranks_i2v_480p"] = time_ring(api, synthetic, torch, "i2v_480p", 8, stream)
        extra["ring_8_ranks_refine_720p"] = time_ring(api, synthetic, torch, "refine_720p", 8,
                                                      stream)
    w = main["w"]
    ms = main["total_ms"] / a.steps
    value = world * main["flops"] * a.steps / (main["total_ms"] * 1e-3) / 1e12
    achieved = main["flops"] / (main["launch_ms"] * 1e-3) / 1e12
    line = {
        "metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": world,
        "steps": a.steps, "warmup": a.warmup, "ms_per_step": round(ms, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) q/k/v, bf16)",
        "config": workload_config(w, world),
        "pct_bf16_peak": round(100.0 * achieved / peak, 2),
        "launch_ms_min_median_max": main["spread"],
        "roofline": {"bound": "tensor", "achieved": round(achieved, 2), "peak": peak,
                     "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
                     "peak_source": peak_src, "traffic": traffic_for(w.name),
                     "kernel": "bsa_sm100_kernel",
                     "algorithmic": "4*64*32*%d FLOP per launch" % main["pairs"]},
        "exp_roofline": exp_roofline(main, clocks),
        "gpu_launches": 2 * a.steps,  # per call: rope_k_kernel (K once) + bsa_sm100_kernel
        "clocks": clocks,
        "e2e": e2e,
        "extra": extra,
    }
    if rank == 0 and world == 1 and not a.no_cpu_baseline:
        tf, sec, threads, sample = cpu_baseline(a.workload)
        line["cpu_baseline"] = {"value": tf, "unit": UNIT, "cores": threads, "kind": "oracle",
                                "sample": sample, "seconds": round(sec, 2)}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


def run_reference(a):
    """The project's reference arm: the fp64 oracle on the host cores.  Each
    step is one head of the workload (cycling through the heads), every 16th
    query row, so that --steps K finishes in a few minutes.  Under torchrun
    only rank 0 works."""
    world, rank, local = dist_env()
    if rank != 0:
        return
    from block_sparse_attention_rope_b200 import synthetic
    w = synthetic.get(a.workload)
    x = synthetic.make_inputs(w)
    for i in range(a.warmup):
        oracle_sample(w, x, [i % w.heads], 64)
    secs, pairs_tot, threads = 0.0, 0, 1
    for i in range(a.steps):
        tf, sec, threads, pairs = oracle_sample(w, x, [i % w.heads], 16)
        secs += sec
        pairs_tot += pairs
    tf = 4.0 * w.head_dim * pairs_tot / secs / 1e12
    sample = ("fp64 oracle (C, OpenMP): %d steps of one head x every 16th query row of %s, "
              "RoPE of the head included" % (a.steps, w.name))
    line = {"metric": METRIC, "value": tf, "unit": UNIT, "n_gpus": world, "steps": a.steps,
            "warmup": a.warmup, "ms_per_step": round(1e3 * secs / a.steps, 2),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded N(0,1) q/k/v, bf16 values upcast to f64)",
            "impl": "reference",
            "config": workload_config(w, world),
            "cpu_baseline": {"value": tf, "unit": UNIT, "cores": threads, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": tf, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    a = parse()
    if a.impl == "reference":
        run_reference(a)
    elif a.backward_only:
        import torch
        torch.cuda.set_device(0)
        from block_sparse_attention_rope_b200 import api, synthetic
        r = time_backward(api, synthetic, torch, a.workload, a.steps, a.warmup,
                          torch.cuda.current_stream())
        print(json.dumps(dict(metric="backward ms per layer", value=r["ms_per_layer"], unit="ms",
                              higher_is_better=False, **r)), flush=True)
    elif a.plan_only:
        import torch
        torch.cuda.set_device(0)
        from block_sparse_attention_rope_b200 import api, synthetic
        w = synthetic.get(a.workload)
        st = torch.cuda.current_stream()
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
        for _ in range(2):  # warm-up (first-call setup outside the timed pass)
            api.Plan(w.T, w.H, w.W, local=w.local, stride=w.stride, n_cond=w.n_cond).close()
            api.Rope3D(w.T, w.H, w.W).close()
        torch.cuda.synchronize()
        n = max(1, a.steps)
        ev[0].record(st)
        plans = [api.Plan(w.T, w.H, w.W, local=w.local, stride=w.stride, n_cond=w.n_cond)
                 for _ in range(n)]
        ev[1].record(st)
        ropes = [api.Rope3D(w.T, w.H, w.W) for _ in range(n)]
        ev[2].record(st)
        torch.cuda.synchronize()
        inf = plans[0].info()
        print(json.dumps(dict(metric="plan build ms", value=round(ev[0].elapsed_time(ev[1]) / n, 4),
                              unit="ms", higher_is_better=False, workload=w.name,
                              rope_tables_ms=round(ev[1].elapsed_time(ev[2]) / n, 4),
                              nnz=inf.nnz, num_q_blocks=inf.num_q_blocks)), flush=True)
    elif a.ring_only:
        import torch
        torch.cuda.set_device(0)
        from block_sparse_attention_rope_b200 import api, synthetic
        r = time_ring(api, synthetic, torch, a.workload, a.ring_only, torch.cuda.current_stream(),
                      reps=max(1, a.steps))
        print(json.dumps(dict(metric="ring ms per rank (slowest)", value=r["ms_per_rank_max"],
                              unit="ms", higher_is_better=False, **r)), flush=True)
    else:
        run_ours(a)


if __name__ == "__main__":
    main()
