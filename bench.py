#!/usr/bin/env python3
"""Benchmark of the paged decode hot path on B200.

One step = one decode step of one attention layer over a batch of sequences: the
cache write of each sequence's new token and paged decode attention over all
cached tokens.  Variants: append (pa_append_decode_v1: the write fused into the
v1 decode, one launch), v1 (pa_reshape_and_cache + pa_decode_v1), v2
(+ pa_decode_v2_partition / pa_decode_v2_merge) and fused (pa_reshape_and_cache +
the persistent pa_decode_fused); auto picks append for many short sequences,
fused for long or few sequences and cascade (pa_decode_cascade) for a batch that
shares a cached prefix.  Default workload: one Qwen3-32B layer (32 seqs, 64 q / 8 kv
heads, head_dim 128, block 16, 12480-block pool, lengths U{512..768}, fp16); the
same line then carries nested blocks for the 32K-context (persistent and split-K
forms), INT8, FP8 and mixed shared-prefix workloads, measured the same way.

Usage:
  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                  [--variant auto|append|v1|v2|fused]
  python bench.py --impl reference ...   # the oracle timed on the host cores

Timing: W untimed warm-up steps, then exactly K steps replayed from CUDA graphs,
bracketed by a barrier and a device synchronise, timed with CUDA events on the
launching stream (max over ranks).  The steps rotate over several input sets
whose KV bytes together exceed L2, so every step reads its KV from HBM.
Prints one JSON line (rank 0).
"""
from __future__ import annotations

import argparse
import copy
import datetime
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from paged_kv_cache_390_b200 import workloads as W  # noqa: E402

L2_BYTES = 126 * 1024 * 1024
METRIC = "paged decode attention effective KV GB/s (% of B200 HBM peak; seq-heads/s)"
FALLBACK_HBM_GBS = 6650.0
NOMINAL_HBM_GBS = 8000.0
# the 32K-context configuration (persistent split-K, and the two-kernel v2 with
# partitions of 512 tokens) and the INT8 / FP8 caches, beside the Qwen3-32B layer
DEFAULT_ALSO = "long_ctx_bf16,long_ctx_bf16@v2,quant_int8,quant_fp8,mixed_f16"
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "decode_traffic.json")
KERNEL_SOURCES = [os.path.join(ROOT, "paged_kv_cache_390_b200", "csrc", f)
                  for f in ("pa_decode.cu", "pa_fused.cu", "pa_tile.cuh", "pa_device.cuh",
                            "pa_write.cuh", "pa_internal.h", "pa_api.cu")]
STEP_DECODE = {"append": "append_decode_v1 (the new token's cache write fused into the v1 "
                         "decode: one launch)",
               "cascade": "decode_cascade (the shared prefix on tcgen05 once per kv head, beside "
                          "each sequence's own tokens on the persistent decode, then a "
                          "log-sum-exp merge: three launches)",
               "v1": "decode_v1",
               "v2": "decode_v2_partition(P={P}) + decode_v2_merge",
               "fused": "decode_fused (persistent, merge fused)"}
DOMINANT_KERNEL = {"append": "decode_tc_kernel (pa_append_decode_v1)",
                   "cascade": "prefill_kernel (shared prefix, tcgen05, on its own SMs) + "
                              "decode_fused_kernel (own tokens, on the other SMs) + "
                              "merge_partials_kernel: the whole call",
                   "v1": "decode_tc_kernel (pa_decode_v1)",
                   "v2": "decode_tc_kernel (pa_decode_v2_partition)",
                   "fused": "decode_fused_kernel (pa_decode_fused)"}


# ----------------------------------------------------------------------------- host logic

def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", str(rank)))
    return rank, world, local


def rank_seed(rank: int, base: int = 0) -> int:
    """Each rank decodes its own independent batch (weak scaling, no data exchange)."""
    return base + 1000 * rank


def max_over_ranks(value: float, device) -> float:
    """Max of a per-rank scalar across the process group (identity without one)."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank: float, world: int, seconds: float) -> float:
    return units_per_rank * world / seconds


def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    for p in KERNEL_SOURCES:
        with open(p, "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(workload: str, variant: str):
    """DRAM bytes per launch of the decode kernel from the committed ncu summary, if
    it was taken on the kernel source as it is now; else None."""
    try:
        with open(TRAFFIC_FILE) as f:
            d = json.load(f)
    except Exception:
        return None
    e = d.get(f"{workload}/{variant}")
    if not e or e.get("kernel_source_sha256_16") != kernel_source_hash():
        return None
    return e.get("dram_bytes_per_launch_full_size")


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 200 ms in the background."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        if not self.lines:
            return None
        sm, mx, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = max(mx, float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ----------------------------------------------------------------------------- our arm

class Step:
    """Device tensors of one input set and the launches of one decode step."""

    def __init__(self, pa, g_caches, batch, wl, variant, partition_size, device):
        self.pa = pa
        self.c = g_caches
        self.wl = wl
        self.q = batch.q.to(device)
        self.tables = batch.block_tables.to(device)
        self.lens = batch.seq_lens.to(device)
        self.nk = batch.new_key.to(device)
        self.nv = batch.new_value.to(device)
        self.slots = batch.new_slots.to(device)
        self.out = torch.empty_like(self.q)
        self.variant = variant
        self.P = partition_size
        S, H, D = self.q.shape
        self.max_len = int(batch.seq_lens.max())
        self.maxp = max(1, -(-self.max_len // self.P)) if variant == "v2" else 1
        self.ws = pa.V2Workspace(S, H, D, self.maxp, device) if variant == "v2" else None
        if variant == "cascade":
            key = ("cascade", S, H, D)
            if key not in Step._fused_ws:
                n = pa.lib().pa_decode_cascade_workspace_bytes(S, H, D)
                Step._fused_ws[key] = torch.zeros(n, dtype=torch.uint8, device=device)
            self.cws = Step._fused_ws[key]
        if variant == "fused":
            key = (S, wl.num_kv_heads, D)
            if key not in Step._fused_ws:         # one workspace serves every input set
                Step._fused_ws[key] = pa.FusedWorkspace(S, wl.num_kv_heads, D, device)
            self.fws = Step._fused_ws[key]

    _fused_ws = {}

    def cache_write(self):
        if self.variant == "append":
            return                                 # fused into decode_main
        c = self.c
        self.pa.reshape_and_cache(self.nk, self.nv, c["kc"], c["vc"], self.slots,
                                  cache_dtype=self.wl.cache_dtype, k_scale=c["ks"],
                                  v_scale=c["vs"])

    def decode_main(self):
        c, wl = self.c, self.wl
        if self.variant == "append":
            self.pa.append_decode_v1(self.q, self.nk, self.nv, self.slots, c["kc"], c["vc"],
                                     self.tables, self.lens, wl.scale, out=self.out,
                                     cache_dtype=wl.cache_dtype, k_scale=c["ks"],
                                     v_scale=c["vs"])
        elif self.variant == "cascade":
            self.pa.decode_cascade(self.q, c["kc"], c["vc"], self.tables, self.lens, wl.scale,
                                   wl.shared_prefix_tokens, out=self.out, workspace=self.cws)
        elif self.variant == "v1":
            self.pa.decode_v1(self.q, c["kc"], c["vc"], self.tables, self.lens, wl.scale,
                              out=self.out, cache_dtype=wl.cache_dtype, k_scale=c["ks"],
                              v_scale=c["vs"])
        elif self.variant == "fused":
            self.pa.decode_fused(self.q, c["kc"], c["vc"], self.tables, self.lens, wl.scale,
                                 out=self.out, workspace=self.fws, cache_dtype=wl.cache_dtype,
                                 k_scale=c["ks"], v_scale=c["vs"])
        else:
            self.pa.decode_v2_partition(self.q, c["kc"], c["vc"], self.tables, self.lens,
                                        wl.scale, self.P, self.ws.tmp_out, self.ws.max_logits,
                                        self.ws.exp_sums, cache_dtype=wl.cache_dtype,
                                        k_scale=c["ks"], v_scale=c["vs"])

    def decode_tail(self):
        if self.variant == "v2":
            self.pa.decode_v2_merge(self.out, self.ws.tmp_out, self.ws.max_logits,
                                    self.ws.exp_sums, self.lens, self.P)

    @property
    def launches(self):
        # cache write + decode (+ merge, or + the prefix kernel)
        return {"v2": 3, "append": 1, "cascade": 3}.get(self.variant, 2)


def workload_overrides(args, base) -> dict:
    """make_problem overrides: --block-size (the block size, and a pool of the same number
    of tokens) and --num-seqs (the batch size, the pool scaled with it)."""
    over = {}
    bs = getattr(args, "block_size", 0)
    if bs and bs != base.block_size:
        over["block_size"] = bs
        if base.num_blocks:
            over["num_blocks"] = base.num_blocks * base.block_size // bs
    ns = getattr(args, "num_seqs", 0)
    if ns and ns != base.num_seqs:
        over["num_seqs"] = ns
        if base.num_blocks:
            over["num_blocks"] = -(-over.get("num_blocks", base.num_blocks) * ns // base.num_seqs)
    return over


def workload_desc(wl_name, wl) -> str:
    return (f"{wl_name}: {wl.num_seqs} seqs, {wl.num_heads} q / {wl.num_kv_heads} kv heads, "
            f"head_dim {wl.head_dim}, block {wl.block_size}, cache {wl.cache_dtype}, lengths "
            f"{wl.lens} [{wl.len_lo},{wl.len_hi}]"
            + (f" after a {wl.shared_prefix_tokens}-token shared prefix"
               if wl.shared_prefix_tokens else ""))


def step_bytes(wl, batch):
    """Algorithmic bytes of one step: K/V (+scales) of every cached token, q read, out
    written, and the new rows read and written by the cache write."""
    lens = batch.seq_lens.numpy()
    kv = W.logical_kv_bytes(wl, lens)
    qo = W.qo_bytes(wl, len(lens))
    row_bytes = wl.num_kv_heads * wl.head_dim * {"f32": 4, "f16": 2, "bf16": 2}[wl.dtype]
    cache_el = W.CACHE_ELEM_BYTES[wl.cache_dtype]
    write = len(lens) * 2 * (row_bytes + wl.num_kv_heads * wl.head_dim * cache_el)
    decode = kv + qo
    return decode, decode + write, W.unique_kv_bytes(wl, lens) + qo


class DecodeSetup:
    """One workload on the device: its pool, with the history rows written by the
    library's cache write, and enough input sets (disjoint blocks) that their KV bytes
    together exceed the 126 MB L2 twice over, so every step reads its KV from HBM."""

    def __init__(self, pa, wl_name, rank, device, over=None, max_sets=8):
        over = over or {}
        base = W.WORKLOADS[wl_name]
        bs = over.get("block_size", base.block_size)
        probe = W.make_problem(wl_name, rank_seed(rank), num_batches=1, **over)
        per_set = W.logical_kv_bytes(probe.wl, probe.batch.seq_lens.numpy())
        n_sets = max(1, min(max_sets, math.ceil(2 * L2_BYTES / max(per_set, 1))))
        pool_tokens = over.get("num_blocks", base.num_blocks) * bs if base.num_blocks else 0
        if pool_tokens:
            fit = pool_tokens // max(1, int(probe.batch.seq_lens.sum()) + base.num_seqs * bs)
            n_sets = max(1, min(n_sets, fit))
        del probe
        p = W.make_problem(wl_name, rank_seed(rank), num_batches=n_sets, **over)
        self.name, self.p, self.wl, self.over = wl_name, p, p.wl, over
        self.device = device
        self.caches = {"kc": p.k_cache.to(device), "vc": p.v_cache.to(device),
                       "ks": p.k_scale.to(device) if p.k_scale is not None else None,
                       "vs": p.v_scale.to(device) if p.v_scale is not None else None}
        c, wl = self.caches, self.wl
        if p.hist_slots.numel():
            pa.reshape_and_cache(p.hist_key.to(device), p.hist_value.to(device), c["kc"],
                                 c["vc"], p.hist_slots.to(device), cache_dtype=wl.cache_dtype,
                                 k_scale=c["ks"], v_scale=c["vs"])
        torch.cuda.synchronize()
        self.max_len = max(int(b.seq_lens.max()) for b in p.batches)
        sb = [step_bytes(wl, b) for b in p.batches]
        # every set has its own lengths: the per-step figures average over the sets
        self.decode_bytes = float(np.mean([x[0] for x in sb]))
        self.bytes_per_step = float(np.mean([x[1] for x in sb]))
        self.unique_bytes = float(np.mean([x[2] for x in sb]))

    def resolve(self, pa, variant, partition_size=0):
        """(variant, P): auto -> cascade for a shared prefix, else the append step (v1
        with the write fused in) or the persistent decode by pick_decode_variant."""
        wl = self.wl
        sms = torch.cuda.get_device_properties(self.device).multi_processor_count
        P = partition_size or wl.partition_size or pa.choose_partition_size(
            self.max_len, wl.num_seqs, wl.num_kv_heads, sms, wl.block_size)
        if variant == "auto":
            if wl.shared_prefix_tokens and wl.cache_dtype in ("f16", "bf16") and wl.head_dim == 128:
                variant = "cascade"
            else:
                pick = pa.pick_decode_variant(wl.num_seqs, wl.num_kv_heads, self.max_len, sms)
                variant = "append" if pick == "v1" else pick
        return variant, P

    def kernel_bytes(self, variant):
        """Algorithmic bytes of the dominant launch: the append launch also moves the new
        rows (its bytes are the whole step's); with a shared prefix every variant counts
        the prefix once (a variant that streams it per sequence reads it from L2)."""
        if self.wl.shared_prefix_tokens:
            return self.unique_bytes
        return self.bytes_per_step if variant == "append" else self.decode_bytes


def event_plan(K, variant, every_arg, run_arg):
    """(every, run) of the in-graph kernel events, or None for none.  A one-launch step
    needs none: the timed region is K back-to-back launches of the kernel, so its
    events give the kernel's average launch duration without an event node inside
    the graph (each such node breaks the PDL overlap of the launches around it and
    costs several microseconds); --event-run / --event-every ask for windows of
    `run` launches every `every` steps instead.  Otherwise the decode launch of every
    `every`-th step is bracketed (0 = adapt to K so a short run still gives several)."""
    if variant == "append":
        if not run_arg and not every_arg:
            return None
        run = run_arg or max(2, min(10, K // 4))
        every = every_arg or (run if K <= 400 else 50)
        return max(every, run), run
    # every event node costs several microseconds of lost overlap: few of them in a
    # short run (two samples at K = 20), one every 50 steps in a long one
    every = every_arg or (50 if K >= 200 else max(1, K // 2))
    return every, 1


def time_decode(pa, setup, variant, P, K, Wm, args, stream, kernel_events=True):
    """W warm-up steps, then exactly K steps replayed from CUDA graphs, bracketed by a
    barrier and a device synchronise; CUDA events on the launching stream, max over
    ranks.

    The timed region runs from the completion of an untimed lead-in step to the
    completion of the K-th timed step: K intervals between consecutive step
    completions, which is the steady-state rate.  When K fits one graph
    (K <= --graph-chunk), the lead-in steps and the K steps are one graph: the start
    event is recorded on a branch that forks off the last lead-in step, so no node
    sits between that step and the first timed step and their launches keep the PDL
    overlap every other pair of consecutive steps has.  Longer runs replay chunks of
    steps, with untimed replays queued ahead of the start event."""
    import torch.distributed as dist
    device = setup.device
    steps = [Step(pa, setup.caches, b, setup.wl, variant, P, device) for b in setup.p.batches]

    def one_step(i, start=None, end=None):
        st = steps[i % len(steps)]
        st.cache_write()
        if start is not None:
            start.record(torch.cuda.current_stream(device))
        st.decode_main()
        if end is not None:
            end.record(torch.cuda.current_stream(device))
        st.decode_tail()

    # eager warm-up (configures the kernels), then chunks of steps captured as graphs;
    # a chunk is a whole number of passes over the input sets, so consecutive steps
    # never reuse a set across a chunk boundary
    for i in range(max(3, len(steps))):
        one_step(i)
    torch.cuda.synchronize()
    chunk = min(K, args.graph_chunk)
    if chunk >= len(steps):
        chunk -= chunk % len(steps)
    tail = K % chunk
    plan = event_plan(K, variant, args.event_every, args.event_run) if kernel_events else None
    every, run = plan if plan else (K, K)

    def capture(n):
        evs = {}
        if plan and n >= run:
            first = 0 if every == run else min(every // 2, n - run)
            evs = {j: (torch.cuda.Event(enable_timing=True, external=True),
                       torch.cuda.Event(enable_timing=True, external=True))
                   for j in range(first, n - run + 1, every)}
        ends = {j + run - 1: e for j, (_, e) in evs.items()}
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for j in range(n):
                one_step(j, evs[j][0] if j in evs else None, ends.get(j))
        return g, evs

    if K <= args.graph_chunk:
        return _time_one_graph(steps, one_step, K, Wm, args, device, plan, every, run)
    # two graphs with their own events alternate, so the host reads one's events
    # while the other replays
    full = [capture(chunk) for _ in range(2 if K > chunk else 1)]
    part = capture(tail) if tail else None
    torch.cuda.synchronize()
    for _ in range(max(1, math.ceil(Wm / chunk))):
        for g, _ in full:
            g.replay()
    if part is not None:
        part[0].replay()
    torch.cuda.synchronize()

    if dist.is_initialized():
        dist.barrier()
    torch.cuda.synchronize()
    kern_ms = []

    def harvest(evs):
        if evs:
            evs[max(evs)][1].synchronize()
            kern_ms.extend(a.elapsed_time(b) / run for a, b in evs.values())

    # untimed replays (at least 64 steps) right before the start event: the GPU is busy
    # again after the barrier's idle time, and the start event waits behind work
    prime = full[-1][0]                            # its events are never read
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    unread = {}
    with ClockSampler(device.index) as clk:
        for _ in range(max(1, math.ceil(args.prime_steps / chunk))):
            prime.replay()
        start.record(stream)
        done, r = 0, 0
        while done < K:
            g, evs = full[r % len(full)] if K - done >= chunk else part
            harvest(unread.pop(id(g), None))     # before this graph re-records its events
            g.replay()
            unread[id(g)] = evs
            done += chunk if K - done >= chunk else tail
            r += 1
        end.record(stream)
        torch.cuda.synchronize()
    for evs in unread.values():
        harvest(evs)
    elapsed_ms = start.elapsed_time(end)
    if kernel_events and plan is None:
        kern_ms.append(elapsed_ms / K)           # K launches back to back, nothing else
    if dist.is_initialized():
        dist.barrier()
    max_ms = max_over_ranks(elapsed_ms, device)
    return {"steps": steps, "max_ms": max_ms, "kern_ms": kern_ms, "chunk": chunk,
            "every": every, "run": run, "region": plan is None, "clocks": clk.summary()}


def _time_one_graph(steps, one_step, K, Wm, args, device, plan, every, run):
    """K <= one graph: lead-in steps, a branch recording the start event after the last
    of them, the K timed steps, the end event (see time_decode)."""
    import torch.distributed as dist
    n_sets = len(steps)
    lead = max(n_sets, math.ceil(max(1, args.prime_steps) / n_sets) * n_sets)
    evs = {}
    if plan and K >= run:
        first = 0 if every == run else min(every // 2, K - run)
        evs = {lead + j: (torch.cuda.Event(enable_timing=True, external=True),
                          torch.cuda.Event(enable_timing=True, external=True))
               for j in range(first, K - run + 1, every)}
    ends = {j + run - 1: e for j, (_, e) in evs.items()}
    start = torch.cuda.Event(enable_timing=True, external=True)
    end = torch.cuda.Event(enable_timing=True, external=True)
    side = torch.cuda.Stream(device)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        main = torch.cuda.current_stream(device)
        for j in range(lead):
            one_step(j)
        fork = torch.cuda.Event()
        fork.record(main)
        side.wait_event(fork)
        start.record(side)                       # off the path of the next launch
        for j in range(lead, lead + K):
            one_step(j, evs[j][0] if j in evs else None, ends.get(j))
        end.record(main)
        main.wait_stream(side)
    torch.cuda.synchronize()
    for _ in range(max(1, math.ceil(Wm / (lead + K)))):
        g.replay()
    torch.cuda.synchronize()
    if dist.is_initialized():
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(device.index) as clk:
        g.replay()
        torch.cuda.synchronize()
    elapsed_ms = start.elapsed_time(end)
    kern_ms = [a.elapsed_time(b) / run for a, b in evs.values()]
    if plan is None:
        kern_ms.append(elapsed_ms / K)           # K launches back to back, nothing else
    if dist.is_initialized():
        dist.barrier()
    max_ms = max_over_ranks(elapsed_ms, device)
    return {"steps": steps, "max_ms": max_ms, "kern_ms": kern_ms, "chunk": lead + K,
            "every": every, "run": run, "region": plan is None, "clocks": clk.summary(),
            "lead": lead}


def roofline_block(setup, variant, t, peak, peak_kind, traffic=None):
    kern_ms = t["kern_ms"]
    if not kern_ms:
        return None
    avg = float(np.mean(kern_ms))
    kb = setup.kernel_bytes(variant)
    achieved = kb / (avg / 1e3) / 1e9
    return {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
            "frac": round(achieved / peak, 4), "traffic": traffic, "peak_source": peak_kind,
            "kernel": DOMINANT_KERNEL[variant],
            "kernel_avg_us": round(avg * 1e3, 3),
            "kernel_median_us": round(float(np.median(kern_ms)) * 1e3, 3),
            "kernel_min_max_us": [round(min(kern_ms) * 1e3, 3), round(max(kern_ms) * 1e3, 3)],
            "kernel_event_samples": len(kern_ms),
            "launches_per_sample": t["run"],
            "bytes_per_launch": kb}


def event_desc(t, variant, on=True):
    if not on:
        return "off"
    if t.get("region"):
        return (f"the timed region's own events: {t['run']} back-to-back launches of the one "
                f"kernel, no event node inside the graphs")
    if t["run"] > 1:
        return f"windows of {t['run']} consecutive launches, one every {t['every']} steps"
    return f"decode timed on every {t['every']}-th step"


def nested_block(pa, args, wl_name, variant, rank, world, device, stream, peak, peak_kind,
                 setup=None, partition_size=0):
    """Another workload measured in the same process, the same way as the headline."""
    setup = setup or DecodeSetup(pa, wl_name, rank, device)
    v, P = setup.resolve(pa, variant, partition_size)
    K, Wm = args.steps, max(3, args.warmup)
    t = time_decode(pa, setup, v, P, K, Wm, args, stream, args.kernel_events)
    gbs = whole_job_rate(setup.bytes_per_step * K, world, t["max_ms"] / 1e3) / 1e9
    wl = setup.wl
    blk = {"workload": workload_desc(wl_name, wl),
           "step": STEP_DECODE[v] if v == "append" else
                   "reshape_and_cache(new token) + " + STEP_DECODE[v].format(P=P),
           "value": round(gbs, 2), "unit": "GB/s", "ms_per_step": t["max_ms"] / K,
           "bytes_per_step": setup.bytes_per_step,
           "pct_of_hbm_peak": round(100.0 * gbs / (world * peak), 2),
           "pct_of_nominal_8tbs": round(100.0 * gbs / (world * NOMINAL_HBM_GBS), 2),
           "seq_heads_per_s": whole_job_rate(wl.num_seqs * wl.num_heads * K, world,
                                             t["max_ms"] / 1e3),
           "gpu_launches": K * t["steps"][0].launches,
           "kernel_events": event_desc(t, v, args.kernel_events),
           "roofline": roofline_block(setup, v, t, peak, peak_kind,
                                      recorded_traffic(wl_name, v)),
           "clocks": t["clocks"]}
    if wl.shared_prefix_tokens:
        blk["unique_kv_gbs"] = round(whole_job_rate(setup.unique_bytes * K, world,
                                                    t["max_ms"] / 1e3) / 1e9, 2)
        blk["unique_pct_of_hbm_peak"] = round(100.0 * blk["unique_kv_gbs"] / (world * peak), 2)
    return blk, setup


def run_ours(args, rank, world, local):
    from paged_kv_cache_390_b200 import build as pa_build
    from paged_kv_cache_390_b200 import pa

    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (the path has no CPU fallback)")
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    pa_build.build()
    pa.lib()
    pa.set_pdl(args.pdl)
    pa.set_prefetch_tiles(args.prefetch)
    pa.set_decode_config(args.warps, args.stages)
    pa.set_cascade_config(args.cascade_splits, args.cascade_suffix)

    wl_name = args.workload
    over = workload_overrides(args, W.WORKLOADS[wl_name])
    setup = DecodeSetup(pa, wl_name, rank, device, over)
    wl, p = setup.wl, setup.p
    args.variant, P = setup.resolve(pa, args.variant, args.partition_size)
    stream = torch.cuda.current_stream(device)
    K, Wm = args.steps, max(3, args.warmup)
    t = time_decode(pa, setup, args.variant, P, K, Wm, args, stream, args.kernel_events)
    steps, max_ms = t["steps"], t["max_ms"]
    ms_per_step = max_ms / K
    gbs = whole_job_rate(setup.bytes_per_step * K, world, max_ms / 1e3) / 1e9
    peak, peak_kind = measured_peaks()

    # the same metric end to end through the public API with host buffers
    e2e = measure_e2e(pa, steps, device, stream, min(K, args.e2e_steps), setup.bytes_per_step)

    res = {
        "metric": METRIC,
        "value": round(gbs, 2),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": K,
        "warmup": Wm,
        "ms_per_step": ms_per_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": wl.cache_dtype if wl.cache_dtype in ("int8", "fp8") else wl.dtype,
        "data": "synthetic (seeded N(0,1) q/K/V, seeded block tables and lengths)",
        "config": {
            "workload": workload_desc(wl_name, wl),
            "step": STEP_DECODE[args.variant] if args.variant == "append" else
                    "reshape_and_cache(new token) + " + STEP_DECODE[args.variant].format(P=P),
            "pool_blocks": int(p.num_blocks),
            "l2": f"{len(steps)} rotating input sets, "
                  f"{len(steps) * setup.decode_bytes / 1e6:.0f} MB of KV in total > 126 MB L2 "
                  f"(no flush kernel)",
            "graph": (f"one CUDA graph: {t['lead']} untimed lead-in steps, then the {K} timed "
                      f"steps; the start event on a branch off the last lead-in step"
                      if "lead" in t else
                      f"CUDA graphs of {t['chunk']} steps; untimed replays (>= "
                      f"{args.prime_steps} steps) queued right ahead of the start event"),
            "kernel_events": event_desc(t, args.variant, args.kernel_events),
            "pdl": {0: "off", 1: "launch overlap", 2: "launch overlap + early table reads"}[args.pdl],
            "parallelism": f"replicas x{world} (independent batches per GPU, no collective)",
        },
        "bytes_per_step": setup.bytes_per_step,
        "pct_of_hbm_peak": round(100.0 * gbs / (world * peak), 2),
        "pct_of_nominal_8tbs": round(100.0 * gbs / (world * NOMINAL_HBM_GBS), 2),
        "seq_heads_per_s": whole_job_rate(wl.num_seqs * wl.num_heads * K, world, max_ms / 1e3),
        "gpu_launches": K * steps[0].launches,
        "e2e": e2e,
    }
    if wl.shared_prefix_tokens:
        res["unique_kv_gbs"] = round(whole_job_rate(setup.unique_bytes * K, world,
                                                    max_ms / 1e3) / 1e9, 2)
        # the shared prefix legitimately comes from L2: the HBM roofline counts it once
        res["unique_pct_of_hbm_peak"] = round(100.0 * res["unique_kv_gbs"] / (world * peak), 2)
    # recorded for the workloads as defined (their own block size)
    roof = roofline_block(setup, args.variant, t, peak, peak_kind,
                          None if over else recorded_traffic(wl_name, args.variant))
    if roof:
        res["roofline"] = roof
    res["clocks"] = t["clocks"]

    # the other configurations, measured the same way in this process (NAME@v2: the
    # split-K form with its workload's partition size; it reuses the pool of a NAME
    # entry just before it)
    if args.also and args.also != "none" and args.path == "decode":
        del steps, t
        extra_launches, prev = 0, None
        for name in [n for n in args.also.split(",") if n and n != wl_name]:
            base_name, _, form = name.partition("@")
            reuse = prev if prev is not None and prev.name == base_name else None
            blk, prev = nested_block(pa, args, base_name, form or "auto", rank, world, device,
                                     stream, peak, peak_kind, setup=reuse)
            res[name.replace("@", "_")] = blk
            extra_launches += blk["gpu_launches"]
        del prev
        torch.cuda.empty_cache()
        res["gpu_launches_with_extra_configs"] = res["gpu_launches"] + extra_launches

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        caches = oracle_caches(p, wl)
        res["cpu_baseline"] = cpu_baseline(p, wl, budget_s=args.cpu_seconds, caches=caches)
        res["cpu_baseline_all_cores"] = cpu_baseline_all_cores(p, wl, budget_s=args.cpu_seconds,
                                                               caches=caches)
    return res


def measure_e2e(pa, steps, device, stream, n, bytes_per_step):
    """The same steps end to end with host buffers.  Per step: one copy of the step's
    inputs (q, new K/V rows, slots, block tables, lengths, packed in one pinned host
    buffer) to the device, the step's kernels, and one copy of out back to pinned host
    memory.  Issued as a serving loop would issue it: host-to-device and
    device-to-host copies run on two more streams into two device buffer sets used in
    turn, so step i+1's inputs and step i-1's output travel while step i computes; the
    loop is captured once into a CUDA graph and replayed.
    The plain eager loop (copies and kernels in one stream) is reported beside it."""
    names = ("q", "nk", "nv", "slots", "tables", "lens")
    width = max(st.tables.shape[1] for st in steps)

    def padded(st, k):
        t = getattr(st, k)
        if k == "tables" and t.shape[1] < width:
            t = torch.nn.functional.pad(t, (0, width - t.shape[1]), value=-1)
        return t

    offs, total = {}, 0
    for k in names:
        t = padded(steps[0], k)
        offs[k] = (total, t.numel() * t.element_size(), t.dtype, tuple(t.shape))
        total += -(-offs[k][1] // 256) * 256
    hosts, outs = [], []
    for st in steps:
        h = torch.empty(total, dtype=torch.uint8).pin_memory()
        for k in names:
            o, nb, _, _ = offs[k]
            h[o:o + nb].copy_(padded(st, k).contiguous().view(-1).view(torch.uint8).cpu())
        hosts.append(h)
        outs.append(torch.empty_like(st.out, device="cpu").pin_memory())
    h2d, d2h = total, outs[0].numel() * outs[0].element_size()

    # two device input buffers, each viewed as one step's tensors
    template = max(steps, key=lambda st: st.maxp)
    pipes = []
    for _ in range(2):
        buf = torch.empty(total, dtype=torch.uint8, device=device)
        st = copy.copy(template)
        for k in names:
            o, nb, dt, shape = offs[k]
            setattr(st, k, buf[o:o + nb].view(dt).view(shape))
        st.out = torch.empty_like(template.out)
        st.buf = buf
        pipes.append(st)
    h2d_stream, d2h_stream = torch.cuda.Stream(device), torch.cuda.Stream(device)

    def pipelined(j, done, cs):
        """Step j of the pipelined loop on compute stream cs.  done[k][b] = events after
        the kernels (k = 0) and the out copy (k = 1) that last used buffer set b."""
        b = j % 2
        st, h, o = pipes[b], hosts[j % len(hosts)], outs[j % len(outs)]
        landed, computed, drained = torch.cuda.Event(), torch.cuda.Event(), torch.cuda.Event()
        with torch.cuda.stream(h2d_stream):
            h2d_stream.wait_event(done[0][b])    # step j-2's kernels are done with buffer b
            st.buf.copy_(h, non_blocking=True)
            landed.record(h2d_stream)
        cs.wait_event(landed)
        cs.wait_event(done[1][b])                # step j-2's out has left buffer b
        st.cache_write()
        st.decode_main()
        st.decode_tail()
        computed.record(cs)
        with torch.cuda.stream(d2h_stream):
            d2h_stream.wait_event(computed)
            o.copy_(st.out, non_blocking=True)
            drained.record(d2h_stream)
        done[0][b], done[1][b] = computed, drained

    def eager(j):
        st, h, o = pipes[0], hosts[j % len(hosts)], outs[j % len(outs)]
        st.buf.copy_(h, non_blocking=True)
        st.cache_write()
        st.decode_main()
        st.decode_tail()
        o.copy_(st.out, non_blocking=True)

    def timed(fn, reps):
        """Device time of `reps` calls; one untimed call is queued first, so the start
        event waits behind work and the host's first submit is not in the figure."""
        torch.cuda.synchronize()
        fn(reps)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for r in range(reps):
            fn(r)
        b.record(stream)
        torch.cuda.synchronize()
        return a.elapsed_time(b)

    for i in range(10):
        eager(i)
    torch.cuda.synchronize()
    eager_ms = timed(eager, n) / n

    m = min(n, 200)
    if m >= len(steps):
        m -= m % len(steps)
    m -= m % 2
    m = max(m, 2)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        cs = torch.cuda.current_stream()
        fork = torch.cuda.Event()
        fork.record(cs)                          # the copy streams join the capture here
        done = [[fork, fork], [fork, fork]]
        for j in range(m):
            pipelined(j, done, cs)
        cs.wait_stream(h2d_stream)               # and rejoin before it ends
        cs.wait_stream(d2h_stream)
    g.replay()
    torch.cuda.synchronize()
    reps = max(1, n // m)
    ms = timed(lambda r: g.replay(), reps) / (reps * m)
    return {"value": round(bytes_per_step / (ms / 1e3) / 1e9, 2), "unit": "GB/s",
            "ms_per_step": ms, "steps": reps * m,
            "issue": f"CUDA graph of {m} steps; inputs and outputs double-buffered, "
                     f"copies on their own streams",
            "eager_value": round(bytes_per_step / (eager_ms / 1e3) / 1e9, 2),
            "eager_ms_per_step": eager_ms,
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h)}


# ----------------------------------------------------------------------------- prefill path

PREFILL_METRIC = "multi-token query (prefix-cached prefill chunk) attention TFLOP/s"


def prefill_flops(lens, qlens, H, D):
    """Attention flops of a causal chunk: each query row at position p touches p + 1
    tokens, 2 * D flops for q.K and 2 * D for p.V, per query head."""
    total = 0
    for n, ql in zip(lens, qlens):
        first = n - ql + 1                       # tokens seen by the chunk's first row
        total += ql * first + ql * (ql - 1) // 2
    return 4.0 * D * H * total


def run_prefill(args, rank, world, local):
    """One step = pa_prefill over a batch of chunks: 8 sequences with 4096 cached
    tokens each compute a 512-token chunk (64 q / 8 kv heads, head_dim 128, bf16 or
    fp16, block 16).  Two input sets with disjoint blocks alternate."""
    from paged_kv_cache_390_b200 import build as pa_build
    from paged_kv_cache_390_b200 import pa

    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    pa_build.build()
    pa.lib()
    pa.set_pdl(1)
    S, ctx, chunk = 8, 4096, 512
    lens = [ctx + chunk] * S
    qlens = [chunk] * S
    dt = args.prefill_dtype
    p = W.make_problem("qwen3_32b_f16", rank_seed(rank), num_batches=2, num_seqs=S,
                       seq_lens=lens, dtype=dt, cache_dtype=dt)
    tdt = torch.bfloat16 if dt == "bf16" else torch.float16
    wl = p.wl
    kc, vc = p.k_cache.to(device), p.v_cache.to(device)
    pa.reshape_and_cache(p.hist_key.to(device), p.hist_value.to(device), kc, vc,
                         p.hist_slots.to(device))
    for b in p.batches:
        pa.reshape_and_cache(b.new_key.to(device), b.new_value.to(device), kc, vc,
                             b.new_slots.to(device))
    gen = torch.Generator().manual_seed(rank_seed(rank) + 7)
    qs = torch.tensor([0] + list(np.cumsum(qlens)), dtype=torch.int32, device=device)
    sets = []
    for b in p.batches:
        q = torch.randn((sum(qlens), wl.num_heads, wl.head_dim), generator=gen).to(tdt).to(device)
        sets.append((q, b.block_tables.to(device), b.seq_lens.to(device), torch.empty_like(q)))

    def step(i):
        q, tb, sl, out = sets[i % len(sets)]
        pa.prefill(q, kc, vc, tb, sl, qs, wl.scale, max_query_len=chunk, out=out)

    K, Wm = args.steps, max(3, args.warmup)
    for i in range(4):
        step(i)
    torch.cuda.synchronize()
    chunk_steps = min(K, 50)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for j in range(chunk_steps):
            step(j)
    for _ in range(max(1, Wm // chunk_steps)):
        g.replay()
    torch.cuda.synchronize()
    reps = max(1, K // chunk_steps)
    stream = torch.cuda.current_stream(device)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        a.record(stream)
        for _ in range(reps):
            g.replay()
        b.record(stream)
        torch.cuda.synchronize()
    ms = max_over_ranks(a.elapsed_time(b), device) / (reps * chunk_steps)
    flops = prefill_flops(lens, qlens, wl.num_heads, wl.head_dim)
    tflops = flops / (ms / 1e3) / 1e12
    peaks = {}
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            peaks = json.load(f)
    except Exception:
        pass
    peak = peaks.get("bf16_tflops", 1590.0)
    return {
        "metric": PREFILL_METRIC, "value": round(tflops * world, 2), "unit": "TFLOP/s",
        "n_gpus": world, "steps": reps * chunk_steps, "warmup": Wm, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": dt,
        "data": "synthetic (seeded N(0,1) q/K/V, seeded block tables)",
        "config": {"workload": f"{S} sequences x ({ctx} cached + {chunk} new) tokens, "
                               f"{wl.num_heads} q / {wl.num_kv_heads} kv heads, head_dim "
                               f"{wl.head_dim}, block {wl.block_size}, {dt}",
                   "step": "pa_prefill (causal chunk over the paged cache, tcgen05)",
                   "graph": f"CUDA graphs of {chunk_steps} steps, 2 alternating input sets"},
        "flops_per_step": flops,
        "gpu_launches": reps * chunk_steps,
        "roofline": {"bound": "tensor", "achieved": round(tflops, 1), "peak": peak,
                     "unit": "TFLOP/s", "frac": round(tflops / peak, 4), "traffic": None,
                     "peak_source": "measured bf16 GEMM (burst)" if "bf16_tflops" in peaks
                     else "fallback"},
        "clocks": clk.summary(),
    }


# ----------------------------------------------------------------------------- oracle arm

def oracle_caches(p, wl):
    """The first input set's caches as the oracle writes them (history, then the step's
    new tokens)."""
    from oracle import oracle as orc
    orc.build()
    kc, vc = p.k_cache.clone(), p.v_cache.clone()
    ks = p.k_scale.clone() if p.k_scale is not None else None
    vs = p.v_scale.clone() if p.v_scale is not None else None
    cd = wl.cache_dtype
    b = p.batches[0]
    orc.reshape_and_cache(p.hist_key, p.hist_value, kc, vc, p.hist_slots, cache_dtype=cd,
                          k_scale=ks, v_scale=vs)
    orc.reshape_and_cache(b.new_key, b.new_value, kc, vc, b.new_slots, cache_dtype=cd,
                          k_scale=ks, v_scale=vs)
    return orc, kc, vc, ks, vs, cd, b


def cpu_baseline(p, wl, budget_s=12.0, sample_seqs=None, caches=None):
    """The oracle (single-threaded C, binary64) on a bounded sample of the workload:
    whole sequences (all heads) of the first input set, as many as fit the budget."""
    orc, kc, vc, ks, vs, cd, b = caches or oracle_caches(p, wl)
    t0 = time.perf_counter()
    done_bytes, done_seqs, i = 0.0, 0, 0
    S = wl.num_seqs
    while time.perf_counter() - t0 < budget_s and (sample_seqs is None or done_seqs < sample_seqs):
        s = i % S
        orc.paged_decode(b.q[s:s + 1], kc, vc, b.block_tables[s:s + 1], b.seq_lens[s:s + 1],
                         wl.scale, cache_dtype=cd, k_scale=ks, v_scale=vs)
        lens = b.seq_lens[s:s + 1].numpy()
        done_bytes += W.logical_kv_bytes(wl, lens) + W.qo_bytes(wl, 1)
        done_seqs += 1
        i += 1
    dt = time.perf_counter() - t0
    return {"value": round(done_bytes / dt / 1e9, 4), "unit": "GB/s", "cores": 1,
            "kind": "oracle",
            "sample": f"{done_seqs} whole sequences (all {wl.num_heads} heads, decode only) of "
                      f"the {wl.name} batch, {dt:.1f} s single-threaded C binary64",
            "seconds": round(dt, 2)}


def cpu_baseline_all_cores(p, wl, budget_s=12.0, threads=None, caches=None):
    """The same oracle on every host core: one thread per core, each decoding whole
    sequences of the first input set in turn (the C call releases the interpreter lock,
    so the threads run in parallel); the caches are shared read-only."""
    import threading
    orc, kc, vc, ks, vs, cd, b = caches or oracle_caches(p, wl)
    T = threads or os.cpu_count() or 1
    S = wl.num_seqs
    done = [[0.0, 0] for _ in range(T)]
    t0 = time.perf_counter()

    def work(k):
        i = k
        while time.perf_counter() - t0 < budget_s:
            s = i % S
            orc.paged_decode(b.q[s:s + 1], kc, vc, b.block_tables[s:s + 1],
                             b.seq_lens[s:s + 1], wl.scale, cache_dtype=cd, k_scale=ks,
                             v_scale=vs)
            done[k][0] += W.logical_kv_bytes(wl, b.seq_lens[s:s + 1].numpy()) + W.qo_bytes(wl, 1)
            done[k][1] += 1
            i += T

    pool = [threading.Thread(target=work, args=(k,)) for k in range(T)]
    for t in pool:
        t.start()
    for t in pool:
        t.join()
    dt = time.perf_counter() - t0
    nbytes, nseq = sum(d[0] for d in done), sum(d[1] for d in done)
    return {"value": round(nbytes / dt / 1e9, 4), "unit": "GB/s", "cores": T, "kind": "oracle",
            "sample": f"{nseq} whole sequences (all {wl.num_heads} heads, decode only) of the "
                      f"{wl.name} batch on {T} threads, {dt:.1f} s of C binary64",
            "seconds": round(dt, 2)}


def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return None
    wl_name = args.workload
    p = W.make_problem(wl_name, rank_seed(0), num_batches=1,
                       **workload_overrides(args, W.WORKLOADS[wl_name]))
    wl = p.wl
    from oracle import oracle as orc
    orc.build()
    kc, vc = p.k_cache.clone(), p.v_cache.clone()
    ks = p.k_scale.clone() if p.k_scale is not None else None
    vs = p.v_scale.clone() if p.v_scale is not None else None
    cd = wl.cache_dtype
    b = p.batch
    orc.reshape_and_cache(p.hist_key, p.hist_value, kc, vc, p.hist_slots, cache_dtype=cd,
                          k_scale=ks, v_scale=vs)

    def step(i):   # bounded sample: the cache write of one sequence's token + its decode
        s = i % wl.num_seqs
        orc.reshape_and_cache(b.new_key[s:s + 1], b.new_value[s:s + 1], kc, vc,
                              b.new_slots[s:s + 1], cache_dtype=cd, k_scale=ks, v_scale=vs)
        orc.paged_decode(b.q[s:s + 1], kc, vc, b.block_tables[s:s + 1], b.seq_lens[s:s + 1],
                         wl.scale, cache_dtype=cd, k_scale=ks, v_scale=vs)
        lens = b.seq_lens[s:s + 1].numpy()
        return W.logical_kv_bytes(wl, lens) + W.qo_bytes(wl, 1)

    K = args.steps
    for i in range(max(3, args.warmup) if args.warmup < 50 else 3):
        step(i)
    t0 = time.perf_counter()
    tot = 0.0
    done = 0
    budget = args.reference_seconds
    for i in range(K):
        tot += step(i)
        done += 1
        if time.perf_counter() - t0 > budget:
            break
    dt = time.perf_counter() - t0
    gbs = tot / dt / 1e9
    sample = (f"{done} steps, each the cache write + decode of ONE sequence (all "
              f"{wl.num_heads} heads) of the {wl_name} batch, single-threaded C binary64")
    return {"impl": "reference", "metric": METRIC, "value": round(gbs, 4), "unit": "GB/s",
            "n_gpus": world, "steps": done, "warmup": args.warmup, "ms_per_step": dt * 1e3 / done,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f64", "data": "synthetic",
            "config": {"workload": workload_desc(wl_name, wl),
                       "sample": "one sequence (the cache write of its new token + its decode) "
                                 "per step"},
            "cpu_baseline": {"value": round(gbs, 4), "unit": "GB/s", "cores": 1,
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": round(gbs, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


# ----------------------------------------------------------------------------- main

def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1,
                    help="ranks (one per GPU); without an outer launcher, N > 1 starts them "
                         "under torch.distributed.run")
    ap.add_argument("--launch-timeout", type=float, default=3600.0,
                    help="seconds after which a self-launched group of ranks is killed")
    ap.add_argument("--steps", type=int, default=40000)
    ap.add_argument("--warmup", type=int, default=400)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--prefill-dtype", choices=["bf16", "f16"], default="bf16")
    ap.add_argument("--path", choices=["decode", "prefill"], default="decode",
                    help="decode: the paged decode step (the default); prefill: the "
                         "multi-token query kernel on its own workload")
    ap.add_argument("--workload", default="qwen3_32b_f16", choices=sorted(W.WORKLOADS))
    ap.add_argument("--num-seqs", type=int, default=0,
                    help="decode path: override the workload's batch size (0 = its own)")
    ap.add_argument("--block-size", type=int, choices=[0, 8, 16, 32], default=0,
                    help="decode path: override the workload's block size (0 = its own)")
    ap.add_argument("--variant", choices=sorted(STEP_DECODE) + ["auto"], default="auto",
                    help="decode entry point; auto = pick_decode_variant: append (v1 with the "
                         "cache write fused in) when one CTA per (sequence, kv head) fills the "
                         "GPU with short sequences, else fused")
    ap.add_argument("--partition-size", type=int, default=0)
    ap.add_argument("--pdl", type=int, choices=[0, 1, 2], default=2,
                    help="programmatic dependent launch mode (pa_set_pdl); 2 lets the decode "
                         "read seq_lens / block_tables while the cache write finishes")
    ap.add_argument("--prefetch", type=int, default=-1,
                    help="KV tiles per decode warp prefetched into L2 before the PDL wait "
                         "(pa_set_prefetch_tiles; -1 = the library default)")
    ap.add_argument("--warps", type=int, default=0,
                    help="decode warps per CTA (pa_set_decode_config; 0 = the library default)")
    ap.add_argument("--stages", type=int, default=0,
                    help="pipeline stages per decode warp (0 = the library default)")
    ap.add_argument("--cascade-splits", type=int, default=0,
                    help="KV splits of the cascade's prefix launch (1..4; 0 = automatic "
                         "placement; -1 = side by side with the suffix whenever it fits)")
    ap.add_argument("--cascade-suffix", type=int, choices=[0, 1], default=0,
                    help="cascade suffix: 0 persistent decode + merge, 1 v1 decode merging "
                         "the prefix partials in its epilogue")
    ap.add_argument("--graph-chunk", type=int, default=400)
    ap.add_argument("--prime-steps", type=int, default=64,
                    help="untimed steps replayed right before the start event (at least one "
                         "graph replay)")
    ap.add_argument("--e2e-steps", type=int, default=2000)
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--reference-seconds", type=float, default=120.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-kernel-events", dest="kernel_events", action="store_false")
    ap.add_argument("--event-every", type=int, default=0,
                    help="time the decode kernel with CUDA events on every n-th step "
                         "(0 = adapt to --steps)")
    ap.add_argument("--event-run", type=int, default=0,
                    help="one-launch steps: consecutive launches bracketed by one event pair "
                         "(0 = adapt to --steps)")
    ap.add_argument("--also", default=DEFAULT_ALSO,
                    help="comma-separated workloads measured after the headline in the same "
                         "run and reported as nested blocks (NAME@v2: the split-K form); "
                         "'none' = none")
    return ap.parse_args(argv)


def free_port() -> int:
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def launch_ranks(n: int, argv, limit_s: float) -> int:
    """`--gpus N` with no launcher around this process: run N ranks of this script
    under torch.distributed.run on this node (one per GPU, rendezvous on 127.0.0.1).
    The ranks run in their own process group, which is killed as a whole if it
    outlives `limit_s` (the ranks' own process-group timeout is far shorter)."""
    import signal
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
           f"--nproc-per-node={n}", "--master-addr", "127.0.0.1",
           "--master-port", str(free_port()), os.path.abspath(__file__), *argv]
    proc = subprocess.Popen(cmd, start_new_session=True)
    try:
        return proc.wait(timeout=limit_s)
    except subprocess.TimeoutExpired:
        os.killpg(proc.pid, signal.SIGTERM)
        try:
            return proc.wait(timeout=60)
        except subprocess.TimeoutExpired:
            os.killpg(proc.pid, signal.SIGKILL)
            return proc.wait()


def main(argv=None):
    raw = list(sys.argv[1:] if argv is None else argv)
    args = parse_args(raw)
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        return launch_ranks(args.gpus, raw, args.launch_timeout)
    if args.impl == "reference":
        res = run_reference(args)
        if res is not None:
            print(json.dumps(res), flush=True)
        return 0
    rank, world, local = dist_env()
    if world > 1:
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    try:
        res = (run_prefill if args.path == "prefill" else run_ours)(args, rank, world, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(res), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
