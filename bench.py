#!/usr/bin/env python3
"""Decode-step benchmark of the paged KV-cache hot path on B200.

One step = one decode iteration of the teaching-model workload: 32 layers,
32 requests with a 4096-token history (growing by one token per step),
H_q 32 / H_kv 8 / d 128, bf16 K/V/Q, block size 16, block tables over a
shuffled pool of 16 GiB + 10 %.  Per step:
  host allocator append (C++; allocate-or-fail) -> block tables mirrored to
  the device (pinned double buffer) -> copy-on-write copies if any -> slot
  mapping -> decode plan -> for each layer: one launch that appends the new
  token's K/V and runs paged decode attention (--unfused: kv_append, then
  attention).

Reported (one JSON line from rank 0):
  value        algorithmic HBM bytes of the step / device step time (GB/s);
               bytes = K/V history read once per KV head + q + out + new
               K/V written + block tables and lengths
  e2e          the same metric with q, new K/V from pinned host buffers and
               the outputs read back to the host inside the timed region
               (per-layer copies on two copy streams, overlapped with the
               other layers' attention)
  roofline     paged decode attention (one partition-kernel launch per layer,
               append and merge folded in): bytes per launch / average launch
               duration, from CUDA events around each step's layer loop in the
               timed region, against the measured HBM peak
  cpu_baseline the float64 oracle on the host cores, on a bounded sample
  clocks       nvidia-smi samples taken during the timed region

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
With N > 1 it runs under torchrun, one rank per GPU, each rank serving its own
32 x 4096 batch (weak scaling; no collective on the data path, only the
barrier and the max-over-ranks of the step time).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np

NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
METRIC = "paged decode-attn achieved HBM GB/s (frac of peak); decode steps/s at 32x4096"


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=100)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--seed", type=int, default=1)
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--cpu-seconds", type=float, default=12.0)
    p.add_argument("--kernel", type=int, default=0, help="0 auto, 1 FMA tiles, 2 tensor-core tiles")
    p.add_argument("--no-extras", action="store_true", help="skip the measurements of the other rows")
    p.add_argument("--extra", default=None,
                   choices=["swap", "allocator", "multi_query", "prefix_cow", "large_serving", "mixed_512",
                            "large_serving_steps", "prefix_cow_steps", "block_size_sweep", "hbm_ceiling"],
                   help="run only this one extra measurement and print its JSON (for profiling captures)")
    p.add_argument("--no-overlap", action="store_true",
                   help="launch every layer's attention without programmatic dependent launch")
    p.add_argument("--unfused", action="store_true",
                   help="append with a separate kv_append launch instead of folding it into attention")
    p.add_argument("--pool-copies", type=int, default=None,
                   help="pool copies the multi_query and prefix_cow extras rotate over (fewer: smaller profiling captures)")
    p.add_argument("--layers", type=int, default=32,
                   help="layers per step (32 for the workload; fewer only for small profiling captures)")
    return p.parse_args()


def read_traffic(key: str):
    """DRAM bytes (read + write) per launch from the committed ncu summary, or None.

    profiles/traffic.txt holds `key value` lines written from one ncu capture of
    the current kernel; it is removed whenever the kernel changes."""
    path = os.path.join(ROOT, "profiles", "traffic.txt")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        for line in f:
            parts = line.split()
            if len(parts) >= 2 and parts[0] == key:
                return float(parts[1])
    return None


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


# -- distributed plumbing -------------------------------------------------------
def dist_init(n):
    if n <= 1:
        return 0, 1, None
    import datetime

    import torch
    import torch.distributed as dist

    rank = int(os.environ["RANK"])
    world = int(os.environ["WORLD_SIZE"])
    local = int(os.environ.get("LOCAL_RANK", rank))
    torch.cuda.set_device(local)
    dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                            device_id=torch.device("cuda", local))
    return rank, world, dist


def _reduce(x: float, dist, op: str, device: str) -> float:
    if dist is None:
        return x
    import torch

    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX if op == "max" else dist.ReduceOp.SUM)
    return float(t.item())


def max_over_ranks(x: float, dist, device: str = "cuda") -> float:
    """The slowest rank's time: a multi-GPU number is timed as the max over ranks."""
    return _reduce(x, dist, "max", device)


def sum_over_ranks(x: float, dist, device: str = "cuda") -> float:
    return _reduce(x, dist, "sum", device)


def shard_requests(num_requests: int, world: int, rank: int) -> range:
    """Requests served by one rank: each rank owns a disjoint, equal block of
    request ids (weak scaling: per-rank work is fixed, the total grows with N).
    Requests are independent, so ranks exchange nothing on the data path."""
    return range(rank * num_requests, (rank + 1) * num_requests)


# -- clocks -----------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_uuid: str):
        self.uuid = device_uuid
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.uuid, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.reader = threading.Thread(target=self._read, daemon=True)
            self.reader.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, smax, power, reasons = [], [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                smax.append(float(parts[1]))
                power.append(float(parts[2]))
            except ValueError:
                continue
            for nm, v in zip(names, parts[4:8]):
                if v.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": float(max(smax)), "samples": len(sm),
                "power_w_max": float(max(power)) if power else None, "reasons": sorted(reasons)}


# -- the workload -------------------------------------------------------------------
class DecodeStep:
    """Multi-layer decode step through the C ABI; all state resident on the device.

    workload: a name of ``workloads.workload`` (its lengths, heads, head_dim,
    block size).  prefix_groups = (groups, branches, prompt): instead of the
    workload's lengths, `groups` prompts of `prompt` tokens are admitted and
    each is forked to `branches` requests that share its blocks (copy-on-write
    of the shared partial tail on the first append).  shared_prefix: attend
    through the shared-prefix call (each group's shared blocks read once per
    layer) after a separate kv_append, instead of the folded append."""

    def __init__(self, steps_budget: int, seed: int, kernel: int, rank: int = 0, world: int = 1,
                 layers: int = 32, fused: bool = True, overlap: bool = True,
                 workload: str = "teaching_32x4096", prefix_groups=None, shared_prefix: bool = False):
        import torch

        import paged_kv_cache_358_b200 as pkv
        import workloads as W

        self.torch, self.pkv = torch, pkv
        self.fused = fused and not shared_prefix
        self.shared_prefix = shared_prefix
        # layers after the first may start while the previous layer's launch
        # finishes (each reads its own pool; the plan, tables and slots were
        # written by kernels that completed before layer 0 started)
        self.overlap = overlap
        pkv.set_decode_kernel(kernel)
        wl = W.workload(workload, decode_steps=steps_budget + 8, seed=seed)
        self.wl = wl
        Hq, Hkv, D, B = wl.num_q_heads, wl.num_kv_heads, wl.head_dim, wl.block_size
        if prefix_groups is not None:
            ng, br, prompt = prefix_groups
            lengths = [prompt] * (ng * br)
            # prompts (full blocks + tail) + per request its copied tail and appends
            N = ng * -(-prompt // B) + ng * br * (-(-(B + steps_budget + 8) // B) + 1)
        else:
            lengths = list(wl.lengths)
            N = wl.pool_blocks
        S, L = len(lengths), layers
        self.S, self.L, self.Hq, self.Hkv, self.D, self.B = S, L, Hq, Hkv, D, B
        self.N = N
        g = W.rng(seed)
        order = W.free_order(g, N)
        self.alloc = pkv.BlockAllocator(N, B, free_order=order)
        self.ids = np.array(list(shard_requests(S, world, rank)), dtype=np.int32)
        if prefix_groups is not None:
            for gi in range(ng):
                root = int(self.ids[gi * br])
                assert self.alloc.add_seq(root, prompt) == 0
                for b in range(1, br):
                    assert self.alloc.fork(root, int(self.ids[gi * br + b])) == 0
            self.group_start = torch.arange(0, S + 1, br, dtype=torch.int32, device="cuda")
            self.prefix_blocks = torch.full((ng,), prompt // B, dtype=torch.int32, device="cuda")
            self.max_group = br
        else:
            for i, n in zip(self.ids, lengths):
                assert self.alloc.add_seq(int(i), n) == 0
        self.max_blocks = -(-(max(lengths) + steps_budget + 8) // B)
        dev = torch.device("cuda")
        gen = torch.Generator(device=dev)
        gen.manual_seed(seed)
        shape = (N, B, Hkv, D)
        self.k_pools, self.v_pools = [], []
        for _ in range(L):
            self.k_pools.append(torch.randn(shape, generator=gen, device=dev, dtype=torch.bfloat16))
            self.v_pools.append(torch.randn(shape, generator=gen, device=dev, dtype=torch.bfloat16))
        # a step's inputs, per layer one packed row [q | k_new | v_new], and its
        # outputs are each one contiguous buffer, two of each: the end-to-end
        # pass moves a step's inputs with one host->device copy and its outputs
        # with one device->host copy, while the neighbouring step computes
        nq, nkv = S * Hq * D, S * Hkv * D
        self.in_d = torch.randn((2, L, nq + 2 * nkv), generator=gen, device=dev, dtype=torch.bfloat16)
        self.q = [[self.in_d[b, i, :nq].view(S, Hq, D) for i in range(L)] for b in range(2)]
        self.k_new = [[self.in_d[b, i, nq:nq + nkv].view(S, Hkv, D) for i in range(L)] for b in range(2)]
        self.v_new = [[self.in_d[b, i, nq + nkv:].view(S, Hkv, D) for i in range(L)] for b in range(2)]
        self.out_d = torch.empty((2, L, S, Hq, D), device=dev, dtype=torch.bfloat16)
        self.out = [[self.out_d[b, i] for i in range(L)] for b in range(2)]
        self.status = np.zeros(S, dtype=np.int32)
        self.copies_h = np.zeros((S, 3), dtype=np.int32)
        # pinned double buffers for the tables and lengths mirrored each step
        self.tab_h = [torch.empty((S, self.max_blocks), dtype=torch.int32).pin_memory() for _ in range(2)]
        self.len_h = [torch.empty((S,), dtype=torch.int32).pin_memory() for _ in range(2)]
        self.pos_h = [torch.empty((S,), dtype=torch.int32).pin_memory() for _ in range(2)]
        self.cp_h = [torch.empty((S, 3), dtype=torch.int32).pin_memory() for _ in range(2)]
        self.h2d_done = [None, None]
        self.tab_d = torch.empty((S, self.max_blocks), dtype=torch.int32, device=dev)
        self.len_d = torch.empty((S,), dtype=torch.int32, device=dev)
        self.pos_d = torch.empty((S,), dtype=torch.int32, device=dev)
        self.cp_d = torch.empty((S, 3), dtype=torch.int32, device=dev)
        self.slots = torch.empty((S,), dtype=torch.int64, device=dev)
        self.ws = pkv.new_workspace(S, Hq, Hkv, D)
        if shared_prefix:
            self.wsp = pkv.shared_prefix_workspace(S, len(self.prefix_blocks), self.max_group, Hq, Hkv, D,
                                                   self.max_blocks)
        self.stream = torch.cuda.current_stream()
        self.parity = 0
        self.launches = 0
        self.bytes_done = 0
        self.attn_bytes = []
        self.attn_events = []
        self.record_attn = False
        self.step_events = None    # when a list: one event recorded at the end of each step
        # e2e host buffers and copy streams: step k's inputs go up on one stream
        # (while step k-1 computes) and its outputs come back on another (while
        # step k+1 computes); events order every copy against the kernels
        self.in_h = self.in_d[0].cpu().pin_memory()
        self.out_h = torch.empty((2, L, S, Hq, D), dtype=torch.bfloat16).pin_memory()
        self.up = torch.cuda.Stream()
        self.down = torch.cuda.Stream()
        self.e2e_k = 0
        self.in_ready = [None, None]    # per buffer: inputs of its current step on the device
        self.tables_copied = None       # the last step's table copies are done
        self.step_done = [None, None]   # per buffer: its step's kernels finished
        self.out_back = [None, None]    # per buffer: its step's outputs on the host
        # the last step's readback, not issued yet: it goes out behind the next
        # step's small table copies, so those never wait for it on a copy engine
        self.pending_readback = None

    def bytes_of_step(self, lens: np.ndarray, copied_rows: int) -> int:
        """Algorithmic bytes: every history slot read once per KV head, q, out, appends,
        metadata, and the copy-on-write copies (`copied_rows` = the sum of n_valid
        over the step's copies: only the valid slots of a shared tail are copied)."""
        e = 2
        kv = int(lens.sum()) * self.Hkv * self.D * e * 2
        qo = self.S * self.Hq * self.D * e * 2
        app = self.S * self.Hkv * self.D * e * 2 * 2
        meta = 4 * int(sum(-(-int(n) // self.B) for n in lens)) + 4 * self.S
        cow = copied_rows * self.Hkv * self.D * e * 2 * 2
        return self.L * (kv + qo + app + meta) + self.L * cow + 8 * self.S

    def attn_bytes_per_launch(self, lens: np.ndarray) -> int:
        """History K/V read once per KV head, q read, out written, table + length; with the
        append folded in, also the new K/V rows read and written."""
        e = 2
        b = (int(lens.sum()) * self.Hkv * self.D * e * 2 + self.S * self.Hq * self.D * e * 2
             + 4 * int(sum(-(-int(n) // self.B) for n in lens)) + 4 * self.S)
        if self.fused:
            b += self.S * self.Hkv * self.D * e * 2 * 2 + 8 * self.S
        return b

    def step(self, e2e: bool = False):
        torch, pkv = self.torch, self.pkv
        rc, nc = self.alloc.append_arrays(self.ids, self.status, self.copies_h)
        if rc != 0:
            raise RuntimeError(f"allocator refused a step: {rc}")
        b = self.parity
        self.parity ^= 1
        if self.h2d_done[b] is not None:
            self.h2d_done[b].synchronize()
        tab, lens = self.alloc.fill_tables(self.ids, self.max_blocks, 0, self.tab_h[b].numpy(),
                                           self.len_h[b].numpy())
        np.subtract(lens, 1, out=self.pos_h[b].numpy())
        self.tab_d.copy_(self.tab_h[b], non_blocking=True)
        self.len_d.copy_(self.len_h[b], non_blocking=True)
        self.pos_d.copy_(self.pos_h[b], non_blocking=True)
        if nc:
            self.cp_h[b].numpy()[:nc] = self.copies_h[:nc]
            self.cp_d[:nc].copy_(self.cp_h[b][:nc], non_blocking=True)
        ev = torch.cuda.Event()
        ev.record(self.stream)
        self.h2d_done[b] = ev
        tables_copied_prev = self.tables_copied
        self.tables_copied = ev
        if self.pending_readback is not None:
            self.read_back(*self.pending_readback, after=ev)
        if nc:
            pkv.block_copy(self.k_pools, self.v_pools, self.cp_d[:nc])
            self.launches += 1
        pkv.slot_mapping(self.tab_d, self.pos_d, self.B, out=self.slots)
        self.launches += 1
        if not self.shared_prefix:      # the shared-prefix call plans inside each layer's call
            pkv.decode_plan(self.len_d, self.Hq, self.Hkv, self.D, pkv.BF16, self.ws)
            self.launches += 1
        eb = 0
        if e2e:
            eb = self.e2e_k % 2
            self.e2e_k += 1
            # upload this step's inputs once the step that last used the buffer is
            # done, and after the previous step's small table copies, so those
            # never queue behind this upload on the copy engine
            if self.step_done[eb] is not None:
                self.up.wait_event(self.step_done[eb])
            if tables_copied_prev is not None:
                self.up.wait_event(tables_copied_prev)
            with torch.cuda.stream(self.up):
                self.in_d[eb].copy_(self.in_h, non_blocking=True)
            self.in_ready[eb] = torch.cuda.Event()
            self.in_ready[eb].record(self.up)
            self.stream.wait_event(self.in_ready[eb])
            if self.out_back[eb] is not None:   # the outputs last written here are on the host
                self.stream.wait_event(self.out_back[eb])
        if self.record_attn:
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(self.stream)
        q, k_new, v_new, out = self.q[eb], self.k_new[eb], self.v_new[eb], self.out[eb]
        for i in range(self.L):
            if not self.fused:
                pkv.kv_append(k_new[i], v_new[i], self.slots, self.k_pools[i], self.v_pools[i])
                self.launches += 1
            if self.shared_prefix:
                # preparation (gather + both plans), two attention passes and
                # the combine (which merges the shared pass's split pieces):
                # four kernels (and a memset)
                pkv.paged_decode_attn_shared_prefix(q[i], self.k_pools[i], self.v_pools[i], self.tab_d,
                                                    self.len_d, self.group_start, self.prefix_blocks,
                                                    self.max_group, self.wl.scale, out=out[i],
                                                    workspace=self.wsp)
                self.launches += 4
                continue
            pkv.set_launch_overlap(self.overlap and i > 0 and self.fused)
            if self.fused:
                pkv.paged_decode_attn_append_run(q[i], k_new[i], v_new[i], self.slots,
                                                 self.k_pools[i], self.v_pools[i], self.tab_d, self.len_d,
                                                 self.wl.scale, out[i], self.ws)
            else:
                pkv.paged_decode_attn_run(q[i], self.k_pools[i], self.v_pools[i], self.tab_d, self.len_d,
                                          self.wl.scale, out[i], self.ws)
            self.launches += 1
        pkv.set_launch_overlap(False)
        if e2e:
            done = torch.cuda.Event()
            done.record(self.stream)
            self.step_done[eb] = done
            self.pending_readback = (eb, done)
        if self.record_attn:
            e1.record(self.stream)
            self.attn_events.append((e0, e1))
            self.attn_bytes.append(self.attn_bytes_per_launch(lens))
        self.bytes_done += self.bytes_of_step(lens, int(self.copies_h[:nc, 2].sum()) if nc else 0)
        if self.step_events is not None:
            ev = torch.cuda.Event(enable_timing=True)
            ev.record(self.stream)
            self.step_events.append(ev)

    def read_back(self, eb: int, done, after=None):
        """Copy buffer eb's outputs to the host on the download stream, once
        their step's kernels are done (and, given `after`, once the next
        step's table copies are: a readback that starts with them delayed
        them by up to its own 0.17 ms on the copy engines)."""
        torch = self.torch
        self.down.wait_event(done)
        if after is not None:
            self.down.wait_event(after)
        with torch.cuda.stream(self.down):
            self.out_h[eb].copy_(self.out_d[eb], non_blocking=True)
        self.out_back[eb] = torch.cuda.Event()
        self.out_back[eb].record(self.down)
        self.pending_readback = None

    def drain(self):
        """Issue the last step's readback and order the compute stream after
        the outputs' copies to the host."""
        if self.pending_readback is not None:
            self.read_back(*self.pending_readback)
        for ev in self.out_back:
            if ev is not None:
                self.stream.wait_event(ev)

    def h2d_d2h_bytes(self):
        e = 2
        per_layer_in = self.S * self.Hq * self.D * e + 2 * self.S * self.Hkv * self.D * e
        meta = self.S * self.max_blocks * 4 + self.S * 4
        return self.L * per_layer_in + meta, self.L * self.S * self.Hq * self.D * e


def timed(fn, steps, dist, stream, finish=None, start=None):
    import torch

    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    w0 = time.perf_counter()
    e0.record(stream)
    if start is not None:
        start()
    for _ in range(steps):
        fn()
    if finish is not None:
        finish()
    e1.record(stream)
    torch.cuda.synchronize()
    wall = time.perf_counter() - w0
    if dist is not None:
        dist.barrier()
    ms = e0.elapsed_time(e1)
    return ms, wall


def step_stats(step_ms) -> dict:
    """Median, 10th and 90th percentile and mean of per-step device times (ms),
    from one CUDA event recorded at the end of every timed step."""
    x = np.asarray(step_ms, dtype=np.float64)
    return {"median": float(np.median(x)), "p10": float(np.percentile(x, 10)),
            "p90": float(np.percentile(x, 90)), "mean": float(x.mean()), "n": int(x.size)}


# -- CPU oracle baseline -----------------------------------------------------------
def _blas_threads():
    try:
        from threadpoolctl import threadpool_info

        return max([d.get("num_threads", 1) for d in threadpool_info()] + [1])
    except Exception:
        return 1


def cpu_baseline(seconds: float):
    """The float64 oracle, as it stands, on a bounded sample of the same workload.

    The 32 request histories (4096 tokens) are drawn once; layer after layer,
    a fresh q is drawn and each request is attended one at a time until
    `seconds` of oracle compute have been spent.  Input generation is not
    timed.
    """
    import workloads as W
    from oracle import attention as oatt

    wl = W.workload("teaching_32x4096")
    g = W.rng(123)
    hist = [(W.normal_bf16_bits(g, (n, wl.num_kv_heads, wl.head_dim)),
             W.normal_bf16_bits(g, (n, wl.num_kv_heads, wl.head_dim))) for n in wl.lengths]
    compute, done_bytes, n_att, layers = 0.0, 0, 0, 0
    while compute < seconds and layers < wl.layers:
        for s, n in enumerate(wl.lengths):
            q = W.normal_bf16_bits(g, (wl.num_q_heads, wl.head_dim))
            t1 = time.perf_counter()
            oatt.dense_decode(q, hist[s][0], hist[s][1], wl.scale)
            compute += time.perf_counter() - t1
            done_bytes += n * wl.num_kv_heads * wl.head_dim * 2 * 2 + 2 * wl.num_q_heads * wl.head_dim * 2
            n_att += 1
            if compute >= seconds:
                break
        layers += 1
    # the two small batches, whole (one layer each)
    others = {}
    for name in ("tiny", "mixed_512"):
        wo = W.workload(name)
        go = W.rng(wo.seed + 100)
        tot = 0.0
        nbytes = 0
        for n in wo.lengths:
            kh, vh = W.kv_history(go, wo, n), W.kv_history(go, wo, n)
            q = (W.normal_bf16_bits if wo.dtype == "bf16" else W.normal_f32)(go, (wo.num_q_heads, wo.head_dim))
            t1 = time.perf_counter()
            oatt.dense_decode(q, kh, vh, wo.scale)
            tot += time.perf_counter() - t1
            es = 2 if wo.dtype == "bf16" else 4
            nbytes += n * wo.num_kv_heads * wo.head_dim * es * 2 + 2 * wo.num_q_heads * wo.head_dim * es
        others[name] = {"seconds": tot, "gb_per_s": nbytes / tot / 1e9, "requests": len(wo.lengths)}
    return {"value": done_bytes / compute / 1e9, "unit": "GB/s", "cores": _blas_threads(),
            "host_cpus": os.cpu_count(), "kind": "oracle",
            "sample": f"float64 NumPy dense decode attention of {n_att} (request, layer) pairs of the "
                      f"32 requests x 4096 history (H_q 32, H_kv 8, d 128; histories drawn once and "
                      f"reused across {layers} layers, fresh q per layer); {compute:.1f} s of CPU work, "
                      f"input generation not timed",
            "other_batches_one_layer": others}


def swap_measurement():
    """Preemption by swap: move 500 MiB of KV (250 blocks of the teaching model,
    32 layers, K and V) to pinned host memory and back; the pages estimate
    19.5 ms one way at 25 GiB/s."""
    import torch

    import paged_kv_cache_358_b200 as pkv

    L, B, Hkv, D, nblk = 32, 16, 8, 128, 250
    kp = [torch.zeros((nblk + 4, B, Hkv, D), dtype=torch.bfloat16, device="cuda") for _ in range(L)]
    vp = [torch.zeros_like(kp[0]) for _ in range(L)]
    blocks = torch.arange(nblk, dtype=torch.int32, device="cuda")
    host = torch.empty(nblk * L * 2 * B * Hkv * D, dtype=torch.bfloat16).pin_memory()
    res = {"mib": host.numel() * 2 / 2**20, "pages_one_way_ms_at_25_gib_per_s": 19.5}
    for name, to_host in (("out", True), ("in", False)):
        pkv.swap_blocks(kp, vp, blocks, host, to_host=to_host)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        pkv.swap_blocks(kp, vp, blocks, host, to_host=to_host)
        e1.record()
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1)
        res[f"{name}_ms"] = ms
        res[f"{name}_gib_per_s"] = res["mib"] / 1024 / (ms / 1000)
    del kp, vp, host
    return res


def multi_query_measurement(reps: int = 20, copies: int = 12):
    """Multi-token query (T tokens per request, causal) on one layer of the
    32 x 4096 teaching shapes: microseconds per call (plan + attention) and
    algorithmic GB/s (history K/V once per KV head, q and out of all T tokens,
    tables), for T = 1, 2, 4.  Pools hold 12 layers' worth of blocks and the
    calls rotate over them, so every call streams from HBM."""
    import torch

    import paged_kv_cache_358_b200 as pkv
    import workloads as W

    wl = W.workload("teaching_32x4096", decode_steps=16)
    S, Hq, Hkv, D, B, N = wl.num_seqs, wl.num_q_heads, wl.num_kv_heads, wl.head_dim, wl.block_size, wl.pool_blocks
    a = pkv.BlockAllocator(N, B, free_order=W.free_order(W.rng(5), N))
    for i, n in enumerate(wl.lengths):
        assert a.add_seq(i, n) == 0
    tables, lens = a.fill_tables(list(range(S)), -(-max(wl.lengths) // B))
    td, ld = torch.from_numpy(tables).cuda(), torch.from_numpy(lens).cuda()
    gen = torch.Generator(device="cuda")
    gen.manual_seed(5)
    kp = [torch.randn((N, B, Hkv, D), generator=gen, device="cuda", dtype=torch.bfloat16) for _ in range(copies)]
    vp = [torch.randn((N, B, Hkv, D), generator=gen, device="cuda", dtype=torch.bfloat16) for _ in range(copies)]
    res = {}
    for T in (1, 2, 4):
        q = torch.randn((S, T, Hq, D), generator=gen, device="cuda", dtype=torch.bfloat16)
        out = torch.empty_like(q)
        ws = torch.zeros(pkv.lib().pkv_multi_query_workspace_bytes(S, T, Hq, Hkv, D), dtype=torch.uint8,
                         device="cuda")
        for i in range(3):
            pkv.paged_attn_multi_query(q, kp[i % copies], vp[i % copies], td, ld, wl.scale, out=out, workspace=ws)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for i in range(reps):
            pkv.paged_attn_multi_query(q, kp[i % copies], vp[i % copies], td, ld, wl.scale, out=out, workspace=ws)
        e1.record()
        torch.cuda.synchronize()
        us = e0.elapsed_time(e1) * 1000 / reps
        nbytes = (int(lens.sum()) * Hkv * D * 2 * 2 + 2 * S * T * Hq * D * 2
                  + 4 * int(sum(-(-int(n) // B) for n in lens)) + 4 * S)
        res[f"T{T}"] = {"us_per_call": us, "gb_per_s": nbytes / (us * 1e-6) / 1e9,
                        "columns_per_kv_head": T * Hq // Hkv}
    del kp, vp
    return res


def _time_decode(pkv, torch, q, pools, tables, lens, scale, ws, reps):
    """Average microseconds of one paged_decode_attn call (plan + attention),
    rotating over the pool copies so every call streams from HBM."""
    for i in range(2):
        pkv.paged_decode_attn(q, pools[i][0], pools[i][1], tables, lens, scale, workspace=ws)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for i in range(reps):
        kp, vp = pools[i % len(pools)]
        pkv.paged_decode_attn(q, kp, vp, tables, lens, scale, workspace=ws)
    e1.record()
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) * 1000 / reps


def prefix_cow_measurement(reps: int = 20, copies: int = 8):
    """Shared prompts: 64 groups x 4 branches fork one 2008-token prompt (full
    blocks shared, the 8-token tail copied on the first append) and append 256
    tokens each; one layer (H_q 16, H_kv 4, d 128, bf16, B 16).  Reports the
    logical KV GB/s (every request's whole history counted) and the unique
    GB/s (each physical block counted once): shared blocks may be served from
    L2 for the later branches of a group."""
    import torch

    import paged_kv_cache_358_b200 as pkv
    import workloads as W

    wl = W.workload("prefix_cow")
    G, BR, P, A = 64, 4, 2008, 256
    S, Hq, Hkv, D, B, N = G * BR, wl.num_q_heads, wl.num_kv_heads, wl.head_dim, wl.block_size, wl.pool_blocks
    a = pkv.BlockAllocator(N, B, free_order=W.free_order(W.rng(wl.seed), N))
    ids = []
    for g in range(G):
        root = g * BR
        assert a.add_seq(root, P) == 0
        for b in range(1, BR):
            assert a.fork(root, root + b) == 0
        ids += list(range(root, root + BR))
    ids = np.array(ids, dtype=np.int32)
    st = np.zeros(S, dtype=np.int32)
    cp = np.zeros((S, 3), dtype=np.int32)
    copies = 0
    for _ in range(A):
        rc, nc = a.append_arrays(ids, st, cp)
        assert rc == 0
        copies += nc
    tables, lens = a.fill_tables(list(ids), -(-(P + A) // B))
    unique_blocks = a.stats()["active"]
    td, ld = torch.from_numpy(tables).cuda(), torch.from_numpy(lens).cuda()
    gen = torch.Generator(device="cuda")
    gen.manual_seed(7)
    pools = [(torch.randn((N, B, Hkv, D), generator=gen, device="cuda", dtype=torch.bfloat16),
              torch.randn((N, B, Hkv, D), generator=gen, device="cuda", dtype=torch.bfloat16)) for _ in range(copies)]
    q = torch.randn((S, Hq, D), generator=gen, device="cuda", dtype=torch.bfloat16)
    ws = pkv.new_workspace(S, Hq, Hkv, D)
    us = _time_decode(pkv, torch, q, pools, td, ld, wl.scale, ws, reps)
    # the same batch through the shared-prefix call: each group's 125 full
    # prompt blocks are read once for its 4 branches
    gs = torch.arange(0, S + 1, BR, dtype=torch.int32, device="cuda")
    pb = torch.full((G,), P // B, dtype=torch.int32, device="cuda")
    wsp = pkv.shared_prefix_workspace(S, G, BR, Hq, Hkv, D, tables.shape[1])
    out = torch.empty((S, Hq, D), dtype=torch.bfloat16, device="cuda")

    def shared(i):
        kp, vp = pools[i % len(pools)]
        pkv.paged_decode_attn_shared_prefix(q, kp, vp, td, ld, gs, pb, BR, wl.scale, out=out, workspace=wsp)

    for i in range(2):
        shared(i)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for i in range(reps):
        shared(i)
    e1.record()
    torch.cuda.synchronize()
    us_shared = e0.elapsed_time(e1) * 1000 / reps
    assert pkv.decode_status(wsp) == 0
    row = Hkv * D * 2 * 2
    logical = int(lens.sum()) * row + 2 * S * Hq * D * 2
    unique = unique_blocks * B * row + 2 * S * Hq * D * 2
    del pools
    return {"us_per_layer": us, "logical_gb_per_s": logical / (us * 1e-6) / 1e9,
            "unique_gb_per_s": unique / (us * 1e-6) / 1e9, "cow_copies": copies,
            "logical_mb": logical / 1e6, "unique_mb": unique / 1e6,
            "shared_prefix_call": {"us_per_layer": us_shared,
                                   "logical_gb_per_s": logical / (us_shared * 1e-6) / 1e9,
                                   "unique_gb_per_s": unique / (us_shared * 1e-6) / 1e9}}


def large_serving_measurement(reps: int = 12):
    """256 requests with lengths uniform in 1..8192, H_q 32, H_kv 4 (G = 8),
    d 128, bf16, B 16, shuffled tables; one layer per call."""
    import torch

    import paged_kv_cache_358_b200 as pkv
    import workloads as W

    wl = W.workload("large_serving")
    S, Hq, Hkv, D, B, N = wl.num_seqs, wl.num_q_heads, wl.num_kv_heads, wl.head_dim, wl.block_size, wl.pool_blocks
    a = pkv.BlockAllocator(N, B, free_order=W.free_order(W.rng(wl.seed), N))
    for i, n in enumerate(wl.lengths):
        assert a.add_seq(i, n) == 0
    tables, lens = a.fill_tables(list(range(S)), -(-max(wl.lengths) // B))
    td, ld = torch.from_numpy(tables).cuda(), torch.from_numpy(lens).cuda()
    gen = torch.Generator(device="cuda")
    gen.manual_seed(9)
    pools = [(torch.randn((N, B, Hkv, D), generator=gen, device="cuda", dtype=torch.bfloat16),
              torch.randn((N, B, Hkv, D), generator=gen, device="cuda", dtype=torch.bfloat16)) for _ in range(3)]
    q = torch.randn((S, Hq, D), generator=gen, device="cuda", dtype=torch.bfloat16)
    ws = pkv.new_workspace(S, Hq, Hkv, D)
    us = _time_decode(pkv, torch, q, pools, td, ld, wl.scale, ws, reps)
    nbytes = (int(lens.sum()) * Hkv * D * 2 * 2 + 2 * S * Hq * D * 2
              + 4 * int(sum(-(-int(n) // B) for n in lens)) + 4 * S)
    del pools
    return {"us_per_layer": us, "gb_per_s": nbytes / (us * 1e-6) / 1e9, "kv_tokens": int(lens.sum())}


def mixed_512_measurement(reps: int = 20):
    """512 requests with lengths uniform in 1..512 (H_q 32, H_kv 8, d 128,
    bf16, B 16): one layer of short ragged histories per call."""
    import torch

    import paged_kv_cache_358_b200 as pkv
    import workloads as W

    wl = W.workload("mixed_512", block_size=16)
    S, Hq, Hkv, D, B, N = wl.num_seqs, wl.num_q_heads, wl.num_kv_heads, wl.head_dim, wl.block_size, wl.pool_blocks
    a = pkv.BlockAllocator(N, B, free_order=W.free_order(W.rng(wl.seed), N))
    for i, n in enumerate(wl.lengths):
        assert a.add_seq(i, n) == 0
    tables, lens = a.fill_tables(list(range(S)), -(-max(wl.lengths) // B))
    td, ld = torch.from_numpy(tables).cuda(), torch.from_numpy(lens).cuda()
    gen = torch.Generator(device="cuda")
    gen.manual_seed(11)
    pools = [(torch.randn((N, B, Hkv, D), generator=gen, device="cuda", dtype=torch.bfloat16),
              torch.randn((N, B, Hkv, D), generator=gen, device="cuda", dtype=torch.bfloat16)) for _ in range(4)]
    q = torch.randn((S, Hq, D), generator=gen, device="cuda", dtype=torch.bfloat16)
    ws = pkv.new_workspace(S, Hq, Hkv, D)
    us = _time_decode(pkv, torch, q, pools, td, ld, wl.scale, ws, reps)
    nbytes = (int(lens.sum()) * Hkv * D * 2 * 2 + 2 * S * Hq * D * 2
              + 4 * int(sum(-(-int(n) // B) for n in lens)) + 4 * S)
    del pools
    return {"us_per_layer": us, "gb_per_s": nbytes / (us * 1e-6) / 1e9, "kv_tokens": int(lens.sum())}


def serving_steps_measurement(kind: str, steps: int, layers: int = 24, shared_prefix: bool = False):
    """Whole decode steps of a serving batch, timed with one CUDA event per step.

    kind "large_serving": 256 requests, lengths U(1..8192), H_q 32 / H_kv 4
    (G = 8), d 128, bf16, B 16, 24 layers; every step appends one token per
    request (allocator, table mirror, slot mapping, plan, then one launch per
    layer with the append folded in).
    kind "prefix_cow": 64 prompts of 2008 tokens, each forked to 4 branches
    (H_q 16 / H_kv 4, d 128, bf16, B 16, 24 layers); the timed steps start at
    the first append, so the copy-on-write of every shared 8-token tail (3 per
    group, in all 24 layers) is inside the timed region.  With shared_prefix
    each layer runs kv_append and the shared-prefix call (each group's 125
    shared blocks read once) instead of the folded append.
    Reports ms per step (median and mean), steps/s, tokens/s and the
    algorithmic GB/s of the step (every request's history counted: logical);
    for prefix_cow also GB/s of the unique blocks of the pool."""
    import torch

    if kind == "prefix_cow":
        ds = DecodeStep(steps + 8, 3, 0, layers=layers, workload="prefix_cow", prefix_groups=(64, 4, 2008),
                        shared_prefix=shared_prefix)
        warm = 0        # the first append (copy-on-write) is timed; the kernels are warm already
    else:
        ds = DecodeStep(steps + 8, 4, 0, layers=layers, workload="large_serving")
        warm = 3
    for _ in range(warm):
        ds.step()
    torch.cuda.synchronize()
    ds.bytes_done = 0
    copies0 = ds.alloc.stats()["cow_copies"]
    start_ev = torch.cuda.Event(enable_timing=True)
    ds.step_events = []
    ms, _ = timed(ds.step, steps, None, ds.stream, start=lambda: start_ev.record(ds.stream))
    marks = [start_ev] + ds.step_events
    step_ms = np.array([a.elapsed_time(b) for a, b in zip(marks[:-1], marks[1:])])
    assert ds.pkv.decode_status(ds.wsp if shared_prefix else ds.ws) == 0
    st = ds.alloc.stats()
    res = {"layers": layers, "requests": ds.S, "steps": steps, "ms_per_step": ms / steps,
           "step_ms": step_stats(step_ms), "steps_per_s": steps / (ms / 1000),
           "tokens_per_s": steps * ds.S / (ms / 1000), "gb_per_s": ds.bytes_done / (ms / 1000) / 1e9,
           "kv_tokens_end": int(sum(ds.alloc.length(int(i)) for i in ds.ids)),
           "cow_copies": int(st["cow_copies"] - copies0)}
    if kind == "prefix_cow":
        # unique bytes: each physical block of the pool read once per layer (upper bound: whole blocks)
        row = ds.Hkv * ds.D * 2 * 2
        res["unique_blocks_end"] = int(st["active"])
        res["unique_gb_per_s_upper"] = (steps * layers * st["active"] * ds.B * row) / (ms / 1000) / 1e9
    del ds
    torch.cuda.empty_cache()
    return res


def block_size_sweep_measurement(reps: int = 20):
    """The 512 short ragged requests (lengths U{1..512}, H_q 32 / H_kv 8, d 128,
    bf16) at block sizes 4, 8, 16, 32, 64: microseconds per layer (plan +
    attention), algorithmic GB/s, and the mean tail waste (slots allocated
    past the length, B * ceil(n / B) - n) beside its expectation (B - 1) / 2."""
    import torch

    import paged_kv_cache_358_b200 as pkv
    import workloads as W

    res = {}
    for B in (4, 8, 16, 32, 64):
        wl = W.workload("mixed_512", block_size=B)
        S, Hq, Hkv, D, N = wl.num_seqs, wl.num_q_heads, wl.num_kv_heads, wl.head_dim, wl.pool_blocks
        a = pkv.BlockAllocator(N, B, free_order=W.free_order(W.rng(wl.seed), N))
        for i, n in enumerate(wl.lengths):
            assert a.add_seq(i, n) == 0
        tables, lens = a.fill_tables(list(range(S)), -(-max(wl.lengths) // B))
        td, ld = torch.from_numpy(tables).cuda(), torch.from_numpy(lens).cuda()
        gen = torch.Generator(device="cuda")
        gen.manual_seed(11 + B)
        pools = [(torch.randn((N, B, Hkv, D), generator=gen, device="cuda", dtype=torch.bfloat16),
                  torch.randn((N, B, Hkv, D), generator=gen, device="cuda", dtype=torch.bfloat16))
                 for _ in range(4)]
        q = torch.randn((S, Hq, D), generator=gen, device="cuda", dtype=torch.bfloat16)
        ws = pkv.new_workspace(S, Hq, Hkv, D)
        us = _time_decode(pkv, torch, q, pools, td, ld, wl.scale, ws, reps)
        nbytes = (int(lens.sum()) * Hkv * D * 2 * 2 + 2 * S * Hq * D * 2
                  + 4 * int(sum(-(-int(n) // B) for n in lens)) + 4 * S)
        waste = [B * -(-int(n) // B) - int(n) for n in lens]
        res[f"B{B}"] = {"us_per_layer": us, "gb_per_s": nbytes / (us * 1e-6) / 1e9,
                        "mean_tail_waste_slots": float(np.mean(waste)), "expected_waste": (B - 1) / 2,
                        "blocks": int(sum(-(-int(n) // B) for n in lens))}
        del pools
    return res


def hbm_ceiling_measurement(reps: int = 10):
    """Context for the roofline: what plain library kernels stream on this GPU.
    A read-only reduction (torch amax over 4 GiB of int32) and a copy (2 GiB
    read + 2 GiB written), each timed with CUDA events over `reps` calls, in
    GB/s of bytes moved.  The decode kernel only reads (its writes are < 1 %),
    so the read-only figure is its practical ceiling."""
    import torch

    n = (4 << 30) // 4
    x = torch.randint(0, 1 << 30, (n,), dtype=torch.int32, device="cuda")
    res = {}
    for name, fn, nbytes in (("read_only_amax", lambda: torch.amax(x), 4 << 30),
                             ("copy", None, 4 << 30)):
        if fn is None:
            src, dst = x[: n // 2], x[n // 2:]
            fn = lambda: dst.copy_(src)
        for _ in range(2):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            fn()
        e1.record()
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / reps
        res[name] = {"ms": ms, "gb_per_s": nbytes / (ms * 1e-3) / 1e9}
    del x
    torch.cuda.empty_cache()
    return res


def allocator_measurement(seconds: float = 1.0):
    """Host allocator throughput (C++): admit with prefix-cache hits, decode
    appends, release, on a 4096-block pool; operations per second."""
    import paged_kv_cache_358_b200 as pkv

    a = pkv.BlockAllocator(4096, 16, enable_cache=True)
    ids = np.arange(64, dtype=np.int32)
    st = np.zeros(64, dtype=np.int32)
    cp = np.zeros((64, 3), dtype=np.int32)
    ops = 0
    t0 = time.perf_counter()
    rnd = 0
    while time.perf_counter() - t0 < seconds:
        for i in ids:
            keys = [(int(i) % 8) * 100 + k for k in range(4)]
            rc, _ = a.add_seq_prefix(int(i), 64 + int(i) % 16, keys)
            if rc == 0:
                for k in range(4):
                    a.set_block_key(int(i), k, keys[k])
        for _ in range(16):
            a.append_arrays(ids, st, cp)
        for i in ids:
            a.free_seq(int(i))
        ops += 64 * 2 + 16 * 64 + 64 * 4
        rnd += 1
    dt = time.perf_counter() - t0
    assert a.check()
    return {"ops_per_s": ops / dt, "note": "admit with prefix hits + 4 key registrations + 16 appends + release, "
                                             "per request, 64 requests per round, through the Python binding",
            "prefix_hits": a.stats()["prefix_hits"]}


def reference_arm(args):
    """--impl reference: the oracle on the host cores, as the comparison arm."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import workloads as W
    from oracle import attention as oatt

    wl = W.workload("teaching_32x4096")
    g = W.rng(321)
    # each step: one layer of a bounded sample (4 requests x 4096 history)
    reqs = 4
    hist = [(W.normal_bf16_bits(g, (4096, 8, 128)), W.normal_bf16_bits(g, (4096, 8, 128)),
             W.normal_bf16_bits(g, (32, 128))) for _ in range(reqs)]
    step_bytes = reqs * (4096 * 8 * 128 * 2 * 2 + 2 * 32 * 128 * 2)

    def step():
        for kh, vh, q in hist:
            oatt.dense_decode(q, kh, vh, wl.scale)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = time.perf_counter() - t0
    value = step_bytes * args.steps / dt / 1e9
    threads = _blas_threads()
    line = {"metric": METRIC, "value": value, "unit": "GB/s", "impl": "reference", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1000,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": {"workload": "teaching_32x4096 (bounded sample: 4 of 32 requests, 1 of 32 layers)",
                       "num_seqs": 32, "history": 4096, "layers": 32, "H_q": 32, "H_kv": 8, "head_dim": 128,
                       "block_size": 16},
            "cpu_baseline": {"value": value, "unit": "GB/s", "cores": threads, "host_cpus": os.cpu_count(),
                             "kind": "oracle",
                             "sample": "each step: float64 NumPy dense decode attention of 4 requests x 4096 "
                                       "history, one layer"},
            "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


EXTRAS = {
    "swap": lambda: swap_measurement(),
    "allocator": lambda: allocator_measurement(),
    "multi_query": lambda: multi_query_measurement(),
    "prefix_cow": lambda: prefix_cow_measurement(),
    "large_serving": lambda: large_serving_measurement(),
    "mixed_512": lambda: mixed_512_measurement(),
    "large_serving_steps": lambda: serving_steps_measurement("large_serving", 64),
    "prefix_cow_steps": lambda: {"plain": serving_steps_measurement("prefix_cow", 256),
                                 "shared_prefix": serving_steps_measurement("prefix_cow", 256,
                                                                            shared_prefix=True)},
    "block_size_sweep": lambda: block_size_sweep_measurement(),
    "hbm_ceiling": lambda: hbm_ceiling_measurement(),
}


def main():
    args = parse()
    if args.impl == "reference":
        reference_arm(args)
        return
    if args.extra is not None:
        if args.extra == "multi_query" and args.pool_copies:
            res = multi_query_measurement(copies=args.pool_copies)
        elif args.extra == "prefix_cow" and args.pool_copies:
            res = prefix_cow_measurement(copies=args.pool_copies)
        else:
            res = EXTRAS[args.extra]()
        print(json.dumps({args.extra: res}), flush=True)
        return
    assert args.warmup >= 3, "at least 3 warm-up steps"
    import torch

    rank, world, dist = dist_init(args.gpus)
    torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
    budget = 2 * (args.warmup + args.steps) + 6
    ds = DecodeStep(budget, args.seed + rank, args.kernel, rank, world, args.layers, not args.unfused,
                    not args.no_overlap)
    stream = ds.stream
    for _ in range(args.warmup):
        ds.step()
    torch.cuda.synchronize()
    assert ds.pkv.decode_status(ds.ws) == 0

    # device-resident timed region: the step exactly as a caller runs it, with
    # one event pair around each step's layer loop for the roofline (in the
    # folded path only the attention launches run between the two events)
    uuid = "GPU-" + str(torch.cuda.get_device_properties(torch.cuda.current_device()).uuid)
    clocks = ClockSampler(uuid)
    clocks.start()
    time.sleep(0.3)
    ds.bytes_done = 0
    ds.launches = 0
    ds.record_attn = True
    start_ev = torch.cuda.Event(enable_timing=True)
    ds.step_events = []

    def first_event():
        start_ev.record(stream)

    ms, wall = timed(ds.step, args.steps, dist, stream, start=first_event)
    ds.record_attn = False
    marks = [start_ev] + ds.step_events
    step_ms = np.array([a.elapsed_time(b) for a, b in zip(marks[:-1], marks[1:])])
    ds.step_events = None
    clk = clocks.stop()
    launches = ds.launches
    step_bytes = ds.bytes_done
    attn_ms = [a.elapsed_time(b) / ds.L for a, b in ds.attn_events]   # per launch
    attn_bytes = ds.attn_bytes
    assert ds.pkv.decode_status(ds.ws) == 0

    # end-to-end timed region: inputs from pinned host buffers, outputs read back
    for _ in range(2):
        ds.step(e2e=True)
    ds.drain()   # the warm-up's last readback goes out before the timed region
    ds.bytes_done = 0
    ms_e2e, _ = timed(lambda: ds.step(e2e=True), args.steps, dist, stream, finish=ds.drain)
    e2e_bytes = ds.bytes_done
    h2d, d2h = ds.h2d_d2h_bytes()

    ms_max = max_over_ranks(ms, dist)
    ms_e2e_max = max_over_ranks(ms_e2e, dist)
    total_bytes = sum_over_ranks(step_bytes, dist)
    total_e2e = sum_over_ranks(e2e_bytes, dist)
    value = total_bytes / (ms_max / 1000) / 1e9
    e2e_value = total_e2e / (ms_e2e_max / 1000) / 1e9
    peak, peak_kind = peaks()
    avg_attn_ms = float(np.mean(attn_ms))
    achieved = float(np.mean(attn_bytes)) / (avg_attn_ms / 1000) / 1e9
    traffic = read_traffic("paged_decode_attn_teaching_32x4096_bytes_per_launch")
    result = None
    if rank == 0:
        cpu = None
        if not args.no_cpu_baseline and world == 1:
            cpu = cpu_baseline(args.cpu_seconds)
        extras = None
        if world == 1 and not args.no_extras:
            # the headline batch's pools are not needed any more
            ds.k_pools = ds.v_pools = None
            torch.cuda.empty_cache()
            extras = {"swap_500mib": swap_measurement(), "allocator": allocator_measurement(),
                      "multi_query_32x4096": multi_query_measurement(),
                      "prefix_cow_256x2264": prefix_cow_measurement(),
                      "large_serving_256xU8192": large_serving_measurement(),
                      "mixed_512xU512": mixed_512_measurement(),
                      "large_serving_steps_24L": serving_steps_measurement("large_serving", 64),
                      "prefix_cow_steps_24L": {
                          "plain": serving_steps_measurement("prefix_cow", 256),
                          "shared_prefix": serving_steps_measurement("prefix_cow", 256, shared_prefix=True)},
                      "mixed_512_block_size_sweep": block_size_sweep_measurement(),
                      "hbm_ceiling_4gib": hbm_ceiling_measurement()}
        steps_per_s = args.steps / (ms_max / 1000) * world
        result = {
            "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_max / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": "teaching_32x4096" if ds.L == 32 else f"teaching_32x4096 ({ds.L} layers)",
                       "layers": ds.L, "num_seqs": ds.S, "history": 4096,
                       "H_q": ds.Hq, "H_kv": ds.Hkv, "head_dim": ds.D, "block_size": ds.B,
                       "pool_blocks_per_layer": ds.N, "kv_pool_gib": round(2 * ds.L * ds.N * ds.B * ds.Hkv * ds.D * 2 / 2**30, 2),
                       "l2": "inputs larger than L2 (KV pool far above 126 MB); no flush",
                       "parallelism": f"replicas x{world} (requests sharded by rank, no collective)",
                       "launch_overlap": bool(ds.overlap and ds.fused)},
            "steps_per_s": steps_per_s, "tokens_per_s": steps_per_s * ds.S,
            "step_ms": step_stats(step_ms),
            "frac_of_nominal_8tbs": value / NOMINAL_HBM_GBS,
            "e2e": {"value": e2e_value, "unit": "GB/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "ms_per_step": ms_e2e_max / args.steps},
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "traffic": traffic, "peak_kind": peak_kind,
                         "kernel": ("paged_decode_attn_append_run (append and merge folded in)" if ds.fused else
                                    "paged_decode_attn_run (merge folded in)") + ", 32x4096, one layer per launch"
                                   + ("; layers 2..32 overlap their predecessor's tail (programmatic dependent "
                                      "launch), so the per-launch time is the layer loop's span / 32"
                                      if ds.overlap and ds.fused else ""),
                         "avg_launch_us": avg_attn_ms * 1000,
                         "frac_of_nominal_8tbs": achieved / NOMINAL_HBM_GBS},
            "cpu_baseline": cpu,
            "clocks": clk,
            "gpu_launches": launches,
            "extras": extras,
            "wall_s_timed": wall,
        }
        print(json.dumps(result), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
