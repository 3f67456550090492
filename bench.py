#!/usr/bin/env python
"""Throughput of the fused ZeRO shard step on B200: params/s, HBM GB/s and the fraction of
the measured HBM roofline.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload gpt2_small|shard_7p5b|flat] [--nd ND] [--bucket B]

One step is one pass of the whole hot path over one batch of synthetic input: the
reduce-scatter of the Nd simulated ranks' fp16 gradients, the unscale, the fp32 Adam update of
every owner's shard, the fp16 cast and the all-gather write-back into the full parameter buffer
(zero_step_fused over the step's range(s), then zero_step_commit), all resident in HBM.

Workloads (synthetic, seeded):
  gpt2_small  GPT-2-small parameter list (psi = 123,653,376), Nd = 8, stage 1 (full local
              gradients, one fused call per step); grads N(0, 1e-3^2) with 1% x100; master
              N(0, 0.02^2), m = v = 0 at the start.               (default)
  shard_7p5b  one owner's view of 7.5e9 parameters at Nd = 64: a 117,187,500-element shard,
              64 separate fp16 gradient slices, written into a 7.5e9-element fp16 buffer at
              r*S (r = 31); master U(-0.05, 0.05), m N(0, 1e-4^2), v |N(0, 1e-6^2)|.
  flat        psi = 2^29 flat buffer, one fused call per bucket of B elements in backward
              order, Nd in {2, 4, 8, 16, 64}; state as shard_7p5b.

Every step reads and writes far more than the 126 MB L2 (5.2 GB for gpt2_small), so no L2 flush
is needed between steps. With N > 1 (torchrun), every rank runs its own replica of the
simulated Nd-rank step on its own GPU (the Nd ranks are simulated on one device; no data
crosses GPUs), and the time is the maximum over ranks.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

FALLBACK_HBM_GBS = 6650.0
CSRC = os.path.join(ROOT, "zero_partitioned_optimizer_plan_b200", "csrc")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.json")
METRIC = "fused ZeRO shard step params/sec"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=["gpt2_small", "shard_7p5b", "flat", "zero2_1p3b",
                                           "zero2_gpt2_small"],
                    default="gpt2_small")
    ap.add_argument("--nd", type=int, default=None)
    ap.add_argument("--bucket", type=int, default=None)
    ap.add_argument("--psi", type=int, default=None, help="flat workload size (default 2^29)")
    ap.add_argument("--graph", action="store_true",
                    help="capture a step's calls in CUDA graphs (constants in device memory)")
    ap.add_argument("--dynamic-scale", action="store_true",
                    help="with --graph: dynamic loss scaling on the device (scaler prepare and "
                         "update kernels in the graph, no host work per step)")
    ap.add_argument("--payload", choices=["fp16", "q8"], default="fp16",
                    help="q8: the owner reduces int8 payloads with one fp32 scale per 128 "
                         "elements (quantized once per rank before timing)")
    ap.add_argument("--stage2-fused", action="store_true",
                    help="stage-2 workloads: the bucket scheduler launches the fused step per "
                         "bucket (zero_sched_create_fused) instead of reduce-scatter + update")
    ap.add_argument("--no-overlap", action="store_true",
                    help="launch the per-bucket calls of a step strictly one after another "
                         "(default: inside a zero_overlap_begin/end region)")
    ap.add_argument("--e2e-steps", type=int, default=None)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    a = ap.parse_args()
    if a.warmup < 3:
        ap.error("--warmup must be >= 3")
    return a


# ---------------------------------------------------------------------------------------------
# workloads
# ---------------------------------------------------------------------------------------------
def workload_config(args) -> dict:
    """The workload's name and sizes as both arms report them (no device needed)."""
    from zero_partitioned_optimizer_plan_b200 import synth
    kind = args.workload
    if kind == "gpt2_small":
        nd = args.nd or 8
        numels = synth.gpt2_small_list()
        cfg = {"workload": "gpt2_small_stage1", "psi": sum(numels), "nd": nd, "stage": 1,
               "calls_per_step": 1, "tensors": len(numels)}
    elif kind == "shard_7p5b":
        nd = args.nd or 64
        total = 7_500_000_000
        cfg = {"workload": "shard_7p5b_rank31", "psi_total": total, "shard": total // nd,
               "nd": nd, "owner": 31, "calls_per_step": 1}
    elif kind in ("zero2_1p3b", "zero2_gpt2_small"):
        small = kind == "zero2_gpt2_small"
        nd = args.nd or (8 if small else 16)
        B = args.bucket or (10_000_000 if small else 50_000_000)
        numels = synth.gpt2_small_list() if small else synth.gpt_1p3b_list()
        psi = sum(numels)
        psi_p = -(-psi // nd) * nd
        nb = -(-psi_p // B)
        cfg = {"workload": kind, "psi": psi, "nd": nd, "stage": 2, "bucket": B, "buckets": nb,
               "calls_per_step": nb + nd}
        if args.stage2_fused:
            cfg["workload"] = kind + "_fused"
            cfg["calls_per_step"] = nb + 1
        cfg["overlap"] = not args.no_overlap
        return cfg
    else:
        nd = args.nd or 16
        psi = args.psi or (1 << 29)
        B = args.bucket or min(psi, 1 << 26)
        cfg = {"workload": "flat_2p29" if psi == 1 << 29 else f"flat_{psi}", "psi": psi,
               "nd": nd, "bucket": B, "calls_per_step": -(-psi // B)}
    if cfg["calls_per_step"] > 1:
        cfg["overlap"] = not args.no_overlap
    if args.payload == "q8":
        cfg["payload"] = "int8 records: 128 values and their fp32 scale"
        cfg["workload"] += "_q8"
    return cfg


class Workload:
    """Device buffers and the per-step call sequence of one workload."""

    def __init__(self, args, dev):
        import torch
        from zero_partitioned_optimizer_plan_b200 import libzero as lz
        from zero_partitioned_optimizer_plan_b200 import synth
        self.torch, self.lz, self.dev = torch, lz, dev
        self.hp = lz.AdamHP()
        kind = args.workload
        self.kind = kind
        if kind == "gpt2_small":
            nd = args.nd or 8
            numels = synth.gpt2_small_list()
            pl = lz.zero_plan_create(numels, nd, 1, 0)
            psi, psi_p, S, nb = lz.zero_plan_info(pl)
            self.nd, self.n, self.psi = nd, psi_p, psi
            self.ranges = [(0, psi_p)]
            self.grads = []
            for r in range(nd):
                g = torch.zeros(psi_p, dtype=torch.float16, device=dev)
                synth.grad_f16(psi, 1e-3, seed=0, rank=r, step=1, spike_frac=0.01,
                               spike_scale=100.0, out=g[:psi])
                self.grads.append(g)
            master, m, v = synth.state_small(psi_p, seed=0, device=dev)
            self.params = torch.empty(psi_p, dtype=torch.float16, device=dev)
            self.param_base = 0
            self.config = workload_config(args)
        elif kind == "shard_7p5b":
            nd = args.nd or 64
            total = 7_500_000_000
            S = total // nd
            r = 31
            self.nd, self.n, self.psi = nd, S, S
            self.ranges = [(0, S)]
            self.grads = [synth.grad_f16(S, 1e-3, seed=0, rank=j, step=1, device=dev)
                          for j in range(nd)]
            master, m, v = synth.state_warm(S, seed=0, device=dev)
            self.full = torch.zeros(total, dtype=torch.float16, device=dev)
            self.params = self.full[r * S:(r + 1) * S]
            self.param_base = r * S
            self.config = workload_config(args)
        elif kind in ("zero2_1p3b", "zero2_gpt2_small"):
            self._init_zero2(args, dev)
            return
        else:
            nd = args.nd or 16
            psi = args.psi or (1 << 29)
            B = args.bucket or min(psi, 1 << 26)
            self.nd, self.n, self.psi = nd, psi, psi
            self.ranges = []
            hi = psi
            while hi > 0:
                lo = max(0, hi - B)
                self.ranges.append((lo, hi))
                hi = lo
            self.grads = [synth.grad_f16(psi, 1e-3, seed=0, rank=j, step=1, device=dev)
                          for j in range(nd)]
            master, m, v = synth.state_warm(psi, seed=0, device=dev)
            self.params = torch.empty(psi, dtype=torch.float16, device=dev)
            self.param_base = 0
            self.config = workload_config(args)
            assert self.config["calls_per_step"] == len(self.ranges)
        self.cur = [master, m, v]
        self.nxt = [torch.empty_like(x) for x in self.cur]
        self.bytes_per_step = (2 * self.nd + 26) * self.n     # algorithmic HBM bytes
        # the dominant kernel: its bytes and launches per step
        self.dominant = "fused_tma_kernel"
        self.dominant_bytes = self.bytes_per_step
        self.dominant_calls = len(self.ranges)
        self.side = None
        self.payload = args.payload
        # the per-bucket calls of a step touch disjoint ranges: declare them independent
        self.overlap = len(self.ranges) > 1 and not args.no_overlap
        if self.payload == "q8":
            self._quantize_payload()

    def _quantize_payload(self):
        """Each rank's gradients as int8 + one fp32 scale per 128 (the senders' work, done once
        before timing and timed on its own)."""
        torch, lz = self.torch, self.lz
        n, nd = self.n, self.nd
        # one payload per range and rank, records counted from the range's first element;
        # self.q[i * nd + r] is range i's payload of rank r
        self.q = [torch.empty(lz.q8_payload_bytes(hi - lo), dtype=torch.uint8, device=self.dev)
                  for lo, hi in self.ranges for _ in range(nd)]
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        lo0, hi0 = self.ranges[0]
        lz.zero_quantize_q8(hi0 - lo0, self.grads[0][lo0:hi0], self.q[0])   # first use untimed
        e0.record()
        for i, (lo, hi) in enumerate(self.ranges):
            for r, g in enumerate(self.grads):
                lz.zero_quantize_q8(hi - lo, g[lo:hi], self.q[i * nd + r])
        e1.record()
        torch.cuda.synchronize()
        recs = sum((hi - lo + 127) // 128 for lo, hi in self.ranges)
        qbytes = nd * (2 * n + 132 * recs)
        self.side = {"kernel": "quant_q8_kernel (senders, once)", "bytes": qbytes,
                     "calls": nd * len(self.ranges), "ms": [(e0, e1)]}
        self.grads = None
        torch.cuda.empty_cache()
        self.bytes_per_step = nd * 132 * recs + 26 * n
        self.dominant = "fused_q8_tma_kernel"
        self.dominant_bytes = self.bytes_per_step

    def inputs(self):
        """The tensors a step consumes that a host would have to upload."""
        if self.payload == "q8":
            return self.q
        return self.grads

    # --- CUDA-graph mode: the step's calls read the Adam constants from device memory -------
    def enable_graph(self, dynamic=False, max_steps=0):
        torch, lz = self.torch, self.lz
        dev = self.cur[0].device
        self.dynamic = dynamic
        self.d_consts = torch.empty(40, dtype=torch.uint8, device=dev)
        self.h_consts = [torch.empty(40, dtype=torch.uint8, pin_memory=True) for _ in range(2)]
        self.h_done = [None, None]
        self.g_status = torch.zeros(1, dtype=torch.int32, device=dev)
        self.g_flags = torch.zeros(1, dtype=torch.int32, device=dev)
        a, b = self.cur, self.nxt
        if dynamic:
            n_tab = max_steps + 2
            tab = lz.zero_adam_consts_table(self.hp, 1, n_tab)
            self.d_table = torch.frombuffer(bytearray(bytes(tab)), dtype=torch.uint8).to(dev)
            self.n_tab = n_tab
            init = lz.ScalerState(self.hp.loss_scale, 0, 1, 0)
            self.d_scaler0 = torch.frombuffer(bytearray(bytes(init)), dtype=torch.uint8).to(dev)
            self.d_scaler = self.d_scaler0.clone()
            self.scaler_prm = lz.ScalerParams(2.0, 0.5, 2000)

        def body(src, dst):
            if dynamic:
                lz.zero_scaler_prepare(self.d_scaler, self.d_table, self.n_tab, self.d_consts,
                                       self.g_status)
            else:
                self.g_status.zero_()
            if self.overlap:
                lz.zero_overlap_begin()
            nd = self.nd
            for i, (lo, hi) in enumerate(self.ranges):
                if self.payload == "q8":
                    lz.zero_step_fused_q8_dc(hi - lo, nd, self.q[i * nd:(i + 1) * nd],
                                             *[x[lo:hi] for x in src], *[x[lo:hi] for x in dst],
                                             self.params[lo:hi], self.d_consts, self.g_status)
                else:
                    lz.zero_step_fused_dc(hi - lo, nd, [g[lo:hi] for g in self.grads],
                                          *[x[lo:hi] for x in src], *[x[lo:hi] for x in dst],
                                          self.params[lo:hi], self.d_consts, self.g_status)
            if self.overlap:
                lz.zero_overlap_end()
            lz.zero_step_commit(self.n, *src, *dst, self.params, self.g_status)
            if dynamic:
                lz.zero_scaler_update(self.d_scaler, self.scaler_prm, self.g_status)
            self.g_flags.bitwise_or_(self.g_status)

        self._load_consts(1)
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            body(a, b)                  # first use outside the capture
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize()
        self.graphs = []
        for src, dst in ((a, b), (b, a)):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                body(src, dst)
            self.graphs.append(g)
        self.g_flags.zero_()
        if dynamic:
            self.d_scaler.copy_(self.d_scaler0)
        self.graph_dir = 0
        self.step = self._graph_step

    def _load_consts(self, t):
        """Copy step t's constants to the device, double-buffered in pinned host memory."""
        torch, lz = self.torch, self.lz
        i = t % 2
        if self.h_done[i] is not None:
            self.h_done[i].synchronize()      # the copy that last read this buffer is done
        c = lz.zero_adam_consts_for_step(self.hp, t)
        self.h_consts[i].copy_(torch.frombuffer(bytearray(bytes(c)), dtype=torch.uint8))
        self.d_consts.copy_(self.h_consts[i], non_blocking=True)
        e = torch.cuda.Event()
        e.record()
        self.h_done[i] = e

    def _graph_step(self, t, status, ev=None, grads=None):
        if grads is not None:
            raise ValueError("graph mode has no host-buffer variant")
        if not self.dynamic:   # with the device scaler, the graph picks t's constants itself
            self._load_consts(t)
        if ev is not None:
            ev[0].record()
        self.graphs[self.graph_dir].replay()
        if ev is not None:
            ev[1].record()
        self.graph_dir ^= 1

    def step(self, t, status, ev=None, grads=None):
        """Enqueue one step on the current stream; ev = (start, end) events around the
        dominant kernel's launches. grads: the step's inputs (as inputs() lists them) when
        they are not the workload's own buffers."""
        lz = self.lz
        if self.payload == "q8":
            pays = grads or self.inputs()
            nd = self.nd
            if ev is not None:
                ev[0].record()
            if self.overlap:
                lz.zero_overlap_begin()
            for i, (lo, hi) in enumerate(self.ranges):
                lz.zero_step_fused_q8(hi - lo, nd, pays[i * nd:(i + 1) * nd],
                                      *[x[lo:hi] for x in self.cur], *[x[lo:hi] for x in self.nxt],
                                      self.params[lo:hi], self.hp, t, status)
            if self.overlap:
                lz.zero_overlap_end()
            if ev is not None:
                ev[1].record()
            lz.zero_step_commit(self.n, *self.cur, *self.nxt, self.params, status)
            self.cur, self.nxt = self.nxt, self.cur
            return
        grads = grads or self.grads
        if ev is not None:
            ev[0].record()
        if self.overlap:
            lz.zero_overlap_begin()
        for lo, hi in self.ranges:
            lz.zero_step_fused(hi - lo, self.nd, [g[lo:hi] for g in grads],
                               *[x[lo:hi] for x in self.cur], *[x[lo:hi] for x in self.nxt],
                               self.params[lo:hi], self.hp, t, status)
        if self.overlap:
            lz.zero_overlap_end()
        if ev is not None:
            ev[1].record()
        lz.zero_step_commit(self.n, *self.cur, *self.nxt, self.params, status)
        self.cur, self.nxt = self.nxt, self.cur


def _init_zero2(self, args, dev):
    """Stage 2 on the 1.3B list (Nd = 16, buckets of 50,000,000 elements), or on the GPT-2-small
    list (Nd = 8, buckets of 10,000,000; a smaller case for profiling). The backward pass's
    output (every bucket's local gradients of every rank) is already in the scheduler's staging
    slots, one slot per bucket; a step is the reduce-scatter of the buckets in backward order
    through the scheduler, then the owners' updates (zero_adam_shard)."""
    torch, lz = self.torch, self.lz
    from zero_partitioned_optimizer_plan_b200 import synth
    if args.payload != "fp16":
        raise SystemExit("the stage-2 workloads take fp16 payloads")
    self.payload = "fp16"
    small = args.workload == "zero2_gpt2_small"
    nd = args.nd or (8 if small else 16)
    B = args.bucket or (10_000_000 if small else 50_000_000)
    numels = synth.gpt2_small_list() if small else synth.gpt_1p3b_list()
    self.plan = pl = lz.zero_plan_create(numels, nd, 2, B)
    psi, psi_p, S, nb = lz.zero_plan_info(pl)
    self.nd, self.n, self.psi, self.S, self.nb = nd, psi_p, psi, S, nb
    self.slot_elems = lz.zero_sched_slot_elems(pl, nb)
    self.slots = torch.empty(self.slot_elems, dtype=torch.float16, device=dev)
    stride = self.slot_elems // (nb * nd)
    for k in range(nb):
        lo, ln, _, _ = lz.zero_plan_bucket(pl, k)
        for r in range(nd):
            base = (k * nd + r) * stride
            synth.grad_f16(ln, 1e-3, seed=0, rank=r, step=1000 + k,
                           out=self.slots[base:base + ln])
    self.master, self.m, self.v = synth.state_small(psi_p, seed=0, device=dev)
    self.params = torch.empty(psi_p, dtype=torch.float16, device=dev)
    self.shards = torch.empty(psi_p, dtype=torch.float32, device=dev)
    self.grads = None
    self.ranges = [(0, psi_p)]
    # the buckets' reduce-scatters (or fused steps) of a step touch disjoint ranges
    self.overlap = not args.no_overlap
    self.param_base = 0
    self.config = workload_config(args)
    assert (self.config["psi"], self.config["buckets"]) == (psi, nb)
    if args.stage2_fused:
        # the scheduler launches the fused step per bucket; ping-pong state, commit at the end
        self.cur = [self.master, self.m, self.v]
        self.nxt = [torch.empty_like(x) for x in self.cur]
        self.d_consts = torch.empty(40, dtype=torch.uint8, device=dev)
        self.h_consts = [torch.empty(40, dtype=torch.uint8, pin_memory=True) for _ in range(2)]
        self.h_done = [None, None]
        self.bytes_per_step = (2 * nd + 26) * psi_p
        self.dominant = "fused_tma_kernel"
        self.dominant_bytes = self.bytes_per_step
        self.dominant_calls = nb
        self.side = None
        self.step = self._step_zero2_fused
        return
    rs_bytes = (2 * nd + 4) * psi_p
    adam_bytes = 30 * psi_p
    self.bytes_per_step = rs_bytes + adam_bytes
    self.dominant = "rs_tma_kernel"
    self.dominant_bytes = rs_bytes
    self.dominant_calls = nb
    self.side = {"kernel": "adam_kernel", "bytes": adam_bytes, "calls": nd, "ms": []}
    self.step = self._step_zero2


def _step_zero2(self, t, status, ev=None, grads=None):
    lz, torch = self.lz, self.torch
    if grads is not None:
        raise ValueError("the stage-2 workload has no host-buffer variant")
    S, nd = self.S, self.nd
    stream = torch.cuda.current_stream()
    sch = lz.zero_sched_create(self.plan, self.slots, self.slot_elems, self.nb,
                               [self.shards[r * S:(r + 1) * S] for r in range(nd)], status,
                               stream)
    if ev is not None:
        ev[0].record()
    if self.overlap:
        lz.zero_overlap_begin(stream)
    for k in range(self.nb):
        lz.zero_sched_begin_bucket(sch, k, stream)
        lz.zero_sched_end_bucket(sch, k, stream)
    if self.overlap:
        lz.zero_overlap_end(stream)
    lz.zero_sched_wait(sch, stream)
    if ev is not None:
        ev[1].record()
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a0.record()
    for r in range(nd):
        sl = slice(r * S, (r + 1) * S)
        lz.zero_adam_shard(S, self.shards[sl], self.master[sl], self.m[sl], self.v[sl],
                           self.params[sl], self.hp, t, status)
    if ev is not None:
        a1.record()
        self.side["ms"].append((a0, a1))
    lz.zero_sched_destroy(sch)


def _step_zero2_fused(self, t, status, ev=None, grads=None):
    """Stage 2 with the fused step per bucket: the scheduler launches each bucket's fused
    kernel as the bucket arrives (its slot released after it), then one commit."""
    lz, torch = self.lz, self.torch
    if grads is not None:
        raise ValueError("the stage-2 workload has no host-buffer variant")
    stream = torch.cuda.current_stream()
    self._load_consts(t)
    sch = lz.zero_sched_create_fused(self.plan, self.slots, self.slot_elems, self.nb, *self.cur,
                                     *self.nxt, self.params, self.d_consts, status, stream)
    if ev is not None:
        ev[0].record()
    if self.overlap:
        lz.zero_overlap_begin(stream)
    for k in range(self.nb):
        lz.zero_sched_begin_bucket(sch, k, stream)
        lz.zero_sched_end_bucket(sch, k, stream)
    if self.overlap:
        lz.zero_overlap_end(stream)
    lz.zero_sched_wait(sch, stream)
    if ev is not None:
        ev[1].record()
    lz.zero_step_commit(self.n, *self.cur, *self.nxt, self.params, status)
    lz.zero_sched_destroy(sch)
    self.cur, self.nxt = self.nxt, self.cur


Workload._init_zero2 = _init_zero2
Workload._step_zero2 = _step_zero2
Workload._step_zero2_fused = _step_zero2_fused


# ---------------------------------------------------------------------------------------------
# clocks during the timed region (NVML, the data nvidia-smi reports)
# ---------------------------------------------------------------------------------------------
REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
           0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
           0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
           0x100: "display_clock_setting"}


class ClockSampler:
    def __init__(self, dev_index):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()
        self.ok = False
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(dev_index).uuid)
            if not uuid.startswith("GPU-"):
                uuid = "GPU-" + uuid
            self.h = pynvml.nvmlDeviceGetHandleByUUID(uuid)
            self.nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # clocks are reported as unavailable, the run still counts
            self.err = repr(e)

    def _run(self):
        nv = self.nv
        get_r = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                bits = get_r(self.h)
                for b, name in REASONS.items():
                    if bits & b:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(0.01)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()

    def report(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "note": self.err}
        med = statistics.median(self.samples) if self.samples else None
        return {"sm_mhz": med, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                "samples": len(self.samples)}


# ---------------------------------------------------------------------------------------------
# helpers
# ---------------------------------------------------------------------------------------------
def measured_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            pk = json.load(f)
        return float(pk["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


# The source files each kernel is built from: a kernel's DRAM counters stay valid while these
# files are unchanged.
KERNEL_SOURCES = {
    "fused_tma_kernel": ("zero_kernels.cu", "zero_device.cuh", "zero_internal.h"),
    "rs_tma_kernel": ("zero_kernels.cu", "zero_device.cuh", "zero_internal.h"),
    "adam_kernel": ("zero_kernels.cu", "zero_device.cuh", "zero_internal.h"),
    "fused_q8_tma_kernel": ("zero_q8.cu", "zero_device.cuh", "zero_internal.h"),
}


def kernel_sources_sha256(kernel: str) -> str:
    """One hash over the sources of `kernel` (the code the ncu counters describe)."""
    h = hashlib.sha256()
    for name in KERNEL_SOURCES[kernel]:
        with open(os.path.join(CSRC, name), "rb") as f:
            h.update(name.encode() + b"\0" + f.read())
    return h.hexdigest()


def traffic_key(wl) -> str:
    """Key of a workload's entry in the traffic table: workload and Nd, and the bucket size
    when a step is several calls (a launch's bytes depend on it)."""
    key = f"{wl.config['workload']}_nd{wl.nd}"
    if wl.config.get("calls_per_step", 1) > 1 and "bucket" in wl.config:
        key += f"_b{wl.config['bucket']}"
    return key


def traffic_per_launch(kernel: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on the current
    kernel source; else None."""
    try:
        with open(TRAFFIC_FILE) as f:
            tab = json.load(f)
        sha = kernel_sources_sha256(kernel)
        ent = tab.get(workload, {}).get(kernel)
        if ent and ent.get("kernel_src_sha256") == sha:
            return ent["dram_bytes_per_launch"]
    except Exception:
        pass
    return None


def host_cpu() -> dict:
    """The host's CPU model and hardware thread count (the oracle itself uses one core)."""
    model = "unknown"
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"cpu": model, "threads": os.cpu_count()}


def cpu_oracle_rate(nd: int, n_sample: int, target_s: float, seed=0):
    """Time the oracle (single-threaded C, as it stands) on n_sample elements of the workload's
    distribution; repeat until target_s seconds have passed. Returns (params/s, reps, secs)."""
    import oracle
    from zero_partitioned_optimizer_plan_b200 import synth
    g = [synth.grad_f16(n_sample, 1e-3, seed=seed, rank=r, step=1, spike_frac=0.01,
                        spike_scale=100.0).numpy() for r in range(nd)]
    master, m, v = (x.numpy() for x in synth.state_small(n_sample, seed=seed))
    hp = oracle.AdamHP()
    reps, total = 0, 0.0
    while total < target_s and reps < 50:
        t0 = time.perf_counter()
        skipped, master, m, v, _ = oracle.step(g, master, m, v, hp, reps + 1)
        total += time.perf_counter() - t0
        reps += 1
    return n_sample * reps / total, reps, total


def dist_setup(args=None):
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def max_over_ranks(ms: float, ws: int, device) -> float:
    """The slowest rank's time: every rank must call this, in the same order."""
    if ws == 1:
        return ms
    import torch
    import torch.distributed as dist
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_rate(ws: int, units_per_rank_step: int, steps: int, ms: float) -> float:
    """Whole-job throughput: every rank's units over the slowest rank's time."""
    return ws * units_per_rank_step * steps / (ms / 1e3)


# ---------------------------------------------------------------------------------------------
# reference arm: the CPU oracle, on the host cores, on a bounded sample per step
# ---------------------------------------------------------------------------------------------
def run_reference(args):
    ws, rank, _ = dist_setup(args)
    if rank != 0:
        return 0
    cfg = workload_config(args)
    nd = cfg["nd"]
    # calibrate, then size each step so that the whole run takes about two minutes
    rate, _, _ = cpu_oracle_rate(nd, 200_000, 0.2)
    per_step_s = max(0.05, 120.0 / (args.steps + args.warmup))
    n_sample = int(min(16_000_000, max(100_000, rate * per_step_s)))
    import oracle
    from zero_partitioned_optimizer_plan_b200 import synth
    g = [synth.grad_f16(n_sample, 1e-3, seed=0, rank=r, step=1, spike_frac=0.01,
                        spike_scale=100.0).numpy() for r in range(nd)]
    master, m, v = (x.numpy() for x in synth.state_small(n_sample, seed=0))
    hp = oracle.AdamHP()
    for t in range(1, args.warmup + 1):
        _, master, m, v, _ = oracle.step(g, master, m, v, hp, t)
    t0 = time.perf_counter()
    for t in range(args.warmup + 1, args.warmup + args.steps + 1):
        _, master, m, v, _ = oracle.step(g, master, m, v, hp, t)
    dt = time.perf_counter() - t0
    value = n_sample * args.steps / dt
    sample = (f"first {n_sample} elements of the {cfg['workload']} workload's gradient "
              f"distribution, Nd={nd}, one oracle step per timed step")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "params/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * dt / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": dict(cfg, sample_elems=n_sample, parallelism="replicas1"),
        "cpu_baseline": {"value": value, "unit": "params/s", "cores": 1, "kind": "oracle",
                         "sample": sample, "host": host_cpu()},
        "e2e": {"value": value, "unit": "params/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------------------------
def run_ours(args):
    import torch
    import torch.distributed as dist
    ws, rank, local = dist_setup(args)
    if ws > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    from zero_partitioned_optimizer_plan_b200 import build as zbuild
    zbuild.build()
    from zero_partitioned_optimizer_plan_b200 import libzero as lz

    wl = Workload(args, dev)
    if args.dynamic_scale and not args.graph:
        raise SystemExit("--dynamic-scale needs --graph")
    if args.graph:
        if wl.grads is None and wl.payload != "q8":
            raise SystemExit("--graph applies to the stage-1 and flat workloads")
        wl.enable_graph(dynamic=args.dynamic_scale, max_steps=args.steps + args.warmup + 4)
    K, W = args.steps, args.warmup
    status = torch.zeros(K + W, dtype=torch.int32, device=dev)   # one status word per step
    torch.cuda.synchronize()

    def barrier():
        if ws > 1:
            dist.barrier(device_ids=[local])

    # warm-up
    for i in range(W):
        wl.step(i + 1, status[i:i + 1])
    torch.cuda.synchronize()

    # timed region: K steps on torch's current stream
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(K)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(local)
    barrier()
    torch.cuda.synchronize()
    launches0 = lz.zero_kernel_launches()
    with sampler:
        start.record()
        for i in range(K):
            wl.step(W + i + 1, status[W + i:W + i + 1], ev=evs[i])
        end.record()
        torch.cuda.synchronize()
    launches = lz.zero_kernel_launches() - launches0
    if args.graph:   # replays launch the captured kernels without the host library
        launches = K * (len(wl.ranges) + 1 + (2 if args.dynamic_scale else 0))
        if int(wl.g_flags.item()) != 0:
            raise RuntimeError(f"unexpected status flags in the timed steps: {wl.g_flags.item()}")
    barrier()
    ms = start.elapsed_time(end)
    kernel_ms = [a.elapsed_time(b) for a, b in evs]
    flags = status.cpu()
    if int((flags != 0).sum()):
        raise RuntimeError(f"unexpected status flags in the timed steps: {set(flags.tolist())}")
    ms = max_over_ranks(ms, ws, dev)
    ms_per_step = ms / K
    value = aggregate_rate(ws, wl.n, K, ms)

    # roofline of the dominant kernel: algorithmic bytes per launch / mean launch time
    calls = wl.dominant_calls
    launch_s = statistics.mean(kernel_ms) / 1e3 / calls
    bytes_per_launch = wl.dominant_bytes / calls
    peak, peak_kind = measured_peak()
    achieved = bytes_per_launch / launch_s / 1e9
    roofline = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                "frac": achieved / peak, "peak_source": peak_kind,
                "traffic": traffic_per_launch(wl.dominant, traffic_key(wl)),
                "kernel": wl.dominant, "bytes_per_launch": bytes_per_launch,
                "kernel_ms_mean": launch_s * 1e3}
    if wl.side is not None:   # the other kernel of the step (or the senders' quantization)
        side_s = statistics.mean(a.elapsed_time(b) for a, b in wl.side["ms"][-K:]) / 1e3
        roofline["other"] = {"kernel": wl.side["kernel"],
                             "achieved": wl.side["bytes"] / side_s / 1e9,
                             "frac": wl.side["bytes"] / side_s / 1e9 / peak,
                             "ms_per_step": side_s * 1e3}

    # end to end through the public API with host buffers: every step uploads its gradients
    # from pinned host memory, runs, and downloads the updated fp16 parameters and its status
    # word, which the host reads. The upload of step i+1 overlaps step i's compute and download
    # (double-buffered device gradients; copies on their own streams, ordered by events).
    e2e = None
    if not args.no_e2e and wl.inputs() is not None and not args.graph:
        E = args.e2e_steps or max(3, min(K, 10))
        h_grads = [torch.empty(g.numel(), dtype=g.dtype, pin_memory=True) for g in wl.inputs()]
        for h, g in zip(h_grads, wl.inputs()):
            h.copy_(g)
        h_params = [torch.empty(wl.params.numel(), dtype=torch.float16, pin_memory=True)
                    for _ in range(2)]
        h_status = [torch.empty(1, dtype=torch.int32, pin_memory=True) for _ in range(2)]
        d_grads = [[torch.empty_like(g) for g in wl.inputs()] for _ in range(2)]
        st = torch.zeros(E, dtype=torch.int32, device=dev)
        main = torch.cuda.current_stream()
        up, down = torch.cuda.Stream(), torch.cuda.Stream()
        ev = lambda: torch.cuda.Event()   # noqa: E731
        up_done, comp_done, down_done = [None, None], [None, None], [None, None]
        torch.cuda.synchronize()
        barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(main)
        up.wait_event(e0)

        def read_result(j):
            down_done[j % 2].synchronize()            # the caller reads step j's result
            if int(h_status[j % 2].item()) != 0:
                raise RuntimeError("unexpected status in the end-to-end steps")

        for i in range(E):
            b = i % 2
            with torch.cuda.stream(up):
                if comp_done[b] is not None:
                    up.wait_event(comp_done[b])     # step i-2 is done with these buffers
                for d, h in zip(d_grads[b], h_grads):
                    d.copy_(h, non_blocking=True)
                up_done[b] = ev()
                up_done[b].record(up)
            main.wait_event(up_done[b])
            if down_done[1 - b] is not None:
                main.wait_event(down_done[1 - b])   # step i-1's parameters are downloaded
            wl.step(W + K + i + 1, st[i:i + 1], grads=d_grads[b])
            comp_done[b] = ev()
            comp_done[b].record(main)
            with torch.cuda.stream(down):
                down.wait_event(comp_done[b])
                h_params[b].copy_(wl.params, non_blocking=True)
                h_status[b].copy_(st[i:i + 1], non_blocking=True)
                down_done[b] = ev()
                down_done[b].record(down)
            if i > 0:
                read_result(i - 1)
        main.wait_event(down_done[(E - 1) % 2])
        e1.record(main)
        read_result(E - 1)
        torch.cuda.synchronize()
        ems = max_over_ranks(e0.elapsed_time(e1), ws, dev)
        e2e = {"value": aggregate_rate(ws, wl.n, E, ems), "unit": "params/s",
               "h2d_bytes_per_step": sum(h.numel() * h.element_size() for h in h_grads),
               "d2h_bytes_per_step": 2 * wl.n + 4,
               "steps": E, "overlap": "upload of step i+1 overlaps compute and download of step i"}

    cpu = None
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        n_sample = 8_000_000
        rate, reps, secs = cpu_oracle_rate(wl.nd, n_sample, 10.0)
        cpu = {"value": rate, "unit": "params/s", "cores": 1, "kind": "oracle",
               "sample": f"{n_sample} elements with the workload's gradient distribution, "
                         f"Nd={wl.nd}, {reps} oracle steps, {secs:.1f} s",
               "host": host_cpu()}

    if rank == 0:
        cfg = dict(wl.config)
        if args.graph:
            cfg["cuda_graph"] = "one replay per step; kernel time includes the commit"
            if args.dynamic_scale:
                cfg["loss_scale"] = "dynamic, on the device (scaler kernels inside the graph)"
        cfg.update({"l2": "no flush: every step streams several GB, far above L2",
                    "bytes_per_step": wl.bytes_per_step, "parallelism": f"replicas{ws}",
                    "hbm_gbs": wl.bytes_per_step / (ms_per_step / 1e3) / 1e9})
        line = {
            "metric": METRIC, "value": value, "unit": "params/s", "n_gpus": ws, "steps": K,
            "warmup": W, "ms_per_step": ms_per_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic (seeded fp16 gradients and fp32 optimizer state)",
            "config": cfg, "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": launches, "clocks": sampler.report(),
        }
        print(json.dumps(line), flush=True)
    if ws > 1:
        dist.destroy_process_group()
    return 0


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
