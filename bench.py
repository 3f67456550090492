#!/usr/bin/env python
"""Throughput of the fused ZeRO shard step on B200: params/s, HBM GB/s and the fraction of
the measured HBM roofline.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload zero2_1p3b|zero2_gpt2_small|zero3_gpt2_small|zero3_1p3b|
                                gpt2_small|tiny|shard_7p5b|flat]
                    [--stage2 fused|unfused] [--payload fp16|q8] [--graph] [--nd ND]
                    [--bucket B] [--layer-buffers L] [--no-sweep]

One step is one pass of the whole hot path over one batch of synthetic input: the
reduce-scatter of the Nd simulated ranks' fp16 gradients, the unscale, the fp32 Adam update of
every owner's shard, the fp16 cast and the all-gather write-back into the full parameter buffer
(zero_step_fused over the step's range(s), then zero_step_commit), all resident in HBM.

Workloads (synthetic, seeded):
  zero2_1p3b  ZeRO stage 2 on a 1.3B GPT-shaped list (24 layers, hidden 2048, FFN 8192, vocab
              50257; psi = 1,311,528,960), Nd = 16, buckets of 50,000,000 elements in backward
              order (27 buckets). The bucket scheduler launches the fused step per bucket as the
              bucket arrives and releases its staging slot after it, then one commit (--stage2
              unfused: the reduce-scatter per bucket, then the 16 owner updates). Grads
              N(0, 1e-3^2); master N(0, 0.02^2), m = v = 0 at the start.    (default)
  zero2_gpt2_small  the same on the GPT-2-small list, Nd = 8, buckets of 10,000,000.
  zero3_gpt2_small  ZeRO stage 3 on the GPT-2-small list, Nd = 8: the fp16 parameters live in
              8 partitions; a step gathers each of the 14 layers (embedding, 12 blocks, final
              LayerNorm) in forward order, then in backward order gathers each layer again and
              runs its fused update into the owners' partitions, then commits. The library's
              layer scheduler runs the gathers one layer ahead on a second stream into four
              layer buffers (--layer-buffers).
  zero3_1p3b  the same on the 1.3B list (26 layers), Nd = 16.
  gpt2_small  GPT-2-small parameter list (psi = 123,653,376), Nd = 8, stage 1 (full local
              gradients, one fused call per step); grads N(0, 1e-3^2) with 1% x100; master
              N(0, 0.02^2), m = v = 0 at the start.
  shard_7p5b  one owner's view of 7.5e9 parameters at Nd = 64: a 117,187,500-element shard,
              64 separate fp16 gradient slices, written into a 7.5e9-element fp16 buffer at
              r*S (r = 31); master U(-0.05, 0.05), m N(0, 1e-4^2), v |N(0, 1e-6^2)|.
  flat        psi = 2^29 flat buffer, one fused call per bucket of B elements in backward
              order, Nd in {2, 4, 8, 16, 64}; state as shard_7p5b.
  tiny        the 2^20-value stage-1 case (4 tensors, Nd = 4), L2-resident.

--payload q8: the owners reduce int8 records (128 values and their fp32 scale) instead of fp16
gradients, quantized once before timing (stage 1, flat, the 7.5B view, stage 2 through the
int8 bucket scheduler, stage 3 per owner part). --graph: each step is one CUDA-graph replay
(the step's constants read from device memory).

The default line also carries the bucket / Nd sweep ("sweep" in config: the flat workload at
Nd in {2, 4, 8, 16, 64} with 128 MiB buckets, each point timed the same way; --no-sweep skips
it). Every step reads and writes far more than the 126 MB L2 (76 GB for zero2_1p3b, 5.2 GB for
gpt2_small), so no L2 flush is needed between steps. With N > 1 (torchrun), every rank runs its own replica of the
simulated Nd-rank step on its own GPU (the Nd ranks are simulated on one device; no data
crosses GPUs), and the time is the maximum over ranks.
"""
from __future__ import annotations

import argparse
import datetime
import gc
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
L2_BYTES = 126 * 1024 * 1024    # B200 L2


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=["tiny", "gpt2_small", "shard_7p5b", "flat",
                                           "zero2_1p3b", "zero2_gpt2_small", "zero3_gpt2_small",
                                           "zero3_1p3b"],
                    default="zero2_1p3b")
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
    ap.add_argument("--stage2", choices=["fused", "unfused"], default="fused",
                    help="stage-2 workloads: the bucket scheduler launches the fused step per "
                         "bucket (zero_sched_create_fused), or the reduce-scatter per bucket "
                         "and then the owner updates")
    ap.add_argument("--replicas", type=int, default=0,
                    help="flat workload: the fused calls store the fp16 parameters into R replica "
                         "buffers (the all-gather in the epilogue, zero_step_fused_replicas)")
    ap.add_argument("--l2", choices=["warm", "flushed"], default="warm",
                    help="flushed: write a buffer larger than L2 between timed steps and time each "
                         "step on its own (for the L2-resident tiny workload)")
    ap.add_argument("--layer-buffers", type=int, default=4,
                    help="stage-3 workloads: layer buffers of the layer scheduler (>= 1)")
    ap.add_argument("--no-sweep", action="store_true",
                    help="leave out the bucket / Nd sweep of the default line")
    ap.add_argument("--sweep-steps", type=int, default=None)
    ap.add_argument("--no-overlap", action="store_true",
                    help="launch the per-bucket calls of a step strictly one after another "
                         "(default: inside a zero_overlap_begin/end region)")
    ap.add_argument("--e2e-steps", type=int, default=None)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    a = ap.parse_args()
    if a.warmup < 3:
        ap.error("--warmup must be >= 3")
    if a.replicas and (a.workload != "flat" or a.payload != "fp16" or a.graph):
        ap.error("--replicas takes the flat workload, fp16 payloads, eager calls")
    if not 0 <= a.replicas <= 64:
        ap.error("--replicas: 1 to 64")
    return a


# ---------------------------------------------------------------------------------------------
# workloads
# ---------------------------------------------------------------------------------------------
def workload_config(args) -> dict:
    """The workload's name and sizes as both arms report them (no device needed)."""
    from zero_partitioned_optimizer_plan_b200 import synth
    kind = args.workload
    if kind in ("gpt2_small", "tiny"):
        nd = args.nd or (8 if kind == "gpt2_small" else 4)
        numels = synth.gpt2_small_list() if kind == "gpt2_small" else synth.TINY_LIST
        cfg = {"workload": kind + "_stage1" if kind == "tiny" else "gpt2_small_stage1",
               "psi": sum(numels), "nd": nd, "stage": 1, "calls_per_step": 1,
               "tensors": len(numels)}
    elif kind == "shard_7p5b":
        nd = args.nd or 64
        total = 7_500_000_000
        cfg = {"workload": "shard_7p5b_rank31", "psi_total": total, "shard": total // nd,
               "nd": nd, "owner": 31, "calls_per_step": 1}
    elif kind in ("zero3_gpt2_small", "zero3_1p3b"):
        small = kind == "zero3_gpt2_small"
        nd = args.nd or (8 if small else 16)
        numels = synth.gpt2_small_list() if small else synth.gpt_1p3b_list()
        layers = synth.gpt2_small_layers() if small else synth.gpt_1p3b_layers()
        cfg = {"workload": kind, "psi": sum(numels), "nd": nd, "stage": 3,
               "layers": len(layers), "calls_per_step": None, "tensors": len(numels)}
        if args.payload == "q8":
            cfg["payload"] = "int8 records: 128 values and their fp32 scale, one segment per owner part"
            cfg["workload"] += "_q8"
        return cfg
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
        if args.stage2 == "fused":
            cfg["workload"] = kind + "_fused"
            cfg["calls_per_step"] = nb + 1
        cfg["overlap"] = not args.no_overlap
        if args.payload == "q8":
            cfg["payload"] = "int8 records: 128 values and their fp32 scale"
            cfg["workload"] += "_q8"
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
    if getattr(args, "replicas", 0):
        cfg["replicas"] = args.replicas
        cfg["workload"] += f"_rep{args.replicas}"
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
        self.e2e = None          # a workload-specific end-to-end leg (stage 2 fused)
        self.kernel_times = None  # per-step dominant-kernel time, when not the ev pair's
        self.replicas = []        # --replicas: the full parameter buffers the fused calls write
        self.time_calls = False   # record per-call events in this step (stage 3)
        if kind in ("gpt2_small", "tiny"):
            tiny = kind == "tiny"
            nd = args.nd or (4 if tiny else 8)
            numels = synth.TINY_LIST if tiny else synth.gpt2_small_list()
            pl = lz.zero_plan_create(numels, nd, 1, 0)
            psi, psi_p, S, nb = lz.zero_plan_info(pl)
            self.nd, self.n, self.psi = nd, psi_p, psi
            self.ranges = [(0, psi_p)]
            self.grads = []
            for r in range(nd):
                g = torch.zeros(psi_p, dtype=torch.float16, device=dev)
                if tiny:     # the tiny stage-1 case: N(0, 0.01^2) gradients, no spikes
                    synth.grad_f16(psi, 0.01, seed=0, rank=r, step=1, out=g[:psi])
                else:
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
        elif kind in ("zero3_gpt2_small", "zero3_1p3b"):
            self._init_zero3(args, dev)
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
            # --replicas R: the all-gather in the epilogue, into R full parameter buffers
            self.replicas = [self.params] + [torch.empty(psi, dtype=torch.float16, device=dev)
                                             for _ in range(args.replicas - 1)] \
                if args.replicas else []
        self.cur = [master, m, v]
        self.nxt = [torch.empty_like(x) for x in self.cur]
        self.state_a0 = self.cur[0].data_ptr()
        self.prepared = [None, None]                          # per ping-pong direction
        # algorithmic HBM bytes: with R replicas the fp16 write is 2 R bytes per value
        self.bytes_per_step = (2 * self.nd + 24 + 2 * max(1, len(self.replicas))) * self.n
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

    def outputs(self):
        """The step's result a host reads back: the fp16 parameters (stage 3: every owner's
        partition)."""
        return self.shards if self.kind.startswith("zero3") else [self.params]

    def inputs(self):
        """The tensors a step consumes that a host would have to upload."""
        if self.payload == "q8" and self.kind.startswith("zero3"):
            return [x for pays in self.q3 for x in pays]       # per layer, per rank
        if self.payload == "q8":
            return self.q
        return self.grads

    # --- CUDA-graph mode: the step's calls read the Adam constants from device memory -------
    def enable_graph(self, dynamic=False, max_steps=0):
        torch, lz = self.torch, self.lz
        dev = self.cur[0].device
        self.dynamic = dynamic
        nb_c = lz.ZERO_ADAM_CONSTS_BYTES
        self.d_consts = torch.empty(nb_c, dtype=torch.uint8, device=dev)
        self.h_consts = [torch.empty(nb_c, dtype=torch.uint8, pin_memory=True) for _ in range(2)]
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
        if self.replicas:
            grads = grads or self.grads
            if ev is not None:
                ev[0].record()
            if self.overlap:
                lz.zero_overlap_begin()
            for lo, hi in self.ranges:
                lz.zero_step_fused_replicas(hi - lo, self.nd, [g[lo:hi] for g in grads],
                                            *[x[lo:hi] for x in self.cur],
                                            *[x[lo:hi] for x in self.nxt],
                                            [r[lo:hi] for r in self.replicas], self.hp, t, status)
            if self.overlap:
                lz.zero_overlap_end()
            if ev is not None:
                ev[1].record()
            lz.zero_step_commit_replicas(self.n, *self.cur, *self.nxt, self.replicas, status)
            self.cur, self.nxt = self.nxt, self.cur
            return
        if grads is None and len(self.ranges) > 1:   # per-bucket calls, marshalled once
            self._step_prepared(t, status, ev)
            return
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


def _step_prepared(self, t, status, ev=None):
    """The per-bucket calls of a step as one zero_step_fused_ranges (int8 payloads:
    zero_step_fused_q8_ranges) call, its range descriptors marshalled once per ping-pong
    direction (a step's host cost is then one entry plus the launches, which matters for 1 MiB
    buckets)."""
    lz, torch = self.lz, self.torch
    d = 0 if self.cur[0].data_ptr() == self.state_a0 else 1
    if self.prepared[d] is None:
        nd = self.nd
        if self.payload == "q8":    # range i's payloads: self.q[i * nd:(i + 1) * nd]
            ins = [self.q[i * nd:(i + 1) * nd] for i in range(len(self.ranges))]
        else:
            ins = [[g[lo:hi] for g in self.grads] for lo, hi in self.ranges]
        self.prepared[d] = lz.PreparedStepRanges(nd, [
            (hi - lo, x, *[y[lo:hi] for y in self.cur], *[y[lo:hi] for y in self.nxt],
             self.params[lo:hi]) for (lo, hi), x in zip(self.ranges, ins)], self.payload)
    sh = lz.stream_handle(torch.cuda.current_stream())
    if ev is not None:
        ev[0].record()
    self.prepared[d](lz.hparams_ref(self.hp), t, lz.status_ptr(status), self.overlap, sh)
    if ev is not None:
        ev[1].record()
    lz.zero_step_commit(self.n, *self.cur, *self.nxt, self.params, status)
    self.cur, self.nxt = self.nxt, self.cur


def _init_zero2(self, args, dev):
    """Stage 2 on the 1.3B list (Nd = 16, buckets of 50,000,000 elements), or on the GPT-2-small
    list (Nd = 8, buckets of 10,000,000; a smaller case for profiling). The backward pass's
    output (every bucket's local gradients of every rank) is already in the scheduler's staging
    slots, one slot per bucket; a step runs the buckets in backward order through the
    scheduler: the fused step per bucket and one commit, or (--stage2 unfused) the
    reduce-scatter per bucket and then the owners' updates (zero_adam_shard). One scheduler
    serves every step; between steps it is rebound to the step's buffers and status word."""
    torch, lz = self.torch, self.lz
    from zero_partitioned_optimizer_plan_b200 import synth
    q8 = args.payload == "q8"
    if q8 and args.stage2 != "fused":
        raise SystemExit("the int8 payload takes the fused stage-2 scheduler")
    self.payload = args.payload
    small = args.workload == "zero2_gpt2_small"
    nd = args.nd or (8 if small else 16)
    B = args.bucket or (10_000_000 if small else 50_000_000)
    numels = synth.gpt2_small_list() if small else synth.gpt_1p3b_list()
    self.plan = pl = lz.zero_plan_create(numels, nd, 2, B)
    psi, psi_p, S, nb = lz.zero_plan_info(pl)
    self.nd, self.n, self.psi, self.S, self.nb = nd, psi_p, psi, S, nb
    self.buckets = [lz.zero_plan_bucket(pl, k)[:2] for k in range(nb)]
    if q8:
        # every bucket's int8 records of every rank, quantized once from the same gradients
        self.slot_elems = lz.zero_sched_slot_bytes_q8(pl, nb)
        self.slots = torch.empty(self.slot_elems, dtype=torch.uint8, device=dev)
        self.stride = self.slot_elems // (nb * nd)         # bytes per rank region
        tmp = torch.empty(max(ln for _, ln in self.buckets), dtype=torch.float16, device=dev)
        for k, (lo, ln) in enumerate(self.buckets):
            for r in range(nd):
                base = (k * nd + r) * self.stride
                synth.grad_f16(ln, 1e-3, seed=0, rank=r, step=1000 + k, out=tmp[:ln])
                lz.zero_quantize_q8(ln, tmp[:ln],
                                    self.slots[base:base + lz.q8_payload_bytes(ln)])
        del tmp
    else:
        self.slot_elems = lz.zero_sched_slot_elems(pl, nb)
        self.slots = torch.empty(self.slot_elems, dtype=torch.float16, device=dev)
        self.stride = self.slot_elems // (nb * nd)
        for k, (lo, ln) in enumerate(self.buckets):
            for r in range(nd):
                base = (k * nd + r) * self.stride
                synth.grad_f16(ln, 1e-3, seed=0, rank=r, step=1000 + k,
                               out=self.slots[base:base + ln])
    self.master, self.m, self.v = synth.state_small(psi_p, seed=0, device=dev)
    self.params = torch.empty(psi_p, dtype=torch.float16, device=dev)
    self.grads = None
    self.ranges = [(0, psi_p)]
    # the buckets' reduce-scatters (or fused steps) of a step touch disjoint ranges
    self.overlap = not args.no_overlap
    self.param_base = 0
    self.config = workload_config(args)
    assert (self.config["psi"], self.config["buckets"]) == (psi, nb)
    stream = torch.cuda.current_stream()
    self.st_create = torch.zeros(1, dtype=torch.int32, device=dev)   # rebound before each step
    if args.stage2 == "fused":
        # the scheduler launches the fused step per bucket; ping-pong state, commit at the end
        self.cur = [self.master, self.m, self.v]
        self.nxt = [torch.empty_like(x) for x in self.cur]
        nb_c = lz.ZERO_ADAM_CONSTS_BYTES
        self.d_consts = torch.empty(nb_c, dtype=torch.uint8, device=dev)
        self.h_consts = [torch.empty(nb_c, dtype=torch.uint8, pin_memory=True) for _ in range(2)]
        self.h_done = [None, None]
        if q8:
            self.sched = lz.zero_sched_create_fused_q8(pl, self.slots, self.slot_elems, nb,
                                                       *self.cur, *self.nxt, self.params,
                                                       self.d_consts, self.st_create, stream)
            self.bytes_per_step = (nd * sum(lz.q8_payload_bytes(ln) for _, ln in self.buckets)
                                   + 26 * psi_p)
            self.dominant = "fused_q8_tma_kernel"
        else:
            self.sched = lz.zero_sched_create_fused(pl, self.slots, self.slot_elems, nb,
                                                    *self.cur, *self.nxt, self.params,
                                                    self.d_consts, self.st_create, stream)
            self.bytes_per_step = (2 * nd + 26) * psi_p
            self.dominant = "fused_tma_kernel"
        self.dominant_bytes = self.bytes_per_step
        self.dominant_calls = nb
        self.side = None
        self.step = self._step_zero2_fused
        self.e2e = self._e2e_zero2_fused
        return
    self.shards = torch.empty(psi_p, dtype=torch.float32, device=dev)
    self.sched = lz.zero_sched_create(pl, self.slots, self.slot_elems, nb,
                                      [self.shards[r * S:(r + 1) * S] for r in range(nd)],
                                      self.st_create, stream)
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
        raise ValueError("the unfused stage-2 workload has no host-buffer variant")
    S, nd, sch = self.S, self.nd, self.sched
    stream = torch.cuda.current_stream()
    lz.zero_sched_rebind_status(sch, status)
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


def _step_zero2_fused(self, t, status, ev=None, grads=None):
    """Stage 2 with the fused step per bucket: the scheduler launches each bucket's fused
    kernel as the bucket arrives (its slot released after it), then one commit."""
    lz, torch = self.lz, self.torch
    if grads is not None:
        raise ValueError("use the workload's e2e() for host buffers")
    stream = torch.cuda.current_stream()
    sch = self.sched
    self._load_consts(t)
    lz.zero_sched_rebind_fused(sch, *self.cur, *self.nxt, self.params, status)
    if ev is not None:
        ev[0].record()
    begin = lz.zero_sched_begin_bucket_q8 if self.payload == "q8" else lz.zero_sched_begin_bucket
    if self.overlap:
        lz.zero_overlap_begin(stream)
    for k in range(self.nb):
        begin(sch, k, stream)
        lz.zero_sched_end_bucket(sch, k, stream)
    if self.overlap:
        lz.zero_overlap_end(stream)
    lz.zero_sched_wait(sch, stream)
    if ev is not None:
        ev[1].record()
    lz.zero_step_commit(self.n, *self.cur, *self.nxt, self.params, status)
    self.cur, self.nxt = self.nxt, self.cur


def _e2e_zero2_fused(self, t0, E, barrier, max_ms):
    """End to end through the C ABI with host buffers: every step uploads each bucket's Nd
    gradient slices from pinned host memory into a staging slot (two slots on the device; the
    upload of a bucket waits, on the upload stream, for the release of its slot by
    zero_sched_begin_bucket), the scheduler launches the bucket's fused step after the upload,
    then the commit; the fp16 parameters and the status word are downloaded and the host reads
    the status. The next step's uploads overlap this step's tail and download."""
    torch, lz = self.torch, self.lz
    dev, nd, pl = self.params.device, self.nd, self.plan
    q8 = self.payload == "q8"        # int8 records uploaded instead of fp16 gradients
    n_slots = 2
    if q8:
        slot_elems = lz.zero_sched_slot_bytes_q8(pl, n_slots)
        d_slots = torch.empty(slot_elems, dtype=torch.uint8, device=dev)
    else:
        slot_elems = lz.zero_sched_slot_elems(pl, n_slots)
        d_slots = torch.empty(slot_elems, dtype=torch.float16, device=dev)
    esize = d_slots.element_size()
    region = nd * self.stride
    # pinned host source: every bucket's gradients when the host has room (42 GB for the 1.3B
    # list at Nd = 16), else as many buckets as half the host's available memory allows per
    # rank, cycled (each step still uploads every bucket's bytes; only the source is reused)
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    try:
        import psutil
        avail = psutil.virtual_memory().available
    except Exception:
        avail = 0
    host_buckets = self.nb
    if avail and self.nb * region * esize > avail // (2 * ws):
        host_buckets = max(2, min(self.nb, (avail // (2 * ws)) // (region * esize)))
    total = host_buckets * region
    h_grads = pinned_host(total, d_slots.dtype)
    h_grads.copy_(self.slots[:total])          # the same gradients as the device-resident run
    h_params = [torch.empty(self.n, dtype=torch.float16, pin_memory=True) for _ in range(2)]
    h_status = [torch.empty(1, dtype=torch.int32, pin_memory=True) for _ in range(2)]
    st = torch.zeros(E, dtype=torch.int32, device=dev)
    main = torch.cuda.current_stream()
    up, down = torch.cuda.Stream(), torch.cuda.Stream()
    create = lz.zero_sched_create_fused_q8 if q8 else lz.zero_sched_create_fused
    begin = lz.zero_sched_begin_bucket_q8 if q8 else lz.zero_sched_begin_bucket
    sch = create(pl, d_slots, slot_elems, n_slots, *self.cur, *self.nxt, self.params,
                 self.d_consts, st[0:1], main)
    h2d = 0
    comp_done, down_done = [None, None], [None, None]
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
        t = t0 + i
        self._load_consts(t)
        lz.zero_sched_rebind_fused(sch, *self.cur, *self.nxt, self.params, st[i:i + 1])
        if down_done[1 - b] is not None:
            main.wait_event(down_done[1 - b])   # step i-1's parameters are downloaded
        if self.overlap:
            lz.zero_overlap_begin(main)
        for k, (lo, ln) in enumerate(self.buckets):
            ptrs = begin(sch, k, up)
            cnt = lz.q8_payload_bytes(ln) if q8 else ln       # elements of a rank's part
            with torch.cuda.stream(up):
                hk = k % host_buckets
                for r in range(nd):
                    off = (ptrs[r] - d_slots.data_ptr()) // esize
                    a = hk * region + r * self.stride
                    d_slots[off:off + cnt].copy_(h_grads[a:a + cnt], non_blocking=True)
                    h2d += esize * cnt if i == 0 else 0
            lz.zero_sched_end_bucket(sch, k, up)
        if self.overlap:
            lz.zero_overlap_end(main)
        lz.zero_sched_wait(sch, main)
        lz.zero_step_commit(self.n, *self.cur, *self.nxt, self.params, st[i:i + 1], main)
        self.cur, self.nxt = self.nxt, self.cur
        comp = torch.cuda.Event()
        comp.record(main)
        comp_done[b] = comp
        with torch.cuda.stream(down):
            down.wait_event(comp)
            h_params[b].copy_(self.params, non_blocking=True)
            h_status[b].copy_(st[i:i + 1], non_blocking=True)
            dd = torch.cuda.Event()
            dd.record(down)
            down_done[b] = dd
        if i > 0:
            read_result(i - 1)
    main.wait_event(down_done[(E - 1) % 2])
    e1.record(main)
    read_result(E - 1)
    torch.cuda.synchronize()
    lz.zero_sched_destroy(sch)
    ems = max_ms(e0.elapsed_time(e1))
    out = {"ms": ems, "steps": E, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": 2 * self.n + 4,
           "overlap": ("bucket uploads (int8 records) into two staging slots, each gated by the "
                       "release of its slot; the next step's uploads overlap this step's tail "
                       "and download") if q8 else
                      ("bucket uploads into two staging slots, each gated by the release of its "
                       "slot; the next step's uploads overlap this step's tail and download"),
           "host_source": (f"all {self.nb} buckets in pinned host memory" if host_buckets ==
                           self.nb else f"{host_buckets} buckets in pinned host memory, cycled")}
    unpin_host(h_grads)
    del h_grads, h_params, d_slots
    return out


def _owner_parts(lo: int, hi: int, shard: int):
    """The owner parts of the flat range [lo, hi), in owner order."""
    out, a = [], lo
    while a < hi:
        b = min(hi, (a // shard + 1) * shard)
        out.append((a, b))
        a = b
    return out


def _init_zero3(self, args, dev):
    """Stage 3 on a GPT-shaped list: every rank's full local gradient is resident (as the
    backward pass would leave it layer by layer); the fp16 parameters are Nd partitions of S
    values; the optimizer state is flat and ping-ponged. The library's layer scheduler gathers
    the layers on a second stream into --layer-buffers layer buffers. A step: every layer acquired in
    forward order (the next one prefetched), then per layer in backward order acquired again
    (the previous one prefetched), released, and updated (zero_stage3_step_fused), then
    zero_stage3_step_commit. Each fused call is timed with its own events in the last step."""
    torch, lz = self.torch, self.lz
    from zero_partitioned_optimizer_plan_b200 import synth
    q8 = args.payload == "q8"
    self.payload = args.payload
    small = args.workload == "zero3_gpt2_small"
    nd = args.nd or (8 if small else 16)
    numels = synth.gpt2_small_list() if small else synth.gpt_1p3b_list()
    split = synth.gpt2_small_layers() if small else synth.gpt_1p3b_layers()
    self.plan = pl = lz.zero_plan_create(numels, nd, 3, 0)
    psi, psi_p, S, _ = lz.zero_plan_info(pl)
    offs = lz.zero_plan_tensor_offsets(pl)
    self.layers, i = [], 0
    for c in split:
        self.layers.append((offs[i], offs[i + c - 1] + numels[i + c - 1]))
        i += c
    self.nd, self.n, self.psi, self.S = nd, psi_p, psi, S
    self.grads = []
    for r in range(nd):
        g = torch.zeros(psi_p, dtype=torch.float16, device=dev)
        synth.grad_f16(psi, 1e-3, seed=0, rank=r, step=1, out=g[:psi])
        self.grads.append(g)
    master, m, v = synth.state_small(psi_p, seed=0, device=dev)
    self.cur = [master, m, v]
    self.nxt = [torch.empty_like(x) for x in self.cur]
    self.shards = []
    for q in range(nd):
        part = torch.empty(S, dtype=torch.float16, device=dev)
        part.copy_(master[q * S:(q + 1) * S])
        self.shards.append(part)
    bounds = [lo for lo, _ in self.layers] + [self.layers[-1][1]]
    nb = args.layer_buffers
    elems = lz.zero_layer_sched_buf_elems(pl, bounds, nb)
    self.layer_mem = torch.empty(elems, dtype=torch.float16, device=dev)
    self.gather_stream = torch.cuda.Stream()
    self.layer_sched = lz.zero_layer_sched_create(pl, bounds, self.shards, self.layer_mem, elems,
                                                  nb, self.gather_stream)
    L = len(self.layers)
    mk = lambda: torch.cuda.Event(enable_timing=True)   # noqa: E731
    self.f_ev = [(mk(), mk()) for _ in range(L)]        # reused by the step that records them
    self.state_a0 = self.cur[0].data_ptr()
    self.layer_views = [None, None]
    self.prepared3 = [None, None]         # per ping-pong direction: the layers' update calls
    self.params = self.shards[0]          # (the e2e leg downloads every partition)
    self.ranges = [(0, psi_p)]
    self.overlap = False
    self.param_base = 0
    self.config = workload_config(args)
    n_fused = sum(((psi_p if l == len(self.layers) - 1 else hi) - 1) // S - lo // S + 1
                  for l, (lo, hi) in enumerate(self.layers))
    self.config["calls_per_step"] = 2 * len(self.layers) + n_fused + 1   # + one commit
    self.config["fused_calls_per_step"] = n_fused
    self.config["layer_buffers"] = nb
    gather_bytes = 2 * 4 * psi              # two gathers: 2 bytes read + 2 written each
    fused_bytes = (2 * nd + 26) * psi_p
    self.dominant = "fused_tma_kernel"
    self.q3 = None
    if q8:
        # every layer's int8 payload of every rank (one segment per owner part), quantized once
        self.q3, pay_bytes = [], 0
        for l, (lo, hi) in enumerate(self.layers):
            ghi = psi_p if l == L - 1 else hi
            nbytes = lz.zero_stage3_payload_bytes_q8(pl, lo, ghi - lo)
            pays = [torch.empty(nbytes, dtype=torch.uint8, device=dev) for _ in range(nd)]
            for r in range(nd):
                lz.zero_stage3_quantize_q8(pl, lo, ghi - lo, self.grads[r][lo:ghi], pays[r])
            self.q3.append(pays)
            pay_bytes += sum(lz.q8_payload_bytes(b - a) for a, b in
                             _owner_parts(lo, ghi, S)) * nd
        fused_bytes = pay_bytes + 26 * psi_p
        self.dominant = "fused_q8_tma_kernel"
    self.bytes_per_step = gather_bytes + fused_bytes
    self.dominant_bytes = fused_bytes
    self.dominant_calls = n_fused
    self.fused_evs = []
    self.side = None                      # the gathers run inside the layer scheduler
    self.step = self._step_zero3
    self.kernel_times = self._kernel_times_zero3


def _step_zero3(self, t, status, ev=None, grads=None):
    """One stage-3 step through the library's layer scheduler: the gathers run on its gather
    stream one layer ahead of the main stream (forward, then backward); each layer's update on
    the main stream follows its release. The backward gather of layer l-1 runs beside layer l's
    update (disjoint ranges of the partitions); the next step's gathers wait for this step's
    commit (zero_layer_sched_begin_step)."""
    lz, torch = self.lz, self.torch
    pl, shards, L, sch = self.plan, self.shards, len(self.layers), self.layer_sched
    if self.q3 is not None:   # int8: the step's inputs are the layers' payloads (inputs())
        pays = self.q3 if grads is None else \
            [grads[l * self.nd:(l + 1) * self.nd] for l in range(L)]
        grads = self.grads    # only the state views of _layer_args are used then
    grads = grads or self.grads
    main = torch.cuda.current_stream()
    # per-call events only in the step that run_ours marks (the last timed one): recording
    # events around every call of every step doubled the host's work per step, which at
    # GPT-2-small sizes then set the step's pace
    timed = ev is not None and self.time_calls
    f_pairs = []
    if ev is not None:
        ev[0].record(main)
    lz.zero_layer_sched_begin_step(sch, status, main)
    for l in range(L):                        # forward: the layer's computation would go here
        lz.zero_layer_sched_acquire(sch, l, l + 1 if l + 1 < L else -1, main)
        lz.zero_layer_sched_release(sch, l, main)
    # the layers' updates touch disjoint ranges: one overlap region on the main stream (event
    # waits and records are allowed inside; an event recorded after an update completes only
    # when every update before it has)
    prepared = self._layer_updates() if grads is self.grads and self.q3 is None else None
    hp_ref, st_ptr, sh = lz.hparams_ref(self.hp), lz.status_ptr(status), lz.stream_handle(main)
    lz.zero_overlap_begin(main)
    for l in range(L - 1, -1, -1):
        lo, _ = self.layers[l]
        lz.zero_layer_sched_acquire(sch, l, l - 1, main)
        lz.zero_layer_sched_release(sch, l, main)
        if timed:
            e = self.f_ev[len(f_pairs)]
            e[0].record(main)
        if prepared is not None:
            prepared[l](hp_ref, t, st_ptr, sh)
        elif self.q3 is not None:          # the owners' update from the int8 payloads
            n, _, *state = self._layer_args(l, grads)
            lz.zero_stage3_step_fused_q8(pl, lo, n, pays[l], *state, shards, self.hp, t,
                                         status, main)
        else:
            lz.zero_stage3_step_fused(pl, lo, *self._layer_args(l, grads), shards, self.hp, t,
                                      status, main)
        if timed:
            e[1].record(main)
            f_pairs.append(e)
    lz.zero_overlap_end(main)
    lz.zero_stage3_step_commit(pl, *self.cur, *self.nxt, shards, status, main)
    if ev is not None:
        ev[1].record(main)
    if timed:
        self.fused_evs.append(list(f_pairs))
    self.cur, self.nxt = self.nxt, self.cur


def _layer_args(self, l, grads):
    """(length, rank gradients, state in, state out) views of layer l's gradient bucket, made
    once per ping-pong direction (the padding rides with the last layer)."""
    if grads is not self.grads:
        lo, hi = self.layers[l]
        ghi = self.n if l == len(self.layers) - 1 else hi
        return (ghi - lo, [g[lo:ghi] for g in grads], *[x[lo:ghi] for x in self.cur],
                *[x[lo:ghi] for x in self.nxt])
    d = 0 if self.cur[0].data_ptr() == self.state_a0 else 1
    if self.layer_views[d] is None:
        views = []
        for k, (lo, hi) in enumerate(self.layers):
            ghi = self.n if k == len(self.layers) - 1 else hi
            views.append((ghi - lo, [g[lo:ghi] for g in self.grads],
                          *[x[lo:ghi] for x in self.cur], *[x[lo:ghi] for x in self.nxt]))
        self.layer_views[d] = views
    return self.layer_views[d][l]


def _enable_graph_zero3(self):
    """Capture the stage-3 step once per ping-pong direction as a CUDA graph on one capture
    stream: the layer scheduler's gathers (on its gather stream), the layers' updates with the
    step's constants in device memory (zero_stage3_step_fused_dc, or _q8_dc from the int8
    payloads), the commit. A replay needs no host work but the constants' copy."""
    torch, lz = self.torch, self.lz
    dev = self.cur[0].device
    self.dynamic = False
    nb_c = lz.ZERO_ADAM_CONSTS_BYTES
    self.d_consts = torch.empty(nb_c, dtype=torch.uint8, device=dev)
    self.h_consts = [torch.empty(nb_c, dtype=torch.uint8, pin_memory=True) for _ in range(2)]
    self.h_done = [None, None]
    self.g_status = torch.zeros(1, dtype=torch.int32, device=dev)
    self.g_flags = torch.zeros(1, dtype=torch.int32, device=dev)
    cap = torch.cuda.Stream()
    pl, sch, L, shards = self.plan, self.layer_sched, len(self.layers), self.shards

    def body(src, dst):
        self.g_status.zero_()
        lz.zero_layer_sched_begin_step(sch, self.g_status, cap)
        for l in range(L):
            lz.zero_layer_sched_acquire(sch, l, l + 1 if l + 1 < L else -1, cap)
            lz.zero_layer_sched_release(sch, l, cap)
        lz.zero_overlap_begin(cap)
        for l in range(L - 1, -1, -1):
            lo, hi = self.layers[l]
            ghi = self.n if l == L - 1 else hi
            lz.zero_layer_sched_acquire(sch, l, l - 1, cap)
            lz.zero_layer_sched_release(sch, l, cap)
            if self.q3 is not None:
                lz.zero_stage3_step_fused_q8_dc(pl, lo, ghi - lo, self.q3[l],
                                                *[x[lo:ghi] for x in src],
                                                *[x[lo:ghi] for x in dst], shards, self.d_consts,
                                                self.g_status, cap)
            else:
                lz.zero_stage3_step_fused_dc(pl, lo, ghi - lo, [g[lo:ghi] for g in self.grads],
                                             *[x[lo:ghi] for x in src],
                                             *[x[lo:ghi] for x in dst], shards, self.d_consts,
                                             self.g_status, cap)
        lz.zero_overlap_end(cap)
        lz.zero_stage3_step_commit(pl, *src, *dst, shards, self.g_status, cap)
        self.g_flags.bitwise_or_(self.g_status)

    a, b = self.cur, self.nxt
    self._load_consts(1)
    cap.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(cap):
        body(a, b)                  # first use outside the capture
    torch.cuda.current_stream().wait_stream(cap)
    torch.cuda.synchronize()
    self.graphs = []
    for src, dst in ((a, b), (b, a)):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=cap):
            body(src, dst)
        self.graphs.append(g)
    self.g_flags.zero_()
    self.graph_dir = 0
    self.step = self._graph_step
    self.kernel_times = None          # the replay's events: the whole step
    self.dominant = "stage-3 step graph (gathers, fused layer updates, commit)"
    self.dominant_bytes = self.bytes_per_step
    self.dominant_calls = 1
    self.graph_launches = 2 * L + self.config["fused_calls_per_step"] + 1


def _layer_updates(self):
    """Each layer's zero_stage3_step_fused call for the current ping-pong direction, its
    arguments marshalled once (PreparedStage3Update)."""
    d = 0 if self.cur[0].data_ptr() == self.state_a0 else 1
    if self.prepared3[d] is None:
        self.prepared3[d] = [
            self.lz.PreparedStage3Update(self.plan, lo, *self._layer_args(l, self.grads),
                                         self.shards)
            for l, (lo, _) in enumerate(self.layers)]
    return self.prepared3[d]


def _kernel_times_zero3(self, evs):
    """Per step: the fused calls' summed durations (ms). Only the last timed step records
    per-call events (time_calls): its durations stand for each timed step."""
    last = sum(a.elapsed_time(b) for a, b in self.fused_evs[-1])
    return [last] * len(evs)


Workload._init_zero3 = _init_zero3
Workload._step_zero3 = _step_zero3
Workload._kernel_times_zero3 = _kernel_times_zero3
Workload._layer_args = _layer_args
Workload._layer_updates = _layer_updates
Workload._enable_graph_zero3 = _enable_graph_zero3
Workload._step_prepared = _step_prepared
Workload._init_zero2 = _init_zero2
Workload._step_zero2 = _step_zero2
Workload._step_zero2_fused = _step_zero2_fused
Workload._e2e_zero2_fused = _e2e_zero2_fused


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
    """One hash over the sources of `kernel` and the build script that holds its compiler
    flags and geometry macros (the code the ncu counters describe)."""
    h = hashlib.sha256()
    for name in KERNEL_SOURCES[kernel]:
        with open(os.path.join(CSRC, name), "rb") as f:
            h.update(name.encode() + b"\0" + f.read())
    with open(os.path.join(os.path.dirname(CSRC), "build.py"), "rb") as f:
        h.update(b"build.py\0" + f.read())
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


def oracle_sample(nd: int, n: int, payload: str = "fp16", seed=0):
    """The oracle's owner step on n elements of the workload's distribution: a function
    step(master, m, v, t) -> (master, m, v) and the initial state. With the int8 payload the
    ranks' records are quantized once here (the senders' part), the step reduces them."""
    import oracle
    from zero_partitioned_optimizer_plan_b200 import synth
    g = [synth.grad_f16(n, 1e-3, seed=seed, rank=r, step=1, spike_frac=0.01,
                        spike_scale=100.0).numpy() for r in range(nd)]
    state = tuple(x.numpy() for x in synth.state_small(n, seed=seed))
    hp = oracle.AdamHP()
    if payload == "q8":
        q = [oracle.quant_q8(x) for x in g]
        qs, scs = [a for a, _ in q], [b for _, b in q]

        def step(w, mm, vv, t):
            _, w, mm, vv, _ = oracle.step_q8(qs, scs, w, mm, vv, hp, t)
            return w, mm, vv
    else:
        def step(w, mm, vv, t):
            _, w, mm, vv, _ = oracle.step(g, w, mm, vv, hp, t)
            return w, mm, vv
    return step, state


def cpu_oracle_rate(nd: int, n_sample: int, target_s: float, seed=0, payload: str = "fp16"):
    """Time the oracle (single-threaded C, as it stands) on n_sample elements of the workload's
    distribution; repeat until target_s seconds have passed. Returns (params/s, reps, secs)."""
    step, (master, m, v) = oracle_sample(nd, n_sample, payload, seed)
    reps, total = 0, 0.0
    while total < target_s and reps < 50:
        t0 = time.perf_counter()
        master, m, v = step(master, m, v, reps + 1)
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


def pinned_host(n: int, dtype):
    """A host tensor of exactly n elements, page-locked with cudaHostRegister (torch's pinned
    allocator rounds a request up to a power of two: 42 GB would take 64 GB)."""
    import torch
    t = torch.empty(n, dtype=dtype)
    err = torch.cuda.cudart().cudaHostRegister(t.data_ptr(), t.numel() * t.element_size(), 0)
    if int(err) != 0:
        raise RuntimeError(f"cudaHostRegister of {t.numel() * t.element_size()} bytes failed "
                           f"({int(err)})")
    return t


def unpin_host(t):
    import torch
    torch.cuda.cudart().cudaHostUnregister(t.data_ptr())


def e2e_resident_inputs(wl, t0, E, barrier, max_ms):
    """End to end for the workloads whose inputs are whole device tensors: the upload of step
    i+1 overlaps step i's compute and download (double-buffered device gradients; copies on
    their own streams, ordered by events)."""
    import torch
    dev = wl.params.device
    h_grads = [torch.empty(g.numel(), dtype=g.dtype, pin_memory=True) for g in wl.inputs()]
    for h, g in zip(h_grads, wl.inputs()):
        h.copy_(g)
    outs = wl.outputs()
    h_params = [[torch.empty(o.numel(), dtype=o.dtype, pin_memory=True) for o in outs]
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
        wl.step(t0 + i, st[i:i + 1], grads=d_grads[b])
        comp_done[b] = ev()
        comp_done[b].record(main)
        with torch.cuda.stream(down):
            down.wait_event(comp_done[b])
            for h, o in zip(h_params[b], outs):
                h.copy_(o, non_blocking=True)
            h_status[b].copy_(st[i:i + 1], non_blocking=True)
            down_done[b] = ev()
            down_done[b].record(down)
        if i > 0:
            read_result(i - 1)
    main.wait_event(down_done[(E - 1) % 2])
    e1.record(main)
    read_result(E - 1)
    torch.cuda.synchronize()
    return {"ms": max_ms(e0.elapsed_time(e1)), "steps": E,
            "h2d_bytes_per_step": sum(h.numel() * h.element_size() for h in h_grads),
            "d2h_bytes_per_step": sum(o.numel() * o.element_size() for o in outs) + 4,
            "overlap": "upload of step i+1 overlaps compute and download of step i"}


SWEEP_ND = (2, 4, 8, 16, 64)
SWEEP_PSI = 1 << 29
SWEEP_BUCKET = 1 << 26      # 128 MiB of fp16 per rank


def run_sweep(args, dev, ws, barrier):
    """The bucket / Nd sweep on the flat workload (psi = 2^29, 128 MiB buckets, one fused call
    per bucket in backward order inside an overlap region, then the commit), each point timed
    like the main line (CUDA events on the stream, max over ranks); the point's buffers are
    freed before the next."""
    import copy

    import torch
    peak, _ = measured_peak()
    K = args.sweep_steps or max(5, min(args.steps, 20))
    W = 3
    out = []
    for nd in SWEEP_ND:
        a = copy.copy(args)
        a.workload, a.nd, a.psi, a.bucket, a.payload = "flat", nd, SWEEP_PSI, SWEEP_BUCKET, "fp16"
        wl = Workload(a, dev)
        status = torch.zeros(K + W, dtype=torch.int32, device=dev)
        for i in range(W):
            wl.step(i + 1, status[i:i + 1])
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(K)]
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        barrier()
        start.record()
        for i in range(K):
            wl.step(W + i + 1, status[W + i:W + i + 1], ev=evs[i])
        end.record()
        torch.cuda.synchronize()
        if int((status != 0).sum().item()):
            raise RuntimeError(f"unexpected status flags in the sweep at Nd={nd}")
        ms = max_over_ranks(start.elapsed_time(end), ws, dev) / K
        kms = max_over_ranks(statistics.mean(x.elapsed_time(y) for x, y in evs), ws, dev)
        gbs = wl.bytes_per_step / (kms / 1e3) / 1e9
        out.append({"nd": nd, "psi": SWEEP_PSI, "bucket": SWEEP_BUCKET,
                    "calls_per_step": len(wl.ranges), "steps": K, "ms_per_step": ms,
                    "params_per_s": aggregate_rate(ws, wl.n, 1, ms),
                    "kernel_gbs": gbs, "frac": gbs / peak,
                    "bytes_per_step": wl.bytes_per_step})
        if ws == 1 and not args.no_cpu_baseline:   # the oracle at this Nd, a short sample
            rate, reps, secs = cpu_oracle_rate(nd, 1_000_000, 2.0)
            out[-1]["cpu_oracle_params_per_s"] = rate
            out[-1]["cpu_oracle_sample"] = f"1,000,000 elements, {reps} steps, {secs:.1f} s, 1 core"
        del wl, status
        gc.collect()
        torch.cuda.empty_cache()
    return out


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
    payload = getattr(args, "payload", "fp16")
    rate, _, _ = cpu_oracle_rate(nd, 200_000, 0.2, payload=payload)
    per_step_s = max(0.05, 120.0 / (args.steps + args.warmup))
    n_sample = int(min(16_000_000, max(100_000, rate * per_step_s)))
    step, (master, m, v) = oracle_sample(nd, n_sample, payload)
    for t in range(1, args.warmup + 1):
        master, m, v = step(master, m, v, t)
    t0 = time.perf_counter()
    for t in range(args.warmup + 1, args.warmup + args.steps + 1):
        master, m, v = step(master, m, v, t)
    dt = time.perf_counter() - t0
    value = n_sample * args.steps / dt
    sample = (f"first {n_sample} elements of the {cfg['workload']} workload's gradient "
              f"distribution, Nd={nd}, one oracle step per timed step"
              + (" (int8 records quantized once before timing)" if payload == "q8" else ""))
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
    if args.graph and wl.kind.startswith("zero3"):
        if args.dynamic_scale:
            raise SystemExit("--dynamic-scale applies to the stage-1 and flat workloads")
        wl._enable_graph_zero3()
    elif args.graph:
        if wl.grads is None and wl.payload != "q8":
            raise SystemExit("--graph applies to the stage-1, stage-3 and flat workloads")
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
    flushed = args.l2 == "flushed"
    if flushed:   # a buffer twice the L2 written between steps; each step timed on its own
        flush_buf = torch.empty(2 * L2_BYTES // 4, dtype=torch.int32, device=dev)
        sevs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                for _ in range(K)]
    sampler = ClockSampler(local)
    barrier()
    torch.cuda.synchronize()
    launches0 = lz.zero_kernel_launches()
    with sampler:
        start.record()
        for i in range(K):
            if flushed:
                flush_buf.fill_(i)
                sevs[i][0].record()
            wl.time_calls = i == K - 1
            wl.step(W + i + 1, status[W + i:W + i + 1], ev=evs[i])
            if flushed:
                sevs[i][1].record()
        end.record()
        torch.cuda.synchronize()
    launches = lz.zero_kernel_launches() - launches0
    if args.graph:   # replays launch the captured kernels without the host library
        launches = K * getattr(wl, "graph_launches",
                               len(wl.ranges) + 1 + (2 if args.dynamic_scale else 0))
        if int(wl.g_flags.item()) != 0:
            raise RuntimeError(f"unexpected status flags in the timed steps: {wl.g_flags.item()}")
    barrier()
    ms = sum(a.elapsed_time(b) for a, b in sevs) if flushed else start.elapsed_time(end)
    kernel_ms = wl.kernel_times(evs) if wl.kernel_times else [a.elapsed_time(b) for a, b in evs]
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
        def dur(x):    # one (start, end) pair per step, or a list of pairs (one per call)
            return x[0].elapsed_time(x[1]) if isinstance(x, tuple) else \
                sum(a.elapsed_time(b) for a, b in x)
        side_s = statistics.mean(dur(x) for x in wl.side["ms"][-K:]) / 1e3
        roofline["other"] = {"kernel": wl.side["kernel"],
                             "achieved": wl.side["bytes"] / side_s / 1e9,
                             "frac": wl.side["bytes"] / side_s / 1e9 / peak,
                             "ms_per_step": side_s * 1e3}

    # end to end through the public API with host buffers: every step uploads its gradients
    # from pinned host memory, runs, and downloads the updated fp16 parameters and its status
    # word, which the host reads.
    e2e = None
    if not args.no_e2e and not args.graph and (wl.e2e is not None or wl.inputs() is not None):
        E = args.e2e_steps or max(3, min(K, 10))
        mx = lambda ms: max_over_ranks(ms, ws, dev)   # noqa: E731
        if wl.e2e is not None:
            r = wl.e2e(W + K + 1, E, barrier, mx)
        else:
            r = e2e_resident_inputs(wl, W + K + 1, E, barrier, mx)
        e2e = {"value": aggregate_rate(ws, wl.n, r["steps"], r["ms"]), "unit": "params/s",
               **{k: v for k, v in r.items() if k != "ms"}}

    cpu = None
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        n_sample = 8_000_000
        rate, reps, secs = cpu_oracle_rate(wl.nd, n_sample, 10.0, payload=wl.payload)
        what = ("the oracle's int8 owner step, records quantized once before timing"
                if wl.payload == "q8" else "the oracle's step is the same element arithmetic "
                "for every stage and bucketing")
        cpu = {"value": rate, "unit": "params/s", "cores": 1, "kind": "oracle",
               "sample": f"{n_sample} elements with the workload's gradient distribution, "
                         f"Nd={wl.nd}, {reps} oracle steps, {secs:.1f} s ({what})",
               "host": host_cpu()}

    main_line = wl.config["workload"].startswith("zero2_1p3b") and args.stage2 == "fused" and \
        not args.graph and args.payload == "fp16"
    sweep = None
    if main_line and not args.no_sweep:
        cfg0, nd0, bytes0 = dict(wl.config), wl.nd, wl.bytes_per_step
        del wl
        gc.collect()            # a workload refers to itself through its bound step method
        torch.cuda.empty_cache()
        sweep = run_sweep(args, dev, ws, barrier)
    else:
        cfg0, nd0, bytes0 = dict(wl.config), wl.nd, wl.bytes_per_step

    if rank == 0:
        cfg = cfg0
        if args.graph:
            cfg["cuda_graph"] = "one replay per step; kernel time includes the commit"
            if args.dynamic_scale:
                cfg["loss_scale"] = "dynamic, on the device (scaler kernels inside the graph)"
        if flushed:
            l2 = (f"flushed: {2 * L2_BYTES >> 20} MiB written between steps, each step timed "
                  "on its own (the flush outside the timed steps)")
        elif bytes0 > 4 * L2_BYTES:
            l2 = "no flush: every step streams several GB, far above L2"
        else:
            l2 = "warm: the step's buffers stay in L2 across steps (no flush)"
        cfg.update({"l2": l2,
                    "bytes_per_step": bytes0, "parallelism": f"replicas{ws}",
                    "hbm_gbs": bytes0 / (ms_per_step / 1e3) / 1e9})
        if sweep is not None:
            cfg["sweep"] = sweep
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
