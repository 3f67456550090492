"""CPU oracle for the ZeRO stage-1/2 data-parallel step (TEST INFRASTRUCTURE ONLY).

Only tests/, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may import
this package. It never imports the CUDA library and the library never imports it; they share
only the seeded input generators, which hold none of the method's arithmetic.

The element arithmetic is plain C (``oracle.c``, built by ``oracle/build.py``); this module
adds the partitioning that ZeRO-DP performs around it, written with numpy slicing:

* ``dp_step``      -- plain data parallelism: every replica all-reduces the full gradient and
                      updates the full model ("ZeRO: particionar estados do treino entre GPUs",
                      section "Como funciona": the baseline DP keeps a full replica).
* ``zero1_step``   -- stage 1 (Pos): full local gradients, one reduce-scatter at the step, each
                      owner updates its 1/Nd shard, an all-gather writes every updated fp16
                      shard back ("Como funciona"; "ZeRO-2" card, "ZeRO-1에서 남은 낭비").
* ``zero2_step``   -- stage 2 (Pos+g): buckets in backward order, each reduce-scattered as soon
                      as it is produced, the owner keeps its slice and the rest is released;
                      then the owner update and the all-gather ("ZeRO-2" card, "Gradient
                      생명주기" and "왜 all-gather는 그대로 필요한가").
* ``zero3_step``   -- stage 3 (Pos+g+p): the fp16 parameters are partitioned as well; each
                      layer's parameters are gathered just in time in the forward pass and again
                      in the backward pass, each layer's gradient is reduce-scattered, and the
                      owners update their partitions ("Como funciona": 16 psi/Nd, 3 psi of
                      communication; "ZeRO" (lastdictionary), main definition).

All four produce the same numbers ("ZeRO" (lastdictionary), "Usage note": ZeRO changes where
state is stored, not how updates are computed); the pins in tests/test_oracle_pins.py check it.

Parity status: every function here is pinned (see tests/test_oracle_pins.py).
"""
from __future__ import annotations

import ctypes as C
import dataclasses
import os
from typing import Callable, List, Sequence

import numpy as np

from . import build as _build

_lib = None

SKIPPED = 1


def lib():
    """Load (building first if needed) the oracle's shared library."""
    global _lib
    if _lib is None:
        _lib = bind(_build.build())
    return _lib


def bind(path: str):
    """Open a build of oracle.c and declare its C signatures."""
    L = C.CDLL(path)
    u64, i64, f32p, u16p = C.c_uint64, C.c_int64, C.POINTER(C.c_float), C.POINTER(C.c_uint16)
    L.orc_h2f.argtypes, L.orc_h2f.restype = [C.c_uint16], C.c_float
    L.orc_f2h.argtypes, L.orc_f2h.restype = [C.c_float], C.c_uint16
    L.orc_h2f_array.argtypes = [u64, u16p, f32p]
    L.orc_f2h_array.argtypes = [u64, f32p, u16p]
    L.orc_state_bytes.argtypes = [u64, C.c_int, C.c_int, C.POINTER(u64), C.POINTER(u64)]
    L.orc_plan.argtypes = [C.POINTER(u64), C.c_int, C.c_int, u64, C.POINTER(u64),
                           C.POINTER(u64), C.POINTER(u64), C.POINTER(u64), C.POINTER(i64)]
    L.orc_bucket.argtypes = [u64, u64, i64, C.POINTER(u64), C.POINTER(u64)]
    L.orc_adam_scalars.argtypes = [C.c_void_p, i64, C.c_void_p]
    L.orc_reduce_mean.argtypes = [u64, C.c_int, C.POINTER(u16p), f32p]
    L.orc_all_finite.argtypes, L.orc_all_finite.restype = [u64, f32p], C.c_int
    L.orc_adam.argtypes = [u64, f32p, f32p, f32p, f32p, u16p, C.c_void_p]
    L.orc_step.argtypes = [u64, C.c_int, C.POINTER(u16p), f32p, f32p, f32p, u16p,
                           C.c_void_p, i64, f32p]
    i8p = C.POINTER(C.c_int8)
    L.orc_quant_q8.argtypes = [u64, u16p, i8p, f32p]
    L.orc_reduce_mean_q8.argtypes = [u64, C.c_int, C.POINTER(i8p), C.POINTER(f32p), f32p]
    L.orc_reduce_mean_q8_gathered.argtypes = [u64, C.c_int, C.POINTER(i8p), C.POINTER(f32p), f32p]
    return L


class _HP(C.Structure):
    _fields_ = [("lr", C.c_double), ("beta1", C.c_double), ("beta2", C.c_double),
                ("eps", C.c_double), ("loss_scale", C.c_double)]


class _Scalars(C.Structure):
    _fields_ = [(k, C.c_float) for k in
                ("b1", "omb1", "b2", "omb2", "step_size", "bc2s", "eps", "loss_scale")]


@dataclasses.dataclass(frozen=True)
class AdamHP:
    """Adam hyperparameters and the static loss scale (defaults: the tiny stage-1 workload)."""
    lr: float = 1e-3
    beta1: float = 0.9
    beta2: float = 0.999
    eps: float = 1e-8
    loss_scale: float = 1024.0

    def _c(self) -> _HP:
        return _HP(self.lr, self.beta1, self.beta2, self.eps, self.loss_scale)


def _f32p(a):
    return a.ctypes.data_as(C.POINTER(C.c_float))


def _u16p(a):
    return a.ctypes.data_as(C.POINTER(C.c_uint16))


def _as_u16(a) -> np.ndarray:
    a = np.asarray(a)
    if a.dtype == np.float16:
        a = a.view(np.uint16)
    assert a.dtype == np.uint16, a.dtype
    return np.ascontiguousarray(a)


# ---------------------------------------------------------------------------------------------
# binary16 conversion
# ---------------------------------------------------------------------------------------------
def h2f(h) -> np.ndarray:
    h = _as_u16(h)
    out = np.empty(h.shape, np.float32)
    lib().orc_h2f_array(h.size, _u16p(h), _f32p(out))
    return out


def f2h(x) -> np.ndarray:
    """binary32 -> binary16 bits (uint16), round to nearest even."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.shape, np.uint16)
    lib().orc_f2h_array(x.size, _f32p(x), _u16p(out))
    return out


# ---------------------------------------------------------------------------------------------
# accounting and plan
# ---------------------------------------------------------------------------------------------
STAGES = ("dp", "pos", "pos_g", "pos_g_p")


def state_bytes(psi: int, nd: int, K: int = 12) -> dict:
    """Per-device bytes of each stage and the per-step communication volume (elements)."""
    b = (C.c_uint64 * 16)()
    c = (C.c_uint64 * 4)()
    rc = lib().orc_state_bytes(psi, nd, K, b, c)
    if rc:
        raise ValueError("orc_state_bytes: invalid arguments")
    out = {}
    for s, name in enumerate(STAGES):
        out[name] = dict(params=b[4 * s], grads=b[4 * s + 1], optim=b[4 * s + 2],
                         total=b[4 * s + 3], comm_elems=c[s])
    return out


@dataclasses.dataclass
class Plan:
    numels: List[int]
    nd: int
    bucket_elems: int
    tensor_off: List[int]
    psi: int
    psi_p: int
    shard: int
    buckets: List[tuple]   # (lo, len) in backward order: bucket 0 is produced first

    def owners(self, k: int) -> tuple:
        lo, ln = self.buckets[k]
        return lo // self.shard, (lo + ln - 1) // self.shard


def plan(numels: Sequence[int], nd: int, bucket_elems: int = 0) -> Plan:
    n = len(numels)
    arr = (C.c_uint64 * max(n, 1))(*numels)
    off = (C.c_uint64 * max(n, 1))()
    psi, psi_p, shard = C.c_uint64(), C.c_uint64(), C.c_uint64()
    nb = C.c_int64()
    rc = lib().orc_plan(arr, n, nd, bucket_elems, off, C.byref(psi), C.byref(psi_p),
                        C.byref(shard), C.byref(nb))
    if rc:
        raise ValueError("orc_plan: invalid arguments")
    buckets = []
    for k in range(nb.value):
        lo, ln = C.c_uint64(), C.c_uint64()
        if lib().orc_bucket(psi_p.value, bucket_elems, k, C.byref(lo), C.byref(ln)):
            raise ValueError("orc_bucket failed")
        buckets.append((lo.value, ln.value))
    return Plan(list(numels), nd, bucket_elems, list(off[:n]), psi.value, psi_p.value,
                shard.value, buckets)


# ---------------------------------------------------------------------------------------------
# element arithmetic
# ---------------------------------------------------------------------------------------------
def adam_scalars(hp: AdamHP, t: int) -> dict:
    s = _Scalars()
    h = hp._c()
    if lib().orc_adam_scalars(C.byref(h), t, C.byref(s)):
        raise ValueError("step t must be >= 1")
    return {k: getattr(s, k) for k, _ in _Scalars._fields_}


def reduce_mean(grads: Sequence[np.ndarray]) -> np.ndarray:
    """Rank-ordered binary32 mean of Nd fp16 gradients (given as float16 or uint16 arrays)."""
    gs = [_as_u16(g) for g in grads]
    n = gs[0].size
    assert all(g.size == n for g in gs)
    ptrs = (C.POINTER(C.c_uint16) * len(gs))(*[_u16p(g) for g in gs])
    red = np.empty(n, np.float32)
    lib().orc_reduce_mean(n, len(gs), ptrs, _f32p(red))
    return red


def all_finite(x: np.ndarray) -> bool:
    x = np.ascontiguousarray(x, dtype=np.float32)
    return bool(lib().orc_all_finite(x.size, _f32p(x)))


def adam(red, master, m, v, hp: AdamHP, t: int):
    """Owner update from reduced gradients; returns new (master, m, v, p16) copies."""
    s = _Scalars()
    h = hp._c()
    if lib().orc_adam_scalars(C.byref(h), t, C.byref(s)):
        raise ValueError("step t must be >= 1")
    red = np.ascontiguousarray(red, np.float32)
    w, mm, vv = (np.array(a, dtype=np.float32, copy=True) for a in (master, m, v))
    p16 = np.empty(red.size, np.uint16)
    lib().orc_adam(red.size, _f32p(red), _f32p(w), _f32p(mm), _f32p(vv), _u16p(p16),
                   C.byref(s))
    return w, mm, vv, p16


def step(grads, master, m, v, hp: AdamHP, t: int):
    """One owner step on a range: returns (skipped, master, m, v, p16 or None)."""
    gs = [_as_u16(g) for g in grads]
    n = gs[0].size
    ptrs = (C.POINTER(C.c_uint16) * len(gs))(*[_u16p(g) for g in gs])
    w, mm, vv = (np.array(a, dtype=np.float32, copy=True) for a in (master, m, v))
    p16 = np.empty(n, np.uint16)
    scratch = np.empty(n, np.float32)
    h = _HP(hp.lr, hp.beta1, hp.beta2, hp.eps, hp.loss_scale)
    rc = lib().orc_step(n, len(gs), ptrs, _f32p(w), _f32p(mm), _f32p(vv), _u16p(p16),
                        C.byref(h), t, _f32p(scratch))
    if rc < 0:
        raise ValueError("step t must be >= 1")
    if rc == SKIPPED:
        return True, np.array(master, np.float32), np.array(m, np.float32), \
            np.array(v, np.float32), None
    return False, w, mm, vv, p16


# ---------------------------------------------------------------------------------------------
# whole-model steps: plain DP and the two ZeRO-DP stages
# ---------------------------------------------------------------------------------------------
@dataclasses.dataclass
class Result:
    skipped: bool
    master: np.ndarray
    m: np.ndarray
    v: np.ndarray
    params16: np.ndarray                 # the full fp16 parameter buffer every replica holds
    reduced: np.ndarray = None           # reduced gradient as kept by its owner (psi_p floats)


def dp_step(local_grads, master, m, v, params16, hp: AdamHP, t: int) -> Result:
    """Plain DP: all-reduce (mean) the full gradient, then every replica updates everything.

    local_grads: Nd arrays of psi_p fp16 values (one full local gradient per rank).
    """
    red = reduce_mean(local_grads)
    if not all_finite(red):
        return Result(True, np.array(master, np.float32), np.array(m, np.float32),
                      np.array(v, np.float32), np.array(params16, np.uint16), red)
    w, mm, vv, p16 = adam(red, master, m, v, hp, t)
    return Result(False, w, mm, vv, p16, red)


def zero1_step(pl: Plan, local_grads, master, m, v, params16, hp: AdamHP, t: int) -> Result:
    """Stage 1: one reduce-scatter of the full local gradients at the step.

    The state arrays hold the Nd owners' shards end to end (owner r: [r*S, (r+1)*S)).
    """
    S, nd = pl.shard, pl.nd
    gs = [_as_u16(g) for g in local_grads]
    assert len(gs) == nd and all(g.size == pl.psi_p for g in gs)
    # reduce-scatter: owner r receives rank j's slice r of the local gradient, for every j
    shards = []
    for r in range(nd):
        shards.append(reduce_mean([g[r * S:(r + 1) * S] for g in gs]))
    # one verdict for the whole step, over every owner's shard
    if not all(all_finite(sh) for sh in shards):
        return Result(True, np.array(master, np.float32), np.array(m, np.float32),
                      np.array(v, np.float32), np.array(params16, np.uint16),
                      np.concatenate(shards))
    w_out = np.array(master, np.float32)
    m_out = np.array(m, np.float32)
    v_out = np.array(v, np.float32)
    p_out = np.array(params16, np.uint16)
    for r in range(nd):
        sl = slice(r * S, (r + 1) * S)
        w, mm, vv, p16 = adam(shards[r], master[sl], m[sl], v[sl], hp, t)
        w_out[sl], m_out[sl], v_out[sl] = w, mm, vv
        p_out[sl] = p16           # all-gather: owner r's updated fp16 shard into the full buffer
    return Result(False, w_out, m_out, v_out, p_out, np.concatenate(shards))


def zero2_step(pl: Plan, bucket_grad: Callable[[int, int], np.ndarray], master, m, v, params16,
               hp: AdamHP, t: int) -> Result:
    """Stage 2: buckets in backward order; each is reduce-scattered when produced.

    bucket_grad(k, rank) returns rank's local fp16 gradient for bucket k (pl.buckets[k][1]
    values). After the reduce-scatter of bucket k only the owners' reduced slices are kept;
    the local bucket gradients are dropped before the next bucket is produced.
    """
    S, nd = pl.shard, pl.nd
    grad_shard = [np.zeros(S, np.float32) for _ in range(nd)]    # owner r's reduced grad shard
    for k, (lo, ln) in enumerate(pl.buckets):
        local = [_as_u16(bucket_grad(k, j)) for j in range(nd)]
        assert all(g.size == ln for g in local)
        o_lo, o_hi = lo // S, (lo + ln - 1) // S
        for r in range(o_lo, o_hi + 1):
            a, b = max(lo, r * S), min(lo + ln, (r + 1) * S)
            grad_shard[r][a - r * S:b - r * S] = reduce_mean([g[a - lo:b - lo] for g in local])
        del local                                                 # release
    if not all(all_finite(sh) for sh in grad_shard):
        return Result(True, np.array(master, np.float32), np.array(m, np.float32),
                      np.array(v, np.float32), np.array(params16, np.uint16),
                      np.concatenate(grad_shard))
    w_out = np.array(master, np.float32)
    m_out = np.array(m, np.float32)
    v_out = np.array(v, np.float32)
    p_out = np.array(params16, np.uint16)
    for r in range(nd):
        sl = slice(r * S, (r + 1) * S)
        w, mm, vv, p16 = adam(grad_shard[r], master[sl], m[sl], v[sl], hp, t)
        w_out[sl], m_out[sl], v_out[sl] = w, mm, vv
        p_out[sl] = p16
    return Result(False, w_out, m_out, v_out, p_out, np.concatenate(grad_shard))


# ---------------------------------------------------------------------------------------------
# stage 3 (Pos+g+p): the parameters are partitioned too
#
# "ZeRO: particionar estados do treino entre GPUs", "Como funciona": in the third stage the
# fp16 parameters are also split among the Nd processes, a process that needs a partition it
# does not own receives it from the owner, and a step moves 3 psi: a parameter all-gather in
# the forward pass, another in the backward pass, and the gradient reduce-scatter (1.5 times the
# 2 psi of plain DP). "ZeRO" (lastdictionary), main definition: each layer's parameters are
# gathered just in time for its computation and discarded afterwards; stage 3 adds about 50 %
# communication.
#
# Readings (the pages are silent on them): a layer is a run of consecutive tensors of the
# forward-order list; the backward pass reduce-scatters each layer's local gradient as soon as
# the layer is done (a bucket per layer, as stage 2 does per bucket); the zero padding at the
# end of the flat list rides with the first gradient bucket of the backward pass, the last
# layer's, as it does in stage 2's bucket map; the owner's update writes its fp16 values into
# its own parameter shard, and nothing gathers them after the step (the next forward pass does,
# layer by layer). Communication counts the model's elements (the padding is not model state).
# ---------------------------------------------------------------------------------------------
def layer_ranges(pl: Plan, layer_tensors: Sequence[int]) -> List[tuple]:
    """Flat ranges [lo, hi) of the layers, in forward order: layer l is the next
    layer_tensors[l] tensors of the plan's list."""
    if sum(layer_tensors) != len(pl.numels) or any(c < 1 for c in layer_tensors):
        raise ValueError("layer_tensors must split the tensor list into non-empty runs")
    out, i = [], 0
    for c in layer_tensors:
        lo = pl.tensor_off[i]
        last = i + c - 1
        out.append((lo, pl.tensor_off[last] + pl.numels[last]))
        i += c
    return out


def grad_buckets(pl: Plan, layers: Sequence[tuple]) -> List[tuple]:
    """The gradient bucket of each layer: its range, the last layer's extended over the zero
    padding to psi_p (the backward pass produces the end of the flat list first)."""
    out = list(layers)
    lo, _ = out[-1]
    out[-1] = (lo, pl.psi_p)
    return out


def gather_params(param_shards, S: int, lo: int, hi: int) -> np.ndarray:
    """The just-in-time all-gather of the flat range [lo, hi): every owner q whose shard
    [q*S, (q+1)*S) meets the range hands over that part; the pieces, in owner order, make up
    the layer's fp16 parameters."""
    out = np.empty(hi - lo, np.uint16)
    for q in range(lo // S, (hi - 1) // S + 1):
        a, b = max(lo, q * S), min(hi, (q + 1) * S)
        out[a - lo:b - lo] = _as_u16(param_shards[q])[a - q * S:b - q * S]
    return out


@dataclasses.dataclass
class Result3:
    skipped: bool
    master: np.ndarray
    m: np.ndarray
    v: np.ndarray
    param_shards: List[np.ndarray]       # owner q's fp16 parameter partition (S values each)
    gathered_fwd: List[np.ndarray]       # layer l's gathered parameters in the forward pass
    gathered_bwd: List[np.ndarray]       # ... and in the backward pass (index l, not order)
    comm_elems: int                      # elements moved by the step's collectives
    reduced: np.ndarray = None           # the owners' reduced gradient shards, end to end


def zero3_step(pl: Plan, layers: Sequence[tuple], layer_grad: Callable[[int, int], np.ndarray],
               master, m, v, param_shards, hp: AdamHP, t: int) -> Result3:
    """Stage 3: forward gathers layer by layer, backward gathers again in reverse order and
    reduce-scatters each layer's local gradient, then every owner updates its shard.

    layers: flat ranges (layer_ranges); layer_grad(l, rank): rank's local fp16 gradient of
    layer l's gradient bucket (grad_buckets: the layer's range, the last one extended over the
    padding); param_shards: Nd arrays of S fp16 values (owner q's partition).
    """
    S, nd = pl.shard, pl.nd
    shards = [_as_u16(p).copy() for p in param_shards]
    assert len(shards) == nd and all(p.size == S for p in shards)
    comm = 0
    fwd, bwd = [None] * len(layers), [None] * len(layers)
    for l, (lo, hi) in enumerate(layers):                    # forward pass
        fwd[l] = gather_params(shards, S, lo, hi)             # used, then discarded
        comm += hi - lo
    grad_shard = [np.zeros(S, np.float32) for _ in range(nd)]
    buckets = grad_buckets(pl, layers)
    for l in reversed(range(len(layers))):                    # backward pass
        lo, hi = layers[l]
        bwd[l] = gather_params(shards, S, lo, hi)
        comm += hi - lo
        _, ghi = buckets[l]
        local = [_as_u16(layer_grad(l, j)) for j in range(nd)]
        assert all(g.size == ghi - lo for g in local)
        for q in range(lo // S, (ghi - 1) // S + 1):          # reduce-scatter of the layer
            a, b = max(lo, q * S), min(ghi, (q + 1) * S)
            grad_shard[q][a - q * S:b - q * S] = reduce_mean([g[a - lo:b - lo] for g in local])
        comm += hi - lo
        del local                                             # released
    w_out = np.array(master, np.float32)
    m_out = np.array(m, np.float32)
    v_out = np.array(v, np.float32)
    red = np.concatenate(grad_shard)
    if not all(all_finite(sh) for sh in grad_shard):
        return Result3(True, w_out, m_out, v_out, shards, fwd, bwd, comm, red)
    for q in range(nd):
        sl = slice(q * S, (q + 1) * S)
        w, mm, vv, p16 = adam(grad_shard[q], master[sl], m[sl], v[sl], hp, t)
        w_out[sl], m_out[sl], v_out[sl] = w, mm, vv
        shards[q] = p16                  # the owner's partition; no all-gather after the step
    return Result3(False, w_out, m_out, v_out, shards, fwd, bwd, comm, red)


def ulp_diff_f32(a, b) -> np.ndarray:
    """Distance in units in the last place between binary32 arrays (ordered-integer metric;
    two NaNs are 0 apart, NaN vs a number is 2**32)."""
    a = np.ascontiguousarray(a, np.float32).view(np.int32).astype(np.int64)
    b = np.ascontiguousarray(b, np.float32).view(np.int32).astype(np.int64)
    oa = np.where(a < 0, -(a & 0x7fffffff), a)
    ob = np.where(b < 0, -(b & 0x7fffffff), b)
    d = np.abs(oa - ob)
    na = ((a & 0x7f800000) == 0x7f800000) & ((a & 0x7fffff) != 0)
    nb = ((b & 0x7f800000) == 0x7f800000) & ((b & 0x7fffff) != 0)
    d = np.where(na & nb, 0, np.where(na ^ nb, 1 << 32, d))
    return d


def ulp_diff_f16(a, b) -> np.ndarray:
    """Same metric for binary16 bit patterns (uint16 or float16 arrays)."""
    a = _as_u16(a).astype(np.int64)
    b = _as_u16(b).astype(np.int64)
    oa = np.where(a & 0x8000, -(a & 0x7fff), a)
    ob = np.where(b & 0x8000, -(b & 0x7fff), b)
    d = np.abs(oa - ob)
    na = ((a & 0x7c00) == 0x7c00) & ((a & 0x3ff) != 0)
    nb = ((b & 0x7c00) == 0x7c00) & ((b & 0x3ff) != 0)
    return np.where(na & nb, 0, np.where(na ^ nb, 1 << 32, d))


# ---------------------------------------------------------------------------------------------
# dynamic loss scaling (the pages say nothing about it; the rule is the one of Micikevicius et
# al., "Mixed Precision Training", ICLR 2018, section 3.2, in the form of torch.cuda.amp's
# GradScaler): an overflowing step is skipped and the scale is multiplied by backoff_factor;
# after growth_interval consecutive applied steps it is multiplied by growth_factor. The Adam
# step t counts applied steps only. The scale is a binary32 number.
# ---------------------------------------------------------------------------------------------
@dataclasses.dataclass
class Scaler:
    scale: float = 1024.0
    good_steps: int = 0
    next_step: int = 1
    skipped_steps: int = 0
    growth_factor: float = 2.0
    backoff_factor: float = 0.5
    growth_interval: int = 2000

    def update(self, overflowed: bool):
        if overflowed:
            self.scale = float(np.float32(self.scale) * np.float32(self.backoff_factor))
            self.good_steps = 0
            self.skipped_steps += 1
        else:
            self.next_step += 1
            self.good_steps += 1
            if self.good_steps >= self.growth_interval:
                self.scale = float(np.float32(self.scale) * np.float32(self.growth_factor))
                self.good_steps = 0


def scaled_step(grads, master, m, v, hp: AdamHP, sc: Scaler):
    """One step under dynamic loss scaling: the gradients carry sc.scale, Adam uses step
    sc.next_step; then the scaler is updated. Returns (skipped, master, m, v, p16)."""
    hp_t = dataclasses.replace(hp, loss_scale=sc.scale)
    skipped, w, mm, vv, p16 = step(grads, master, m, v, hp_t, sc.next_step)
    sc.update(skipped)
    return skipped, w, mm, vv, p16


# ---------------------------------------------------------------------------------------------
# compressed reduce-scatter payload: int8 with one fp32 scale per block of 128 elements
# ("ZeRO" (lastdictionary): extensions compress communication, ZeRO++; the format is this
# library's reading, see oracle.c)
# ---------------------------------------------------------------------------------------------
QB = 128


def quant_q8(g):
    """A rank's fp16 slice -> (int8 values, fp32 scale per block of 128)."""
    g = _as_u16(g)
    q = np.empty(g.size, np.int8)
    sc = np.empty((g.size + QB - 1) // QB, np.float32)
    lib().orc_quant_q8(g.size, _u16p(g), q.ctypes.data_as(C.POINTER(C.c_int8)), _f32p(sc))
    return q, sc


def reduce_mean_q8(qs, scales):
    n = qs[0].size
    qs = [np.ascontiguousarray(q, np.int8) for q in qs]
    scales = [np.ascontiguousarray(s, np.float32) for s in scales]
    qp = (C.POINTER(C.c_int8) * len(qs))(*[q.ctypes.data_as(C.POINTER(C.c_int8)) for q in qs])
    sp = (C.POINTER(C.c_float) * len(qs))(*[_f32p(s) for s in scales])
    red = np.empty(n, np.float32)
    lib().orc_reduce_mean_q8(n, len(qs), qp, sp, _f32p(red))
    return red


def step_q8(qs, scales, master, m, v, hp: AdamHP, t: int):
    """The owner's step from int8 payloads: (skipped, master, m, v, p16 or None)."""
    red = reduce_mean_q8(qs, scales)
    if not all_finite(red):
        return True, np.array(master, np.float32), np.array(m, np.float32), \
            np.array(v, np.float32), None
    w, mm, vv, p16 = adam(red, master, m, v, hp, t)
    return False, w, mm, vv, p16


def step_q8_gathered(qs, scale_of_elem, master, m, v, hp: AdamHP, t: int):
    """step_q8 on gathered samples: scale_of_elem[r][i] is the scale of sample i's block."""
    n = qs[0].size
    qs = [np.ascontiguousarray(q, np.int8) for q in qs]
    sc = [np.ascontiguousarray(s, np.float32) for s in scale_of_elem]
    qp = (C.POINTER(C.c_int8) * len(qs))(*[q.ctypes.data_as(C.POINTER(C.c_int8)) for q in qs])
    sp = (C.POINTER(C.c_float) * len(qs))(*[_f32p(s) for s in sc])
    red = np.empty(n, np.float32)
    lib().orc_reduce_mean_q8_gathered(n, len(qs), qp, sp, _f32p(red))
    if not all_finite(red):
        return True, np.array(master, np.float32), np.array(m, np.float32), \
            np.array(v, np.float32), None
    w, mm, vv, p16 = adam(red, master, m, v, hp, t)
    return False, w, mm, vv, p16
