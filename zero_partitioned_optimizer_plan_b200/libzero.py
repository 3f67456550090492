"""Python binding of libzero.so (argument marshalling only).

Every function has the name of the C entry point it calls (include/libzero.h) and does no
arithmetic of its own. Device buffers are given as torch tensors (their data_ptr() is passed)
or as raw integer addresses; streams as torch.cuda.Stream, a raw cudaStream_t integer, or None
for torch's current stream. A non-OK status raises ZeroError, except zero_step_status, which
returns it.

Importing this module loads the in-tree libzero.so and fails loudly if it has not been built
(``python -m zero_partitioned_optimizer_plan_b200.build``): there is no fallback.
"""
from __future__ import annotations

import ctypes as C
import dataclasses
import os
from typing import List, Sequence

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "lib", "libzero.so")

ZERO_OK = 0
ZERO_EINVAL = 1
ZERO_EALIGN = 2
ZERO_ECUDA = 3
ZERO_ENOMEM = 4
ZERO_STEP_SKIPPED = 5

ZERO_FLAG_OVERFLOW = 0x1
ZERO_FLAG_SKIPPED = 0x2
ZERO_FLAG_TIMEOUT = 0x4
ZERO_FLAG_BOUNDS = 0x8

ZERO_MAX_RANKS = 64
ZERO_Q8_BLOCK = 128
ZERO_Q8_RECORD = 132


def q8_payload_bytes(n: int) -> int:
    """ZERO_Q8_PAYLOAD_BYTES(n)."""
    return (n + 127) // 128 * 132

# every symbol include/libzero.h declares
SYMBOLS = (
    "zero_status_string", "zero_kernel_launches", "zero_last_error",
    "zero_plan_create", "zero_plan_destroy", "zero_plan_info", "zero_plan_tensor_offsets",
    "zero_plan_bucket", "zero_state_bytes",
    "zero_reduce_scatter_bucket", "zero_adam_shard", "zero_step_fused", "zero_step_commit",
    "zero_step_status", "zero_adam_consts_for_step", "zero_adam_shard_dc", "zero_step_fused_dc",
    "zero_selftest_timeout", "zero_adam_consts_table", "zero_scaler_prepare",
    "zero_scaler_update", "zero_quantize_q8", "zero_step_fused_q8", "zero_step_fused_q8_dc",
    "zero_overlap_begin", "zero_overlap_end",
    "zero_gather_params", "zero_stage3_step_fused", "zero_stage3_step_commit",
    "zero_stage3_step_fused_dc", "zero_stage3_payload_bytes_q8", "zero_stage3_quantize_q8",
    "zero_stage3_step_fused_q8", "zero_stage3_step_fused_q8_dc",
    "zero_step_fused_ranges", "zero_step_fused_q8_ranges",
    "zero_step_fused_replicas", "zero_step_commit_replicas",
    "zero_sched_slot_elems", "zero_sched_create", "zero_sched_create_fused",
    "zero_sched_begin_bucket", "zero_sched_rebind_fused", "zero_sched_rebind_status",
    "zero_sched_end_bucket", "zero_sched_wait", "zero_sched_launches", "zero_sched_destroy",
    "zero_sched_slot_bytes_q8", "zero_sched_create_fused_q8", "zero_sched_begin_bucket_q8",
    "zero_layer_sched_buf_elems", "zero_layer_sched_create", "zero_layer_sched_begin_step",
    "zero_layer_sched_acquire", "zero_layer_sched_release", "zero_layer_sched_gathers",
    "zero_layer_sched_destroy",
)


class ZeroError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        msg = f"{where}: {zero_status_string(code)}"
        if code == ZERO_ECUDA:
            msg += f" ({zero_last_error()})"
        super().__init__(msg)


class _Bytes(C.Structure):
    _fields_ = [("params", C.c_uint64), ("grads", C.c_uint64), ("optim", C.c_uint64),
                ("total", C.c_uint64)]


class _Report(C.Structure):
    _fields_ = [("stage", _Bytes * 4), ("comm_elems", C.c_uint64 * 4),
                ("comm_bytes_fp16", C.c_uint64 * 4)]


class _HP(C.Structure):
    _fields_ = [("lr", C.c_double), ("beta1", C.c_double), ("beta2", C.c_double),
                ("eps", C.c_double), ("loss_scale", C.c_double)]


class AdamConsts(C.Structure):
    """zero_adam_consts: one step's fp32 constants (copy into device memory for the _dc calls;
    bytes(obj) gives its ZERO_ADAM_CONSTS_BYTES-byte image)."""
    _fields_ = [("beta1", C.c_float), ("one_minus_beta1", C.c_float), ("beta2", C.c_float),
                ("one_minus_beta2", C.c_float), ("step_size", C.c_float),
                ("bias2_sqrt", C.c_float), ("eps", C.c_float), ("loss_scale", C.c_float),
                ("inv_loss_scale", C.c_float), ("loss_scale_pow2", C.c_int32)]


ZERO_ADAM_CONSTS_BYTES = C.sizeof(AdamConsts)


class ScalerState(C.Structure):
    """zero_scaler_state (24 bytes; copy into 8-byte-aligned device memory)."""
    _fields_ = [("scale", C.c_float), ("good_steps", C.c_int32), ("next_step", C.c_int64),
                ("skipped_steps", C.c_int64)]


class FusedRange(C.Structure):
    """zero_fused_range: one range of a step for zero_step_fused_ranges."""
    _fields_ = [("n", C.c_uint64), ("rank_grads", C.POINTER(C.c_void_p)),
                ("master_in", C.c_void_p), ("m_in", C.c_void_p), ("v_in", C.c_void_p),
                ("master_out", C.c_void_p), ("m_out", C.c_void_p), ("v_out", C.c_void_p),
                ("param_out", C.c_void_p)]


class FusedQ8Range(C.Structure):
    """zero_fused_q8_range: one range of a step for zero_step_fused_q8_ranges."""
    _fields_ = [("n", C.c_uint64), ("rank_payload", C.POINTER(C.c_void_p)),
                ("master_in", C.c_void_p), ("m_in", C.c_void_p), ("v_in", C.c_void_p),
                ("master_out", C.c_void_p), ("m_out", C.c_void_p), ("v_out", C.c_void_p),
                ("param_out", C.c_void_p)]


class ScalerParams(C.Structure):
    _fields_ = [("growth_factor", C.c_float), ("backoff_factor", C.c_float),
                ("growth_interval", C.c_int32)]


@dataclasses.dataclass(frozen=True)
class AdamHP:
    lr: float = 1e-3
    beta1: float = 0.9
    beta2: float = 0.999
    eps: float = 1e-8
    loss_scale: float = 1024.0

    def _c(self):
        return _HP(self.lr, self.beta1, self.beta2, self.eps, self.loss_scale)


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"libzero.so is not built ({LIB_PATH}); run "
            "`python -m zero_partitioned_optimizer_plan_b200.build` (needs nvcc)")
    L = C.CDLL(LIB_PATH)
    u64, i64, vp, i32 = C.c_uint64, C.c_int64, C.c_void_p, C.c_int
    P = C.POINTER
    L.zero_status_string.argtypes, L.zero_status_string.restype = [i32], C.c_char_p
    L.zero_kernel_launches.argtypes, L.zero_kernel_launches.restype = [], u64
    L.zero_last_error.argtypes, L.zero_last_error.restype = [], C.c_char_p
    L.zero_plan_create.argtypes = [P(u64), i32, i32, i32, u64, P(vp)]
    L.zero_plan_destroy.argtypes, L.zero_plan_destroy.restype = [vp], None
    L.zero_plan_info.argtypes = [vp, P(u64), P(u64), P(u64), P(i32)]
    L.zero_plan_tensor_offsets.argtypes = [vp, P(u64)]
    L.zero_plan_bucket.argtypes = [vp, i32, P(u64), P(u64), P(i32), P(i32)]
    L.zero_state_bytes.argtypes = [u64, i32, i32, P(_Report)]
    L.zero_reduce_scatter_bucket.argtypes = [vp, i32, P(vp), P(vp), vp, vp]
    L.zero_adam_shard.argtypes = [u64, vp, vp, vp, vp, vp, P(_HP), i64, vp, vp]
    L.zero_step_fused.argtypes = [u64, i32, P(vp), vp, vp, vp, vp, vp, vp, vp, P(_HP), i64,
                                  vp, vp]
    L.zero_step_commit.argtypes = [u64, vp, vp, vp, vp, vp, vp, vp, vp, vp]
    L.zero_step_status.argtypes = [vp, vp, P(C.c_uint32)]
    L.zero_adam_consts_for_step.argtypes = [P(_HP), i64, P(AdamConsts)]
    L.zero_adam_shard_dc.argtypes = [u64, vp, vp, vp, vp, vp, vp, vp, vp]
    L.zero_step_fused_dc.argtypes = [u64, i32, P(vp), vp, vp, vp, vp, vp, vp, vp, vp, vp, vp]
    L.zero_selftest_timeout.argtypes = [vp, vp]
    L.zero_quantize_q8.argtypes = [u64, vp, vp, vp]
    L.zero_step_fused_q8.argtypes = [u64, i32, P(vp), vp, vp, vp, vp, vp, vp, vp,
                                     P(_HP), i64, vp, vp]
    L.zero_step_fused_q8_dc.argtypes = [u64, i32, P(vp), vp, vp, vp, vp, vp, vp, vp, vp, vp, vp]
    L.zero_adam_consts_table.argtypes = [P(_HP), i64, i64, P(AdamConsts)]
    L.zero_scaler_prepare.argtypes = [vp, vp, i64, vp, vp, vp]
    L.zero_scaler_update.argtypes = [vp, P(ScalerParams), vp, vp]
    L.zero_step_fused_ranges.argtypes = [i32, i32, P(FusedRange), P(_HP), i64, vp, i32, vp]
    L.zero_step_fused_q8_ranges.argtypes = [i32, i32, P(FusedQ8Range), P(_HP), i64, vp, i32, vp]
    L.zero_step_fused_replicas.argtypes = [u64, i32, P(vp), vp, vp, vp, vp, vp, vp, i32, P(vp),
                                           P(_HP), i64, vp, vp]
    L.zero_step_commit_replicas.argtypes = [u64, vp, vp, vp, vp, vp, vp, i32, P(vp), vp, vp]
    L.zero_gather_params.argtypes = [vp, u64, u64, P(vp), vp, vp, vp]
    L.zero_stage3_step_fused.argtypes = [vp, u64, u64, P(vp), vp, vp, vp, vp, vp, vp, P(vp), P(_HP),
                                   i64, vp, vp]
    L.zero_stage3_step_commit.argtypes = [vp, vp, vp, vp, vp, vp, vp, P(vp), vp, vp]
    L.zero_stage3_step_fused_dc.argtypes = [vp, u64, u64, P(vp), vp, vp, vp, vp, vp, vp, P(vp),
                                            vp, vp, vp]
    L.zero_stage3_payload_bytes_q8.argtypes = [vp, u64, u64, P(u64)]
    L.zero_stage3_quantize_q8.argtypes = [vp, u64, u64, vp, vp, vp]
    L.zero_stage3_step_fused_q8.argtypes = [vp, u64, u64, P(vp), vp, vp, vp, vp, vp, vp, P(vp),
                                            P(_HP), i64, vp, vp]
    L.zero_stage3_step_fused_q8_dc.argtypes = [vp, u64, u64, P(vp), vp, vp, vp, vp, vp, vp,
                                               P(vp), vp, vp, vp]
    L.zero_overlap_begin.argtypes = [vp]
    L.zero_overlap_end.argtypes = [vp]
    L.zero_sched_slot_elems.argtypes = [vp, i32, P(u64)]
    L.zero_sched_create.argtypes = [vp, vp, u64, i32, P(vp), vp, vp, P(vp)]
    L.zero_sched_create_fused.argtypes = [vp, vp, u64, i32, vp, vp, vp, vp, vp, vp, vp, vp, vp,
                                          vp, P(vp)]
    L.zero_sched_rebind_fused.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp]
    L.zero_sched_rebind_status.argtypes = [vp, vp]
    L.zero_sched_begin_bucket.argtypes = [vp, i32, vp, P(vp)]
    L.zero_sched_end_bucket.argtypes = [vp, i32, vp]
    L.zero_sched_wait.argtypes = [vp, vp]
    L.zero_sched_launches.argtypes = [vp, P(u64)]
    L.zero_sched_destroy.argtypes, L.zero_sched_destroy.restype = [vp], None
    L.zero_sched_slot_bytes_q8.argtypes = [vp, i32, P(u64)]
    L.zero_sched_create_fused_q8.argtypes = [vp, vp, u64, i32, vp, vp, vp, vp, vp, vp, vp, vp,
                                             vp, vp, P(vp)]
    L.zero_sched_begin_bucket_q8.argtypes = [vp, i32, vp, P(vp)]
    L.zero_layer_sched_buf_elems.argtypes = [vp, i32, P(u64), i32, P(u64)]
    L.zero_layer_sched_create.argtypes = [vp, i32, P(u64), P(vp), vp, u64, i32, vp, P(vp)]
    L.zero_layer_sched_begin_step.argtypes = [vp, vp, vp]
    L.zero_layer_sched_acquire.argtypes = [vp, i32, i32, vp, P(vp)]
    L.zero_layer_sched_release.argtypes = [vp, i32, vp]
    L.zero_layer_sched_gathers.argtypes = [vp, P(u64)]
    L.zero_layer_sched_destroy.argtypes, L.zero_layer_sched_destroy.restype = [vp], None
    # every other entry point returns a zero_status: ctypes' default int restype
    return L


_lib = _load()


# ---------------------------------------------------------------------------------------------
# marshalling helpers
# ---------------------------------------------------------------------------------------------
def _ptr(x, elem_size: int | None = None) -> int:
    if x is None:
        return 0
    if hasattr(x, "data_ptr"):
        if elem_size is not None and x.element_size() != elem_size:
            raise TypeError(f"expected a tensor of {elem_size}-byte elements, got {x.dtype}")
        if not x.is_contiguous():
            raise TypeError("tensor must be contiguous")
        return int(x.data_ptr())
    return int(x)


def _stream(s) -> int:
    if s is None:
        import torch
        return int(torch.cuda.current_stream().cuda_stream)
    if hasattr(s, "cuda_stream"):
        return int(s.cuda_stream)
    return int(s)


def _ptr_array(xs, elem_size=None):
    return (C.c_void_p * max(len(xs), 1))(*[_ptr(x, elem_size) for x in xs])


def _check(code: int, where: str):
    if code != ZERO_OK:
        raise ZeroError(code, where)


def zero_status_string(code: int) -> str:
    return _lib.zero_status_string(int(code)).decode()


def zero_kernel_launches() -> int:
    return int(_lib.zero_kernel_launches())


def zero_last_error() -> str:
    return _lib.zero_last_error().decode()


# ---------------------------------------------------------------------------------------------
# plan and accounting
# ---------------------------------------------------------------------------------------------
class Plan:
    """Owns a zero_plan handle (host memory)."""

    def __init__(self, handle: int, n_tensors: int):
        self.handle = handle
        self.n_tensors = n_tensors

    def __del__(self):
        if getattr(self, "handle", None):
            _lib.zero_plan_destroy(self.handle)
            self.handle = None


def zero_plan_create(numels: Sequence[int], nd: int, stage: int = 1, bucket_elems: int = 0) -> Plan:
    arr = (C.c_uint64 * max(len(numels), 1))(*[int(x) for x in numels])
    h = C.c_void_p()
    _check(_lib.zero_plan_create(arr, len(numels), nd, stage, bucket_elems, C.byref(h)),
           "zero_plan_create")
    return Plan(h.value, len(numels))


def zero_plan_destroy(plan: Plan):
    if plan.handle:
        _lib.zero_plan_destroy(plan.handle)
        plan.handle = None


def zero_plan_info(plan: Plan):
    psi, psi_p, shard = C.c_uint64(), C.c_uint64(), C.c_uint64()
    nb = C.c_int()
    _check(_lib.zero_plan_info(plan.handle, C.byref(psi), C.byref(psi_p), C.byref(shard),
                               C.byref(nb)), "zero_plan_info")
    return psi.value, psi_p.value, shard.value, nb.value


def zero_plan_tensor_offsets(plan: Plan) -> List[int]:
    out = (C.c_uint64 * max(plan.n_tensors, 1))()
    _check(_lib.zero_plan_tensor_offsets(plan.handle, out), "zero_plan_tensor_offsets")
    return list(out[:plan.n_tensors])


def zero_plan_bucket(plan: Plan, k: int):
    lo, ln = C.c_uint64(), C.c_uint64()
    olo, ohi = C.c_int(), C.c_int()
    _check(_lib.zero_plan_bucket(plan.handle, k, C.byref(lo), C.byref(ln), C.byref(olo),
                                 C.byref(ohi)), "zero_plan_bucket")
    return lo.value, ln.value, olo.value, ohi.value


STAGES = ("dp", "pos", "pos_g", "pos_g_p")


def zero_state_bytes(psi: int, nd: int, K: int = 12) -> dict:
    rep = _Report()
    _check(_lib.zero_state_bytes(psi, nd, K, C.byref(rep)), "zero_state_bytes")
    out = {}
    for s, name in enumerate(STAGES):
        b = rep.stage[s]
        out[name] = dict(params=b.params, grads=b.grads, optim=b.optim, total=b.total,
                         comm_elems=rep.comm_elems[s], comm_bytes_fp16=rep.comm_bytes_fp16[s])
    return out


# ---------------------------------------------------------------------------------------------
# data path
# ---------------------------------------------------------------------------------------------
def zero_reduce_scatter_bucket(plan: Plan, k: int, rank_grads, owner_grad_shards, d_status,
                               stream=None):
    _check(_lib.zero_reduce_scatter_bucket(plan.handle, k, _ptr_array(rank_grads, 2),
                                           _ptr_array(owner_grad_shards, 4), _ptr(d_status, 4),
                                           _stream(stream)), "zero_reduce_scatter_bucket")


def zero_adam_shard(n: int, grad, master, m, v, param_out, hp: AdamHP, step: int, d_status,
                    stream=None):
    h = hp._c()
    _check(_lib.zero_adam_shard(n, _ptr(grad, 4), _ptr(master, 4), _ptr(m, 4), _ptr(v, 4),
                                _ptr(param_out, 2), C.byref(h), step, _ptr(d_status, 4),
                                _stream(stream)), "zero_adam_shard")


def zero_step_fused(n: int, nd: int, rank_grads, master_in, m_in, v_in, master_out, m_out,
                    v_out, param_out, hp: AdamHP, step: int, d_status, stream=None):
    h = hp._c()
    _check(_lib.zero_step_fused(n, nd, _ptr_array(rank_grads, 2), _ptr(master_in, 4),
                                _ptr(m_in, 4), _ptr(v_in, 4), _ptr(master_out, 4),
                                _ptr(m_out, 4), _ptr(v_out, 4), _ptr(param_out, 2), C.byref(h),
                                step, _ptr(d_status, 4), _stream(stream)), "zero_step_fused")


class PreparedStepRanges:
    """zero_step_fused_ranges (payload "fp16") or zero_step_fused_q8_ranges (payload "q8") with
    its range descriptors marshalled once: each item of `ranges` is (n, rank inputs, master_in,
    m_in, v_in, master_out, m_out, v_out, param_out) as zero_step_fused / zero_step_fused_q8
    take them (rank inputs: the ranks' fp16 gradients, or their int8 payloads). Calling it
    launches every range of the step in one C call."""

    def __init__(self, nd: int, ranges, payload: str = "fp16"):
        if payload not in ("fp16", "q8"):
            raise ValueError(f"payload {payload!r}")
        self.nd = nd
        q8 = payload == "q8"
        self._name = "zero_step_fused_q8_ranges" if q8 else "zero_step_fused_ranges"
        self._fn = getattr(_lib, self._name)
        Range = FusedQ8Range if q8 else FusedRange
        self._in_arrays = [_ptr_array(r[1], 1 if q8 else 2) for r in ranges]   # kept alive
        arr = (Range * max(len(ranges), 1))()
        for i, (r, g) in enumerate(zip(ranges, self._in_arrays)):
            arr[i] = Range(r[0], C.cast(g, C.POINTER(C.c_void_p)), *[
                _ptr(x, 4) for x in r[2:8]], _ptr(r[8], 2))
        self._arr = arr
        self.count = len(ranges)

    def __call__(self, hp_ref, step: int, d_status: int, overlap: bool, stream: int):
        code = self._fn(self.nd, self.count, self._arr, hp_ref, step, d_status,
                        1 if overlap else 0, stream)
        if code:
            raise ZeroError(code, self._name)


def zero_step_fused_ranges(nd: int, ranges, hp: AdamHP, step: int, d_status, overlap=True,
                           stream=None):
    PreparedStepRanges(nd, ranges)(hparams_ref(hp), step, _ptr(d_status, 4), overlap,
                                   _stream(stream))


def zero_step_fused_replicas(n: int, nd: int, rank_grads, master_in, m_in, v_in, master_out, m_out,
                             v_out, replicas, hp: AdamHP, step: int, d_status, stream=None):
    """zero_step_fused with the fp16 write-back stored into every replica (the all-gather in the
    epilogue); replicas: tensors or device addresses of this range in each replica."""
    h = hp._c()
    _check(_lib.zero_step_fused_replicas(n, nd, _ptr_array(rank_grads, 2), _ptr(master_in, 4),
                                         _ptr(m_in, 4), _ptr(v_in, 4), _ptr(master_out, 4),
                                         _ptr(m_out, 4), _ptr(v_out, 4), len(replicas),
                                         _ptr_array(replicas, 2), C.byref(h), step,
                                         _ptr(d_status, 4), _stream(stream)),
           "zero_step_fused_replicas")


def zero_step_commit_replicas(n: int, master_in, m_in, v_in, master_out, m_out, v_out, replicas,
                              d_status, stream=None):
    _check(_lib.zero_step_commit_replicas(n, _ptr(master_in, 4), _ptr(m_in, 4), _ptr(v_in, 4),
                                          _ptr(master_out, 4), _ptr(m_out, 4), _ptr(v_out, 4),
                                          len(replicas), _ptr_array(replicas, 2),
                                          _ptr(d_status, 4), _stream(stream)),
           "zero_step_commit_replicas")


def zero_step_fused_q8_ranges(nd: int, ranges, hp: AdamHP, step: int, d_status, overlap=True,
                              stream=None):
    PreparedStepRanges(nd, ranges, "q8")(hparams_ref(hp), step, _ptr(d_status, 4), overlap,
                                         _stream(stream))


def hparams_ref(hp: AdamHP):
    """The C struct of hp, by reference, for prepared calls (build once per step)."""
    return C.byref(hp._c())


def status_ptr(d_status) -> int:
    return _ptr(d_status, 4)


def stream_handle(stream=None) -> int:
    return _stream(stream)


def zero_adam_consts_for_step(hp: AdamHP, step: int) -> AdamConsts:
    out = AdamConsts()
    h = hp._c()
    _check(_lib.zero_adam_consts_for_step(C.byref(h), step, C.byref(out)),
           "zero_adam_consts_for_step")
    return out


def zero_adam_shard_dc(n: int, grad, master, m, v, param_out, d_consts, d_status, stream=None):
    _check(_lib.zero_adam_shard_dc(n, _ptr(grad, 4), _ptr(master, 4), _ptr(m, 4), _ptr(v, 4),
                                   _ptr(param_out, 2), _ptr(d_consts), _ptr(d_status, 4),
                                   _stream(stream)), "zero_adam_shard_dc")


def zero_step_fused_dc(n: int, nd: int, rank_grads, master_in, m_in, v_in, master_out, m_out,
                       v_out, param_out, d_consts, d_status, stream=None):
    _check(_lib.zero_step_fused_dc(n, nd, _ptr_array(rank_grads, 2), _ptr(master_in, 4),
                                   _ptr(m_in, 4), _ptr(v_in, 4), _ptr(master_out, 4),
                                   _ptr(m_out, 4), _ptr(v_out, 4), _ptr(param_out, 2),
                                   _ptr(d_consts), _ptr(d_status, 4), _stream(stream)),
           "zero_step_fused_dc")


def zero_quantize_q8(n: int, grad, payload, stream=None):
    _check(_lib.zero_quantize_q8(n, _ptr(grad, 2), _ptr(payload, 1), _stream(stream)),
           "zero_quantize_q8")


def zero_step_fused_q8(n: int, nd: int, rank_payload, master_in, m_in, v_in, master_out, m_out,
                       v_out, param_out, hp: AdamHP, step: int, d_status, stream=None):
    h = hp._c()
    _check(_lib.zero_step_fused_q8(n, nd, _ptr_array(rank_payload, 1), _ptr(master_in, 4),
                                   _ptr(m_in, 4), _ptr(v_in, 4), _ptr(master_out, 4),
                                   _ptr(m_out, 4), _ptr(v_out, 4), _ptr(param_out, 2),
                                   C.byref(h), step, _ptr(d_status, 4), _stream(stream)),
           "zero_step_fused_q8")


def zero_step_fused_q8_dc(n: int, nd: int, rank_payload, master_in, m_in, v_in, master_out,
                          m_out, v_out, param_out, d_consts, d_status, stream=None):
    _check(_lib.zero_step_fused_q8_dc(n, nd, _ptr_array(rank_payload, 1), _ptr(master_in, 4),
                                      _ptr(m_in, 4), _ptr(v_in, 4), _ptr(master_out, 4),
                                      _ptr(m_out, 4), _ptr(v_out, 4), _ptr(param_out, 2),
                                      _ptr(d_consts), _ptr(d_status, 4), _stream(stream)),
           "zero_step_fused_q8_dc")


def zero_step_commit(n: int, master_in, m_in, v_in, master_out, m_out, v_out, param_out,
                     d_status, stream=None):
    _check(_lib.zero_step_commit(n, _ptr(master_in, 4), _ptr(m_in, 4), _ptr(v_in, 4),
                                 _ptr(master_out, 4), _ptr(m_out, 4), _ptr(v_out, 4),
                                 _ptr(param_out, 2), _ptr(d_status, 4), _stream(stream)),
           "zero_step_commit")


def zero_step_status(d_status, stream=None):
    """Blocks until `stream` is done; returns (zero_status code, flags)."""
    flags = C.c_uint32()
    code = _lib.zero_step_status(_ptr(d_status, 4), _stream(stream), C.byref(flags))
    return int(code), int(flags.value)


def zero_adam_consts_table(hp: AdamHP, first_step: int, count: int):
    out = (AdamConsts * max(count, 1))()
    h = hp._c()
    _check(_lib.zero_adam_consts_table(C.byref(h), first_step, count, out),
           "zero_adam_consts_table")
    return out


def zero_scaler_prepare(d_state, d_table, table_len: int, d_consts, d_status, stream=None):
    _check(_lib.zero_scaler_prepare(_ptr(d_state), _ptr(d_table), table_len, _ptr(d_consts),
                                    _ptr(d_status, 4), _stream(stream)), "zero_scaler_prepare")


def zero_scaler_update(d_state, params: ScalerParams, d_status, stream=None):
    _check(_lib.zero_scaler_update(_ptr(d_state), C.byref(params), _ptr(d_status, 4),
                                   _stream(stream)), "zero_scaler_update")


def zero_selftest_timeout(d_status, stream=None):
    _check(_lib.zero_selftest_timeout(_ptr(d_status, 4), _stream(stream)), "zero_selftest_timeout")


def zero_gather_params(plan: Plan, flat_lo: int, length: int, param_shards, out, d_status,
                       stream=None):
    _check(_lib.zero_gather_params(plan.handle, flat_lo, length, _ptr_array(param_shards, 2),
                                   _ptr(out, 2), _ptr(d_status, 4), _stream(stream)),
           "zero_gather_params")


def zero_stage3_step_fused(plan: Plan, flat_lo: int, length: int, rank_grads, master_in, m_in, v_in,
                     master_out, m_out, v_out, param_shards, hp: AdamHP, step: int, d_status,
                     stream=None):
    h = hp._c()
    _check(_lib.zero_stage3_step_fused(plan.handle, flat_lo, length, _ptr_array(rank_grads, 2),
                                 _ptr(master_in, 4), _ptr(m_in, 4), _ptr(v_in, 4),
                                 _ptr(master_out, 4), _ptr(m_out, 4), _ptr(v_out, 4),
                                 _ptr_array(param_shards, 2), C.byref(h), step,
                                 _ptr(d_status, 4), _stream(stream)), "zero_stage3_step_fused")


def zero_stage3_step_fused_dc(plan: Plan, flat_lo: int, length: int, rank_grads, master_in,
                              m_in, v_in, master_out, m_out, v_out, param_shards, d_consts,
                              d_status, stream=None):
    _check(_lib.zero_stage3_step_fused_dc(plan.handle, flat_lo, length,
                                          _ptr_array(rank_grads, 2), _ptr(master_in, 4),
                                          _ptr(m_in, 4), _ptr(v_in, 4), _ptr(master_out, 4),
                                          _ptr(m_out, 4), _ptr(v_out, 4),
                                          _ptr_array(param_shards, 2), _ptr(d_consts),
                                          _ptr(d_status, 4), _stream(stream)),
           "zero_stage3_step_fused_dc")


def zero_stage3_payload_bytes_q8(plan: Plan, flat_lo: int, length: int) -> int:
    out = C.c_uint64()
    _check(_lib.zero_stage3_payload_bytes_q8(plan.handle, flat_lo, length, C.byref(out)),
           "zero_stage3_payload_bytes_q8")
    return out.value


def zero_stage3_quantize_q8(plan: Plan, flat_lo: int, length: int, grad, payload, stream=None):
    _check(_lib.zero_stage3_quantize_q8(plan.handle, flat_lo, length, _ptr(grad, 2),
                                        _ptr(payload, 1), _stream(stream)),
           "zero_stage3_quantize_q8")


def zero_stage3_step_fused_q8(plan: Plan, flat_lo: int, length: int, rank_payload, master_in,
                              m_in, v_in, master_out, m_out, v_out, param_shards, hp: AdamHP,
                              step: int, d_status, stream=None):
    h = hp._c()
    _check(_lib.zero_stage3_step_fused_q8(plan.handle, flat_lo, length,
                                          _ptr_array(rank_payload, 1), _ptr(master_in, 4),
                                          _ptr(m_in, 4), _ptr(v_in, 4), _ptr(master_out, 4),
                                          _ptr(m_out, 4), _ptr(v_out, 4),
                                          _ptr_array(param_shards, 2), C.byref(h), step,
                                          _ptr(d_status, 4), _stream(stream)),
           "zero_stage3_step_fused_q8")


def zero_stage3_step_fused_q8_dc(plan: Plan, flat_lo: int, length: int, rank_payload,
                                 master_in, m_in, v_in, master_out, m_out, v_out, param_shards,
                                 d_consts, d_status, stream=None):
    _check(_lib.zero_stage3_step_fused_q8_dc(plan.handle, flat_lo, length,
                                             _ptr_array(rank_payload, 1), _ptr(master_in, 4),
                                             _ptr(m_in, 4), _ptr(v_in, 4), _ptr(master_out, 4),
                                             _ptr(m_out, 4), _ptr(v_out, 4),
                                             _ptr_array(param_shards, 2), _ptr(d_consts),
                                             _ptr(d_status, 4), _stream(stream)),
           "zero_stage3_step_fused_q8_dc")


class PreparedStage3Update:
    """zero_stage3_step_fused with its pointer arguments marshalled once (e.g. one layer's
    update in one ping-pong direction); calling it with the step's hyperparameters (hparams_ref),
    step, status address and stream handle makes the same C call."""

    def __init__(self, plan: Plan, flat_lo: int, length: int, rank_grads, master_in, m_in, v_in,
                 master_out, m_out, v_out, param_shards):
        self._plan = plan                                     # kept alive with the handle
        self._grads = _ptr_array(rank_grads, 2)
        self._shards = _ptr_array(param_shards, 2)
        self._args = (plan.handle, flat_lo, length, self._grads, _ptr(master_in, 4),
                      _ptr(m_in, 4), _ptr(v_in, 4), _ptr(master_out, 4), _ptr(m_out, 4),
                      _ptr(v_out, 4), self._shards)

    def __call__(self, hp_ref, step: int, d_status: int, stream: int):
        code = _lib.zero_stage3_step_fused(*self._args, hp_ref, step, d_status, stream)
        if code:
            raise ZeroError(code, "zero_stage3_step_fused")


def zero_stage3_step_commit(plan: Plan, master_in, m_in, v_in, master_out, m_out, v_out, param_shards,
                      d_status, stream=None):
    _check(_lib.zero_stage3_step_commit(plan.handle, _ptr(master_in, 4), _ptr(m_in, 4), _ptr(v_in, 4),
                                  _ptr(master_out, 4), _ptr(m_out, 4), _ptr(v_out, 4),
                                  _ptr_array(param_shards, 2), _ptr(d_status, 4),
                                  _stream(stream)), "zero_stage3_step_commit")


def zero_overlap_begin(stream=None):
    _check(_lib.zero_overlap_begin(_stream(stream)), "zero_overlap_begin")


def zero_overlap_end(stream=None):
    _check(_lib.zero_overlap_end(_stream(stream)), "zero_overlap_end")


class overlap:
    """Context manager: zero_overlap_begin(stream) ... zero_overlap_end(stream)."""

    def __init__(self, stream=None):
        self.stream = _stream(stream)

    def __enter__(self):
        zero_overlap_begin(self.stream)
        return self

    def __exit__(self, *exc):
        zero_overlap_end(self.stream)
        return False


# ---------------------------------------------------------------------------------------------
# stage-2 bucket scheduler
# ---------------------------------------------------------------------------------------------
class Sched:
    def __init__(self, handle: int, nd: int):
        self.handle = handle
        self.nd = nd

    def __del__(self):
        if getattr(self, "handle", None):
            _lib.zero_sched_destroy(self.handle)
            self.handle = None


def zero_sched_slot_elems(plan: Plan, n_slots: int) -> int:
    out = C.c_uint64()
    _check(_lib.zero_sched_slot_elems(plan.handle, n_slots, C.byref(out)),
           "zero_sched_slot_elems")
    return out.value


def zero_sched_create(plan: Plan, slot_mem, slot_mem_elems: int, n_slots: int,
                      owner_grad_shards, d_status, rs_stream=None) -> Sched:
    h = C.c_void_p()
    _check(_lib.zero_sched_create(plan.handle, _ptr(slot_mem, 2), slot_mem_elems, n_slots,
                                  _ptr_array(owner_grad_shards, 4), _ptr(d_status, 4),
                                  _stream(rs_stream), C.byref(h)), "zero_sched_create")
    return Sched(h.value, len(owner_grad_shards))


def zero_sched_create_fused(plan: Plan, slot_mem, slot_mem_elems: int, n_slots: int,
                            master_in, m_in, v_in, master_out, m_out, v_out, param_out,
                            d_consts, d_status, stream=None) -> Sched:
    h = C.c_void_p()
    _check(_lib.zero_sched_create_fused(plan.handle, _ptr(slot_mem, 2), slot_mem_elems, n_slots,
                                        _ptr(master_in, 4), _ptr(m_in, 4), _ptr(v_in, 4),
                                        _ptr(master_out, 4), _ptr(m_out, 4), _ptr(v_out, 4),
                                        _ptr(param_out, 2), _ptr(d_consts), _ptr(d_status, 4),
                                        _stream(stream), C.byref(h)), "zero_sched_create_fused")
    _, psi_p, shard, _ = zero_plan_info(plan)
    return Sched(h.value, psi_p // shard if shard else 1)


def zero_sched_slot_bytes_q8(plan: Plan, n_slots: int) -> int:
    out = C.c_uint64()
    _check(_lib.zero_sched_slot_bytes_q8(plan.handle, n_slots, C.byref(out)),
           "zero_sched_slot_bytes_q8")
    return out.value


def zero_sched_create_fused_q8(plan: Plan, slot_mem, slot_mem_bytes: int, n_slots: int,
                               master_in, m_in, v_in, master_out, m_out, v_out, param_out,
                               d_consts, d_status, stream=None) -> Sched:
    h = C.c_void_p()
    _check(_lib.zero_sched_create_fused_q8(plan.handle, _ptr(slot_mem, 1), slot_mem_bytes,
                                           n_slots, _ptr(master_in, 4), _ptr(m_in, 4),
                                           _ptr(v_in, 4), _ptr(master_out, 4), _ptr(m_out, 4),
                                           _ptr(v_out, 4), _ptr(param_out, 2), _ptr(d_consts),
                                           _ptr(d_status, 4), _stream(stream), C.byref(h)),
           "zero_sched_create_fused_q8")
    _, psi_p, shard, _ = zero_plan_info(plan)
    return Sched(h.value, psi_p // shard if shard else 1)


def zero_sched_begin_bucket_q8(s: Sched, k: int, producer=None) -> List[int]:
    out = (C.c_void_p * s.nd)()
    _check(_lib.zero_sched_begin_bucket_q8(s.handle, k, _stream(producer), out),
           "zero_sched_begin_bucket_q8")
    return [int(p) for p in out]


def zero_sched_rebind_fused(s: Sched, master_in, m_in, v_in, master_out, m_out, v_out,
                            param_out, d_status):
    _check(_lib.zero_sched_rebind_fused(s.handle, _ptr(master_in, 4), _ptr(m_in, 4),
                                        _ptr(v_in, 4), _ptr(master_out, 4), _ptr(m_out, 4),
                                        _ptr(v_out, 4), _ptr(param_out, 2), _ptr(d_status, 4)),
           "zero_sched_rebind_fused")


def zero_sched_rebind_status(s: Sched, d_status):
    _check(_lib.zero_sched_rebind_status(s.handle, _ptr(d_status, 4)), "zero_sched_rebind_status")


def zero_sched_begin_bucket(s: Sched, k: int, producer=None) -> List[int]:
    out = (C.c_void_p * s.nd)()
    _check(_lib.zero_sched_begin_bucket(s.handle, k, _stream(producer), out),
           "zero_sched_begin_bucket")
    return [int(p) for p in out]


def zero_sched_end_bucket(s: Sched, k: int, producer=None):
    _check(_lib.zero_sched_end_bucket(s.handle, k, _stream(producer)), "zero_sched_end_bucket")


def zero_sched_wait(s: Sched, stream=None):
    _check(_lib.zero_sched_wait(s.handle, _stream(stream)), "zero_sched_wait")


def zero_sched_launches(s: Sched) -> int:
    out = C.c_uint64()
    _check(_lib.zero_sched_launches(s.handle, C.byref(out)), "zero_sched_launches")
    return out.value


class LayerSched:
    """Handle of a stage-3 layer scheduler (destroyed with this object)."""

    def __init__(self, handle: int, n_layers: int):
        self.handle = handle
        self.n_layers = n_layers
        self._out = C.c_void_p()

    def __del__(self):
        if getattr(self, "handle", None):
            _lib.zero_layer_sched_destroy(self.handle)
            self.handle = None


def zero_layer_sched_buf_elems(plan: Plan, layer_bounds, n_bufs: int) -> int:
    b = (C.c_uint64 * len(layer_bounds))(*layer_bounds)
    out = C.c_uint64()
    _check(_lib.zero_layer_sched_buf_elems(plan.handle, len(layer_bounds) - 1, b, n_bufs,
                                           C.byref(out)), "zero_layer_sched_buf_elems")
    return out.value


def zero_layer_sched_create(plan: Plan, layer_bounds, param_shards, buf_mem, buf_mem_elems: int,
                            n_bufs: int, gather_stream=None) -> LayerSched:
    b = (C.c_uint64 * len(layer_bounds))(*layer_bounds)
    h = C.c_void_p()
    _check(_lib.zero_layer_sched_create(plan.handle, len(layer_bounds) - 1, b,
                                        _ptr_array(param_shards, 2), _ptr(buf_mem, 2),
                                        buf_mem_elems, n_bufs, _stream(gather_stream),
                                        C.byref(h)), "zero_layer_sched_create")
    return LayerSched(h.value, len(layer_bounds) - 1)


def zero_layer_sched_begin_step(s: LayerSched, d_status, stream=None):
    _check(_lib.zero_layer_sched_begin_step(s.handle, _ptr(d_status, 4), _stream(stream)),
           "zero_layer_sched_begin_step")


def zero_layer_sched_acquire(s: LayerSched, layer: int, prefetch: int = -1,
                             compute=None) -> int:
    """Returns the device address of the layer's gathered fp16 values."""
    _check(_lib.zero_layer_sched_acquire(s.handle, layer, prefetch, _stream(compute),
                                         C.byref(s._out)), "zero_layer_sched_acquire")
    return int(s._out.value)


def zero_layer_sched_release(s: LayerSched, layer: int, compute=None):
    _check(_lib.zero_layer_sched_release(s.handle, layer, _stream(compute)),
           "zero_layer_sched_release")


def zero_layer_sched_gathers(s: LayerSched) -> int:
    out = C.c_uint64()
    _check(_lib.zero_layer_sched_gathers(s.handle, C.byref(out)), "zero_layer_sched_gathers")
    return out.value


def zero_sched_destroy(s: Sched):
    if s.handle:
        _lib.zero_sched_destroy(s.handle)
        s.handle = None
