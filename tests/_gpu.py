"""Helpers for the GPU parity tests: buffers, calls through the C ABI, and ulp comparisons
against the oracle. Test infrastructure only."""
import numpy as np
import torch

import oracle
from zero_partitioned_optimizer_plan_b200 import build as zbuild

zbuild.build()
from zero_partitioned_optimizer_plan_b200 import libzero as lz  # noqa: E402

DEV = "cuda:0"
TOL_F32_ULP = 2    # fp32 master, m, v
TOL_F16_ULP = 1    # fp16 parameters

HP = lz.AdamHP()
ORC_HP = oracle.AdamHP()


def require_gpu():
    if not torch.cuda.is_available():
        raise RuntimeError("GPU test run without a CUDA device")


def status_word():
    return torch.zeros(1, dtype=torch.int32, device=DEV)


def status_flags(st) -> int:
    return int(st.item()) & 0xffffffff


def f16np(t) -> np.ndarray:
    """uint16 bits of a float16 tensor."""
    return t.detach().cpu().numpy().view(np.uint16)


def f32np(t) -> np.ndarray:
    return t.detach().cpu().numpy()


def check_f32(name, got, want, tol=TOL_F32_ULP) -> int:
    d = oracle.ulp_diff_f32(got, want)
    worst = int(d.max()) if d.size else 0
    if worst > tol:
        i = int(d.argmax())
        raise AssertionError(f"{name}: {worst} ulp at {i}: got {np.float32(got[i])!r} "
                             f"want {np.float32(want[i])!r}")
    return worst


def check_f16(name, got, want, tol=TOL_F16_ULP) -> int:
    d = oracle.ulp_diff_f16(got, want)
    worst = int(d.max()) if d.size else 0
    if worst > tol:
        i = int(d.argmax())
        raise AssertionError(f"{name}: {worst} ulp at {i}: got {hex(int(got[i]))} "
                             f"want {hex(int(want[i]))}")
    return worst


def check_bitexact_f32(name, got, want):
    g = np.ascontiguousarray(got, np.float32).view(np.uint32)
    w = np.ascontiguousarray(want, np.float32).view(np.uint32)
    bad = np.nonzero(g != w)[0]
    if bad.size:
        i = int(bad[0])
        raise AssertionError(f"{name}: {bad.size} values differ, first at {i}: "
                             f"got {hex(int(g[i]))} want {hex(int(w[i]))}")


class PingPong:
    """fp32 master/m/v in two device copies: zero_step_fused reads one and writes the other."""

    def __init__(self, master, m, v):
        self.cur = [x.to(DEV).contiguous() for x in (master, m, v)]
        self.nxt = [torch.empty_like(x) for x in self.cur]

    def swap(self):
        self.cur, self.nxt = self.nxt, self.cur

    def numpy(self):
        return [f32np(x) for x in self.cur]


def fused_step(n, grads, pp: PingPong, params, hp, t, status, stream=None, lo=0):
    """One stage-1 step through the C ABI over elements [lo, lo+n) of the state arrays."""
    ins = [x[lo:lo + n] for x in pp.cur]
    outs = [x[lo:lo + n] for x in pp.nxt]
    lz.zero_step_fused(n, len(grads), grads, *ins, *outs, params, hp, t, status, stream)
    lz.zero_step_commit(n, *ins, *outs, params, status, stream)
