"""Dynamic loss scaling on the device: a sequence of steps with overflows injected, run with
no host read between steps (eagerly, and as CUDA-graph replays), against the oracle's scaled
steps and scaler. Tolerances as in test_gpu_parity.py."""
import ctypes as C

import numpy as np
import pytest
import torch

import oracle
from tests._gpu import (DEV, HP, ORC_HP, check_f16, check_f32, f16np, f32np, lz, require_gpu,
                        status_word)
from zero_partitioned_optimizer_plan_b200 import synth

pytestmark = pytest.mark.gpu

OVERFLOW = [False, False, False, True, True, False, False, False, True, False]


@pytest.fixture(autouse=True)
def _gpu():
    require_gpu()
    torch.cuda.set_device(0)
    yield
    torch.cuda.synchronize()


def _to_dev(struct_obj):
    return torch.frombuffer(bytearray(bytes(struct_obj)), dtype=torch.uint8).to(DEV)


def _state_from_dev(t):
    s = lz.ScalerState()
    C.memmove(C.addressof(s), bytes(t.cpu().numpy().tobytes()), C.sizeof(s))
    return s


def _grads(n, nd, step, bad):
    gs = [synth.grad_f16(n, 1e-2, seed=91, rank=r, step=step) for r in range(nd)]
    if bad:
        gs[nd - 1][n // 3] = float("inf")
    return gs


@pytest.mark.parametrize("init_scale", [1024.0, 1000.0])
@pytest.mark.parametrize("graph", [False, True])
def test_device_scaler_sequence(init_scale, graph):
    nd, n, B = 4, 2048 * 12 + 5, 7000
    interval = 2
    master, m, v = synth.state_warm(n, seed=92)
    bufs = [[x.to(DEV) for x in (master, m, v)], [torch.empty(n, device=DEV) for _ in range(3)]]
    grads = [torch.empty(n, dtype=torch.float16, device=DEV) for _ in range(nd)]
    params = torch.empty(n, dtype=torch.float16, device=DEV)
    table = lz.zero_adam_consts_table(HP, 1, 32)
    d_table = torch.frombuffer(bytearray(bytes(table)), dtype=torch.uint8).to(DEV)
    d_consts = torch.empty(lz.ZERO_ADAM_CONSTS_BYTES, dtype=torch.uint8, device=DEV)
    d_state = _to_dev(lz.ScalerState(init_scale, 0, 1, 0))
    prm = lz.ScalerParams(2.0, 0.5, interval)
    st = status_word()
    bounds, hi = [], n
    while hi > 0:
        bounds.append((max(0, hi - B), hi))
        hi = max(0, hi - B)

    def step(src, dst):
        lz.zero_scaler_prepare(d_state, d_table, 32, d_consts, st)
        for lo, hi in bounds:
            lz.zero_step_fused_dc(hi - lo, nd, [g[lo:hi] for g in grads],
                                  *[x[lo:hi] for x in src], *[x[lo:hi] for x in dst],
                                  params[lo:hi], d_consts, st)
        lz.zero_step_commit(n, *src, *dst, params, st)
        lz.zero_scaler_update(d_state, prm, st)

    graphs = None
    if graph:
        snap = _to_dev(lz.ScalerState(init_scale, 0, 1, 0))
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            step(bufs[0], bufs[1])
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize()
        graphs = []
        for src, dst in ((bufs[0], bufs[1]), (bufs[1], bufs[0])):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                step(src, dst)
            graphs.append(g)
        for x, y in zip(bufs[0], (master, m, v)):
            x.copy_(y.to(DEV))
        d_state.copy_(snap)
        torch.cuda.synchronize()

    sc = oracle.Scaler(scale=init_scale, growth_interval=interval)
    w_r, m_r, v_r = master.numpy(), m.numpy(), v.numpy()
    p_r = None
    for i, bad in enumerate(OVERFLOW):
        g_cpu = _grads(n, nd, i, bad)
        for d, s in zip(grads, g_cpu):
            d.copy_(s.to(DEV), non_blocking=False)
        if graph:
            graphs[i % 2].replay()
        else:
            step(bufs[i % 2], bufs[(i + 1) % 2])
        skipped, w_r, m_r, v_r, p = oracle.scaled_step([g.numpy() for g in g_cpu], w_r, m_r,
                                                       v_r, ORC_HP, sc)
        assert skipped == bad
        if p is not None:
            p_r = p
    torch.cuda.synchronize()
    out = bufs[len(OVERFLOW) % 2]
    check_f32("master", f32np(out[0]), w_r)
    check_f32("m", f32np(out[1]), m_r)
    check_f32("v", f32np(out[2]), v_r)
    check_f16("params", f16np(params), p_r)
    s = _state_from_dev(d_state)
    assert (s.scale, s.good_steps, s.next_step, s.skipped_steps) == \
        (np.float32(sc.scale), sc.good_steps, sc.next_step, sc.skipped_steps)


def test_table_exhausted_refuses_the_step():
    n, nd = 4096 * 2, 2
    table = lz.zero_adam_consts_table(HP, 1, 2)
    d_table = torch.frombuffer(bytearray(bytes(table)), dtype=torch.uint8).to(DEV)
    d_consts = torch.empty(lz.ZERO_ADAM_CONSTS_BYTES, dtype=torch.uint8, device=DEV)
    d_state = _to_dev(lz.ScalerState(1024.0, 0, 3, 0))     # t = 3, the table holds 1..2
    st = status_word()
    cur = [x.to(DEV) for x in synth.state_warm(n, seed=93)]
    nxt = [torch.empty_like(x) for x in cur]
    params = torch.zeros(n, dtype=torch.float16, device=DEV)
    grads = [synth.grad_f16(n, 1e-2, seed=94, rank=r).to(DEV) for r in range(nd)]
    lz.zero_scaler_prepare(d_state, d_table, 2, d_consts, st)
    lz.zero_step_fused_dc(n, nd, grads, *cur, *nxt, params, d_consts, st)
    lz.zero_step_commit(n, *cur, *nxt, params, st)
    lz.zero_scaler_update(d_state, lz.ScalerParams(2.0, 0.5, 10), st)
    code, flags = lz.zero_step_status(st)
    assert code == lz.ZERO_ECUDA and flags & lz.ZERO_FLAG_BOUNDS and flags & lz.ZERO_FLAG_SKIPPED
    for a, b in zip(cur, nxt):
        assert torch.equal(a, b)
    s = _state_from_dev(d_state)
    assert (s.scale, s.good_steps, s.next_step, s.skipped_steps) == (1024.0, 0, 3, 0)
