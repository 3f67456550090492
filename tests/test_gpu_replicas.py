"""The parameter all-gather in the fused step's epilogue (zero_step_fused_replicas and
zero_step_commit_replicas) against the oracle: every replica's range holds the oracle's fp16
parameters (0 ulp) and nothing outside the ranges is written; the same bits as the one-buffer
call; a void step's commit repairs every replica. The replicas here are ranges of local
buffers (one 4- or 8-byte aligned, so the common store width drops) standing for the peers'
full parameter buffers."""
import numpy as np
import pytest
import torch

import oracle
from tests._gpu import (DEV, HP, ORC_HP, PingPong, check_f16, check_f32, f16np, f32np, lz,
                        require_gpu, status_flags, status_word)
from zero_partitioned_optimizer_plan_b200 import synth

pytestmark = pytest.mark.gpu
SENTINEL = 0x7e01      # an fp16 NaN pattern the step never writes


@pytest.fixture(autouse=True)
def _gpu():
    require_gpu()
    torch.cuda.set_device(0)
    yield
    torch.cuda.synchronize()
    torch.cuda.empty_cache()


def _replicas(n, k, skew):
    """k ranges of n fp16 values inside one sentinel-filled buffer; replica 1 starts `skew`
    elements past a 16-byte boundary."""
    stride = (n + 63) // 8 * 8 + 64
    buf = torch.full((k * stride + 64,), SENTINEL, dtype=torch.int16, device=DEV)
    offs = [d * stride + (skew if d == 1 else 0) for d in range(k)]
    return buf, offs, [buf[o:o + n].view(torch.float16) for o in offs]


@pytest.mark.parametrize("skew", [0, 2, 4])
@pytest.mark.parametrize("nd", [2, 8])
@pytest.mark.parametrize("n", [1000, 4096 + 300, 1_900_000 + 77])
def test_replicas_vs_oracle(n, nd, skew):
    """Sizes for the plain kernel (1000), the small-call shape and the large shape."""
    k = 3
    seed = 3 * n + nd + skew
    master, m, v = synth.state_warm(n, seed=seed)
    g_cpu = [synth.grad_f16(n, 1e-3, seed=seed, rank=r, step=1) for r in range(nd)]
    g_dev = [g.to(DEV) for g in g_cpu]
    pp = PingPong(master, m, v)
    buf, offs, reps = _replicas(n, k, skew)
    st = status_word()
    lz.zero_step_fused_replicas(n, nd, g_dev, *pp.cur, *pp.nxt, reps, HP, 1, st)
    lz.zero_step_commit_replicas(n, *pp.cur, *pp.nxt, reps, st)
    one = torch.empty(n, dtype=torch.float16, device=DEV)        # the one-buffer call
    outs1 = [torch.empty_like(x) for x in pp.cur]
    st1 = status_word()
    lz.zero_step_fused(n, nd, g_dev, *pp.cur, *outs1, one, HP, 1, st1)
    torch.cuda.synchronize()
    assert status_flags(st) == 0 and status_flags(st1) == 0
    ref = oracle.dp_step([g.numpy() for g in g_cpu], master.numpy(), m.numpy(), v.numpy(),
                         oracle.f2h(master.numpy()), ORC_HP, 1)
    assert not ref.skipped
    for name, got, want in zip(("master", "m", "v"), pp.nxt, (ref.master, ref.m, ref.v)):
        check_f32(name, f32np(got), want, tol=0)
    host = buf.cpu().numpy().view(np.uint16)
    mask = np.ones(host.size, bool)
    for o in offs:
        check_f16("replica", host[o:o + n], ref.params16, tol=0)
        assert np.array_equal(host[o:o + n], f16np(one))
        mask[o:o + n] = False
    assert (host[mask] == SENTINEL).all()          # nothing outside the replicas
    for a, b in zip(outs1, pp.nxt):
        assert torch.equal(a.view(torch.int32), b.view(torch.int32))


@pytest.mark.parametrize("n", [1000, 1_900_000 + 77])
def test_replicas_void_step_repaired_everywhere(n):
    """An inf in one rank's gradient: the commit restores the state and writes fp16(master_in)
    into every replica (the fused kernel had already written the step's values there)."""
    nd, k = 4, 5
    master, m, v = synth.state_warm(n, seed=77)
    g_dev = [synth.grad_f16(n, 1e-3, seed=78, rank=r, step=1).to(DEV) for r in range(nd)]
    g_dev[2][n // 3] = float("inf")
    pp = PingPong(master, m, v)
    buf, offs, reps = _replicas(n, k, 2)
    st = status_word()
    lz.zero_step_fused_replicas(n, nd, g_dev, *pp.cur, *pp.nxt, reps, HP, 1, st)
    lz.zero_step_commit_replicas(n, *pp.cur, *pp.nxt, reps, st)
    assert lz.zero_step_status(st)[0] == lz.ZERO_STEP_SKIPPED
    for a, b in zip(pp.cur, pp.nxt):
        assert torch.equal(a, b)
    host = buf.cpu().numpy().view(np.uint16)
    want = oracle.f2h(master.numpy())
    for o in offs:
        assert np.array_equal(host[o:o + n], want)


def test_replicas_at_full_fan_out():
    """64 replicas (the ABI's maximum), Nd = 64, a large-shape range."""
    n, nd, k = 300_000, 64, 64
    master, m, v = synth.state_warm(n, seed=90)
    g_cpu = [synth.grad_f16(n, 1e-3, seed=91, rank=r, step=1) for r in range(nd)]
    pp = PingPong(master, m, v)
    buf, offs, reps = _replicas(n, k, 0)
    st = status_word()
    lz.zero_step_fused_replicas(n, nd, [g.to(DEV) for g in g_cpu], *pp.cur, *pp.nxt, reps, HP, 1,
                                st)
    lz.zero_step_commit_replicas(n, *pp.cur, *pp.nxt, reps, st)
    torch.cuda.synchronize()
    assert status_flags(st) == 0
    ref = oracle.dp_step([g.numpy() for g in g_cpu], master.numpy(), m.numpy(), v.numpy(),
                         oracle.f2h(master.numpy()), ORC_HP, 1)
    host = buf.cpu().numpy().view(np.uint16)
    for o in offs:
        check_f16("replica", host[o:o + n], ref.params16, tol=0)
