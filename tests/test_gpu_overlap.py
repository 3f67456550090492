"""Launch overlap (programmatic dependent launch) against the oracle.

Every bulk-copy kernel is launched so that it may be scheduled while the previous kernel on the
stream drains; outside a zero_overlap_begin/end region it must still wait for that kernel, so
back-to-back calls that depend on each other give the oracle's sequential result. Inside a
region the per-bucket calls of one step run alongside one another; the step (with bucket
ranges that take the plain-load kernels, an overflow, graph capture, the reduce-scatter and the
int8-payload calls) still equals the oracle's step. Same tolerances as the other parity tests."""
import numpy as np
import pytest
import torch

import oracle
from tests._gpu import (DEV, HP, ORC_HP, PingPong, check_bitexact_f32, check_f16, check_f32,
                        f16np, f32np, lz, require_gpu, status_flags, status_word)
from zero_partitioned_optimizer_plan_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True, scope="module")
def _gpu():
    require_gpu()
    torch.cuda.set_device(0)
    yield
    torch.cuda.synchronize()
    torch.cuda.empty_cache()


def _grads(n, nd, seed, step):
    return [synth.grad_f16(n, 1e-3, seed=seed, rank=r, step=step) for r in range(nd)]


def _buckets(n, sizes):
    """Ranges of the given lengths (cycled) from the start of [0, n), the last one short,
    listed in backward order."""
    out, lo, i = [], 0, 0
    while lo < n:
        hi = min(n, lo + sizes[i % len(sizes)])
        out.append((lo, hi))
        lo, i = hi, i + 1
    return out[::-1]


def test_dependent_calls_back_to_back_stay_ordered():
    """Five steps, each one zero_step_fused call reading the previous call's outputs and
    writing over its inputs, enqueued with nothing in between. Each step uses another Nd, so
    each launch tiles the range differently (16, 20 or 24 consumer warps): a kernel that ran
    ahead of its predecessor would read state rows another CTA has not written yet."""
    n = 1 << 21
    nds = [8, 2, 64, 3, 16]
    master, m, v = synth.state_warm(n, seed=501)
    pp = PingPong(master, m, v)
    params = torch.empty(n, dtype=torch.float16, device=DEV)
    g_cpu = [_grads(n, nd, 502, t + 1) for t, nd in enumerate(nds)]
    g_dev = [[g.to(DEV) for g in gs] for gs in g_cpu]
    st = status_word()
    torch.cuda.synchronize()
    for t, nd in enumerate(nds):
        lz.zero_step_fused(n, nd, g_dev[t], *pp.cur, *pp.nxt, params, HP, t + 1, st)
        pp.swap()
    torch.cuda.synchronize()
    assert status_flags(st) == 0
    w, mm, vv = master.numpy(), m.numpy(), v.numpy()
    for t, nd in enumerate(nds):
        skipped, w, mm, vv, p = oracle.step([g.numpy() for g in g_cpu[t]], w, mm, vv, ORC_HP,
                                            t + 1)
        assert not skipped
    got = pp.numpy()
    check_f32("master", got[0], w)
    check_f32("m", got[1], mm)
    check_f32("v", got[2], vv)
    check_f16("params", f16np(params), p)


@pytest.mark.parametrize("nd", [2, 8, 64])
def test_region_of_bucket_calls_vs_oracle(nd):
    """One step as per-bucket zero_step_fused calls inside a region: bulk-copy ranges with and
    without a ragged tail, a range on unaligned pointers and a one-element range (plain-load
    kernel) between them; three steps; then a NaN in a middle bucket skips the whole step."""
    n = 3072 * 40 + 13
    cuts = [0, 21504, 25603, 25703, 25704, 34928, 61440, 90000, n]
    bounds = [(a, b) for a, b in zip(cuts[:-1], cuts[1:])][::-1]
    master, m, v = synth.state_warm(n, seed=510 + nd)
    pp = PingPong(master, m, v)
    params = torch.empty(n, dtype=torch.float16, device=DEV)
    w, mm, vv = master.numpy(), m.numpy(), v.numpy()
    for t in (1, 2, 3):
        g_cpu = _grads(n, nd, 511, t)
        g_dev = [g.to(DEV) for g in g_cpu]
        st = status_word()
        with lz.overlap():
            for lo, hi in bounds:
                lz.zero_step_fused(hi - lo, nd, [g[lo:hi] for g in g_dev],
                                   *[x[lo:hi] for x in pp.cur], *[x[lo:hi] for x in pp.nxt],
                                   params[lo:hi], HP, t, st)
        lz.zero_step_commit(n, *pp.cur, *pp.nxt, params, st)
        torch.cuda.synchronize()
        assert status_flags(st) == 0
        pp.swap()
        skipped, w, mm, vv, p = oracle.step([g.numpy() for g in g_cpu], w, mm, vv, ORC_HP, t)
        got = pp.numpy()
        check_f32(f"step {t} master", got[0], w)
        check_f32(f"step {t} m", got[1], mm)
        check_f32(f"step {t} v", got[2], vv)
        check_f16(f"step {t} params", f16np(params), p)
    # overflow in a bucket in the middle of the region: the step is skipped everywhere
    g_dev = [g.to(DEV) for g in _grads(n, nd, 511, 4)]
    lo_mid = bounds[2][0] + 77            # a bulk-copy range chained to the ones before it
    g_dev[nd - 1][lo_mid] = float("nan")
    st = status_word()
    with lz.overlap():
        for lo, hi in bounds:
            lz.zero_step_fused(hi - lo, nd, [g[lo:hi] for g in g_dev],
                               *[x[lo:hi] for x in pp.cur], *[x[lo:hi] for x in pp.nxt],
                               params[lo:hi], HP, 4, st)
    lz.zero_step_commit(n, *pp.cur, *pp.nxt, params, st)
    assert lz.zero_step_status(st)[0] == lz.ZERO_STEP_SKIPPED
    for a, b in zip(pp.cur, pp.nxt):
        assert torch.equal(a, b)
    assert np.array_equal(f16np(params), oracle.f2h(w))


def test_consecutive_regions_are_ordered():
    """Step t+1's region reads what step t's region wrote, with no commit or other kernel in
    between: the first call of a region waits for everything before it."""
    nd, n = 8, 3072 * 60 + 5
    bounds = _buckets(n, [3072 * 5, 3072 * 4 + 16])
    master, m, v = synth.state_warm(n, seed=520)
    pp = PingPong(master, m, v)
    params = torch.empty(n, dtype=torch.float16, device=DEV)
    g_cpu = [_grads(n, nd, 521, t) for t in (1, 2, 3, 4)]
    g_dev = [[g.to(DEV) for g in gs] for gs in g_cpu]
    st = status_word()
    torch.cuda.synchronize()
    for t in (1, 2, 3, 4):
        with lz.overlap():
            # alternate the walk direction so consecutive regions tile differently
            for lo, hi in (bounds if t % 2 else bounds[::-1]):
                lz.zero_step_fused(hi - lo, nd, [g[lo:hi] for g in g_dev[t - 1]],
                                   *[x[lo:hi] for x in pp.cur], *[x[lo:hi] for x in pp.nxt],
                                   params[lo:hi], HP, t, st)
        pp.swap()
    torch.cuda.synchronize()
    assert status_flags(st) == 0
    w, mm, vv = master.numpy(), m.numpy(), v.numpy()
    for t in (1, 2, 3, 4):
        skipped, w, mm, vv, p = oracle.step([g.numpy() for g in g_cpu[t - 1]], w, mm, vv,
                                            ORC_HP, t)
    got = pp.numpy()
    check_f32("master", got[0], w)
    check_f32("m", got[1], mm)
    check_f32("v", got[2], vv)
    check_f16("params", f16np(params), p)


def test_region_captured_in_graph():
    """Per-bucket zero_step_fused_dc calls inside a region plus the commit, captured as CUDA
    graphs (one per ping-pong direction) and replayed for t = 1..4 equal the oracle."""
    nd, n = 4, 2560 * 48 + 9
    bounds = _buckets(n, [2560 * 3, 8192, 2560 * 2 + 8])
    master, m, v = synth.state_warm(n, seed=530)
    bufs = [[x.to(DEV) for x in (master, m, v)], [torch.empty(n, device=DEV) for _ in range(3)]]
    grads = [torch.empty(n, dtype=torch.float16, device=DEV) for _ in range(nd)]
    params = torch.empty(n, dtype=torch.float16, device=DEV)
    dc = torch.empty(lz.ZERO_ADAM_CONSTS_BYTES, dtype=torch.uint8, device=DEV)
    st = status_word()
    flags = status_word()

    def consts(t):
        c = lz.zero_adam_consts_for_step(HP, t)
        return torch.frombuffer(bytearray(bytes(c)), dtype=torch.uint8).to(DEV)

    def step(src, dst):
        st.zero_()
        with lz.overlap():
            for lo, hi in bounds:
                lz.zero_step_fused_dc(hi - lo, nd, [g[lo:hi] for g in grads],
                                      *[x[lo:hi] for x in src], *[x[lo:hi] for x in dst],
                                      params[lo:hi], dc, st)
        lz.zero_step_commit(n, *src, *dst, params, st)
        flags.bitwise_or_(st)

    dc.copy_(consts(1))
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
    flags.zero_()
    w, mm, vv = master.numpy(), m.numpy(), v.numpy()
    for t in (1, 2, 3, 4):
        g_cpu = _grads(n, nd, 531, t)
        for d, s in zip(grads, g_cpu):
            d.copy_(s.to(DEV))
        dc.copy_(consts(t))
        graphs[(t - 1) % 2].replay()
        torch.cuda.synchronize()
        assert status_flags(flags) == 0
        skipped, w, mm, vv, p = oracle.step([g.numpy() for g in g_cpu], w, mm, vv, ORC_HP, t)
        out = bufs[t % 2]
        check_f32(f"step {t} master", f32np(out[0]), w)
        check_f32(f"step {t} m", f32np(out[1]), mm)
        check_f32(f"step {t} v", f32np(out[2]), vv)
        check_f16(f"step {t} params", f16np(params), p)
    del graphs


@pytest.mark.parametrize("nd", [3, 16])
def test_region_of_reduce_scatter_buckets(nd):
    """Every bucket's zero_reduce_scatter_bucket inside one region, then the owners' updates:
    the reduced shards are bit-exact and the state equals the oracle's stage-2 step."""
    numels = [70001, 4099, 12345, 300000]
    bucket = 9000
    pl = lz.zero_plan_create(numels, nd, 2, bucket)
    psi, psi_p, S, nb = lz.zero_plan_info(pl)
    ref_plan = oracle.plan(numels, nd, bucket)
    g_cpu = []
    for r in range(nd):
        g = torch.zeros(psi_p, dtype=torch.float16)
        g[:psi] = synth.grad_f16(psi, 1e-3, seed=540, rank=r, step=1)
        g_cpu.append(g)
    g_dev = [g.to(DEV) for g in g_cpu]
    master = torch.zeros(psi_p)
    master[:psi] = synth.normal_f32(psi, 0.02, seed=541)
    m = torch.zeros(psi_p)
    v = torch.zeros(psi_p)
    shards = torch.empty(psi_p, dtype=torch.float32, device=DEV)
    views = [shards[r * S:(r + 1) * S] for r in range(nd)]
    st = status_word()
    with lz.overlap():
        for k in range(nb):
            lo, ln, _, _ = lz.zero_plan_bucket(pl, k)
            lz.zero_reduce_scatter_bucket(pl, k, [g[lo:lo + ln] for g in g_dev], views, st)
    dm, dmm, dv = master.to(DEV), m.to(DEV), v.to(DEV)
    params = torch.zeros(psi_p, dtype=torch.float16, device=DEV)
    for r in range(nd):
        sl = slice(r * S, (r + 1) * S)
        lz.zero_adam_shard(S, shards[sl], dm[sl], dmm[sl], dv[sl], params[sl], HP, 1, st)
    ref = oracle.zero2_step(ref_plan, lambda k, r: g_cpu[r].numpy()[
        ref_plan.buckets[k][0]:sum(ref_plan.buckets[k])], master.numpy(), m.numpy(), v.numpy(),
        oracle.f2h(master.numpy()), ORC_HP, 1)
    torch.cuda.synchronize()
    assert status_flags(st) == 0 and not ref.skipped
    check_bitexact_f32("reduced grad", f32np(shards), ref.reduced)
    check_f32("master", f32np(dm), ref.master)
    check_f32("m", f32np(dmm), ref.m)
    check_f32("v", f32np(dv), ref.v)
    check_f16("params", f16np(params), ref.params16)


def test_region_of_q8_bucket_calls():
    """Per-bucket zero_step_fused_q8 calls inside a region (each bucket's payload quantized from
    its own range, as the senders would) equal the oracle's per-bucket owner steps."""
    nd, n = 8, 3072 * 30 + 640
    bounds = _buckets(n, [3072 * 4, 3072 * 2 + 512, 1000])
    g_cpu = _grads(n, nd, 550, 1)
    master, m, v = synth.state_warm(n, seed=551)
    pp = PingPong(master, m, v)
    params = torch.empty(n, dtype=torch.float16, device=DEV)
    pays = {}
    for lo, hi in bounds:
        pays[lo] = []
        for g in g_cpu:
            pay = torch.empty(lz.q8_payload_bytes(hi - lo), dtype=torch.uint8, device=DEV)
            lz.zero_quantize_q8(hi - lo, g[lo:hi].to(DEV), pay)
            pays[lo].append(pay)
    st = status_word()
    torch.cuda.synchronize()
    with lz.overlap():
        for lo, hi in bounds:
            lz.zero_step_fused_q8(hi - lo, nd, pays[lo], *[x[lo:hi] for x in pp.cur],
                                  *[x[lo:hi] for x in pp.nxt], params[lo:hi], HP, 1, st)
    lz.zero_step_commit(n, *pp.cur, *pp.nxt, params, st)
    torch.cuda.synchronize()
    assert status_flags(st) == 0
    w, mm, vv = master.numpy().copy(), m.numpy().copy(), v.numpy().copy()
    p = np.empty(n, np.uint16)
    for lo, hi in bounds:
        ref = [oracle.quant_q8(g.numpy()[lo:hi]) for g in g_cpu]
        skipped, w[lo:hi], mm[lo:hi], vv[lo:hi], p[lo:hi] = oracle.step_q8(
            [q for q, _ in ref], [s for _, s in ref], w[lo:hi], mm[lo:hi], vv[lo:hi], ORC_HP, 1)
        assert not skipped
    got = [f32np(x) for x in pp.nxt]
    check_f32("master", got[0], w)
    check_f32("m", got[1], mm)
    check_f32("v", got[2], vv)
    check_f16("params", f16np(params), p)
