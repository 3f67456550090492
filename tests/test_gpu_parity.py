"""Parity of the CUDA path (called through the C ABI) with the CPU oracle, element by element,
on seeded inputs that span several tiles and a ragged tail, plus the edge cases: Nd = 1,
non-power-of-two Nd, the largest Nd, pointers without 16-byte alignment, parameter buffers at
2/4/8-byte offsets, overflow anywhere in the range, and the stage-2 bucket scheduler.

Tolerances: reduced gradients bit-exact; fp32 master, m, v within 2 ulp; fp16 parameters
within 1 ulp of the oracle (ulp = distance in the ordered-integer representation)."""
import numpy as np
import pytest
import torch

import oracle
from tests._gpu import (DEV, HP, ORC_HP, PingPong, check_bitexact_f32, check_f16, check_f32,
                        f16np, f32np, fused_step, lz, require_gpu, status_flags, status_word)
from zero_partitioned_optimizer_plan_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True, scope="module")
def _gpu():
    require_gpu()
    torch.cuda.set_device(0)
    yield
    torch.cuda.synchronize()
    torch.cuda.empty_cache()


def _rank_grads_cpu(n, nd, seed, step, sigma=1e-3, spike=0.0):
    return [synth.grad_f16(n, sigma, seed=seed, rank=r, step=step, spike_frac=spike,
                           spike_scale=100.0) for r in range(nd)]


SIZES = [1, 9, 4096, 4101, 20003, 2048 * 150 + 7]
NDS = [1, 2, 3, 4, 7, 8, 9, 16, 24, 25, 33, 64]


@pytest.mark.parametrize("nd", NDS)
@pytest.mark.parametrize("n", SIZES)
def test_fused_step_vs_oracle(n, nd):
    seed = 1000 * nd + n
    master, m, v = synth.state_warm(n, seed=seed)
    pp = PingPong(master, m, v)
    w_ref, m_ref, v_ref = master.numpy(), m.numpy(), v.numpy()
    params = torch.empty(n, dtype=torch.float16, device=DEV)
    worst = [0, 0]
    for t in (1, 2, 3):
        g_cpu = _rank_grads_cpu(n, nd, seed, t)
        g_dev = [g.to(DEV) for g in g_cpu]
        st = status_word()
        fused_step(n, g_dev, pp, params, HP, t, st)
        torch.cuda.synchronize()
        assert status_flags(st) == 0
        pp.swap()
        skipped, w_ref, m_ref, v_ref, p_ref = oracle.step([g.numpy() for g in g_cpu], w_ref,
                                                          m_ref, v_ref, ORC_HP, t)
        assert not skipped
        w, mm, vv = pp.numpy()
        worst[0] = max(worst[0], check_f32("master", w, w_ref), check_f32("m", mm, m_ref),
                       check_f32("v", vv, v_ref))
        worst[1] = max(worst[1], check_f16("param", f16np(params), p_ref))
    print(f"PARITY fused n={n} nd={nd}: max ulp fp32 {worst[0]}, fp16 {worst[1]}")


def _large_shape_elems(nd):
    """Smallest call that takes the large (per-Nd table) pipeline shape rather than the
    small-call shape, plus a ragged remainder: tiles of 32 * warps * 4 elements, at least 32
    tiles per SM at Nd <= 2 and 4 above."""
    warps = 20 if nd <= 2 else 16 if nd <= 4 else 24 if nd <= 8 else 16 if nd <= 16 else 20
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    return (32 if nd <= 2 else 4) * sms * 32 * warps * 4 + 1000 + 5


@pytest.mark.parametrize("nd", [1, 2, 4, 8, 16, 64])
def test_fused_step_large_shape_vs_oracle(nd):
    """The large shape (full shared-memory budget, 16-24 consumer warps, every SM busy) on
    every element of a call just above its threshold, two steps."""
    n = _large_shape_elems(nd)
    seed = 7000 + nd
    master, m, v = synth.state_warm(n, seed=seed)
    pp = PingPong(master, m, v)
    w_ref, m_ref, v_ref = master.numpy(), m.numpy(), v.numpy()
    params = torch.empty(n, dtype=torch.float16, device=DEV)
    for t in (1, 2):
        g_cpu = _rank_grads_cpu(n, nd, seed, t, spike=0.01)
        st = status_word()
        fused_step(n, [g.to(DEV) for g in g_cpu], pp, params, HP, t, st)
        torch.cuda.synchronize()
        assert status_flags(st) == 0
        pp.swap()
        skipped, w_ref, m_ref, v_ref, p_ref = oracle.step([g.numpy() for g in g_cpu], w_ref,
                                                          m_ref, v_ref, ORC_HP, t)
        w, mm, vv = pp.numpy()
        check_f32("master", w, w_ref)
        check_f32("m", mm, m_ref)
        check_f32("v", vv, v_ref)
        check_f16("param", f16np(params), p_ref)


@pytest.mark.parametrize("nd", [1, 3, 4, 16, 64])
@pytest.mark.parametrize("numels,bucket", [([1000, 37, 4099, 12345], 0),
                                           ([1000, 37, 4099, 12345], 4096),
                                           ([70001, 3], 7),
                                           ([300000, 250000, 250000, 248576], 100000)])
def test_reduce_scatter_and_adam_vs_oracle(numels, bucket, nd):
    """Every owner's reduced shard bit for bit, then the owner updates; the 7-element buckets
    give about 10^4 bucket calls, each touching one or two owners' shards."""
    pl = lz.zero_plan_create(numels, nd, 2, bucket)
    psi, psi_p, S, nb = lz.zero_plan_info(pl)
    ref_plan = oracle.plan(numels, nd, bucket)
    seed = psi + nd
    g_cpu = []
    for r in range(nd):
        g = torch.zeros(psi_p, dtype=torch.float16)
        g[:psi] = synth.grad_f16(psi, 1e-3, seed=seed, rank=r, step=1)
        g_cpu.append(g)
    g_dev = [g.to(DEV) for g in g_cpu]
    master = torch.zeros(psi_p)
    master[:psi] = synth.normal_f32(psi, 0.02, seed=seed)
    m = torch.zeros(psi_p)
    v = torch.zeros(psi_p)
    shards = torch.empty(psi_p, dtype=torch.float32, device=DEV)   # owner r: [r*S, (r+1)*S)
    shard_views = [shards[r * S:(r + 1) * S] for r in range(nd)]
    st = status_word()
    base = [g.data_ptr() for g in g_dev]      # raw addresses: ~10^4 calls stay quick
    shard_ptrs = [x.data_ptr() for x in shard_views]
    for k in range(nb):
        lo, ln, _, _ = lz.zero_plan_bucket(pl, k)
        lz.zero_reduce_scatter_bucket(pl, k, [b + 2 * lo for b in base], shard_ptrs, st)
    ref = oracle.zero2_step(ref_plan, lambda k, r: g_cpu[r].numpy()[
        ref_plan.buckets[k][0]:sum(ref_plan.buckets[k])], master.numpy(), m.numpy(), v.numpy(),
        oracle.f2h(master.numpy()), ORC_HP, 1)
    torch.cuda.synchronize()
    assert status_flags(st) == 0 and not ref.skipped
    check_bitexact_f32("reduced grad", f32np(shards), ref.reduced)
    # owner updates, one call per owner, writing into the full parameter buffer
    dm, dmm, dv = master.to(DEV), m.to(DEV), v.to(DEV)
    params = torch.zeros(psi_p, dtype=torch.float16, device=DEV)
    for r in range(nd):
        sl = slice(r * S, (r + 1) * S)
        lz.zero_adam_shard(S, shards[sl], dm[sl], dmm[sl], dv[sl], params[sl], HP, 1, st)
    torch.cuda.synchronize()
    assert status_flags(st) == 0
    check_f32("master", f32np(dm), ref.master)
    check_f32("m", f32np(dmm), ref.m)
    check_f32("v", f32np(dv), ref.v)
    check_f16("params", f16np(params), ref.params16)


def test_tiny_stage1_workload_three_steps():
    """4 tensors of 300000/250000/250000/248576, Nd = 4, fp16 grads N(0, 0.01^2) per rank,
    master N(0, 0.02^2), m = v = 0, Adam 1e-3/0.9/0.999/1e-8, loss scale 1024, 3 steps; both
    the fused call and the reduce-scatter + owner-update pair against the oracle's stage-1
    step."""
    numels, nd = synth.TINY_LIST, 4
    pl = lz.zero_plan_create(numels, nd, 1, 0)
    psi, psi_p, S, nb = lz.zero_plan_info(pl)
    assert (psi, psi_p, S, nb) == (1048576, 1048576, 262144, 1)
    ref_plan = oracle.plan(numels, nd)
    master, m, v = synth.state_small(psi_p, seed=7)
    pp = PingPong(master, m, v)
    um, umm, uv = master.to(DEV), m.to(DEV), v.to(DEV)      # unfused path, in place
    p_fused = torch.empty(psi_p, dtype=torch.float16, device=DEV)
    p_unf = torch.empty(psi_p, dtype=torch.float16, device=DEV)
    shards = torch.empty(psi_p, dtype=torch.float32, device=DEV)
    ref = oracle.Result(False, master.numpy(), m.numpy(), v.numpy(), oracle.f2h(master.numpy()))
    for t in (1, 2, 3):
        g_cpu = [synth.grad_f16(psi_p, 0.01, seed=7, rank=r, step=t) for r in range(nd)]
        g_dev = [g.to(DEV) for g in g_cpu]
        st = status_word()
        fused_step(psi_p, g_dev, pp, p_fused, HP, t, st)
        pp.swap()
        st2 = status_word()
        lz.zero_reduce_scatter_bucket(pl, 0, g_dev, [shards[r * S:(r + 1) * S] for r in range(nd)],
                                      st2)
        lz.zero_adam_shard(psi_p, shards, um, umm, uv, p_unf, HP, t, st2)
        ref = oracle.zero1_step(ref_plan, [g.numpy() for g in g_cpu], ref.master, ref.m, ref.v,
                                ref.params16, ORC_HP, t)
        torch.cuda.synchronize()
        assert status_flags(st) == 0 and status_flags(st2) == 0 and not ref.skipped
        check_bitexact_f32("reduced grad", f32np(shards), ref.reduced)
        w, mm, vv = pp.numpy()
        for name, a, b in (("master", w, ref.master), ("m", mm, ref.m), ("v", vv, ref.v),
                           ("master unfused", f32np(um), ref.master),
                           ("m unfused", f32np(umm), ref.m), ("v unfused", f32np(uv), ref.v)):
            check_f32(f"step {t} {name}", a, b)
        check_f16(f"step {t} params", f16np(p_fused), ref.params16)
        check_f16(f"step {t} params unfused", f16np(p_unf), ref.params16)


@pytest.mark.parametrize("where", ["first", "middle", "tail", "last_tile"])
@pytest.mark.parametrize("bad", [0x7c00, 0xfc00, 0x7e01])
@pytest.mark.parametrize("nd", [3, 8, 64])
def test_fused_overflow_skips_the_step(where, bad, nd):
    n = 2048 * 40 + 5
    idx = {"first": 0, "middle": n // 2 + 1, "tail": n - 1, "last_tile": n - 13}[where]
    master, m, v = synth.state_warm(n, seed=nd)
    pp = PingPong(master, m, v)
    g_dev = [g.to(DEV) for g in _rank_grads_cpu(n, nd, 5, 1)]
    g_dev[nd - 1].view(torch.int16)[idx] = torch.tensor(bad, dtype=torch.int32).to(torch.int16)
    params = torch.zeros(n, dtype=torch.float16, device=DEV)
    st = status_word()
    fused_step(n, g_dev, pp, params, HP, 1, st)
    code, flags = lz.zero_step_status(st)
    assert code == lz.ZERO_STEP_SKIPPED
    assert flags == lz.ZERO_FLAG_OVERFLOW | lz.ZERO_FLAG_SKIPPED
    # the step did not happen: outputs equal inputs, parameters are fp16(master)
    for a, b in zip(pp.cur, pp.nxt):
        assert torch.equal(a.view(torch.int32), b.view(torch.int32))
    assert np.array_equal(f16np(params), oracle.f2h(master.numpy()))
    # and the next step runs normally (same t: the counter does not advance on a skip)
    pp.swap()
    g_dev[nd - 1].view(torch.int16)[idx] = 0
    st = status_word()
    fused_step(n, g_dev, pp, params, HP, 1, st)
    assert lz.zero_step_status(st) == (lz.ZERO_OK, 0)


def test_unfused_overflow_skips_the_step():
    numels, nd = [5000, 3001], 4
    pl = lz.zero_plan_create(numels, nd, 2, 1024)
    psi, psi_p, S, nb = lz.zero_plan_info(pl)
    g_dev = [synth.grad_f16(psi_p, 1e-3, seed=1, rank=r).to(DEV) for r in range(nd)]
    g_dev[2][psi_p - 1] = float("nan")
    shards = torch.empty(psi_p, dtype=torch.float32, device=DEV)
    master, m, v = (x.to(DEV) for x in synth.state_warm(psi_p, seed=2))
    m0, v0, w0 = m.clone(), v.clone(), master.clone()
    params = torch.zeros(psi_p, dtype=torch.float16, device=DEV)
    st = status_word()
    for k in range(nb):
        lo, ln, _, _ = lz.zero_plan_bucket(pl, k)
        lz.zero_reduce_scatter_bucket(pl, k, [g[lo:lo + ln] for g in g_dev],
                                      [shards[r * S:(r + 1) * S] for r in range(nd)], st)
    for r in range(nd):
        sl = slice(r * S, (r + 1) * S)
        lz.zero_adam_shard(S, shards[sl], master[sl], m[sl], v[sl], params[sl], HP, 3, st)
    code, flags = lz.zero_step_status(st)
    assert code == lz.ZERO_STEP_SKIPPED and flags == 3
    assert torch.equal(master, w0) and torch.equal(m, m0) and torch.equal(v, v0)
    assert not params.view(torch.int16).any()


@pytest.mark.parametrize("grad_off,state_off,param_off", [(1, 0, 0), (0, 1, 0), (0, 0, 1),
                                                          (0, 0, 2), (0, 0, 4), (3, 2, 3)])
def test_alignment_variants(grad_off, state_off, param_off):
    """Pointers that are only element-aligned take the plain-load kernel; parameter buffers at
    2/4/8-byte alignment take narrower stores. Results are the same as the oracle's."""
    n, nd = 50007, 5
    g_cpu = _rank_grads_cpu(n, nd, 11, 1)
    g_big = [torch.zeros(n + 8, dtype=torch.float16, device=DEV) for _ in range(nd)]
    for gb, g in zip(g_big, g_cpu):
        gb[grad_off:grad_off + n] = g.to(DEV)
    g_dev = [gb[grad_off:grad_off + n] for gb in g_big]
    master, m, v = synth.state_warm(n, seed=12)
    big = [torch.zeros(n + 8, device=DEV) for _ in range(6)]
    for b, x in zip(big[:3], (master, m, v)):
        b[state_off:state_off + n] = x.to(DEV)
    ins = [b[state_off:state_off + n] for b in big[:3]]
    outs = [b[state_off:state_off + n] for b in big[3:]]
    pbig = torch.zeros(n + 8, dtype=torch.float16, device=DEV)
    params = pbig[param_off:param_off + n]
    st = status_word()
    lz.zero_step_fused(n, nd, g_dev, *ins, *outs, params, HP, 1, st)
    lz.zero_step_commit(n, *ins, *outs, params, st)
    torch.cuda.synchronize()
    assert status_flags(st) == 0
    skipped, w, mm, vv, p = oracle.step([g.numpy() for g in g_cpu], master.numpy(), m.numpy(),
                                        v.numpy(), ORC_HP, 1)
    check_f32("master", f32np(outs[0]), w)
    check_f32("m", f32np(outs[1]), mm)
    check_f32("v", f32np(outs[2]), vv)
    check_f16("params", f16np(params), p)
    # nothing written outside the range
    assert not pbig[:param_off].view(torch.int16).any()
    assert not pbig[param_off + n:].view(torch.int16).any()


@pytest.mark.parametrize("overlap", [False, True])
@pytest.mark.parametrize("n_slots", [1, 2, 3])
def test_stage2_scheduler_vs_oracle(n_slots, overlap):
    """Buckets in backward order through the scheduler: the producer fills a staging slot on
    its own stream, the reduce-scatter runs on the scheduler's stream after it, the slot is
    released for a later bucket when the reduce-scatter is done; then the owner updates. With
    `overlap` the scheduler's stream is an overlap region (the bucket kernels chained), so the
    release events follow kernels that may overlap the next bucket's."""
    numels, nd, bucket = [40000, 1234, 30000, 777], 6, 9000
    pl = lz.zero_plan_create(numels, nd, 2, bucket)
    psi, psi_p, S, nb = lz.zero_plan_info(pl)
    ref_plan = oracle.plan(numels, nd, bucket)
    g_cpu = []
    for r in range(nd):
        g = torch.zeros(psi_p, dtype=torch.float16)
        g[:psi] = synth.grad_f16(psi, 1e-3, seed=21, rank=r)
        g_cpu.append(g)
    g_src = [g.to(DEV) for g in g_cpu]
    slot_elems = lz.zero_sched_slot_elems(pl, n_slots)
    slots = torch.empty(slot_elems, dtype=torch.float16, device=DEV)
    shards = torch.empty(psi_p, dtype=torch.float32, device=DEV)
    st = status_word()
    producer = torch.cuda.Stream()
    rs = torch.cuda.Stream()
    torch.cuda.synchronize()
    sch = lz.zero_sched_create(pl, slots, slot_elems, n_slots,
                               [shards[r * S:(r + 1) * S] for r in range(nd)], st, rs)
    if overlap:
        lz.zero_overlap_begin(rs)
    with torch.cuda.stream(producer):
        for k in range(nb):
            lo, ln, _, _ = lz.zero_plan_bucket(pl, k)
            ptrs = lz.zero_sched_begin_bucket(sch, k, producer)
            for r in range(nd):
                dst = torch.empty(0, dtype=torch.float16, device=DEV).set_(
                    slots.untyped_storage(), (ptrs[r] - slots.data_ptr()) // 2, (ln,))
                dst.copy_(g_src[r][lo:lo + ln])      # the "backward pass" writes bucket k
            lz.zero_sched_end_bucket(sch, k, producer)
    if overlap:
        lz.zero_overlap_end(rs)
    main = torch.cuda.current_stream()
    lz.zero_sched_wait(sch, main)
    assert lz.zero_sched_launches(sch) == nb
    master, m, v = (x.to(DEV) for x in synth.state_warm(psi_p, seed=22))
    m_np, v_np, w_np = f32np(m), f32np(v), f32np(master)
    params = torch.empty(psi_p, dtype=torch.float16, device=DEV)
    lz.zero_adam_shard(psi_p, shards, master, m, v, params, HP, 2, st)
    torch.cuda.synchronize()
    assert status_flags(st) == 0
    ref = oracle.zero2_step(ref_plan, lambda k, r: g_cpu[r].numpy()[
        ref_plan.buckets[k][0]:sum(ref_plan.buckets[k])], w_np, m_np, v_np,
        oracle.f2h(w_np), ORC_HP, 2)
    check_bitexact_f32("reduced grad", f32np(shards), ref.reduced)
    check_f32("master", f32np(master), ref.master)
    check_f32("m", f32np(m), ref.m)
    check_f32("v", f32np(v), ref.v)
    check_f16("params", f16np(params), ref.params16)
    lz.zero_sched_destroy(sch)


@pytest.mark.parametrize("overlap", [False, True])
@pytest.mark.parametrize("n_slots", [1, 3])
def test_stage2_fused_scheduler_vs_oracle(n_slots, overlap):
    """The scheduler in fused mode: each bucket's kernel is the fused step over its range (the
    reduced gradient never stored), slots released after it; commit after the last bucket.
    Equals the oracle's stage-2 step; then an inf in one bucket skips the whole step."""
    numels, nd, bucket = [40000, 1234, 30000, 777], 6, 9000
    pl = lz.zero_plan_create(numels, nd, 2, bucket)
    psi, psi_p, S, nb = lz.zero_plan_info(pl)
    ref_plan = oracle.plan(numels, nd, bucket)
    g_cpu = []
    for r in range(nd):
        g = torch.zeros(psi_p, dtype=torch.float16)
        g[:psi] = synth.grad_f16(psi, 1e-3, seed=23, rank=r)
        g_cpu.append(g)
    master, m, v = synth.state_warm(psi_p, seed=24)
    w_np, m_np, v_np = master.numpy(), m.numpy(), v.numpy()
    slot_elems = lz.zero_sched_slot_elems(pl, n_slots)
    slots = torch.empty(slot_elems, dtype=torch.float16, device=DEV)
    dc = torch.frombuffer(bytearray(bytes(lz.zero_adam_consts_for_step(HP, 3))),
                          dtype=torch.uint8).to(DEV)

    def run(g_src):
        ins = [x.to(DEV) for x in (master, m, v)]
        outs = [torch.full_like(x, float("nan")) for x in ins]
        params = torch.zeros(psi_p, dtype=torch.float16, device=DEV)
        st = status_word()
        producer, stream = torch.cuda.Stream(), torch.cuda.Stream()
        torch.cuda.synchronize()
        sch = lz.zero_sched_create_fused(pl, slots, slot_elems, n_slots, *ins, *outs, params,
                                         dc, st, stream)
        if overlap:
            lz.zero_overlap_begin(stream)
        with torch.cuda.stream(producer):
            for k in range(nb):
                lo, ln, _, _ = lz.zero_plan_bucket(pl, k)
                ptrs = lz.zero_sched_begin_bucket(sch, k, producer)
                for r in range(nd):
                    dst = torch.empty(0, dtype=torch.float16, device=DEV).set_(
                        slots.untyped_storage(), (ptrs[r] - slots.data_ptr()) // 2, (ln,))
                    dst.copy_(g_src[r][lo:lo + ln])
                lz.zero_sched_end_bucket(sch, k, producer)
        if overlap:
            lz.zero_overlap_end(stream)
        main = torch.cuda.current_stream()
        lz.zero_sched_wait(sch, main)
        lz.zero_step_commit(psi_p, *ins, *outs, params, st)
        code, flags = lz.zero_step_status(st)
        assert lz.zero_sched_launches(sch) == nb
        lz.zero_sched_destroy(sch)
        return code, flags, ins, outs, params

    code, flags, ins, outs, params = run([g.to(DEV) for g in g_cpu])
    assert code == lz.ZERO_OK and flags == 0
    ref = oracle.zero2_step(ref_plan, lambda k, r: g_cpu[r].numpy()[
        ref_plan.buckets[k][0]:sum(ref_plan.buckets[k])], w_np, m_np, v_np,
        oracle.f2h(w_np), ORC_HP, 3)
    check_f32("master", f32np(outs[0]), ref.master)
    check_f32("m", f32np(outs[1]), ref.m)
    check_f32("v", f32np(outs[2]), ref.v)
    check_f16("params", f16np(params), ref.params16)
    # an inf in the middle bucket's gradient of rank 2: the whole step is skipped
    g_bad = [g.to(DEV) for g in g_cpu]
    lo_mid, _, _, _ = lz.zero_plan_bucket(pl, nb // 2)
    g_bad[2][lo_mid + 5] = float("inf")
    code, flags, ins, outs, params = run(g_bad)
    assert code == lz.ZERO_STEP_SKIPPED
    for a, b in zip(ins, outs):
        assert torch.equal(a, b)
    assert np.array_equal(f16np(params), oracle.f2h(w_np))


@pytest.mark.parametrize("nd", [3, 8])
@pytest.mark.parametrize("loss_scale", [1000.0, 1024.0, 1.0])
def test_fused_step_special_values(nd, loss_scale):
    """Gradients made of special fp16 values -- +0, -0, subnormals (the smallest, the largest),
    the smallest and largest normals, 65504 and its negation, and values whose sum cancels --
    with a non-power-of-two Nd (the mean by division) and a loss scale that is not a power of
    two (the unscale by division), over a range that takes the bulk-copy pipeline with a
    ragged tail. Zero gradients with zero m and v leave master unchanged."""
    n = 3072 * 9 + 5
    special = np.array([0x0000, 0x8000, 0x0001, 0x8001, 0x03ff, 0x83ff, 0x0400, 0x8400,
                        0x7bff, 0xfbff, 0x3c00, 0xbc00, 0x1400, 0x9400], np.uint16)
    rng = np.random.default_rng(1000 + nd)
    g_cpu = []
    for r in range(nd):
        pick = special[rng.integers(0, special.size, size=n)]
        g = torch.from_numpy(pick.view(np.int16).copy()).view(torch.float16)
        g_cpu.append(g)
    # a block of exact cancellation: rank r holds (-1)^r * 65504 (Nd = 8: sum 0)
    for r in range(nd):
        g_cpu[r][100:200] = 65504.0 if r % 2 == 0 else -65504.0
    # a block of all-zero gradients at all ranks
    for r in range(nd):
        g_cpu[r][3000:3100] = 0.0
    master, m, v = synth.state_warm(n, seed=77)
    m[3000:3050] = 0.0
    v[3000:3050] = 0.0
    hp = lz.AdamHP(loss_scale=loss_scale)
    ohp = oracle.AdamHP(loss_scale=loss_scale)
    pp = PingPong(master, m, v)
    params = torch.empty(n, dtype=torch.float16, device=DEV)
    st = status_word()
    fused_step(n, [g.to(DEV) for g in g_cpu], pp, params, hp, 2, st)
    torch.cuda.synchronize()
    assert status_flags(st) == 0
    pp.swap()
    skipped, w, mm, vv, p = oracle.step([g.numpy() for g in g_cpu], master.numpy(), m.numpy(),
                                        v.numpy(), ohp, 2)
    assert not skipped
    got = pp.numpy()
    check_f32("master", got[0], w)
    check_f32("m", got[1], mm)
    check_f32("v", got[2], vv)
    check_f16("params", f16np(params), p)
    assert np.array_equal(got[0][3000:3050], master.numpy()[3000:3050])


def test_step_split_into_bucket_calls():
    """One step made of several zero_step_fused calls (one per bucket, backward order) and one
    commit equals the single-call step; an overflow in a late bucket skips all of it."""
    nd, n, B = 8, 2048 * 37 + 3, 10000
    g_cpu = _rank_grads_cpu(n, nd, 31, 1)
    g_dev = [g.to(DEV) for g in g_cpu]
    master, m, v = synth.state_warm(n, seed=32)
    pp = PingPong(master, m, v)
    params = torch.empty(n, dtype=torch.float16, device=DEV)
    st = status_word()
    bounds = []
    hi = n
    while hi > 0:
        lo = max(0, hi - B)
        bounds.append((lo, hi))
        hi = lo
    for lo, hi in bounds:
        lz.zero_step_fused(hi - lo, nd, [g[lo:hi] for g in g_dev], *[x[lo:hi] for x in pp.cur],
                           *[x[lo:hi] for x in pp.nxt], params[lo:hi], HP, 1, st)
    lz.zero_step_commit(n, *pp.cur, *pp.nxt, params, st)
    torch.cuda.synchronize()
    assert status_flags(st) == 0
    skipped, w, mm, vv, p = oracle.step([g.numpy() for g in g_cpu], master.numpy(), m.numpy(),
                                        v.numpy(), ORC_HP, 1)
    check_f32("master", f32np(pp.nxt[0]), w)
    check_f16("params", f16np(params), p)
    # overflow in the last bucket processed (the lowest range): everything is rolled back
    g_dev[5][3] = float("inf")
    st = status_word()
    for lo, hi in bounds:
        lz.zero_step_fused(hi - lo, nd, [g[lo:hi] for g in g_dev], *[x[lo:hi] for x in pp.cur],
                           *[x[lo:hi] for x in pp.nxt], params[lo:hi], HP, 1, st)
    lz.zero_step_commit(n, *pp.cur, *pp.nxt, params, st)
    assert lz.zero_step_status(st)[0] == lz.ZERO_STEP_SKIPPED
    for a, b in zip(pp.cur, pp.nxt):
        assert torch.equal(a, b)
    assert np.array_equal(f16np(params), oracle.f2h(master.numpy()))


def test_launch_sizes_in_any_order():
    """Nd changes the pipeline's shared-memory size; alternating sizes on the same kernel
    must keep launching (each size within the device's opt-in limit)."""
    n = 2048 * 9 + 5
    for nd in (1, 2, 1, 7, 6, 1, 64, 33, 64, 25):
        master, m, v = synth.state_warm(n, seed=nd)
        pp = PingPong(master, m, v)
        g_cpu = _rank_grads_cpu(n, nd, 41, 1)
        params = torch.empty(n, dtype=torch.float16, device=DEV)
        st = status_word()
        fused_step(n, [g.to(DEV) for g in g_cpu], pp, params, HP, 1, st)
        torch.cuda.synchronize()
        assert status_flags(st) == 0
        skipped, w, mm, vv, p = oracle.step([g.numpy() for g in g_cpu], master.numpy(),
                                            m.numpy(), v.numpy(), ORC_HP, 1)
        check_f32("master", f32np(pp.nxt[0]), w)
        check_f16("params", f16np(params), p)


def _consts_on_device(t):
    c = lz.zero_adam_consts_for_step(HP, t)
    host = torch.frombuffer(bytearray(bytes(c)), dtype=torch.uint8)
    return host.to(DEV)


@pytest.mark.parametrize("nd", [2, 8, 64])
def test_device_constants_variants_match(nd):
    """zero_step_fused_dc / zero_adam_shard_dc (constants read from device memory) give the
    same bits as the calls that take the hyperparameters and t."""
    n = 2048 * 21 + 3
    g_dev = [g.to(DEV) for g in _rank_grads_cpu(n, nd, 61, 1)]
    master, m, v = (x.to(DEV) for x in synth.state_warm(n, seed=62))
    for t in (1, 7):
        dc = _consts_on_device(t)
        outs_a = [torch.empty_like(x) for x in (master, m, v)]
        outs_b = [torch.empty_like(x) for x in (master, m, v)]
        pa = torch.empty(n, dtype=torch.float16, device=DEV)
        pb = torch.empty(n, dtype=torch.float16, device=DEV)
        st = status_word()
        lz.zero_step_fused(n, nd, g_dev, master, m, v, *outs_a, pa, HP, t, st)
        lz.zero_step_fused_dc(n, nd, g_dev, master, m, v, *outs_b, pb, dc, st)
        red = torch.full((n,), 3e-6, device=DEV)
        ua = [x.clone() for x in (master, m, v)]
        ub = [x.clone() for x in (master, m, v)]
        qa = torch.empty(n, dtype=torch.float16, device=DEV)
        qb = torch.empty(n, dtype=torch.float16, device=DEV)
        lz.zero_adam_shard(n, red, *ua, qa, HP, t, st)
        lz.zero_adam_shard_dc(n, red, *ub, qb, dc, st)
        torch.cuda.synchronize()
        assert status_flags(st) == 0
        for a, b in list(zip(outs_a, outs_b)) + list(zip(ua, ub)) + [(pa, pb), (qa, qb)]:
            assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_graph_replay_of_bucketed_step():
    """A step of per-bucket zero_step_fused_dc calls and a commit, captured once per direction
    of the ping-pong as CUDA graphs and replayed for t = 1, 2, 3 with that step's constants
    copied in before each replay, equals the oracle's three steps."""
    nd, n, B = 4, 2048 * 30 + 7, 9000
    master, m, v = synth.state_warm(n, seed=71)
    bufs = [[x.to(DEV) for x in (master, m, v)], [torch.empty(n, device=DEV) for _ in range(3)]]
    grads = [torch.empty(n, dtype=torch.float16, device=DEV) for _ in range(nd)]
    params = torch.empty(n, dtype=torch.float16, device=DEV)
    dc = torch.empty(lz.ZERO_ADAM_CONSTS_BYTES, dtype=torch.uint8, device=DEV)
    st = status_word()
    flags = status_word()
    bounds, hi = [], n
    while hi > 0:
        bounds.append((max(0, hi - B), hi))
        hi = max(0, hi - B)

    def step(src, dst):
        st.zero_()
        for lo, hi in bounds:
            lz.zero_step_fused_dc(hi - lo, nd, [g[lo:hi] for g in grads],
                                  *[x[lo:hi] for x in src], *[x[lo:hi] for x in dst],
                                  params[lo:hi], dc, st)
        lz.zero_step_commit(n, *src, *dst, params, st)
        flags.bitwise_or_(st)

    dc.copy_(_consts_on_device(1))
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step(bufs[0], bufs[1])        # warm-up outside capture (sets launch attributes)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    graphs = []
    for src, dst in ((bufs[0], bufs[1]), (bufs[1], bufs[0])):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            step(src, dst)
        graphs.append(g)
    # restore the state the warm-up overwrote, then run three steps by replay
    for x, y in zip(bufs[0], (master, m, v)):
        x.copy_(y.to(DEV))
    flags.zero_()
    w_r, m_r, v_r = master.numpy(), m.numpy(), v.numpy()
    for t in (1, 2, 3):
        g_cpu = _rank_grads_cpu(n, nd, 72, t)
        for d, s in zip(grads, g_cpu):
            d.copy_(s.to(DEV))
        dc.copy_(_consts_on_device(t))
        graphs[(t - 1) % 2].replay()
        torch.cuda.synchronize()
        assert status_flags(flags) == 0
        skipped, w_r, m_r, v_r, p_r = oracle.step([g.numpy() for g in g_cpu], w_r, m_r, v_r,
                                                  ORC_HP, t)
        out = bufs[t % 2]
        check_f32(f"step {t} master", f32np(out[0]), w_r)
        check_f32(f"step {t} m", f32np(out[1]), m_r)
        check_f32(f"step {t} v", f32np(out[2]), v_r)
        check_f16(f"step {t} params", f16np(params), p_r)


def test_bounded_wait_expires_and_context_survives():
    """Failure detection without a fault: the pipeline's wait for data that never comes gives up
    after about a second with ZERO_FLAG_TIMEOUT, and the next step on the same context works."""
    import time
    st = status_word()
    t0 = time.perf_counter()
    lz.zero_selftest_timeout(st)
    code, flags = lz.zero_step_status(st)
    dt = time.perf_counter() - t0
    assert code == lz.ZERO_ECUDA and flags == lz.ZERO_FLAG_TIMEOUT
    assert 0.5 < dt < 30.0
    # the context is still usable
    n, nd = 5000, 3
    master, m, v = synth.state_warm(n, seed=81)
    pp = PingPong(master, m, v)
    g_cpu = _rank_grads_cpu(n, nd, 82, 1)
    params = torch.empty(n, dtype=torch.float16, device=DEV)
    st = status_word()
    fused_step(n, [g.to(DEV) for g in g_cpu], pp, params, HP, 1, st)
    assert lz.zero_step_status(st) == (lz.ZERO_OK, 0)
    skipped, w, mm, vv, p = oracle.step([g.numpy() for g in g_cpu], master.numpy(), m.numpy(),
                                        v.numpy(), ORC_HP, 1)
    check_f32("master", f32np(pp.nxt[0]), w)
    check_f16("params", f16np(params), p)


@pytest.mark.parametrize("mode", ["ordered", "overlap", "inside_region"])
def test_step_fused_ranges_vs_oracle(mode):
    """zero_step_fused_ranges: a step's bucket calls (backward order, ragged last bucket, the
    small-call and the plain shapes mixed) in one C call equal the oracle's step, launched
    ordered, as an overlap region, or joining a region the caller opened."""
    n, nd, B = 300_007, 5, 65_536
    master, m, v = synth.state_warm(n, seed=91)
    pp = PingPong(master, m, v)
    g_cpu = _rank_grads_cpu(n, nd, 92, 1)
    g_dev = [g.to(DEV) for g in g_cpu]
    params = torch.empty(n, dtype=torch.float16, device=DEV)
    cuts, hi = [], n
    while hi > 0:
        cuts.append((max(0, hi - B), hi))
        hi = max(0, hi - B)
    cuts.append((0, 0))                                   # an empty range is allowed
    ranges = [(hi - lo, [g[lo:hi] if hi > lo else g for g in g_dev],
               *[x[lo:hi] if hi > lo else x for x in pp.cur],
               *[x[lo:hi] if hi > lo else x for x in pp.nxt],
               params[lo:hi] if hi > lo else params) for lo, hi in cuts]
    st = status_word()
    before = lz.zero_kernel_launches()
    if mode == "inside_region":
        with lz.overlap():
            lz.zero_step_fused_ranges(nd, ranges, HP, 1, st, overlap=True)
    else:
        lz.zero_step_fused_ranges(nd, ranges, HP, 1, st, overlap=(mode == "overlap"))
    lz.zero_step_commit(n, *pp.cur, *pp.nxt, params, st)
    assert lz.zero_step_status(st) == (lz.ZERO_OK, 0)
    assert lz.zero_kernel_launches() - before == len(cuts) - 1 + 1
    skipped, w, mm, vv, p = oracle.step([g.numpy() for g in g_cpu], master.numpy(), m.numpy(),
                                        v.numpy(), ORC_HP, 1)
    check_f32("master", f32np(pp.nxt[0]), w)
    check_f32("m", f32np(pp.nxt[1]), mm)
    check_f32("v", f32np(pp.nxt[2]), vv)
    check_f16("params", f16np(params), p)
