"""The step protocol around the kernels, through the C ABI: one stage-2 scheduler reused for
every step (rebound to the swapped ping-pong buffers and a fresh status word), the skip of a
step whose kernels reported a failure (not only an overflow), and the scheduler's refusal to
hand out a slot that still holds an unfinished bucket. Against the oracle's stage-2 step
("ZeRO-2" card, "Gradient 생명주기"); tolerances as in test_gpu_parity.py."""
import numpy as np
import pytest
import torch

import oracle
from tests._gpu import (DEV, HP, ORC_HP, PingPong, check_f16, check_f32, f16np, f32np, lz,
                        require_gpu, status_word)
from zero_partitioned_optimizer_plan_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _gpu():
    require_gpu()
    torch.cuda.set_device(0)
    yield
    torch.cuda.synchronize()


def _slot_view(slots, ptr, n):
    return torch.empty(0, dtype=torch.float16, device=DEV).set_(
        slots.untyped_storage(), (ptr - slots.data_ptr()) // 2, (n,))


@pytest.mark.parametrize("n_slots", [1, 2])
def test_stage2_fused_scheduler_reused_across_steps(n_slots):
    """One fused scheduler for four steps: t = 1, an overflowing attempt at t = 2 (skipped,
    t not advanced), then t = 2 and t = 3; between steps it is rebound to the swapped state
    and a new status word. Every step equals the oracle's stage-2 step."""
    numels, nd, bucket = [40000, 1234, 30000, 777], 6, 9000
    pl = lz.zero_plan_create(numels, nd, 2, bucket)
    psi, psi_p, S, nb = lz.zero_plan_info(pl)
    ref_plan = oracle.plan(numels, nd, bucket)
    master, m, v = synth.state_warm(psi_p, seed=31)
    pp = PingPong(master, m, v)
    params = torch.from_numpy(oracle.f2h(master.numpy()).view(np.float16)).to(DEV)
    slot_elems = lz.zero_sched_slot_elems(pl, n_slots)
    slots = torch.empty(slot_elems, dtype=torch.float16, device=DEV)
    d_consts = torch.empty(lz.ZERO_ADAM_CONSTS_BYTES, dtype=torch.uint8, device=DEV)
    producer, stream = torch.cuda.Stream(), torch.cuda.Stream()
    main = torch.cuda.current_stream()
    st0 = status_word()
    sch = lz.zero_sched_create_fused(pl, slots, slot_elems, n_slots, *pp.cur, *pp.nxt, params,
                                     d_consts, st0, stream)
    ref = (master.numpy(), m.numpy(), v.numpy(), oracle.f2h(master.numpy()))
    attempts = [(1, None), (2, (nb // 2, 4)), (2, None), (3, None)]
    for i, (t, bad) in enumerate(attempts):
        g = []
        for r in range(nd):
            x = torch.zeros(psi_p, dtype=torch.float16)
            x[:psi] = synth.grad_f16(psi, 1e-3, seed=32, rank=r, step=10 * i + t)
            g.append(x)
        if bad is not None:
            k, r = bad
            g[r][lz.zero_plan_bucket(pl, k)[0] + 3] = float("inf")
        st = status_word()
        c = lz.zero_adam_consts_for_step(HP, t)
        d_consts.copy_(torch.frombuffer(bytearray(bytes(c)), dtype=torch.uint8))
        torch.cuda.synchronize()
        lz.zero_sched_rebind_fused(sch, *pp.cur, *pp.nxt, params, st)
        g_dev = [x.to(DEV) for x in g]
        torch.cuda.synchronize()
        lz.zero_overlap_begin(stream)
        with torch.cuda.stream(producer):
            for k in range(nb):
                lo, ln, _, _ = lz.zero_plan_bucket(pl, k)
                ptrs = lz.zero_sched_begin_bucket(sch, k, producer)
                for r in range(nd):
                    _slot_view(slots, ptrs[r], ln).copy_(g_dev[r][lo:lo + ln])
                lz.zero_sched_end_bucket(sch, k, producer)
        lz.zero_overlap_end(stream)
        lz.zero_sched_wait(sch, main)
        lz.zero_step_commit(psi_p, *pp.cur, *pp.nxt, params, st, main)
        code, flags = lz.zero_step_status(st, main)
        res = oracle.zero2_step(ref_plan, lambda kk, rr: g[rr].numpy()[
            ref_plan.buckets[kk][0]:sum(ref_plan.buckets[kk])], *ref[:3], ref[3], ORC_HP, t)
        if bad is not None:
            assert res.skipped
            assert code == lz.ZERO_STEP_SKIPPED
            assert flags == lz.ZERO_FLAG_OVERFLOW | lz.ZERO_FLAG_SKIPPED
        else:
            assert not res.skipped and (code, flags) == (lz.ZERO_OK, 0)
            ref = (res.master, res.m, res.v, res.params16)
        pp.swap()
        check_f32(f"attempt {i} master", f32np(pp.cur[0]), ref[0])
        check_f32(f"attempt {i} m", f32np(pp.cur[1]), ref[1])
        check_f32(f"attempt {i} v", f32np(pp.cur[2]), ref[2])
        check_f16(f"attempt {i} params", f16np(params), ref[3])
    assert lz.zero_sched_launches(sch) == nb * len(attempts)
    assert int(st0.item()) == 0     # the creation status word was never written after rebinding
    lz.zero_sched_destroy(sch)


def test_stage2_upload_from_pinned_host_through_two_slots():
    """The end-to-end leg's data path: each bucket's Nd gradient slices copied from pinned host
    memory into one of two staging slots on an upload stream (each copy waits, on that stream,
    for the release of its slot), the fused bucket kernels on the scheduler's stream, the
    commit, and the fp16 parameters downloaded. Two steps equal the oracle's stage-2 step."""
    numels, nd, bucket = [40000, 1234, 30000, 777, 9999], 5, 7000
    pl = lz.zero_plan_create(numels, nd, 2, bucket)
    psi, psi_p, S, nb = lz.zero_plan_info(pl)
    ref_plan = oracle.plan(numels, nd, bucket)
    master, m, v = synth.state_warm(psi_p, seed=35)
    pp = PingPong(master, m, v)
    params = torch.from_numpy(oracle.f2h(master.numpy()).view(np.float16)).to(DEV)
    slot_elems = lz.zero_sched_slot_elems(pl, 2)
    slots = torch.empty(slot_elems, dtype=torch.float16, device=DEV)
    d_consts = torch.empty(lz.ZERO_ADAM_CONSTS_BYTES, dtype=torch.uint8, device=DEV)
    up, main = torch.cuda.Stream(), torch.cuda.current_stream()
    st = status_word()
    sch = lz.zero_sched_create_fused(pl, slots, slot_elems, 2, *pp.cur, *pp.nxt, params,
                                     d_consts, st, main)
    ref = (master.numpy(), m.numpy(), v.numpy(), oracle.f2h(master.numpy()))
    for t in (1, 2):
        g = []
        for r in range(nd):
            x = torch.zeros(psi_p, dtype=torch.float16)
            x[:psi] = synth.grad_f16(psi, 1e-3, seed=36, rank=r, step=t)
            g.append(x.pin_memory())
        st = status_word()
        c = lz.zero_adam_consts_for_step(HP, t)
        d_consts.copy_(torch.frombuffer(bytearray(bytes(c)), dtype=torch.uint8))
        lz.zero_sched_rebind_fused(sch, *pp.cur, *pp.nxt, params, st)
        lz.zero_overlap_begin(main)
        for k in range(nb):
            lo, ln, _, _ = lz.zero_plan_bucket(pl, k)
            ptrs = lz.zero_sched_begin_bucket(sch, k, up)
            with torch.cuda.stream(up):
                for r in range(nd):
                    _slot_view(slots, ptrs[r], ln).copy_(g[r][lo:lo + ln], non_blocking=True)
            lz.zero_sched_end_bucket(sch, k, up)
        lz.zero_overlap_end(main)
        lz.zero_sched_wait(sch, main)
        lz.zero_step_commit(psi_p, *pp.cur, *pp.nxt, params, st, main)
        h_params = torch.empty(psi_p, dtype=torch.float16, pin_memory=True)
        h_params.copy_(params, non_blocking=True)
        assert lz.zero_step_status(st, main) == (lz.ZERO_OK, 0)
        res = oracle.zero2_step(ref_plan, lambda kk, rr: g[rr].numpy()[
            ref_plan.buckets[kk][0]:sum(ref_plan.buckets[kk])], *ref[:3], ref[3], ORC_HP, t)
        ref = (res.master, res.m, res.v, res.params16)
        pp.swap()
        check_f32(f"step {t} master", f32np(pp.cur[0]), ref[0])
        check_f32(f"step {t} v", f32np(pp.cur[2]), ref[2])
        check_f16(f"step {t} downloaded params", h_params.numpy().view(np.uint16), ref[3])
    lz.zero_sched_destroy(sch)


def test_scheduler_refuses_a_slot_still_in_use():
    """With one slot, beginning bucket 1 while bucket 0 has been begun but not ended would drop
    bucket 0's fill: EINVAL. Rebinding in the middle of a bucket is refused too."""
    numels, nd, bucket = [5000, 3000], 2, 4000
    pl = lz.zero_plan_create(numels, nd, 2, bucket)
    psi, psi_p, S, nb = lz.zero_plan_info(pl)
    slot_elems = lz.zero_sched_slot_elems(pl, 1)
    slots = torch.zeros(slot_elems, dtype=torch.float16, device=DEV)
    shards = torch.empty(psi_p, dtype=torch.float32, device=DEV)
    st = status_word()
    sch = lz.zero_sched_create(pl, slots, slot_elems, 1, [shards[:S], shards[S:]], st)
    lz.zero_sched_begin_bucket(sch, 0)
    with pytest.raises(lz.ZeroError) as e:
        lz.zero_sched_begin_bucket(sch, 1)
    assert e.value.code == lz.ZERO_EINVAL
    with pytest.raises(lz.ZeroError) as e:
        lz.zero_sched_rebind_status(sch, status_word())
    assert e.value.code == lz.ZERO_EINVAL
    with pytest.raises(lz.ZeroError) as e:     # not a fused scheduler
        lz.zero_sched_rebind_fused(sch, shards, shards, shards, shards, shards, shards,
                                   slots, st)
    assert e.value.code == lz.ZERO_EINVAL
    lz.zero_sched_end_bucket(sch, 0)
    lz.zero_sched_begin_bucket(sch, 1)          # the slot is free again (after bucket 0's kernel)
    lz.zero_sched_end_bucket(sch, 1)
    st2 = status_word()
    lz.zero_sched_rebind_status(sch, st2)
    torch.cuda.synchronize()
    lz.zero_sched_destroy(sch)


@pytest.mark.parametrize("bit", ["timeout", "bounds"])
def test_commit_restores_a_failed_step(bit):
    """A step whose status word carries the timeout or bounds bit (its kernels left outputs
    unwritten) is voided by the commit like an overflowing one: outputs = inputs, fp16
    parameters = fp16(master_in), skipped bit set; zero_step_status reports the failure."""
    flag = {"timeout": lz.ZERO_FLAG_TIMEOUT, "bounds": lz.ZERO_FLAG_BOUNDS}[bit]
    n, nd = 70_000, 4
    master, m, v = synth.state_warm(n, seed=41)
    pp = PingPong(master, m, v)
    grads = [synth.grad_f16(n, 1e-3, seed=42, rank=r).to(DEV) for r in range(nd)]
    params = torch.zeros(n, dtype=torch.float16, device=DEV)
    st = torch.full((1,), flag, dtype=torch.int32, device=DEV)   # as a failed kernel leaves it
    lz.zero_step_fused(n, nd, grads, *pp.cur, *pp.nxt, params, HP, 1, st)
    lz.zero_step_commit(n, *pp.cur, *pp.nxt, params, st)
    code, flags = lz.zero_step_status(st)
    assert code == lz.ZERO_ECUDA
    assert flags == flag | lz.ZERO_FLAG_SKIPPED
    for a, b in zip(pp.cur, pp.nxt):
        assert torch.equal(a.view(torch.int32), b.view(torch.int32))
    assert np.array_equal(f16np(params), oracle.f2h(master.numpy()))


def test_unfused_update_skips_a_failed_reduce_scatter():
    """zero_adam_shard leaves the shard alone when the step's status carries the timeout bit
    (a reduce-scatter of the step gave up, so its reduced shard is incomplete)."""
    n = 50_000
    master, m, v = (x.to(DEV) for x in synth.state_warm(n, seed=43))
    keep = [x.clone() for x in (master, m, v)]
    grad = torch.randn(n, device=DEV) * 1e-3
    params = torch.zeros(n, dtype=torch.float16, device=DEV)
    st = torch.full((1,), lz.ZERO_FLAG_TIMEOUT, dtype=torch.int32, device=DEV)
    lz.zero_adam_shard(n, grad, master, m, v, params, HP, 1, st)
    code, flags = lz.zero_step_status(st)
    assert code == lz.ZERO_ECUDA and flags == lz.ZERO_FLAG_TIMEOUT | lz.ZERO_FLAG_SKIPPED
    for a, b in zip((master, m, v), keep):
        assert torch.equal(a, b)
    assert int(torch.count_nonzero(params)) == 0
