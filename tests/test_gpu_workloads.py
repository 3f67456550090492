"""The workloads at their full sizes, through the C ABI in the launch configuration bench.py
times, checked against the oracle on sampled elements (each element's result depends only on
its own inputs, so the oracle evaluates the sample one by one): random positions plus every
tensor, shard and bucket boundary and both ends. Whole-buffer properties (nothing written
outside the owner's range, nothing changed by a skipped step) are checked on all elements.

Tolerances as in test_gpu_parity.py: reduced gradients bit-exact, fp32 state within 2 ulp,
fp16 parameters within 1 ulp."""
import numpy as np
import pytest
import torch

import oracle
from tests._gpu import (DEV, HP, ORC_HP, check_bitexact_f32, check_f16, check_f32, lz,
                        require_gpu, status_flags, status_word)
from zero_partitioned_optimizer_plan_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _gpu():
    require_gpu()
    torch.cuda.set_device(0)
    torch.cuda.empty_cache()
    yield
    torch.cuda.synchronize()
    torch.cuda.empty_cache()


def sample_idx(n, k, seed, boundaries=()):
    rng = np.random.default_rng(seed)
    pts = [rng.integers(0, n, size=k)]
    near = np.array([b + d for b in boundaries for d in (-2, -1, 0, 1, 2)], dtype=np.int64)
    ends = np.concatenate([np.arange(0, min(n, 64)), np.arange(max(0, n - 64), n)])
    allx = np.concatenate(pts + [near, ends.astype(np.int64)])
    allx = allx[(allx >= 0) & (allx < n)]
    return np.unique(allx)


def gather(t, idx_dev):
    x = t[idx_dev].cpu()
    return x.numpy().view(np.uint16) if t.dtype == torch.float16 else x.numpy()


def view_at(base, ptr, n):
    """fp16 tensor of n elements at device address ptr inside base's storage."""
    off = (ptr - base.data_ptr()) // base.element_size()
    assert 0 <= off and off + n <= base.numel()
    return base[off:off + n]


def test_gpt2_small_stage1_ten_steps():
    """GPT-2-small list (Psi = 123,653,376), Nd = 8, stage 1: one fused call per step over the
    whole padded range, 10 steps, gradients N(0, 1e-3^2) with 1% x100, new each step."""
    numels, nd = synth.gpt2_small_list(), 8
    pl = lz.zero_plan_create(numels, nd, 1, 0)
    psi, psi_p, S, nb = lz.zero_plan_info(pl)
    offs = lz.zero_plan_tensor_offsets(pl)
    idx = sample_idx(psi_p, 200_000, 1, boundaries=offs + [r * S for r in range(nd + 1)])
    idx_dev = torch.from_numpy(idx).to(DEV)
    cur = list(synth.state_small(psi_p, seed=2, device=DEV))
    nxt = [torch.empty_like(x) for x in cur]
    params = torch.empty(psi_p, dtype=torch.float16, device=DEV)
    grads = [torch.zeros(psi_p, dtype=torch.float16, device=DEV) for _ in range(nd)]
    shards = torch.empty(psi_p, dtype=torch.float32, device=DEV)
    w_s, m_s, v_s = (gather(x, idx_dev) for x in cur)
    for t in range(1, 11):
        for r in range(nd):
            synth.grad_f16(psi, 1e-3, seed=2, rank=r, step=t, spike_frac=0.01, spike_scale=100.0,
                           out=grads[r][:psi])
        st = status_word()
        lz.zero_step_fused(psi_p, nd, grads, *cur, *nxt, params, HP, t, st)
        lz.zero_step_commit(psi_p, *cur, *nxt, params, st)
        if t == 1:   # the reduced gradient itself, from the bucketed reduce-scatter
            lz.zero_reduce_scatter_bucket(pl, 0, grads,
                                          [shards[r * S:(r + 1) * S] for r in range(nd)], st)
        torch.cuda.synchronize()
        assert status_flags(st) == 0
        cur, nxt = nxt, cur
        gs = [gather(g, idx_dev) for g in grads]
        if t == 1:
            check_bitexact_f32("reduced grad", gather(shards, idx_dev), oracle.reduce_mean(gs))
        skipped, w_s, m_s, v_s, p_s = oracle.step(gs, w_s, m_s, v_s, ORC_HP, t)
        assert not skipped
        check_f32(f"step {t} master", gather(cur[0], idx_dev), w_s)
        check_f32(f"step {t} m", gather(cur[1], idx_dev), m_s)
        check_f32(f"step {t} v", gather(cur[2], idx_dev), v_s)
        check_f16(f"step {t} params", gather(params, idx_dev), p_s)
    print(f"PARITY gpt2-small stage 1: {idx.size} sampled elements x 10 steps within tolerance")


def test_1p3b_stage2_fused_scheduler_with_overflow_run():
    """The same 1.3B stage-2 step with the scheduler in fused mode (the launch configuration of
    bench.py --workload zero2_1p3b --stage2-fused): each bucket's fused step is launched as the
    bucket arrives, two staging slots, then one commit. An overflow run (+inf in rank 3, first
    element of bucket 7) leaves the state unchanged; then 3 steps against the oracle."""
    numels, nd, B = synth.gpt_1p3b_list(), 16, 50_000_000
    pl = lz.zero_plan_create(numels, nd, 2, B)
    psi, psi_p, S, nb = lz.zero_plan_info(pl)
    bounds = [lz.zero_plan_bucket(pl, k)[0] for k in range(nb)] + [r * S for r in range(nd + 1)]
    idx = sample_idx(psi_p, 200_000, 5, boundaries=bounds + lz.zero_plan_tensor_offsets(pl))
    idx_dev = torch.from_numpy(idx).to(DEV)
    cur = list(synth.state_small(psi_p, seed=5, device=DEV))
    nxt = [torch.empty_like(x) for x in cur]
    params = torch.zeros(psi_p, dtype=torch.float16, device=DEV)
    n_slots = 2
    slot_elems = lz.zero_sched_slot_elems(pl, n_slots)
    slots = torch.empty(slot_elems, dtype=torch.float16, device=DEV)
    d_consts = torch.empty(lz.ZERO_ADAM_CONSTS_BYTES, dtype=torch.uint8, device=DEV)
    producer, stream = torch.cuda.Stream(), torch.cuda.Stream()
    main = torch.cuda.current_stream()

    def run_step(t, inject):
        st = status_word()
        c = lz.zero_adam_consts_for_step(HP, t)
        d_consts.copy_(torch.frombuffer(bytearray(bytes(c)), dtype=torch.uint8))
        torch.cuda.synchronize()
        sch = lz.zero_sched_create_fused(pl, slots, slot_elems, n_slots, *cur, *nxt, params,
                                         d_consts, st, stream)
        gathered = [np.empty(idx.size, np.uint16) for _ in range(nd)]
        lz.zero_overlap_begin(stream)      # as bench.py: the bucket kernels chained
        with torch.cuda.stream(producer):
            for k in range(nb):
                lo, ln, _, _ = lz.zero_plan_bucket(pl, k)
                ptrs = lz.zero_sched_begin_bucket(sch, k, producer)
                views = [view_at(slots, p, ln) for p in ptrs]
                for r in range(nd):
                    synth.grad_f16(ln, 1e-3, seed=5, rank=r, step=1000 * t + k, out=views[r])
                if inject and k == 7:
                    views[3][0] = float("inf")
                sel = np.nonzero((idx >= lo) & (idx < lo + ln))[0]
                local = torch.from_numpy(idx[sel] - lo).to(DEV)
                for r in range(nd):
                    gathered[r][sel] = views[r][local].cpu().numpy().view(np.uint16)
                lz.zero_sched_end_bucket(sch, k, producer)
        lz.zero_overlap_end(stream)
        lz.zero_sched_wait(sch, main)
        lz.zero_step_commit(psi_p, *cur, *nxt, params, st, main)
        code, flags = lz.zero_step_status(st, main)
        assert lz.zero_sched_launches(sch) == nb
        lz.zero_sched_destroy(sch)
        return code, flags, gathered

    code, flags, _ = run_step(1, inject=True)
    assert code == lz.ZERO_STEP_SKIPPED and flags == lz.ZERO_FLAG_OVERFLOW | lz.ZERO_FLAG_SKIPPED
    for a, b in zip(cur, nxt):    # the commit restored every element
        assert torch.equal(a.view(torch.int32), b.view(torch.int32))
    w_s, m_s, v_s = (gather(x, idx_dev) for x in cur)
    check_f16("skipped step params", gather(params, idx_dev), oracle.f2h(w_s))
    for t in range(1, 4):
        code, flags, gs = run_step(t, inject=False)
        assert (code, flags) == (lz.ZERO_OK, 0)
        cur, nxt = nxt, cur
        skipped, w_s, m_s, v_s, p_s = oracle.step(gs, w_s, m_s, v_s, ORC_HP, t)
        assert not skipped
        check_f32(f"step {t} master", gather(cur[0], idx_dev), w_s)
        check_f32(f"step {t} m", gather(cur[1], idx_dev), m_s)
        check_f32(f"step {t} v", gather(cur[2], idx_dev), v_s)
        check_f16(f"step {t} params", gather(params, idx_dev), p_s)
    print(f"PARITY 1.3B stage 2 fused scheduler: skip run + 3 steps, {idx.size} sampled elements")


def test_1p3b_stage2_buckets_with_overflow_run():
    """1.3B list (Psi = 1,311,528,960), Nd = 16, stage 2, buckets of 50,000,000 elements in
    backward order through the scheduler (two staging slots, producer and reduce-scatter on
    their own streams), then the owners' updates. First a run with +inf in rank 3's gradient
    at the first element of bucket 7: the step is skipped and nothing changes. Then 5 steps."""
    numels, nd, B = synth.gpt_1p3b_list(), 16, 50_000_000
    pl = lz.zero_plan_create(numels, nd, 2, B)
    psi, psi_p, S, nb = lz.zero_plan_info(pl)
    assert nb == 27
    lo7, ln7, o7, _ = lz.zero_plan_bucket(pl, 7)
    assert (lo7, o7) == (911_528_960, 11)
    bounds = [lz.zero_plan_bucket(pl, k)[0] for k in range(nb)] + [r * S for r in range(nd + 1)]
    idx = sample_idx(psi_p, 200_000, 3, boundaries=bounds + lz.zero_plan_tensor_offsets(pl))
    idx_dev = torch.from_numpy(idx).to(DEV)
    master, m, v = synth.state_small(psi_p, seed=3, device=DEV)
    params = torch.zeros(psi_p, dtype=torch.float16, device=DEV)
    shards = torch.empty(psi_p, dtype=torch.float32, device=DEV)
    n_slots = 2
    slot_elems = lz.zero_sched_slot_elems(pl, n_slots)
    slots = torch.empty(slot_elems, dtype=torch.float16, device=DEV)
    producer, rs = torch.cuda.Stream(), torch.cuda.Stream()
    main = torch.cuda.current_stream()

    def run_step(t, inject):
        st = status_word()
        torch.cuda.synchronize()
        sch = lz.zero_sched_create(pl, slots, slot_elems, n_slots,
                                   [shards[r * S:(r + 1) * S] for r in range(nd)], st, rs)
        gathered = [np.empty(idx.size, np.uint16) for _ in range(nd)]
        lz.zero_overlap_begin(rs)          # as bench.py: the bucket kernels chained
        with torch.cuda.stream(producer):
            for k in range(nb):
                lo, ln, _, _ = lz.zero_plan_bucket(pl, k)
                ptrs = lz.zero_sched_begin_bucket(sch, k, producer)
                views = [view_at(slots, p, ln) for p in ptrs]
                for r in range(nd):   # the backward pass produces bucket k of every rank
                    synth.grad_f16(ln, 1e-3, seed=3, rank=r, step=1000 * t + k, out=views[r])
                if inject and k == 7:
                    views[3][0] = float("inf")
                sel = np.nonzero((idx >= lo) & (idx < lo + ln))[0]
                local = torch.from_numpy(idx[sel] - lo).to(DEV)
                for r in range(nd):
                    gathered[r][sel] = views[r][local].cpu().numpy().view(np.uint16)
                lz.zero_sched_end_bucket(sch, k, producer)
        lz.zero_overlap_end(rs)
        lz.zero_sched_wait(sch, main)
        assert lz.zero_sched_launches(sch) == nb
        for r in range(nd):   # each owner updates its shard and writes it into the full buffer
            sl = slice(r * S, (r + 1) * S)
            lz.zero_adam_shard(S, shards[sl], master[sl], m[sl], v[sl], params[sl], HP, t, st)
        code, flags = lz.zero_step_status(st, main)
        lz.zero_sched_destroy(sch)
        return code, flags, gathered

    # the overflow run: skipped, every element unchanged
    snap = [x.clone() for x in (master, m, v, params)]
    code, flags, _ = run_step(1, inject=True)
    assert code == lz.ZERO_STEP_SKIPPED and flags == lz.ZERO_FLAG_OVERFLOW | lz.ZERO_FLAG_SKIPPED
    for a, b in zip((master, m, v, params), snap):
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    del snap
    torch.cuda.empty_cache()
    # then 5 steps, t not advanced by the skipped one
    w_s, m_s, v_s = (gather(x, idx_dev) for x in (master, m, v))
    for t in range(1, 6):
        code, flags, gs = run_step(t, inject=False)
        assert (code, flags) == (lz.ZERO_OK, 0)
        check_bitexact_f32(f"step {t} reduced grad", gather(shards, idx_dev),
                           oracle.reduce_mean(gs))
        skipped, w_s, m_s, v_s, p_s = oracle.step(gs, w_s, m_s, v_s, ORC_HP, t)
        assert not skipped
        check_f32(f"step {t} master", gather(master, idx_dev), w_s)
        check_f32(f"step {t} m", gather(m, idx_dev), m_s)
        check_f32(f"step {t} v", gather(v, idx_dev), v_s)
        check_f16(f"step {t} params", gather(params, idx_dev), p_s)
    print(f"PARITY 1.3B stage 2: skip run + {idx.size} sampled elements x 5 steps")


@pytest.fixture(scope="module")
def big_7p5b():
    require_gpu()
    total, nd = 7_500_000_000, 64
    S = total // nd
    full = torch.zeros(total, dtype=torch.float16, device=DEV)
    grads = [torch.empty(S, dtype=torch.float16, device=DEV) for _ in range(nd)]
    yield total, nd, S, full, grads
    del full, grads
    torch.cuda.empty_cache()


@pytest.mark.parametrize("owner", [0, 31, 63])
def test_7p5b_shard_view(big_7p5b, owner):
    """One owner of 7.5e9 parameters at Nd = 64: its 117,187,500-element shard of fp32 state,
    64 separate fp16 gradient slices (one per simulated rank), its updated fp16 shard written
    into the 7.5e9-element parameter buffer at owner*S (8-byte aligned for odd owners)."""
    total, nd, S, full, grads = big_7p5b
    full.zero_()
    for j in range(nd):
        synth.grad_f16(S, 1e-3, seed=4, rank=j, step=owner, out=grads[j])
    cur = list(synth.state_warm(S, seed=40 + owner, device=DEV))
    nxt = [torch.empty_like(x) for x in cur]
    idx = sample_idx(S, 200_000, owner)
    idx_dev = torch.from_numpy(idx).to(DEV)
    w0, m0, v0 = (gather(x, idx_dev) for x in cur)
    out = full[owner * S:(owner + 1) * S]
    st = status_word()
    lz.zero_step_fused(S, nd, grads, *cur, *nxt, out, HP, 1, st)
    lz.zero_step_commit(S, *cur, *nxt, out, st)
    torch.cuda.synchronize()
    assert status_flags(st) == 0
    gs = [gather(g, idx_dev) for g in grads]
    skipped, w, mm, vv, p = oracle.step(gs, w0, m0, v0, ORC_HP, 1)
    assert not skipped
    check_f32("master", gather(nxt[0], idx_dev), w)
    check_f32("m", gather(nxt[1], idx_dev), mm)
    check_f32("v", gather(nxt[2], idx_dev), vv)
    check_f16("params", gather(out, idx_dev), p)
    # the all-gather write-back touched exactly the owner's range of the full buffer
    assert int(torch.count_nonzero(full[:owner * S].view(torch.int16))) == 0
    assert int(torch.count_nonzero(full[(owner + 1) * S:].view(torch.int16))) == 0
    assert int(torch.count_nonzero(out.view(torch.int16))) > S // 2


@pytest.mark.parametrize("nd", [2, 4, 8, 16, 64])
def test_flat_sweep_bucketed_calls(nd):
    """Psi = 2^29 flat buffer, one fused call per bucket of B in {2^19, 2^23, 2^26, 2^29}
    elements (1 MB ... 1 GB of fp16 gradient per rank) in backward order inside an overlap
    region, then one commit -- the launch configuration bench.py times, eagerly and, for the
    two smaller bucket sizes, as a CUDA-graph replay of zero_step_fused_dc calls (outputs
    poisoned with NaN before the replay); every bucketing gives the oracle's step on the
    sample."""
    psi = 1 << 29
    grads = [synth.grad_f16(psi, 1e-3, seed=5, rank=r, step=nd, device=DEV) for r in range(nd)]
    init = list(synth.state_warm(psi, seed=50 + nd, device=DEV))
    bounds = [k * (1 << 19) for k in range(0, 1 << 10, 97)]
    idx = sample_idx(psi, 100_000, nd, boundaries=bounds)
    idx_dev = torch.from_numpy(idx).to(DEV)
    gs = [gather(g, idx_dev) for g in grads]
    skipped, w, mm, vv, p = oracle.step(gs, *(gather(x, idx_dev) for x in init), ORC_HP, 1)
    assert not skipped
    params = torch.empty(psi, dtype=torch.float16, device=DEV)
    nxt = [torch.empty_like(x) for x in init]
    c = lz.zero_adam_consts_for_step(HP, 1)
    d_consts = torch.frombuffer(bytearray(bytes(c)), dtype=torch.uint8).to(DEV)
    for B in (1 << 19, 1 << 23, 1 << 26, 1 << 29):
        ranges = []
        hi = psi
        while hi > 0:
            ranges.append((max(0, hi - B), hi))
            hi = max(0, hi - B)
        assert len(ranges) == psi // B
        st = status_word()

        def step(dc):
            st.zero_()
            with lz.overlap():
                for lo, hi in ranges:
                    if dc:
                        lz.zero_step_fused_dc(hi - lo, nd, [g[lo:hi] for g in grads],
                                              *[x[lo:hi] for x in init], *[x[lo:hi] for x in nxt],
                                              params[lo:hi], d_consts, st)
                    else:
                        lz.zero_step_fused(hi - lo, nd, [g[lo:hi] for g in grads],
                                           *[x[lo:hi] for x in init], *[x[lo:hi] for x in nxt],
                                           params[lo:hi], HP, 1, st)
            lz.zero_step_commit(psi, *init, *nxt, params, st)

        modes = ["eager", "graph"] if B <= 1 << 23 else ["eager"]
        for mode in modes:
            if mode == "eager":
                step(False)
            else:
                side = torch.cuda.Stream()
                side.wait_stream(torch.cuda.current_stream())
                with torch.cuda.stream(side):
                    step(True)
                torch.cuda.current_stream().wait_stream(side)
                torch.cuda.synchronize()
                graph = torch.cuda.CUDAGraph()
                with torch.cuda.graph(graph):
                    step(True)
                for x in nxt:
                    x.fill_(float("nan"))
                params.fill_(float("nan"))
                graph.replay()
            torch.cuda.synchronize()
            assert status_flags(st) == 0
            check_f32(f"B={B} {mode} master", gather(nxt[0], idx_dev), w)
            check_f32(f"B={B} {mode} m", gather(nxt[1], idx_dev), mm)
            check_f32(f"B={B} {mode} v", gather(nxt[2], idx_dev), vv)
            check_f16(f"B={B} {mode} params", gather(params, idx_dev), p)
            if mode == "graph":
                del graph
    print(f"PARITY flat 2^29 Nd={nd}: 4 bucket sizes (2 also by graph), {idx.size} sampled elements")


def test_fused_call_beyond_2p31_elements():
    """Maximum size: one zero_step_fused call over 2^31 + 4101 elements (Nd = 2; 64 GB on the
    device), so every element index past 2^31 goes through the tile, copy and store arithmetic;
    sampled around 2^31, tile boundaries and the end, then the commit."""
    nd, n = 2, (1 << 31) + 4101
    grads = [synth.grad_f16(n, 1e-3, seed=9, rank=r, step=1, device=DEV) for r in range(nd)]
    cur = list(synth.state_warm(n, seed=90, device=DEV))
    nxt = [torch.empty_like(x) for x in cur]
    params = torch.empty(n, dtype=torch.float16, device=DEV)
    idx = sample_idx(n, 100_000, 9, boundaries=[1 << 31, (1 << 31) - 2560 * 7, n - 4101,
                                                 n - 5, (1 << 30) * 3 // 2])
    idx_dev = torch.from_numpy(idx).to(DEV)
    st = status_word()
    lz.zero_step_fused(n, nd, grads, *cur, *nxt, params, HP, 1, st)
    lz.zero_step_commit(n, *cur, *nxt, params, st)
    torch.cuda.synchronize()
    assert status_flags(st) == 0
    skipped, w, mm, vv, p = oracle.step([gather(g, idx_dev) for g in grads],
                                        *(gather(x, idx_dev) for x in cur), ORC_HP, 1)
    assert not skipped
    check_f32("master", gather(nxt[0], idx_dev), w)
    check_f32("m", gather(nxt[1], idx_dev), mm)
    check_f32("v", gather(nxt[2], idx_dev), vv)
    check_f16("params", gather(params, idx_dev), p)
    print(f"PARITY fused call of {n} elements: {idx.size} sampled")

