"""The stage-3 layer scheduler (zero_layer_sched_*) on the GPU against the oracle: whole
stage-3 steps in which every layer is acquired through the scheduler in the forward pass (the
next layer prefetched) and again in the backward pass (the previous layer prefetched, each
layer's fused update after its release), with 1 to 4 layer buffers. Every acquired layer is
copied out on the compute stream at the point where a layer's computation would read it, and
equals the oracle's gathered layer bit for bit ("ZeRO" (lastdictionary): layers gathered just
in time and discarded; "Como funciona": gathered in the forward and again in the backward
pass); state and partitions equal zero3_step. Tolerances as in test_gpu_parity.py."""
import numpy as np
import pytest
import torch

import oracle
from tests._gpu import (DEV, HP, ORC_HP, check_f16, check_f32, f16np, f32np, lz, require_gpu,
                        status_word)
from zero_partitioned_optimizer_plan_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _gpu():
    require_gpu()
    torch.cuda.set_device(0)
    yield
    torch.cuda.synchronize()


class _Pool:
    """The scheduler's buffer memory as a torch tensor, so that an acquired layer's address maps
    back to a view (the scheduler returns device addresses)."""

    def __init__(self, pl, bounds, n_bufs):
        self.elems = lz.zero_layer_sched_buf_elems(pl, bounds, n_bufs)
        self.mem = torch.empty(self.elems + 8, dtype=torch.float16, device=DEV)
        self.base = self.mem.data_ptr()

    def view(self, addr, n):
        off = addr - self.base
        assert off % 2 == 0 and 0 <= off // 2 and off // 2 + n <= self.elems
        return self.mem[off // 2:off // 2 + n]


def _run_step(sched, pool, pl, layers, gb, grads, cur, nxt, shards, t, st, main,
              prepared=False):
    """One stage-3 step through the scheduler; returns the layers as acquired (copied on the
    compute stream right after each acquire, where the layer's computation would run).
    prepared: the updates through PreparedStage3Update (arguments marshalled once), as
    bench.py makes them."""
    L = len(layers)
    fwd, bwd = [None] * L, [None] * L
    lz.zero_layer_sched_begin_step(sched, st, main)
    for l in range(L):
        lo, hi = layers[l]
        p = lz.zero_layer_sched_acquire(sched, l, l + 1 if l + 1 < L else -1, main)
        fwd[l] = pool.view(p, hi - lo).clone()
        lz.zero_layer_sched_release(sched, l, main)
    for l in reversed(range(L)):
        lo, hi = layers[l]
        p = lz.zero_layer_sched_acquire(sched, l, l - 1, main)
        bwd[l] = pool.view(p, hi - lo).clone()
        lz.zero_layer_sched_release(sched, l, main)
        _, ghi = gb[l]
        args = (pl, lo, ghi - lo, [g[lo:ghi] for g in grads], *[x[lo:ghi] for x in cur],
                *[x[lo:ghi] for x in nxt], shards)
        if prepared:
            lz.PreparedStage3Update(*args)(lz.hparams_ref(HP), t, lz.status_ptr(st),
                                           lz.stream_handle(main))
        else:
            lz.zero_stage3_step_fused(*args, HP, t, st, main)
    lz.zero_stage3_step_commit(pl, *cur, *nxt, shards, st, main)
    return fwd, bwd


def _partitions(p16, nd, S):
    out = []
    for q in range(nd):
        buf = torch.zeros(S + 8, dtype=torch.float16, device=DEV)
        view = buf[2 * (q % 3):2 * (q % 3) + S]        # 4-byte and 2-byte offsets too
        view.copy_(torch.from_numpy(p16[q * S:(q + 1) * S].view(np.float16)))
        out.append(view)
    return out


@pytest.mark.parametrize("nd,n_bufs", [(3, 2), (8, 2), (8, 3), (8, 4), (5, 1)])
def test_layer_scheduler_steps_vs_oracle(nd, n_bufs):
    """Three attempts -- t = 1, an overflowing t = 2 (skipped), t = 2 -- through one scheduler
    on a side gather stream, layers straddling owners; with one buffer every prefetch is
    skipped and each acquire gathers. Gathers per step: 2 per layer (none wasted)."""
    numels, split = [40000, 1234, 30000, 777, 5003, 999, 4096], [1, 2, 2, 2]
    pl = lz.zero_plan_create(numels, nd, 3, 0)
    psi, psi_p, S, _ = lz.zero_plan_info(pl)
    opl = oracle.plan(numels, nd, 0)
    layers = oracle.layer_ranges(opl, split)
    gb = oracle.grad_buckets(opl, layers)
    L = len(layers)
    bounds = [lo for lo, _ in layers] + [layers[-1][1]]
    master, m, v = synth.state_warm(psi_p, seed=81)
    w_r, m_r, v_r = master.numpy(), m.numpy(), v.numpy()
    p16 = oracle.f2h(w_r)
    ref_shards = [p16[q * S:(q + 1) * S].copy() for q in range(nd)]
    shards = _partitions(p16, nd, S)
    cur = [x.to(DEV) for x in (master, m, v)]
    nxt = [torch.empty_like(x) for x in cur]
    pool = _Pool(pl, bounds, n_bufs)
    gs = torch.cuda.Stream()
    sched = lz.zero_layer_sched_create(pl, bounds, shards, pool.mem, pool.elems, n_bufs, gs)
    main = torch.cuda.current_stream()
    for i, (t, bad) in enumerate([(1, False), (2, True), (2, False)]):
        g_cpu = []
        for r in range(nd):
            g = torch.zeros(psi_p, dtype=torch.float16)
            g[:psi] = synth.grad_f16(psi, 1e-3, seed=82, rank=r, step=10 * i + t)
            g_cpu.append(g)
        if bad:
            g_cpu[1][layers[2][0] + 3] = float("nan")
        grads = [g.to(DEV) for g in g_cpu]
        st = status_word()
        n0 = lz.zero_layer_sched_gathers(sched)
        fwd, bwd = _run_step(sched, pool, pl, layers, gb, grads, cur, nxt, shards, t, st, main)
        assert lz.zero_layer_sched_gathers(sched) - n0 == 2 * L
        code, flags = lz.zero_step_status(st)
        ref = oracle.zero3_step(opl, layers, lambda l, r: g_cpu[r].numpy()[gb[l][0]:gb[l][1]],
                                w_r, m_r, v_r, ref_shards, ORC_HP, t)
        for l in range(L):
            assert np.array_equal(f16np(fwd[l]), ref.gathered_fwd[l]), ("fwd", i, l)
            assert np.array_equal(f16np(bwd[l]), ref.gathered_bwd[l]), ("bwd", i, l)
        assert ref.skipped == bad
        assert code == (lz.ZERO_STEP_SKIPPED if bad else lz.ZERO_OK)
        cur, nxt = nxt, cur
        check_f32(f"attempt {i} master", f32np(cur[0]), ref.master)
        check_f32(f"attempt {i} m", f32np(cur[1]), ref.m)
        check_f32(f"attempt {i} v", f32np(cur[2]), ref.v)
        for q in range(nd):
            check_f16(f"attempt {i} partition {q}", f16np(shards[q]), ref.param_shards[q])
        w_r, m_r, v_r, ref_shards = ref.master, ref.m, ref.v, ref.param_shards


@pytest.mark.parametrize("n_bufs", [2, 3])
def test_layer_scheduler_two_compute_streams(n_bufs):
    """Layers acquired and released on two compute streams in turn (a release on one stream
    does not order the other's): every layer as acquired, forward and backward, equals the
    partitions' values, three steps in a row through one scheduler."""
    numels, nd = [3000, 7001, 512, 9000, 2048, 4000], 4
    pl = lz.zero_plan_create(numels, nd, 3, 0)
    psi, psi_p, S, _ = lz.zero_plan_info(pl)
    offs = lz.zero_plan_tensor_offsets(pl)
    bounds = list(offs) + [psi_p]
    L = len(bounds) - 1
    pool = _Pool(pl, bounds, n_bufs)
    gs = torch.cuda.Stream()
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    main = torch.cuda.current_stream()
    st = status_word()
    for step in range(3):
        full = torch.randint(-(1 << 15), 1 << 15, (psi_p,), dtype=torch.int16,
                             device=DEV).view(torch.float16)
        shards = [full[q * S:(q + 1) * S].clone() for q in range(nd)]
        if step == 0:
            sched = lz.zero_layer_sched_create(pl, bounds, shards, pool.mem, pool.elems, n_bufs,
                                               gs)
            keep = shards
        else:                       # new values in the same partitions, as an update would write
            for k, x in zip(keep, shards):
                k.copy_(x)
        for c in streams:
            c.wait_stream(main)
        lz.zero_layer_sched_begin_step(sched, st, main)
        seen = []
        order = list(range(L)) + list(reversed(range(L)))
        for i, l in enumerate(order):
            c = streams[i % 2]
            nxt = order[i + 1] if i + 1 < len(order) else -1
            p = lz.zero_layer_sched_acquire(sched, l, nxt, c)
            with torch.cuda.stream(c):
                seen.append((l, pool.view(p, bounds[l + 1] - bounds[l]).clone()))
            lz.zero_layer_sched_release(sched, l, c)
        for c in streams:
            main.wait_stream(c)
        torch.cuda.synchronize()
        for l, got in seen:
            lo, hi = bounds[l], bounds[l + 1]
            assert torch.equal(got.view(torch.int16), full[lo:hi].view(torch.int16)), (step, l)
    assert lz.zero_step_status(st) == (lz.ZERO_OK, 0)


def test_layer_scheduler_bookkeeping():
    """Host-side rules on a live scheduler: a layer cannot be acquired twice or released
    unacquired; a step cannot begin while a layer is held; with every buffer held the next
    acquire reports ZERO_ENOMEM; an unused prefetch is dropped, and a dropped or released layer
    is gathered again when acquired."""
    numels, nd = [1000, 3000, 500, 2000], 4
    pl = lz.zero_plan_create(numels, nd, 3, 0)
    psi, psi_p, S, _ = lz.zero_plan_info(pl)
    bounds = [0, 1000, 4000, 4500, psi_p]
    full = torch.randint(-(1 << 15), 1 << 15, (psi_p,), dtype=torch.int16,
                         device=DEV).view(torch.float16)
    shards = [full[q * S:(q + 1) * S].clone() for q in range(nd)]
    pool = _Pool(pl, bounds, 2)
    sched = lz.zero_layer_sched_create(pl, bounds, shards, pool.mem, pool.elems, 2, None)
    st = status_word()

    def rejects(code, fn, *a):
        with pytest.raises(lz.ZeroError) as e:
            fn(*a)
        assert e.value.code == code

    rejects(lz.ZERO_EINVAL, lz.zero_layer_sched_acquire, sched, 0, -1, None)  # before a step
    lz.zero_layer_sched_begin_step(sched, st)
    p0 = lz.zero_layer_sched_acquire(sched, 0, 2)          # gathers 0, prefetches 2
    assert lz.zero_layer_sched_gathers(sched) == 2
    rejects(lz.ZERO_EINVAL, lz.zero_layer_sched_acquire, sched, 0, -1, None)
    rejects(lz.ZERO_EINVAL, lz.zero_layer_sched_release, sched, 1, None)
    rejects(lz.ZERO_EINVAL, lz.zero_layer_sched_acquire, sched, 4, -1, None)
    rejects(lz.ZERO_EINVAL, lz.zero_layer_sched_begin_step, sched, st, None)
    p1 = lz.zero_layer_sched_acquire(sched, 1, -1)         # drops the unused prefetch of 2
    assert lz.zero_layer_sched_gathers(sched) == 3
    rejects(lz.ZERO_ENOMEM, lz.zero_layer_sched_acquire, sched, 3, -1, None)
    torch.cuda.synchronize()
    for l, p in ((0, p0), (1, p1)):
        lo, hi = bounds[l], bounds[l + 1]
        assert torch.equal(pool.view(p, hi - lo).view(torch.int16), full[lo:hi].view(torch.int16))
    lz.zero_layer_sched_release(sched, 0)
    lz.zero_layer_sched_release(sched, 1)
    p2 = lz.zero_layer_sched_acquire(sched, 2, 3)          # 2 again (dropped), 3 prefetched
    assert lz.zero_layer_sched_gathers(sched) == 5
    lz.zero_layer_sched_release(sched, 2)
    p3 = lz.zero_layer_sched_acquire(sched, 3, -1)         # from the prefetch: no gather
    assert lz.zero_layer_sched_gathers(sched) == 5
    torch.cuda.synchronize()
    for l, p in ((2, p2), (3, p3)):
        lo, hi = bounds[l], bounds[l + 1]
        assert torch.equal(pool.view(p, hi - lo).view(torch.int16), full[lo:hi].view(torch.int16))
    lz.zero_layer_sched_release(sched, 3)
    lz.zero_layer_sched_begin_step(sched, st)              # nothing held: a new step may begin
    assert lz.zero_step_status(st) == (lz.ZERO_OK, 0)


def test_layer_scheduler_gpt2_small_layers():
    """The GPT-2-small list at Nd = 8 (14 layers) through the scheduler with two buffers, as
    bench.py times it: one step, every acquired layer equal to the partitions' values, state
    and partitions against the oracle's element arithmetic on sampled elements."""
    numels, nd = synth.gpt2_small_list(), 8
    pl = lz.zero_plan_create(numels, nd, 3, 0)
    psi, psi_p, S, _ = lz.zero_plan_info(pl)
    opl = oracle.plan(numels, nd, 0)
    layers = oracle.layer_ranges(opl, synth.gpt2_small_layers())
    gb = oracle.grad_buckets(opl, layers)
    bounds = [lo for lo, _ in layers] + [layers[-1][1]]
    rng = np.random.default_rng(91)
    idx = np.unique(np.concatenate([rng.integers(0, psi_p, 50_000),
                                    np.array([lo for lo, _ in layers]),
                                    np.arange(psi_p - 8, psi_p)]))
    idx_dev = torch.from_numpy(idx).to(DEV)
    cur = list(synth.state_small(psi_p, seed=92, device=DEV))
    nxt = [torch.empty_like(x) for x in cur]
    full = torch.empty(psi_p, dtype=torch.float16, device=DEV)
    full.copy_(cur[0])
    shards = [full[q * S:(q + 1) * S].clone() for q in range(nd)]
    grads = [torch.zeros(psi_p, dtype=torch.float16, device=DEV) for _ in range(nd)]
    for r in range(nd):
        synth.grad_f16(psi, 1e-3, seed=93, rank=r, step=1, out=grads[r][:psi])
    w_s, m_s, v_s = (cur[k][idx_dev].cpu().numpy() for k in range(3))
    gsmp = [g[idx_dev].cpu().numpy() for g in grads]
    pool = _Pool(pl, bounds, 2)
    gs = torch.cuda.Stream()
    sched = lz.zero_layer_sched_create(pl, bounds, shards, pool.mem, pool.elems, 2, gs)
    main = torch.cuda.current_stream()
    st = status_word()
    fwd, bwd = _run_step(sched, pool, pl, layers, gb, grads, cur, nxt, shards, 1, st, main,
                         prepared=True)
    assert lz.zero_step_status(st) == (lz.ZERO_OK, 0)
    for l, (lo, hi) in enumerate(layers):
        assert torch.equal(fwd[l].view(torch.int16), full[lo:hi].view(torch.int16)), l
        assert torch.equal(bwd[l].view(torch.int16), full[lo:hi].view(torch.int16)), l
    skipped, w_s, m_s, v_s, p_s = oracle.step(gsmp, w_s, m_s, v_s, ORC_HP, 1)
    assert not skipped
    check_f32("master", nxt[0][idx_dev].cpu().numpy(), w_s)
    check_f32("m", nxt[1][idx_dev].cpu().numpy(), m_s)
    check_f32("v", nxt[2][idx_dev].cpu().numpy(), v_s)
    check_f16("params", f16np(torch.cat(shards)[idx_dev]), p_s)


def test_stage3_step_captured_in_a_graph():
    """A whole stage-3 step -- the layer scheduler's forward and backward gathers on its gather
    stream, each layer's update with the step's constants in device memory
    (zero_stage3_step_fused_dc), the commit -- captured once per ping-pong direction as a CUDA
    graph on one capture stream and replayed: an eager first step, then replays at t = 2, an
    attempt whose gradients hold an inf (skipped, t not advanced), t = 3 and t = 4, each against
    zero3_step (state and partitions)."""
    numels, split, nd = [40000, 1234, 30000, 777, 5003, 999, 4096], [1, 2, 2, 2], 4
    pl = lz.zero_plan_create(numels, nd, 3, 0)
    psi, psi_p, S, _ = lz.zero_plan_info(pl)
    opl = oracle.plan(numels, nd, 0)
    layers = oracle.layer_ranges(opl, split)
    gb = oracle.grad_buckets(opl, layers)
    L = len(layers)
    bounds = [lo for lo, _ in layers] + [layers[-1][1]]
    master, m, v = synth.state_warm(psi_p, seed=101)
    w_r, m_r, v_r = master.numpy(), m.numpy(), v.numpy()
    p16 = oracle.f2h(w_r)
    ref_shards = [p16[q * S:(q + 1) * S].copy() for q in range(nd)]
    shards = _partitions(p16, nd, S)
    bufs = [[x.to(DEV) for x in (master, m, v)], [torch.empty(psi_p, dtype=torch.float32,
                                                              device=DEV) for _ in range(3)]]
    grads = [torch.zeros(psi_p, dtype=torch.float16, device=DEV) for _ in range(nd)]
    d_consts = torch.empty(lz.ZERO_ADAM_CONSTS_BYTES, dtype=torch.uint8, device=DEV)
    st = status_word()
    pool = _Pool(pl, bounds, 2)
    gs, cap = torch.cuda.Stream(), torch.cuda.Stream()
    sched = lz.zero_layer_sched_create(pl, bounds, shards, pool.mem, pool.elems, 2, gs)

    def body(d):
        cur, nxt = bufs[d], bufs[1 - d]
        st.zero_()
        lz.zero_layer_sched_begin_step(sched, st, cap)
        for l in range(L):
            lz.zero_layer_sched_acquire(sched, l, l + 1 if l + 1 < L else -1, cap)
            lz.zero_layer_sched_release(sched, l, cap)
        for l in reversed(range(L)):
            lo, _ = layers[l]
            _, ghi = gb[l]
            lz.zero_layer_sched_acquire(sched, l, l - 1, cap)
            lz.zero_layer_sched_release(sched, l, cap)
            lz.zero_stage3_step_fused_dc(pl, lo, ghi - lo, [g[lo:ghi] for g in grads],
                                         *[x[lo:ghi] for x in cur], *[x[lo:ghi] for x in nxt],
                                         shards, d_consts, st, cap)
        lz.zero_stage3_step_commit(pl, *cur, *nxt, shards, st, cap)

    def load(t, i, bad):
        g_cpu = []
        for r in range(nd):
            x = torch.zeros(psi_p, dtype=torch.float16)
            x[:psi] = synth.grad_f16(psi, 1e-3, seed=102, rank=r, step=10 * i + t)
            g_cpu.append(x)
        if bad:
            g_cpu[2][layers[1][0] + 9] = float("inf")
        c = lz.zero_adam_consts_for_step(HP, t)
        with torch.cuda.stream(cap):
            for g, x in zip(grads, g_cpu):
                g.copy_(x)
            d_consts.copy_(torch.frombuffer(bytearray(bytes(c)), dtype=torch.uint8))
        return g_cpu

    graphs = [None, None]
    attempts = [(1, False), (2, False), (3, True), (3, False), (4, False)]
    for i, (t, bad) in enumerate(attempts):
        d = i % 2
        g_cpu = load(t, i, bad)
        if i == 0:                                   # first use outside any capture
            with torch.cuda.stream(cap):
                body(d)
            cap.synchronize()
            for dd in (1, 0):
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g, stream=cap):
                    body(dd)
                graphs[dd] = g
            # the capture enqueued nothing: state and partitions hold step 1's results
        else:
            with torch.cuda.stream(cap):
                graphs[d].replay()
        cap.synchronize()
        code, flags = lz.zero_step_status(st, cap)
        ref = oracle.zero3_step(opl, layers, lambda l, r: g_cpu[r].numpy()[gb[l][0]:gb[l][1]],
                                w_r, m_r, v_r, ref_shards, ORC_HP, t)
        assert ref.skipped == bad
        assert code == (lz.ZERO_STEP_SKIPPED if bad else lz.ZERO_OK), (i, code, flags)
        out = bufs[1 - d]
        check_f32(f"attempt {i} master", f32np(out[0]), ref.master)
        check_f32(f"attempt {i} m", f32np(out[1]), ref.m)
        check_f32(f"attempt {i} v", f32np(out[2]), ref.v)
        for q in range(nd):
            check_f16(f"attempt {i} partition {q}", f16np(shards[q]), ref.param_shards[q])
        w_r, m_r, v_r, ref_shards = ref.master, ref.m, ref.v, ref.param_shards


def test_layer_scheduler_from_c(tmp_path):
    """A stage-3 step driven from C through the C ABI (tests/layer_sched_c.c, no Python in the
    loop): every layer as acquired equals the uploaded parameters, the steps end with status
    OK, two gathers per layer and step, and the host time of an acquire and of a release."""
    import json
    import os
    import subprocess
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    cuda = os.environ.get("CUDA_HOME", "/usr/local/cuda")
    libdir = os.path.dirname(lz.LIB_PATH)
    exe = str(tmp_path / "layer_sched_c")
    subprocess.check_call(["gcc", "-O2", "-std=c11", os.path.join(root, "tests", "layer_sched_c.c"),
                           "-I", os.path.join(root, "include"), "-I", os.path.join(cuda, "include"),
                           "-L", libdir, "-lzero", "-Wl,-rpath," + libdir,
                           "-L", os.path.join(cuda, "lib64"), "-lcudart",
                           "-Wl,-rpath," + os.path.join(cuda, "lib64"), "-o", exe])
    r = subprocess.run([exe, "8", "50"], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stdout + r.stderr
    d = json.loads(r.stdout.strip().splitlines()[-1])
    print("LAYER SCHED FROM C", json.dumps(d))
    assert d["ok"] and d["status"] == 0 and d["flags"] == 0
    assert d["gathers"] == d["steps"] * 2 * d["layers"]
    # an acquire records, waits and launches at most one or two gathers: a few microseconds
    assert d["host_us_acquire"] < 50 and d["host_us_release"] < 50
