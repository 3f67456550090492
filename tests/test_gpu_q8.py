"""The compressed (int8 + per-128 fp32 scale) reduce-scatter payload on the GPU against the
oracle: the quantizer bit for bit, the owner's fused step from the payload within the usual
tolerances (fp32 state 2 ulp, fp16 params 1 ulp), overflow carried through a poisoned block,
unaligned fallbacks, and the 7.5B shard view at Nd = 64 on sampled elements."""
import numpy as np
import pytest
import torch

import oracle
from tests._gpu import (DEV, HP, ORC_HP, PingPong, check_f16, check_f32, f16np, f32np, lz,
                        require_gpu, status_flags, status_word)
from zero_partitioned_optimizer_plan_b200 import synth

pytestmark = pytest.mark.gpu
QB = 128


@pytest.fixture(autouse=True)
def _gpu():
    require_gpu()
    torch.cuda.set_device(0)
    yield
    torch.cuda.synchronize()
    torch.cuda.empty_cache()


def _quant_dev(g_dev, off=0):
    """A rank's payload on the device (optionally at a byte offset inside a larger buffer)."""
    n = g_dev.numel()
    nbytes = lz.q8_payload_bytes(n)
    big = torch.zeros(nbytes + 32, dtype=torch.uint8, device=DEV)
    pay = big[off:off + nbytes]
    lz.zero_quantize_q8(n, g_dev, pay)
    return pay


def _q_of(codes):
    """Stored bytes (q + 128) -> q as int8."""
    return (codes.astype(np.int16) - 128).astype(np.int8)


def _split(pay, n):
    """Payload records -> (int8 values of the n elements, fp32 scale per block)."""
    rec = pay.cpu().numpy().reshape(-1, 132)
    q = _q_of(rec[:, :128].reshape(-1)[:n])
    sc = np.ascontiguousarray(rec[:, 128:]).view(np.float32).reshape(-1)
    return q, sc


def _same_scales(a, b):
    return np.array_equal(np.isnan(a), np.isnan(b)) and \
        np.array_equal(a[~np.isnan(a)].view(np.uint32), b[~np.isnan(b)].view(np.uint32))


@pytest.mark.parametrize("n", [1, 127, 128, 129, 4096 + 77, 300_005])
@pytest.mark.parametrize("kind", ["normal", "zeros", "poisoned", "unaligned"])
def test_quantize_bit_exact(n, kind):
    rng_seed = n + len(kind)
    g = synth.grad_f16(n, 1e-2, seed=rng_seed)
    if kind == "zeros":
        g[: min(n, 300)] = 0
    if kind == "poisoned":
        g[n // 2] = float("nan")
        g[0] = float("-inf")
    goff = 1 if kind == "unaligned" else 0
    gbig = torch.zeros(n + 8, dtype=torch.float16, device=DEV)
    gbig[goff:goff + n] = g.to(DEV)
    pay = _quant_dev(gbig[goff:goff + n], off=4 if kind == "unaligned" else 0)
    torch.cuda.synchronize()
    q, sc = _split(pay, n)
    q_ref, sc_ref = oracle.quant_q8(g.numpy())
    assert np.array_equal(q, q_ref)
    assert _same_scales(sc, sc_ref)
    # the stored bytes are q + 128; a short last block's unused bytes hold q = 0
    tail = n % 128
    if tail:
        assert (pay.cpu().numpy().reshape(-1, 132)[-1, tail:128] == 128).all()


def _near_tie_blocks(nblocks, seed):
    """Blocks of fp16 values that divide by their block's scale to within 2^-12 of a
    half-integer, some exactly onto one: the rounding decisions the quantizer must take as the
    IEEE quotient does. Each block's first value is its max |x|. Selection only: the expected
    bytes come from the oracle."""
    rng = np.random.default_rng(seed)
    pos = np.arange(1, 0x7c00, dtype=np.uint16).view(np.float16)   # positive finite fp16
    out = []
    while len(out) < nblocks:
        amax = pos[rng.integers(0x0400, 0x7c00 - 1)]
        s = np.float32(amax) / np.float32(127)
        cand = pos[pos <= amax]
        y = cand.astype(np.float32) / s
        near = cand[np.abs(y - np.floor(y) - np.float32(0.5)) < 2.0 ** -12]
        if near.size < 4:
            continue
        blk = near[rng.integers(0, near.size, 127)]
        blk = np.where(rng.random(127) < 0.5, -blk, blk).astype(np.float16)
        out.append(np.concatenate([[amax], blk]).astype(np.float16))
    return np.concatenate(out)


@pytest.mark.parametrize("off", [0, 1])
def test_quantize_near_ties_bit_exact(off):
    """Quotients at and next to half-integers (where a quotient formed by a reciprocal could
    round the other way) give the oracle's bytes, 16-byte aligned and not."""
    g = torch.from_numpy(_near_tie_blocks(600, seed=31 + off))
    n = g.numel() - 5                                   # and a short last block
    gbig = torch.zeros(g.numel() + 8, dtype=torch.float16, device=DEV)
    gbig[off:off + n] = g[:n].to(DEV)
    pay = _quant_dev(gbig[off:off + n])
    torch.cuda.synchronize()
    q, sc = _split(pay, n)
    q_ref, sc_ref = oracle.quant_q8(g[:n].numpy())
    assert np.array_equal(q, q_ref)
    assert _same_scales(sc, sc_ref)


@pytest.mark.parametrize("nd", [1, 2, 3, 8, 16, 25, 64])
@pytest.mark.parametrize("n", [9, 4096, 4096 + 300, 4096 + 511, 2048 * 40 + 777,
                               1_900_000 + 77])
def test_fused_q8_vs_oracle(n, nd):
    """Sizes for the plain kernel (9), the small-call shape (its tail of up to 511 elements
    past the last whole tile taken in several passes by 8 or 12 warps) and the large shape
    (1.9 M elements, above 4 tiles per SM)."""
    seed = 7 * n + nd
    master, m, v = synth.state_warm(n, seed=seed)
    pp = PingPong(master, m, v)
    w_r, m_r, v_r = master.numpy(), m.numpy(), v.numpy()
    params = torch.empty(n, dtype=torch.float16, device=DEV)
    for t in (1, 2):
        g_cpu = [synth.grad_f16(n, 1e-2, seed=seed, rank=r, step=t) for r in range(nd)]
        pay = [_quant_dev(g.to(DEV)) for g in g_cpu]
        st = status_word()
        ins, outs = pp.cur, pp.nxt
        lz.zero_step_fused_q8(n, nd, pay, *ins, *outs, params, HP, t, st)
        lz.zero_step_commit(n, *ins, *outs, params, st)
        torch.cuda.synchronize()
        assert status_flags(st) == 0
        pp.swap()
        ref_pay = [oracle.quant_q8(g.numpy()) for g in g_cpu]      # the oracle's own payload
        skipped, w_r, m_r, v_r, p_r = oracle.step_q8([q for q, _ in ref_pay],
                                                     [s for _, s in ref_pay], w_r, m_r, v_r,
                                                     ORC_HP, t)
        assert not skipped
        w, mm, vv = pp.numpy()
        # the kernel runs the oracle's operations in the oracle's order (one fma per rank in
        # rank order, the packed two-wide instructions being two ordinary IEEE operations), so
        # the results are held to 0 ulp, not to the general 2 / 1 ulp bound
        check_f32("master", w, w_r, tol=0)
        check_f32("m", mm, m_r, tol=0)
        check_f32("v", vv, v_r, tol=0)
        check_f16("params", f16np(params), p_r, tol=0)


def test_fused_q8_overflow_through_poisoned_block():
    n, nd = 2048 * 9 + 3, 4
    master, m, v = synth.state_warm(n, seed=5)
    pp = PingPong(master, m, v)
    g_dev = [synth.grad_f16(n, 1e-2, seed=6, rank=r).to(DEV) for r in range(nd)]
    g_dev[2][5000] = float("inf")
    pay = [_quant_dev(g) for g in g_dev]
    params = torch.zeros(n, dtype=torch.float16, device=DEV)
    st = status_word()
    lz.zero_step_fused_q8(n, nd, pay, *pp.cur, *pp.nxt, params, HP, 1, st)
    lz.zero_step_commit(n, *pp.cur, *pp.nxt, params, st)
    assert lz.zero_step_status(st)[0] == lz.ZERO_STEP_SKIPPED
    for a, b in zip(pp.cur, pp.nxt):
        assert torch.equal(a, b)
    assert np.array_equal(f16np(params), oracle.f2h(master.numpy()))


def test_fused_q8_unaligned_payload_takes_plain_kernel():
    n, nd = 50_000, 3
    master, m, v = synth.state_warm(n, seed=8)
    pp = PingPong(master, m, v)
    g_cpu = [synth.grad_f16(n, 1e-2, seed=9, rank=r) for r in range(nd)]
    pay = [_quant_dev(g.to(DEV), off=4) for g in g_cpu]     # 4- but not 16-byte aligned
    params = torch.empty(n, dtype=torch.float16, device=DEV)
    st = status_word()
    lz.zero_step_fused_q8(n, nd, pay, *pp.cur, *pp.nxt, params, HP, 1, st)
    torch.cuda.synchronize()
    assert status_flags(st) == 0
    ref = [oracle.quant_q8(g.numpy()) for g in g_cpu]
    skipped, w, mm, vv, p = oracle.step_q8([q for q, _ in ref], [s for _, s in ref],
                                           master.numpy(), m.numpy(), v.numpy(), ORC_HP, 1)
    check_f32("master", f32np(pp.nxt[0]), w)
    check_f16("params", f16np(params), p)


def test_7p5b_shard_view_q8_sampled():
    """Owner 63 of 7.5e9 parameters at Nd = 64 from int8 payloads, in the bench's launch
    configuration; sampled elements against the oracle on the gathered payload."""
    total, nd = 7_500_000_000, 64
    S = total // nd
    owner = 63
    full = torch.zeros(total, dtype=torch.float16, device=DEV)
    pays = []
    g = torch.empty(S, dtype=torch.float16, device=DEV)
    for r in range(nd):
        synth.grad_f16(S, 1e-3, seed=11, rank=r, out=g)
        pay = torch.empty(lz.q8_payload_bytes(S), dtype=torch.uint8, device=DEV)
        lz.zero_quantize_q8(S, g, pay)
        pays.append(pay)
    del g
    cur = list(synth.state_warm(S, seed=12, device=DEV))
    nxt = [torch.empty_like(x) for x in cur]
    rng = np.random.default_rng(13)
    idx = np.unique(np.concatenate([rng.integers(0, S, 100_000), np.arange(S - 600, S),
                                    np.arange(0, 256)]))
    idx_dev = torch.from_numpy(idx).to(DEV)
    qpos = torch.from_numpy((idx // QB) * 132 + idx % QB).to(DEV)
    spos = torch.from_numpy(((idx // QB) * 132 + 128)[:, None] + np.arange(4)).to(DEV)
    w0, m0, v0 = (x[idx_dev].cpu().numpy() for x in cur)
    out = full[owner * S:(owner + 1) * S]
    st = status_word()
    lz.zero_step_fused_q8(S, nd, pays, *cur, *nxt, out, HP, 1, st)
    lz.zero_step_commit(S, *cur, *nxt, out, st)
    torch.cuda.synchronize()
    assert status_flags(st) == 0
    gq = [_q_of(p[qpos].cpu().numpy()) for p in pays]
    gs = [np.ascontiguousarray(p[spos].cpu().numpy()).view(np.float32).reshape(-1) for p in pays]
    skipped, w, mm, vv, p = oracle.step_q8_gathered(gq, gs, w0, m0, v0, ORC_HP, 1)
    assert not skipped
    check_f32("master", nxt[0][idx_dev].cpu().numpy(), w)
    check_f32("m", nxt[1][idx_dev].cpu().numpy(), mm)
    check_f32("v", nxt[2][idx_dev].cpu().numpy(), vv)
    check_f16("params", out[idx_dev].cpu().numpy().view(np.uint16), p)
    assert int(torch.count_nonzero(full[:owner * S].view(torch.int16))) == 0


@pytest.mark.parametrize("nd", [2, 64])
def test_q8_device_constants_match(nd):
    """zero_step_fused_q8_dc (constants from device memory) gives the same bits as
    zero_step_fused_q8 with the hyperparameters and t, for the small and the large shape."""
    for n in (2048 * 21 + 3, 1_900_000 + 77):
        g_dev = [synth.grad_f16(n, 1e-2, seed=81, rank=r, step=1).to(DEV) for r in range(nd)]
        pay = [_quant_dev(g) for g in g_dev]
        master, m, v = (x.to(DEV) for x in synth.state_warm(n, seed=82))
        for t in (1, 7):
            c = lz.zero_adam_consts_for_step(HP, t)
            dc = torch.frombuffer(bytearray(bytes(c)), dtype=torch.uint8).to(DEV)
            outs_a = [torch.empty_like(x) for x in (master, m, v)]
            outs_b = [torch.empty_like(x) for x in (master, m, v)]
            pa = torch.empty(n, dtype=torch.float16, device=DEV)
            pb = torch.empty(n, dtype=torch.float16, device=DEV)
            st = status_word()
            lz.zero_step_fused_q8(n, nd, pay, master, m, v, *outs_a, pa, HP, t, st)
            lz.zero_step_fused_q8_dc(n, nd, pay, master, m, v, *outs_b, pb, dc, st)
            torch.cuda.synchronize()
            assert status_flags(st) == 0
            for a, b in list(zip(outs_a, outs_b)) + [(pa, pb)]:
                assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_q8_graph_with_device_scaler():
    """Per-bucket int8 steps in an overlap region between zero_scaler_prepare and
    zero_scaler_update, captured as CUDA graphs and replayed for ten steps, three of them with
    an inf in a rank's gradient (its block poisoned by the quantizer): state, parameters and
    scaler equal the oracle's int8 steps under the same scaling rule."""
    import dataclasses
    nd, n, B = 4, 2048 * 12 + 5, 7168
    overflow = [False, False, False, True, True, False, False, False, True, False]
    bounds = [(lo, min(n, lo + B)) for lo in range(0, n, B)][::-1]
    master, m, v = synth.state_warm(n, seed=83)
    bufs = [[x.to(DEV) for x in (master, m, v)], [torch.empty(n, device=DEV) for _ in range(3)]]
    grads = [torch.empty(n, dtype=torch.float16, device=DEV) for _ in range(nd)]
    pays = {lo: [torch.empty(lz.q8_payload_bytes(hi - lo), dtype=torch.uint8, device=DEV)
                 for _ in range(nd)] for lo, hi in bounds}
    params = torch.empty(n, dtype=torch.float16, device=DEV)
    table = lz.zero_adam_consts_table(HP, 1, 32)
    d_table = torch.frombuffer(bytearray(bytes(table)), dtype=torch.uint8).to(DEV)
    d_consts = torch.empty(lz.ZERO_ADAM_CONSTS_BYTES, dtype=torch.uint8, device=DEV)
    init = lz.ScalerState(1024.0, 0, 1, 0)
    d_state = torch.frombuffer(bytearray(bytes(init)), dtype=torch.uint8).to(DEV)
    prm = lz.ScalerParams(2.0, 0.5, 2)
    st = status_word()

    def step(src, dst):
        lz.zero_scaler_prepare(d_state, d_table, 32, d_consts, st)
        with lz.overlap():
            for lo, hi in bounds:
                lz.zero_step_fused_q8_dc(hi - lo, nd, pays[lo], *[x[lo:hi] for x in src],
                                         *[x[lo:hi] for x in dst], params[lo:hi], d_consts, st)
        lz.zero_step_commit(n, *src, *dst, params, st)
        lz.zero_scaler_update(d_state, prm, st)

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
    d_state.copy_(torch.frombuffer(bytearray(bytes(init)), dtype=torch.uint8).to(DEV))
    torch.cuda.synchronize()

    sc = oracle.Scaler(scale=1024.0, growth_interval=2)
    w_r, m_r, v_r = master.numpy(), m.numpy(), v.numpy()
    p_r = None
    for i, bad in enumerate(overflow):
        g_cpu = [synth.grad_f16(n, 1e-2, seed=84, rank=r, step=i) for r in range(nd)]
        if bad:
            g_cpu[nd - 1][n // 3] = float("inf")
        for d, s in zip(grads, g_cpu):
            d.copy_(s.to(DEV))
        for lo, hi in bounds:                    # the senders quantize each bucket
            for r in range(nd):
                lz.zero_quantize_q8(hi - lo, grads[r][lo:hi], pays[lo][r])
        graphs[i % 2].replay()
        # oracle: each bucket's payload from its own range; one skip decision for the step
        hp_t = dataclasses.replace(ORC_HP, loss_scale=sc.scale)
        parts, skipped = {}, False
        for lo, hi in bounds:
            ref = [oracle.quant_q8(g.numpy()[lo:hi]) for g in g_cpu]
            sk, w, mm, vv, p = oracle.step_q8([q for q, _ in ref], [s for _, s in ref],
                                              w_r[lo:hi], m_r[lo:hi], v_r[lo:hi], hp_t,
                                              sc.next_step)
            skipped |= sk
            parts[lo] = (w, mm, vv, p)
        assert skipped == bad
        if not skipped:
            w_r, m_r, v_r = (np.concatenate([parts[lo][k] for lo, _ in bounds[::-1]])
                             for k in range(3))
            p_r = np.concatenate([parts[lo][3] for lo, _ in bounds[::-1]])
        sc.update(skipped)
    torch.cuda.synchronize()
    out = bufs[len(overflow) % 2]
    check_f32("master", f32np(out[0]), w_r)
    check_f32("m", f32np(out[1]), m_r)
    check_f32("v", f32np(out[2]), v_r)
    check_f16("params", f16np(params), p_r)
    s = lz.ScalerState()
    import ctypes as C
    C.memmove(C.addressof(s), bytes(d_state.cpu().numpy().tobytes()), C.sizeof(s))
    assert (s.scale, s.good_steps, s.next_step, s.skipped_steps) == \
        (np.float32(sc.scale), sc.good_steps, sc.next_step, sc.skipped_steps)
    del graphs


@pytest.mark.parametrize("nd", [8, 64])
def test_step_fused_q8_ranges_vs_oracle(nd):
    """zero_step_fused_q8_ranges over buckets of every kernel shape (one above 4 tiles per SM,
    small-call ones, one under 4096 elements for the plain kernel), each bucket's payload
    quantized from its own range: the same bits as per-bucket zero_step_fused_q8 calls in a
    region, and the oracle's per-bucket owner steps (0 ulp)."""
    sizes = [1_900_032, 3072 * 4, 3072 * 2 + 512, 1000]
    n = sum(sizes) + 333
    bounds, lo = [], 0
    for sz in sizes + [333]:
        bounds.append((lo, lo + sz))
        lo += sz
    bounds = bounds[::-1]                                   # backward order
    g_cpu = [synth.grad_f16(n, 1e-2, seed=91, rank=r, step=1) for r in range(nd)]
    g_dev = [g.to(DEV) for g in g_cpu]
    pays = {}
    for lo, hi in bounds:
        pays[lo] = []
        for g in g_dev:
            pay = torch.empty(lz.q8_payload_bytes(hi - lo), dtype=torch.uint8, device=DEV)
            lz.zero_quantize_q8(hi - lo, g[lo:hi], pay)
            pays[lo].append(pay)
    del g_dev
    master, m, v = synth.state_warm(n, seed=92)
    ins = [x.to(DEV) for x in (master, m, v)]
    outs_a = [torch.empty_like(x) for x in ins]
    outs_b = [torch.empty_like(x) for x in ins]
    pa = torch.empty(n, dtype=torch.float16, device=DEV)
    pb = torch.empty(n, dtype=torch.float16, device=DEV)
    st = status_word()
    lz.zero_step_fused_q8_ranges(nd, [
        (hi - lo, pays[lo], *[x[lo:hi] for x in ins], *[x[lo:hi] for x in outs_a], pa[lo:hi])
        for lo, hi in bounds], HP, 1, st)
    with lz.overlap():
        for lo, hi in bounds:
            lz.zero_step_fused_q8(hi - lo, nd, pays[lo], *[x[lo:hi] for x in ins],
                                  *[x[lo:hi] for x in outs_b], pb[lo:hi], HP, 1, st)
    torch.cuda.synchronize()
    assert status_flags(st) == 0
    for a, b in list(zip(outs_a, outs_b)) + [(pa, pb)]:
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    w, mm, vv = master.numpy().copy(), m.numpy().copy(), v.numpy().copy()
    p = np.empty(n, np.uint16)
    for lo, hi in bounds:
        ref = [oracle.quant_q8(g.numpy()[lo:hi]) for g in g_cpu]
        skipped, w[lo:hi], mm[lo:hi], vv[lo:hi], p[lo:hi] = oracle.step_q8(
            [q for q, _ in ref], [s for _, s in ref], w[lo:hi], mm[lo:hi], vv[lo:hi], ORC_HP, 1)
        assert not skipped
    check_f32("master", f32np(outs_a[0]), w, tol=0)
    check_f32("m", f32np(outs_a[1]), mm, tol=0)
    check_f32("v", f32np(outs_a[2]), vv, tol=0)
    check_f16("params", f16np(pa), p, tol=0)


def _byte_view(slots, ptr, n):
    off = ptr - slots.data_ptr()
    assert 0 <= off and off + n <= slots.numel()
    return slots[off:off + n]


@pytest.mark.parametrize("n_slots", [1, 2])
def test_q8_bucket_scheduler_vs_oracle(n_slots):
    """Stage 2 with the int8 payload through one scheduler (zero_sched_create_fused_q8): each
    bucket's part of every rank's gradient quantized into the slot region that
    zero_sched_begin_bucket_q8 hands out (records counted from the bucket's first element), the
    int8 fused step launched per bucket, one commit. Four attempts -- t = 1, an attempt with a
    poisoned block (skipped, t not advanced), t = 2, t = 3 -- against the oracle's quantizer and
    int8 step over the same buckets; the state bit for bit (one fma per rank, as the oracle)."""
    numels, nd, bucket = [40000, 1234, 30000, 777], 6, 9000
    pl = lz.zero_plan_create(numels, nd, 2, bucket)
    psi, psi_p, S, nb = lz.zero_plan_info(pl)
    master, m, v = synth.state_warm(psi_p, seed=141)
    pp = PingPong(master, m, v)
    params = torch.from_numpy(oracle.f2h(master.numpy()).view(np.float16)).to(DEV)
    nbytes = lz.zero_sched_slot_bytes_q8(pl, n_slots)
    slots = torch.empty(nbytes, dtype=torch.uint8, device=DEV)
    d_consts = torch.empty(lz.ZERO_ADAM_CONSTS_BYTES, dtype=torch.uint8, device=DEV)
    producer, stream = torch.cuda.Stream(), torch.cuda.Stream()
    main = torch.cuda.current_stream()
    sch = lz.zero_sched_create_fused_q8(pl, slots, nbytes, n_slots, *pp.cur, *pp.nxt, params,
                                        d_consts, status_word(), stream)
    with pytest.raises(lz.ZeroError):             # the fp16 hand-out is refused here
        lz.zero_sched_begin_bucket(sch, 0, producer)
    w, mm, vv = master.numpy(), m.numpy(), v.numpy()
    p16 = oracle.f2h(w)
    buckets = [lz.zero_plan_bucket(pl, k)[:2] for k in range(nb)]
    for i, (t, bad) in enumerate([(1, None), (2, (nb // 2, 4)), (2, None), (3, None)]):
        g = []
        for r in range(nd):
            x = torch.zeros(psi_p, dtype=torch.float16)
            x[:psi] = synth.grad_f16(psi, 1e-3, seed=142, rank=r, step=10 * i + t)
            g.append(x)
        if bad is not None:
            k, r = bad
            g[r][buckets[k][0] + 5] = float("nan")
        st = status_word()
        c = lz.zero_adam_consts_for_step(HP, t)
        d_consts.copy_(torch.frombuffer(bytearray(bytes(c)), dtype=torch.uint8))
        torch.cuda.synchronize()
        lz.zero_sched_rebind_fused(sch, *pp.cur, *pp.nxt, params, st)
        g_dev = [x.to(DEV) for x in g]
        torch.cuda.synchronize()
        lz.zero_overlap_begin(stream)
        with torch.cuda.stream(producer):
            for k, (lo, ln) in enumerate(buckets):
                ptrs = lz.zero_sched_begin_bucket_q8(sch, k, producer)
                for r in range(nd):
                    lz.zero_quantize_q8(ln, g_dev[r][lo:lo + ln],
                                        _byte_view(slots, ptrs[r], lz.q8_payload_bytes(ln)),
                                        producer)
                lz.zero_sched_end_bucket(sch, k, producer)
        lz.zero_overlap_end(stream)
        lz.zero_sched_wait(sch, main)
        lz.zero_step_commit(psi_p, *pp.cur, *pp.nxt, params, st, main)
        code, flags = lz.zero_step_status(st, main)
        # the oracle: each bucket's parts quantized from the bucket's first element, the int8
        # step per bucket; any overflow skips the whole step
        w2, m2, v2, p2 = w.copy(), mm.copy(), vv.copy(), p16.copy()
        skipped = False
        for lo, ln in buckets:
            qs = [oracle.quant_q8(x.numpy()[lo:lo + ln]) for x in g]
            sk, wb, mb, vb, pb = oracle.step_q8([q for q, _ in qs], [sc for _, sc in qs],
                                                w[lo:lo + ln], mm[lo:lo + ln], vv[lo:lo + ln],
                                                ORC_HP, t)
            skipped |= sk
            if not sk:
                w2[lo:lo + ln], m2[lo:lo + ln], v2[lo:lo + ln], p2[lo:lo + ln] = wb, mb, vb, pb
        assert skipped == (bad is not None)
        if skipped:
            assert code == lz.ZERO_STEP_SKIPPED
        else:
            assert (code, flags) == (lz.ZERO_OK, 0)
            w, mm, vv, p16 = w2, m2, v2, p2
        pp.swap()
        check_f32(f"attempt {i} master", f32np(pp.cur[0]), w, tol=0)
        check_f32(f"attempt {i} m", f32np(pp.cur[1]), mm, tol=0)
        check_f32(f"attempt {i} v", f32np(pp.cur[2]), vv, tol=0)
        check_f16(f"attempt {i} params", f16np(params), p16, tol=0)
    lz.zero_sched_destroy(sch)


@pytest.mark.parametrize("nd", [3, 8])
def test_stage3_q8_steps_vs_oracle(nd):
    """Stage 3 with the int8 gradient payload: per layer in backward order each rank's gradient
    bucket quantized into one segment per owner part (zero_stage3_quantize_q8; the segments
    bit for bit against the oracle's quantizer of each part), then the owners' int8 fused
    update into their partitions (zero_stage3_step_fused_q8), then the commit. Three attempts
    (t = 1, a poisoned block at t = 2 that skips the step, t = 2): state and partitions
    against the oracle's int8 step over the same parts, bit for bit."""
    numels, split = [40000, 1234, 30000, 777, 5003], [1, 2, 2]
    pl = lz.zero_plan_create(numels, nd, 3, 0)
    psi, psi_p, S, _ = lz.zero_plan_info(pl)
    opl = oracle.plan(numels, nd, 0)
    layers = oracle.layer_ranges(opl, split)
    gb = oracle.grad_buckets(opl, layers)
    master, m, v = synth.state_warm(psi_p, seed=151)
    w, mm, vv = master.numpy(), m.numpy(), v.numpy()
    p16 = oracle.f2h(w)
    shards = [torch.from_numpy(p16[q * S:(q + 1) * S].view(np.float16)).to(DEV)
              for q in range(nd)]
    pp = PingPong(master, m, v)

    def parts(lo, hi):                  # the owner parts of [lo, hi), in owner order
        out, a = [], lo
        while a < hi:
            b = min(hi, (a // S + 1) * S)
            out.append((a, b))
            a = b
        return out

    for i, (t, bad) in enumerate([(1, False), (2, True), (2, False)]):
        g = []
        for r in range(nd):
            x = torch.zeros(psi_p, dtype=torch.float16)
            x[:psi] = synth.grad_f16(psi, 1e-3, seed=152, rank=r, step=10 * i + t)
            g.append(x)
        if bad:
            g[nd - 1][layers[1][0] + 11] = float("nan")
        g_dev = [x.to(DEV) for x in g]
        st = status_word()
        for l in reversed(range(len(layers))):
            lo, ghi = gb[l]
            nb = lz.zero_stage3_payload_bytes_q8(pl, lo, ghi - lo)
            assert nb == sum((lz.q8_payload_bytes(b - a) + 15) // 16 * 16 for a, b in parts(lo, ghi))
            pays = [torch.empty(nb, dtype=torch.uint8, device=DEV) for _ in range(nd)]
            for r in range(nd):
                lz.zero_stage3_quantize_q8(pl, lo, ghi - lo, g_dev[r][lo:ghi], pays[r])
            if l == 0:                  # the segments of rank 0 against the oracle's quantizer
                got, off = pays[0].cpu().numpy(), 0
                for a, b in parts(lo, ghi):
                    q, sc = oracle.quant_q8(g[0].numpy()[a:b])
                    rec = got[off:off + lz.q8_payload_bytes(b - a)].reshape(-1, 132)
                    assert np.array_equal(_q_of(rec[:, :128]).reshape(-1)[:b - a], q)
                    assert np.array_equal(rec[:, 128:].copy().view(np.float32).reshape(-1), sc)
                    off += (lz.q8_payload_bytes(b - a) + 15) // 16 * 16
            lz.zero_stage3_step_fused_q8(pl, lo, ghi - lo, pays, *[x[lo:ghi] for x in pp.cur],
                                         *[x[lo:ghi] for x in pp.nxt], shards, HP, t, st)
        lz.zero_stage3_step_commit(pl, *pp.cur, *pp.nxt, shards, st)
        code, flags = lz.zero_step_status(st)
        w2, m2, v2, p2 = w.copy(), mm.copy(), vv.copy(), p16.copy()
        skipped = False
        for lo, ghi in gb:
            for a, b in parts(lo, ghi):
                qs = [oracle.quant_q8(x.numpy()[a:b]) for x in g]
                sk, wb, mb, vb, pb = oracle.step_q8([q for q, _ in qs], [c for _, c in qs],
                                                    w[a:b], mm[a:b], vv[a:b], ORC_HP, t)
                skipped |= sk
                if not sk:
                    w2[a:b], m2[a:b], v2[a:b], p2[a:b] = wb, mb, vb, pb
        assert skipped == bad
        assert code == (lz.ZERO_STEP_SKIPPED if bad else lz.ZERO_OK), (code, flags)
        if not bad:
            w, mm, vv, p16 = w2, m2, v2, p2
        pp.swap()
        check_f32(f"attempt {i} master", f32np(pp.cur[0]), w, tol=0)
        check_f32(f"attempt {i} m", f32np(pp.cur[1]), mm, tol=0)
        check_f32(f"attempt {i} v", f32np(pp.cur[2]), vv, tol=0)
        for q in range(nd):
            check_f16(f"attempt {i} partition {q}", f16np(shards[q]), p16[q * S:(q + 1) * S],
                      tol=0)


def test_stage3_q8_step_captured_in_a_graph():
    """A stage-3 step from int8 payloads with the constants in device memory
    (zero_stage3_step_fused_q8_dc), the layer gathers by the layer scheduler and the commit,
    captured as a CUDA graph per ping-pong direction and replayed at t = 1, 2, 3 (the payloads
    rewritten in place between replays): state and partitions against the oracle's int8 step
    per owner part, bit for bit."""
    numels, split, nd = [40000, 1234, 30000, 777, 5003], [1, 2, 2], 4
    pl = lz.zero_plan_create(numels, nd, 3, 0)
    psi, psi_p, S, _ = lz.zero_plan_info(pl)
    opl = oracle.plan(numels, nd, 0)
    layers = oracle.layer_ranges(opl, split)
    gb = oracle.grad_buckets(opl, layers)
    L = len(layers)
    bounds = [lo for lo, _ in layers] + [layers[-1][1]]
    master, m, v = synth.state_warm(psi_p, seed=161)
    w, mm, vv = master.numpy(), m.numpy(), v.numpy()
    p16 = oracle.f2h(w)
    shards = [torch.from_numpy(p16[q * S:(q + 1) * S].view(np.float16)).to(DEV)
              for q in range(nd)]
    bufs = [[x.to(DEV) for x in (master, m, v)],
            [torch.empty(psi_p, dtype=torch.float32, device=DEV) for _ in range(3)]]
    g_dev = [torch.zeros(psi_p, dtype=torch.float16, device=DEV) for _ in range(nd)]
    pays = [[torch.empty(lz.zero_stage3_payload_bytes_q8(pl, lo, hi - lo), dtype=torch.uint8,
                         device=DEV) for _ in range(nd)] for lo, hi in gb]
    d_consts = torch.empty(lz.ZERO_ADAM_CONSTS_BYTES, dtype=torch.uint8, device=DEV)
    st = status_word()
    elems = lz.zero_layer_sched_buf_elems(pl, bounds, 2)
    pool = torch.empty(elems, dtype=torch.float16, device=DEV)
    gs, cap = torch.cuda.Stream(), torch.cuda.Stream()
    sched = lz.zero_layer_sched_create(pl, bounds, shards, pool, elems, 2, gs)

    def body(d):
        cur, nxt = bufs[d], bufs[1 - d]
        st.zero_()
        lz.zero_layer_sched_begin_step(sched, st, cap)
        for l in range(L):
            lz.zero_layer_sched_acquire(sched, l, l + 1 if l + 1 < L else -1, cap)
            lz.zero_layer_sched_release(sched, l, cap)
        for l in reversed(range(L)):
            lo, ghi = gb[l]
            lz.zero_layer_sched_acquire(sched, l, l - 1, cap)
            lz.zero_layer_sched_release(sched, l, cap)
            lz.zero_stage3_step_fused_q8_dc(pl, lo, ghi - lo, pays[l], *[x[lo:ghi] for x in cur],
                                            *[x[lo:ghi] for x in nxt], shards, d_consts, st, cap)
        lz.zero_stage3_step_commit(pl, *cur, *nxt, shards, st, cap)

    def parts(lo, hi):
        out, a = [], lo
        while a < hi:
            b = min(hi, (a // S + 1) * S)
            out.append((a, b))
            a = b
        return out

    graphs = [None, None]
    for i, t in enumerate((1, 2, 3)):
        d = i % 2
        g = []
        for r in range(nd):
            x = torch.zeros(psi_p, dtype=torch.float16)
            x[:psi] = synth.grad_f16(psi, 1e-3, seed=162, rank=r, step=t)
            g.append(x)
        c = lz.zero_adam_consts_for_step(HP, t)
        with torch.cuda.stream(cap):
            for gd, x in zip(g_dev, g):
                gd.copy_(x)
            for (lo, ghi), pl_pays in zip(gb, pays):
                for r in range(nd):
                    lz.zero_stage3_quantize_q8(pl, lo, ghi - lo, g_dev[r][lo:ghi], pl_pays[r], cap)
            d_consts.copy_(torch.frombuffer(bytearray(bytes(c)), dtype=torch.uint8))
        if i == 0:                                   # first use outside any capture
            with torch.cuda.stream(cap):
                body(d)
            cap.synchronize()
            for dd in (1, 0):
                gr = torch.cuda.CUDAGraph()
                with torch.cuda.graph(gr, stream=cap):
                    body(dd)
                graphs[dd] = gr
        else:
            with torch.cuda.stream(cap):
                graphs[d].replay()
        cap.synchronize()
        assert lz.zero_step_status(st, cap) == (lz.ZERO_OK, 0)
        w2, m2, v2, p2 = w.copy(), mm.copy(), vv.copy(), p16.copy()
        for lo, ghi in gb:
            for a, b in parts(lo, ghi):
                qs = [oracle.quant_q8(x.numpy()[a:b]) for x in g]
                sk, wb, mb, vb, pb = oracle.step_q8([q for q, _ in qs], [s_ for _, s_ in qs],
                                                    w[a:b], mm[a:b], vv[a:b], ORC_HP, t)
                assert not sk
                w2[a:b], m2[a:b], v2[a:b], p2[a:b] = wb, mb, vb, pb
        w, mm, vv, p16 = w2, m2, v2, p2
        out = bufs[1 - d]
        check_f32(f"step {t} master", f32np(out[0]), w, tol=0)
        check_f32(f"step {t} m", f32np(out[1]), mm, tol=0)
        check_f32(f"step {t} v", f32np(out[2]), vv, tol=0)
        for q in range(nd):
            check_f16(f"step {t} partition {q}", f16np(shards[q]), p16[q * S:(q + 1) * S], tol=0)
