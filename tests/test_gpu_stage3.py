"""Stage 3 (Pos+g+p) through the C ABI against the oracle: the just-in-time parameter gather
bit for bit (ragged ranges, layers across owners, unaligned partitions and outputs, up to 64
owners, the GPT-2-small layers), and whole stage-3 steps -- forward gathers, backward gathers
with each layer's fused update into the owners' partitions, commit -- against zero3_step
("Como funciona": parameters partitioned, 3 psi per step; "ZeRO" (lastdictionary): layers
gathered just in time). Tolerances as in test_gpu_parity.py (measured: 0 ulp)."""
import numpy as np
import pytest
import torch

import oracle
from tests._gpu import (DEV, HP, ORC_HP, check_f16, check_f32, f16np, f32np, lz, require_gpu,
                        status_flags, status_word)
from zero_partitioned_optimizer_plan_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _gpu():
    require_gpu()
    torch.cuda.set_device(0)
    yield
    torch.cuda.synchronize()


def _partitions(full16_cpu, nd, shift_elems=()):
    """The owners' partitions as separate device buffers; partition q starts shift_elems[q]
    elements into its allocation (to make its address 2-, 4- or 8-byte aligned)."""
    S = full16_cpu.numel() // nd
    out = []
    for q in range(nd):
        sh = shift_elems[q] if shift_elems else 0
        buf = torch.zeros(S + 8, dtype=torch.float16, device=DEV)
        view = buf[sh:sh + S]
        view.copy_(full16_cpu[q * S:(q + 1) * S])
        out.append(view)
    return out


CASES = [  # numels, nd, (flat_lo, len) ranges as fractions or exact
    ([1000, 3, 999, 5], 3), ([7], 3), ([5, 40, 1, 17, 3, 90, 2], 8), ([123457], 64),
    ([4096 * 5 + 3], 2), ([300000, 250000, 250000, 248576], 4), ([65536 * 3 + 17], 5),
]


@pytest.mark.parametrize("numels,nd", CASES)
@pytest.mark.parametrize("shift", [0, 1, 2, 3])
def test_gather_params_bit_exact(numels, nd, shift):
    """Random ranges (single elements, shorter than a 16-byte chunk, within one partition,
    across several) into outputs at every 2-byte offset; partitions shifted by `shift` * q
    elements. Bit-exact against the oracle's gather; nothing outside the output written."""
    pl = lz.zero_plan_create(numels, nd, 3, 0)
    psi, psi_p, S, _ = lz.zero_plan_info(pl)
    rng = np.random.default_rng(psi + nd + shift)
    full = torch.from_numpy(rng.integers(0, 1 << 16, psi_p, dtype=np.uint16).view(np.int16)
                            ).view(torch.float16)
    shards = _partitions(full, nd, [(shift * q) % 8 for q in range(nd)])
    ref_shards = [f16np(x) for x in shards]
    ranges = [(0, psi_p), (0, 1), (psi_p - 1, 1), (S - 1, 2) if nd > 1 else (0, 2)]
    for _ in range(12):
        lo = int(rng.integers(0, psi_p))
        ranges.append((lo, int(rng.integers(1, psi_p - lo + 1))))
    for _ in range(6):
        lo = int(rng.integers(0, psi_p))
        ranges.append((lo, int(min(psi_p - lo, rng.integers(1, 24)))))
    st = status_word()
    for lo, n in ranges:
        for off in (0, 1, 3, 7):
            buf = torch.full((n + 16,), -1.0, dtype=torch.float16, device=DEV)
            out = buf[off:off + n]
            lz.zero_gather_params(pl, lo, n, shards, out, st)
            got = f16np(buf)
            want = oracle.gather_params(ref_shards, S, lo, lo + n)
            assert np.array_equal(got[off:off + n], want), (lo, n, off)
            assert (got[:off] == 0xbc00).all() and (got[off + n:] == 0xbc00).all()
    torch.cuda.synchronize()
    assert status_flags(st) == 0


def test_gather_gpt2_small_layers():
    """The GPT-2-small list at Nd = 8, cut into its 14 layers (embedding, 12 blocks, final
    LayerNorm): every layer gathered from the 8 partitions equals the full buffer's slice."""
    numels, nd = synth.gpt2_small_list(), 8
    pl = lz.zero_plan_create(numels, nd, 3, 0)
    psi, psi_p, S, _ = lz.zero_plan_info(pl)
    full = torch.randint(-(1 << 15), 1 << 15, (psi_p,), dtype=torch.int16,
                         device=DEV).view(torch.float16)
    shards = [full[q * S:(q + 1) * S].clone() for q in range(nd)]
    opl = oracle.plan(numels, nd, 0)
    layers = oracle.layer_ranges(opl, synth.gpt2_small_layers())
    assert len(layers) == 14 and layers[-1][1] == psi
    buf = torch.empty(max(hi - lo for lo, hi in layers), dtype=torch.float16, device=DEV)
    st = status_word()
    for lo, hi in layers:
        lz.zero_gather_params(pl, lo, hi - lo, shards, buf, st)
        assert torch.equal(buf[:hi - lo].view(torch.int16), full[lo:hi].view(torch.int16))
    assert status_flags(st) == 0


def _run_stage3_step(pl, layers, gb, grads, cur, nxt, shards, buf, t, st):
    """One stage-3 step through the C ABI; returns the gathered layers (forward, backward).
    gb: each layer's gradient bucket (its range; the last one extended over the padding)."""
    fwd, bwd = [None] * len(layers), [None] * len(layers)
    for l, (lo, hi) in enumerate(layers):
        lz.zero_gather_params(pl, lo, hi - lo, shards, buf, st)
        fwd[l] = f16np(buf[:hi - lo]).copy()
    for l in reversed(range(len(layers))):
        lo, hi = layers[l]
        lz.zero_gather_params(pl, lo, hi - lo, shards, buf, st)
        bwd[l] = f16np(buf[:hi - lo]).copy()
        _, ghi = gb[l]
        lz.zero_stage3_step_fused(pl, lo, ghi - lo, [g[lo:ghi] for g in grads],
                                  *[x[lo:ghi] for x in cur], *[x[lo:ghi] for x in nxt], shards,
                                  HP, t, st)
    lz.zero_stage3_step_commit(pl, *cur, *nxt, shards, st)
    return fwd, bwd


@pytest.mark.parametrize("nd", [1, 3, 8])
def test_stage3_steps_vs_oracle(nd):
    """Three attempts -- t = 1, an overflowing t = 2 (skipped), t = 2 -- with layers that
    straddle owners: every gathered layer, the state and the partitions equal zero3_step."""
    numels, split = [40000, 1234, 30000, 777, 5003], [1, 2, 2]   # psi = 77014
    pl = lz.zero_plan_create(numels, nd, 3, 0)
    psi, psi_p, S, _ = lz.zero_plan_info(pl)
    opl = oracle.plan(numels, nd, 0)
    layers = oracle.layer_ranges(opl, split)
    gb = oracle.grad_buckets(opl, layers)
    master, m, v = synth.state_warm(psi_p, seed=51)    # non-zero state in the padding too
    w_r, m_r, v_r = master.numpy(), m.numpy(), v.numpy()
    p16 = oracle.f2h(w_r)
    ref_shards = [p16[q * S:(q + 1) * S].copy() for q in range(nd)]
    shards = _partitions(torch.from_numpy(p16.view(np.float16)), nd,
                         [2 * (q % 2) for q in range(nd)])
    cur = [x.to(DEV) for x in (master, m, v)]
    nxt = [torch.empty_like(x) for x in cur]
    buf = torch.empty(max(hi - lo for lo, hi in layers), dtype=torch.float16, device=DEV)
    for i, (t, bad) in enumerate([(1, False), (2, True), (2, False)]):
        g_cpu = []
        for r in range(nd):
            g = torch.zeros(psi_p, dtype=torch.float16)
            g[:psi] = synth.grad_f16(psi, 1e-3, seed=52, rank=r, step=10 * i + t)
            g_cpu.append(g)
        if bad:
            g_cpu[nd - 1][layers[1][0] + 7] = float("-inf")
        grads = [g.to(DEV) for g in g_cpu]
        st = status_word()
        fwd, bwd = _run_stage3_step(pl, layers, gb, grads, cur, nxt, shards, buf, t, st)
        code, flags = lz.zero_step_status(st)
        ref = oracle.zero3_step(opl, layers, lambda l, r: g_cpu[r].numpy()[gb[l][0]:gb[l][1]],
                                w_r, m_r, v_r, ref_shards, ORC_HP, t)
        for l in range(len(layers)):
            assert np.array_equal(fwd[l], ref.gathered_fwd[l])
            assert np.array_equal(bwd[l], ref.gathered_bwd[l])
        assert ref.skipped == bad
        if bad:
            assert code == lz.ZERO_STEP_SKIPPED
        else:
            assert (code, flags) == (lz.ZERO_OK, 0)
        cur, nxt = nxt, cur
        check_f32(f"attempt {i} master", f32np(cur[0]), ref.master)
        check_f32(f"attempt {i} m", f32np(cur[1]), ref.m)
        check_f32(f"attempt {i} v", f32np(cur[2]), ref.v)
        for q in range(nd):
            check_f16(f"attempt {i} partition {q}", f16np(shards[q]), ref.param_shards[q])
        w_r, m_r, v_r, ref_shards = ref.master, ref.m, ref.v, ref.param_shards


def test_stage3_gpt2_small_sampled():
    """The GPT-2-small list at Nd = 8 in the launch configuration bench.py times (14 layers,
    gathered forward and backward, each layer's fused update into the partitions): two steps,
    the state and partitions compared with the oracle's element arithmetic on sampled
    elements (every tensor, layer and shard boundary), every gathered layer compared in full
    with the partitions it came from."""
    numels, nd = synth.gpt2_small_list(), 8
    pl = lz.zero_plan_create(numels, nd, 3, 0)
    psi, psi_p, S, _ = lz.zero_plan_info(pl)
    opl = oracle.plan(numels, nd, 0)
    layers = oracle.layer_ranges(opl, synth.gpt2_small_layers())
    rng = np.random.default_rng(61)
    bounds = [lo for lo, _ in layers] + [r * S for r in range(nd + 1)] + opl.tensor_off
    idx = np.unique(np.concatenate([rng.integers(0, psi_p, 100_000),
                                    np.array([b + d for b in bounds for d in (-2, -1, 0, 1)]),
                                    np.arange(psi_p - 8, psi_p)]))
    idx = idx[(idx >= 0) & (idx < psi_p)]
    idx_dev = torch.from_numpy(idx).to(DEV)
    cur = list(synth.state_small(psi_p, seed=62, device=DEV))
    nxt = [torch.empty_like(x) for x in cur]
    full = torch.empty(psi_p, dtype=torch.float16, device=DEV)
    full.copy_(cur[0])                       # fp16 of the master weights: the initial params
    shards = [full[q * S:(q + 1) * S].clone() for q in range(nd)]
    grads = [torch.zeros(psi_p, dtype=torch.float16, device=DEV) for _ in range(nd)]
    buf = torch.empty(max(hi - lo for lo, hi in layers), dtype=torch.float16, device=DEV)
    w_s, m_s, v_s = (cur[k][idx_dev].cpu().numpy() for k in range(3))
    for t in (1, 2):
        for r in range(nd):
            synth.grad_f16(psi, 1e-3, seed=63, rank=r, step=t, out=grads[r][:psi])
        gs = [g[idx_dev].cpu().numpy() for g in grads]
        before = torch.cat(shards)
        st = status_word()
        for l, (lo, hi) in enumerate(layers):
            lz.zero_gather_params(pl, lo, hi - lo, shards, buf, st)
            assert torch.equal(buf[:hi - lo].view(torch.int16), before[lo:hi].view(torch.int16))
        for l in reversed(range(len(layers))):
            lo, hi = layers[l]
            lz.zero_gather_params(pl, lo, hi - lo, shards, buf, st)
            assert torch.equal(buf[:hi - lo].view(torch.int16), before[lo:hi].view(torch.int16))
            ghi = psi_p if l == len(layers) - 1 else hi
            lz.zero_stage3_step_fused(pl, lo, ghi - lo, [g[lo:ghi] for g in grads],
                                      *[x[lo:ghi] for x in cur], *[x[lo:ghi] for x in nxt],
                                      shards, HP, t, st)
        lz.zero_stage3_step_commit(pl, *cur, *nxt, shards, st)
        assert lz.zero_step_status(st) == (lz.ZERO_OK, 0)
        cur, nxt = nxt, cur
        skipped, w_s, m_s, v_s, p_s = oracle.step(gs, w_s, m_s, v_s, ORC_HP, t)
        assert not skipped
        check_f32(f"step {t} master", cur[0][idx_dev].cpu().numpy(), w_s)
        check_f32(f"step {t} m", cur[1][idx_dev].cpu().numpy(), m_s)
        check_f32(f"step {t} v", cur[2][idx_dev].cpu().numpy(), v_s)
        check_f16(f"step {t} params", f16np(torch.cat(shards)[idx_dev]), p_s)


@pytest.mark.parametrize("nd", [3, 8])
def test_stage3_prefetch_schedule_vs_oracle(nd):
    """The two-stream schedule bench.py times: forward gathers, then backward gathers one layer
    ahead on a side stream while the main stream runs the previous layer's update (gather of
    layer l-1 beside the update of layer l; each update waits for its own layer's gather).
    Two steps; every gathered layer, the state and the partitions equal zero3_step."""
    numels, split = [40000, 1234, 30000, 777, 5003, 999, 4096], [1, 2, 2, 2]
    pl = lz.zero_plan_create(numels, nd, 3, 0)
    psi, psi_p, S, _ = lz.zero_plan_info(pl)
    opl = oracle.plan(numels, nd, 0)
    layers = oracle.layer_ranges(opl, split)
    gb = oracle.grad_buckets(opl, layers)
    L = len(layers)
    master, m, v = synth.state_warm(psi_p, seed=71)
    w_r, m_r, v_r = master.numpy(), m.numpy(), v.numpy()
    p16 = oracle.f2h(w_r)
    ref_shards = [p16[q * S:(q + 1) * S].copy() for q in range(nd)]
    shards = _partitions(torch.from_numpy(p16.view(np.float16)), nd)
    cur = [x.to(DEV) for x in (master, m, v)]
    nxt = [torch.empty_like(x) for x in cur]
    main, gs = torch.cuda.current_stream(), torch.cuda.Stream()
    ev = lambda: torch.cuda.Event()   # noqa: E731
    for t in (1, 2):
        g_cpu = []
        for r in range(nd):
            g = torch.zeros(psi_p, dtype=torch.float16)
            g[:psi] = synth.grad_f16(psi, 1e-3, seed=72, rank=r, step=t)
            g_cpu.append(g)
        grads = [g.to(DEV) for g in g_cpu]
        fwd = [torch.empty(hi - lo, dtype=torch.float16, device=DEV) for lo, hi in layers]
        bwd = [torch.empty(hi - lo, dtype=torch.float16, device=DEV) for lo, hi in layers]
        st = status_word()
        start = ev()
        start.record(main)
        gs.wait_event(start)
        g_done = [ev() for _ in range(L)]

        def gather(l, out):
            lo, hi = layers[l]
            lz.zero_gather_params(pl, lo, hi - lo, shards, out, st, gs)

        for l in range(L):
            gather(l, fwd[l])
        gather(L - 1, bwd[L - 1])
        g_done[L - 1].record(gs)
        lz.zero_overlap_begin(main)            # the updates chained, as in bench.py
        for l in range(L - 1, -1, -1):
            lo, _ = layers[l]
            _, ghi = gb[l]
            main.wait_event(g_done[l])
            lz.zero_stage3_step_fused(pl, lo, ghi - lo, [g[lo:ghi] for g in grads],
                                      *[x[lo:ghi] for x in cur], *[x[lo:ghi] for x in nxt],
                                      shards, HP, t, st, main)
            if l > 0:
                gather(l - 1, bwd[l - 1])      # beside layer l's update
                g_done[l - 1].record(gs)
        lz.zero_overlap_end(main)
        lz.zero_stage3_step_commit(pl, *cur, *nxt, shards, st, main)
        main.wait_stream(gs)
        assert lz.zero_step_status(st) == (lz.ZERO_OK, 0)
        ref = oracle.zero3_step(opl, layers, lambda l, r: g_cpu[r].numpy()[gb[l][0]:gb[l][1]],
                                w_r, m_r, v_r, ref_shards, ORC_HP, t)
        for l in range(L):
            assert np.array_equal(f16np(fwd[l]), ref.gathered_fwd[l])
            assert np.array_equal(f16np(bwd[l]), ref.gathered_bwd[l])
        cur, nxt = nxt, cur
        check_f32(f"step {t} master", f32np(cur[0]), ref.master)
        check_f32(f"step {t} v", f32np(cur[2]), ref.v)
        for q in range(nd):
            check_f16(f"step {t} partition {q}", f16np(shards[q]), ref.param_shards[q])
        w_r, m_r, v_r, ref_shards = ref.master, ref.m, ref.v, ref.param_shards
