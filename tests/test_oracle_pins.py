"""Pins for the CPU oracle: facts the pages, exact arithmetic or closed forms fix.

None of these re-types the oracle's formulas. Each pin is chosen so that a plausible slip in
the oracle (a dropped term, a wrong sign, a swapped beta, a wrong index or offset, a wrong
summation order or rounding rule) makes at least one of them fail; tests/test_oracle_mutants.py
plants such slips in a copy of the oracle and checks that they are caught.
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
from tests._exact import frac, round_f16, round_f32

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# ---------------------------------------------------------------------------------------------
# binary16 conversion
# ---------------------------------------------------------------------------------------------
def test_h2f_exhaustive_vs_numpy():
    h = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    ours = oracle.h2f(h)
    ref = h.view(np.float16).astype(np.float32)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan].view(np.uint32), ref[~nan].view(np.uint32))


def _f2h_chunk_check(lo, hi):
    bits = np.arange(lo, hi, dtype=np.uint64).astype(np.uint32)
    x = bits.view(np.float32)
    ours = oracle.f2h(x)
    with np.errstate(over="ignore", invalid="ignore"):
        ref = x.astype(np.float16).view(np.uint16)
    xnan = np.isnan(x)
    assert np.all(((ours[xnan] & 0x7c00) == 0x7c00) & ((ours[xnan] & 0x3ff) != 0))
    bad = np.nonzero((ours != ref) & ~xnan)[0]
    assert bad.size == 0, f"first mismatch at bits {hex(int(bits[bad[0]]))}"


def test_f2h_strided_vs_numpy():
    # every binary32 exponent and sign, dense in the low mantissa bits
    for lo in range(0, 1 << 32, 1 << 23):
        _f2h_chunk_check(lo, lo + 4096)
    # the whole binary16 range, around every representable value and midpoint
    for lo in range(0x33000000, 0x47800000 + 1, 1 << 24):
        _f2h_chunk_check(lo, lo + (1 << 24))


def _f2h_chunk_worker(lo_hi):
    _f2h_chunk_check(*lo_hi)
    return lo_hi


def test_f2h_exhaustive_vs_numpy():
    # all 2^32 binary32 bit patterns, spread over the host's cores (spawned workers, each
    # loading its own copy of the oracle)
    import concurrent.futures as cf
    import multiprocessing as mp
    step = 1 << 25
    chunks = [(lo, lo + step) for lo in range(0, 1 << 32, step)]
    workers = max(1, min(16, os.cpu_count() or 1))
    with cf.ProcessPoolExecutor(workers, mp_context=mp.get_context("spawn")) as ex:
        done = list(ex.map(_f2h_chunk_worker, chunks))
    assert len(done) == len(chunks)


def test_f2h_vs_exact_rounding_at_midpoints():
    # every binary16 midpoint between consecutive finite values, and a hair either side
    h = np.arange(0, 0x7bff, dtype=np.uint16)
    a = h.view(np.float16).astype(np.float64)
    b = (h + 1).view(np.float16).astype(np.float64)
    mids = ((a + b) / 2).astype(np.float32)   # exact: binary16 midpoints fit in binary32
    for x in list(mids[::97]) + [np.float32(65520.0), np.float32(65519.99)]:
        for y in (x, np.nextafter(x, np.float32(np.inf)), np.nextafter(x, np.float32(0))):
            want = round_f16(frac(y))
            got = oracle.f2h(np.array([y], np.float32))[0]
            assert got == np.array([want], np.float16).view(np.uint16)[0], (y, hex(got))


# ---------------------------------------------------------------------------------------------
# accounting: the pages' numbers and closed forms
# ---------------------------------------------------------------------------------------------
def test_memory_figures_of_the_7p5b_example():
    g = _golden("memory_7p5b_nd64.json")
    rep = oracle.state_bytes(g["psi"], g["nd"], g["K"])
    for stage, gb in g["gb_one_decimal"].items():
        assert round(rep[stage]["total"] / 1e9, 1) == gb, stage
    # the exact bytes behind the rounded figures
    assert rep["dp"]["total"] == 120_000_000_000
    assert rep["pos"]["total"] == 31_406_250_000
    assert rep["pos_g"]["total"] == 16_640_625_000
    assert rep["pos_g_p"]["total"] == 1_875_000_000


def test_bytes_per_param_and_reduction_limits():
    g = _golden("reduction_and_comm.json")
    bpp = g["bytes_per_param"]
    psi = 1_000_000
    rep = oracle.state_bytes(psi, 1, bpp["optimizer_K"])
    assert rep["dp"]["params"] == bpp["fp16_params"] * psi
    assert rep["dp"]["grads"] == bpp["fp16_grads"] * psi
    assert rep["dp"]["total"] == bpp["total"] * psi
    # with one process every stage holds everything
    for s in oracle.STAGES:
        assert rep[s]["total"] == 16 * psi
    # limits as Nd grows: 4x, 8x and linear
    nd = 1 << 20
    psi = nd * 1000
    rep = oracle.state_bytes(psi, nd, 12)
    dp = rep["dp"]["total"]
    assert abs(dp / rep["pos"]["total"] - g["max_reduction"]["pos"]) < 1e-4
    assert abs(dp / rep["pos_g"]["total"] - g["max_reduction"]["pos_g"]) < 1e-4
    assert dp / rep["pos_g_p"]["total"] == nd
    # monotone in Nd and never above the limit
    prev = [0, 0]
    for nd in (1, 2, 4, 8, 64, 1024):
        rep = oracle.state_bytes(nd * 1000, nd, 12)
        r1 = rep["dp"]["total"] / rep["pos"]["total"]
        r2 = rep["dp"]["total"] / rep["pos_g"]["total"]
        assert prev[0] <= r1 < 4 + 1e-12 and prev[1] <= r2 < 8 + 1e-12
        prev = [r1, r2]


@pytest.mark.parametrize("psi,nd", [(7_500_000_000, 64), (123_653_376, 8), (1000, 3), (7, 4)])
def test_partitioned_bytes_per_stage(psi, nd):
    rep = oracle.state_bytes(psi, nd, 12)
    shard = -(-psi // nd)
    # which quantity is split in which stage: Pos splits optimizer state, Pos+g adds the
    # gradients, Pos+g+p adds the parameters
    assert (rep["pos"]["params"], rep["pos"]["grads"], rep["pos"]["optim"]) == \
        (2 * psi, 2 * psi, 12 * shard)
    assert (rep["pos_g"]["params"], rep["pos_g"]["grads"], rep["pos_g"]["optim"]) == \
        (2 * psi, 2 * shard, 12 * shard)
    assert (rep["pos_g_p"]["params"], rep["pos_g_p"]["grads"], rep["pos_g_p"]["optim"]) == \
        (2 * shard, 2 * shard, 12 * shard)
    if psi % nd == 0:   # the pages' closed forms, exactly
        assert rep["pos"]["total"] * nd == 4 * psi * nd + 12 * psi
        assert rep["pos_g"]["total"] * nd == 2 * psi * nd + 14 * psi
        assert rep["pos_g_p"]["total"] * nd == 16 * psi


def test_communication_volume():
    g = _golden("reduction_and_comm.json")
    psi = 123_456_789
    rep = oracle.state_bytes(psi, 16, 12)
    for s, k in g["comm_elems_per_psi"].items():
        assert rep[s]["comm_elems"] == k * psi
    assert rep["pos_g_p"]["comm_elems"] * 2 == 3 * rep["dp"]["comm_elems"]   # 1.5x


# ---------------------------------------------------------------------------------------------
# plan
# ---------------------------------------------------------------------------------------------
def _gpt_closed_form(V, h, L, f):
    # token embedding + per layer (two LayerNorms, qkv, proj, two MLP matrices, biases) + ln_f
    return V * h + L * (4 * h * h + 2 * h * f + 9 * h + f) + 2 * h


def test_plan_gpt_shapes_closed_form():
    from zero_partitioned_optimizer_plan_b200 import synth
    pl = oracle.plan(synth.gpt2_small_list(), 8)
    assert len(pl.numels) == 1 + 12 * 12 + 2
    assert pl.psi == _gpt_closed_form(50257, 768, 12, 3072) == 123_653_376
    assert pl.psi_p == pl.psi and pl.shard == pl.psi // 8
    pl = oracle.plan(synth.gpt_1p3b_list(), 16, 50_000_000)
    assert len(pl.numels) == 1 + 24 * 12 + 2
    assert pl.psi == _gpt_closed_form(50257, 2048, 24, 8192) == 1_311_528_960
    assert len(pl.buckets) == math.ceil(pl.psi_p / 50_000_000) == 27
    assert pl.buckets[-1] == (0, pl.psi_p - 26 * 50_000_000)


@pytest.mark.parametrize("seed", range(20))
def test_plan_brute_force(seed):
    rng = np.random.default_rng(seed)
    n = int(rng.integers(0, 8))
    numels = [int(x) for x in rng.integers(0, 40, n)]
    nd = int(rng.integers(1, 9))
    bucket = int(rng.integers(0, 12))
    pl = oracle.plan(numels, nd, bucket)
    # element by element: which tensor and offset each flat index belongs to
    flat = [(t, j) for t, c in enumerate(numels) for j in range(c)]
    assert pl.psi == len(flat)
    for t, off in enumerate(pl.tensor_off):
        for j in range(numels[t]):
            assert flat[off + j] == (t, j)
    # padding to a multiple of nd, shards of equal length covering everything once
    assert pl.psi_p % nd == 0 and pl.psi <= pl.psi_p < pl.psi + nd
    assert pl.shard * nd == pl.psi_p
    owner = [i // pl.shard for i in range(pl.psi_p)] if pl.shard else []
    for r in range(nd):
        assert owner.count(r) == pl.shard
    # buckets: produced from the end of the flat list backwards, disjoint, covering all
    covered = []
    prev_lo = pl.psi_p
    B = bucket or pl.psi_p
    for k, (lo, ln) in enumerate(pl.buckets):
        assert lo + ln == prev_lo and ln > 0 and ln <= B
        assert lo == max(0, pl.psi_p - (k + 1) * B)
        covered.extend(range(lo, lo + ln))
        prev_lo = lo
        o_lo, o_hi = pl.owners(k)
        assert o_lo == owner[lo] and o_hi == owner[lo + ln - 1]
    assert prev_lo == 0 if pl.psi_p else pl.buckets == []
    assert sorted(covered) == list(range(pl.psi_p))


def test_three_gpu_picture():
    g = _golden("three_gpu_picture.json")
    nd = g["nd"]
    layer = 5                        # three layers of five parameters, one bucket per layer
    pl = oracle.plan([layer] * 3, nd, layer)
    assert pl.shard == layer
    for name, r in g["owner_of_shard"].items():
        lo = g["shard_names"].index(name) * pl.shard
        assert lo // pl.shard == r
    produced = [g["layers_forward_order"][lo // layer] for lo, _ in pl.buckets]
    assert produced == g["bucket_production_order"]


# ---------------------------------------------------------------------------------------------
# reduced gradient
# ---------------------------------------------------------------------------------------------
def test_sum_order_golden():
    g = _golden("sum_order.json")
    for case in g["cases"]:
        ranks = [np.array([int(b, 16)], np.uint16) for b in case["rank_values_f16_bits"]]
        red = oracle.reduce_mean(ranks)
        if case.get("expected_mean_is_nan"):
            assert np.isnan(red[0]), case["name"]
        else:
            assert red.view(np.uint32)[0] == int(case["expected_mean_f32_bits"], 16), case["name"]


@pytest.mark.parametrize("nd", [1, 2, 3, 4, 7, 8, 16, 64])
def test_exact_sums_closed_form(nd):
    # multiples of 2^-10 below 2 in magnitude are exact in fp16 and every partial sum is exact
    # in binary32, so the rank-ordered sum is the exact sum; the mean is the exact quotient
    # rounded once (exact for power-of-two Nd)
    rng = np.random.default_rng(nd)
    n = 257
    k = rng.integers(-2047, 2048, size=(nd, n))
    ranks = [(k[r] * 2.0 ** -10).astype(np.float16) for r in range(nd)]
    red = oracle.reduce_mean(ranks)
    for i in range(n):
        exact = Fraction(int(k[:, i].sum()), 1024 * nd)
        assert red[i] == round_f32(exact), (i, red[i], exact)


@pytest.mark.parametrize("seed", range(6))
def test_reduce_brute_force_exact_rationals(seed):
    # generic fp16 inputs: evaluate the rank-ordered binary32 sum with exact rationals,
    # rounding after every addition, and the single division at the end
    rng = np.random.default_rng(100 + seed)
    nd = int(rng.integers(1, 20))
    n = 64
    ranks = [(rng.standard_normal(n) * 10.0 ** rng.uniform(-6, 3, n)).astype(np.float16)
             for _ in range(nd)]
    red = oracle.reduce_mean(ranks)
    for i in range(n):
        s = Fraction(0)
        for r in range(nd):
            s = frac(round_f32(s + frac(ranks[r][i])))
        assert red[i] == round_f32(s / nd)


# ---------------------------------------------------------------------------------------------
# Adam
# ---------------------------------------------------------------------------------------------
HP = oracle.AdamHP()
U = 2.0 ** -24


def _ulp(x):
    return np.spacing(np.abs(np.float32(x))).astype(np.float64)


def test_adam_first_step_from_zero_state():
    # t = 1, m = v = 0: the bias-corrected moments are g and g^2, so the update is
    # lr * g / (|g| + eps) exactly (Kingma & Ba), whatever beta1 and beta2 are
    rng = np.random.default_rng(1)
    n = 4096
    g16 = (rng.standard_normal(n) * 1e-2).astype(np.float16)
    master = (rng.standard_normal(n) * 0.02).astype(np.float32)
    z = np.zeros(n, np.float32)
    for hp in (HP, oracle.AdamHP(lr=3e-4, beta1=0.8, beta2=0.95, eps=1e-6, loss_scale=1.0)):
        skipped, w, m, v, p16 = oracle.step([g16], master, z, z, hp, 1)
        assert not skipped
        g = g16.astype(np.float64) / hp.loss_scale        # Nd = 1: the reduced grad is g16
        upd = hp.lr * g / (np.abs(g) + hp.eps)
        ref = master.astype(np.float64) - upd
        bound = 0.5 * _ulp(ref) + 16 * U * np.abs(upd) + 1e-30
        assert np.all(np.abs(w.astype(np.float64) - ref) <= bound)
        assert np.all(np.abs(m - (1 - hp.beta1) * g) <= 4 * U * np.abs((1 - hp.beta1) * g))
        assert np.all(np.abs(v - (1 - hp.beta2) * g * g) <= 4 * U * (1 - hp.beta2) * g * g)
        assert np.array_equal(p16, oracle.f2h(w))


def test_adam_constant_gradient_many_steps():
    # constant g from zero state: m_t = (1 - beta1^t) g and v_t = (1 - beta2^t) g^2 exactly,
    # so every bias-corrected step moves by lr * g/(|g| + eps); a wrong bias correction
    # (missing, off by one step, the wrong beta or no square root) breaks this at some t
    rng = np.random.default_rng(2)
    n = 2048
    g16 = (rng.standard_normal(n) * 1e-1).astype(np.float16)
    master0 = (rng.standard_normal(n)).astype(np.float32)
    w, m, v = master0, np.zeros(n, np.float32), np.zeros(n, np.float32)
    g = g16.astype(np.float64) / HP.loss_scale
    T = 12
    for t in range(1, T + 1):
        skipped, w, m, v, _ = oracle.step([g16, g16], w, m, v, HP, t)
        assert not skipped
        mt = (1 - HP.beta1 ** t) * g
        vt = (1 - HP.beta2 ** t) * g * g
        assert np.all(np.abs(m - mt) <= 6 * t * U * np.abs(mt))
        assert np.all(np.abs(v - vt) <= 6 * t * U * vt)
    upd = HP.lr * g / (np.abs(g) + HP.eps)
    ref = master0.astype(np.float64) - T * upd
    # each step rounds once to half an ulp of its result; the path may cross a binade, so
    # take the larger ulp of its two ends
    bound = T * (0.5 * np.maximum(_ulp(ref), _ulp(master0)) + 64 * U * np.abs(upd))
    assert np.all(np.abs(w.astype(np.float64) - ref) <= bound)


@pytest.mark.parametrize("t", [1, 2, 5, 100, 10000])
def test_adam_vs_textbook_fp64(t):
    # warm state, mixed signs: Kingma & Ba's algorithm in float64 with the exact constants;
    # the oracle's binary32 result must sit within the forward rounding-error bound
    rng = np.random.default_rng(t)
    n = 8192
    hp = HP
    g16 = (rng.standard_normal(n) * 1e-3).astype(np.float16)
    master = rng.uniform(-0.05, 0.05, n).astype(np.float32)
    m0 = (rng.standard_normal(n) * 1e-4 / hp.loss_scale).astype(np.float32)
    v0 = (np.abs(rng.standard_normal(n)) * 1e-6 / hp.loss_scale ** 2).astype(np.float32)
    skipped, w, m, v, p16 = oracle.step([g16], master, m0, v0, hp, t)
    assert not skipped
    g = g16.astype(np.float64) / hp.loss_scale
    M0, V0, W0 = (a.astype(np.float64) for a in (m0, v0, master))
    m_ref = hp.beta1 * M0 + (1 - hp.beta1) * g
    v_ref = hp.beta2 * V0 + (1 - hp.beta2) * g * g
    mhat = m_ref / (1 - hp.beta1 ** t)
    vhat = v_ref / (1 - hp.beta2 ** t)
    upd = hp.lr * mhat / (np.sqrt(vhat) + hp.eps)
    w_ref = W0 - upd
    em = 4 * U * (np.abs(hp.beta1 * M0) + np.abs((1 - hp.beta1) * g))
    ev = 4 * U * (hp.beta2 * V0 + (1 - hp.beta2) * g * g)
    assert np.all(np.abs(m - m_ref) <= em)
    assert np.all(np.abs(v - v_ref) <= ev)
    denom = np.sqrt(vhat) + hp.eps
    e_upd = hp.lr / (1 - hp.beta1 ** t) * em / denom + 16 * U * np.abs(upd) \
        + np.abs(upd) * (ev / v_ref)
    bound = 0.5 * _ulp(w_ref) + 2 * e_upd
    assert np.all(np.abs(w.astype(np.float64) - w_ref) <= bound)
    assert np.array_equal(p16, oracle.f2h(w))


def test_zero_gradient_changes_nothing():
    # the zero-padded tail: g = m = v = 0 leaves the master where it is
    n = 1000
    master = np.linspace(-1, 1, n, dtype=np.float32)
    z = np.zeros(n, np.float32)
    zero16 = np.zeros(n, np.float16)
    for t in (1, 7):
        skipped, w, m, v, p16 = oracle.step([zero16] * 3, master, z, z, HP, t)
        assert not skipped
        assert np.array_equal(w, master) and not m.any() and not v.any()
        assert np.array_equal(p16, master.astype(np.float16).view(np.uint16))


# ---------------------------------------------------------------------------------------------
# overflow skip
# ---------------------------------------------------------------------------------------------
@pytest.mark.parametrize("bad", [0x7c00, 0xfc00, 0x7e00])
def test_overflow_skips_whole_step(bad):
    rng = np.random.default_rng(3)
    n, nd = 300, 5
    ranks = [(rng.standard_normal(n) * 1e-2).astype(np.float16) for _ in range(nd)]
    ranks[3].view(np.uint16)[217] = bad
    master = rng.standard_normal(n).astype(np.float32)
    m = rng.standard_normal(n).astype(np.float32) * 1e-3
    v = np.abs(rng.standard_normal(n)).astype(np.float32) * 1e-6
    skipped, w, mm, vv, p16 = oracle.step(ranks, master, m, v, HP, 4)
    assert skipped and p16 is None
    assert np.array_equal(w, master) and np.array_equal(mm, m) and np.array_equal(vv, v)


def test_largest_finite_gradients_do_not_skip():
    n, nd = 16, 64
    ranks = [np.full(n, 65504.0, np.float16) for _ in range(nd)]
    skipped, *_ = oracle.step(ranks, np.zeros(n, np.float32), np.zeros(n, np.float32),
                              np.zeros(n, np.float32), HP, 1)
    assert not skipped


# ---------------------------------------------------------------------------------------------
# ZeRO changes where state lives, not the update: every stage equals plain DP, bitwise
# ---------------------------------------------------------------------------------------------
def _random_model(rng, numels, nd, bucket):
    pl = oracle.plan(numels, nd, bucket)
    grads = []
    for _ in range(nd):
        g = np.zeros(pl.psi_p, np.float16)
        g[:pl.psi] = (rng.standard_normal(pl.psi) * 1e-2).astype(np.float16)
        grads.append(g)
    master = np.zeros(pl.psi_p, np.float32)
    master[:pl.psi] = rng.standard_normal(pl.psi) * 0.02
    m = np.zeros(pl.psi_p, np.float32)
    m[:pl.psi] = rng.standard_normal(pl.psi) * 1e-7
    v = np.zeros(pl.psi_p, np.float32)
    v[:pl.psi] = np.abs(rng.standard_normal(pl.psi)) * 1e-12
    p16 = oracle.f2h(master)
    return pl, grads, master, m, v, p16


@pytest.mark.parametrize("nd", [1, 2, 3, 4, 7, 8])
@pytest.mark.parametrize("numels,bucket", [([300, 250, 250, 249], 0), ([7], 3),
                                            ([50, 1, 64, 13], 17), ([1000], 999)])
def test_zero_stages_equal_plain_dp(nd, numels, bucket):
    rng = np.random.default_rng(nd * 1000 + sum(numels))
    pl, grads, master, m, v, p16 = _random_model(rng, numels, nd, bucket)
    for t in (1, 2):
        dp = oracle.dp_step(grads, master, m, v, p16, HP, t)
        z1 = oracle.zero1_step(pl, grads, master, m, v, p16, HP, t)

        def bucket_grad(k, r):
            lo, ln = pl.buckets[k]
            return grads[r][lo:lo + ln]
        z2 = oracle.zero2_step(pl, bucket_grad, master, m, v, p16, HP, t)
        for z in (z1, z2):
            assert z.skipped == dp.skipped is False
            for a, b in ((z.master, dp.master), (z.m, dp.m), (z.v, dp.v), (z.reduced, dp.reduced)):
                assert np.array_equal(a.view(np.uint32), b.view(np.uint32))
            assert np.array_equal(z.params16, dp.params16)
        # the zero-padded tail stays zero
        assert not dp.master[pl.psi:].any() and not dp.m[pl.psi:].any()
        master, m, v, p16 = dp.master, dp.m, dp.v, dp.params16


def test_zero_stages_skip_together():
    rng = np.random.default_rng(9)
    pl, grads, master, m, v, p16 = _random_model(rng, [40, 40, 21], 4, 16)
    grads[2][77] = np.float16(np.inf)
    dp = oracle.dp_step(grads, master, m, v, p16, HP, 1)
    z1 = oracle.zero1_step(pl, grads, master, m, v, p16, HP, 1)
    z2 = oracle.zero2_step(pl, lambda k, r: grads[r][pl.buckets[k][0]:sum(pl.buckets[k])],
                           master, m, v, p16, HP, 1)
    for z in (dp, z1, z2):
        assert z.skipped
        assert np.array_equal(z.master, master) and np.array_equal(z.params16, p16)


# ---------------------------------------------------------------------------------------------
# stage 3 (Pos+g+p): parameters partitioned too, gathered just in time per layer
# ("Como funciona": 16 psi/Nd and 3 psi of communication; "ZeRO" (lastdictionary), main
# definition: layers gathered just in time and discarded, about 50 % more communication)
# ---------------------------------------------------------------------------------------------
def _split_shards(full16, nd):
    """The owners' fp16 partitions of a flat padded buffer (numpy's split, not the oracle's
    gather, so that the gather is checked against an independent partitioning)."""
    return [x.copy() for x in np.split(full16, nd)]


@pytest.mark.parametrize("nd", [1, 2, 3, 4, 7, 8])
@pytest.mark.parametrize("numels,layer_tensors", [([300, 250, 250, 249], [1, 2, 1]),
                                                   ([7], [1]),
                                                   ([50, 1, 64, 13], [2, 1, 1]),
                                                   ([1000, 3, 999, 5], [1, 3])])
def test_stage3_equals_plain_dp(nd, numels, layer_tensors):
    """ZeRO changes where state lives, not the update ("ZeRO" (lastdictionary), "Usage note"):
    two stage-3 steps give plain DP's master, m, v, reduced gradients and fp16 parameters bit
    for bit, the parameters held as Nd partitions."""
    rng = np.random.default_rng(nd * 7919 + sum(numels))
    pl, grads, master, m, v, p16 = _random_model(rng, numels, nd, 0)
    layers = oracle.layer_ranges(pl, layer_tensors)
    gb = oracle.grad_buckets(pl, layers)
    shards = _split_shards(p16, nd)
    for t in (1, 2):
        dp = oracle.dp_step(grads, master, m, v, p16, HP, t)
        z3 = oracle.zero3_step(pl, layers, lambda l, r: grads[r][gb[l][0]:gb[l][1]],
                               master, m, v, shards, HP, t)
        assert z3.skipped == dp.skipped is False
        for a, b in ((z3.master, dp.master), (z3.m, dp.m), (z3.v, dp.v),
                     (z3.reduced, dp.reduced)):
            assert np.array_equal(a.view(np.uint32), b.view(np.uint32))
        assert np.array_equal(np.concatenate(z3.param_shards), dp.params16)
        master, m, v, p16, shards = dp.master, dp.m, dp.v, dp.params16, z3.param_shards


@pytest.mark.parametrize("nd", [1, 3, 4, 8])
def test_stage3_gathers_are_the_layer_parameters(nd):
    """Every gathered layer, forward and backward, is exactly the layer's slice of the full
    fp16 buffer the partitions were cut from -- including layers that straddle owners, a layer
    smaller than a shard and one larger than several shards; values that encode their own flat
    index make any misplaced element visible."""
    numels = [5, 40, 1, 17, 3, 90, 2]
    pl = oracle.plan(numels, nd, 0)
    full = np.arange(1, pl.psi_p + 1, dtype=np.uint16)          # element i holds i + 1
    full[pl.psi:] = 0
    shards = _split_shards(full, nd)
    for split in ([1] * 7, [2, 2, 3], [7], [3, 1, 3]):
        layers = oracle.layer_ranges(pl, split)
        assert layers[0][0] == 0 and layers[-1][1] == pl.psi
        z = np.zeros(pl.psi_p, np.float32)
        gb = oracle.grad_buckets(pl, layers)
        res = oracle.zero3_step(pl, layers,
                                lambda l, r: np.zeros(gb[l][1] - gb[l][0], np.float16),
                                z, z, z, shards, HP, 1)
        for l, (lo, hi) in enumerate(layers):
            want = np.arange(lo + 1, hi + 1, dtype=np.uint16)
            assert np.array_equal(res.gathered_fwd[l], want)
            assert np.array_equal(res.gathered_bwd[l], want)


@pytest.mark.parametrize("nd,numels", [(4, [300, 250, 250, 249]), (3, [50, 1, 64, 13]),
                                       (8, [1000, 3, 999, 5])])
def test_stage3_moves_three_psi(nd, numels):
    """The step's collectives move 3 psi elements -- the forward and backward parameter
    all-gathers and the gradient reduce-scatter -- which is zero_state_bytes' closed form and
    1.5 times the 2 psi of stages 0-2 ("Como funciona"; "ZeRO" (lastdictionary): stage 3 adds
    about 50 %)."""
    rng = np.random.default_rng(nd)
    pl, grads, master, m, v, p16 = _random_model(rng, numels, nd, 0)
    layers = oracle.layer_ranges(pl, [1] * len(numels))
    gb = oracle.grad_buckets(pl, layers)
    res = oracle.zero3_step(pl, layers, lambda l, r: grads[r][gb[l][0]:gb[l][1]],
                            master, m, v, _split_shards(p16, nd), HP, 1)
    acct = oracle.state_bytes(pl.psi, nd)
    assert res.comm_elems == 3 * pl.psi == acct["pos_g_p"]["comm_elems"]
    assert 2 * res.comm_elems == 3 * acct["pos_g"]["comm_elems"] == 3 * acct["dp"]["comm_elems"]


@pytest.mark.parametrize("nd", [3, 4, 7])
def test_stage3_padding_is_updated_like_plain_dp(nd):
    """The zero padding at the end of the flat list rides with the first backward bucket, so
    it is updated exactly as plain DP updates it, even from non-zero state."""
    rng = np.random.default_rng(100 + nd)
    pl, grads, master, m, v, p16 = _random_model(rng, [50, 1, 64, 15], nd, 0)
    assert pl.psi_p > pl.psi
    master[pl.psi:] = 0.5
    m[pl.psi:] = 1e-3
    v[pl.psi:] = 1e-6
    layers = oracle.layer_ranges(pl, [2, 2])
    gb = oracle.grad_buckets(pl, layers)
    assert gb[-1] == (layers[-1][0], pl.psi_p) and gb[:-1] == layers[:-1]
    z3 = oracle.zero3_step(pl, layers, lambda l, r: grads[r][gb[l][0]:gb[l][1]], master, m, v,
                           _split_shards(oracle.f2h(master), nd), HP, 1)
    dp = oracle.dp_step(grads, master, m, v, oracle.f2h(master), HP, 1)
    assert np.array_equal(z3.master.view(np.uint32), dp.master.view(np.uint32))
    assert np.array_equal(np.concatenate(z3.param_shards), dp.params16)
    assert not np.array_equal(dp.master[pl.psi:], master[pl.psi:])   # it did move


def test_stage3_skips_together():
    """An inf in one rank's gradient of one layer skips the whole stage-3 step: state and every
    parameter partition unchanged, like plain DP."""
    rng = np.random.default_rng(19)
    pl, grads, master, m, v, p16 = _random_model(rng, [40, 40, 21], 4, 0)
    grads[1][45] = np.float16(np.inf)
    layers = oracle.layer_ranges(pl, [1, 1, 1])
    gb = oracle.grad_buckets(pl, layers)
    shards = _split_shards(p16, 4)
    z3 = oracle.zero3_step(pl, layers, lambda l, r: grads[r][gb[l][0]:gb[l][1]],
                           master, m, v, shards, HP, 1)
    dp = oracle.dp_step(grads, master, m, v, p16, HP, 1)
    assert z3.skipped and dp.skipped
    assert np.array_equal(z3.master, master) and np.array_equal(z3.v, v)
    assert np.array_equal(np.concatenate(z3.param_shards), p16)


def test_ulp_metric():
    a = np.array([1.0, -0.0, np.nan, 1.0], np.float32)
    b = np.array([np.nextafter(np.float32(1), np.float32(2)), 0.0, np.nan, np.nan], np.float32)
    assert list(oracle.ulp_diff_f32(a, b)) == [1, 0, 0, 1 << 32]
    h = np.array([0x3c00, 0x8000, 0x0001], np.uint16)
    k = np.array([0x3c01, 0x0000, 0x8001], np.uint16)
    assert list(oracle.ulp_diff_f16(h, k)) == [1, 0, 2]


def test_dynamic_scale_golden_sequence():
    g = _golden("dynamic_scale_sequence.json")
    sc = oracle.Scaler(scale=g["init_scale"], growth_factor=g["growth_factor"],
                       backoff_factor=g["backoff_factor"], growth_interval=g["growth_interval"])
    for ovf, s_before, t in zip(g["overflow"], g["scale_before_step"], g["adam_t_of_step"]):
        assert sc.scale == s_before
        if t is not None:
            assert sc.next_step == t
        sc.update(ovf)
    assert (sc.scale, sc.good_steps, sc.next_step, sc.skipped_steps) == tuple(g["final"].values())


def test_scaled_step_unscales_by_the_current_scale():
    # the same gradients at scale 2S against halved inputs at scale S give the same update:
    # the update only sees g = red / scale
    rng = np.random.default_rng(5)
    n = 512
    g16 = (rng.standard_normal(n) * 1e-2).astype(np.float16)
    half = (g16.astype(np.float32) / 2).astype(np.float16)
    ok = g16.astype(np.float32) / 2 == half.astype(np.float32)   # exactly halved elements
    master = rng.standard_normal(n).astype(np.float32)
    z = np.zeros(n, np.float32)
    a = oracle.scaled_step([g16], master, z, z, HP, oracle.Scaler(scale=2048.0))
    b = oracle.scaled_step([half], master, z, z, HP, oracle.Scaler(scale=1024.0))
    assert np.array_equal(a[1][ok].view(np.uint32), b[1][ok].view(np.uint32))
    # a skipped step leaves t where it was and halves the scale
    bad = g16.copy()
    bad[7] = np.float16(np.inf)
    sc = oracle.Scaler(scale=1024.0)
    skipped, *_ = oracle.scaled_step([bad], master, z, z, HP, sc)
    assert skipped and sc.next_step == 1 and sc.scale == 512.0 and sc.skipped_steps == 1


# ---------------------------------------------------------------------------------------------
# compressed payload: int8 + one fp32 scale per block of 128
# ---------------------------------------------------------------------------------------------
def _rint_half_even(fr: Fraction) -> int:
    n = fr.numerator // fr.denominator
    rem = fr - n
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and n % 2 == 1):
        n += 1
    return n


@pytest.mark.parametrize("seed", range(4))
def test_quant_q8_brute_force(seed):
    # every q from the definition with exact rationals: scale = fl(amax / 127),
    # q = half-even integer of fl(x / scale), clamped; blocks of 128 from element 0
    rng = np.random.default_rng(200 + seed)
    n = 128 * 3 + 37
    g = (rng.standard_normal(n) * 10.0 ** rng.uniform(-4, 1)).astype(np.float16)
    g[128:256] = 0                                    # a zero block
    q, sc = oracle.quant_q8(g)
    assert sc.size == 4
    for b in range(4):
        blk = g[128 * b:128 * (b + 1)].astype(np.float64)
        amax = Fraction(float(np.max(np.abs(blk))))
        scale = round_f32(amax / 127)
        assert sc[b] == scale
        for j, x in enumerate(blk):
            i = 128 * b + j
            if scale == 0:
                assert q[i] == 0
                continue
            k = _rint_half_even(frac(round_f32(Fraction(float(x)) / frac(scale))))
            assert q[i] == max(-127, min(127, k)), (i, x, q[i], k)


def test_quant_q8_grid_values_round_trip_exactly():
    # values k * 2^-7 with max |k| = 127: scale is exactly 2^-7 and every q is exactly k
    rng = np.random.default_rng(7)
    k = rng.integers(-127, 128, size=256)
    k[0], k[128] = 127, -127
    x = (k * 2.0 ** -7).astype(np.float16)
    q, sc = oracle.quant_q8(x)
    assert np.all(sc == np.float32(2.0 ** -7)) and np.array_equal(q.astype(np.int64), k)


def test_quant_q8_ties_go_to_even():
    x = np.zeros(128, np.float16)
    x[0] = 127 * 2.0 ** -7                        # scale 2^-7
    x[1], x[2], x[3], x[4] = 2.5 * 2.0 ** -7, 3.5 * 2.0 ** -7, -2.5 * 2.0 ** -7, 0.5 * 2.0 ** -7
    q, _ = oracle.quant_q8(x)
    assert list(q[:5]) == [127, 2, 4, -2, 0]


def test_quant_q8_poisoned_block_skips_the_step():
    rng = np.random.default_rng(8)
    g = [(rng.standard_normal(300) * 1e-2).astype(np.float16) for _ in range(3)]
    g[1][200] = np.float16(np.inf)
    qs, scs = zip(*[oracle.quant_q8(x) for x in g])
    assert np.isnan(scs[1][1]) and not np.isnan(scs[1][0]) and not scs[1][1:2].size == 0
    assert not qs[1][128:256].any()
    master = rng.standard_normal(300).astype(np.float32)
    z = np.zeros(300, np.float32)
    skipped, w, *_ = oracle.step_q8(qs, scs, master, z, z, HP, 1)
    assert skipped and np.array_equal(w, master)


@pytest.mark.parametrize("nd", [1, 3, 8])
def test_reduce_mean_q8_brute_force(nd):
    # per rank in order: the exact product q*scale added to the running sum, rounded once
    # (a fused multiply-add); then one division
    rng = np.random.default_rng(300 + nd)
    n = 128 * 2 + 5
    g = [(rng.standard_normal(n) * 1e-2).astype(np.float16) for _ in range(nd)]
    qs, scs = zip(*[oracle.quant_q8(x) for x in g])
    red = oracle.reduce_mean_q8(qs, scs)
    for i in range(n):
        s = Fraction(0)
        for r in range(nd):
            s = frac(round_f32(s + Fraction(int(qs[r][i])) * frac(scs[r][i // 128])))
        assert red[i] == round_f32(s / nd)
    # and the payload is close to the fp16 gradients it stands for (half a step per element)
    for r in range(nd):
        deq = qs[r].astype(np.float64) * np.repeat(scs[r].astype(np.float64), 128)[:n]
        err = np.abs(deq - g[r].astype(np.float64))
        assert np.all(err <= 0.5 * np.repeat(scs[r], 128)[:n] * (1 + 2.0 ** -20) + 1e-30)
