"""C-ABI checks that need no GPU: the library loads, exports every symbol include/*.h
declares, its planner and accounting agree bit-exactly with the oracle's independent ones, and
host-detectable argument errors return their status codes without launching anything."""
import glob
import os
import re
import subprocess

import numpy as np
import pytest

import oracle
from zero_partitioned_optimizer_plan_b200 import build as zbuild
from zero_partitioned_optimizer_plan_b200 import synth

zbuild.build()
from zero_partitioned_optimizer_plan_b200 import libzero as lz  # noqa: E402

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        src = open(h).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        for m in re.finditer(r"^[A-Za-z_][\w\s\*]*?\b(zero_\w+)\s*\(", src, flags=re.M):
            names.add(m.group(1))
    return names


def test_header_declares_the_entry_points():
    names = _declared_functions()
    for must in ("zero_plan_create", "zero_state_bytes", "zero_reduce_scatter_bucket",
                 "zero_adam_shard", "zero_step_fused"):
        assert must in names
    assert names == set(lz.SYMBOLS)


def test_library_exports_every_declared_symbol():
    out = subprocess.run(["nm", "-D", "--defined-only", lz.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    missing = _declared_functions() - exported
    assert not missing, missing
    for name in _declared_functions():
        assert hasattr(lz._lib, name)


def test_library_is_built_for_sm100a():
    assert "arch=compute_100a,code=sm_100a" in " ".join(zbuild.NVCC_FLAGS)
    log = open(os.path.join(zbuild.BUILD, "ptxas.log")).read()
    assert "for 'sm_100a'" in log and "spill stores" in log
    # no kernel spills registers to local memory
    assert all(" 0 bytes spill stores" in ln for ln in log.splitlines() if "spill stores" in ln)


# ---------------------------------------------------------------------------------------------
# planner and accounting: two independent implementations agree exactly
# ---------------------------------------------------------------------------------------------
def _compare_plans(numels, nd, bucket):
    ref = oracle.plan(numels, nd, bucket)
    pl = lz.zero_plan_create(numels, nd, 2, bucket)
    psi, psi_p, shard, nb = lz.zero_plan_info(pl)
    assert (psi, psi_p, shard, nb) == (ref.psi, ref.psi_p, ref.shard, len(ref.buckets))
    assert lz.zero_plan_tensor_offsets(pl) == ref.tensor_off
    for k, (lo, ln) in enumerate(ref.buckets):
        assert lz.zero_plan_bucket(pl, k) == (lo, ln, *ref.owners(k))
    with pytest.raises(lz.ZeroError):
        lz.zero_plan_bucket(pl, nb)


@pytest.mark.parametrize("seed", range(40))
def test_plan_matches_oracle_random(seed):
    rng = np.random.default_rng(seed)
    n = int(rng.integers(1, 12))
    numels = [int(x) for x in rng.integers(0, 10 ** int(rng.integers(1, 7)), n)]
    if sum(numels) == 0:
        numels[0] = 1
    nd = int(rng.integers(1, 65))
    total = sum(numels)
    # at most ~300 buckets: the oracle walks them one by one
    small = max(1, -(-total // 300))
    bucket = int(rng.choice([0, small, small + 7, 8 * small, int(rng.integers(small, total + 10))]))
    _compare_plans(numels, nd, bucket)


def test_plan_matches_oracle_workloads():
    _compare_plans(synth.TINY_LIST, 4, 0)
    _compare_plans(synth.gpt2_small_list(), 8, 0)
    _compare_plans(synth.gpt_1p3b_list(), 16, 50_000_000)
    _compare_plans([7_500_000_000], 64, 0)
    _compare_plans([1 << 29], 64, 1 << 19)
    _compare_plans([7], 4, 3)


@pytest.mark.parametrize("psi,nd,K", [(7_500_000_000, 64, 12), (123_653_376, 8, 12),
                                      (1_311_528_960, 16, 12), (1, 64, 12), (7, 4, 12),
                                      (1000, 3, 8), (0, 5, 12)])
def test_state_bytes_matches_oracle(psi, nd, K):
    a = lz.zero_state_bytes(psi, nd, K)
    b = oracle.state_bytes(psi, nd, K)
    for s in lz.STAGES:
        for key in ("params", "grads", "optim", "total", "comm_elems"):
            assert a[s][key] == b[s][key], (s, key)
        assert a[s]["comm_bytes_fp16"] == 2 * b[s]["comm_elems"]


def test_plan_rejects_bad_arguments():
    for args in [([], 4, 1, 0), ([5], 0, 1, 0), ([5], 65, 1, 0), ([5], 4, 4, 0), ([5], 4, 0, 0),
                 ([0, 0], 2, 1, 0)]:
        with pytest.raises(lz.ZeroError) as e:
            lz.zero_plan_create(*args)
        assert e.value.code == lz.ZERO_EINVAL
    with pytest.raises(lz.ZeroError):
        lz.zero_state_bytes(10, 0)


# ---------------------------------------------------------------------------------------------
# data-path argument errors (all caught on the host before any CUDA call)
# ---------------------------------------------------------------------------------------------
HP = lz.AdamHP()
A = 1 << 32          # fake, 256-byte aligned device addresses far apart
MB = 1 << 24


def _fused(n=1000, nd=2, grads=None, ins=None, outs=None, p=None, hp=HP, step=1, st=None):
    grads = grads if grads is not None else [A + i * MB for i in range(nd)]
    ins = ins or [A + 100 * MB, A + 101 * MB, A + 102 * MB]
    outs = outs or [A + 110 * MB, A + 111 * MB, A + 112 * MB]
    p = p if p is not None else A + 120 * MB
    st = st if st is not None else A + 130 * MB
    lz.zero_step_fused(n, nd, grads, *ins, *outs, p, hp, step, st, 0)


@pytest.mark.parametrize("kw,code", [
    (dict(nd=0), lz.ZERO_EINVAL),
    (dict(nd=65), lz.ZERO_EINVAL),
    (dict(step=0), lz.ZERO_EINVAL),
    (dict(st=0), lz.ZERO_EINVAL),
    (dict(hp=lz.AdamHP(beta1=1.0)), lz.ZERO_EINVAL),
    (dict(hp=lz.AdamHP(loss_scale=0.0)), lz.ZERO_EINVAL),
    (dict(hp=lz.AdamHP(lr=float("nan"))), lz.ZERO_EINVAL),
    (dict(hp=lz.AdamHP(eps=-1.0)), lz.ZERO_EINVAL),
    (dict(grads=[A, 0]), lz.ZERO_EINVAL),
    (dict(grads=[A, A + 1]), lz.ZERO_EALIGN),
    (dict(p=A + 120 * MB + 1), lz.ZERO_EALIGN),
    (dict(ins=[A + 100 * MB + 2, A + 101 * MB, A + 102 * MB]), lz.ZERO_EALIGN),
    (dict(outs=[A + 100 * MB, A + 111 * MB, A + 112 * MB]), lz.ZERO_EINVAL),      # out == in
    (dict(outs=[A + 110 * MB, A + 110 * MB + 400, A + 112 * MB]), lz.ZERO_EINVAL),  # outs overlap
    (dict(p=A), lz.ZERO_EINVAL),                                                    # param over grads
    (dict(st=A + 110 * MB + 8), lz.ZERO_EINVAL),                                    # status in out
])
def test_fused_rejects(kw, code):
    with pytest.raises(lz.ZeroError) as e:
        _fused(**kw)
    assert e.value.code == code


def test_zero_length_launches_nothing():
    before = lz.zero_kernel_launches()
    _fused(n=0)
    lz.zero_adam_shard(0, A, A + MB, A + 2 * MB, A + 3 * MB, A + 4 * MB, HP, 1, A + 5 * MB, 0)
    lz.zero_step_commit(0, A, A + MB, A + 2 * MB, A + 3 * MB, A + 4 * MB, A + 5 * MB,
                        A + 6 * MB, A + 7 * MB, 0)
    assert lz.zero_kernel_launches() == before


@pytest.mark.parametrize("args,code", [
    ((10, 0, A + MB, A + 2 * MB, A + 3 * MB, A + 4 * MB), lz.ZERO_EINVAL),        # null grad
    ((10, A, A + MB + 2, A + 2 * MB, A + 3 * MB, A + 4 * MB), lz.ZERO_EALIGN),
    ((10, A, A + MB, A + MB + 20, A + 3 * MB, A + 4 * MB), lz.ZERO_EINVAL),        # m over master
    ((10, A, A + MB, A + 2 * MB, A + 3 * MB, A + 4 * MB + 1), lz.ZERO_EALIGN),
])
def test_adam_rejects(args, code):
    with pytest.raises(lz.ZeroError) as e:
        lz.zero_adam_shard(*args, HP, 1, A + 9 * MB, 0)
    assert e.value.code == code
    with pytest.raises(lz.ZeroError) as e:
        lz.zero_adam_shard(10, A, A + MB, A + 2 * MB, A + 3 * MB, A + 4 * MB, HP, 0, A + 9 * MB, 0)
    assert e.value.code == lz.ZERO_EINVAL


def test_reduce_scatter_rejects():
    pl = lz.zero_plan_create([100, 28], 4, 2, 32)
    grads = [A + i * MB for i in range(4)]
    shards = [A + (10 + i) * MB for i in range(4)]
    st = A + 50 * MB
    for k, g, s, code in [(4, grads, shards, lz.ZERO_EINVAL),       # bucket out of range
                          (-1, grads, shards, lz.ZERO_EINVAL),
                          (0, grads[:3] + [0], shards, lz.ZERO_EINVAL),
                          (0, grads, shards[:3] + [A + 10 * MB + 2], lz.ZERO_EALIGN),
                          (0, grads, shards[:3] + [A + 10 * MB + 8], lz.ZERO_EINVAL),  # overlap
                          (0, grads, shards[:3] + [A + 4], lz.ZERO_EINVAL)]:            # over grads
        with pytest.raises(lz.ZeroError) as e:
            lz.zero_reduce_scatter_bucket(pl, k, g, s, st, 0)
        assert e.value.code == code


def test_scheduler_rejects():
    pl = lz.zero_plan_create([100, 28], 4, 2, 32)
    need = lz.zero_sched_slot_elems(pl, 2)
    assert need == 2 * 4 * 32
    shards = [A + (10 + i) * MB for i in range(4)]
    with pytest.raises(lz.ZeroError) as e:
        lz.zero_sched_create(pl, A, need - 1, 2, shards, A + 50 * MB, 0)
    assert e.value.code == lz.ZERO_ENOMEM
    with pytest.raises(lz.ZeroError) as e:
        lz.zero_sched_create(pl, A + 8, need, 2, shards, A + 50 * MB, 0)
    assert e.value.code == lz.ZERO_EALIGN
    with pytest.raises(lz.ZeroError) as e:
        lz.zero_sched_create(pl, A, need, 0, shards, A + 50 * MB, 0)
    assert e.value.code == lz.ZERO_EINVAL


def test_status_strings():
    for code in range(6):
        assert lz.zero_status_string(code).startswith("ZERO_")


@pytest.mark.parametrize("t", [1, 2, 3, 10, 1000, 123456])
@pytest.mark.parametrize("hp", [lz.AdamHP(), lz.AdamHP(lr=3e-4, beta1=0.8, beta2=0.95, eps=1e-6,
                                                     loss_scale=1000.0),
                                lz.AdamHP(loss_scale=0.5)])
def test_adam_consts_match_oracle_bitwise(hp, t):
    c = lz.zero_adam_consts_for_step(hp, t)
    o = oracle.adam_scalars(oracle.AdamHP(hp.lr, hp.beta1, hp.beta2, hp.eps, hp.loss_scale), t)
    pairs = [("beta1", "b1"), ("one_minus_beta1", "omb1"), ("beta2", "b2"),
             ("one_minus_beta2", "omb2"), ("step_size", "step_size"), ("bias2_sqrt", "bc2s"),
             ("eps", "eps"), ("loss_scale", "loss_scale")]
    for a, b in pairs:
        assert np.float32(getattr(c, a)).view(np.uint32) == np.float32(o[b]).view(np.uint32), a
    pow2 = hp.loss_scale in (1024.0, 0.5)
    assert c.loss_scale_pow2 == int(pow2)
    if pow2:
        assert c.inv_loss_scale == 1.0 / hp.loss_scale


def test_dc_variants_reject():
    with pytest.raises(lz.ZeroError) as e:
        lz.zero_adam_consts_for_step(HP, 0)
    assert e.value.code == lz.ZERO_EINVAL
    grads = [A + i * MB for i in range(2)]
    ins = [A + 100 * MB, A + 101 * MB, A + 102 * MB]
    outs = [A + 110 * MB, A + 111 * MB, A + 112 * MB]
    for dc, code in [(0, lz.ZERO_EINVAL), (A + 140 * MB + 2, lz.ZERO_EALIGN)]:
        with pytest.raises(lz.ZeroError) as e:
            lz.zero_step_fused_dc(1000, 2, grads, *ins, *outs, A + 120 * MB, dc, A + 130 * MB, 0)
        assert e.value.code == code
        with pytest.raises(lz.ZeroError) as e:
            lz.zero_adam_shard_dc(10, A, A + MB, A + 2 * MB, A + 3 * MB, A + 4 * MB, dc,
                                  A + 5 * MB, 0)
        assert e.value.code == code


def test_consts_table_matches_per_step():
    tab = lz.zero_adam_consts_table(HP, 5, 20)
    for i in range(20):
        c = lz.zero_adam_consts_for_step(HP, 5 + i)
        assert bytes(tab[i]) == bytes(c)
    with pytest.raises(lz.ZeroError):
        lz.zero_adam_consts_table(HP, 0, 3)


def test_scaler_rejects():
    ok = lz.ScalerParams(2.0, 0.5, 2000)
    for args, code in [((0, A, 10, A + MB, A + 2 * MB), lz.ZERO_EINVAL),
                       ((A, A, 0, A + MB, A + 2 * MB), lz.ZERO_EINVAL),
                       ((A + 4, A, 10, A + MB, A + 2 * MB), lz.ZERO_EALIGN),
                       ((A, A + MB, 10, A + MB + 40, A + 2 * MB), lz.ZERO_EINVAL)]:  # in table
        with pytest.raises(lz.ZeroError) as e:
            lz.zero_scaler_prepare(*args, 0)
        assert e.value.code == code
    for prm, code in [(lz.ScalerParams(2.0, 0.5, 0), lz.ZERO_EINVAL),
                      (lz.ScalerParams(float("inf"), 0.5, 10), lz.ZERO_EINVAL),
                      (lz.ScalerParams(2.0, -0.5, 10), lz.ZERO_EINVAL)]:
        with pytest.raises(lz.ZeroError) as e:
            lz.zero_scaler_update(A, prm, A + MB, 0)
        assert e.value.code == code
    with pytest.raises(lz.ZeroError) as e:
        lz.zero_scaler_update(A + 4, ok, A + MB, 0)
    assert e.value.code == lz.ZERO_EALIGN


def test_q8_rejects():
    with pytest.raises(lz.ZeroError) as e:
        lz.zero_quantize_q8(100, A, A + MB + 2, 0)
    assert e.value.code == lz.ZERO_EALIGN
    with pytest.raises(lz.ZeroError) as e:
        lz.zero_quantize_q8(100, A, A + 100, 0)                     # payload over grad
    assert e.value.code == lz.ZERO_EINVAL
    assert lz.q8_payload_bytes(1) == 132 and lz.q8_payload_bytes(256) == 264
    ps = [A + i * MB for i in range(2)]
    ins = [A + 100 * MB, A + 101 * MB, A + 102 * MB]
    outs = [A + 110 * MB, A + 111 * MB, A + 112 * MB]
    for pay, code in [(ps[:1] + [0], lz.ZERO_EINVAL), (ps[:1] + [A + MB + 2], lz.ZERO_EALIGN),
                      ([A + 110 * MB, ps[1]], lz.ZERO_EINVAL)]:
        with pytest.raises(lz.ZeroError) as e:
            lz.zero_step_fused_q8(1000, 2, pay, *ins, *outs, A + 120 * MB, HP, 1, A + 130 * MB, 0)
        assert e.value.code == code


def test_overlap_region_bookkeeping():
    """zero_overlap_begin/end keep one open region per stream and reject misuse; they touch
    no device (host-side flags only)."""
    s1, s2 = 0x1000, 0x2000
    lz.zero_overlap_begin(s1)
    with pytest.raises(lz.ZeroError) as e:
        lz.zero_overlap_begin(s1)                  # already open on this stream
    assert e.value.code == lz.ZERO_EINVAL
    lz.zero_overlap_begin(s2)                      # another stream is independent
    lz.zero_overlap_end(s1)
    with pytest.raises(lz.ZeroError) as e:
        lz.zero_overlap_end(s1)                    # closed already
    assert e.value.code == lz.ZERO_EINVAL
    with lz.overlap(s1):
        pass
    lz.zero_overlap_end(s2)
    with pytest.raises(lz.ZeroError) as e:
        lz.zero_overlap_end(0)                     # never opened
    assert e.value.code == lz.ZERO_EINVAL


def test_q8_scheduler_sizes_and_rejects():
    """zero_sched_create_fused_q8: slots of n_slots x nd regions of the longest bucket's int8
    records rounded up to 16 bytes, and the fp16 fused mode's argument checks."""
    pl = lz.zero_plan_create([100, 28], 4, 2, 32)     # psi_p = 128, buckets of 32
    assert lz.zero_sched_slot_bytes_q8(pl, 2) == 2 * 4 * 144    # one 132-byte record -> 144
    pl2 = lz.zero_plan_create([1000, 300], 2, 2, 600)          # longest bucket 600: 5 records
    assert lz.zero_sched_slot_bytes_q8(pl2, 3) == 3 * 2 * 672   # 660 -> 672
    need = lz.zero_sched_slot_bytes_q8(pl, 2)
    slots = A
    ins = [A + 10 * MB, A + 11 * MB, A + 12 * MB]
    outs = [A + 20 * MB, A + 21 * MB, A + 22 * MB]
    par, dc, st = A + 30 * MB, A + 31 * MB, A + 32 * MB
    ok = dict(slots=slots, size=need, master_in=ins[0], master_out=outs[0], param_out=par,
              d_consts=dc, d_status=st)

    def call(**kw):
        a = dict(ok, **kw)
        return lz.zero_sched_create_fused_q8(pl, a["slots"], a["size"], 2, a["master_in"], ins[1],
                                             ins[2], a["master_out"], outs[1], outs[2],
                                             a["param_out"], a["d_consts"], a["d_status"], 0)

    for kw, code in [({"size": need - 1}, lz.ZERO_ENOMEM), ({"slots": slots + 8}, lz.ZERO_EALIGN),
                     ({"slots": 0}, lz.ZERO_EINVAL), ({"d_consts": 0}, lz.ZERO_EINVAL),
                     ({"master_in": 0}, lz.ZERO_EINVAL),
                     ({"master_out": ins[0]}, lz.ZERO_EINVAL),        # output over an input
                     ({"param_out": slots + 100}, lz.ZERO_EINVAL),    # output over the slots
                     ({"d_status": slots + need - 4}, lz.ZERO_EINVAL)]:
        with pytest.raises(lz.ZeroError) as e:
            call(**kw)
        assert e.value.code == code, kw


def test_fused_scheduler_rejects():
    """zero_sched_create_fused checks the plan, the state arrays (psi_p values each), the
    constants pointer and that no output overlaps an input, another output or the slots."""
    pl = lz.zero_plan_create([100, 28], 4, 2, 32)     # psi_p = 128
    need = lz.zero_sched_slot_elems(pl, 2)
    slots = A
    ins = [A + 10 * MB, A + 11 * MB, A + 12 * MB]
    outs = [A + 20 * MB, A + 21 * MB, A + 22 * MB]
    par, dc, st = A + 30 * MB, A + 31 * MB, A + 32 * MB
    ok = dict(master_in=ins[0], m_in=ins[1], v_in=ins[2], master_out=outs[0], m_out=outs[1],
              v_out=outs[2], param_out=par, d_consts=dc, d_status=st)

    def call(**kw):
        a = dict(ok, **kw)
        return lz.zero_sched_create_fused(pl, slots, need, 2, a["master_in"], a["m_in"],
                                          a["v_in"], a["master_out"], a["m_out"], a["v_out"],
                                          a["param_out"], a["d_consts"], a["d_status"], 0)

    for kw, code in [({"d_consts": 0}, lz.ZERO_EINVAL), ({"d_consts": dc + 2}, lz.ZERO_EALIGN),
                     ({"master_in": 0}, lz.ZERO_EINVAL), ({"m_out": outs[1] + 2}, lz.ZERO_EALIGN),
                     ({"v_out": ins[2] + 4}, lz.ZERO_EINVAL),          # output over an input
                     ({"param_out": outs[0] + 100}, lz.ZERO_EINVAL),   # over another output
                     ({"master_out": slots + 64}, lz.ZERO_EINVAL),     # over the slots
                     ({"d_status": slots + 16}, lz.ZERO_EINVAL)]:
        with pytest.raises(lz.ZeroError) as e:
            call(**kw)
        assert e.value.code == code, kw
    with pytest.raises(lz.ZeroError) as e:
        lz.zero_sched_create_fused(pl, slots, need - 1, 2, *ins, *outs, par, dc, st, 0)
    assert e.value.code == lz.ZERO_ENOMEM


def test_q8_dc_rejects():
    ins = [A + 100 * MB, A + 101 * MB, A + 102 * MB]
    outs = [A + 110 * MB, A + 111 * MB, A + 112 * MB]
    pays = [A + i * MB for i in range(2)]
    for dc, code in [(0, lz.ZERO_EINVAL), (A + 140 * MB + 2, lz.ZERO_EALIGN)]:
        with pytest.raises(lz.ZeroError) as e:
            lz.zero_step_fused_q8_dc(1000, 2, pays, *ins, *outs, A + 120 * MB, dc, A + 130 * MB, 0)
        assert e.value.code == code
    lz.zero_step_fused_q8_dc(0, 2, pays, *ins, *outs, A + 120 * MB, A + 140 * MB, A + 130 * MB, 0)


def test_state_bytes_rejects_overflowing_sizes():
    K = 12
    lim = (2**64 - 1) // (K + 6)
    rep = lz.zero_state_bytes(lim, 8, K)
    assert rep[lz.STAGES[0]]["total"] == 16 * lim
    with pytest.raises(lz.ZeroError) as e:
        lz.zero_state_bytes(lim + 1, 8, K)
    assert e.value.code == lz.ZERO_EINVAL


# ---------------------------------------------------------------------------------------------
# stage 3: gather and the per-owner update, argument errors on the host
# ---------------------------------------------------------------------------------------------
def _stage3_plan():
    return lz.zero_plan_create([100, 28], 4, 3, 0)     # psi_p = 128, S = 32


@pytest.mark.parametrize("lo,n,shards,out,st,code", [
    (0, 129, None, A + 50 * MB, A + 60 * MB, lz.ZERO_EINVAL),        # beyond psi_padded
    (127, 2, None, A + 50 * MB, A + 60 * MB, lz.ZERO_EINVAL),
    (0, 40, [A, 0, A + 2 * MB, A + 3 * MB], A + 50 * MB, A + 60 * MB, lz.ZERO_EINVAL),
    (0, 10, None, A + 50 * MB + 1, A + 60 * MB, lz.ZERO_EALIGN),     # out not 2-byte aligned
    (0, 10, [A + 1, A + MB, A + 2 * MB, A + 3 * MB], A + 50 * MB, A + 60 * MB, lz.ZERO_EALIGN),
    (0, 10, None, A + 10, A + 60 * MB, lz.ZERO_EINVAL),              # out over partition 0
    (0, 10, None, A + 50 * MB, A + 8, lz.ZERO_EINVAL),               # status in partition 0
    (0, 10, None, A + 50 * MB, 0, lz.ZERO_EINVAL),
])
def test_gather_params_rejects(lo, n, shards, out, st, code):
    pl = _stage3_plan()
    shards = shards or [A + q * MB for q in range(4)]
    before = lz.zero_kernel_launches()
    with pytest.raises(lz.ZeroError) as e:
        lz.zero_gather_params(pl, lo, n, shards, out, st, 0)
    assert e.value.code == code
    assert lz.zero_kernel_launches() == before


def test_stage3_update_rejects_and_launches_nothing():
    pl = _stage3_plan()
    grads = [A + (10 + r) * MB for r in range(4)]
    ins = [A + 20 * MB, A + 21 * MB, A + 22 * MB]
    outs = [A + 23 * MB, A + 24 * MB, A + 25 * MB]
    parts = [A + q * MB for q in range(4)]
    st = A + 30 * MB
    before = lz.zero_kernel_launches()
    for kw, code in [(dict(lo=100, n=29), lz.ZERO_EINVAL),            # beyond psi_padded
                     (dict(parts=[A, A + 16, A + 2 * MB, A + 3 * MB]), lz.ZERO_EINVAL),
                     (dict(parts=[A, A + MB, 0, A + 3 * MB]), lz.ZERO_EINVAL),
                     (dict(step=0), lz.ZERO_EINVAL),
                     (dict(outs=[A + 20 * MB, A + 24 * MB, A + 25 * MB]), lz.ZERO_EINVAL)]:
        a = dict(lo=10, n=60, parts=parts, step=1, outs=outs)
        a.update(kw)
        with pytest.raises(lz.ZeroError) as e:
            lz.zero_stage3_step_fused(pl, a["lo"], a["n"], grads, *ins, *a["outs"], a["parts"],
                                      HP, a["step"], st, 0)
        assert e.value.code == code, kw
    with pytest.raises(lz.ZeroError) as e:       # overlapping partitions in the commit
        lz.zero_stage3_step_commit(pl, *ins, *outs, [A, A + 32, A + 2 * MB, A + 3 * MB], st, 0)
    assert e.value.code == lz.ZERO_EINVAL
    lz.zero_gather_params(pl, 5, 0, parts, A + 50 * MB, st, 0)          # zero length: nothing
    lz.zero_stage3_step_fused(pl, 5, 0, grads, *ins, *outs, parts, HP, 1, st, 0)
    assert lz.zero_kernel_launches() == before


def test_layer_scheduler_sizes_and_rejects():
    """The stage-3 layer scheduler's buffer size (n_bufs buffers of the longest layer rounded
    up to 8 values) and its argument errors, all found before any CUDA call."""
    pl = _stage3_plan()                                  # psi = 128 = psi_p, S = 32
    parts = [A + q * MB for q in range(4)]
    good = [0, 17, 100, 128]                             # longest layer 83 -> 88 per buffer
    assert lz.zero_layer_sched_buf_elems(pl, good, 2) == 176
    assert lz.zero_layer_sched_buf_elems(pl, [0, 128], 3) == 3 * 128
    for bounds in ([1, 17, 128], [0, 17, 17, 128], [0, 17, 127], [0, 17, 129], [0, 40, 20, 128],
                   [0]):
        with pytest.raises(lz.ZeroError) as e:
            lz.zero_layer_sched_buf_elems(pl, bounds, 2)
        assert e.value.code == lz.ZERO_EINVAL, bounds
    with pytest.raises(lz.ZeroError) as e:
        lz.zero_layer_sched_buf_elems(pl, good, 0)
    assert e.value.code == lz.ZERO_EINVAL
    buf = A + 50 * MB
    for kw, code in [(dict(elems=175), lz.ZERO_ENOMEM),
                     (dict(buf=buf + 8), lz.ZERO_EALIGN),
                     (dict(buf=0), lz.ZERO_EINVAL),
                     (dict(n_bufs=0), lz.ZERO_EINVAL),
                     (dict(parts=[A, 0, A + 2 * MB, A + 3 * MB]), lz.ZERO_EINVAL),
                     (dict(parts=[A + 1, A + MB, A + 2 * MB, A + 3 * MB]), lz.ZERO_EALIGN),
                     (dict(buf=A + 2 * MB - 64), lz.ZERO_EINVAL),     # buffers over partition 2
                     (dict(bounds=[0, 200]), lz.ZERO_EINVAL)]:
        a = dict(elems=176, buf=buf, n_bufs=2, parts=parts, bounds=good)
        a.update(kw)
        with pytest.raises(lz.ZeroError) as e:
            lz.zero_layer_sched_create(pl, a["bounds"], a["parts"], a["buf"], a["elems"],
                                       a["n_bufs"], 0)
        assert e.value.code == code, kw


def test_stage3_q8_payload_sizes_and_rejects():
    """The stage-3 int8 payload of a range: one segment per owner part, the part's records
    rounded up to 16 bytes; the quantizer's and the step's argument errors."""
    pl = _stage3_plan()                                  # psi_p = 128, S = 32, Nd = 4
    assert lz.zero_stage3_payload_bytes_q8(pl, 10, 60) == 3 * 144   # parts of 22, 32 and 6
    assert lz.zero_stage3_payload_bytes_q8(pl, 0, 128) == 4 * 144
    assert lz.zero_stage3_payload_bytes_q8(pl, 5, 0) == 0
    with pytest.raises(lz.ZeroError) as e:
        lz.zero_stage3_payload_bytes_q8(pl, 100, 29)
    assert e.value.code == lz.ZERO_EINVAL
    before = lz.zero_kernel_launches()
    for args, code in [((10, 60, A, A + 50 * MB + 4), lz.ZERO_EALIGN),      # payload not 16-aligned
                       ((10, 60, A + 1, A + 50 * MB), lz.ZERO_EALIGN),
                       ((10, 60, 0, A + 50 * MB), lz.ZERO_EINVAL),
                       ((10, 60, A, A + 16), lz.ZERO_EINVAL),              # payload over the grads
                       ((120, 9, A, A + 50 * MB), lz.ZERO_EINVAL)]:        # beyond psi_padded
        with pytest.raises(lz.ZeroError) as e:
            lz.zero_stage3_quantize_q8(pl, *args, 0)
        assert e.value.code == code, args
    pays = [A + (10 + r) * MB for r in range(4)]
    ins = [A + 20 * MB, A + 21 * MB, A + 22 * MB]
    outs = [A + 23 * MB, A + 24 * MB, A + 25 * MB]
    parts = [A + q * MB for q in range(4)]
    st = A + 30 * MB
    for kw, code in [(dict(pays=pays[:3] + [0]), lz.ZERO_EINVAL),
                     (dict(pays=pays[:3] + [pays[3] + 2]), lz.ZERO_EALIGN),
                     (dict(step=0), lz.ZERO_EINVAL),
                     (dict(outs=[ins[0]] + outs[1:]), lz.ZERO_EINVAL),
                     (dict(parts=[A, A + 16, A + 2 * MB, A + 3 * MB]), lz.ZERO_EINVAL)]:
        a = dict(pays=pays, step=1, outs=outs, parts=parts)
        a.update(kw)
        with pytest.raises(lz.ZeroError) as e:
            lz.zero_stage3_step_fused_q8(pl, 10, 60, a["pays"], *ins, *a["outs"], a["parts"], HP,
                                         a["step"], st, 0)
        assert e.value.code == code, kw
    assert lz.zero_kernel_launches() == before


def test_step_fused_ranges_rejects_before_launching():
    grads = [A + i * MB for i in range(2)]
    good = (1000, grads, A + 100 * MB, A + 101 * MB, A + 102 * MB, A + 110 * MB, A + 111 * MB,
            A + 112 * MB, A + 120 * MB)
    bad_out = (1000, grads, A + 200 * MB, A + 201 * MB, A + 202 * MB, A + 200 * MB,
               A + 211 * MB, A + 212 * MB, A + 220 * MB)                  # out == in
    before = lz.zero_kernel_launches()
    for ranges, kw, code in [([good, bad_out], {}, lz.ZERO_EINVAL),
                             ([good], dict(step=0), lz.ZERO_EINVAL),
                             ([good], dict(st=A + 110 * MB + 4), lz.ZERO_EINVAL),
                             ([good[:1] + ([A, A + 1],) + good[2:]], {}, lz.ZERO_EALIGN)]:
        with pytest.raises(lz.ZeroError) as e:
            lz.zero_step_fused_ranges(2, ranges, HP, kw.get("step", 1),
                                      kw.get("st", A + 130 * MB), True, 0)
        assert e.value.code == code
    assert lz.zero_kernel_launches() == before
    lz.zero_step_fused_ranges(2, [], HP, 1, A + 130 * MB, True, 0)     # nothing to do
    assert lz.zero_kernel_launches() == before


def test_step_fused_q8_ranges_rejects_before_launching():
    pays = [A + i * MB for i in range(2)]
    good = (1000, pays, A + 100 * MB, A + 101 * MB, A + 102 * MB, A + 110 * MB, A + 111 * MB,
            A + 112 * MB, A + 120 * MB)
    pay_on_out = (1000, [A + 210 * MB, pays[1]], A + 200 * MB, A + 201 * MB, A + 202 * MB,
                  A + 210 * MB, A + 211 * MB, A + 212 * MB, A + 220 * MB)   # payload == master_out
    before = lz.zero_kernel_launches()
    for ranges, kw, code in [([good, pay_on_out], {}, lz.ZERO_EINVAL),
                             ([good], dict(step=0), lz.ZERO_EINVAL),
                             ([good[:1] + ([A, A + MB + 2],) + good[2:]], {}, lz.ZERO_EALIGN),
                             ([good[:1] + ([A, 0],) + good[2:]], {}, lz.ZERO_EINVAL)]:
        with pytest.raises(lz.ZeroError) as e:
            lz.zero_step_fused_q8_ranges(2, ranges, HP, kw.get("step", 1), A + 130 * MB, True, 0)
        assert e.value.code == code
    assert lz.zero_kernel_launches() == before
    lz.zero_step_fused_q8_ranges(2, [], HP, 1, A + 130 * MB, True, 0)   # nothing to do
    assert lz.zero_kernel_launches() == before
    with pytest.raises(ValueError):
        lz.PreparedStepRanges(2, [good], "bf16")


def test_step_fused_replicas_rejects_before_launching():
    """The epilogue all-gather's replica list: 1..64 distinct, aligned ranges, each checked
    like a param_out; anything else is refused with nothing launched."""
    grads = [A + i * MB for i in range(2)]
    ins = [A + 100 * MB, A + 101 * MB, A + 102 * MB]
    outs = [A + 110 * MB, A + 111 * MB, A + 112 * MB]
    st = A + 130 * MB
    reps = [A + 120 * MB, A + 121 * MB, A + 122 * MB]
    before = lz.zero_kernel_launches()
    for replicas, code in [([], lz.ZERO_EINVAL),
                           ([A + 120 * MB + 2 * k * 1000 for k in range(65)], lz.ZERO_EINVAL),
                           (reps[:1] + [0], lz.ZERO_EINVAL),
                           (reps[:1] + [A + 120 * MB + 500], lz.ZERO_EINVAL),   # overlapping
                           (reps[:1] + [A + 110 * MB], lz.ZERO_EINVAL),         # on master_out
                           (reps[:1] + [A + 123 * MB + 1], lz.ZERO_EALIGN)]:
        with pytest.raises(lz.ZeroError) as e:
            lz.zero_step_fused_replicas(1000, 2, grads, *ins, *outs, replicas, HP, 1, st, 0)
        assert e.value.code == code, replicas[:3]
        with pytest.raises(lz.ZeroError) as e:
            lz.zero_step_commit_replicas(1000, *ins, *outs, replicas, st, 0)
        assert e.value.code == code, replicas[:3]
    with pytest.raises(lz.ZeroError) as e:     # a replica on a rank's gradient (the step only)
        lz.zero_step_fused_replicas(1000, 2, grads, *ins, *outs, reps[:1] + [A + 1 * MB + 100],
                                    HP, 1, st, 0)
    assert e.value.code == lz.ZERO_EINVAL
    with pytest.raises(lz.ZeroError) as e:
        lz.zero_step_fused_replicas(1000, 2, grads, *ins, *outs, reps, HP, 0, st, 0)   # t = 0
    assert e.value.code == lz.ZERO_EINVAL
    lz.zero_step_fused_replicas(0, 2, grads, *ins, *outs, reps, HP, 1, st, 0)   # nothing to do
    assert lz.zero_kernel_launches() == before
