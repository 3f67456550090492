"""The oracle's pins must catch plausible slips: each case plants one slip in a COPY of the
oracle (its C source, or the partitioning code of its Python module), builds it on the CPU and
checks that at least one pin from tests/test_oracle_pins.py fails against it.

Nothing here touches the real oracle, the CUDA library or a GPU.
"""
import importlib.util
import os
import subprocess
import sys

import numpy as np
import pytest

import oracle
from oracle import build as obuild
from tests import test_oracle_pins as pins

ORACLE_DIR = os.path.dirname(oracle.__file__)

# (name, original text, planted slip, pins expected to notice)
C_MUTANTS = [
    ("swapped beta in momentum", "float m_keep = s->b1 * m[i];", "float m_keep = s->b2 * m[i];",
     ["adam_textbook"]),
    ("update sign flipped", "float w = master[i] - delta;", "float w = master[i] + delta;",
     ["adam_first", "adam_textbook"]),
    ("no square root in bias correction", "s->bc2s = (float)sqrt(bc2);", "s->bc2s = (float)bc2;",
     ["adam_first"]),
    ("bias correction one step late", "double bc1 = 1.0 - pow(hp->beta1, (double)t);",
     "double bc1 = 1.0 - pow(hp->beta1, (double)(t + 1));", ["adam_const", "adam_first"]),
    ("eps dropped", "float denom = root / s->bc2s + s->eps;", "float denom = root / s->bc2s;",
     ["adam_first"]),
    ("gradient not unscaled", "float g = red[i] / s->loss_scale;", "float g = red[i];",
     ["adam_first", "adam_textbook"]),
    ("variance takes g, not g squared", "float v_new = s->omb2 * gsq;",
     "float v_new = s->omb2 * g;", ["adam_textbook"]),
    ("ranks summed in reverse order", "for (int r = 0; r < nd; r++) s = s + orc_h2f(g[r][i]);",
     "for (int r = nd - 1; r >= 0; r--) s = s + orc_h2f(g[r][i]);", ["sum_order"]),
    ("sum, not mean", "s = s + orc_h2f(g[r][i]);\n        red[i] = s / fnd;",
     "s = s + orc_h2f(g[r][i]);\n        red[i] = s;", ["exact_sums"]),
    ("ties rounded away from zero in the fp16 cast",
     "if (rem > half || (rem == half && (n & 1u))) n += 1u;", "if (rem >= half) n += 1u;",
     ["f2h_mid"]),
    ("no padding to a multiple of Nd", "*psi_p = s * (uint64_t)nd;", "*psi_p = total;",
     ["plan_bf"]),
    ("stage 2 keeps full gradients", "{p_full, g_sh, o_sh},", "{p_full, g_full, o_sh},",
     ["memory"]),
    ("overflow check ignores NaN", "if (((u >> 23) & 0xffu) == 0xffu) return 0;",
     "if (u == 0x7f800000u || u == 0xff800000u) return 0;", ["overflow_nan"]),
    ("payload scale divides by 128", "float scale = poisoned ? float_of(0x7fc00000u) : amax / 127.0f;",
     "float scale = poisoned ? float_of(0x7fc00000u) : amax / 128.0f;", ["q8_bf"]),
    ("payload ties rounded away from zero",
     "if (r > 0.5f || (r == 0.5f && ((int32_t)f & 1))) f = f + 1.0f;",
     "if (r >= 0.5f) f = f + 1.0f;", ["q8_ties"]),
    ("payload scale of the wrong block", "s = fmaf((float)q[r][i], scales[r][i / ORC_QB], s);",
     "s = fmaf((float)q[r][i], scales[r][(i + 1) / ORC_QB], s);", ["q8_red"]),
    ("payload product rounded before the sum",
     "s = fmaf((float)q[r][i], scales[r][i / ORC_QB], s);",
     "{ float x = (float)q[r][i] * scales[r][i / ORC_QB]; s = s + x; }", ["q8_red"]),
]

PINS = {
    "adam_textbook": lambda: pins.test_adam_vs_textbook_fp64(5),
    "adam_first": pins.test_adam_first_step_from_zero_state,
    "adam_const": pins.test_adam_constant_gradient_many_steps,
    "sum_order": pins.test_sum_order_golden,
    "exact_sums": lambda: pins.test_exact_sums_closed_form(4),
    "f2h_mid": pins.test_f2h_vs_exact_rounding_at_midpoints,
    "plan_bf": lambda: [pins.test_plan_brute_force(s) for s in range(20)],
    "memory": pins.test_memory_figures_of_the_7p5b_example,
    "overflow_nan": lambda: pins.test_overflow_skips_whole_step(0x7e00),
    "q8_bf": lambda: pins.test_quant_q8_brute_force(0),
    "q8_ties": pins.test_quant_q8_ties_go_to_even,
    "q8_red": lambda: pins.test_reduce_mean_q8_brute_force(3),
}


def _build_mutant(tmp_path, old, new):
    with open(obuild.SRC) as f:
        src = f.read()
    assert src.count(old) == 1, old
    path = tmp_path / "oracle_mutant.c"
    path.write_text(src.replace(old, new))
    lib = tmp_path / "liboracle_mutant.so"
    subprocess.check_call(["gcc", *obuild.CFLAGS, str(path), "-o", str(lib), "-lm"])
    return str(lib)


@pytest.mark.parametrize("name,old,new,expect", C_MUTANTS, ids=[m[0] for m in C_MUTANTS])
def test_c_mutant_is_caught(tmp_path, name, old, new, expect):
    # the pin passes on the real oracle ...
    for p in expect:
        PINS[p]()
    saved = oracle._lib
    oracle._lib = oracle.bind(_build_mutant(tmp_path, old, new))
    try:
        caught = []
        for p in expect:
            try:
                PINS[p]()
            except AssertionError:
                caught.append(p)
        # ... and fails on the mutant
        assert caught, f"slip '{name}' went unnoticed by {expect}"
    finally:
        oracle._lib = saved


# slips in the partitioning around the element arithmetic (Python side of the oracle)
PY_MUTANTS = [
    ("owner reads the neighbour's slice",
     "shards.append(reduce_mean([g[r * S:(r + 1) * S] for g in gs]))",
     "shards.append(reduce_mean([g[(r + 1) % nd * S:((r + 1) % nd + 1) * S] for g in gs]))"),
    ("all-gather skipped", "        p_out[sl] = p16           # all-gather",
     "        pass                      # all-gather"),
    ("bucket slice kept by the wrong owner",
     "grad_shard[r][a - r * S:b - r * S] = reduce_mean([g[a - lo:b - lo] for g in local])",
     "grad_shard[(r + 1) % nd][a - r * S:b - r * S] = reduce_mean([g[a - lo:b - lo] for g in local])"),
    ("one rank left out of the bucket reduce-scatter",
     "local = [_as_u16(bucket_grad(k, j)) for j in range(nd)]",
     "local = [_as_u16(bucket_grad(k, j)) for j in range(max(1, nd - 1))]"),
]


@pytest.mark.parametrize("name,old,new", PY_MUTANTS, ids=[m[0] for m in PY_MUTANTS])
def test_partition_mutant_is_caught(name, old, new, monkeypatch):
    with open(os.path.join(ORACLE_DIR, "__init__.py")) as f:
        src = f.read()
    assert src.count(old) == 1, old
    spec = importlib.util.spec_from_loader("oracle._mutant", loader=None)
    mod = importlib.util.module_from_spec(spec)
    mod.__package__ = "oracle"
    monkeypatch.setitem(sys.modules, "oracle._mutant", mod)
    exec(compile(src.replace(old, new), "oracle_mutant.py", "exec"), mod.__dict__)
    monkeypatch.setattr(pins, "oracle", mod)
    failed = 0
    for nd in (3, 4):
        try:
            pins.test_zero_stages_equal_plain_dp(nd, [50, 1, 64, 13], 17)
        except (AssertionError, ValueError):
            failed += 1
    assert failed, f"slip '{name}' went unnoticed"


# slips in the stage-3 partitioning (parameters partitioned and gathered per layer)
STAGE3_MUTANTS = [
    ("gather takes the neighbour's partition",
     "out[a - lo:b - lo] = _as_u16(param_shards[q])[a - q * S:b - q * S]",
     "out[a - lo:b - lo] = _as_u16(param_shards[(q + 1) % len(param_shards)])[a - q * S:b - q * S]"),
    ("backward parameter all-gather not counted",
     "        bwd[l] = gather_params(shards, S, lo, hi)\n        comm += hi - lo",
     "        bwd[l] = gather_params(shards, S, lo, hi)"),
    ("updated partition stored at the wrong owner",
     "        shards[q] = p16                  # the owner's partition",
     "        shards[(q + 1) % nd] = p16       # the owner's partition"),
    ("layer gradient reduced from the wrong slice",
     "grad_shard[q][a - q * S:b - q * S] = reduce_mean([g[a - lo:b - lo] for g in local])",
     "grad_shard[q][a - q * S:b - q * S] = reduce_mean([g[::-1][a - lo:b - lo] for g in local])"),
]


@pytest.mark.parametrize("name,old,new", STAGE3_MUTANTS, ids=[m[0] for m in STAGE3_MUTANTS])
def test_stage3_mutant_is_caught(name, old, new, monkeypatch):
    with open(os.path.join(ORACLE_DIR, "__init__.py")) as f:
        src = f.read()
    assert src.count(old) == 1, old
    spec = importlib.util.spec_from_loader("oracle._mutant3", loader=None)
    mod = importlib.util.module_from_spec(spec)
    mod.__package__ = "oracle"
    monkeypatch.setitem(sys.modules, "oracle._mutant3", mod)
    exec(compile(src.replace(old, new), "oracle_mutant3.py", "exec"), mod.__dict__)
    monkeypatch.setattr(pins, "oracle", mod)
    failed = 0
    checks = [lambda: pins.test_stage3_equals_plain_dp(3, [50, 1, 64, 13], [2, 1, 1]),
              lambda: pins.test_stage3_gathers_are_the_layer_parameters(3),
              lambda: pins.test_stage3_moves_three_psi(4, [300, 250, 250, 249])]
    for c in checks:
        try:
            c()
        except (AssertionError, ValueError):
            failed += 1
    assert failed, f"slip '{name}' went unnoticed"
