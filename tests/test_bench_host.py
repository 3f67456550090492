"""bench.py's host side on the CPU: the workload names and sizes both arms report, and the
reference arm's line (the oracle on a bounded sample) for the small workloads."""
import json
import os
import subprocess
import sys
import types

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _args(**kw):
    base = dict(workload="zero2_1p3b", nd=None, bucket=None, psi=None, payload="fp16",
                stage2="fused", no_overlap=False, graph=False, l2="warm")
    base.update(kw)
    return types.SimpleNamespace(**base)


def test_workload_configs():
    tiny = bench.workload_config(_args(workload="tiny"))
    assert (tiny["workload"], tiny["psi"], tiny["nd"], tiny["stage"]) == \
        ("tiny_stage1", 1 << 20, 4, 1)
    g2 = bench.workload_config(_args(workload="gpt2_small"))
    assert (g2["psi"], g2["nd"], g2["tensors"]) == (123_653_376, 8, 147)
    d = bench.workload_config(_args())
    assert (d["workload"], d["psi"], d["nd"], d["buckets"]) == \
        ("zero2_1p3b_fused", 1_311_528_960, 16, 27)
    fq = bench.workload_config(_args(workload="flat", psi=1 << 28, nd=64, payload="q8"))
    assert fq["workload"] == "flat_268435456_q8" and fq["calls_per_step"] == 4
    s3 = bench.workload_config(_args(workload="zero3_gpt2_small"))
    assert (s3["stage"], s3["layers"]) == (3, 14)
    dq = bench.workload_config(_args(payload="q8"))
    assert (dq["workload"], dq["buckets"], dq["calls_per_step"]) == ("zero2_1p3b_fused_q8", 27, 28)
    assert bench.traffic_key(types.SimpleNamespace(config=dq, nd=16)) == \
        "zero2_1p3b_fused_q8_nd16_b50000000"     # the key profiles/traffic.json holds


def test_traffic_keys_name_the_bucket_only_for_multi_call_steps():
    wl = types.SimpleNamespace(config={"workload": "flat_2p29", "calls_per_step": 8,
                                       "bucket": 1 << 26}, nd=16)
    assert bench.traffic_key(wl) == "flat_2p29_nd16_b67108864"
    wl1 = types.SimpleNamespace(config={"workload": "shard_7p5b_rank31_q8",
                                        "calls_per_step": 1}, nd=64)
    assert bench.traffic_key(wl1) == "shard_7p5b_rank31_q8_nd64"


@pytest.mark.parametrize("extra", [["--workload", "tiny"], ["--workload", "tiny", "--l2", "flushed"]])
def test_reference_arm_line_for_the_tiny_case(extra):
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "3", "--warmup", "3", *extra],
                       capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["config"]["workload"] == "tiny_stage1"
    assert d["value"] > 0 and d["higher_is_better"] is True
    assert d["cpu_baseline"]["kind"] == "oracle" and d["e2e"]["h2d_bytes_per_step"] == 0
