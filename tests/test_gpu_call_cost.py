"""Host cost of a data-path call through the C ABI, measured by a small C program
(tests/call_cost.c) so that Python's ctypes marshalling is not part of it: zero_step_fused on a
1 MiB bucket per rank at Nd = 8, outside and inside an overlap region, and the device time per
call of the region's calls."""
import json
import os
import subprocess

import pytest

from tests._gpu import lz, require_gpu

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CUDA = os.environ.get("CUDA_HOME", "/usr/local/cuda")


def _build(tmp_path):
    exe = str(tmp_path / "call_cost")
    libdir = os.path.dirname(lz.LIB_PATH)
    subprocess.check_call(["gcc", "-O2", "-std=c11", os.path.join(ROOT, "tests", "call_cost.c"),
                           "-I", os.path.join(ROOT, "include"), "-I", os.path.join(CUDA, "include"),
                           "-L", libdir, "-lzero", "-Wl,-rpath," + libdir,
                           "-L", os.path.join(CUDA, "lib64"), "-lcudart",
                           "-Wl,-rpath," + os.path.join(CUDA, "lib64"), "-o", exe])
    return exe


@pytest.mark.parametrize("n,nd", [(1 << 19, 8), (1 << 19, 64), (1 << 23, 8)])
def test_c_call_cost(tmp_path, n, nd):
    require_gpu()
    exe = _build(tmp_path)
    r = subprocess.run([exe, str(n), str(nd), "400"], capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0, r.stderr
    d = json.loads(r.stdout.strip().splitlines()[-1])
    print("CALL COST", json.dumps(d))
    assert d["status"] == 0
    # a launch costs a few microseconds of host time; anything near 50 us means a lock, an
    # allocation or a synchronisation crept onto the launch path
    assert d["host_us_ordered"] < 50 and d["host_us_region"] < 50
