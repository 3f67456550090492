"""The N > 1 host logic of bench.py, on the CPU with world-size-2 gloo process groups (the
replicas share nothing on the data path; only the timing is reduced across ranks)."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, ws, port, times, out):
    import datetime
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(ws), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=ws,
                            timeout=datetime.timedelta(seconds=60))
    try:
        assert bench.dist_setup() == (ws, rank, rank)
        ms = bench.max_over_ranks(times[rank], ws, "cpu")
        rate = bench.aggregate_rate(ws, 1000, 10, ms)
        out.put((rank, ms, rate))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_aggregate_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.SimpleQueue()
    port = _free_port()
    times = [12.5, 20.0]
    procs = [ctx.Process(target=_worker, args=(r, 2, port, times, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get() for _ in range(2))
    for rank, ms, rate in res:
        assert ms == 20.0                                  # the slowest rank's time on every rank
        assert rate == pytest.approx(2 * 1000 * 10 / 0.020)  # all ranks' units / that time


def test_reference_arm_under_torchrun_prints_once():
    env = dict(os.environ, PYTHONPATH=ROOT)
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()),
           os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
           "--steps", "3", "--warmup", "3"]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=600, env=env, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["e2e"]["h2d_bytes_per_step"] == 0


def _worker_failing(rank, ws, port, mode, out):
    """Rank 1 fails on the host: it exits before the timing collective ("dies") or before
    joining the process group at all ("never_joins"); rank 0 must get an error, not hang."""
    import datetime
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(ws), LOCAL_RANK=str(rank))
    if rank == 1 and mode == "never_joins":
        os._exit(3)
    try:
        dist.init_process_group("gloo", rank=rank, world_size=ws,
                                timeout=datetime.timedelta(seconds=10))
    except Exception as e:   # the rendezvous gives up on the missing rank
        out.put((rank, "error", type(e).__name__))
        return
    if rank == 1:
        os._exit(3)           # dies between steps, with no collective in flight
    try:
        bench.max_over_ranks(1.0, ws, "cpu")
        out.put((rank, "no error", ""))
    except Exception as e:
        out.put((rank, "error", type(e).__name__))


@pytest.mark.parametrize("mode", ["dies", "never_joins"])
def test_failed_rank_is_detected_on_the_host(mode):
    import time
    ctx = mp.get_context("spawn")
    q = ctx.SimpleQueue()
    port = _free_port()
    t0 = time.monotonic()
    procs = [ctx.Process(target=_worker_failing, args=(r, 2, port, mode, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(180)
    assert all(p.exitcode is not None for p in procs), "a rank hung"
    assert procs[1].exitcode == 3
    assert procs[0].exitcode == 0
    rank, verdict, _ = q.get()
    assert (rank, verdict) == (0, "error")
    assert time.monotonic() - t0 < 170
