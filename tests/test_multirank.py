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


# ---------------------------------------------------------------------------------------------
# the distributed step (dist.py): its exchange on CPU processes over gloo, with the owner's
# fused step and commit done by the oracle (the library needs a GPU)
# ---------------------------------------------------------------------------------------------
def _pack_q8(q, scales):
    """The library's payload records (128 bytes q + 128, then the fp32 scale; a short last
    block padded with q = 0) from the oracle's logical q and scales."""
    import numpy as np
    nb = scales.size
    rec = np.zeros((nb, 132), np.uint8)
    rec[:, :128] = 128
    codes = (q.astype(np.int16) + 128).astype(np.uint8)
    for b in range(nb):
        blk = codes[128 * b:128 * (b + 1)]
        rec[b, :blk.size] = blk
    rec[:, 128:] = np.ascontiguousarray(scales, np.float32).view(np.uint8).reshape(nb, 4)
    return rec.reshape(-1)


def _unpack_q8(payload, n):
    import numpy as np
    rec = np.asarray(payload).reshape(-1, 132)
    q = (rec[:, :128].astype(np.int16) - 128).astype(np.int8).reshape(-1)[:n]
    return q, np.ascontiguousarray(rec[:, 128:]).view(np.float32).reshape(-1)


class _OracleCompute:
    def __init__(self, fail=False):
        self.fail = fail     # report a kernel timeout (as a library kernel that gave up would)

    def fused(self, n, rows, state_in, state_out, params, hp, t, status):
        import numpy as np
        import oracle
        if self.fail:
            status |= 4
            state_out[0].fill_(float("nan"))    # a half-written output
            return
        red = oracle.reduce_mean([row.numpy() for row in rows])
        if not oracle.all_finite(red):
            status |= 1
            return
        w, m, v, p16 = oracle.adam(red, *(x.numpy() for x in state_in), hp, t)
        for dst, src in zip(state_out, (w, m, v)):
            dst.copy_(__import__("torch").from_numpy(np.ascontiguousarray(src)))
        params.view(__import__("torch").int16).copy_(
            __import__("torch").from_numpy(np.ascontiguousarray(p16).view(np.int16)))

    def gather(self, numels, nd, lo, n, partitions, out, status):
        import torch
        import oracle
        S = partitions[0].numel()
        g = oracle.gather_params([p.numpy() for p in partitions], S, lo, lo + n)
        out.view(torch.int16).copy_(torch.from_numpy(g.view("int16")))

    def fused_replicas(self, n, rows, state_in, state_out, replicas, hp, t, status):
        import torch
        own = torch.empty(n, dtype=torch.float16)
        before = int(status.item())
        self.fused(n, rows, state_in, state_out, own, hp, t, status)
        if int(status.item()) == before:         # written: the all-gather in the epilogue
            for rep in replicas:
                rep.copy_(own)

    def commit_replicas(self, n, state_in, state_out, replicas, status):
        import numpy as np
        import torch
        import oracle
        if int(status.item()) & (1 | 4 | 8):
            for dst, src in zip(state_out, state_in):
                dst.copy_(src)
            p16 = torch.from_numpy(oracle.f2h(state_in[0].numpy()).view(np.int16))
            for rep in replicas:
                rep.view(torch.int16).copy_(p16)
            status |= 2

    def quantize(self, n, grad, payload):
        import torch
        import oracle
        q, sc = oracle.quant_q8(grad.numpy())
        payload.copy_(torch.from_numpy(_pack_q8(q, sc)))

    def fused_q8(self, n, payloads, state_in, state_out, params, hp, t, status):
        import numpy as np
        import torch
        import oracle
        qs, scs = zip(*[_unpack_q8(p.numpy(), n) for p in payloads])
        skipped, w, m, v, p16 = oracle.step_q8(list(qs), list(scs),
                                               *(x.numpy() for x in state_in), hp, t)
        if skipped:
            status |= 1
            return
        for dst, src in zip(state_out, (w, m, v)):
            dst.copy_(torch.from_numpy(np.ascontiguousarray(src)))
        params.view(torch.int16).copy_(torch.from_numpy(np.ascontiguousarray(p16).view(np.int16)))

    def commit(self, n, state_in, state_out, params, status):
        import numpy as np
        import torch
        import oracle
        if int(status.item()) & (1 | 4 | 8):
            for dst, src in zip(state_out, state_in):
                dst.copy_(src)
            params.view(torch.int16).copy_(
                torch.from_numpy(oracle.f2h(state_in[0].numpy()).view(np.int16)))
            status |= 2


def _dist_case(numels, ws, bad_rank):
    """Every rank's inputs of the case, the same on every process (seeded)."""
    import torch
    from zero_partitioned_optimizer_plan_b200 import synth
    psi = sum(numels)
    psi_p = -(-psi // ws) * ws
    grads = []
    for r in range(ws):
        g = torch.zeros(psi_p, dtype=torch.float16)
        g[:psi] = synth.grad_f16(psi, 1e-3, seed=7, rank=r, step=1)
        if r == bad_rank:
            g[psi // 2] = float("inf")
        grads.append(g)
    master, m, v = synth.state_warm(psi_p, seed=8)
    return psi_p, grads, master, m, v


def _worker_dist(rank, ws, port, numels, bucket, bad_rank, out, payload="fp16"):
    import datetime
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import oracle
    from zero_partitioned_optimizer_plan_b200.dist import DistZeroStep
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=ws,
                            timeout=datetime.timedelta(seconds=60))
    try:
        psi_p, grads, master, m, v = _dist_case(numels, ws, bad_rank)
        S = psi_p // ws
        st_in = [x[rank * S:(rank + 1) * S].clone() for x in (master, m, v)]
        st_out = [torch.full_like(x, float("nan")) for x in st_in]
        params = torch.zeros(psi_p, dtype=torch.float16)
        params[rank * S:(rank + 1) * S] = torch.from_numpy(
            oracle.f2h(st_in[0].numpy()).view("float16"))
        status = torch.zeros(1, dtype=torch.int32)
        step = DistZeroStep(psi_p, bucket, compute=_OracleCompute(), payload=payload)
        flag = step.step(grads[rank], st_in, st_out, params, oracle.AdamHP(), 1, status)
        out.put((rank, int(flag.item()), int(status.item()), [x.numpy() for x in st_out],
                 params.numpy().view("uint16")))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("ws,bucket,bad_rank", [(2, 0, -1), (3, 0, -1), (2, 3000, -1),
                                                (3, 2500, -1), (3, 2500, 1)])
def test_distributed_step_exchange_gloo(ws, bucket, bad_rank):
    """The distributed step's all-to-all / all-reduce / all-gather on gloo ranks gives the
    single-process data-parallel step of the oracle (all ranks' gradients summed in rank
    order): every rank's shard of the state and every rank's full fp16 parameters; an inf in
    one rank's gradient skips the step on every rank."""
    import numpy as np
    import oracle
    numels = [1000, 37, 4099, 12345]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker_dist, args=(r, ws, port, numels, bucket, bad_rank, q))
             for r in range(ws)]
    for p in procs:
        p.start()
    try:   # read before joining: a result larger than the pipe buffer blocks its sender
        res = sorted((q.get(timeout=240) for _ in range(ws)), key=lambda x: x[0])
    finally:
        for p in procs:
            p.join(60)
            if p.exitcode is None:
                p.kill()
    assert all(p.exitcode == 0 for p in procs)
    psi_p, grads, master, m, v = _dist_case(numels, ws, bad_rank)
    ref = oracle.dp_step([g.numpy() for g in grads], master.numpy(), m.numpy(), v.numpy(),
                         oracle.f2h(master.numpy()), oracle.AdamHP(), 1)
    S = psi_p // ws
    for rank, flag, status, shard, params in res:
        assert flag == (1 if bad_rank >= 0 else 0)
        assert bool(status & 2) == ref.skipped == (bad_rank >= 0)
        for got, want in zip(shard, (ref.master, ref.m, ref.v)):
            assert np.array_equal(got.view(np.uint32),
                                  want[rank * S:(rank + 1) * S].view(np.uint32))
        assert np.array_equal(params, ref.params16)


def _worker_dist_fail(rank, ws, port, numels, bucket, fail_rank, out):
    import datetime
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import oracle
    from zero_partitioned_optimizer_plan_b200.dist import DistStepError, DistZeroStep
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=ws,
                            timeout=datetime.timedelta(seconds=60))
    try:
        psi_p, grads, master, m, v = _dist_case(numels, ws, -1)
        S = psi_p // ws
        st_in = [x[rank * S:(rank + 1) * S].clone() for x in (master, m, v)]
        st_out = [torch.full_like(x, float("nan")) for x in st_in]
        params = torch.zeros(psi_p, dtype=torch.float16)
        status = torch.zeros(1, dtype=torch.int32)
        step = DistZeroStep(psi_p, bucket, compute=_OracleCompute(fail=rank == fail_rank))
        raised = None
        try:
            step.step(grads[rank], st_in, st_out, params, oracle.AdamHP(), 1, status)
        except DistStepError as e:
            raised = e.bits
        # the ranks are still in step: one more collective completes on every rank
        t = torch.ones(1)
        dist.all_reduce(t)
        out.put((rank, raised, int(status.item()), [x.numpy() for x in st_in],
                 [x.numpy() for x in st_out], params.numpy().view("uint16"), float(t.item())))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("ws,fail_rank", [(2, 1), (3, 0)])
def test_distributed_step_failure_on_one_rank_voids_it_everywhere(ws, fail_rank):
    """One rank's kernels report a timeout (made on the host: the fake compute sets the bit and
    leaves a half-written output). Every rank learns it from the combined status, restores its
    shard through the commit, skips the parameter all-gather and raises DistStepError; the
    ranks stay in step (a later collective completes)."""
    import numpy as np
    import oracle
    numels = [1000, 37, 4099, 12345]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker_dist_fail,
                         args=(r, ws, port, numels, 3000, fail_rank, q)) for r in range(ws)]
    for p in procs:
        p.start()
    try:
        res = sorted((q.get(timeout=240) for _ in range(ws)), key=lambda x: x[0])
    finally:
        for p in procs:
            p.join(60)
            if p.exitcode is None:
                p.kill()
    assert all(p.exitcode == 0 for p in procs)
    psi_p = sum(numels) + (-sum(numels)) % ws
    S = psi_p // ws
    for rank, raised, status, st_in, st_out, params, t in res:
        assert raised == 4                       # the timeout bit, seen on every rank
        assert status == 4 | 2                   # combined bits + skipped
        for a, b in zip(st_in, st_out):          # the commit restored the shard
            assert np.array_equal(a.view(np.uint32), b.view(np.uint32))
        own = params[rank * S:(rank + 1) * S]
        assert np.array_equal(own, oracle.f2h(st_in[0]))
        rest = np.concatenate([params[:rank * S], params[(rank + 1) * S:]])
        assert not rest.any()                    # no all-gather ran
        assert t == ws


def _worker_dist_peer(rank, ws, port, numels, bucket, bad_rank, bufs, out):
    import datetime
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import oracle
    from zero_partitioned_optimizer_plan_b200.dist import DistZeroStep, SharedPeerBuffers
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=ws,
                            timeout=datetime.timedelta(seconds=60))
    try:
        psi_p, grads, master, m, v = _dist_case(numels, ws, bad_rank)
        S = psi_p // ws
        peers = SharedPeerBuffers(bufs, rank)
        peers.local.copy_(grads[rank])        # this rank's backward pass, into its own buffer
        st_in = [x[rank * S:(rank + 1) * S].clone() for x in (master, m, v)]
        st_out = [torch.full_like(x, float("nan")) for x in st_in]
        params = torch.zeros(psi_p, dtype=torch.float16)
        status = torch.zeros(1, dtype=torch.int32)
        step = DistZeroStep(psi_p, bucket, compute=_OracleCompute(), peers=peers)
        flag = step.step(peers.local, st_in, st_out, params, oracle.AdamHP(), 1, status)
        out.put((rank, int(flag.item()), int(status.item()), [x.numpy() for x in st_out],
                 params.numpy().view("uint16"), step._recv is None))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("ws,bucket,bad_rank", [(2, 0, -1), (3, 2500, -1), (3, 2500, 2)])
def test_distributed_step_peer_reads_gloo(ws, bucket, bad_rank):
    """The peer-read form of the distributed step: each rank writes its gradient into its own
    buffer, readable by every rank (here CPU tensors in memory the processes share, standing
    for NVLink peer mappings); per bucket a barrier, then each owner reduces its part straight
    from the peers' buffers -- no all-to-all, no receive buffers. Every rank's shard and full
    fp16 parameters equal the oracle's data-parallel step bit for bit; an inf on one rank
    skips the step everywhere."""
    import numpy as np
    import torch
    import oracle
    numels = [1000, 37, 4099, 12345]
    psi_p = -(-sum(numels) // ws) * ws
    bufs = [torch.zeros(psi_p, dtype=torch.float16).share_memory_() for _ in range(ws)]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker_dist_peer,
                         args=(r, ws, port, numels, bucket, bad_rank, bufs, q)) for r in range(ws)]
    for p in procs:
        p.start()
    try:
        res = sorted((q.get(timeout=240) for _ in range(ws)), key=lambda x: x[0])
    finally:
        for p in procs:
            p.join(60)
            if p.exitcode is None:
                p.kill()
    assert all(p.exitcode == 0 for p in procs)
    psi_p, grads, master, m, v = _dist_case(numels, ws, bad_rank)
    ref = oracle.dp_step([g.numpy() for g in grads], master.numpy(), m.numpy(), v.numpy(),
                         oracle.f2h(master.numpy()), oracle.AdamHP(), 1)
    S = psi_p // ws
    for rank, flag, status, shard, params, no_recv in res:
        assert no_recv
        assert flag == (1 if bad_rank >= 0 else 0)
        assert bool(status & 2) == ref.skipped == (bad_rank >= 0)
        for got, want in zip(shard, (ref.master, ref.m, ref.v)):
            assert np.array_equal(got.view(np.uint32),
                                  want[rank * S:(rank + 1) * S].view(np.uint32))
        assert np.array_equal(params, ref.params16)


def test_dist_bucket_map_matches_the_plan():
    """dist.py's bucket ranges and per-owner split sizes agree with the oracle's plan (backward
    order, element-granular, last bucket short) for several sizes, bucket lengths and Nd."""
    import oracle
    from zero_partitioned_optimizer_plan_b200.dist import bucket_ranges, owner_parts
    for numels, nd, bucket in [([1000, 37, 4099, 12345], 3, 2500), ([70001, 3], 4, 7),
                               ([300000, 250000, 250000, 248576], 4, 100000),
                               ([5, 5, 5], 2, 0), ([123457], 64, 1000)]:
        pl = oracle.plan(numels, nd, bucket)
        psi_p, S = pl.psi_p, pl.shard
        got = bucket_ranges(psi_p, bucket)
        want = [(lo, lo + ln) for lo, ln in pl.buckets]
        assert got == want
        for lo, hi in got:
            parts = owner_parts(lo, hi, S, nd)
            assert sum(parts) == hi - lo
            owned = [q for q in range(nd) if parts[q] > 0]
            assert owned == list(range(lo // S, (hi - 1) // S + 1))


@pytest.mark.parametrize("ws,bucket,bad_rank", [(2, 0, -1), (3, 2500, -1), (3, 2500, 2)])
def test_distributed_step_int8_payload_gloo(ws, bucket, bad_rank):
    """payload="q8": every rank quantizes its slice of each bucket for each owner (records
    counted from the owner's part), the all-to-all moves the records, the owner steps from the
    Nd payloads. Against the oracle's quantizer and int8 owner step over the same
    (bucket, owner) parts, bit for bit; an inf in one rank's gradient skips the step on every
    rank."""
    numels = [1000, 37, 4099, 12345]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker_dist,
                         args=(r, ws, port, numels, bucket, bad_rank, q, "q8"))
             for r in range(ws)]
    for p in procs:
        p.start()
    try:
        res = sorted((q.get(timeout=240) for _ in range(ws)), key=lambda x: x[0])
    finally:
        for p in procs:
            p.join(60)
            if p.exitcode is None:
                p.kill()
    assert all(p.exitcode == 0 for p in procs)
    _check_q8_result(res, numels, ws, bucket, bad_rank)


def _check_q8_result(res, numels, ws, bucket, bad_rank):
    """Every rank's shard and full fp16 parameters against the oracle's quantizer and int8
    owner step over the (bucket, owner) parts; one overflow skips the step everywhere."""
    import numpy as np
    import oracle
    from zero_partitioned_optimizer_plan_b200.dist import bucket_ranges
    psi_p, grads, master, m, v = _dist_case(numels, ws, bad_rank)
    S = psi_p // ws
    w, mm, vv = master.numpy().copy(), m.numpy().copy(), v.numpy().copy()
    p16 = oracle.f2h(master.numpy())
    skipped = False
    for lo, hi in bucket_ranges(psi_p, bucket):
        for o in range(ws):
            a, b = max(lo, o * S), min(hi, (o + 1) * S)
            if a >= b:
                continue
            pay = [oracle.quant_q8(g.numpy()[a:b]) for g in grads]
            sk, wn, mn, vn, pn = oracle.step_q8([x for x, _ in pay], [s for _, s in pay],
                                                w[a:b], mm[a:b], vv[a:b], oracle.AdamHP(), 1)
            skipped |= sk
            if not sk:
                w[a:b], mm[a:b], vv[a:b], p16[a:b] = wn, mn, vn, pn
    if skipped:
        w, mm, vv = master.numpy(), m.numpy(), v.numpy()
        p16 = oracle.f2h(master.numpy())
    assert skipped == (bad_rank >= 0)
    for rank, flag, status, shard, params in (x[:5] for x in res):
        assert flag == (1 if skipped else 0)
        assert bool(status & 2) == skipped
        for got, want in zip(shard, (w, mm, vv)):
            assert np.array_equal(got.view(np.uint32), want[rank * S:(rank + 1) * S].view(np.uint32))
        assert np.array_equal(params, p16)


def _worker_dist_q8_peer(rank, ws, port, numels, bucket, bad_rank, bufs, out):
    import datetime
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import oracle
    from zero_partitioned_optimizer_plan_b200.dist import DistZeroStep, SharedPeerBuffers
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=ws,
                            timeout=datetime.timedelta(seconds=60))
    try:
        psi_p, grads, master, m, v = _dist_case(numels, ws, bad_rank)
        S = psi_p // ws
        peers = SharedPeerBuffers(bufs, rank)
        st_in = [x[rank * S:(rank + 1) * S].clone() for x in (master, m, v)]
        st_out = [torch.full_like(x, float("nan")) for x in st_in]
        params = torch.zeros(psi_p, dtype=torch.float16)
        params[rank * S:(rank + 1) * S] = torch.from_numpy(
            oracle.f2h(st_in[0].numpy()).view("float16"))
        status = torch.zeros(1, dtype=torch.int32)
        step = DistZeroStep(psi_p, bucket, compute=_OracleCompute(), peers=peers, payload="q8")
        flag = step.step(grads[rank], st_in, st_out, params, oracle.AdamHP(), 1, status)
        out.put((rank, int(flag.item()), int(status.item()), [x.numpy() for x in st_out],
                 params.numpy().view("uint16"), step._recv is None and step._send is None))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("ws,bucket,bad_rank", [(2, 0, -1), (3, 2500, -1), (3, 2500, 0)])
def test_distributed_step_int8_peer_reads_gloo(ws, bucket, bad_rank):
    """The int8 peer-read form: each rank quantizes every (bucket, owner) part into its own
    buffer (CPU tensors shared by the processes, standing for NVLink peer mappings) at offsets
    every rank computes alike; per bucket a barrier, then the owner's int8 step reads the Nd
    payloads of its part in the peers' buffers -- no all-to-all, no send or receive buffers.
    The same results as the oracle's quantizer and int8 step over the parts, bit for bit."""
    import torch
    from zero_partitioned_optimizer_plan_b200.dist import q8_peer_bytes
    numels = [1000, 37, 4099, 12345]
    psi_p = -(-sum(numels) // ws) * ws
    nbytes = q8_peer_bytes(psi_p, bucket, ws)
    bufs = [torch.zeros(nbytes, dtype=torch.uint8).share_memory_() for _ in range(ws)]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker_dist_q8_peer,
                         args=(r, ws, port, numels, bucket, bad_rank, bufs, q))
             for r in range(ws)]
    for p in procs:
        p.start()
    try:
        res = sorted((q.get(timeout=240) for _ in range(ws)), key=lambda x: x[0])
    finally:
        for p in procs:
            p.join(60)
            if p.exitcode is None:
                p.kill()
    assert all(p.exitcode == 0 for p in procs)
    assert all(x[5] for x in res)          # nothing exchanged but the barriers
    _check_q8_result(res, numels, ws, bucket, bad_rank)


def test_q8_peer_layout_tiles_every_part():
    """The peer buffer's layout: one 16-byte-aligned segment per (bucket, owner) part, in
    order, each holding that part's records, none overlapping."""
    from zero_partitioned_optimizer_plan_b200.dist import (bucket_ranges, owner_parts,
                                                           q8_bytes, q8_peer_layout)
    for psi_p, bucket, nd in [(17481, 0, 1), (17484, 2500, 3), (10_000_000, 1_000_003, 8),
                              (4096, 128, 64 // 16)]:
        offs, total = q8_peer_layout(psi_p, bucket, nd)
        spans = []
        for k, (lo, hi) in enumerate(bucket_ranges(psi_p, bucket)):
            for q, x in enumerate(owner_parts(lo, hi, psi_p // nd, nd)):
                assert offs[k][q] % 16 == 0
                if x:
                    spans.append((offs[k][q], offs[k][q] + q8_bytes(x)))
        spans.sort()
        assert all(a[1] <= b[0] for a, b in zip(spans, spans[1:]))
        assert spans[-1][1] <= total


def _worker_dist_replicas(rank, ws, port, numels, bucket, bad_rank, gbufs, pbufs, fail_rank, out):
    import datetime
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import oracle
    from zero_partitioned_optimizer_plan_b200.dist import (DistStepError, DistZeroStep,
                                                           SharedPeerBuffers)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=ws,
                            timeout=datetime.timedelta(seconds=60))
    try:
        psi_p, grads, master, m, v = _dist_case(numels, ws, bad_rank)
        S = psi_p // ws
        peers = SharedPeerBuffers(gbufs, rank)
        peers.local.copy_(grads[rank])
        params = SharedPeerBuffers(pbufs, rank)
        st_in = [x[rank * S:(rank + 1) * S].clone() for x in (master, m, v)]
        st_out = [torch.full_like(x, float("nan")) for x in st_in]
        status = torch.zeros(1, dtype=torch.int32)
        step = DistZeroStep(psi_p, bucket, compute=_OracleCompute(fail=rank == fail_rank),
                            peers=peers, param_peers=params)
        raised = 0
        try:
            flag = int(step.step(peers.local, st_in, st_out, params.local, oracle.AdamHP(), 1,
                                 status).item())
        except DistStepError as e:
            flag, raised = e.bits, 1
        out.put((rank, flag, int(status.item()), [x.numpy() for x in st_out],
                 params.local.numpy().view("uint16").copy(), raised))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("ws,bucket,bad_rank,fail_rank", [(2, 0, -1, -1), (3, 2500, -1, -1),
                                                          (3, 2500, 1, -1), (3, 2500, -1, 2)])
def test_distributed_step_all_gather_in_epilogue_gloo(ws, bucket, bad_rank, fail_rank):
    """param_peers: each owner's step writes its fp16 values into every rank's full parameter
    buffer (CPU tensors shared by the processes, standing for NVLink peer mappings), with no
    all-gather collective. Every rank's full buffer equals the oracle's data-parallel step; an
    inf on one rank leaves fp16(master) in every replica (the commit repairs them all); a
    failure reported by one rank's kernels raises on every rank after the same repair."""
    import numpy as np
    import torch
    import oracle
    numels = [1000, 37, 4099, 12345]
    psi_p = -(-sum(numels) // ws) * ws
    _, _, master0, _, _ = _dist_case(numels, ws, bad_rank)
    p0 = torch.from_numpy(oracle.f2h(master0.numpy()).view(np.int16)).view(torch.float16)
    gbufs = [torch.zeros(psi_p, dtype=torch.float16).share_memory_() for _ in range(ws)]
    pbufs = [p0.clone().share_memory_() for _ in range(ws)]   # every replica starts at fp16(master)
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker_dist_replicas,
                         args=(r, ws, port, numels, bucket, bad_rank, gbufs, pbufs, fail_rank, q))
             for r in range(ws)]
    for p in procs:
        p.start()
    try:
        res = sorted((q.get(timeout=240) for _ in range(ws)), key=lambda x: x[0])
    finally:
        for p in procs:
            p.join(60)
            if p.exitcode is None:
                p.kill()
    assert all(p.exitcode == 0 for p in procs)
    psi_p, grads, master, m, v = _dist_case(numels, ws, bad_rank)
    ref = oracle.dp_step([g.numpy() for g in grads], master.numpy(), m.numpy(), v.numpy(),
                         oracle.f2h(master.numpy()), oracle.AdamHP(), 1)
    S = psi_p // ws
    void = ref.skipped or fail_rank >= 0
    for rank, flag, status, shard, params, raised in res:
        assert raised == (1 if fail_rank >= 0 else 0)
        assert bool(status & 2) == void
        want = (master.numpy(), m.numpy(), v.numpy()) if void else (ref.master, ref.m, ref.v)
        for got, w in zip(shard, want):
            assert np.array_equal(got.view(np.uint32), w[rank * S:(rank + 1) * S].view(np.uint32))
        assert np.array_equal(params, oracle.f2h(master.numpy()) if void else ref.params16)


S3_NUMELS = [1000, 37, 4099, 12345, 6000, 7]
S3_LAYERS = [1, 2, 1, 2]


def _worker_stage3(rank, ws, port, bad_rank, pbufs, gbufs, out, payload="fp16"):
    import datetime
    import numpy as np
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import oracle
    from zero_partitioned_optimizer_plan_b200.dist import DistStage3Step, SharedPeerBuffers
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=ws,
                            timeout=datetime.timedelta(seconds=60))
    try:
        psi_p, grads, master, m, v = _dist_case(S3_NUMELS, ws, bad_rank)
        S = psi_p // ws
        parts = SharedPeerBuffers(pbufs, rank)
        st_in = [x[rank * S:(rank + 1) * S].clone() for x in (master, m, v)]
        st_out = [torch.full_like(x, float("nan")) for x in st_in]
        status = torch.zeros(1, dtype=torch.int32)
        peers = None
        if gbufs is not None:      # gradients read in place from the peers' buffers
            peers = SharedPeerBuffers(gbufs, rank)
            if payload == "fp16":
                peers.local.copy_(grads[rank])
        step = DistStage3Step(S3_NUMELS, S3_LAYERS, parts, compute=_OracleCompute(), peers=peers,
                              payload=payload)
        big = max(hi - lo for lo, hi in step.layers)
        layer_buf = torch.zeros(big, dtype=torch.float16)
        rec = []
        local = peers.local if peers is not None and payload == "fp16" else grads[rank]
        flag = step.step(local, st_in, st_out, oracle.AdamHP(), 1, status, layer_buf, rec)
        dist.barrier()    # every owner's partition is final before it is read back
        out.put((rank, int(flag.item()), int(status.item()), [x.numpy() for x in st_out],
                 [p.numpy().view(np.uint16).copy() for p in parts.tensors],
                 [r.numpy().view(np.uint16) for r in rec]))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("peer", [False, True])
@pytest.mark.parametrize("ws,bad_rank", [(2, -1), (3, -1), (3, 1)])
def test_distributed_stage3_gloo(ws, bad_rank, peer):
    """DistStage3Step on gloo ranks, the partitions in CPU tensors shared by the processes
    (standing for NVLink peer mappings): every gathered layer (forward and backward), every
    owner's final partition and state shard equal the oracle's stage-3 step (zero3_step) bit
    for bit; an inf on one rank skips the step everywhere and leaves the partitions as they
    were."""
    import numpy as np
    import torch
    import oracle
    psi_p, grads, master, m, v = _dist_case(S3_NUMELS, ws, bad_rank)
    S = psi_p // ws
    p16 = oracle.f2h(master.numpy())
    pbufs = [torch.from_numpy(p16[q * S:(q + 1) * S].copy().view(np.int16)).view(torch.float16)
             .share_memory_() for q in range(ws)]
    gbufs = [torch.zeros(psi_p, dtype=torch.float16).share_memory_() for _ in range(ws)] \
        if peer else None
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker_stage3, args=(r, ws, port, bad_rank, pbufs, gbufs, q))
             for r in range(ws)]
    for p in procs:
        p.start()
    try:
        res = sorted((q.get(timeout=240) for _ in range(ws)), key=lambda x: x[0])
    finally:
        for p in procs:
            p.join(60)
            if p.exitcode is None:
                p.kill()
    assert all(p.exitcode == 0 for p in procs)
    pl = oracle.plan(S3_NUMELS, ws)
    layers = oracle.layer_ranges(pl, S3_LAYERS)
    buckets = oracle.grad_buckets(pl, layers)
    ref = oracle.zero3_step(pl, layers,
                            lambda l, j: grads[j].numpy()[buckets[l][0]:buckets[l][1]],
                            master.numpy(), m.numpy(), v.numpy(),
                            [p16[q * S:(q + 1) * S] for q in range(ws)], oracle.AdamHP(), 1)
    assert ref.skipped == (bad_rank >= 0)
    L = len(layers)
    for rank, flag, status, shard, parts, rec in res:
        assert flag == (1 if ref.skipped else 0)
        assert bool(status & 2) == ref.skipped
        for got, want in zip(shard, (ref.master, ref.m, ref.v)):
            assert np.array_equal(got.view(np.uint32), want[rank * S:(rank + 1) * S].view(np.uint32))
        for qq in range(ws):
            assert np.array_equal(parts[qq], ref.param_shards[qq].view(np.uint16))
        assert len(rec) == 2 * L
        for l in range(L):
            assert np.array_equal(rec[l], ref.gathered_fwd[l])
            assert np.array_equal(rec[L + (L - 1 - l)], ref.gathered_bwd[l])


@pytest.mark.parametrize("peer", [False, True])
@pytest.mark.parametrize("ws,bad_rank", [(2, -1), (3, 1)])
def test_distributed_stage3_int8_gloo(ws, bad_rank, peer):
    """DistStage3Step with the int8 payload on gloo ranks (the layers' gradient buckets
    exchanged, or read from the peers' buffers, as int8 records): every owner's partition and
    state shard against the oracle's quantizer and int8 step over the (layer bucket, owner)
    parts, bit for bit; an inf on one rank skips the step everywhere."""
    import numpy as np
    import torch
    import oracle
    from zero_partitioned_optimizer_plan_b200.dist import q8_peer_layout
    psi_p, grads, master, m, v = _dist_case(S3_NUMELS, ws, bad_rank)
    S = psi_p // ws
    p16 = oracle.f2h(master.numpy())
    pbufs = [torch.from_numpy(p16[q * S:(q + 1) * S].copy().view(np.int16)).view(torch.float16)
             .share_memory_() for q in range(ws)]
    pl = oracle.plan(S3_NUMELS, ws)
    layers = oracle.layer_ranges(pl, S3_LAYERS)
    buckets = oracle.grad_buckets(pl, layers)
    gbufs = None
    if peer:
        _, need = q8_peer_layout(psi_p, 0, ws, buckets[::-1])
        gbufs = [torch.zeros(need, dtype=torch.uint8).share_memory_() for _ in range(ws)]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker_stage3,
                         args=(r, ws, port, bad_rank, pbufs, gbufs, q, "q8"))
             for r in range(ws)]
    for p in procs:
        p.start()
    try:
        res = sorted((q.get(timeout=240) for _ in range(ws)), key=lambda x: x[0])
    finally:
        for p in procs:
            p.join(60)
            if p.exitcode is None:
                p.kill()
    assert all(p.exitcode == 0 for p in procs)
    w, mm, vv = master.numpy().copy(), m.numpy().copy(), v.numpy().copy()
    pw = p16.copy()
    skipped = False
    for lo, hi in buckets:
        for o in range(ws):
            a, b = max(lo, o * S), min(hi, (o + 1) * S)
            if a >= b:
                continue
            pay = [oracle.quant_q8(g.numpy()[a:b]) for g in grads]
            sk, wn, mn, vn, pn = oracle.step_q8([x for x, _ in pay], [c for _, c in pay],
                                                w[a:b], mm[a:b], vv[a:b], oracle.AdamHP(), 1)
            skipped |= sk
            if not sk:
                w[a:b], mm[a:b], vv[a:b], pw[a:b] = wn, mn, vn, pn
    if skipped:
        w, mm, vv, pw = master.numpy(), m.numpy(), v.numpy(), p16
    assert skipped == (bad_rank >= 0)
    for rank, flag, status, shard, parts, rec in res:
        assert flag == (1 if skipped else 0)
        assert bool(status & 2) == skipped
        for got, want in zip(shard, (w, mm, vv)):
            assert np.array_equal(got.view(np.uint32), want[rank * S:(rank + 1) * S].view(np.uint32))
        for qq in range(ws):
            assert np.array_equal(parts[qq], pw[qq * S:(qq + 1) * S].view(np.uint16))
