"""The distributed step (dist.py) on the GPU through NCCL and the library's kernels, with the one
rank a single-GPU run allows (the all-to-all, all-reduce and all-gather then move data only
within the rank); the exchange between several ranks is tested on CPU processes over gloo
(test_multirank.py). Against the oracle's data-parallel step, tolerances as in
test_gpu_parity.py."""
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

pytestmark = pytest.mark.gpu


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _case(numels):
    import torch
    from zero_partitioned_optimizer_plan_b200 import synth
    psi = sum(numels)
    grad = synth.grad_f16(psi, 1e-3, seed=11, rank=0, step=1)
    master, m, v = synth.state_warm(psi, seed=12)
    return psi, grad, master, m, v, torch


def _worker(port, numels, bucket, out, peer=False, payload="fp16", replicas=False):
    import datetime
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    from zero_partitioned_optimizer_plan_b200 import libzero as lz
    from zero_partitioned_optimizer_plan_b200.dist import DistZeroStep
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    torch.cuda.set_device(0)
    dist.init_process_group("nccl", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60),
                            device_id=torch.device("cuda", 0))
    try:
        psi, grad, master, m, v, _ = _case(numels)
        dev = "cuda:0"
        st_in = [x.to(dev) for x in (master, m, v)]
        st_out = [torch.full_like(x, float("nan")) for x in st_in]
        params = torch.zeros(psi, dtype=torch.float16, device=dev)
        status = torch.zeros(1, dtype=torch.int32, device=dev)
        if replicas:   # the fp16 write-back stored by the kernel into symmetric memory
            from zero_partitioned_optimizer_plan_b200.dist import SymmetricPeerBuffers
            pp = SymmetricPeerBuffers(psi, torch.float16, dev)
            pp.local.zero_()
            gpeers = None
            if peer:
                gpeers = SymmetricPeerBuffers(psi, torch.float16, dev)
                gpeers.local.copy_(grad.to(dev))
            step = DistZeroStep(psi, bucket, peers=gpeers, param_peers=pp)
            flag = step.step(gpeers.local if peer else grad.to(dev), st_in, st_out, pp.local,
                             lz.AdamHP(), 1, status)
            params = pp.local
        elif peer and payload == "q8":   # int8 records quantized into symmetric memory
            from zero_partitioned_optimizer_plan_b200.dist import (SymmetricPeerBuffers,
                                                                   q8_peer_bytes)
            peers = SymmetricPeerBuffers(q8_peer_bytes(psi, bucket, 1), torch.uint8, dev)
            step = DistZeroStep(psi, bucket, peers=peers, payload="q8")
            flag = step.step(grad.to(dev), st_in, st_out, params, lz.AdamHP(), 1, status)
        elif peer:    # gradients produced into symmetric memory; the owner reads them in place
            from zero_partitioned_optimizer_plan_b200.dist import SymmetricPeerBuffers
            peers = SymmetricPeerBuffers(psi, torch.float16, dev)
            peers.local.copy_(grad.to(dev))
            step = DistZeroStep(psi, bucket, peers=peers)
            flag = step.step(peers.local, st_in, st_out, params, lz.AdamHP(), 1, status)
        else:
            step = DistZeroStep(psi, bucket, payload=payload)
            flag = step.step(grad.to(dev), st_in, st_out, params, lz.AdamHP(), 1, status)
        torch.cuda.synchronize()
        out.put((int(flag.item()), int(status.item()), [x.cpu().numpy() for x in st_out],
                 params.cpu().numpy().view(np.uint16)))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("peer", [False, True])
@pytest.mark.parametrize("bucket", [0, 3000])
def test_distributed_step_one_rank_nccl(bucket, peer):
    """The all-to-all form and the peer-read form (the rank's gradient in torch symmetric
    memory, read by the owner's kernel through its symmetric address)."""
    import oracle
    numels = [1000, 37, 4099, 12345]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    p = ctx.Process(target=_worker, args=(_free_port(), numels, bucket, q, peer))
    p.start()
    try:
        flag, status, shard, params = q.get(timeout=240)
    finally:
        p.join(60)
        if p.exitcode is None:
            p.kill()
    assert p.exitcode == 0
    psi, grad, master, m, v, _ = _case(numels)
    ref = oracle.dp_step([grad.numpy()], master.numpy(), m.numpy(), v.numpy(),
                         oracle.f2h(master.numpy()), oracle.AdamHP(), 1)
    assert (flag, status) == (0, 0) and not ref.skipped
    for name, got, want in zip(("master", "m", "v"), shard, (ref.master, ref.m, ref.v)):
        d = oracle.ulp_diff_f32(got, want)
        assert int(d.max()) <= 2, name
    assert int(oracle.ulp_diff_f16(params, ref.params16).max()) <= 1


@pytest.mark.parametrize("peer", [False, True])
@pytest.mark.parametrize("bucket", [0, 3000])
def test_distributed_step_int8_payload_one_rank_nccl(bucket, peer):
    """payload="q8" on one NCCL rank: the library's quantizer fills the send buffer, the
    all-to-all moves the records, the library's int8 step runs on the received payloads (or,
    peer-read form, the quantizer writes into torch symmetric memory and the int8 step reads
    the payloads there); against the oracle's quantizer and int8 step per bucket (0 ulp)."""
    import oracle
    from zero_partitioned_optimizer_plan_b200.dist import bucket_ranges
    numels = [1000, 37, 4099, 12345]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    p = ctx.Process(target=_worker, args=(_free_port(), numels, bucket, q, peer, "q8"))
    p.start()
    try:
        flag, status, shard, params = q.get(timeout=240)
    finally:
        p.join(60)
        if p.exitcode is None:
            p.kill()
    assert p.exitcode == 0
    psi, grad, master, m, v, _ = _case(numels)
    w, mm, vv = master.numpy().copy(), m.numpy().copy(), v.numpy().copy()
    p16 = oracle.f2h(master.numpy())
    for lo, hi in bucket_ranges(psi, bucket):
        qq, sc = oracle.quant_q8(grad.numpy()[lo:hi])
        skipped, w[lo:hi], mm[lo:hi], vv[lo:hi], p16[lo:hi] = oracle.step_q8(
            [qq], [sc], w[lo:hi], mm[lo:hi], vv[lo:hi], oracle.AdamHP(), 1)
        assert not skipped
    assert (flag, status) == (0, 0)
    for name, got, want in zip(("master", "m", "v"), shard, (w, mm, vv)):
        assert int(oracle.ulp_diff_f32(got, want).max()) == 0, name
    assert int(oracle.ulp_diff_f16(params, p16).max()) == 0


@pytest.mark.parametrize("peer", [False, True])
@pytest.mark.parametrize("bucket", [0, 3000])
def test_distributed_step_all_gather_in_epilogue_one_rank_nccl(bucket, peer):
    """param_peers on one NCCL rank: the owner's kernel stores the fp16 values into the full
    parameter buffer in torch symmetric memory (no all-gather collective), the gradients
    exchanged by all-to-all or read in place from symmetric memory; against the oracle's
    data-parallel step."""
    import oracle
    numels = [1000, 37, 4099, 12345]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    p = ctx.Process(target=_worker, args=(_free_port(), numels, bucket, q, peer, "fp16", True))
    p.start()
    try:
        flag, status, shard, params = q.get(timeout=240)
    finally:
        p.join(60)
        if p.exitcode is None:
            p.kill()
    assert p.exitcode == 0
    psi, grad, master, m, v, _ = _case(numels)
    ref = oracle.dp_step([grad.numpy()], master.numpy(), m.numpy(), v.numpy(),
                         oracle.f2h(master.numpy()), oracle.AdamHP(), 1)
    assert (flag, status) == (0, 0) and not ref.skipped
    for name, got, want in zip(("master", "m", "v"), shard, (ref.master, ref.m, ref.v)):
        assert int(oracle.ulp_diff_f32(got, want).max()) == 0, name
    assert int(oracle.ulp_diff_f16(params, ref.params16).max()) == 0


def _worker_stage3(port, numels, layer_tensors, out, payload="fp16"):
    import datetime
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import oracle
    from zero_partitioned_optimizer_plan_b200 import libzero as lz
    from zero_partitioned_optimizer_plan_b200.dist import DistStage3Step, SymmetricPeerBuffers
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    torch.cuda.set_device(0)
    dist.init_process_group("nccl", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60),
                            device_id=torch.device("cuda", 0))
    try:
        psi, grad, master, m, v, _ = _case(numels)
        dev = "cuda:0"
        parts = SymmetricPeerBuffers(psi, torch.float16, dev)
        parts.local.copy_(torch.from_numpy(oracle.f2h(master.numpy()).view("float16")).to(dev))
        st_in = [x.to(dev) for x in (master, m, v)]
        st_out = [torch.full_like(x, float("nan")) for x in st_in]
        status = torch.zeros(1, dtype=torch.int32, device=dev)
        step = DistStage3Step(numels, layer_tensors, parts, payload=payload)
        layer_buf = torch.zeros(max(hi - lo for lo, hi in step.layers), dtype=torch.float16,
                                device=dev)
        rec = []
        flag = step.step(grad.to(dev), st_in, st_out, lz.AdamHP(), 1, status, layer_buf, rec)
        torch.cuda.synchronize()
        out.put((int(flag.item()), int(status.item()), [x.cpu().numpy() for x in st_out],
                 parts.local.cpu().numpy().view(np.uint16),
                 [r.cpu().numpy().view(np.uint16) for r in rec]))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("payload", ["fp16", "q8"])
def test_distributed_stage3_one_rank_nccl(payload):
    """DistStage3Step on one NCCL rank: the partition in torch symmetric memory, each layer
    gathered by the library's gather kernel from the owner's partition address, the layers'
    gradient buckets exchanged (fp16, or int8 records quantized by the library) and the owner's
    update written into its partition; gathered layers, partition and state against the
    oracle's zero3_step, or its quantizer and int8 step per bucket (0 ulp)."""
    import oracle
    numels, layer_tensors = [1000, 37, 4099, 12345], [1, 2, 1]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    p = ctx.Process(target=_worker_stage3, args=(_free_port(), numels, layer_tensors, q, payload))
    p.start()
    try:
        flag, status, shard, part, rec = q.get(timeout=240)
    finally:
        p.join(60)
        if p.exitcode is None:
            p.kill()
    assert p.exitcode == 0
    psi, grad, master, m, v, _ = _case(numels)
    pl = oracle.plan(numels, 1)
    layers = oracle.layer_ranges(pl, layer_tensors)
    buckets = oracle.grad_buckets(pl, layers)
    ref = oracle.zero3_step(pl, layers, lambda l, j: grad.numpy()[buckets[l][0]:buckets[l][1]],
                            master.numpy(), m.numpy(), v.numpy(),
                            [oracle.f2h(master.numpy())], oracle.AdamHP(), 1)
    assert (flag, status) == (0, 0) and not ref.skipped
    want_state, want_part = (ref.master, ref.m, ref.v), ref.param_shards[0]
    if payload == "q8":                  # one owner: each layer bucket is one int8 part
        w, mm, vv = master.numpy().copy(), m.numpy().copy(), v.numpy().copy()
        p16 = oracle.f2h(master.numpy())
        for lo, hi in buckets:
            qq, sc = oracle.quant_q8(grad.numpy()[lo:hi])
            sk, w[lo:hi], mm[lo:hi], vv[lo:hi], p16[lo:hi] = oracle.step_q8(
                [qq], [sc], w[lo:hi], mm[lo:hi], vv[lo:hi], oracle.AdamHP(), 1)
            assert not sk
        want_state, want_part = (w, mm, vv), p16
    for name, got, want in zip(("master", "m", "v"), shard, want_state):
        assert int(oracle.ulp_diff_f32(got, want).max()) == 0, name
    assert int(oracle.ulp_diff_f16(part, want_part).max()) == 0
    L = len(layers)
    for l in range(L):
        assert np.array_equal(rec[l], ref.gathered_fwd[l])
        assert np.array_equal(rec[L + (L - 1 - l)], ref.gathered_bwd[l])
