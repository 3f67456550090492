"""The ZeRO stage-1/2 step across processes, one rank per GPU, over torch.distributed.

"ZeRO: particionar estados do treino entre GPUs" (upskillscore.com), "Como funciona": each of the
Nd ranks keeps 1/Nd of the optimizer state; gradients are reduce-scattered so that each
partition is reduced only on its owner, the owner updates its partition, and the updated fp16
parameters are all-gathered into every replica. "ZeRO-2" (llm-engineer.pages.dev), "Gradient
생명주기": the reduce-scatter goes bucket by bucket in backward order.

Here every rank is a process with its own full local fp16 gradient (psi_p values, the flat
padded list) and its own shard [r*S, (r+1)*S) of the fp32 master, m and v. A step:

  1. per bucket, in backward order: an all-to-all moves each rank's slice of the bucket that
     falls in owner q's shard to owner q; owner q receives the Nd slices in rank order;
  2. per bucket: the owner's fused step over its part of the bucket (the library's
     zero_step_fused: rank-ordered fp32 sum over the received rows, mean, unscale, Adam, fp16
     cast into its own range of the full parameter buffer) -- the reduction runs in the
     library kernel, not in the collective, so the sum order (rank 0 first) and hence every
     bit match the single-device step;
  3. one skip decision for the whole job: the overflow bit of every rank's status word is
     combined with an all-reduce (max), then each owner commits its shard (restoring it and
     its fp16 parameters if any rank overflowed);
  4. an all-gather of the fp16 shards into every rank's full parameter buffer.

The collectives are torch.distributed calls (NCCL on GPUs, gloo on CPUs); the arithmetic is the
library's. ``compute`` replaces the two library calls (the tests run the exchange on CPU
processes with another implementation of them).
"""
from __future__ import annotations

from typing import List, Sequence, Tuple

ZERO_FLAG_OVERFLOW = 0x1


def bucket_ranges(psi_p: int, bucket: int) -> List[Tuple[int, int]]:
    """Buckets of the flat padded list in backward order: [max(0, psi_p-(k+1)B), psi_p-kB)."""
    b = bucket if bucket > 0 else psi_p
    out, hi = [], psi_p
    while hi > 0:
        lo = max(0, hi - b)
        out.append((lo, hi))
        hi = lo
    return out


def owner_parts(lo: int, hi: int, shard: int, nd: int) -> List[int]:
    """Length of bucket [lo, hi) inside each owner's shard (the all-to-all split sizes)."""
    return [max(0, min(hi, (q + 1) * shard) - max(lo, q * shard)) for q in range(nd)]


class LibzeroCompute:
    """The owner's fused step and commit through the library (CUDA tensors)."""

    def __init__(self):
        from zero_partitioned_optimizer_plan_b200 import libzero
        self.lz = libzero

    def fused(self, n, rows, state_in, state_out, params, hp, t, status):
        self.lz.zero_step_fused(n, len(rows), rows, *state_in, *state_out, params, hp, t,
                                status)

    def commit(self, n, state_in, state_out, params, status):
        self.lz.zero_step_commit(n, *state_in, *state_out, params, status)


class DistZeroStep:
    """One rank's side of the distributed step. psi_p: the flat padded length (a multiple of
    the world size); bucket: elements per bucket (0: one bucket, stage 1)."""

    def __init__(self, psi_p: int, bucket: int = 0, group=None, compute=None):
        import torch.distributed as dist
        self.dist = dist
        self.group = group
        self.nd = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        if psi_p % self.nd:
            raise ValueError("psi_p must be a multiple of the world size")
        self.psi_p = psi_p
        self.shard = psi_p // self.nd
        self.buckets = bucket_ranges(psi_p, bucket)
        self.compute = compute or LibzeroCompute()

    def step(self, local_grad, state_in: Sequence, state_out: Sequence, params_full, hp,
             t: int, status):
        """local_grad: this rank's fp16 gradient (psi_p); state_in / state_out: this rank's
        fp32 master, m, v shards (S each, distinct buffers); params_full: the fp16 parameter
        buffer (psi_p), whose own range is updated and the rest gathered; status: this rank's
        zeroed int32 status word, which ends with the job-wide overflow bit and, if set, the
        skipped bit (every rank agrees). Returns the job-wide overflow flag (a one-element
        tensor on the status word's device; reading it waits for the step)."""
        import torch
        dist, nd, r, S = self.dist, self.nd, self.rank, self.shard
        own = params_full[r * S:(r + 1) * S]
        for lo, hi in self.buckets:
            parts = owner_parts(lo, hi, S, nd)
            mine = parts[r]
            recv = torch.empty(nd * mine, dtype=local_grad.dtype, device=local_grad.device)
            dist.all_to_all_single(recv, local_grad[lo:hi].contiguous(),
                                   output_split_sizes=[mine] * nd, input_split_sizes=parts,
                                   group=self.group)
            if mine == 0:
                continue
            a = max(lo, r * S) - r * S            # the bucket's part of my shard
            rows = [recv[j * mine:(j + 1) * mine] for j in range(nd)]
            self.compute.fused(mine, rows, [x[a:a + mine] for x in state_in],
                               [x[a:a + mine] for x in state_out], own[a:a + mine], hp, t,
                               status)
        flag = torch.bitwise_and(status, ZERO_FLAG_OVERFLOW)
        dist.all_reduce(flag, op=dist.ReduceOp.MAX, group=self.group)
        status.bitwise_or_(flag)
        self.compute.commit(S, state_in, state_out, own, status)
        dist.all_gather_into_tensor(params_full, own.clone(), group=self.group)
        return flag
