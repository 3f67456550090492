"""Seeded synthetic inputs for the ZeRO step (gradients and optimizer state).

This module holds none of the method's arithmetic: it only draws random numbers. Both the
CUDA path and the CPU oracle consume the bytes it returns; neither regenerates them.

Every draw is keyed by (seed, stream, rank, step): a splitmix64 hash of the key seeds a
fresh ``torch.Generator`` on the requested device, so any rank's gradient of any step can be
produced on its own. CPU and CUDA generators give different streams for the same key; a test
that compares the two paths always hands both the same materialised bytes (generated on the
CPU and uploaded, or generated on the GPU and gathered back at the sampled indices).

Distributions (as the workloads state them):
  gradients        N(0, sigma^2) rounded to fp16, optionally a fraction of elements x spike
  master weights   N(0, 0.02^2) or U(-0.05, 0.05), fp32
  momentum         0 or N(0, 1e-4^2), fp32
  variance         0 or |N(0, 1e-6^2)|, fp32
"""
from __future__ import annotations

import torch

_MASK64 = (1 << 64) - 1

STREAM_GRAD = 1
STREAM_MASTER = 2
STREAM_M = 3
STREAM_V = 4
STREAM_SPIKE = 5


def _splitmix64(x: int) -> int:
    x = (x + 0x9E3779B97F4A7C15) & _MASK64
    x = ((x ^ (x >> 30)) * 0xBF58476D1CE4E5B9) & _MASK64
    x = ((x ^ (x >> 27)) * 0x94D049BB133111EB) & _MASK64
    return x ^ (x >> 31)


def key(seed: int, stream: int, rank: int = 0, step: int = 0, chunk: int = 0) -> int:
    h = _splitmix64(seed & _MASK64)
    for part in (stream, rank, step, chunk):
        h = _splitmix64(h ^ (part & _MASK64))
    return h & ((1 << 63) - 1)


def _gen(device, k: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(k)
    return g


# Draws are made in chunks so that GPU-side generation of multi-GB buffers needs little extra
# memory; the chunk index is part of the key.
_CHUNK = 1 << 26


def grad_f16(n: int, sigma: float, *, seed: int = 0, rank: int = 0, step: int = 0,
             spike_frac: float = 0.0, spike_scale: float = 1.0, device="cpu",
             out: torch.Tensor | None = None) -> torch.Tensor:
    """One rank's local fp16 gradient: N(0, sigma^2), a spike_frac share of elements
    multiplied by spike_scale before the fp16 rounding."""
    if out is None:
        out = torch.empty(n, dtype=torch.float16, device=device)
    assert out.numel() == n and out.dtype == torch.float16
    dev = out.device
    for c, lo in enumerate(range(0, n, _CHUNK)):
        hi = min(n, lo + _CHUNK)
        x = torch.randn(hi - lo, dtype=torch.float32, device=dev,
                        generator=_gen(dev, key(seed, STREAM_GRAD, rank, step, c)))
        x.mul_(sigma)
        if spike_frac > 0.0:
            u = torch.rand(hi - lo, dtype=torch.float32, device=dev,
                           generator=_gen(dev, key(seed, STREAM_SPIKE, rank, step, c)))
            x = torch.where(u < spike_frac, x * spike_scale, x)
        out[lo:hi].copy_(x)
    return out


def normal_f32(n: int, sigma: float, *, seed: int = 0, stream: int = STREAM_MASTER,
               absolute: bool = False, device="cpu", out: torch.Tensor | None = None):
    if out is None:
        out = torch.empty(n, dtype=torch.float32, device=device)
    dev = out.device
    for c, lo in enumerate(range(0, n, _CHUNK)):
        hi = min(n, lo + _CHUNK)
        x = torch.randn(hi - lo, dtype=torch.float32, device=dev,
                        generator=_gen(dev, key(seed, stream, 0, 0, c)))
        x.mul_(sigma)
        if absolute:
            x.abs_()
        out[lo:hi].copy_(x)
    return out


def uniform_f32(n: int, lo_val: float, hi_val: float, *, seed: int = 0,
                stream: int = STREAM_MASTER, device="cpu", out: torch.Tensor | None = None):
    if out is None:
        out = torch.empty(n, dtype=torch.float32, device=device)
    dev = out.device
    for c, lo in enumerate(range(0, n, _CHUNK)):
        hi = min(n, lo + _CHUNK)
        x = torch.rand(hi - lo, dtype=torch.float32, device=dev,
                       generator=_gen(dev, key(seed, stream, 0, 0, c)))
        x.mul_(hi_val - lo_val).add_(lo_val)
        out[lo:hi].copy_(x)
    return out


def state_small(n: int, *, seed: int = 0, device="cpu"):
    """master N(0, 0.02^2), m = v = 0 (the tiny, GPT-2-small and 1.3B workloads)."""
    master = normal_f32(n, 0.02, seed=seed, stream=STREAM_MASTER, device=device)
    m = torch.zeros(n, dtype=torch.float32, device=device)
    v = torch.zeros(n, dtype=torch.float32, device=device)
    return master, m, v


def state_warm(n: int, *, seed: int = 0, device="cpu", out=None):
    """master U(-0.05, 0.05), m N(0, 1e-4^2), v |N(0, 1e-6^2)| (the 7.5B shard and the sweep)."""
    if out is None:
        out = [None, None, None]
    master = uniform_f32(n, -0.05, 0.05, seed=seed, stream=STREAM_MASTER, device=device,
                         out=out[0])
    m = normal_f32(n, 1e-4, seed=seed, stream=STREAM_M, device=device, out=out[1])
    v = normal_f32(n, 1e-6, seed=seed, stream=STREAM_V, absolute=True, device=device,
                   out=out[2])
    return master, m, v


# Parameter lists of the GPT-shaped workloads, in forward order (flatten order). The
# position embedding is not part of the listed tensors.
def gpt_param_list(vocab: int, hidden: int, layers: int, ffn: int):
    shapes = [vocab * hidden]                          # token embedding
    for _ in range(layers):
        shapes += [hidden, hidden,                     # ln1 weight, bias
                   hidden * 3 * hidden, 3 * hidden,    # qkv W, b
                   hidden * hidden, hidden,            # attention proj W, b
                   hidden, hidden,                     # ln2 weight, bias
                   hidden * ffn, ffn,                  # MLP fc W, b
                   ffn * hidden, hidden]               # MLP proj W, b
    shapes += [hidden, hidden]                         # final LayerNorm
    return shapes


def gpt_layer_tensors(layers: int):
    """How many consecutive tensors of gpt_param_list make up each layer, in forward order:
    the embedding, one transformer block (12 tensors) per layer, the final LayerNorm."""
    return [1] + [12] * layers + [2]


def gpt2_small_list():
    return gpt_param_list(50257, 768, 12, 3072)


def gpt2_small_layers():
    return gpt_layer_tensors(12)


def gpt_1p3b_list():
    return gpt_param_list(50257, 2048, 24, 8192)


def gpt_1p3b_layers():
    return gpt_layer_tensors(24)


TINY_LIST = [300000, 250000, 250000, 248576]
