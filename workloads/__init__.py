"""Seeded synthetic inputs shaped like the pages' workloads.

This module only draws random inputs: it holds none of the NVFP4 arithmetic
(no quantisation, no GEMM, no routing gather). The CUDA path's tests, the
benchmark and the oracle's tests all draw their inputs from here, so both
sides always see the same tensors.

Workloads (GLM-5-style MoE layer: 256 experts, hidden 6144, intermediate 2048,
top-8; "Peering into the CUTLASS Kernel", Context: 256 experts, 16-64 tokens
per expert in decode; "Peering into the CUTLASS Kernel Scheduler", Context:
~16 tokens/expert at 512 concurrent requests, ~32 at 1024):

- ``tiny``: 4 experts x 16 rows, K = N = 256, plain epilogue.
- ``dense``: one 8192^3 GEMM (a single expert holding every row).
- ``moe_decode_t512``: 512 tokens, uniform top-8 routing (~16 rows/expert).
- ``moe_zipf_t1024``: 1024 tokens, expert popularity ~ rank^-1.1 over a seeded
  permutation; the two least popular experts get probability 0 so some experts
  are always empty.
- ``moe_prefill_t8192``: 8192 tokens, uniform top-8 routing (~256 rows/expert).

Values: activations N(0, 1), weights N(0, 0.02), drawn in FP32 and rounded to
BF16 (round-to-nearest-even). Router logits N(0, 1); uniform routing takes the
top-k logits (lower expert index wins ties) and softmax-renormalised weights
over the k chosen; Zipf routing takes the top-k of log p_e + Gumbel(0, 1)
(Gumbel-top-k sampling without replacement) with the same renormalised softmax.
"""
from __future__ import annotations

import numpy as np

CONFIGS = {
    "tiny": dict(kind="grouped", E=4, rows_per_expert=16, N=256, K=256, swiglu=False),
    "dense": dict(kind="dense", M=8192, N=8192, K=8192),
    "moe_decode_t512": dict(kind="moe", T=512, H=6144, I=2048, E=256, k=8, routing="uniform"),
    "moe_zipf_t1024": dict(kind="moe", T=1024, H=6144, I=2048, E=256, k=8, routing="zipf", zipf_s=1.1,
                           zero_experts=2),
    "moe_prefill_t8192": dict(kind="moe", T=8192, H=6144, I=2048, E=256, k=8, routing="uniform"),
}

ACT_STD = 1.0
WEIGHT_STD = 0.02

# Stream tags keep every tensor of a workload on its own seed.
TAG_ROUTER = 1
TAG_X = 2
TAG_W13 = 3
TAG_W2 = 4
TAG_A = 5
TAG_B = 6


def derive_seed(seed: int, tag: int, index: int = 0) -> int:
    return (int(seed) * 1_000_003 + int(tag) * 10_007 + int(index)) & 0x7FFF_FFFF_FFFF


def router_logits(T: int, E: int, kind: str = "uniform", seed: int = 0, zipf_s: float = 1.1,
                  zero_experts: int = 0) -> np.ndarray:
    """Router logits [T, E] (float64): N(0, 1) for uniform routing; log p_e + Gumbel(0, 1) for Zipf routing
    (experts with p_e = 0 get -inf)."""
    rng = np.random.Generator(np.random.PCG64(derive_seed(seed, TAG_ROUTER)))
    if kind == "uniform":
        return rng.standard_normal((T, E))
    if kind == "zipf":
        order = rng.permutation(E)                  # order[r] = expert with popularity rank r
        p = np.zeros(E)
        ranks = np.arange(1, E + 1, dtype=np.float64)
        p[order] = ranks ** (-zipf_s)
        if zero_experts:
            p[order[E - zero_experts:]] = 0.0
        p /= p.sum()
        with np.errstate(divide="ignore"):
            logp = np.log(p)
        gumbel = -np.log(-np.log(rng.uniform(np.finfo(np.float64).tiny, 1.0, size=(T, E))))
        return logp[None, :] + gumbel
    raise ValueError(kind)


def routing(T: int, E: int, k: int, kind: str = "uniform", seed: int = 0, zipf_s: float = 1.1,
            zero_experts: int = 0):
    """Return (topk_ids int32 [T, k], topk_w float32 [T, k]) drawn on the host from router_logits()."""
    z = router_logits(T, E, kind, seed, zipf_s, zero_experts)
    ids = np.argsort(-z, axis=1, kind="stable")[:, :k].astype(np.int32)
    zs = np.take_along_axis(z, ids, axis=1)
    zs = zs - zs.max(axis=1, keepdims=True)
    w = np.exp(zs)
    w = (w / w.sum(axis=1, keepdims=True)).astype(np.float32)
    return ids, w


def config_routing(name: str, seed: int = 0):
    c = CONFIGS[name]
    return routing(c["T"], c["E"], c["k"], c["routing"], seed, c.get("zipf_s", 1.1), c.get("zero_experts", 0))


def normal_bf16(shape, std: float, seed: int, tag: int, index: int = 0, device="cpu"):
    """N(0, std) drawn in FP32 by torch's generator on `device`, rounded to BF16."""
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(derive_seed(seed, tag, index))
    x = torch.randn(tuple(shape), generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    return x.to(torch.bfloat16)


def bf16_bits(t) -> np.ndarray:
    """torch BF16 tensor -> numpy uint16 bit patterns (host copy)."""
    import torch
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def random_bf16_bits(shape, seed: int, std: float = 1.0, tag: int = 99) -> np.ndarray:
    """Host-side BF16 bit patterns of N(0, std) samples (small test inputs)."""
    return bf16_bits(normal_bf16(shape, std, seed, tag))
