"""Seeded synthetic inputs for the NVFP4 linear-layer workloads.

This module only draws random numbers and rounds them to bf16 bit patterns; it
holds none of the quantization, transform or GEMM arithmetic.  Both the CPU
oracle tests and the CUDA parity tests / bench take their inputs from here, so
the two sides see identical bf16 bits.

Recipes (distributions and shapes of the workloads the pages describe):
  * linear 256^3 with outliers: N(0,1), each entry x50 with probability 1%.
  * quantize sweep 8192^2: N(0,1), Student-t(nu=3), Laplace(0,1), seeds 0/1/2.
  * 12B-class MLP up-projection: X ~ N(0,1) [8192x5120], W ~ N(0,0.02^2)
    [20480x5120], dY ~ N(0,1e-3^2) [8192x20480].
  * MoE: 64 experts, hidden 2048, expert FFN 1024, 16384 tokens, top-4 routing
    from Zipf(1.1) expert popularity.
  * GEMM sweep: N(0,1) square n^3 and skinny wgrad shapes.
"""
from __future__ import annotations

import numpy as np


def _rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(int(seed)))


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (nearest, ties to even); returns uint16 bits."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    bias = np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))
    return ((u + bias) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(
        np.float32)


def normal_bf16(shape, seed, std=1.0, outlier_prob=0.0, outlier_mult=50.0):
    rng = _rng(seed)
    z = rng.standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        z *= np.float32(std)
    if outlier_prob > 0.0:
        mask = rng.random(size=shape, dtype=np.float32) < np.float32(outlier_prob)
        z[mask] *= np.float32(outlier_mult)
    return f32_to_bf16_bits(z)


def student_t_bf16(shape, seed, nu=3.0):
    return f32_to_bf16_bits(_rng(seed).standard_t(nu, size=shape).astype(np.float32))


def laplace_bf16(shape, seed, scale=1.0):
    return f32_to_bf16_bits(_rng(seed).laplace(0.0, scale, size=shape).astype(np.float32))


def rht_signs(seed) -> np.ndarray:
    """16 random +-1 signs for the Hadamard rotation (int8)."""
    return (_rng(seed).integers(0, 2, size=16) * 2 - 1).astype(np.int8)


def moe_topk_ids(n_tokens=16384, n_experts=64, topk=4, zipf_s=1.1, seed=0) -> np.ndarray:
    """Experts of every token, [n_tokens, topk] int32: `topk` distinct experts drawn
    without replacement, expert e with probability proportional to (e+1)^-zipf_s
    (Gumbel top-k sampling)."""
    rng = _rng(seed)
    logp = -zipf_s * np.log(np.arange(1, n_experts + 1, dtype=np.float64))
    gumbel = rng.gumbel(size=(n_tokens, n_experts))
    return np.argsort(-(logp[None, :] + gumbel), axis=1)[:, :topk].astype(np.int32)


def moe_group_sizes(n_tokens=16384, n_experts=64, topk=4, zipf_s=1.1, seed=0) -> np.ndarray:
    """Tokens routed to each expert (no padding)."""
    ids = moe_topk_ids(n_tokens, n_experts, topk, zipf_s, seed)
    return np.bincount(ids.ravel(), minlength=n_experts).astype(np.int64)


def moe_layout(topk_ids: np.ndarray, n_experts: int, pad: int = 64):
    """Expert-contiguous row layout of the routed copies of every token.

    Returns (group_rows [E] int64, row_src [rows] int32, slots [T, topk] int32):
    expert e owns rows [off_e, off_e + group_rows[e]) (its tokens in token order,
    then zero rows up to a multiple of `pad`); row_src[i] is the token whose row
    lands at permuted row i (-1 for padding); slots[t, j] is the permuted row of
    the j-th routed copy of token t."""
    T, k = topk_ids.shape
    flat = topk_ids.ravel().astype(np.int64)
    counts = np.bincount(flat, minlength=n_experts).astype(np.int64)
    group_rows = (counts + pad - 1) // pad * pad
    offsets = np.concatenate([[0], np.cumsum(group_rows)[:-1]])
    order = np.argsort(flat, kind="stable")            # copies grouped by expert, token order
    expert_of = flat[order]
    first = np.concatenate([[0], np.cumsum(counts)[:-1]])
    rank_in_group = np.arange(flat.size) - first[expert_of]
    dest = offsets[expert_of] + rank_in_group
    row_src = np.full(int(group_rows.sum()), -1, dtype=np.int32)
    row_src[dest] = (order // k).astype(np.int32)
    slots = np.empty(flat.size, dtype=np.int32)
    slots[order] = dest.astype(np.int32)
    return group_rows, row_src, slots.reshape(T, k)


# Workload table: the shapes the parity tests and the bench use.
LINEAR_SMALL = dict(M=256, K=256, N=256)            # outlier case
MLP_12B = dict(M=8192, K=5120, N=20480)             # dense up-projection step
QUANT_SWEEP = dict(rows=8192, cols=8192)
MOE = dict(experts=64, hidden=2048, ffn=1024, tokens=16384, topk=4, zipf_s=1.1)


def moe_inputs(tokens, experts, hidden, ffn, topk, zipf_s, seed=0, pad=64):
    """Token activations X [T, hidden] ~ N(0,1), expert weights W [E, ffn, hidden] ~
    N(0, 0.02^2), routing, and the permuted output gradient dY [rows, ffn] ~ N(0,1)
    with zero padding rows."""
    ids = moe_topk_ids(tokens, experts, topk, zipf_s, seed)
    group_rows, row_src, slots = moe_layout(ids, experts, pad)
    X = normal_bf16((tokens, hidden), seed + 1)
    W = normal_bf16((experts, ffn, hidden), seed + 2, std=0.02)
    dY = normal_bf16((int(group_rows.sum()), ffn), seed + 3)
    dY[row_src < 0] = 0
    return dict(X=X, W=W, dY=dY, group_rows=group_rows, row_src=row_src, slots=slots, ids=ids)


GEMM_SQUARE = (1024, 2048, 4096, 8192, 16384)
GEMM_SKINNY_WGRAD = [(4096, 4096), (4096, 8192), (8192, 4096), (8192, 8192)]  # (N, K), red=32768


def mlp_inputs(M, K, N, seed=0):
    """X ~ N(0,1), W ~ N(0, 0.02^2), dY ~ N(0, 1e-3^2) as bf16 bits."""
    X = normal_bf16((M, K), seed)
    W = normal_bf16((N, K), seed + 1, std=0.02)
    dY = normal_bf16((M, N), seed + 2, std=1e-3)
    return X, W, dY


def linear_small_inputs(seed=0):
    s = LINEAR_SMALL
    X = normal_bf16((s["M"], s["K"]), seed, outlier_prob=0.01)
    W = normal_bf16((s["N"], s["K"]), seed + 1, outlier_prob=0.01)
    dY = normal_bf16((s["M"], s["N"]), seed + 2, outlier_prob=0.01)
    return X, W, dY


def device_bf16(kind, shape, seed, device, std=1.0):
    """Benchmark-scale inputs drawn on the GPU with torch's seeded generator (same
    distributions as the host recipes above, not the same values): kind "normal"
    N(0, std^2), "student_t" with nu = 3 (Z0 / sqrt((Z1^2 + Z2^2 + Z3^2) / 3)),
    "laplace" Laplace(0, 1) (the difference of two unit exponentials).  Drawn in
    fp32, rounded to bf16 (nearest, ties to even).  Parity tests use the host
    recipes; these only feed throughput measurements."""
    import torch

    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    if kind == "normal":
        z = torch.randn(shape, generator=g, device=device, dtype=torch.float32) * std
    elif kind == "student_t":
        z0 = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
        v = torch.zeros(shape, device=device, dtype=torch.float32)
        for _ in range(3):
            v += torch.randn(shape, generator=g, device=device, dtype=torch.float32) ** 2
        z = z0 / torch.sqrt(v / 3.0)
        del z0, v
    elif kind == "laplace":
        e1 = -torch.log1p(-torch.rand(shape, generator=g, device=device, dtype=torch.float32))
        e2 = -torch.log1p(-torch.rand(shape, generator=g, device=device, dtype=torch.float32))
        z = e1 - e2
        del e1, e2
    else:
        raise ValueError(kind)
    return z.to(torch.bfloat16)
