"""Seeded synthetic inputs shared by the tests, the smoke check and the benchmark.

This module draws random numbers and nothing else: it holds none of the
quantization arithmetic, so the CPU oracle and the CUDA path can both be fed
from it.  Every array is numpy; bf16 tensors are returned as ``uint16`` bit
patterns produced by torch's CPU bf16 cast (round to nearest even).

Workloads (shapes and distributions of the quantization pages' use cases):

* ``nvfp4_matrix``   -- [256, 2048] N(0,1), 1 % of entries x20 (outliers).
* ``expert_weights`` -- [E, N, K] N(0, 0.02^2) times a per-(expert,row) factor
  log-uniform in [0.5, 2], plus 16 exact-zero 32-blocks per expert.
* ``cache_acts``     -- [B, T, C] N(0,1) times a per-channel factor
  log-uniform in [0.1, 10] shared over B and T, and an independent N(0,1)
  gradient of the same shape.
* ``linear_weight``  -- [out, in] N(0, 0.01^2) with 0.1 % of entries x50.
* ``moe_problem``    -- activations [T, K] N(0,1), Zipf(1.1)-skewed routing
  over E experts with at least one empty expert (int32 cumulative ``offs``),
  expert weights [E, N, K] N(0, 0.02^2), and grad_out [T, N] N(0,1).

Seeds: workload i uses ``numpy.random.default_rng(20260000 + i)`` unless a
seed is given.
"""
from __future__ import annotations

import numpy as np
import torch

SEED_BASE = 20260000


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit patterns (uint16), round to nearest even (torch CPU cast)."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def _rng(seed, i):
    return np.random.default_rng(SEED_BASE + i if seed is None else seed)


def _scatter_outliers(rng, x: np.ndarray, frac: float, factor: float):
    flat = x.reshape(-1)
    n = int(round(frac * flat.size))
    if n:
        idx = rng.choice(flat.size, size=n, replace=False)
        flat[idx] *= factor
    return x


def nvfp4_matrix(rows=256, cols=2048, seed=None) -> np.ndarray:
    rng = _rng(seed, 1)
    x = rng.standard_normal((rows, cols), dtype=np.float32)
    _scatter_outliers(rng, x, 0.01, 20.0)
    return to_bf16_bits(x)


def expert_weights(E=8, N=2048, K=7168, zero_blocks=16, seed=None, block=32) -> np.ndarray:
    rng = _rng(seed, 2)
    w = rng.standard_normal((E, N, K), dtype=np.float32)
    w *= np.float32(0.02)
    lo, hi = np.log(0.5), np.log(2.0)
    w *= np.exp(rng.uniform(lo, hi, size=(E, N, 1))).astype(np.float32)
    nb = N * (K // block)
    for e in range(E):
        pick = rng.choice(nb, size=min(zero_blocks, nb), replace=False)
        for p in pick:
            r, b = divmod(int(p), K // block)
            w[e, r, b * block:(b + 1) * block] = 0.0
    return to_bf16_bits(w)


def cache_acts(B=4, T=8192, C=512, seed=None):
    rng = _rng(seed, 3)
    x = rng.standard_normal((B, T, C), dtype=np.float32)
    x *= np.exp(rng.uniform(np.log(0.1), np.log(10.0), size=(1, 1, C))).astype(np.float32)
    g = rng.standard_normal((B, T, C), dtype=np.float32)
    return to_bf16_bits(x), to_bf16_bits(g)


def linear_weight(out=7168, inp=18432, seed=None) -> np.ndarray:
    rng = _rng(seed, 4)
    w = rng.standard_normal((out, inp), dtype=np.float32)
    w *= np.float32(0.01)
    _scatter_outliers(rng, w, 0.001, 50.0)
    return to_bf16_bits(w)


def zipf_offs(rng, tokens: int, E: int, s: float = 1.1) -> np.ndarray:
    """int32 cumulative token counts: Zipf(s) expert popularity with ranks
    permuted, multinomial counts, and the smallest expert emptied into the
    largest so at least one expert has no tokens."""
    ranks = rng.permutation(E) + 1
    p = ranks.astype(np.float64) ** (-s)
    p /= p.sum()
    counts = rng.multinomial(tokens, p).astype(np.int64)
    lo, hi = int(np.argmin(counts)), int(np.argmax(counts))
    if lo == hi:
        hi = (lo + 1) % E
    counts[hi] += counts[lo]
    counts[lo] = 0
    return np.cumsum(counts).astype(np.int32)


def skew_offs(rng, kind: str, tokens: int, E: int) -> np.ndarray:
    """int32 cumulative token counts for a routing skew:
    "uniform"  every expert the same share (the remainder to the first ones);
    "zipf"     zipf_offs above (Zipf 1.1, one expert emptied);
    "hot"      one expert (seeded) holds half the tokens, the rest are spread
               uniformly at random over the others;
    "tiny"     half the experts get 1-16 tokens each (seeded), the other half
               share the rest evenly."""
    if kind == "zipf":
        return zipf_offs(rng, tokens, E)
    counts = np.zeros(E, np.int64)
    if kind == "uniform":
        counts[:] = tokens // E
        counts[: tokens - counts.sum()] += 1
    elif kind == "hot":
        h = int(rng.integers(0, E))
        counts[h] = tokens // 2
        rest = [e for e in range(E) if e != h]
        counts[rest] = rng.multinomial(tokens - counts[h], np.full(E - 1, 1.0 / (E - 1)))
    elif kind == "tiny":
        small = rng.permutation(E)[: E // 2]
        counts[small] = rng.integers(1, 17, small.size)
        big = np.setdiff1d(np.arange(E), small)
        left = tokens - counts.sum()
        counts[big] = left // big.size
        counts[big[: left - counts[big].sum()]] += 1
    else:
        raise ValueError(f"unknown routing skew {kind!r}")
    assert counts.sum() == tokens
    return np.cumsum(counts).astype(np.int32)


def moe_problem(T=16384, K=7168, N=2048, E=32, seed=None, with_weights=True):
    """Returns dict(x bf16 [T,K], offs int32 [E], w bf16 [E,N,K] or None, grad_out bf16 [T,N])."""
    rng = _rng(seed, 5)
    offs = zipf_offs(rng, T, E)
    x = to_bf16_bits(rng.standard_normal((T, K), dtype=np.float32))
    w = None
    if with_weights:
        wf = rng.standard_normal((E, N, K), dtype=np.float32)
        wf *= np.float32(0.02)
        w = to_bf16_bits(wf)
        del wf
    go = to_bf16_bits(rng.standard_normal((T, N), dtype=np.float32))
    return {"x": x, "offs": offs, "w": w, "grad_out": go}


# --------------------------------------------------------------------------
# Device-side variants for the benchmark: the same recipes drawn with torch's
# CUDA generator (same distributions and structure; different random numbers
# from the numpy variants above, which feed the parity tests).

def _bf16(t):
    return t.to(torch.bfloat16)


def nvfp4_matrix_torch(rows=256, cols=2048, generator=None, device="cuda"):
    x = torch.randn((rows, cols), generator=generator, device=device)
    n = int(round(0.01 * x.numel()))
    idx = torch.randperm(x.numel(), generator=generator, device=device)[:n]
    x.view(-1)[idx] *= 20.0
    return _bf16(x)


def expert_weights_torch(E=8, N=2048, K=7168, zero_blocks=16, generator=None, device="cuda", block=32):
    w = torch.randn((E, N, K), generator=generator, device=device)
    w *= 0.02
    lo, hi = float(np.log(0.5)), float(np.log(2.0))
    f = torch.empty((E, N, 1), device=device).uniform_(lo, hi, generator=generator).exp_()
    w *= f
    nb = N * (K // block)
    for e in range(E):
        pick = torch.randperm(nb, generator=generator, device=device)[:zero_blocks].tolist()
        for p in pick:
            r, b = divmod(int(p), K // block)
            w[e, r, b * block:(b + 1) * block] = 0.0
    return _bf16(w)


def cache_acts_torch(B=4, T=8192, C=512, generator=None, device="cuda"):
    x = torch.randn((B, T, C), generator=generator, device=device)
    f = torch.empty((1, 1, C), device=device).uniform_(float(np.log(0.1)), float(np.log(10.0)),
                                                       generator=generator).exp_()
    return _bf16(x * f)


def linear_weight_torch(out=7168, inp=18432, generator=None, device="cuda"):
    w = torch.randn((out, inp), generator=generator, device=device)
    w *= 0.01
    n = int(round(0.001 * w.numel()))
    idx = torch.randint(0, w.numel(), (n,), generator=generator, device=device)
    w.view(-1)[idx] *= 50.0
    return _bf16(w)
