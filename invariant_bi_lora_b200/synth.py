"""Seeded synthetic inputs shaped like the workloads of the LoRA / batch-invariance pages.

This module holds no arithmetic of the method: it only draws random numbers
(numpy PCG64, ``default_rng``) and stores them as fp32 or as bf16 bit patterns
(uint16; the float -> bf16 rounding is torch's round-to-nearest-even).  Both
the CUDA tests and the CPU oracle take their inputs from here.

Distribution notation N(mu, sigma): the second parameter is the standard
deviation.  Every array is drawn from its own generator, seeded with
``(seed, tag)``, so one array can be regenerated without the others.
"""
from __future__ import annotations

import numpy as np
import torch


def rng(seed: int, tag: int) -> np.random.Generator:
    return np.random.default_rng(np.random.SeedSequence([int(seed), int(tag)]))


def to_bf16_bits(values: np.ndarray) -> np.ndarray:
    """fp32/fp64 values -> bf16 bit patterns (uint16), torch's RNE rounding."""
    t = torch.from_numpy(np.ascontiguousarray(values, dtype=np.float32))
    return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def normal_f32(shape, std: float, mean: float = 0.0, seed: int = 0, tag: int = 0) -> np.ndarray:
    g = rng(seed, tag)
    return (g.standard_normal(shape, dtype=np.float32) * np.float32(std) + np.float32(mean))


def normal_bf16(shape, std: float, mean: float = 0.0, seed: int = 0, tag: int = 0) -> np.ndarray:
    return to_bf16_bits(normal_f32(shape, std, mean, seed, tag))


def integer_bf16(shape, lo: int, hi: int, seed: int = 0, tag: int = 0) -> np.ndarray:
    """Small integers in [lo, hi] as bf16 (exactly representable)."""
    g = rng(seed, tag)
    return to_bf16_bits(g.integers(lo, hi + 1, size=shape).astype(np.float32))


def integer_f32(shape, lo: int, hi: int, seed: int = 0, tag: int = 0) -> np.ndarray:
    g = rng(seed, tag)
    return g.integers(lo, hi + 1, size=shape).astype(np.float32)


def adapter_ids(M: int, n_adapters: int, seed: int = 0, tag: int = 7) -> np.ndarray:
    """Uniform random adapter id per token, int32 in [0, n_adapters)."""
    return rng(seed, tag).integers(0, n_adapters, size=M).astype(np.int32)


# ----------------------------------------------------------------------
# Workload recipes.  Tags keep each array's stream separate.
# ----------------------------------------------------------------------

TAG_X, TAG_A, TAG_B, TAG_W, TAG_IDS, TAG_NORMW, TAG_LOGITS = 1, 2, 3, 4, 7, 5, 6


def lora_inputs(M: int, K: int, r: int, n_adapters: int = 1, N: int = 0, seed: int = 0):
    """LoRA shrink / expand inputs.

    x  bf16 [M, K]            ~ N(0, 1)
    at bf16 [n_ad, r, K]      ~ N(0, 1/sqrt(K))   (A stored rank-major)
    bt bf16 [n_ad, N, r]      ~ N(0, 1/sqrt(r))   (LoRA-B, out x in layout)
    ids int32 [M]             uniform in [0, n_ad)
    """
    x = normal_bf16((M, K), 1.0, seed=seed, tag=TAG_X)
    at = normal_bf16((n_adapters, r, K), 1.0 / np.sqrt(K), seed=seed, tag=TAG_A)
    out = {"x": x, "at": at}
    if N:
        out["bt"] = normal_bf16((n_adapters, N, r), 1.0 / np.sqrt(r), seed=seed, tag=TAG_B)
    out["ids"] = adapter_ids(M, n_adapters, seed=seed, tag=TAG_IDS)
    return out


def gemm_inputs(M: int, N: int, K: int, seed: int = 0):
    """A bf16 [M, K] and W bf16 [N, K], both ~ N(0, 1/sqrt(K))."""
    a = normal_bf16((M, K), 1.0 / np.sqrt(K), seed=seed, tag=TAG_X)
    w = normal_bf16((N, K), 1.0 / np.sqrt(K), seed=seed, tag=TAG_W)
    return a, w


def rmsnorm_inputs(R: int, n: int = 4096, seed: int = 0):
    """x bf16 [R, n] ~ N(0, 1); weight bf16 [n] ~ N(1, 0.1)."""
    x = normal_bf16((R, n), 1.0, seed=seed, tag=TAG_X)
    w = normal_bf16((n,), 0.1, mean=1.0, seed=seed, tag=TAG_NORMW)
    return x, w


def logits_inputs(R: int, n: int = 151936, seed: int = 0):
    """fp32 logits [R, n] ~ N(0, 3)."""
    return normal_f32((R, n), 3.0, seed=seed, tag=TAG_LOGITS)
