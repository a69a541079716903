"""Seeded synthetic inputs shaped like DeepSeek-R1 / Qwen3-8B linear layers.

This module only draws random numbers and stores them in the input formats
the method consumes (bf16 activations and weights, fp16 decode activations,
FP8-E4M3 checkpoint bytes with fp32 128x128 block scales, int8 weights with
fp16 group scales).  It holds none of the quantization or GEMM arithmetic:
both the CUDA path and the CPU oracle take their inputs from here, and
neither is imported by it.

Random source: numpy's PCG64 (``numpy.random.default_rng``), seeded with
``seed * 2 + stream`` so that X (stream 0) and W (stream 1) of one workload
are independent.  Float-format conversions use torch's CPU casts, which
round to nearest even.

Outliers ("0.1% of entries x50"): each entry is independently selected with
probability ``outlier_p`` and multiplied by ``outlier_mult`` before the cast.
"""
from __future__ import annotations

import numpy as np
import torch

STREAM_X = 0
STREAM_W = 1


def _rng(seed: int, stream: int) -> np.random.Generator:
    return np.random.default_rng(seed * 2 + stream)


def _f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def _f32_to_f16_bits(a: np.ndarray) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float32).astype(np.float16).view(np.uint16)


def activation_bf16(M: int, K: int, seed: int, outlier_p: float = 0.001,
                    outlier_mult: float = 50.0, sigma: float = 1.0,
                    stream: int = STREAM_X) -> np.ndarray:
    """X ~ N(0, sigma) with Bernoulli(outlier_p) entries scaled by outlier_mult; bf16 bits [M, K]."""
    rng = _rng(seed, stream)
    x = rng.standard_normal((M, K), dtype=np.float32)
    if sigma != 1.0:
        x *= np.float32(sigma)
    if outlier_p > 0:
        sel = rng.random((M, K), dtype=np.float32) < outlier_p
        x[sel] *= np.float32(outlier_mult)
    return _f32_to_bf16_bits(x)


def weight_bf16(N: int, K: int, seed: int, sigma: float = 0.02,
                stream: int = STREAM_W) -> np.ndarray:
    """W ~ N(0, sigma); bf16 bits [N, K]."""
    rng = _rng(seed, stream)
    w = rng.standard_normal((N, K), dtype=np.float32)
    w *= np.float32(sigma)
    return _f32_to_bf16_bits(w)


def fp8_checkpoint(N: int, K: int, seed: int, sigma: float = 0.02,
                   scale_lo: float = 1e-4, scale_hi: float = 1e-2,
                   stream: int = STREAM_W):
    """A DeepSeek-style FP8 checkpoint tensor.

    Block scales sf[nb, kb] ~ U(scale_lo, scale_hi) (fp32, one per 128x128
    block, ceil-divided shape); bytes = E4M3(N(0, sigma) / sf), where the
    value is first clamped to the format's finite range +-448 (torch's cast
    does not saturate on its own).  Returns (e4m3 bytes uint8 [N, K],
    sf float32 [ceil(N/128), ceil(K/128)]).
    """
    rng = _rng(seed, stream)
    nb, kb = -(-N // 128), -(-K // 128)
    sf = rng.uniform(scale_lo, scale_hi, size=(nb, kb)).astype(np.float32)
    w = rng.standard_normal((N, K), dtype=np.float32)
    w *= np.float32(sigma)
    rows = np.arange(N) // 128
    for b in range(kb):
        cols = slice(b * 128, min(K, (b + 1) * 128))
        w[:, cols] /= sf[rows, b][:, None]
    np.clip(w, -448.0, 448.0, out=w)
    t = torch.from_numpy(w).to(torch.float8_e4m3fn)
    return t.view(torch.uint8).numpy(), sf


def activation_f16(M: int, K: int, seed: int, sigma: float = 1.0,
                   stream: int = STREAM_X) -> np.ndarray:
    """Decode activations X ~ N(0, sigma); fp16 bits [M, K]."""
    rng = _rng(seed, stream)
    x = rng.standard_normal((M, K), dtype=np.float32)
    if sigma != 1.0:
        x *= np.float32(sigma)
    return _f32_to_f16_bits(x)


def int8_weight_groups(N: int, K: int, seed: int, group: int = 128,
                       sigma: float = 0.02, stream: int = STREAM_W, scale_fmt: str = "fp16"):
    """A stored symmetric group-wise INT8 weight (W8A16 checkpoint format).

    Codes are drawn directly as integers: a rounded N(0, 42) clipped to
    +-127, with one entry per group forced to +-127 as a symmetric absmax
    quantizer would leave it.  Group scales are fp16 (or, with
    scale_fmt="bf16", bf16) values of U(2.5*sigma, 4.5*sigma) / 127, i.e. the
    scale an absmax quantizer gives a N(0, sigma) group.
    Returns (wq int8 [N, K], s fp16 / bf16 bits [N, K/group]).
    """
    assert K % group == 0
    rng = _rng(seed, stream)
    g = K // group
    q = np.clip(np.rint(rng.normal(0.0, 42.0, size=(N, K))), -127, 127).astype(np.int8)
    pos = rng.integers(0, group, size=(N, g))
    sign = np.where(rng.random((N, g)) < 0.5, -127, 127).astype(np.int8)
    qv = q.reshape(N, g, group)
    qv[np.arange(N)[:, None], np.arange(g)[None, :], pos] = sign
    s = rng.uniform(2.5 * sigma, 4.5 * sigma, size=(N, g)).astype(np.float32) / np.float32(127.0)
    return q, (_f32_to_bf16_bits(s) if scale_fmt == "bf16" else _f32_to_f16_bits(s))


def activation_bf16_plain(M: int, K: int, seed: int, sigma: float = 1.0, stream: int = STREAM_X) -> np.ndarray:
    """Activations X ~ N(0, sigma) without outliers (bf16 W8A16 inputs); bf16 bits [M, K]."""
    return activation_bf16(M, K, seed, outlier_p=0.0, sigma=sigma, stream=stream)


def token_counts(E: int, total: int, seed: int, stream: int = STREAM_X) -> np.ndarray:
    """Per-expert token counts for a grouped (MoE) GEMM: a seeded multinomial split of ``total``."""
    rng = _rng(seed, stream)
    p = rng.dirichlet(np.full(E, 0.7))
    return rng.multinomial(total, p).astype(np.int64)
