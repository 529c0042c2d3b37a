"""Seeded synthetic inputs shared by the tests, the smoke check and the bench.

This module holds no arithmetic of the method (no quantization, packing or
matmul); it only draws inputs.  Values are drawn with numpy's PCG64 generator
(``np.random.default_rng([seed, stream])``, normal deviates in fp64) and
rounded to bf16, ties to even, straight from fp64.  Independent streams:
X = 1, W = 2, dY = 3, bias = 4.  Distributions follow the workloads the
pages benchmark: activations and output gradients N(0, 1), weights
N(0, 0.02), bias N(0, 0.01).

bf16 values are returned as numpy ``uint16`` bit patterns.
"""
from __future__ import annotations

import hashlib

import numpy as np

STREAM_X = 1
STREAM_W = 2
STREAM_DY = 3
STREAM_BIAS = 4

_CHUNK = 1 << 23


def f64_to_bf16_bits(v: np.ndarray) -> np.ndarray:
    """Round fp64 values to bf16 bit patterns, ties to even (finite inputs)."""
    v = np.asarray(v, dtype=np.float64)
    neg = np.signbit(v)
    a = np.abs(v)
    b = a.view(np.uint64)
    lsb = (b >> np.uint64(45)) & np.uint64(1)
    r = (b + np.uint64((1 << 44) - 1) + lsb) & ~np.uint64((1 << 45) - 1)
    rounded = r.view(np.float64)
    tiny = a < 2.0 ** -126
    if tiny.any():
        rounded = np.where(tiny, np.round(a * 2.0 ** 133) * 2.0 ** -133, rounded)
    with np.errstate(over="ignore"):
        f = rounded.astype(np.float32)
    out = (f.view(np.uint32) >> np.uint32(16)).astype(np.uint16)
    out[neg] |= np.uint16(0x8000)
    return out


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def normal_bf16(shape, mean: float, std: float, seed: int, stream: int) -> np.ndarray:
    """Seeded N(mean, std^2) values rounded to bf16 bits, shape ``shape``."""
    shape = tuple(int(d) for d in shape)
    n = int(np.prod(shape)) if shape else 1
    rng = np.random.default_rng([int(seed), int(stream)])
    out = np.empty(n, np.uint16)
    for lo in range(0, n, _CHUNK):
        hi = min(n, lo + _CHUNK)
        z = rng.standard_normal(hi - lo)
        out[lo:hi] = f64_to_bf16_bits(mean + std * z)
    return out.reshape(shape)


def config_seed(*key) -> int:
    """Seed of a workload: 0 for the tiny correctness case, else a hash of its key."""
    if not key:
        return 0
    h = hashlib.sha256(repr(key).encode()).digest()
    return int.from_bytes(h[:4], "little")


def activations(M: int, K: int, seed: int) -> np.ndarray:
    return normal_bf16((M, K), 0.0, 1.0, seed, STREAM_X)


def weights(N: int, K: int, seed: int) -> np.ndarray:
    return normal_bf16((N, K), 0.0, 0.02, seed, STREAM_W)


def grads(M: int, N: int, seed: int) -> np.ndarray:
    return normal_bf16((M, N), 0.0, 1.0, seed, STREAM_DY)


def bias(n: int, seed: int) -> np.ndarray:
    return normal_bf16((n,), 0.0, 0.01, seed, STREAM_BIAS)


def plant_structure(W: np.ndarray, g: int, seed: int) -> np.ndarray:
    """Copy of bf16 W with edge structure planted for tail coverage.

    Row 0 all zero; row 1 constant per group (alternating sign); one group
    of row 2 holds an outlier 50x the weight std; the last row is all
    positive (shifted by 0.1).  Needs N >= 4.
    """
    W = np.array(W, dtype=np.uint16, copy=True)
    N, K = W.shape
    rng = np.random.default_rng([int(seed), 99])
    W[0, :] = 0
    for gi in range(K // g):
        c = 0.015 * (1 if gi % 2 == 0 else -1)
        W[1, gi * g:(gi + 1) * g] = f64_to_bf16_bits(np.array([c]))[0]
    W[2, int(rng.integers(0, K))] = f64_to_bf16_bits(np.array([1.0]))[0]
    last = bf16_bits_to_f32(W[N - 1]).astype(np.float64)
    W[N - 1] = f64_to_bf16_bits(np.abs(last) + 0.1)
    return W


def offset_groups(W: np.ndarray, g: int, seed: int, share: float = 0.25, amp: float = 0.08) -> np.ndarray:
    """Copy of bf16 W where a seeded ``share`` of the g-long groups is shifted by an
    offset uniform in [-amp, amp] (groups that do not straddle zero, whose min-max
    zero point then lies far outside the code range)."""
    W = np.array(W, dtype=np.uint16, copy=True)
    N, K = W.shape
    rng = np.random.default_rng([int(seed), 55])
    G = K // g
    pick = rng.random((N, G)) < share
    off = rng.uniform(-amp, amp, (N, G)) * pick
    vals = bf16_bits_to_f32(W).astype(np.float64) + np.repeat(off, g, axis=1)
    return f64_to_bf16_bits(vals)


def outlier_activations(M: int, K: int, seed: int, exp: int, period: int = 128,
                        stream: int = STREAM_X) -> tuple[np.ndarray, np.ndarray]:
    """N(0, 1) bf16 rows with one entry of magnitude 2^exp (random sign) in every
    ``period`` consecutive entries, at a seeded position; returns (values, the
    outlier positions along the row).  Activation outliers of this kind are what
    decode-time LLM activations show."""
    A = normal_bf16((M, K), 0.0, 1.0, seed, stream)
    rng = np.random.default_rng([int(seed), 77])
    blocks = (K + period - 1) // period
    pos = np.minimum(np.arange(blocks) * period + rng.integers(0, period, blocks), K - 1)
    sign = np.where(rng.integers(0, 2, (M, blocks)) == 1, np.uint16(0x8000), np.uint16(0))
    big = f64_to_bf16_bits(np.array([2.0 ** exp]))[0]
    A[:, pos] = big | sign
    return A, pos


def mixed_range_activations(M: int, K: int, seed: int, lo_exp: int = -20, hi_exp: int = 4,
                            every: int = 8, stream: int = STREAM_X) -> tuple[np.ndarray, np.ndarray]:
    """bf16 rows mixing N(0, 2^(2 lo_exp)) values with N(0, 2^(2 hi_exp)) ones at a
    seeded one in ``every`` positions (the same positions in every row); returns
    (values, the large positions)."""
    rng = np.random.default_rng([int(seed), 78])
    z = rng.standard_normal((M, K))
    pos = np.flatnonzero(rng.integers(0, every, K) == 0)
    scale = np.full(K, 2.0 ** lo_exp)
    scale[pos] = 2.0 ** hi_exp
    return f64_to_bf16_bits(z * scale[None, :]), pos


def spread_rows(W: np.ndarray, seed: int, binades: int = 10) -> np.ndarray:
    """Copy of bf16 W with each row scaled by a seeded power of two in
    [2^(-binades/2), 2^(binades/2)], so that the rows' quantization scales
    spread over ``binades`` binades (exact: powers of two)."""
    rng = np.random.default_rng([int(seed), 79])
    e = rng.integers(-(binades // 2), binades // 2 + 1, W.shape[0])
    v = bf16_bits_to_f32(W).astype(np.float64) * (2.0 ** e)[:, None]
    return f64_to_bf16_bits(v)
