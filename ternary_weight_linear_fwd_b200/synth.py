"""Seeded synthetic inputs for the BitLinear workloads.

This module only draws random numbers; it holds none of the forward pass's
arithmetic.  Both the CUDA path and the oracle receive the arrays it makes.

Generator: SplitMix64 used as a counter-based stream (Steele, Lea and Flood,
"Fast splittable pseudorandom number generators", OOPSLA 2014): value i of
stream s is mix64(key(seed, s) + (i + 1) * 0x9E3779B97F4A7C15), where mix64
is the SplitMix64 finaliser.  Uniforms take the top 53 bits; normals use the
Box-Muller transform in fp64.

Workload recipes (the pages' layer shapes; trained weights are not available,
so magnitudes follow the stated distributions):
  * latent weights   W ~ N(0, 0.02) fp32
  * activations      x ~ N(0, 1), each entry x10 with probability 1%, bf16
  * direct ternary   P(0) = 0.42, P(+1) = P(-1) = 0.29, alpha ~ U(0.01, 0.05)
"""
from __future__ import annotations

import numpy as np

_GOLDEN = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)


def _mix64(z: np.ndarray) -> np.ndarray:
    z = (z ^ (z >> np.uint64(30))) * _M1
    z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def _key(seed: int, stream: int) -> np.uint64:
    with np.errstate(over="ignore"):
        base = np.array([np.uint64(seed & 0xFFFFFFFFFFFFFFFF)], dtype=np.uint64)
        k = _mix64(base ^ np.uint64((stream * 0xD1B54A32D192ED03) & 0xFFFFFFFFFFFFFFFF))
    return k[0]


def splitmix64(seed: int, stream: int, count: int) -> np.ndarray:
    """count uint64 values of stream ``stream`` under ``seed``."""
    with np.errstate(over="ignore"):
        i = np.arange(1, count + 1, dtype=np.uint64)
        return _mix64(_key(seed, stream) + i * _GOLDEN)


def uniform(seed: int, stream: int, count: int) -> np.ndarray:
    """fp64 uniforms in [0, 1)."""
    return (splitmix64(seed, stream, count) >> np.uint64(11)).astype(np.float64) * (2.0 ** -53)


def normal(seed: int, stream: int, count: int) -> np.ndarray:
    """fp64 standard normals (Box-Muller on consecutive uniform pairs)."""
    half = (count + 1) // 2
    u = uniform(seed, stream, 2 * half)
    u1, u2 = u[0::2], u[1::2]
    r = np.sqrt(-2.0 * np.log1p(-u1))
    th = 2.0 * np.pi * u2
    z = np.empty(2 * half, dtype=np.float64)
    z[0::2] = r * np.cos(th)
    z[1::2] = r * np.sin(th)
    return z[:count]


def to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round fp32 values to the nearest bf16 (ties to even); returns uint16 bit patterns."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = (u + np.uint64(0x7FFF) + ((u >> np.uint64(16)) & np.uint64(1))) >> np.uint64(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


# ---------------------------------------------------------------------------
# Workload inputs
# ---------------------------------------------------------------------------

def latent_weights(N: int, K: int, seed: int, sigma: float = 0.02, stream: int = 1) -> np.ndarray:
    """fp32 [N, K] latent weights ~ N(0, sigma)."""
    return (normal(seed, stream, N * K) * sigma).astype(np.float32).reshape(N, K)


def activations(M: int, K: int, seed: int, outlier_p: float = 0.01, outlier_scale: float = 10.0,
                stream: int = 2) -> np.ndarray:
    """bf16 bits [M, K]: N(0, 1) with each entry scaled by outlier_scale with probability outlier_p."""
    z = normal(seed, stream, M * K)
    if outlier_p > 0.0:
        hit = uniform(seed, stream + 100, M * K) < outlier_p
        z = np.where(hit, z * outlier_scale, z)
    return to_bf16_bits(z.astype(np.float32)).reshape(M, K)


def ternary_weights(N: int, K: int, seed: int, p0: float = 0.42, stream: int = 3) -> np.ndarray:
    """int8 [N, K] in {-1, 0, +1} with P(0) = p0 and P(+1) = P(-1) = (1 - p0) / 2."""
    u = uniform(seed, stream, N * K)
    pm = (1.0 - p0) / 2.0
    t = np.where(u < pm, -1, np.where(u < pm + p0, 0, 1)).astype(np.int8)
    return t.reshape(N, K)


def alpha_uniform(seed: int, lo: float = 0.01, hi: float = 0.05, stream: int = 4) -> np.float32:
    return np.float32(lo + (hi - lo) * uniform(seed, stream, 1)[0])


# The pages' layer shapes (BitNet b1.58 2B4T: hidden 2560, FFN 6912, 20 query
# heads and 5 key/value heads of 128; Qwen2.5-3B MLP: 2048 <-> 11008).
B2B4T_LAYER = {
    "q": (2560, 2560), "k": (2560, 640), "v": (2560, 640), "o": (2560, 2560),
    "gate": (2560, 6912), "up": (2560, 6912), "down": (6912, 2560),
}  # name -> (K, N)
QWEN25_3B_MLP = {"up": (2048, 11008), "down": (11008, 2048)}
