"""Seeded synthetic inputs shared by the CUDA path's tests/bench and the oracle.

This module holds no attention arithmetic.  It only draws numbers:

* ``splitmix64(seed, n)``      -- the SplitMix64 counter generator (Steele, Lea
  and Flood, "Fast splittable pseudorandom number generators", OOPSLA 2014):
  output i is the 64-bit finaliser applied to ``seed + (i+1)*0x9E3779B97F4A7C15``.
* ``uniform01`` / ``normal``  -- 53-bit uniforms in (0,1) and Box-Muller
  normals (fp64) built on that stream.
* ``normal_bf16``             -- iid N(0,1) draws rounded to fp32 and then
  round-to-nearest-even to bfloat16, returned as raw uint16 bit patterns.
* ``outlier_columns``         -- the seeded choice of feature columns that the
  FP8 workload scales by 20 before rounding (1 % of the H*d columns).
* ``hadamard_signs``          -- the seeded random +-1 diagonal used by the
  incoherent-processing rotation.  The sign vector is an *input* to both the
  oracle and the CUDA quantiser; neither side draws it.

Seed scheme: base seed S; Q = S, K = S+1, V = S+2, Hadamard signs = S+3,
outlier columns = S+4.  The default base seed is 140.
"""
from __future__ import annotations

import numpy as np

BASE_SEED = 140
_GOLDEN = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)


def splitmix64(seed: int, n: int, offset: int = 0) -> np.ndarray:
    """Outputs offset .. offset+n-1 of the SplitMix64 stream started at ``seed``."""
    with np.errstate(over="ignore"):
        idx = np.arange(offset + 1, offset + n + 1, dtype=np.uint64)
        z = np.uint64(seed & 0xFFFFFFFFFFFFFFFF) + idx * _GOLDEN
        z = (z ^ (z >> np.uint64(30))) * _M1
        z = (z ^ (z >> np.uint64(27))) * _M2
        z = z ^ (z >> np.uint64(31))
    return z


def uniform01(seed: int, n: int, offset: int = 0) -> np.ndarray:
    """Uniforms strictly inside (0, 1): ((z >> 11) + 0.5) * 2^-53."""
    z = splitmix64(seed, n, offset)
    return ((z >> np.uint64(11)).astype(np.float64) + 0.5) * (2.0 ** -53)


def normal(seed: int, n: int) -> np.ndarray:
    """n iid N(0,1) fp64 draws, Box-Muller on consecutive uniform pairs."""
    m = (n + 1) // 2
    u = uniform01(seed, 2 * m)
    u1, u2 = u[0::2], u[1::2]
    r = np.sqrt(-2.0 * np.log(u1))
    t = 2.0 * np.pi * u2
    out = np.empty(2 * m, dtype=np.float64)
    out[0::2] = r * np.cos(t)
    out[1::2] = r * np.sin(t)
    return out[:n]


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 values to bfloat16 (nearest, ties to even); raw uint16 bits."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    b = (b + np.uint64(0x7FFF) + ((b >> np.uint64(16)) & np.uint64(1))) >> np.uint64(16)
    return b.astype(np.uint16)


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bfloat16 bit patterns to fp64."""
    u = np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return u.view(np.float32).astype(np.float64)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    u = np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return u.view(np.float32)


def normal_bf16(seed: int, shape, column_scale: np.ndarray | None = None) -> np.ndarray:
    """iid N(0,1) in ``shape`` as bf16 bits.  ``column_scale`` (length shape[-2]*shape[-1],
    i.e. one factor per (head, channel) feature column) multiplies each draw before rounding."""
    n = int(np.prod(shape))
    x = normal(seed, n).reshape(shape)
    if column_scale is not None:
        if column_scale.size != shape[-2] * shape[-1]:
            raise ValueError("column_scale needs one factor per (head, channel) column")
        x = x * column_scale.reshape((1,) * (len(shape) - 2) + (shape[-2], shape[-1]))
    return f32_to_bf16_bits(x.astype(np.float32))


def outlier_columns(seed: int, H: int, d: int, frac: float = 0.01) -> np.ndarray:
    """round(frac*H*d) distinct flattened (head, channel) column indices, seeded."""
    n_feat = H * d
    k = int(round(frac * n_feat))
    keys = splitmix64(seed, n_feat)
    return np.sort(np.argsort(keys, kind="stable")[:k])


def outlier_scale(seed: int, H: int, d: int, factor: float = 20.0, frac: float = 0.01) -> np.ndarray:
    s = np.ones(H * d, dtype=np.float64)
    s[outlier_columns(seed, H, d, frac)] = factor
    return s


def hadamard_signs(seed: int, d: int) -> np.ndarray:
    """Random +-1 vector of length d (fp32): sign = top bit of the SplitMix64 output."""
    z = splitmix64(seed, d)
    return np.where((z >> np.uint64(63)) == 1, -1.0, 1.0).astype(np.float32)


def qkv_bf16(B: int, Hq: int, Hkv: int, Nq: int, Nk: int, d: int, seed: int = BASE_SEED,
             outliers: bool = False):
    """Q [B,Nq,Hq,d], K and V [B,Nk,Hkv,d] as bf16 bits from seeds S, S+1, S+2."""
    cq = outlier_scale(seed + 4, Hq, d) if outliers else None
    ck = outlier_scale(seed + 4, Hkv, d) if outliers else None
    q = normal_bf16(seed, (B, Nq, Hq, d), cq)
    k = normal_bf16(seed + 1, (B, Nk, Hkv, d), ck)
    v = normal_bf16(seed + 2, (B, Nk, Hkv, d), ck)
    return q, k, v
