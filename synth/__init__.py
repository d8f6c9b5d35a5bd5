"""Seeded synthetic inputs shared by the oracle tests, the GPU parity tests and the benchmark.

This module holds none of the attention, RoPE or mask arithmetic. It only turns a
(seed, element index) pair into a number:

* SplitMix64 (Steele, Lea and Flood, "Fast splittable pseudorandom number
  generators", OOPSLA 2014) as a counter-based generator: element ``i`` of stream
  ``seed`` is the SplitMix64 output for state ``seed + (i + 1) * 0x9E3779B97F4A7C15``.
* A uniform double in (0, 1] from the top 53 bits.
* The Box-Muller transform (Box and Muller, 1958) to N(0, 1): element ``2p`` takes the
  cosine branch and ``2p + 1`` the sine branch of pair ``p``.
* Rounding float64 -> float32 -> bfloat16, each step round-to-nearest-even, so the
  oracle (which widens the bf16 bits back to float64) and the GPU see identical values.

Because every value depends only on (seed, index), any slice of a tensor can be
generated on its own; ``normal`` generates in blocks to bound host memory.

Tensor layout convention used by every caller: [tokens, heads, head_dim], token order
frame-major, then patch row h, then patch column w.
"""
from __future__ import annotations

import numpy as np

_GOLDEN = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)
_BLOCK = 1 << 22


def splitmix64(seed: int, start: int, n: int) -> np.ndarray:
    """Outputs ``start .. start+n-1`` of the SplitMix64 stream ``seed`` (uint64 array)."""
    with np.errstate(over="ignore"):
        idx = np.arange(start + 1, start + n + 1, dtype=np.uint64)
        z = np.uint64(seed & 0xFFFFFFFFFFFFFFFF) + idx * _GOLDEN
        z = (z ^ (z >> np.uint64(30))) * _M1
        z = (z ^ (z >> np.uint64(27))) * _M2
        z = z ^ (z >> np.uint64(31))
    return z


def uniform01(seed: int, start: int, n: int) -> np.ndarray:
    """Uniform float64 in (0, 1]: (top 53 bits + 1) * 2**-53."""
    z = splitmix64(seed, start, n)
    return ((z >> np.uint64(11)).astype(np.float64) + 1.0) * (2.0 ** -53)


def _normal_block(seed: int, start: int, n: int) -> np.ndarray:
    # element i belongs to Box-Muller pair i // 2; generate whole pairs, then slice
    p0 = start // 2
    p1 = (start + n + 1) // 2
    u = uniform01(seed, 2 * p0, 2 * (p1 - p0))
    u1 = u[0::2]
    u2 = u[1::2]
    r = np.sqrt(-2.0 * np.log(u1))
    out = np.empty(2 * (p1 - p0), dtype=np.float64)
    out[0::2] = r * np.cos(2.0 * np.pi * u2)
    out[1::2] = r * np.sin(2.0 * np.pi * u2)
    off = start - 2 * p0
    return out[off:off + n]


def normal(seed: int, n: int, start: int = 0) -> np.ndarray:
    """N(0, 1) float64 values ``start .. start+n-1`` of stream ``seed``."""
    out = np.empty(n, dtype=np.float64)
    for b in range(0, n, _BLOCK):
        m = min(_BLOCK, n - b)
        out[b:b + m] = _normal_block(seed, start + b, m)
    return out


def f32_to_bf16_bits(x32: np.ndarray) -> np.ndarray:
    """Round float32 to bfloat16 (nearest, ties to even); returns the uint16 bit patterns.

    Inputs here are finite normals, so no NaN handling is needed."""
    b = np.ascontiguousarray(x32, dtype=np.float32).view(np.uint32)
    lsb = (b >> np.uint32(16)) & np.uint32(1)
    r = (b + np.uint32(0x7FFF) + lsb) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bfloat16 bit patterns to float64."""
    return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def normal_bf16(seed: int, n: int, start: int = 0, scale: float = 1.0) -> np.ndarray:
    """N(0, scale^2) values rounded float64 -> float32 -> bfloat16; uint16 bit patterns."""
    out = np.empty(n, dtype=np.uint16)
    for b in range(0, n, _BLOCK):
        m = min(_BLOCK, n - b)
        x = _normal_block(seed, start + b, m) * scale
        out[b:b + m] = f32_to_bf16_bits(x.astype(np.float32))
    return out


def tensor_seed(workload: int, which: str) -> int:
    """Seed of one input tensor: 1000 * workload id + {q: 0, k: 1, v: 2}."""
    return 1000 * workload + {"q": 0, "k": 1, "v": 2}[which]


def qkv_bf16(workload: int, n_tokens: int, heads: int, head_dim: int,
             which: str, token_offset: int = 0, scale: float = 1.0) -> np.ndarray:
    """A [n_tokens, heads, head_dim] bf16 tensor (uint16 bits) from the stream of ``which``.

    ``token_offset`` selects a slice of a longer sequence: token ``n`` of the result is
    token ``token_offset + n`` of the full stream, so a chunk of frames generated alone
    equals the same frames cut out of the whole clip."""
    row = heads * head_dim
    bits = normal_bf16(tensor_seed(workload, which), n_tokens * row,
                       start=token_offset * row, scale=scale)
    return bits.reshape(n_tokens, heads, head_dim)
