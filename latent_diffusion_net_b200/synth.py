"""Seeded synthetic inputs and random-init weights.

This module holds no arithmetic of the denoiser itself. It only draws the random
numbers that both the CPU oracle and the CUDA path receive as inputs, so that the
two sides start from bit-identical BF16 values.

Generator (counter-based, so any element can be drawn independently):

* Tensor ``k`` gets its own SplitMix64 stream (Steele, Lea & Flood, "Fast
  splittable pseudorandom number generators", OOPSLA 2014) whose starting state is
  ``s_k = seed * 0x9E3779B97F4A7C15 XOR (k + 1)`` (mod 2**64).
* Draw ``i`` (0-based) of that stream is the SplitMix64 output for the state
  ``s_k + (i + 1) * 0x9E3779B97F4A7C15``.
* A uniform in (0, 1] is ``((z >> 11) + 1) * 2**-53``.
* Normal ``j`` is Box-Muller on draws ``2j`` and ``2j + 1``:
  ``sqrt(-2 ln u1) * cos(2 pi u2)``.
* A value ``sigma * n`` is formed in float64, rounded to float32 and then to
  BF16 with round-to-nearest-even.

Tensor indices: inputs use 0..7, weights start at 16 and follow the enumeration
order of the parameter table.
"""
from __future__ import annotations

import math
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

GOLDEN = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)
WEIGHT_INDEX_BASE = 16

# Input tensor indices (stable: stored expected values depend on them).
IDX_X = 0          # block input x, or the U-Net latent
IDX_CTX = 1        # text context
IDX_NOISY = 2      # inpaint: noisy latent
IDX_MASKED = 3     # inpaint: masked latent
IDX_MASK = 4       # inpaint: mask rectangle draws
IDX_TEXT = 5       # SDXL: pooled text embedding
IDX_NOISE = 6      # sampler: the noise z of each reverse step (one stream, step-major)
IDX_CTX_UNCOND = 7  # sampler: the unconditional context of guidance


def stream_seed(seed: int, k: int) -> np.uint64:
    s = (int(seed) * 0x9E3779B97F4A7C15) & 0xFFFFFFFFFFFFFFFF
    return np.uint64(s ^ ((k + 1) & 0xFFFFFFFFFFFFFFFF))


def splitmix64(s0: np.uint64, start: int, count: int) -> np.ndarray:
    """SplitMix64 outputs for draws start .. start+count-1 of stream s0."""
    with np.errstate(over="ignore"):
        i = np.arange(start + 1, start + count + 1, dtype=np.uint64)
        z = s0 + i * GOLDEN
        z = (z ^ (z >> np.uint64(30))) * _M1
        z = (z ^ (z >> np.uint64(27))) * _M2
        z = z ^ (z >> np.uint64(31))
    return z


def uniforms(s0: np.uint64, start: int, count: int) -> np.ndarray:
    z = splitmix64(s0, start, count)
    return ((z >> np.uint64(11)).astype(np.float64) + 1.0) * (2.0 ** -53)


def _normals_chunk(s0: np.uint64, j0: int, n: int) -> np.ndarray:
    u = uniforms(s0, 2 * j0, 2 * n)
    u1 = u[0::2]
    u2 = u[1::2]
    return np.sqrt(-2.0 * np.log(u1)) * np.cos(2.0 * math.pi * u2)


def f32_to_bf16_bits(x32: np.ndarray) -> np.ndarray:
    """Round float32 to BF16 (round-to-nearest-even); returns uint16 bit patterns."""
    b = np.ascontiguousarray(x32, dtype=np.float32).view(np.uint32)
    rounding = np.uint32(0x7FFF) + ((b >> np.uint32(16)) & np.uint32(1))
    with np.errstate(over="ignore"):
        out = ((b + rounding) >> np.uint32(16)).astype(np.uint16)
    nan = np.isnan(x32)
    if nan.any():
        out[nan] = 0x7FC0
    return out


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


_POOL = None


def _pool():
    global _POOL
    if _POOL is None:
        _POOL = ThreadPoolExecutor(max_workers=max(1, min(16, os.cpu_count() or 1)))
    return _POOL


def normal_bf16_bits(seed: int, k: int, count: int, sigma: float = 1.0) -> np.ndarray:
    """``count`` N(0, sigma^2) values of tensor ``k``, as BF16 bit patterns."""
    s0 = stream_seed(seed, k)
    chunk = 1 << 21
    if count <= chunk:
        n = _normals_chunk(s0, 0, count)
        return f32_to_bf16_bits((sigma * n).astype(np.float32))
    out = np.empty(count, dtype=np.uint16)

    def work(j0):
        n = min(chunk, count - j0)
        v = _normals_chunk(s0, j0, n)
        out[j0:j0 + n] = f32_to_bf16_bits((sigma * v).astype(np.float32))

    list(_pool().map(work, range(0, count, chunk)))
    return out


def normal_bf16(seed: int, k: int, shape, sigma: float = 1.0) -> np.ndarray:
    """N(0, sigma^2) values rounded to BF16, returned as float32 of ``shape``."""
    count = int(np.prod(shape)) if len(shape) else 1
    return bf16_bits_to_f32(normal_bf16_bits(seed, k, count, sigma)).reshape(shape)


def mask_rectangle(seed: int, height: int = 128, width: int = 128):
    """Inpaint mask: a rectangle with top-left (y0, x0) uniform in {0..63} and
    height/width uniform in {32..64}; 1.0 inside, 0.0 outside (clipped to the
    image). Returns (mask [height, width] float32, (y0, x0, h, w))."""
    u = uniforms(stream_seed(seed, IDX_MASK), 0, 4)
    y0 = int(u[0] * 64) % 64
    x0 = int(u[1] * 64) % 64
    h = 32 + int(u[2] * 33) % 33
    w = 32 + int(u[3] * 33) % 33
    m = np.zeros((height, width), dtype=np.float32)
    m[y0:min(height, y0 + h), x0:min(width, x0 + w)] = 1.0
    return m, (y0, x0, h, w)


def param_value(seed: int, k: int, shape, kind: str, fan_in: int, affine_noise: bool = False):
    """Random-init value of parameter number ``k`` (0-based in the table order).

    Convolution and linear weights and biases ~ N(0, 1/fan_in); norm gains are
    1 and norm shifts 0, unless ``affine_noise`` asks for gain 1 + 0.1 N and
    shift 0.1 N (used by unit tests that exercise the affine path)."""
    idx = WEIGHT_INDEX_BASE + k
    if kind in ("weight", "bias"):
        return normal_bf16(seed, idx, shape, 1.0 / math.sqrt(fan_in))
    if kind == "norm_gamma":
        if affine_noise:
            n = normal_bf16(seed, idx, shape, 0.1).astype(np.float64) + 1.0
            return bf16_bits_to_f32(f32_to_bf16_bits(n.astype(np.float32))).reshape(shape)
        return np.ones(shape, dtype=np.float32)
    if kind == "norm_beta":
        if affine_noise:
            return normal_bf16(seed, idx, shape, 0.1)
        return np.zeros(shape, dtype=np.float32)
    raise ValueError(kind)


def canonical_weights(rows, seed: int, affine_noise: bool = False, index_base: int = 0) -> np.ndarray:
    """Canonical BF16 buffer (uint16 bit patterns) for a weight table.

    ``rows`` is a sequence of (shape, kind, fan_in) in table order; tensor ``i``
    uses generator stream ``WEIGHT_INDEX_BASE + index_base + i``."""
    sizes = [int(np.prod(s)) for s, _, _ in rows]
    out = np.empty(sum(sizes), dtype=np.uint16)
    off = 0
    for i, ((shape, kind, fan), n) in enumerate(zip(rows, sizes)):
        v = param_value(seed, index_base + i, tuple(shape), kind, fan, affine_noise)
        out[off:off + n] = f32_to_bf16_bits(np.ascontiguousarray(v, dtype=np.float32).reshape(-1))
        off += n
    return out
