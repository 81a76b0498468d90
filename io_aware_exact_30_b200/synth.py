"""Seeded synthetic inputs shared by the CUDA path, its tests and the oracle.

This module holds only random-number generation and dtype rounding: none of
the attention arithmetic lives here, so the oracle and the kernels can both
draw their inputs from it without sharing any of the method.

Definition (counter-addressable, so any slice can be regenerated alone):

* ``splitmix64`` word ``c`` of stream ``(seed, s)`` is
  ``mix64(base + (c + 1) * GAMMA)`` with
  ``base = mix64(mix64(seed) ^ ((s + 1) * GAMMA))``, where ``mix64`` is the
  splitmix64 output finaliser (Steele, Lea, Flood, "Fast splittable
  pseudorandom number generators", OOPSLA 2014) and ``GAMMA`` its golden-ratio
  increment.
* Gaussian pair ``p`` takes words ``2p`` and ``2p+1``:
  ``u1 = ((w0 >> 11) + 1) * 2**-53`` in (0, 1], ``u2 = (w1 >> 11) * 2**-53``
  in [0, 1); Box-Muller gives ``z0 = r cos(2 pi u2)``, ``z1 = r sin(2 pi u2)``
  with ``r = sqrt(-2 ln u1)``. Element ``2p`` is ``z0``, element ``2p+1`` is
  ``z1``.
* ``x = sigma * z`` in float64, then rounded to the storage dtype:
  fp16 by one round-to-nearest-even step from float64; bf16 by
  round-to-nearest-even to float32 and then round-to-nearest-even to bf16.

Stream ids: Q = 0, K = 1, V = 2, dO = 3; the random signs of the FP8
rotation use stream 4 (word t >> 63 picks the sign of coordinate t).
"""

from __future__ import annotations

import numpy as np

GAMMA = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)

STREAM_Q, STREAM_K, STREAM_V, STREAM_DO, STREAM_SIGNS = 0, 1, 2, 3, 4

_CHUNK = 1 << 22  # elements generated per numpy pass (bounds host memory)


def mix64(z):
    """splitmix64 finaliser on a numpy uint64 scalar or array (wrapping)."""
    z = np.asarray(z, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = (z ^ (z >> np.uint64(30))) * _M1
        z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def stream_base(seed: int, stream: int) -> np.uint64:
    with np.errstate(over="ignore"):
        s = np.uint64((stream + 1) & 0xFFFFFFFFFFFFFFFF) * GAMMA
    return np.uint64(mix64(mix64(np.uint64(seed & 0xFFFFFFFFFFFFFFFF)) ^ s))


def words(seed: int, stream: int, start: int, count: int) -> np.ndarray:
    """splitmix64 words ``start .. start+count-1`` of stream ``(seed, stream)``."""
    base = stream_base(seed, stream)
    c = np.arange(start + 1, start + count + 1, dtype=np.uint64)
    with np.errstate(over="ignore"):
        return mix64(base + c * GAMMA)


def gaussian(seed: int, stream: int, n: int, sigma: float = 1.0) -> np.ndarray:
    """``n`` float64 samples of N(0, sigma^2) from stream ``(seed, stream)``."""
    out = np.empty(n, dtype=np.float64)
    two53 = 2.0 ** -53
    for e0 in range(0, n, _CHUNK):
        e1 = min(n, e0 + _CHUNK)
        p0, p1 = e0 // 2, (e1 + 1) // 2
        w = words(seed, stream, 2 * p0, 2 * (p1 - p0))
        u1 = ((w[0::2] >> np.uint64(11)).astype(np.float64) + 1.0) * two53
        u2 = (w[1::2] >> np.uint64(11)).astype(np.float64) * two53
        r = np.sqrt(-2.0 * np.log(u1))
        z = np.empty(2 * (p1 - p0), dtype=np.float64)
        z[0::2] = r * np.cos(2.0 * np.pi * u2)
        z[1::2] = r * np.sin(2.0 * np.pi * u2)
        out[e0:e1] = z[e0 - 2 * p0: e1 - 2 * p0]
    if sigma != 1.0:
        out *= sigma
    return out


def round_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float64 -> bf16 bit patterns (uint16): RNE to float32, then RNE to bf16."""
    b = np.ascontiguousarray(x, dtype=np.float64).astype(np.float32).view(np.uint32)
    lsb = (b >> np.uint32(16)) & np.uint32(1)
    with np.errstate(over="ignore"):
        r = (b + np.uint32(0x7FFF) + lsb) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact upcast of bf16 bit patterns to float64."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def tensor(seed: int, stream: int, shape, sigma: float = 1.0, dtype: str = "bf16") -> np.ndarray:
    """Seeded tensor as its storage array, shaped ``shape`` and C-contiguous:
    uint16 bf16 bit patterns for ``"bf16"``, float16 values for ``"fp16"``.
    :func:`to_f64` gives the exact float64 values."""
    n = int(np.prod(shape))
    z = gaussian(seed, stream, n, sigma)
    if dtype == "bf16":
        return round_bf16_bits(z).reshape(shape)
    if dtype == "fp16":
        return z.astype(np.float16).reshape(shape)
    raise ValueError(f"unsupported dtype {dtype!r}")


def to_f64(stored: np.ndarray, dtype: str) -> np.ndarray:
    """Exact float64 view of what :func:`tensor` stored."""
    if dtype == "bf16":
        return bf16_bits_to_f64(stored).reshape(stored.shape)
    if dtype == "fp16":
        return np.asarray(stored, dtype=np.float16).astype(np.float64)
    raise ValueError(f"unsupported dtype {dtype!r}")


def attention_inputs(B: int, H: int, N: int, d: int, *, seed: int = 0, sigma: float = 1.0,
                     dtype: str = "bf16", with_dout: bool = False, dout_sigma: float = 1.0):
    """Q, K, V (and dO) of shape (B, H, N, d) as storage arrays, streams 0..3."""
    shape = (B, H, N, d)
    out = [tensor(seed, s, shape, sigma, dtype) for s in (STREAM_Q, STREAM_K, STREAM_V)]
    if with_dout:
        out.append(tensor(seed, STREAM_DO, shape, dout_sigma, dtype))
    return out


def random_signs(d: int, seed: int = 0) -> np.ndarray:
    """d random signs (int8, +1 or -1) from stream (seed, 4): the top bit of
    splitmix64 word t set gives -1."""
    w = words(seed, STREAM_SIGNS, 0, d)
    return np.where((w >> np.uint64(63)) == np.uint64(1), -1, 1).astype(np.int8)
