"""Seeded, counter-based synthetic inputs (host side, numpy).

This module is the only code shared by the CPU oracle and the CUDA path. It
holds no arithmetic of the Medusa method itself: it only draws numbers.

Generator definition (the device twin in ``gen_kernels.cu`` implements the
same definition and must produce identical bits):

* ``mix64`` is the splitmix64 finaliser (Steele, Lea and Flood, "Fast
  splittable pseudorandom number generators", OOPSLA 2014):
  ``z ^= z >> 30; z *= 0xBF58476D1CE4E5B9; z ^= z >> 27;
  z *= 0x94D049BB133111EB; z ^= z >> 31`` (all mod 2^64).
* A tensor is a (seed, stream) pair. Its key is
  ``mix64(mix64(seed) ^ (stream * 0xD1B54A32D192ED03))``.
* Element ``i`` (row-major flat index of the tensor's logical layout) draws
  ``r_i = mix64(key + (i + 1) * 0x9E3779B97F4A7C15)``.
* Approximately normal values use the Irwin-Hall sum of the four 16-bit
  fields of ``r_i``: ``c = f0 + f1 + f2 + f3 - 131070`` (an exact integer,
  mean 0, standard deviation ``sqrt(4 * (65536**2 - 1) / 12)``). The value is
  ``fp64(c) * scale`` with ``scale = sigma / sd`` computed once in fp64 on the
  host (one correctly rounded multiply), then rounded to fp32 with
  round-to-nearest-even, then (for bf16 tensors) fp32 -> bf16 with
  round-to-nearest-even on the bit pattern.
* Uniform integers in ``[0, n)`` are ``((r >> 32) * n) >> 32`` (Lemire's
  multiply-shift map, exact in 64-bit integers).
* Uniform reals in ``[0, 1)`` are ``(r >> 11) * 2**-53``.

The distribution is a 4-term Irwin-Hall approximation of N(0, sigma): its
tails stop at about 3.46 sigma. Every step above is exact integer arithmetic
or a single IEEE-rounded operation, which is what lets the host and device
versions agree bit for bit.
"""
from __future__ import annotations

import math

import numpy as np

MASK64 = (1 << 64) - 1
GOLDEN = 0x9E3779B97F4A7C15
STREAM_MULT = 0xD1B54A32D192ED03
IH_SD = math.sqrt(4.0 * (65536.0 ** 2 - 1.0) / 12.0)
IH_CENTER = 2 * 65535

# Stream ids: one per named tensor, fixed forever so that seeds reproduce.
STREAMS = {
    "h": 1,
    "W1": 2,
    "b1": 3,
    "Wv": 4,
    "q": 5,
    "k_cache": 6,
    "v_cache": 7,
    "logits": 8,
    "plant": 9,
    "root_token": 10,
    "prefix_len": 11,
    "tokens": 12,
    "plant_pick": 13,
    "E": 14,
    "head_logits": 15,
}

_U64 = np.uint64
_CHUNK = 1 << 22


def mix64_int(z: int) -> int:
    """splitmix64 finaliser on a Python int (mod 2^64)."""
    z &= MASK64
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & MASK64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & MASK64
    return z ^ (z >> 31)


def stream_key(seed: int, stream: int | str) -> int:
    """64-bit key of the tensor (seed, stream)."""
    if isinstance(stream, str):
        stream = STREAMS[stream]
    return mix64_int(mix64_int(seed) ^ ((stream * STREAM_MULT) & MASK64))


def normal_scale(sigma: float) -> float:
    """fp64 factor that maps the centred Irwin-Hall integer to N(0, sigma)."""
    return float(sigma) / IH_SD


def _mix64(z: np.ndarray) -> np.ndarray:
    z = (z ^ (z >> _U64(30))) * _U64(0xBF58476D1CE4E5B9)
    z = (z ^ (z >> _U64(27))) * _U64(0x94D049BB133111EB)
    return z ^ (z >> _U64(31))


def raw_u64(key: int, idx: np.ndarray) -> np.ndarray:
    """r_i for an array of flat indices (uint64)."""
    idx = np.asarray(idx, dtype=_U64)
    with np.errstate(over="ignore"):
        return _mix64(_U64(key) + (idx + _U64(1)) * _U64(GOLDEN))


def _centred(r: np.ndarray) -> np.ndarray:
    m = _U64(0xFFFF)
    s = (r & m) + ((r >> _U64(16)) & m) + ((r >> _U64(32)) & m) + (r >> _U64(48))
    return s.astype(np.int64) - IH_CENTER


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (nearest even) and return the 16-bit patterns.

    Inputs here are always finite.
    """
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    lsb = (b >> np.uint32(16)) & np.uint32(1)
    return ((b + np.uint32(0x7FFF) + lsb) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to fp32."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def normal_f32_at(key: int, idx: np.ndarray, sigma: float) -> np.ndarray:
    c = _centred(raw_u64(key, idx))
    return (c.astype(np.float64) * normal_scale(sigma)).astype(np.float32)


def normal_bf16_at(key: int, idx: np.ndarray, sigma: float) -> np.ndarray:
    return f32_to_bf16_bits(normal_f32_at(key, idx, sigma))


def uniform_int_at(key: int, idx: np.ndarray, n: int) -> np.ndarray:
    if not (0 < n < (1 << 32)):
        raise ValueError("uniform_int_at: n must be in [1, 2^32)")
    r = raw_u64(key, idx)
    return (((r >> _U64(32)) * _U64(n)) >> _U64(32)).astype(np.int64)


def uniform_unit_at(key: int, idx: np.ndarray) -> np.ndarray:
    r = raw_u64(key, idx)
    return (r >> _U64(11)).astype(np.float64) * (2.0 ** -53)


def _fill(shape, fn, dtype, start: int = 0) -> np.ndarray:
    n = int(np.prod(shape, dtype=np.int64)) if len(shape) else 1
    out = np.empty(n, dtype=dtype)
    for lo in range(0, n, _CHUNK):
        hi = min(n, lo + _CHUNK)
        out[lo:hi] = fn(np.arange(start + lo, start + hi, dtype=_U64))
    return out.reshape(shape)


def normal_bf16(seed: int, stream, shape, sigma: float) -> np.ndarray:
    """bf16 bit patterns (uint16) of a whole tensor."""
    key = stream_key(seed, stream)
    return _fill(tuple(shape), lambda i: normal_bf16_at(key, i, sigma), np.uint16)


def normal_f32(seed: int, stream, shape, sigma: float) -> np.ndarray:
    key = stream_key(seed, stream)
    return _fill(tuple(shape), lambda i: normal_f32_at(key, i, sigma), np.float32)


def uniform_int(seed: int, stream, shape, lo: int, hi: int) -> np.ndarray:
    """Integers uniform in [lo, hi] (inclusive), int64."""
    key = stream_key(seed, stream)
    return _fill(tuple(shape), lambda i: uniform_int_at(key, i, hi - lo + 1) + lo, np.int64)
