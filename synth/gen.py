"""Counter-based random streams for the synthetic decode workloads.

This module is shared by the CPU oracle tests and the GPU path. It holds no step of the
attention method (no RoPE, no index projection, no scoring, no selection, no softmax):
only a seed-addressable random-number stream, bf16 storage rounding of the generated values,
and the planted-cluster shift that gives the index scores their structure.

Random stream (one definition, two implementations: this NumPy file and
``synth/csrc/synth_fill.cu``; a GPU test checks they agree bit for bit):

* ``mix64`` is the splitmix64 output function (Steele, Lea and Flood, "Fast splittable
  pseudorandom number generators", OOPSLA 2014): xor-shift 30, multiply by
  0xBF58476D1CE4E5B9, xor-shift 27, multiply by 0x94D049BB133111EB, xor-shift 31.
* A stream key folds (seed, tensor id, layer, sequence, head) into 64 bits through ``mix64``.
* Element ``c`` of a stream is ``mix64(key + GOLDEN * (c + 1))``.
* A near-normal float32 value takes the four 16-bit fields of that word, sums them
  (Irwin-Hall with four terms), centres the sum and scales it to unit variance with one
  float32 multiplication. Every step is integer or a single correctly rounded float32
  operation, so both implementations produce identical bits.
"""
from __future__ import annotations

import numpy as np

U64 = np.uint64
GOLDEN = U64(0x9E3779B97F4A7C15)
_M1 = U64(0xBF58476D1CE4E5B9)
_M2 = U64(0x94D049BB133111EB)
_KEY_SALT = U64(0xD1B54A32D192ED03)

# 1 / std of the sum of four independent uniforms on {0, ..., 65535}: var = 4 (65536^2 - 1) / 12.
INV_STD = np.float32(1.0 / np.sqrt((65536.0 ** 2 - 1.0) / 3.0))
IH_CENTRE = 2 * 65535

# Tensor ids of the streams.
T_KPRE, T_V, T_QPRE, T_WQIDX, T_WKIDX, T_QPROMPT = 1, 2, 3, 4, 5, 6


def mix64(z):
    """splitmix64 output function on uint64 values (wrapping arithmetic)."""
    z = np.asarray(z, dtype=U64)
    with np.errstate(over="ignore"):
        z = (z ^ (z >> U64(30))) * _M1
        z = (z ^ (z >> U64(27))) * _M2
    return z ^ (z >> U64(31))


def stream_key(seed: int, tensor: int, layer: int = 0, seq: int = 0, head: int = 0) -> int:
    """64-bit key of one stream; all ids are non-negative ints."""
    k = mix64(U64(seed) ^ _KEY_SALT)
    with np.errstate(over="ignore"):
        for v in (tensor, layer, seq, head):
            k = mix64(k + GOLDEN * U64(v + 1))
    return int(k)


def stream_bits(key: int, counters) -> np.ndarray:
    """uint64 word of each counter of the stream ``key``."""
    c = np.asarray(counters, dtype=U64)
    with np.errstate(over="ignore"):
        return mix64(U64(key) + GOLDEN * (c + U64(1)))


def normal_f32(key: int, counters) -> np.ndarray:
    """Near-normal float32 values (mean 0, variance 1, bounded at about 3.46)."""
    h = np.ascontiguousarray(stream_bits(key, counters))
    shape = h.shape
    # the four 16-bit fields of each word (little-endian view), summed exactly in int32
    f = h.reshape(-1).view(np.uint16).reshape(-1, 4)
    s = f[:, 0].astype(np.int32)
    s += f[:, 1]
    s += f[:, 2]
    s += f[:, 3]
    s -= IH_CENTRE
    return (s.astype(np.float32) * INV_STD).reshape(shape)


def f32_to_bf16_bits(x) -> np.ndarray:
    """float32 -> bfloat16 bit patterns, round to nearest even (finite inputs)."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    b = b + U64(0x7FFF) + ((b >> U64(16)) & U64(1))
    return (b >> U64(16)).astype(np.uint16)


def bf16_bits_to_f32(bits) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def token_rows_bits(key: int, t0: int, t1: int, dim: int, shifts=None) -> np.ndarray:
    """bf16 bits [t1 - t0][dim] of rows t0..t1-1 of stream ``key`` (element c = t * dim + d).

    ``shifts`` is an optional list of (start, length, delta float32[dim]): rows inside
    [start, start + length) get ``delta`` added (one float32 addition) before rounding.
    """
    c = np.arange(t0 * dim, t1 * dim, dtype=np.uint64).reshape(t1 - t0, dim)
    x = normal_f32(key, c)
    if shifts:
        for (start, length, delta) in shifts:
            a, b = max(start, t0), min(start + length, t1)
            if a < b:
                x[a - t0:b - t0] = x[a - t0:b - t0] + np.asarray(delta, dtype=np.float32)[None, :]
    return f32_to_bf16_bits(x)
