"""Seeded synthetic inputs for the DSA hot path (host side, numpy).

This module is the only code that both the CPU oracle's tests and the CUDA path's tests
and benchmark use.  It contains no part of the method's arithmetic: it only turns
(seed, tensor id, flat element index) into values, with integer operations alone, so
that the device fill kernels in ``synth_fill.cu`` produce bit-identical tensors.

Generator (counter based, SplitMix64 of Steele, Lea and Flood, OOPSLA 2014):
    mix64(z)      = z ^= z>>30; z *= 0xBF58476D1CE4E5B9; z ^= z>>27;
                    z *= 0x94D049BB133111EB; z ^= z>>31
    key(seed,tid) = mix64((seed ^ 0x5EEDD5A05EEDD5A0) + GAMMA*(tid+1))
    draw(key, j)  = mix64(key + GAMMA*(j+1))          GAMMA = 0x9E3779B97F4A7C15
Distributions, for the element with flat index i:
    int17   (integer-valued bf16, uniform on -8..8):  ((draw(key,i) >> 32) mod 17) - 8
            (int17_e4m3: the same integers as E4M3 bytes)
    pow2    (float32 head weight, 2^-1 .. 2^-6):      2^-(1 + ((draw(key,i) >> 32) mod 6))
    normal  (bf16, approximately N(0,1)): the sum S of the twelve 16-bit fields of
            draw(key,3i), draw(key,3i+1), draw(key,3i+2) (Irwin-Hall with 12 terms),
            x = (S - 393210) * 2^-16 (exact in float32), rounded to bf16 to nearest-even
    unit    (float32 in [-0.5, 0.5) with 24-bit resolution): (draw(key,i) >> 40)*2^-24 - 0.5
"""
from __future__ import annotations

import numpy as np

GAMMA = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)
_SALT = 0x5EEDD5A05EEDD5A0
_MASK64 = (1 << 64) - 1

# tensor kinds of a DSA group workload
KIND_IQ, KIND_W, KIND_IK, KIND_Q, KIND_KV, KIND_SCORES = 1, 2, 3, 4, 5, 6


def tensor_id(kind: int, group: int = 0, layer: int = 0, step: int = 0) -> int:
    return (kind << 24) | (group << 16) | (layer << 8) | step


def _mix64_int(z: int) -> int:
    z &= _MASK64
    z ^= z >> 30
    z = (z * 0xBF58476D1CE4E5B9) & _MASK64
    z ^= z >> 27
    z = (z * 0x94D049BB133111EB) & _MASK64
    z ^= z >> 31
    return z


def stream_key(seed: int, tid: int) -> int:
    return _mix64_int(((seed ^ _SALT) + 0x9E3779B97F4A7C15 * (tid + 1)) & _MASK64)


def _mix64(z: np.ndarray) -> np.ndarray:
    with np.errstate(over="ignore"):
        z = z ^ (z >> np.uint64(30))
        z = z * _M1
        z = z ^ (z >> np.uint64(27))
        z = z * _M2
        z = z ^ (z >> np.uint64(31))
    return z


def draws(key: int, j: np.ndarray) -> np.ndarray:
    j = np.asarray(j, dtype=np.uint64)
    with np.errstate(over="ignore"):
        return _mix64(np.uint64(key) + GAMMA * (j + np.uint64(1)))


def _flat(shape_or_idx) -> np.ndarray:
    if isinstance(shape_or_idx, np.ndarray):
        return shape_or_idx.astype(np.uint64, copy=False)
    n = int(np.prod(shape_or_idx))
    return np.arange(n, dtype=np.uint64)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bf16 (nearest, ties to even) with integer operations."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = (u + np.uint64(0x7FFF) + ((u >> np.uint64(16)) & np.uint64(1))) >> np.uint64(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def int17_bf16(key: int, shape=None, index: np.ndarray = None) -> np.ndarray:
    """Integer-valued bf16 bits, uniform on {-8..8}.  Either a full tensor of `shape`
    or the elements at flat indices `index`."""
    i = _flat(index if index is not None else shape)
    v = ((draws(key, i) >> np.uint64(32)) % np.uint64(17)).astype(np.int64) - 8
    out = f32_to_bf16_bits(v.astype(np.float32))
    return out.reshape(shape) if index is None else out


# E4M3 bytes of the integers 0..8 (1 sign, 4 exponent bits with bias 7, 3 mantissa bits)
E4M3_OF_INT = np.array([0x00, 0x38, 0x40, 0x44, 0x48, 0x4A, 0x4C, 0x4E, 0x50], dtype=np.uint8)


def int17_e4m3(key: int, shape=None, index: np.ndarray = None) -> np.ndarray:
    """The same integers as int17_bf16 (same key, same draws), as E4M3 bytes."""
    i = _flat(index if index is not None else shape)
    v = ((draws(key, i) >> np.uint64(32)) % np.uint64(17)).astype(np.int64) - 8
    out = E4M3_OF_INT[np.abs(v)] | np.where(v < 0, np.uint8(0x80), np.uint8(0))
    out = out.astype(np.uint8)
    return out.reshape(shape) if index is None else out


def pow2_f32(key: int, shape=None, index: np.ndarray = None) -> np.ndarray:
    i = _flat(index if index is not None else shape)
    e = ((draws(key, i) >> np.uint64(32)) % np.uint64(6)).astype(np.int32)
    out = np.ldexp(np.float32(1.0), -(1 + e)).astype(np.float32)
    return out.reshape(shape) if index is None else out


def normal_bf16(key: int, shape=None, index: np.ndarray = None) -> np.ndarray:
    i = _flat(index if index is not None else shape)
    s = np.zeros(i.shape, dtype=np.int64)
    for sub in range(3):
        h = draws(key, i * np.uint64(3) + np.uint64(sub))
        for f in range(4):
            s += ((h >> np.uint64(16 * f)) & np.uint64(0xFFFF)).astype(np.int64)
    x = ((s - 393210).astype(np.float64) * 2.0 ** -16).astype(np.float32)
    out = f32_to_bf16_bits(x)
    return out.reshape(shape) if index is None else out


def unit_f32(key: int, shape=None, index: np.ndarray = None) -> np.ndarray:
    i = _flat(index if index is not None else shape)
    v = (draws(key, i) >> np.uint64(40)).astype(np.float64) * 2.0 ** -24 - 0.5
    out = v.astype(np.float32)
    return out.reshape(shape) if index is None else out


def rows_index(row_ids: np.ndarray, row_len: int) -> np.ndarray:
    """Flat element indices of whole rows (row-major tensor with rows of row_len)."""
    r = np.asarray(row_ids, dtype=np.uint64)[:, None] * np.uint64(row_len)
    return (r + np.arange(row_len, dtype=np.uint64)[None, :]).reshape(-1)
