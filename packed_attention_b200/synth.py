"""Seeded synthetic inputs for the packed joint text+image attention forward.

This module holds only random-number generation and bf16 rounding. It holds
none of the method's arithmetic (no normalisation, rotation or attention), so
both the CUDA path and the fp64 oracle can be fed from it without sharing any
computation.

Generator
---------
* Uniform 64-bit words: SplitMix64 (Steele, Lea & Flood, "Fast splittable
  pseudorandom number generators", OOPSLA 2014). Its n-th output is a pure
  function of ``key + n * 0x9E3779B97F4A7C15`` passed through the published
  64-bit finaliser, so a stream can be evaluated at any counter in parallel.
  Each (seed, stream id) pair gets its own key.
* Normals: Box-Muller in fp64 on consecutive pairs of words,
  ``u1 = (w0 >> 11 + 1) * 2^-53`` in (0, 1], ``u2 = (w1 >> 11) * 2^-53``,
  ``z0 = sqrt(-2 ln u1) cos(2 pi u2)``, ``z1 = sqrt(-2 ln u1) sin(2 pi u2)``.
* bf16: round-to-nearest-even directly from fp64 (one rounding).
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

_GOLDEN = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)
_CHUNK = 1 << 22

# Stream ids: one independent SplitMix64 stream per drawn quantity.
STREAM_Q, STREAM_K, STREAM_V = 0, 1, 2
STREAM_GQ_TEXT, STREAM_GQ_IMG, STREAM_GK_TEXT, STREAM_GK_IMG = 3, 4, 5, 6
STREAM_OUTLIER_ROWS = 7


def _mix64(z: np.ndarray) -> np.ndarray:
    """SplitMix64 finaliser on a uint64 array (wrapping arithmetic)."""
    z = (z ^ (z >> np.uint64(30))) * _M1
    z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def _stream_key(seed: int, stream: int) -> np.uint64:
    base = np.array([(seed * 0x100000001B3 + stream * 0x632BE59BD9B4E019) & 0xFFFFFFFFFFFFFFFF],
                    dtype=np.uint64)
    with np.errstate(over="ignore"):
        return _mix64(base)[0]


def splitmix64(seed: int, stream: int, n: int, offset: int = 0) -> np.ndarray:
    """Outputs ``offset+1 .. offset+n`` of the SplitMix64 stream (seed, stream)."""
    key = _stream_key(seed, stream)
    out = np.empty(n, dtype=np.uint64)
    with np.errstate(over="ignore"):
        for lo in range(0, n, _CHUNK):
            hi = min(n, lo + _CHUNK)
            idx = np.arange(offset + lo + 1, offset + hi + 1, dtype=np.uint64)
            out[lo:hi] = _mix64(key + idx * _GOLDEN)
    return out


def normals(seed: int, stream: int, n: int) -> np.ndarray:
    """``n`` standard normal fp64 values from stream (seed, stream), Box-Muller.

    Chunks are independent (the stream is counter-based), so they are filled
    by a thread pool; the result does not depend on the thread count.
    """
    m = (n + 1) // 2
    out = np.empty(2 * m, dtype=np.float64)
    two_pi = 2.0 * np.pi

    def fill(lo):
        hi = min(m, lo + _CHUNK)
        w = splitmix64(seed, stream, 2 * (hi - lo), offset=2 * lo)
        u1 = ((w[0::2] >> np.uint64(11)) + np.uint64(1)).astype(np.float64) * 2.0 ** -53
        u2 = (w[1::2] >> np.uint64(11)).astype(np.float64) * 2.0 ** -53
        r = np.sqrt(-2.0 * np.log(u1))
        out[2 * lo:2 * hi:2] = r * np.cos(two_pi * u2)
        out[2 * lo + 1:2 * hi:2] = r * np.sin(two_pi * u2)

    starts = list(range(0, m, _CHUNK))
    if len(starts) > 1:
        with ThreadPoolExecutor(max_workers=min(len(starts), os.cpu_count() or 1)) as ex:
            list(ex.map(fill, starts))
    elif starts:
        fill(0)
    return out[:n]


def f64_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp64 to bf16 (round-to-nearest-even, one rounding), as uint16 bits.

    Valid for zero and for magnitudes in bf16's normal range, which covers every
    value drawn here; anything else raises.
    """
    x = np.ascontiguousarray(x, dtype=np.float64)
    ax = np.abs(x)
    bad = (ax != 0) & ((ax < 2.0 ** -126) | (ax >= 2.0 ** 128) | ~np.isfinite(ax))
    if np.any(bad):
        raise ValueError("value outside the bf16 normal range")
    bits = x.view(np.uint64)
    # fp64 has 52 stored fraction bits, bf16 has 7: drop 45 with RNE.
    lsb = (bits >> np.uint64(45)) & np.uint64(1)
    rounded = (bits + np.uint64((1 << 44) - 1) + lsb) & ~np.uint64((1 << 45) - 1)
    f32 = rounded.view(np.float64).astype(np.float32)  # exact: 8 significant bits
    return (f32.view(np.uint32) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f64(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def choose_rows(seed: int, stream: int, n_total: int, n_pick: int) -> np.ndarray:
    """``n_pick`` distinct indices of [0, n_total): the smallest hashed keys win."""
    keys = splitmix64(seed, stream, n_total)
    order = np.lexsort((np.arange(n_total), keys))
    return np.sort(order[:n_pick]).astype(np.int64)
