"""Counter-based random numbers for the synthetic workloads.

Every random value used by the tests and the benchmark comes from here, so
that the oracle and the CUDA library are fed identical inputs.  The module
holds no arithmetic of the ranking method itself: only integer hashing,
uniform and normal variates, and sampling helpers.

Generator (stated so it can be re-implemented elsewhere):

* ``mix(z)`` is the SplitMix64 output function (Steele, Lea and Flood,
  "Fast splittable pseudorandom number generators", OOPSLA 2014):
  ``z ^= z >> 30; z *= 0xBF58476D1CE4E5B9; z ^= z >> 27;
  z *= 0x94D049BB133111EB; z ^= z >> 31`` (all mod 2**64).
* A stream is named by ``(seed, tag)``; its key is
  ``mix(seed + (tag + 1) * G)`` with ``G = 0x9E3779B97F4A7C15``.
* Element ``i`` of the stream is ``mix(key + (i + 1) * G)``, i.e. the
  ``i``-th output of a SplitMix64 generator whose state starts at ``key``.
* Uniform doubles in [0, 1) take the top 53 bits: ``(u >> 11) * 2**-53``.
* Normals use the Box-Muller transform on consecutive uniform pairs
  ``(u1, u2)``: ``r = sqrt(-2 ln(1 - u1))``, giving ``r cos(2 pi u2)`` and
  ``r sin(2 pi u2)`` as elements ``2j`` and ``2j + 1``.
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

GOLDEN = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)


def mix(z: np.ndarray) -> np.ndarray:
    """SplitMix64 output function, elementwise on uint64 (wrapping)."""
    z = np.asarray(z, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = (z ^ (z >> np.uint64(30))) * _M1
        z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def stream_key(seed: int, tag: int) -> np.uint64:
    with np.errstate(over="ignore"):
        base = np.uint64(seed % 2**64) + np.uint64((tag + 1) % 2**64) * GOLDEN
    return np.uint64(mix(np.array([base], dtype=np.uint64))[0])


class Stream:
    """One counter-based stream; each call hands out the next elements."""

    def __init__(self, seed: int, tag: int):
        self.key = stream_key(seed, tag)
        self.pos = 0

    def u64(self, n: int) -> np.ndarray:
        idx = np.arange(self.pos + 1, self.pos + 1 + n, dtype=np.uint64)
        self.pos += n
        with np.errstate(over="ignore"):
            return mix(self.key + idx * GOLDEN)

    def _u64_at(self, start: int, n: int) -> np.ndarray:
        idx = np.arange(start + 1, start + 1 + n, dtype=np.uint64)
        with np.errstate(over="ignore"):
            return mix(self.key + idx * GOLDEN)

    def uniform(self, n: int) -> np.ndarray:
        """n doubles uniform in [0, 1)."""
        return (self.u64(n) >> np.uint64(11)).astype(np.float64) * (2.0 ** -53)

    def _normal_at(self, start_pair: int, pairs: int) -> np.ndarray:
        u = (self._u64_at(2 * start_pair, 2 * pairs) >> np.uint64(11)).astype(np.float64)
        u = (u * (2.0 ** -53)).reshape(pairs, 2)
        r = np.sqrt(-2.0 * np.log1p(-u[:, 0]))
        ang = (2.0 * np.pi) * u[:, 1]
        z = np.empty((pairs, 2), dtype=np.float64)
        z[:, 0] = r * np.cos(ang)
        z[:, 1] = r * np.sin(ang)
        return z.reshape(-1)

    def normal(self, n: int, chunk_pairs: int = 1 << 21) -> np.ndarray:
        """n standard normals (Box-Muller on uniform pairs), float64.

        Element 2j and 2j+1 come from uniforms 2j and 2j+1 of the stream, so
        the chunks are independent and are computed on a thread pool."""
        if self.pos % 2:
            self.pos += 1  # normals start on an even element
        pairs = (n + 1) // 2
        first = self.pos // 2
        out = np.empty(2 * pairs, dtype=np.float64)
        starts = list(range(0, pairs, chunk_pairs))

        def work(c0):
            c1 = min(c0 + chunk_pairs, pairs)
            out[2 * c0:2 * c1] = self._normal_at(first + c0, c1 - c0)

        if len(starts) == 1:
            work(0)
        else:
            with ThreadPoolExecutor(max_workers=min(len(starts), os.cpu_count() or 1)) as ex:
                list(ex.map(work, starts))
        self.pos += 2 * pairs
        return out[:n]

    def integers(self, n: int, low: int, high: int) -> np.ndarray:
        """n integers uniform in [low, high) (multiply-shift on 53-bit uniforms)."""
        span = high - low
        if span <= 0:
            raise ValueError("empty range")
        v = np.floor(self.uniform(n) * span).astype(np.int64)
        return np.minimum(v, span - 1) + low

    def distinct(self, n: int, low: int, high: int, exclude=()) -> np.ndarray:
        """n distinct integers in [low, high), none in ``exclude``, in draw order.

        Draws one at a time and redraws on a collision, so the result does
        not depend on how many values are requested later.
        """
        if high - low - len(set(exclude)) < n:
            raise ValueError("range too small for distinct draw")
        seen = set(int(e) for e in exclude)
        out = []
        while len(out) < n:
            v = int(self.integers(1, low, high)[0])
            if v not in seen:
                seen.add(v)
                out.append(v)
        return np.array(out, dtype=np.int64)


def bf16_round(x: np.ndarray) -> np.ndarray:
    """Round float values to the nearest bfloat16 (ties to even), returned as
    uint16 bit patterns.  Input is first rounded to float32 (exact for the
    N(0, 0.02) draws up to that rounding); NaN does not occur here."""
    f = np.ascontiguousarray(np.asarray(x, dtype=np.float32))
    b = f.view(np.uint32)
    lsb = (b >> np.uint32(16)) & np.uint32(1)
    # finite inputs stay below 2**32 after the bias (largest is 0xFF7FFFFF + 0x8000)
    b = (b + np.uint32(0x7FFF) + lsb) >> np.uint32(16)
    return b.astype(np.uint16)


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bfloat16 bit patterns to float32."""
    b = np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32)


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bfloat16 bit patterns to float64."""
    return bf16_to_f32(bits).astype(np.float64)
