"""Seeded synthetic inputs for the tests, the smoke check and the benchmark.

Every element is a pure function of ``(key, flat_index)``: a SplitMix64 counter
stream (the generator of Steele, Lea and Flood, "Fast splittable pseudorandom
number generators", OOPSLA 2014, with the finaliser constants of Vigna's public
``splitmix64``) gives a 32-bit uniform ``r``, and ``r`` is mapped to a bf16 value
by an inverse-CDF table of the standard normal distribution quantised to bf16
with round-to-nearest-even.  A value therefore has exactly the law of
``RN_bf16(N(0, 1))`` (up to the 2^-32 resolution of ``r``).

The mapping uses only integer arithmetic and a table lookup, so the device
generator in ``csrc/synth.cu`` produces the same bytes from the same table;
``tests/test_gpu_synth.py`` checks that on the GPU.  Any subset of a tensor can
be regenerated on its own (the oracle side of a full-size parity test draws only
the heads it checks).

This module holds no attention, cache or Euler arithmetic.
"""
from __future__ import annotations

import math
from functools import lru_cache

import numpy as np

MASK64 = (1 << 64) - 1
GOLDEN_GAMMA = 0x9E3779B97F4A7C15
_MIX1 = 0xBF58476D1CE4E5B9
_MIX2 = 0x94D049BB133111EB

# Stream kinds: one per logical input tensor of the unit step.
KIND_Q = 1
KIND_K_NEW = 2
KIND_V_NEW = 3
KIND_COND_K = 4
KIND_COND_V = 5
KIND_COMMIT_K = 6
KIND_COMMIT_V = 7
KIND_X = 8
KIND_VEL = 9
KIND_MISC = 10


def _mix_scalar(z: int) -> int:
    z &= MASK64
    z = ((z ^ (z >> 30)) * _MIX1) & MASK64
    z = ((z ^ (z >> 27)) * _MIX2) & MASK64
    return z ^ (z >> 31)


def stream_key(seed: int, kind: int, unit: int = 0, layer: int = 0, step: int = 0) -> int:
    """64-bit key of one logical tensor.  Fields are packed, then mixed with the seed."""
    if not (0 <= kind < 256 and 0 <= layer < 65536 and 0 <= step < 256):
        raise ValueError("stream field out of range")
    sid = kind | (layer << 8) | (step << 24) | ((unit & 0xFFFFFFFF) << 32)
    return _mix_scalar((seed * GOLDEN_GAMMA + _mix_scalar(sid)) & MASK64)


def uniform_u32(key: int, idx: np.ndarray) -> np.ndarray:
    """Top 32 bits of the SplitMix64 output for counter ``idx`` (uint64 array)."""
    idx = np.asarray(idx, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = np.uint64(key) + (idx + np.uint64(1)) * np.uint64(GOLDEN_GAMMA)
        z = (z ^ (z >> np.uint64(30))) * np.uint64(_MIX1)
        z = (z ^ (z >> np.uint64(27))) * np.uint64(_MIX2)
        z = z ^ (z >> np.uint64(31))
    return (z >> np.uint64(32)).astype(np.uint32)


def _bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint32) << 16).view(np.float32).astype(np.float64)


@lru_cache(maxsize=1)
def normal_table() -> tuple[np.ndarray, np.ndarray]:
    """(thresholds uint64 ascending, bf16 bit patterns uint16).

    Entry k receives the uniforms ``thresholds[k-1] <= r < thresholds[k]``: the
    2^32-scaled normal probability of the reals that round (RNE) to value k.
    Values whose scaled mass rounds to zero are dropped.
    """
    bits = np.arange(0, 0x7F80, dtype=np.uint32)          # +0 .. largest finite
    pos = _bf16_bits_to_f64(bits)
    neg = -pos[1:][::-1]                                   # no -0: it is the same real as +0
    vals = np.concatenate([neg, pos])
    vbits = np.concatenate([(bits[1:][::-1] | 0x8000), bits]).astype(np.uint16)
    mids = 0.5 * (vals[:-1] + vals[1:])                    # exact in fp64
    cdf = np.array([0.5 * math.erfc(-m / math.sqrt(2.0)) for m in mids])
    thr = np.rint(cdf * 4294967296.0).astype(np.uint64)
    thr = np.append(thr, np.uint64(1 << 32))
    prev = np.concatenate([[np.uint64(0)], thr[:-1]])
    keep = thr > prev
    return thr[keep].copy(), vbits[keep].copy()


def normal_bf16(key: int, idx: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) of the elements at flat indices ``idx`` of stream ``key``."""
    thr, vb = normal_table()
    r = uniform_u32(key, idx).astype(np.uint64)
    return vb[np.searchsorted(thr, r, side="right")]


def normal_tensor(key: int, shape, offset: int = 0) -> np.ndarray:
    """A whole tensor (flat indices offset .. offset+size-1) as uint16 bf16 bits."""
    n = int(np.prod(shape)) if len(shape) else 1
    idx = np.arange(offset, offset + n, dtype=np.uint64)
    return normal_bf16(key, idx).reshape(shape)


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float64 (for statistics in tests)."""
    return _bf16_bits_to_f64(bits)
