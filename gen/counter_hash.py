"""Host-side counter-based generator (numpy).

Generator definition (the device twin in ``gen/device.cu`` implements the
same definition independently):

* Stream.  A tensor is identified by ``(seed, tid)``; its stream state is
  ``s0 = (seed << 32) | tid`` (both 32-bit).  Output ``i`` of the stream is
  SplitMix64 after ``i + 1`` steps: ``mix64(s0 + (i + 1) * GAMMA)`` modulo
  2**64.  SplitMix64 is the generator of Steele, Lea and Flood, "Fast
  splittable pseudorandom number generators" (OOPSLA 2014); ``mix64`` is the
  output finaliser with the constants of Stafford's "variant 13" used by the
  public-domain ``splitmix64.c``.  With ``seed = tid = 0`` this is the plain
  SplitMix64 stream seeded with 0.
* Integers in ``[lo, hi]``: element ``i`` draws ``u = out(i)`` and takes
  ``lo + floor((u >> 32) * (hi - lo + 1) / 2**32)``.
* Normal-like reals: element ``i`` draws ``out(3i)``, ``out(3i+1)``,
  ``out(3i+2)``, splits each into four 16-bit uniforms, sums the twelve into
  ``S`` and takes ``x = (S - 6 * 65536) / 65536`` (Irwin-Hall with n = 12,
  on a 2**-16 grid; mean ~0, variance ~1, support [-6, 6]).  ``x`` is exact
  in fp32 and is rounded to bfloat16 with round-to-nearest-even.

All values are returned as bfloat16 bit patterns (``uint16``).
"""
from __future__ import annotations

import numpy as np

GAMMA = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)
_MASK32 = np.uint64(0xFFFFFFFF)


def mix64(z: np.ndarray) -> np.ndarray:
    """SplitMix64 output finaliser on a uint64 array (wrapping arithmetic)."""
    z = np.asarray(z, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = (z ^ (z >> np.uint64(30))) * _M1
        z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def stream_state(seed: int, tid: int) -> np.uint64:
    if not (0 <= seed < 2**32 and 0 <= tid < 2**32):
        raise ValueError("seed and tid must be 32-bit unsigned")
    return np.uint64((seed << 32) | tid)


def stream_outputs(seed: int, tid: int, counters: np.ndarray) -> np.ndarray:
    """Outputs ``out(i)`` for each counter ``i`` (uint64 array)."""
    s0 = stream_state(seed, tid)
    c = np.asarray(counters, dtype=np.uint64)
    with np.errstate(over="ignore"):
        return mix64(s0 + (c + np.uint64(1)) * GAMMA)


def _counters(start: int, count: int | None, index: np.ndarray | None) -> np.ndarray:
    if index is not None:
        return np.asarray(index, dtype=np.uint64)
    return np.arange(start, start + count, dtype=np.uint64)


def int_values(seed: int, tid: int, start: int = 0, count: int | None = None,
               index: np.ndarray | None = None, lo: int = -4, hi: int = 4) -> np.ndarray:
    """Uniform integers in [lo, hi] for elements ``start..start+count-1``
    (or the given flat ``index`` array), as int64."""
    i = _counters(start, count, index)
    u = stream_outputs(seed, tid, i)
    span = np.uint64(hi - lo + 1)
    with np.errstate(over="ignore"):
        v = ((u >> np.uint64(32)) * span) >> np.uint64(32)
    return v.astype(np.int64) + lo


def normal_values(seed: int, tid: int, start: int = 0, count: int | None = None,
                  index: np.ndarray | None = None) -> np.ndarray:
    """Irwin-Hall(12) reals on a 2**-16 grid, as exact float64 (before bf16)."""
    i = _counters(start, count, index)
    s = np.zeros(i.shape, dtype=np.int64)
    with np.errstate(over="ignore"):
        for r in range(3):
            u = stream_outputs(seed, tid, np.uint64(3) * i + np.uint64(r))
            for c in range(4):
                s += ((u >> np.uint64(16 * c)) & np.uint64(0xFFFF)).astype(np.int64)
    return (s - 6 * 65536).astype(np.float64) / 65536.0


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float -> bfloat16 bits, round to nearest even (finite inputs only)."""
    b = np.asarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = (b + np.uint64(0x7FFF) + ((b >> np.uint64(16)) & np.uint64(1))) >> np.uint64(16)
    return r.astype(np.uint16)


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)


def e4m3_codes(x: np.ndarray) -> np.ndarray:
    """Values exactly representable in OCP FP8 E4M3 -> their codes (uint8):
    sign bit, 4-bit exponent field with bias 7 (0 for subnormals, steps of
    2^-9), 3-bit mantissa.  Zero is +0.  Raises for values E4M3 cannot hold
    exactly."""
    v = np.asarray(x, dtype=np.float64)
    a = np.abs(v)
    out = np.zeros(v.shape, dtype=np.uint8)
    nz = a > 0
    e = np.floor(np.log2(np.where(nz, a, 1.0))).astype(np.int64)
    normal = nz & (e >= -6)
    m_norm = (a / np.exp2(e.astype(np.float64)) - 1.0) * 8.0
    m_sub = a / 2.0 ** -9
    m = np.where(normal, m_norm, m_sub)
    ok = ~nz | ((m == np.round(m)) & np.where(normal, (e <= 8) & (m <= 7) & ~((e == 8) & (m == 7)), m <= 7))
    if not ok.all():
        raise ValueError("values not exactly representable in E4M3")
    field = np.where(normal, e + 7, 0)
    code = (np.where(v < 0, 0x80, 0) | (field << 3) | np.round(m).astype(np.int64)).astype(np.uint8)
    return np.where(nz, code, 0).astype(np.uint8)


def int_e4m3(seed: int, tid: int, start: int = 0, count: int | None = None,
             index: np.ndarray | None = None, lo: int = -4, hi: int = 4) -> np.ndarray:
    """The integer values of int_bf16 (same stream), as E4M3 codes."""
    return e4m3_codes(int_values(seed, tid, start, count, index, lo, hi))


def int_bf16(seed: int, tid: int, start: int = 0, count: int | None = None,
             index: np.ndarray | None = None, lo: int = -4, hi: int = 4) -> np.ndarray:
    """Integer values stored as bfloat16 bits (exact for |v| <= 256)."""
    return f32_to_bf16_bits(int_values(seed, tid, start, count, index, lo, hi))


def normal_bf16(seed: int, tid: int, start: int = 0, count: int | None = None,
                index: np.ndarray | None = None) -> np.ndarray:
    return f32_to_bf16_bits(normal_values(seed, tid, start, count, index))
