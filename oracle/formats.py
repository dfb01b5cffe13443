"""Element and scale codes used by SharQ's FP4 formats: E2M1, E4M3 and E8M0.

TEST INFRASTRUCTURE. This module is part of the CPU oracle: only ``tests/``,
``__graft_entry__.smoke()`` and the ``cpu_baseline`` / ``--impl reference``
legs of ``bench.py`` may import it. The product path never does.

The SharQ pages name the formats (NVFP4, MXFP4; "SharQ: Bridging Activation
Sparsity and FP4 Quantization for LLM Inference", Abstract) but never define
them. The definitions below are the public ones:

* E2M1 (FP4): 1 sign, 2 exponent (bias 1), 1 mantissa bit, no inf/NaN;
  magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6 (OCP Microscaling Formats v1.0,
  section "FP4 E2M1").
* E4M3: 1 sign, 4 exponent (bias 7), 3 mantissa bits, max 448, no inf,
  S.1111.111 is NaN, subnormals down to 2^-9 (OCP 8-bit Floating Point
  Specification, "E4M3").
* E8M0: 8 exponent bits, value 2^(e-127), 0xFF is NaN (OCP Microscaling
  Formats v1.0, "E8M0 scale").

Encoders round to nearest with ties to the even code (the code whose
lowest bit is 0) and saturate finite values beyond the largest magnitude to
it ("satfinite"). The sign bit of the input is kept, so a negative input
that rounds to zero encodes as negative zero. NaN inputs are outside the
contract. Tables are built by enumerating codes; encoding searches them, so
a reader can check every step by hand.
"""
from __future__ import annotations

import numpy as np


def _e2m1_magnitude(code: int) -> float:
    """Magnitude of the 3 low bits of an E2M1 code, from the bit fields."""
    e = (code >> 1) & 0x3
    m = code & 0x1
    if e == 0:  # subnormal: m * 2^(1-bias) * 1/2 with bias 1
        return m * 0.5
    return (1.0 + m / 2.0) * 2.0 ** (e - 1)


def _e4m3_magnitude(code: int) -> float:
    """Magnitude of the 7 low bits of an E4M3 code (0x7F is NaN)."""
    e = (code >> 3) & 0xF
    m = code & 0x7
    if e == 0xF and m == 0x7:
        return float("nan")
    if e == 0:  # subnormal: m/8 * 2^(1-7)
        return (m / 8.0) * 2.0 ** -6
    return (1.0 + m / 8.0) * 2.0 ** (e - 7)


# Magnitudes indexed by the code's low bits; ascending, so index == code.
E2M1_MAGNITUDES = np.array([_e2m1_magnitude(c) for c in range(8)], dtype=np.float64)
E4M3_MAGNITUDES = np.array([_e4m3_magnitude(c) for c in range(127)], dtype=np.float64)  # 0x00..0x7E
E2M1_MAX = float(E2M1_MAGNITUDES[-1])   # 6
E4M3_MAX = float(E4M3_MAGNITUDES[-1])   # 448


def _rne_search(mag: np.ndarray, table: np.ndarray) -> np.ndarray:
    """Index of the nearest table entry to each non-negative ``mag``.

    Ties go to the even index; values above the last entry saturate to it.
    ``mag`` and ``table`` are float64 and every difference taken here is exact
    (the inputs are float32 values, the tables small dyadic rationals).
    """
    mag = np.asarray(mag, dtype=np.float64)
    hi = np.searchsorted(table, mag, side="left")          # table[hi] >= mag
    hi = np.minimum(hi, len(table) - 1)                     # saturate
    lo = np.maximum(hi - 1, 0)
    d_lo = mag - table[lo]
    d_hi = table[hi] - mag
    out = np.where(d_lo < d_hi, lo, hi)
    tie = (d_lo == d_hi) & (lo != hi)
    even = np.where(lo % 2 == 0, lo, hi)
    out = np.where(tie, even, out)
    # exact hits and saturation: table[hi] == mag, or mag beyond the last entry
    out = np.where(table[hi] == mag, hi, out)
    out = np.where(mag > table[-1], len(table) - 1, out)
    return out.astype(np.uint8)


def e2m1_encode(v) -> np.ndarray:
    """E2M1 code (uint8 in 0..15) of each float32 value: RNE, satfinite, signed zero kept."""
    v = np.asarray(v, dtype=np.float32)
    sign = np.signbit(v).astype(np.uint8) << 3
    return (_rne_search(np.abs(v).astype(np.float64), E2M1_MAGNITUDES) | sign).astype(np.uint8)


def e2m1_decode(code) -> np.ndarray:
    """Value (float64) of each E2M1 code."""
    code = np.asarray(code, dtype=np.uint8)
    mag = E2M1_MAGNITUDES[code & 0x7]
    return np.where((code & 0x8) != 0, -mag, mag)


def e4m3_encode(v) -> np.ndarray:
    """E4M3 code (uint8) of each float32 value: RNE, satfinite to 448, signed zero kept."""
    v = np.asarray(v, dtype=np.float32)
    sign = np.signbit(v).astype(np.uint8) << 7
    return (_rne_search(np.abs(v).astype(np.float64), E4M3_MAGNITUDES) | sign).astype(np.uint8)


def e4m3_decode(code) -> np.ndarray:
    """Value (float64) of each E4M3 code; 0x7F / 0xFF decode to NaN."""
    code = np.asarray(code, dtype=np.uint8)
    low = code & 0x7F
    mag = np.where(low == 0x7F, np.nan, E4M3_MAGNITUDES[np.minimum(low, 126)])
    return np.where((code & 0x80) != 0, -mag, mag)


def e8m0_decode(code) -> np.ndarray:
    """Value (float64) of each E8M0 scale code: 2^(e-127); 0xFF is NaN."""
    code = np.asarray(code, dtype=np.int64)
    return np.where(code == 0xFF, np.nan, np.ldexp(1.0, code - 127))
