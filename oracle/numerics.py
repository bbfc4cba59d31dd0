"""Rounding helpers and comparison metrics for the oracle (test infrastructure).

bf16 is the upper half of an IEEE binary32 word. Rounding a binary32 value to
bf16 with round-to-nearest-even is written out here on the bit pattern so a
reader can check it by eye: add 0x7FFF plus the lowest kept bit, then drop the
16 low bits. NaNs are kept quiet NaNs. No library bf16 type is used.
"""

import numpy as np


def bf16_bits(x):
    """Round float32 values to bf16 (round-to-nearest-even); return uint16 bits."""
    f = np.ascontiguousarray(np.asarray(x, dtype=np.float32))
    u = f.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    rounded = ((u + 0x7FFF + lsb) >> 16).astype(np.uint32)
    nan = np.isnan(f)
    if nan.any():
        # keep the sign and force a quiet-NaN payload bit
        rounded = np.where(nan, ((u >> 16).astype(np.uint32) | 0x0040), rounded)
    return rounded.astype(np.uint16)


def bf16_from_bits(bits):
    """Widen bf16 bit patterns (uint16) to float32 values (exact)."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32)


def bf16_round(x):
    """float32 -> nearest bf16 (ties to even), returned as float32 values."""
    return bf16_from_bits(bf16_bits(x))


def fp16_round(x):
    """float32 -> nearest binary16 (ties to even), returned as float32 values."""
    return np.asarray(x, dtype=np.float32).astype(np.float16).astype(np.float32)


def compare(y, y_ref):
    """Relative Frobenius error and max-abs error per unit RMS of the reference.

    Both are taken in fp64 over all elements: ``||y - y_ref||_F / ||y_ref||_F``
    and ``max|y - y_ref| / rms(y_ref)``.
    """
    y = np.asarray(y, dtype=np.float64)
    r = np.asarray(y_ref, dtype=np.float64)
    diff = y - r
    ref_norm = np.sqrt(np.sum(r * r))
    rms = ref_norm / np.sqrt(max(r.size, 1))
    rel_fro = float(np.sqrt(np.sum(diff * diff)) / ref_norm) if ref_norm > 0 else float(
        np.sqrt(np.sum(diff * diff)))
    max_rel = float(np.max(np.abs(diff)) / rms) if rms > 0 else float(np.max(np.abs(diff)))
    return rel_fro, max_rel


def bf16_ulp(v):
    """Spacing of bf16 numbers at |v| (for element-wise one-ulp checks).

    bf16 keeps 8 significant bits, so in the binade [2^e, 2^(e+1)) its numbers
    are 2^(e-7) apart; below 2^-126 (subnormals) they are 2^-133 apart. The
    binade comes from frexp (|v| = m 2^f with m in [0.5, 1), so e = f - 1),
    which is exact; a floating log2 can round up into the next binade for
    values just below a power of two."""
    a = np.abs(np.asarray(v, dtype=np.float64))
    a = np.maximum(a, np.finfo(np.float32).tiny)
    _, f = np.frexp(a)
    return np.ldexp(1.0, f - 1 - 7)
