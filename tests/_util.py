"""Small helpers for the tests: fixtures, exact binary32 rounding of
rationals, INT4 unpacking.  None of this is the operator's arithmetic."""
import json
import os
from fractions import Fraction

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def f32_of_fraction(fr: Fraction) -> np.float32:
    """Exact round-to-nearest-even of a rational to binary32 (normal range)."""
    fr = Fraction(fr)
    if fr == 0:
        return np.float32(0.0)
    sign = -1 if fr < 0 else 1
    a = abs(fr)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    # a in [2^e, 2^(e+1)); keep 24 significant bits
    m = a / Fraction(2) ** (e - 23)
    fl = m.numerator // m.denominator
    rem = m - fl
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2 == 1):
        fl += 1
    return np.float32(sign * float(Fraction(fl) * Fraction(2) ** (e - 23)))


def unpack_int4(packed: np.ndarray) -> np.ndarray:
    """Packed bytes [..., n/2] -> signed codes [..., n]; the even index sits in
    the low nibble, nibbles are two's complement."""
    p = np.asarray(packed, dtype=np.uint8)
    lo = (p & 0xF).astype(np.int16)
    hi = (p >> 4).astype(np.int16)
    lo = np.where(lo >= 8, lo - 16, lo)
    hi = np.where(hi >= 8, hi - 16, hi)
    out = np.empty(p.shape[:-1] + (p.shape[-1] * 2,), np.int16)
    out[..., 0::2] = lo
    out[..., 1::2] = hi
    return out


def unpack_int4_words(words: np.ndarray) -> np.ndarray:
    """32-bit words [..., n/8] -> signed codes [..., n]: code k of a word is its
    bits 4k..4k+3, a two's-complement nibble (shifts on the word value, not a
    reading of its bytes)."""
    w = np.asarray(words).view(np.uint32).astype(np.int64)
    out = np.empty(w.shape[:-1] + (w.shape[-1] * 8,), np.int16)
    for k in range(8):
        nib = (w >> (4 * k)) & 0xF
        out[..., k::8] = np.where(nib >= 8, nib - 16, nib)
    return out


def codes(y, qdtype):
    """Signed integer codes of an output tensor (int8 as is; INT4 unpacked)."""
    if qdtype == "int8":
        return np.asarray(y).view(np.int8).astype(np.int16)
    if qdtype == "int4_int32":
        return unpack_int4_words(y)
    return unpack_int4(y)
