"""Exact-arithmetic helpers for pinning the oracle (test-only).

These restate IEEE-754 rounding and the LSB-first bitstream with Python
integers and fractions, so that the oracle's C arithmetic is checked against
a computation that shares none of its machinery.
"""
from __future__ import annotations

import math
import struct
from fractions import Fraction

import numpy as np


def f32_bits(v: float) -> int:
    return struct.unpack("<I", struct.pack("<f", v))[0]


def round_binary(fr: Fraction, mant_bits: int, emin: int) -> Fraction:
    """Round a rational to the nearest binary floating value with `mant_bits`
    significant bits (incl. the implicit one), ties to even; subnormals below
    2**emin.  Overflow is not handled (callers stay in range)."""
    if fr == 0:
        return Fraction(0)
    sign = -1 if fr < 0 else 1
    a = abs(fr)
    e = math.floor(math.log2(a.numerator) - math.log2(a.denominator))
    # fix up floating log2 error
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    e = max(e, emin)
    quantum = Fraction(2) ** (e - (mant_bits - 1))
    q = a / quantum
    n = q.numerator // q.denominator
    rem = q - n
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and n % 2 == 1):
        n += 1
    return sign * n * quantum


def rf32(fr) -> Fraction:
    return round_binary(Fraction(fr), 24, -126)


def rbf16(fr) -> Fraction:
    return round_binary(Fraction(fr), 8, -126)


def rf16(fr) -> Fraction:
    return round_binary(Fraction(fr), 11, -14)


def round_half_away(fr: Fraction) -> int:
    n = math.floor(abs(fr) + Fraction(1, 2))
    return n if fr >= 0 else -n


def pack_bigint(codes, bits: int) -> list[int]:
    """LSB-first bitstream: code i at bits [i*bits, (i+1)*bits) of one big integer,
    cut into little-endian 32-bit words."""
    stream = 0
    for i, q in enumerate(codes):
        stream |= int(q) << (i * bits)
    nw = len(codes) * bits // 32
    return [(stream >> (32 * j)) & 0xFFFFFFFF for j in range(nw)]


def unpack_bigint(words, bits: int, n: int) -> list[int]:
    stream = 0
    for j, w in enumerate(words):
        stream |= int(w) << (32 * j)
    mask = (1 << bits) - 1
    return [(stream >> (i * bits)) & mask for i in range(n)]


def bf16_bits_to_fraction(h: int) -> Fraction:
    return Fraction(float(np.array([int(h) << 16], dtype=np.uint32).view(np.float32)[0]))


def f16_bits_to_fraction(h: int) -> Fraction:
    return Fraction(float(np.array([int(h)], dtype=np.uint16).view(np.float16)[0]))


def storage_to_fraction(v, dtype: str) -> Fraction:
    if dtype == "f32":
        return Fraction(float(np.float32(v)))
    if dtype == "bf16":
        return bf16_bits_to_fraction(int(v))
    return f16_bits_to_fraction(int(v))
