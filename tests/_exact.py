"""Exact-arithmetic helpers for pinning the oracle (pure Python, no numpy math).

These re-derive IEEE binary32 rounding from its definition with
``fractions.Fraction`` so that the oracle's numpy arithmetic can be checked
against something other than itself.
"""
from __future__ import annotations

import math
import struct
from fractions import Fraction

F32_MANT = 23
F32_EMIN = -126          # smallest normal exponent
F32_EMAX = 127
SUB_ULP = Fraction(1, 2 ** 149)


def f32_bits(v: float) -> int:
    return struct.unpack("<I", struct.pack("<f", v))[0]


def f32_from_bits(u: int) -> float:
    return struct.unpack("<f", struct.pack("<I", u))[0]


def frac_of_f32(v: float) -> Fraction:
    """Exact value of a binary32 (given as a Python float holding it)."""
    return Fraction(v)


def round_to_f32(r: Fraction) -> Fraction:
    """Round an exact rational to the nearest binary32, ties to even.

    Returns the exact value (as Fraction) or raises OverflowError when the
    result is not finite.  Written from the definition: pick the exponent of
    |r|, scale so the significand has 24 bits (or use the fixed subnormal
    spacing 2^-149), round the scaled value half-to-even.
    """
    if r == 0:
        return Fraction(0)
    sign = -1 if r < 0 else 1
    a = abs(r)
    # exponent e with 2^e <= a < 2^(e+1)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    if e < F32_EMIN:
        spacing = SUB_ULP
    else:
        spacing = Fraction(2) ** (e - F32_MANT)
    m = round(a / spacing)            # Python rounds Fractions half to even
    v = m * spacing
    if v >= Fraction(2) ** (F32_EMAX + 1):
        raise OverflowError("rounds to infinity")
    return sign * v


def exact_scale(row, b: int) -> Fraction:
    """fl32(max|w| / Q) by exact arithmetic; zero row -> fl32(1/Q)."""
    Q = (1 << (b - 1)) - 1
    m = max((abs(Fraction(float(v))) for v in row), default=Fraction(0))
    if m == 0:
        return round_to_f32(Fraction(1, Q))
    return round_to_f32(m / Q)


def exact_codes(row, b: int):
    """Codes of one row by exact arithmetic (see the oracle's readings)."""
    Q = (1 << (b - 1)) - 1
    s = exact_scale(row, b)
    out = []
    for v in row:
        w = Fraction(float(v))
        if s == 0:
            out.append(0 if w == 0 else (Q if w > 0 else -Q))
            continue
        try:
            t = round_to_f32(w / s)
        except OverflowError:
            out.append(Q if w > 0 else -Q)
            continue
        q = round(t)                   # half to even
        out.append(max(-Q, min(Q, q)))
    return out, s


def pack_row_int(codes, b: int, K: int) -> bytes:
    """Canonical packed row built as one big Python integer."""
    acc = 0
    for k, q in enumerate(codes):
        acc |= (q % (1 << b)) << (k * b)
    rb = 16 * math.ceil(K * b / 128)
    return acc.to_bytes(rb, "little")


def unpack_row_int(data: bytes, b: int, K: int):
    acc = int.from_bytes(data, "little")
    out = []
    for k in range(K):
        u = (acc >> (k * b)) & ((1 << b) - 1)
        out.append(u - (1 << b) if u >= (1 << (b - 1)) else u)
    return out


def pack_paired_row_int(codes, b: int) -> bytes:
    """Paired-halves row written with Python integers: per 32-code group, the
    even codes form one integer stream and the odd codes another; each 32-bit
    word takes 16 bits of each, low half from the even stream."""
    assert len(codes) % 32 == 0
    mask = (1 << b) - 1
    words = []
    for g0 in range(0, len(codes), 32):
        even = 0
        odd = 0
        for i in range(16):
            even += (codes[g0 + 2 * i] & mask) * 2 ** (i * b)
            odd += (codes[g0 + 2 * i + 1] & mask) * 2 ** (i * b)
        for h in range(b):
            lo = (even // 2 ** (16 * h)) % 2 ** 16
            hi = (odd // 2 ** (16 * h)) % 2 ** 16
            words.append(lo + hi * 2 ** 16)
    return b"".join(w.to_bytes(4, "little") for w in words)
