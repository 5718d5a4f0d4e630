"""Exact-rational arithmetic used to pin the fp64 oracle (test helper).

Everything here is written independently of ``oracle/far_oracle.c``: values
are Python ``Fraction``s, rounding is done on rationals, and the one square
root is bracketed with ``decimal`` at 60 significant digits.  The formats
follow their published definitions (bfloat16 1-8-7, IEEE binary16 1-5-10,
binary32 1-8-23, OCP FP8 E4M3 "fn" 1-4-3 with max 448 and no infinity).
"""
from __future__ import annotations

from decimal import Decimal, localcontext
from fractions import Fraction

# (significand bits incl. the hidden one, exponent of the smallest normal,
#  largest finite value, exponent-field bias, stored fraction bits)
FORMATS = {
    "bf16": (8, -126, (2 - Fraction(1, 2 ** 7)) * Fraction(2) ** 127, 127, 7),
    "fp16": (11, -14, Fraction(65504), 15, 10),
    "fp32": (24, -126, (2 - Fraction(1, 2 ** 23)) * Fraction(2) ** 127, 127, 23),
    "e4m3": (4, -6, Fraction(448), 7, 3),
}

INF = float("inf")


def floor_log2(a: Fraction) -> int:
    """Largest e with 2**e <= a, for a > 0."""
    e = a.numerator.bit_length() - a.denominator.bit_length()
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    return e


def rne(x: Fraction, fmt: str):
    """Round x to the nearest value of ``fmt``, ties to even.

    Returns a Fraction, or +-INF when the rounded magnitude exceeds the
    largest finite value (e4m3 saturates instead, as the satfinite reading
    requires)."""
    p, emin, maxv, _, _ = FORMATS[fmt]
    if x == 0:
        return Fraction(0)
    s = -1 if x < 0 else 1
    a = abs(x)
    e = max(floor_log2(a), emin)
    q = Fraction(2) ** (e - (p - 1))
    n = a / q
    fl = n.numerator // n.denominator
    rem = n - fl
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2 == 1):
        fl += 1
    v = fl * q
    if v > maxv:
        if fmt == "e4m3":
            return s * maxv
        return s * INF
    return s * v


def e4m3_sat(x: Fraction) -> Fraction:
    """e4m3 with saturation of any magnitude >= 448 (also for huge inputs)."""
    if abs(x) >= 448:
        return Fraction(448) if x > 0 else Fraction(-448)
    return rne(x, "e4m3")


def encode(v, fmt: str, negative_zero: bool = False) -> int:
    """Bit pattern of a value that is exactly representable in ``fmt``."""
    p, emin, maxv, bias, mbits = FORMATS[fmt]
    width = {"bf16": 16, "fp16": 16, "fp32": 32, "e4m3": 8}[fmt]
    ebits = width - 1 - mbits
    sign_bit = 1 << (width - 1)
    if v == INF or v == -INF:
        assert fmt != "e4m3"
        return (sign_bit if v < 0 else 0) | (((1 << ebits) - 1) << mbits)
    v = Fraction(v)
    sign = sign_bit if (v < 0 or (v == 0 and negative_zero)) else 0
    a = abs(v)
    if a == 0:
        return sign
    e = floor_log2(a)
    if e < emin:
        m = a / Fraction(2) ** (emin - mbits)
        assert m.denominator == 1, "not representable"
        return sign | int(m)
    m = (a / Fraction(2) ** e - 1) * 2 ** mbits
    assert m.denominator == 1, "not representable"
    return sign | ((e + bias) << mbits) | int(m)


def decode(bits: int, fmt: str):
    """Exact value of a bit pattern (None for NaN, +-INF for infinities)."""
    p, emin, maxv, bias, mbits = FORMATS[fmt]
    width = {"bf16": 16, "fp16": 16, "fp32": 32, "e4m3": 8}[fmt]
    ebits = width - 1 - mbits
    sign = -1 if (bits >> (width - 1)) & 1 else 1
    E = (bits >> mbits) & ((1 << ebits) - 1)
    M = bits & ((1 << mbits) - 1)
    if fmt == "e4m3":
        if E == 0xF and M == 0x7:
            return None
    elif E == (1 << ebits) - 1:
        return None if M else sign * INF
    if E == 0:
        return sign * Fraction(M) * Fraction(2) ** (emin - mbits)
    return sign * (1 + Fraction(M, 2 ** mbits)) * Fraction(2) ** (E - bias)


def inv_sqrt_bracket(x: Fraction, digits: int = 60):
    """(lo, hi) Fractions with lo <= 1/sqrt(x) <= hi, hi/lo - 1 < 1e-(digits-3)."""
    with localcontext() as ctx:
        ctx.prec = digits
        d = Decimal(x.numerator) / Decimal(x.denominator)
        r = Decimal(1) / d.sqrt()
    r = Fraction(r)
    tol = Fraction(1, 10 ** (digits - 4))
    return r * (1 - tol), r * (1 + tol)


def rne_bracket(lo: Fraction, hi: Fraction, fmt: str):
    """Correctly rounded value of any number in [lo, hi], or None when the
    bracket straddles a rounding boundary (then the test skips that element)."""
    a, b = rne(lo, fmt), rne(hi, fmt)
    return a if a == b else None


def f32(x: float) -> Fraction:
    """The fp32 value of a Python float (as numpy.float32 would store it)."""
    import struct
    return Fraction(struct.unpack("<f", struct.pack("<f", x))[0])
