"""Exact-rational reference rounding for the oracle's pins (tests only).

Every binary floating-point format used on the path is described by three
numbers: p (significand bits, implicit bit included), emin (exponent of the
smallest normal value) and the largest finite value.  ``rn`` rounds an exact
rational to the nearest member with ties to the even integral significand,
which is IEEE 754 roundTiesToEven.  This is a different algorithm from the
oracle's table-and-midpoint search and from bit manipulation, so agreement
pins both.

Formats (from their standard definitions):
  FP32: p=24, emin=-126, max=(2-2^-23)*2^127, overflow -> inf
  BF16: p=8,  emin=-126, max=(2-2^-7)*2^127,  overflow -> inf
  E4M3 (FN): p=4, emin=-6, max=448, saturating (the ".satfinite" reading)
  E2M1: p=2, emin=0, max=6, saturating
"""
from fractions import Fraction
import math
import struct

INF = float("inf")


class Fmt:
    def __init__(self, p, emin, maxval, saturate):
        self.p, self.emin, self.maxval, self.saturate = p, emin, Fraction(maxval), saturate


FP32 = Fmt(24, -126, (2 - Fraction(1, 2 ** 23)) * Fraction(2) ** 127, False)
BF16 = Fmt(8, -126, (2 - Fraction(1, 2 ** 7)) * Fraction(2) ** 127, False)
E4M3 = Fmt(4, -6, 448, True)
E2M1 = Fmt(2, 0, 6, True)


def floor_log2(a: Fraction) -> int:
    e = a.numerator.bit_length() - a.denominator.bit_length()
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    return e


def rn_mag(a: Fraction, fmt: Fmt):
    """Round a non-negative rational; returns a Fraction or INF."""
    if a == INF:
        return INF
    if a == 0:
        return Fraction(0)
    e = max(floor_log2(a), fmt.emin)
    quantum = Fraction(2) ** (e - fmt.p + 1)
    n = a / quantum
    fl = n.numerator // n.denominator
    rem = n - fl
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2 == 1):
        fl += 1
    r = fl * quantum
    if r > fmt.maxval:
        return fmt.maxval if fmt.saturate else INF
    return r


def rn(v, fmt: Fmt):
    """Round (sign, magnitude): returns (negative: bool, magnitude Fraction|INF)."""
    neg, mag = v
    return neg, rn_mag(mag, fmt)


# ---- conversions between Python floats / bit patterns and (neg, Fraction)

def f32_bits_to_exact(u: int):
    f = struct.unpack("<f", struct.pack("<I", u))[0]
    return (u >> 31) == 1, Fraction(abs(f))


def bf16_bits_to_exact(b: int):
    return f32_bits_to_exact(b << 16)


def exact_to_f32_bits(v) -> int:
    neg, mag = v
    if mag == INF:
        u = 0x7F800000
    else:
        u = struct.unpack("<I", struct.pack("<f", float(mag)))[0]
        assert Fraction(struct.unpack("<f", struct.pack("<I", u))[0]) == mag, "not an FP32 value"
    return u | (0x80000000 if neg else 0)


def exact_to_bf16_bits(v) -> int:
    u = exact_to_f32_bits(v)
    assert u & 0xFFFF == 0, "not a BF16 value"
    return u >> 16


def e4m3_value(code: int) -> Fraction:
    """Magnitude of an E4M3 code from the format definition (bias 7)."""
    e, m = (code >> 3) & 0xF, code & 7
    if e == 0:
        return Fraction(m, 2 ** 9)
    return (1 + Fraction(m, 8)) * Fraction(2) ** (e - 7)


E4M3_CODE_OF = {e4m3_value(c): c for c in range(0x7F)}
E2M1_GRID = [Fraction(0), Fraction(1, 2), Fraction(1), Fraction(3, 2), Fraction(2), Fraction(3),
             Fraction(4), Fraction(6)]
E2M1_CODE_OF = {v: c for c, v in enumerate(E2M1_GRID)}


def e4m3_code(v) -> int:
    """Code of an already-rounded E4M3 value (neg, magnitude)."""
    neg, mag = v
    return E4M3_CODE_OF[mag] | (0x80 if neg else 0)


def e2m1_code(v) -> int:
    neg, mag = v
    return E2M1_CODE_OF[mag] | (0x8 if neg else 0)


def mul(a, b):
    if INF in (a[1], b[1]):
        return (a[0] != b[0], INF)
    return (a[0] != b[0], a[1] * b[1])


def div(a, b):
    assert b[1] != 0
    return (a[0] != b[0], a[1] / b[1])


def f32(v):
    """fl(): one IEEE binary32 RN rounding of an exact value."""
    return rn(v, FP32)


def is_zero(v):
    return v[1] == 0


def to_rational(v) -> Fraction:
    """(neg, finite magnitude) -> signed Fraction."""
    assert v[1] != INF
    return -v[1] if v[0] else v[1]


def add(a, b):
    """Exact sum of two finite signed values.  A zero sum of operands with
    different signs is +0, as IEEE addition gives under round-to-nearest;
    -0 + -0 = -0."""
    s = to_rational(a) + to_rational(b)
    if s == 0:
        return (a[0] and b[0], Fraction(0))
    return (s < 0, abs(s))


def neg(a):
    return (not a[0], a[1])


def f32_value_to_exact(x) -> tuple:
    """A Python / numpy binary32 value -> (neg, magnitude)."""
    u = struct.unpack("<I", struct.pack("<f", float(x)))[0]
    return f32_bits_to_exact(u)
