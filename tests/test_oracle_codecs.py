"""Pins for the oracle's element codecs (CPU only).

Each codec is checked against something other than itself:
  * BF16 and E4M3 rounding against torch's own float->bfloat16 and
    float->float8_e4m3fn conversions (round-to-nearest-even library routines),
  * every E4M3 / E2M1 / BF16 rounding boundary against exact-rational IEEE
    rounding (tests/exact.py),
  * E2M1 against a closed form built on numpy's round-half-even,
  * the UE8M0 exponent against a brute-force search in exact rationals,
  * the decoders against the grid printed on the verl NVFP4 QAT article,
    section 2.3, and against torch's float8 decoder.
"""
from fractions import Fraction
import struct

import numpy as np
import pytest
import torch

from oracle import oracle as O
import exact as X

pytestmark = pytest.mark.filterwarnings("ignore")


def f32_from_bits(u):
    return np.asarray(u, dtype=np.uint32).view(np.float32)


def torch_e4m3(v: np.ndarray) -> np.ndarray:
    """torch's RNE float32 -> float8_e4m3fn, made saturating: torch returns NaN
    above 464, where the satfinite reading returns the largest value 448."""
    t = torch.from_numpy(np.ascontiguousarray(v, dtype=np.float32))
    q = t.to(torch.float8_e4m3fn).view(torch.uint8).numpy().copy()
    big = np.abs(v) > 464.0
    q[big] = np.where(np.signbit(v[big]), 0xFE, 0x7E).astype(np.uint8)
    return q


def test_fp_environment():
    assert O.fp_env_ok()


# ------------------------------------------------------------------ BF16

def test_bf16_every_exponent_and_tie_pattern_matches_torch():
    hi = np.arange(0, 1 << 16, dtype=np.uint32)
    hi = hi[(hi & 0x7F80) != 0x7F80]               # finite inputs only
    lows = np.array([0x0000, 0x0001, 0x3FFF, 0x7FFF, 0x8000, 0x8001, 0xBFFF, 0xFFFF],
                    dtype=np.uint32)
    u = (hi[:, None] << 16 | lows[None, :]).ravel()
    v = f32_from_bits(u)
    want = torch.from_numpy(v.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = O.bf16_round(v)
    bad = np.nonzero(got != want)[0]
    assert bad.size == 0, [(hex(u[i]), hex(got[i]), hex(want[i])) for i in bad[:8]]


def test_bf16_random_matches_torch():
    rng = np.random.default_rng(7)
    u = rng.integers(0, 1 << 32, size=4_000_000, dtype=np.uint64).astype(np.uint32)
    u = u[(u & 0x7F800000) != 0x7F800000]
    v = f32_from_bits(u)
    want = torch.from_numpy(v.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(O.bf16_round(v), want)


def test_bf16_overflow_and_subnormals_exact():
    cases = [0x7F7F7FFF, 0x7F7F8000, 0x7F7F8001, 0x7F7FFFFF, 0x00008000, 0x00018000,
             0x00007FFF, 0x00000001, 0x80008000, 0x80018000]
    for u in cases:
        v = X.f32_bits_to_exact(u)
        want = X.exact_to_f32_bits(X.rn(v, X.BF16)) >> 16
        assert int(O.bf16_round(f32_from_bits([u]))[0]) == want, hex(u)


# ------------------------------------------------------------------ E4M3

def test_e4m3_decode_matches_torch_for_every_code():
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)
    ref = torch.from_numpy(codes.copy()).view(torch.float8_e4m3fn).float().numpy()
    got = np.array([O.e4m3_decode(c) for c in codes])
    assert np.array_equal(got, ref.astype(np.float64))
    # -0 keeps its sign
    assert np.signbit(O.e4m3_decode(0x80))


def _e4m3_boundaries():
    vals = sorted(set(X.e4m3_value(c) for c in range(0x7F)))
    pts = []
    for a, b in zip(vals, vals[1:]):
        mid = (a + b) / 2
        pts.append(mid)
    pts += vals + [Fraction(464), Fraction(448) + Fraction(1, 64), Fraction(480), Fraction(2 ** 20)]
    out = []
    for p in pts:
        f = np.float32(float(p))
        assert Fraction(float(f)) == p            # every midpoint is an FP32 value
        out += [f, np.nextafter(f, np.float32(0)), np.nextafter(f, np.float32(np.inf))]
    out = np.array(out, dtype=np.float32)
    return np.concatenate([out, -out])


def test_e4m3_every_rounding_boundary_exact():
    v = _e4m3_boundaries()
    got = O.e4m3_encode(v)
    for x, g in zip(v, got):
        neg = bool(np.signbit(x))
        want = X.e4m3_code(X.rn((neg, Fraction(abs(float(x)))), X.E4M3))
        assert int(g) == want, (float(x), hex(g), hex(want))
    assert np.array_equal(got, torch_e4m3(v))


def test_e4m3_dense_sweep_matches_torch():
    # every 7th FP32 pattern of the binades E4M3 can reach (2^-12 .. 2^10),
    # both signs (the ties themselves are covered by the boundary test)
    lo, hi = (127 - 12) << 23, (127 + 10) << 23
    u = np.arange(lo, hi, 7, dtype=np.uint32)
    u = np.concatenate([u, u | 0x80000000])
    v = f32_from_bits(u)
    got = O.e4m3_encode(v)
    want = torch_e4m3(v)
    bad = np.nonzero(got != want)[0]
    assert bad.size == 0, [(float(v[i]), hex(got[i]), hex(want[i])) for i in bad[:8]]


def test_e4m3_random_full_range_and_signed_zero():
    rng = np.random.default_rng(11)
    u = rng.integers(0, 1 << 32, size=2_000_000, dtype=np.uint64).astype(np.uint32)
    u = u[(u & 0x7F800000) != 0x7F800000]
    v = f32_from_bits(u)
    assert np.array_equal(O.e4m3_encode(v), torch_e4m3(v))
    z = O.e4m3_encode(np.array([0.0, -0.0, -1e-30, 1e-30, -2.0 ** -11], dtype=np.float32))
    assert list(z) == [0x00, 0x80, 0x80, 0x00, 0x80]


# ------------------------------------------------------------------ E2M1

GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def e2m1_closed_form(v: np.ndarray) -> np.ndarray:
    """Piecewise closed form with numpy's round-half-to-even (np.rint):
    spacing 0.5 on [0,2), 1 on [2,4), 2 on [4,6], saturating at 6.  Ties go to
    the even code, which on each piece is the even multiple of the spacing."""
    a = np.abs(v.astype(np.float64))
    r = np.where(a < 2.0, np.rint(a * 2.0) / 2.0,
                 np.where(a < 4.0, np.rint(a), 2.0 * np.rint(a / 2.0)))
    r = np.minimum(r, 6.0)
    code = np.searchsorted(GRID, r).astype(np.uint8)
    assert np.array_equal(GRID[code], r)
    return code | np.where(np.signbit(v), 8, 0).astype(np.uint8)


def test_e2m1_decode_is_the_published_grid():
    # verl NVFP4 QAT article, section 2.3: the E2M1 steps 0, 0.5, 1, 1.5, 2, 3, 4, 6
    assert [O.e2m1_decode(c) for c in range(8)] == [0, 0.5, 1, 1.5, 2, 3, 4, 6]
    assert [O.e2m1_decode(c | 8) for c in range(8)] == [-0.0, -0.5, -1, -1.5, -2, -3, -4, -6]
    assert np.signbit(O.e2m1_decode(8))


def test_e2m1_every_rounding_boundary_exact():
    mids = [Fraction(1, 4), Fraction(3, 4), Fraction(5, 4), Fraction(7, 4), Fraction(5, 2),
            Fraction(7, 2), Fraction(5), Fraction(6), Fraction(7)] + list(X.E2M1_GRID)
    vs = []
    for m in mids:
        f = np.float32(float(m))
        vs += [f, np.nextafter(f, np.float32(0)), np.nextafter(f, np.float32(np.inf))]
    v = np.array(vs, dtype=np.float32)
    v = np.concatenate([v, -v])
    got = O.e2m1_encode(v)
    for x, g in zip(v, got):
        want = X.e2m1_code(X.rn((bool(np.signbit(x)), Fraction(abs(float(x)))), X.E2M1))
        assert int(g) == want, (float(x), g, want)
    # the worked ties: 0.25->0, 0.75->1, 1.25->1, 1.75->2, 2.5->2, 3.5->4, 5->4
    t = O.e2m1_encode(np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0], dtype=np.float32))
    assert [GRID[c] for c in t] == [0, 1, 1, 2, 2, 4, 4]


def test_e2m1_every_fp32_in_the_active_binades():
    # all FP32 magnitudes in [2^-3, 8) (everything E2M1 can tell apart), both signs
    for e in range(127 - 3, 127 + 3):
        u = np.arange(e << 23, (e + 1) << 23, dtype=np.uint32)
        for s in (0, 0x80000000):
            v = f32_from_bits(u | s)
            got = O.e2m1_encode(v)
            want = e2m1_closed_form(v)
            bad = np.nonzero(got != want)[0]
            assert bad.size == 0, [(float(v[i]), got[i], want[i]) for i in bad[:8]]


def test_e2m1_far_ranges():
    rng = np.random.default_rng(5)
    u = rng.integers(0, 1 << 32, size=1_000_000, dtype=np.uint64).astype(np.uint32)
    u = u[(u & 0x7F800000) != 0x7F800000]
    v = f32_from_bits(u)
    assert np.array_equal(O.e2m1_encode(v), e2m1_closed_form(v))


# ------------------------------------------------------------------ UE8M0

def ue8m0_bruteforce(amax_bits16: int) -> int:
    a = Fraction(struct.unpack("<f", struct.pack("<I", amax_bits16 << 16))[0])
    # start well below any candidate (448 = 1.75 * 2^8) and walk up
    k = (X.floor_log2(a) - 12) if a > 0 else -200
    while not (a <= 448 * Fraction(2) ** k):
        k += 1
    return min(max(k, -127), 127) + 127


def test_ue8m0_every_bf16_amax():
    b = np.arange(0, 0x7F80, dtype=np.uint32)      # +0 and every positive finite BF16
    amax = f32_from_bits(b << 16)
    got = O.ue8m0_byte(amax)
    want = np.array([ue8m0_bruteforce(int(x)) for x in b], dtype=np.uint8)
    bad = np.nonzero(got != want)[0]
    assert bad.size == 0, [(hex(b[i]), got[i], want[i]) for i in bad[:8]]
    # the byte never lets the block maximum exceed 448 after scaling, and the
    # next smaller exponent would (round-up reading), unless clamped
    for x, e in zip(amax[1:], got[1:].astype(int) - 127):
        a, e = Fraction(float(x)), int(e)
        assert a <= 448 * Fraction(2) ** e
        assert e == -127 or a > 448 * Fraction(2) ** (e - 1)


def test_ue8m0_matches_ceil_log2_of_float_quotient():
    # a second, independent formulation: ceil(log2(fl(amax / 448))) over every
    # positive normal BF16 amax whose quotient stays normal
    b = np.arange(0x0080, 0x7F80, dtype=np.uint32)
    amax = f32_from_bits(b << 16)
    q = (amax / np.float32(448.0)).astype(np.float32)
    ok = q >= np.float32(2.0 ** -126)
    m, ex = np.frexp(q[ok].astype(np.float64))
    ceil_log2 = np.where(m == 0.5, ex - 1, ex)
    want = np.clip(ceil_log2, -127, 127) + 127
    assert np.array_equal(O.ue8m0_byte(amax[ok]).astype(np.int64), want.astype(np.int64))
