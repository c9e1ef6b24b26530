"""Pins for the oracle's NVFP4 "4over6" variant (CPU only).

Source: vime pull request #503, NVFP4 QDQ config thread (NVTE_NVFP4_4OVER6
and NVTE_NVFP4_4OVER6_E4M3_USE_256, which makes the E4M3 maximum of the
global scale 256 instead of 448).  The pages give the flag and the constant
only; the per-block rule -- scale the block amax to 6 or to 4 and keep the
candidate whose dequantised values have the smaller sum of squared errors,
summed left to right in binary32, ties keeping 6 -- is a reading (R19-R21
in pwq_oracle.c), so this part is parity unpinned against the pages.  What
is pinned here:

  * brute force: every scale byte, code, choice, error and dequantised value
    of small matrices recomputed in exact rationals with one explicit IEEE
    rounding per step (tests/exact.py);
  * the rule against its mathematical meaning: wherever the two exact
    (unrounded) squared errors differ by more than the binary32 summation
    can blur, the kept candidate is the one with the smaller exact error;
  * closed forms: a block on the scaled E2M1 grid of 4 (of 6) comes back
    exactly and keeps 4 (6);
  * reductions: with E = 448, blocks that keep 6 are the plain NVFP4 blocks,
    and no block's error exceeds plain NVFP4's;
  * symmetries: x -> -x and x, A -> 2^j x, 2^j A;
  * the worked example W4 (tests/golden/w4_nvfp4_4over6.txt), derived by
    hand from the reading.
"""
from fractions import Fraction
import os
import struct

import numpy as np
import pytest

from oracle import oracle as O
import exact as X


def _input(shape, seed, spread=4):
    """Normal values over several binades, with zeros of both signs, BF16
    subnormals and outliers."""
    rng = np.random.default_rng(seed)
    v = (rng.standard_normal(shape) * np.exp2(rng.integers(-spread, spread, size=shape))).astype(np.float32)
    x = O.bf16_round(v)
    flat = x.reshape(-1)
    n = flat.size
    idx = rng.choice(n, size=max(1, n // 40), replace=False)
    flat[idx[0::4]] = 0x0000
    flat[idx[1::4]] = 0x8000
    flat[idx[2::4]] = rng.integers(1, 0x80, size=idx[2::4].size) | (rng.integers(0, 2, size=idx[2::4].size) << 15)
    flat[idx[3::4]] = O.bf16_round(rng.standard_normal(idx[3::4].size).astype(np.float32) * 200)
    return x


def _bf16_bits(v):
    u = struct.unpack("<I", struct.pack("<f", float(v)))[0]
    assert u & 0xFFFF == 0, v
    return u >> 16


# ------------------------------------------------------------------ exact restatement

def _ex_candidate(blk, gs, t):
    """R20 for one candidate t: (sb code, codes, values (neg, mag), error)."""
    amax_b = max(v[1] for v in blk)
    if X.is_zero(gs):
        sbc = 0
    else:
        t_gs = X.f32(X.mul((False, Fraction(t)), gs))
        sbc = X.e4m3_code(X.rn(X.f32(X.div((False, amax_b), t_gs)), X.E4M3))
    sbv = (False, X.e4m3_value(sbc))
    d = X.f32(X.mul(sbv, gs))
    codes, ys = [], []
    for xv in blk:
        if X.is_zero(d):
            c = 0x8 if xv[0] else 0x0
        else:
            c = X.e2m1_code(X.rn(X.f32(X.div(xv, d)), X.E2M1))
        cv = (bool(c & 8), X.E2M1_GRID[c & 7])
        codes.append(c)
        ys.append(X.rn(X.f32(X.mul(X.mul(cv, sbv), gs)), X.BF16))
    # R21: fl(fl(x - y)^2) summed left to right in binary32
    err = (False, Fraction(0))
    for xv, y in zip(blk, ys):
        dl = X.f32(X.add(xv, X.neg(y)))
        err = X.f32(X.add(err, X.f32(X.mul(dl, dl))))
    return sbc, codes, ys, err


def ex_4over6(members, E):
    """members: list of uint16 [M][N] sharing one group amax."""
    A = max((X.bf16_bits_to_exact(int(v))[1] for m in members for v in m.ravel()), default=Fraction(0))
    gs = X.f32((False, A / (6 * E)))
    out = []
    for x in members:
        M, N = x.shape
        codes = np.zeros((M, N), np.uint8)
        sb = np.zeros((M, N // 16), np.uint8)
        choice = np.zeros((M, N // 16), np.uint8)
        err = np.zeros((M, N // 16, 2), np.uint32)
        y = np.zeros((M, N), np.uint16)
        for r in range(M):
            for k in range(N // 16):
                blk = [X.bf16_bits_to_exact(int(v)) for v in x[r, k * 16:(k + 1) * 16]]
                c6 = _ex_candidate(blk, gs, 6)
                c4 = _ex_candidate(blk, gs, 4)
                four = c4[3][1] < c6[3][1]
                keep = c4 if four else c6
                sb[r, k] = keep[0]
                choice[r, k] = 4 if four else 6
                codes[r, k * 16:(k + 1) * 16] = keep[1]
                y[r, k * 16:(k + 1) * 16] = [X.exact_to_bf16_bits(v) for v in keep[2]]
                err[r, k] = [X.exact_to_f32_bits(c6[3]), X.exact_to_f32_bits(c4[3])]
        packed = (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)
        out.append((packed, sb, choice, err, y))
    return X.exact_to_f32_bits(gs), out


CASES = [([(1, 16)], 256), ([(2, 48)], 256), ([(3, 64), (2, 32)], 256), ([(4, 64)], 448),
         ([(2, 32), (2, 32), (1, 16)], 448)]


@pytest.mark.parametrize("shapes,E", CASES, ids=lambda c: str(c))
def test_4over6_bruteforce(shapes, E):
    xs = [_input(s, seed=700 + 7 * i + s[0] * s[1] + E) for i, s in enumerate(shapes)]
    A = O.nvfp4_group_amax(xs)
    egs, eouts = ex_4over6(xs, E)
    for x, (epk, esb, ech, eerr, ey) in zip(xs, eouts):
        packed, sb, gs, choice, err = O.nvfp4_4over6_quant(x, A, E, details=True)
        assert np.float32(gs).view(np.uint32) == egs
        assert np.array_equal(sb, esb)
        assert np.array_equal(choice, ech)
        assert np.array_equal(err.view(np.uint32), eerr)
        assert np.array_equal(packed, epk)
        assert np.array_equal(O.nvfp4_dequant(packed, sb, gs, x.shape[-1]), ey)
        assert np.array_equal(O.nvfp4_4over6_fake_quant(x, A, E), ey)
    # both candidates must occur in these inputs, or the test pins only one
    allch = np.concatenate([o[2].ravel() for o in eouts])
    if allch.size >= 8:
        assert (allch == 4).any() and (allch == 6).any()


def test_4over6_degenerate_bruteforce():
    x = np.zeros((4, 32), np.uint16)
    x[0, :16] = 0x8000                                   # a zero block in a live group
    x[0, 16:] = np.arange(1, 17, dtype=np.uint16)        # BF16 subnormals
    x[1] = _bf16_bits(0.0029296875)                      # 3 * 2^-10, constant rows
    x[2, ::2] = 0x4C00                                   # 2^25, the group amax
    x[3, :] = 0x0001
    for E in (256, 448):
        A = O.amax_bf16(x)
        packed, sb, gs, choice, err = O.nvfp4_4over6_quant(x, A, E, details=True)
        egs, eouts = ex_4over6([x], E)
        assert np.float32(gs).view(np.uint32) == egs
        assert np.array_equal(sb, eouts[0][1]) and np.array_equal(packed, eouts[0][0])
        assert np.array_equal(choice, eouts[0][2])
        assert np.array_equal(O.nvfp4_4over6_fake_quant(x, A, E), eouts[0][4])
    # an all-zero group: gs = 0, sb = 0, 6 kept (equal errors), signs kept
    z = np.zeros((1, 16), np.uint16)
    z[0, 5] = 0x8000
    packed, sb, gs, choice, err = O.nvfp4_4over6_quant(z, 0.0, 256, details=True)
    assert gs == 0.0 and not sb.any() and choice[0, 0] == 6 and not err.any()
    assert list(O.unpack_e2m1(packed)[0]) == [8 if i == 5 else 0 for i in range(16)]


# ------------------------------------------------------------------ the rule's meaning

def _exact_sse(xbits, ybits):
    s = Fraction(0)
    for a, b in zip(xbits, ybits):
        d = X.to_rational(X.bf16_bits_to_exact(int(a))) - X.to_rational(X.bf16_bits_to_exact(int(b)))
        s += d * d
    return s


@pytest.mark.parametrize("E", [256, 448])
def test_4over6_keeps_the_smaller_exact_error(E):
    """Each candidate's values come from the plain NVFP4 rule with the block
    amax mapped to t; the kept one must have the smaller unrounded squared
    error wherever binary32 summation cannot blur the comparison (16 terms,
    each step relative error 2^-24: a relative gap above 2^-18 is safe)."""
    x = _input((64, 64), seed=91 + E, spread=3)
    A = O.amax_bf16(x)
    packed, sb, gs, choice, _ = O.nvfp4_4over6_quant(x, A, E, details=True)
    codes = O.unpack_e2m1(packed)
    decided = 0
    for r in range(x.shape[0]):
        for k in range(x.shape[1] // 16):
            blk = x[r, 16 * k:16 * (k + 1)]
            ys = {}
            for t in (6, 4):
                # the candidate t, through an exact restatement of R20 alone
                _, _, yv, _ = _ex_candidate([X.bf16_bits_to_exact(int(v)) for v in blk],
                                            X.f32((False, X.to_rational(X.f32_value_to_exact(A)) / (6 * E))), t)
                ys[t] = [X.exact_to_bf16_bits(v) for v in yv]
            e6, e4 = _exact_sse(blk, ys[6]), _exact_sse(blk, ys[4])
            kept = ys[int(choice[r, k])]
            y_out = O.nvfp4_dequant(packed[r:r + 1, 8 * k:8 * (k + 1)], sb[r:r + 1, k:k + 1], gs, 16)[0]
            assert list(y_out) == kept
            if abs(e4 - e6) > Fraction(1, 2 ** 18) * max(e4, e6):
                decided += 1
                assert int(choice[r, k]) == (4 if e4 < e6 else 6), (r, k, float(e6), float(e4))
    assert decided > 200


# ------------------------------------------------------------------ closed forms

def _grid_block(grid, s, gs, seed):
    """16 values g * s * gs with g drawn from the signed grid, one of them
    +max(grid), as BF16 bits (exact: g has at most 2 significant bits, s an
    E4M3 value at most 4 and gs is a power of two)."""
    rng = np.random.default_rng(seed)
    g = rng.choice(grid, size=16)
    g = g * rng.choice([-1.0, 1.0], size=16)
    g[rng.integers(16)] = max(grid)
    return np.array([_bf16_bits(v * s * gs) for v in g], np.uint16)


@pytest.mark.parametrize("E", [256, 448])
def test_4over6_grid_blocks_come_back_exactly(E):
    """gs a power of two (A = 6 E 2^k).  A block on the grid of 4 scaled by
    s gs has sb_4 = s, every quotient on the E2M1 grid and error 0: it keeps
    4 and fake-quantises to itself.  A block on the grid of 6 has error 0 for
    t = 6 and keeps 6 (4 would need a negative error)."""
    k = -9
    gs = 2.0 ** k
    A = 6 * E * gs
    anchor = np.full(16, _bf16_bits(A), np.uint16)            # holds the group amax
    grid4 = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0]
    grid6 = grid4 + [6.0]
    rows = [anchor]
    want = [None]
    seeds = iter(range(1000))
    for s in (1.0, 1.125, 1.75, 3.5, 13.0, 0.3125):
        if 4 * s > E * 1.5:                                   # keep sb_4 = s representable in range
            continue
        rows.append(_grid_block(grid4, s, gs, next(seeds)))
        want.append(4)
        rows.append(_grid_block(grid6, s, gs, next(seeds)))
        want.append(6)
    x = np.stack(rows)
    assert O.amax_bf16(x) == A
    packed, sb, gsv, choice, err = O.nvfp4_4over6_quant(x, A, E, details=True)
    assert gsv == gs
    y = O.nvfp4_4over6_fake_quant(x, A, E)
    for r in range(1, x.shape[0]):
        assert np.array_equal(y[r], x[r]), r
        assert choice[r, 0] == want[r], (r, choice[r, 0])
        assert err[r, 0, 0 if want[r] == 6 else 1] == 0.0
        if want[r] == 4:
            assert err[r, 0, 0] > 0.0                          # 6 was strictly worse


# ------------------------------------------------------------------ reductions and symmetries

def test_4over6_e448_six_blocks_are_plain_nvfp4():
    x = _input((32, 128), seed=5, spread=3)
    A = O.amax_bf16(x)
    packed, sb, gs, choice, err = O.nvfp4_4over6_quant(x, A, 448, details=True)
    p0, s0, g0 = O.nvfp4_quant(x, A)
    assert gs == g0
    six = choice == 6
    assert six.any() and (~six).any()
    assert np.array_equal(sb[six], s0[six])
    c, c0 = O.unpack_e2m1(packed), O.unpack_e2m1(p0)
    six_el = np.repeat(six, 16, axis=1)
    assert np.array_equal(c[six_el], c0[six_el])
    # the plain NVFP4 error is the t = 6 candidate's error: no block is worse
    y, y0 = O.nvfp4_4over6_fake_quant(x, A, 448), O.nvfp4_fake_quant(x, A)
    for r in range(x.shape[0]):
        for k in range(x.shape[1] // 16):
            sl = slice(16 * k, 16 * (k + 1))
            assert _exact_sse(x[r, sl], y[r, sl]) <= _exact_sse(x[r, sl], y0[r, sl]) * (1 + Fraction(1, 2 ** 18))


@pytest.mark.parametrize("E", [256, 448])
def test_4over6_sign_and_power_of_two_symmetry(E):
    x = _input((16, 64), seed=17 + E, spread=2)
    x[(x & 0x7F80) == 0] &= np.uint16(0x8000)               # BF16 subnormals -> signed zeros
    A = O.amax_bf16(x)
    packed, sb, gs, choice, _ = O.nvfp4_4over6_quant(x, A, E, details=True)
    y = O.nvfp4_4over6_fake_quant(x, A, E)
    # negation: same scales and choices, every code's sign bit flipped
    xn = x ^ np.uint16(0x8000)
    pn, sbn, gsn, chn, _ = O.nvfp4_4over6_quant(xn, A, E, details=True)
    assert gsn == gs and np.array_equal(sbn, sb) and np.array_equal(chn, choice)
    assert np.array_equal(O.unpack_e2m1(pn), O.unpack_e2m1(packed) ^ 8)
    assert np.array_equal(O.nvfp4_4over6_fake_quant(xn, A, E), y ^ np.uint16(0x8000))
    # x, A -> 2^j x, 2^j A: codes, scales and choices unchanged (no value
    # leaves the normal range), gs and every output scaled by 2^j
    for j in (-3, 5):
        f = np.float32(2.0 ** j)
        xs = O.bf16_round(O.bf16_to_f32(x) * f)
        assert np.array_equal(O.bf16_to_f32(xs), O.bf16_to_f32(x) * f)
        ps, sbs, gss, chs, _ = O.nvfp4_4over6_quant(xs, A * float(f), E, details=True)
        assert gss == gs * float(f)
        assert np.array_equal(ps, packed) and np.array_equal(sbs, sb) and np.array_equal(chs, choice)


def test_4over6_sibling_group_shares_the_amax():
    xs = [_input((3, 32), seed=s) for s in (1, 2, 3)]
    xs[1][0, 0] = _bf16_bits(512.0)
    A, outs = O.nvfp4_4over6_quant_group(xs, 256)
    assert A == 512.0
    for x, (packed, sb, gs) in zip(xs, outs):
        assert gs == O.nvfp4_4over6_global_scale(512.0, 256) == np.float32(512.0) / np.float32(1536.0)
        p1, s1, _ = O.nvfp4_4over6_quant(x, A, 256)
        assert np.array_equal(packed, p1) and np.array_equal(sb, s1)


# ------------------------------------------------------------------ worked example W4

GOLDEN_W4 = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "w4_nvfp4_4over6.txt")


def read_w4():
    """The fields of tests/golden/w4_nvfp4_4over6.txt as a dict of token lists."""
    out = {}
    for line in open(GOLDEN_W4):
        line = line.split("#")[0].strip()
        if line:
            key, *vals = line.split()
            out[key] = vals
    return out


def test_4over6_w4_worked_example():
    w = read_w4()
    E = int(w["e4m3_max"][0])
    x = np.array([_bf16_bits(v) for v in w["x"]], np.uint16)[None]
    A = O.amax_bf16(x)
    assert A == float(w["group_amax"][0])
    packed, sb, gs, choice, err = O.nvfp4_4over6_quant(x, A, E, details=True)
    assert int(np.float32(gs).view(np.uint32)) == int(w["global_scale"][0], 16)
    assert list(choice[0]) == [int(v) for v in w["choice"]]
    assert list(err[0, :, 0]) == [float(v) for v in w["err6"]]
    assert list(err[0, :, 1]) == [float(v) for v in w["err4"]]
    assert [int(v) for v in sb[0]] == [int(v, 16) for v in w["sb"]]
    assert list(O.unpack_e2m1(packed)[0]) == [int(v, 16) for v in w["codes"]]
    assert list(packed[0]) == [int(v, 16) for v in w["packed"]]
    assert list(O.nvfp4_4over6_fake_quant(x, A, E)[0]) == [_bf16_bits(v) for v in w["y"]]
    # and the exact-rational restatement agrees
    egs, eouts = ex_4over6([x], E)
    assert egs == int(w["global_scale"][0], 16)
    assert list(eouts[0][2][0]) == [int(v) for v in w["choice"]]
