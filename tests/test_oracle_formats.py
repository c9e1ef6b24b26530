"""Pins for the oracle's three formats (CPU only).

  * worked examples W1-W3 (tests/golden/, derived by hand from the pages'
    definitions, each file citing its source) reproduced by the oracle and
    by an exact-rational restatement,
  * brute force: every code, scale and dequantised value of small matrices
    (several tiles, ragged edges, batches, degenerate tiles) recomputed in
    exact rationals with one explicit IEEE rounding per step (tests/exact.py),
  * invariants: scale == tile amax / 448, the rounding error bound,
    idempotence of QDQ, fake-quant == dequant(quant), sibling amax == max of
    the members' amax.
"""
from fractions import Fraction
import os
import struct

import numpy as np
import pytest

from oracle import oracle as O
import exact as X
import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def bf16_bits_of(values):
    """Exact BF16 values (decimal strings / floats) -> uint16 bit patterns."""
    out = []
    for v in values:
        f = float(v)
        u = struct.unpack("<I", struct.pack("<f", f))[0]
        assert u & 0xFFFF == 0, ("not an exact BF16 value", v)
        out.append(u >> 16)
    return np.array(out, dtype=np.uint16)


def f32_of_bits16(b):
    return O.bf16_to_f32(b)


# ------------------------------------------------------------------ exact restatements

def xval(bits16):
    return X.bf16_bits_to_exact(int(bits16))


def ex_fp8_block(x):
    """x: uint16 [B][M][N].  Exact-rational FP8 block-wise quantisation."""
    B, M, N = x.shape
    TM, TN = -(-M // 128), -(-N // 128)
    q = np.zeros(x.shape, np.uint8)
    s = np.zeros((B, TM, TN), np.uint32)
    y = np.zeros(x.shape, np.uint16)
    for b in range(B):
        for tm in range(TM):
            for tn in range(TN):
                tile = x[b, tm * 128:(tm + 1) * 128, tn * 128:(tn + 1) * 128]
                amax = max((xval(v)[1] for v in tile.ravel()), default=Fraction(0))
                sc = X.f32((False, amax / 448))
                s[b, tm, tn] = X.exact_to_f32_bits(sc)
                for (i, j), v in np.ndenumerate(tile):
                    xv = xval(v)
                    if X.is_zero(sc):
                        code = 0x80 if xv[0] else 0x00
                    else:
                        code = X.e4m3_code(X.rn(X.f32(X.div(xv, sc)), X.E4M3))
                    dq = (bool(code & 0x80), X.e4m3_value(code & 0x7F))
                    r, c = tm * 128 + i, tn * 128 + j
                    q[b, r, c] = code
                    y[b, r, c] = X.exact_to_bf16_bits(X.rn(X.f32(X.mul(dq, sc)), X.BF16))
    return q, s, y


def ex_ue8m0(amax: Fraction) -> int:
    k = (X.floor_log2(amax) - 12) if amax > 0 else -200
    while not (amax <= 448 * Fraction(2) ** k):
        k += 1
    return min(max(k, -127), 127)


def ex_mxfp8(x):
    B, M, N = x.shape
    q = np.zeros(x.shape, np.uint8)
    e = np.zeros((B, M, N // 32), np.uint8)
    y = np.zeros(x.shape, np.uint16)
    for b in range(B):
        for r in range(M):
            for k in range(N // 32):
                blk = [xval(v) for v in x[b, r, k * 32:(k + 1) * 32]]
                ex = ex_ue8m0(max(v[1] for v in blk))
                e[b, r, k] = ex + 127
                p2 = Fraction(2) ** ex
                for j, xv in enumerate(blk):
                    code = X.e4m3_code(X.rn((xv[0], xv[1] / p2), X.E4M3))
                    dq = (bool(code & 0x80), X.e4m3_value(code & 0x7F))
                    q[b, r, k * 32 + j] = code
                    y[b, r, k * 32 + j] = X.exact_to_bf16_bits(
                        X.rn(X.f32((dq[0], dq[1] * p2)), X.BF16))
    return q, e, y


def ex_nvfp4(members):
    """members: list of uint16 [M][N] sharing one group amax."""
    A = max((xval(v)[1] for m in members for v in m.ravel()), default=Fraction(0))
    gs = X.f32((False, A / 2688))
    out = []
    for x in members:
        M, N = x.shape
        codes = np.zeros((M, N), np.uint8)
        sb = np.zeros((M, N // 16), np.uint8)
        y = np.zeros((M, N), np.uint16)
        for r in range(M):
            for k in range(N // 16):
                blk = [xval(v) for v in x[r, k * 16:(k + 1) * 16]]
                amax_b = max(v[1] for v in blk)
                if X.is_zero(gs):
                    sbc = 0
                else:
                    six_gs = X.f32(X.mul((False, Fraction(6)), gs))
                    sbc = X.e4m3_code(X.rn(X.f32(X.div((False, amax_b), six_gs)), X.E4M3))
                sb[r, k] = sbc
                sbv = (False, X.e4m3_value(sbc))
                d = X.f32(X.mul(sbv, gs))
                for j, xv in enumerate(blk):
                    if X.is_zero(d):
                        c = 0x8 if xv[0] else 0x0
                    else:
                        c = X.e2m1_code(X.rn(X.f32(X.div(xv, d)), X.E2M1))
                    codes[r, k * 16 + j] = c
                    cv = (bool(c & 8), X.E2M1_GRID[c & 7])
                    inner = X.mul(cv, sbv)                       # exact
                    y[r, k * 16 + j] = X.exact_to_bf16_bits(X.rn(X.f32(X.mul(inner, gs)), X.BF16))
        packed = (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)
        out.append((packed, sb, y))
    return X.exact_to_f32_bits(gs), out


# ------------------------------------------------------------------ golden files

def _read_blocks(name):
    blocks, cur = [], None
    for line in open(os.path.join(GOLDEN, name)):
        line = line.split("#")[0].strip()
        if not line:
            continue
        parts = line.split()
        if parts[0] in ("tile", "block"):
            cur = {"scale": int(parts[-1], 16), "rows": []}
        elif parts[0] == "end":
            blocks.append(cur)
            cur = None
        else:
            cur["rows"].append((parts[0], int(parts[1], 16), parts[2]))
    return blocks


def test_w1_fp8_block_golden():
    for blk in _read_blocks("w1_fp8_block.txt"):
        x = np.zeros((1, 128, 128), np.uint16)
        vals = [r[0] for r in blk["rows"]]
        n = len(vals)
        x[0, 0, :n] = bf16_bits_of(vals)
        q, s = O.fp8_block_quant(x)
        y = O.fp8_block_dequant(q, s)
        assert s.view(np.uint32)[0, 0, 0] == blk["scale"]
        assert list(q[0, 0, :n]) == [r[1] for r in blk["rows"]]
        assert np.array_equal(y[0, 0, :n], bf16_bits_of([r[2] for r in blk["rows"]]))
        assert not q[0, 1:].any() and not q[0, 0, n:].any()
        # the exact restatement agrees on the whole tile
        eq, es, ey = ex_fp8_block(x[:, :1, :])  # one-row tile: same amax (other rows are 0)
        assert es[0, 0, 0] == blk["scale"]
        assert np.array_equal(eq[0, 0], q[0, 0]) and np.array_equal(ey[0, 0], y[0, 0])


def test_w2_mxfp8_golden():
    blocks = _read_blocks("w2_mxfp8.txt")
    x = np.zeros((len(blocks), 32), np.uint16)
    for i, blk in enumerate(blocks):
        vals = [r[0] for r in blk["rows"]]
        x[i, :len(vals)] = bf16_bits_of(vals)
    q, e = O.mxfp8_quant(x)
    y = O.mxfp8_dequant(q, e)
    eq, ee, ey = ex_mxfp8(x[None])
    assert np.array_equal(q, eq[0]) and np.array_equal(e, ee[0]) and np.array_equal(y, ey[0])
    for i, blk in enumerate(blocks):
        n = len(blk["rows"])
        assert e[i, 0] == blk["scale"]
        assert list(q[i, :n]) == [r[1] for r in blk["rows"]]
        assert np.array_equal(y[i, :n], bf16_bits_of([r[2] for r in blk["rows"]]))


def _read_w3():
    d, members, cur = {}, [], None
    for line in open(os.path.join(GOLDEN, "w3_nvfp4.txt")):
        line = line.split("#")[0].strip()
        if not line:
            continue
        k, *v = line.split()
        if k == "member":
            cur = {"name": v[0]}
            members.append(cur)
        elif cur is None:
            d[k] = v
        else:
            cur[k] = v
    return d, members


def test_w3_nvfp4_sibling_golden():
    d, members = _read_w3()
    xs = [bf16_bits_of(m["x"])[None, :] for m in members]
    A, outs = O.nvfp4_quant_group(xs)
    assert A == float(d["group_amax"][0])
    gs_bits = np.float32(outs[0][2]).view(np.uint32)
    assert gs_bits == int(d["global_scale"][0], 16)
    egs, eouts = ex_nvfp4(xs)
    assert egs == gs_bits
    for m, x, (packed, sb, gs), (epk, esb, ey) in zip(members, xs, outs, eouts):
        assert sb[0, 0] == int(m["sb"][0], 16)
        assert list(O.unpack_e2m1(packed)[0]) == [int(c, 16) for c in m["codes"]]
        assert list(packed[0]) == [int(c, 16) for c in m["packed"]]
        y = O.nvfp4_dequant(packed, sb, gs, 16)
        assert np.array_equal(y[0], bf16_bits_of(m["y"]))
        assert np.array_equal(O.nvfp4_fake_quant(x, A)[0], y[0])
        assert np.array_equal(epk, packed) and np.array_equal(esb, sb) and np.array_equal(ey, y)


# ------------------------------------------------------------------ brute force

def _tiny_input(shape, seed):
    """Normal values spanning several binades, plus exact zeros, negative
    zeros, BF16 subnormals and a few large outliers."""
    rng = np.random.default_rng(seed)
    v = (rng.standard_normal(shape) * np.exp2(rng.integers(-6, 4, size=shape))).astype(np.float32)
    x = O.bf16_round(v)
    flat = x.reshape(-1)
    n = flat.size
    idx = rng.choice(n, size=max(1, n // 50), replace=False)
    flat[idx[0::4]] = 0x0000
    flat[idx[1::4]] = 0x8000
    flat[idx[2::4]] = rng.integers(1, 0x80, size=idx[2::4].size) | (rng.integers(0, 2, size=idx[2::4].size) << 15)
    flat[idx[3::4]] = O.bf16_round(rng.standard_normal(idx[3::4].size).astype(np.float32) * 300)
    return x


FP8_SHAPES = [(1, 1, 16), (1, 1, 32), (1, 2, 48), (1, 128, 128), (1, 130, 260), (3, 129, 131)]


@pytest.mark.parametrize("shape", FP8_SHAPES)
def test_fp8_block_bruteforce(shape):
    x = _tiny_input(shape, seed=sum(shape))
    q, s = O.fp8_block_quant(x)
    y = O.fp8_block_dequant(q, s)
    eq, es, ey = ex_fp8_block(x)
    assert np.array_equal(s.view(np.uint32), es)
    assert np.array_equal(q, eq)
    assert np.array_equal(y, ey)


def test_fp8_block_degenerate_tiles_bruteforce():
    x = np.zeros((1, 256, 256), np.uint16)
    x[0, :128, :128] = 0x8000                                   # all negative zero
    x[0, :128, 128:] = np.array([1, 0x8003, 0x7F, 0x0002], np.uint16)[np.arange(128 * 128) % 4].reshape(128, 128)  # subnormal amax
    x[0, 128:, :128] = 0x7F7F                                   # largest finite BF16
    x[0, 128:, 128:] = np.arange(128 * 128, dtype=np.uint16).reshape(128, 128) % 0x7F00
    q, s = O.fp8_block_quant(x)
    y = O.fp8_block_dequant(q, s)
    eq, es, ey = ex_fp8_block(x)
    assert np.array_equal(s.view(np.uint32), es)
    assert np.array_equal(q, eq) and np.array_equal(y, ey)
    assert s[0, 0, 0] == 0 and (q[0, :128, :128] == 0x80).all() and (y[0, :128, :128] == 0x8000).all()


MX_SHAPES = [(1, 1, 32), (1, 2, 64), (1, 7, 96), (3, 5, 128)]


@pytest.mark.parametrize("shape", MX_SHAPES)
def test_mxfp8_bruteforce(shape):
    x = _tiny_input(shape, seed=7 + sum(shape))
    q, e = O.mxfp8_quant(x)
    y = O.mxfp8_dequant(q, e)
    eq, ee, ey = ex_mxfp8(x)
    assert np.array_equal(e, ee) and np.array_equal(q, eq) and np.array_equal(y, ey)


def test_mxfp8_extreme_blocks_bruteforce():
    x = np.zeros((1, 4, 32), np.uint16)
    x[0, 0] = 0x7F7F                      # near the BF16 maximum: e = 120
    x[0, 0, 1::2] = 0xFF00                # -2^127 and friends
    x[0, 1] = np.arange(1, 33, dtype=np.uint16)          # subnormal block: clamps to -127
    x[0, 2, ::3] = 0x8000
    x[0, 3] = bf16_bits_of([448.0] * 16 + [-0.0078125] * 16)
    q, e = O.mxfp8_quant(x)
    y = O.mxfp8_dequant(q, e)
    eq, ee, ey = ex_mxfp8(x)
    assert np.array_equal(e, ee) and np.array_equal(q, eq) and np.array_equal(y, ey)
    assert e[0, 1, 0] == 0 and e[0, 0, 0] == 120 + 127


NV_CASES = [[(1, 16)], [(1, 32)], [(2, 48)], [(3, 64), (2, 64), (2, 64)], [(5, 128), (4, 128)]]


@pytest.mark.parametrize("shapes", NV_CASES, ids=lambda c: "+".join("%dx%d" % s for s in c))
def test_nvfp4_bruteforce(shapes):
    xs = [_tiny_input(s, seed=31 + i + s[0] * s[1]) for i, s in enumerate(shapes)]
    A, outs = O.nvfp4_quant_group(xs)
    egs, eouts = ex_nvfp4(xs)
    assert np.float32(outs[0][2]).view(np.uint32) == egs
    for x, (packed, sb, gs), (epk, esb, ey) in zip(xs, outs, eouts):
        assert np.array_equal(sb, esb)
        assert np.array_equal(packed, epk)
        y = O.nvfp4_dequant(packed, sb, gs, x.shape[-1])
        assert np.array_equal(y, ey)
        assert np.array_equal(O.nvfp4_fake_quant(x, A), ey)


def test_nvfp4_degenerate_bruteforce():
    x = np.zeros((4, 32), np.uint16)
    x[0, :16] = 0x8000                                   # zero block in a live group
    x[0, 16:] = np.arange(1, 17, dtype=np.uint16)        # subnormal block: sb rounds to 0
    x[1] = bf16_bits_of([0.0029296875] * 32)            # 3 * 2^-10
    x[2, ::2] = 0x4C00                                   # 2^25
    x[3, :] = 0x0001
    A, outs = O.nvfp4_quant_group([x])
    _, eouts = ex_nvfp4([x])
    packed, sb, gs = outs[0]
    assert np.array_equal(packed, eouts[0][0]) and np.array_equal(sb, eouts[0][1])
    assert np.array_equal(O.nvfp4_dequant(packed, sb, gs, 32), eouts[0][2])
    # an all-zero group: gs = 0, sb = 0, codes keep the sign, dequant is +-0
    z = np.zeros((1, 16), np.uint16)
    z[0, 3] = 0x8000
    Az, oz = O.nvfp4_quant_group([z])
    assert Az == 0.0 and oz[0][2] == 0.0 and not oz[0][1].any()
    assert list(O.unpack_e2m1(oz[0][0])[0]) == [8 if i == 3 else 0 for i in range(16)]
    assert list(O.nvfp4_fake_quant(z, 0.0)[0]) == [0x8000 if i == 3 else 0 for i in range(16)]


# ------------------------------------------------------------------ invariants

def test_fp8_scale_is_tile_amax_over_448():
    x = W.bits(W.small_matrix())
    q, s = O.fp8_block_quant(x)
    xf = f32_of_bits16(x)
    for tm in range(2):
        for tn in range(4):
            amax = np.abs(xf[tm * 128:(tm + 1) * 128, tn * 128:(tn + 1) * 128]).max()
            assert s[tm, tn] == np.float32(amax) / np.float32(448.0)


def _ulp_e4m3(v):
    a = np.abs(v)
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -6)))
    return np.exp2(e - 3)


def _ulp_bf16(v):
    a = np.abs(v).astype(np.float64)
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -126)))
    return np.exp2(e - 7)


def test_fp8_block_error_bound():
    x = W.bits(W.small_matrix())
    q, s = O.fp8_block_quant(x)
    y = f32_of_bits16(O.fp8_block_dequant(q, s)).astype(np.float64)
    xf = f32_of_bits16(x).astype(np.float64)
    sc = np.repeat(np.repeat(s.astype(np.float64), 128, 0), 128, 1)[:256, :512]
    bound = (0.5 * _ulp_e4m3(xf / sc) + np.abs(xf / sc) * 2.0 ** -23) * sc + 0.5 * _ulp_bf16(y)
    assert (np.abs(y - xf) <= bound * (1 + 1e-12)).all()


def test_mxfp8_error_bound():
    x = W.bits(W.small_matrix())
    q, e = O.mxfp8_quant(x)
    y = f32_of_bits16(O.mxfp8_dequant(q, e)).astype(np.float64)
    xf = f32_of_bits16(x).astype(np.float64)
    p2 = np.exp2(np.repeat(e.astype(np.float64) - 127, 32, axis=1))
    bound = 0.5 * _ulp_e4m3(xf / p2) * p2 + 0.5 * _ulp_bf16(y)
    assert (np.abs(y - xf) <= bound * (1 + 1e-12)).all()
    # round-up exponent: no element saturates
    assert (np.abs(xf / p2) <= 448).all()


def test_nvfp4_error_bound():
    x = W.bits(W.small_matrix())
    A = O.nvfp4_group_amax([x])
    packed, sb, gs = O.nvfp4_quant(x, A)
    y = f32_of_bits16(O.nvfp4_dequant(packed, sb, gs, 512)).astype(np.float64)
    xf = f32_of_bits16(x).astype(np.float64)
    sbv = np.array([O.e4m3_decode(c) for c in range(128)])[sb]
    d = np.repeat(sbv * gs, 16, axis=1)
    r = np.abs(xf) / d
    step = np.where(r < 2, 0.5, np.where(r < 4, 1.0, 2.0))
    inside = r <= 6
    bound = 0.5 * step * d * (1 + 2.0 ** -20) + 0.5 * _ulp_bf16(y)
    assert (np.abs(y - xf)[inside] <= bound[inside]).all()
    # outside the grid only the block scale's own E4M3 rounding can push |x| past 6d
    assert (r[~inside] <= 6 * (1 + 2.0 ** -4)).all()


def test_fp8_block_qdq_idempotent():
    x = W.bits(W.small_matrix())
    y1 = O.fp8_block_dequant(*O.fp8_block_quant(x))
    q2, s2 = O.fp8_block_quant(y1)
    y2 = O.fp8_block_dequant(q2, s2)
    assert np.array_equal(y1, y2)
    assert np.array_equal(O.fp8_block_quant(x)[1], s2)


def test_mxfp8_dequantised_values_idempotent():
    x = W.bits(W.small_matrix())
    y1 = O.mxfp8_dequant(*O.mxfp8_quant(x))
    y2 = O.mxfp8_dequant(*O.mxfp8_quant(y1))
    assert np.array_equal(y1, y2)


def test_nvfp4_qdq_idempotent_when_block_scales_are_normal():
    x = W.bits(W.small_matrix())
    A = O.nvfp4_group_amax([x])
    packed, sb, gs = O.nvfp4_quant(x, A)
    assert ((sb & 0x78) != 0).all()                    # every block scale E4M3-normal
    y1 = O.nvfp4_fake_quant(x, A)
    A2 = O.nvfp4_group_amax([y1])
    assert A2 == A
    y2 = O.nvfp4_fake_quant(y1, A2)
    assert np.array_equal(y1, y2)
    p2, sb2, _ = O.nvfp4_quant(y1, A2)
    assert np.array_equal(p2, packed) and np.array_equal(sb2, sb)


def test_nvfp4_fake_quant_equals_dequant_of_quant():
    for seed in range(3):
        x = _tiny_input((64, 256), seed=100 + seed)
        A = O.nvfp4_group_amax([x])
        packed, sb, gs = O.nvfp4_quant(x, A)
        assert np.array_equal(O.nvfp4_fake_quant(x, A), O.nvfp4_dequant(packed, sb, gs, 256))


def test_sibling_amax_is_max_of_members():
    xs = [W.bits(W.random_bf16((8, 64), seed=s, std=0.02 * (s + 1))) for s in range(3)]
    A = O.nvfp4_group_amax(xs)
    assert A == max(float(np.abs(f32_of_bits16(x)).max()) for x in xs)
    assert A == float(np.abs(f32_of_bits16(np.concatenate([x.ravel() for x in xs]))).max())
