"""Pins for the oracle's FP8 block -> rollout-format re-quantisation (CPU).

The re-quantisation is defined as dequantise-then-quantise ("低精度训练与
Rollout", "FP8 训练 + FP8 Rollout" / "实现说明" item 3).  Pinned here by facts
that do not come from the oracle itself:
  * power-of-two tile scales: the dequantised values are the E4M3 values
    times 2^k exactly, so FP8 -> FP8 gives back the same codes and scales and
    FP8 -> MXFP8 keeps the codes of blocks that hold a +-448 code, with
    exponent k;
  * scaling every tile scale by 2^j scales every output scale by 2^j
    (FP8 block, NVFP4 global) or shifts every UE8M0 exponent by j, and leaves
    every code and NVFP4 block scale unchanged;
  * FP8 -> FP8 is idempotent: a second re-quantisation changes nothing;
  * brute force: every output of small inputs recomputed in exact rationals
    (tests/exact.py) through the composition, one IEEE rounding per step.
"""
from fractions import Fraction

import numpy as np
import pytest

from oracle import oracle as O
import exact as X
import workloads as W
from test_oracle_formats import ex_fp8_block, ex_mxfp8, ex_nvfp4


def random_codes(shape, seed, with_max=True):
    """E4M3 codes (no NaN), every 128x128 tile holding a +-448 code."""
    rng = np.random.default_rng(seed)
    q = rng.integers(0, 0x7F, size=shape, dtype=np.uint8)          # 0x00..0x7E
    q |= (rng.integers(0, 2, size=shape, dtype=np.uint8) << 7)
    if with_max:
        B, M, N = q.shape
        for tm in range(0, M, 128):
            for tn in range(0, N, 128):
                q[:, tm, tn] = 0x7E | (q[:, tm, tn] & 0x80)
    return q


def tile_shape(q):
    B, M, N = q.shape
    return B, -(-M // 128), -(-N // 128)


@pytest.mark.parametrize("shape", [(1, 256, 256), (2, 130, 200), (1, 1, 8)])
def test_fp8_power_of_two_scales_round_trip(shape):
    q = random_codes(shape, seed=11)
    rng = np.random.default_rng(12)
    k = rng.integers(-60, 20, size=tile_shape(q))
    s = np.ldexp(np.ones(tile_shape(q), np.float32), k).astype(np.float32)
    q2, s2 = O.fp8_block_requant(q, s)
    assert np.array_equal(q2, q)
    assert np.array_equal(s2.view(np.uint32), s.view(np.uint32))


@pytest.mark.parametrize("shape", [(1, 256, 384), (3, 130, 200)])
def test_fp8_tiles_holding_448_map_codes_to_themselves(shape):
    """Any scale with normal products, not only powers of two: when a tile
    holds a +-448 code, y = dec(q) * s * (1 + d) with |d| <= 2^-8 (one BF16
    rounding), the new scale is fl(bf16(fl(448 s)) / 448), and each quotient
    is dec(q) times a factor within about 2^-7 of 1, inside the half-step of
    E4M3 (at least 2^-5 relative for normal codes, 2^-10 absolute for
    subnormal ones): every code comes back unchanged.  The expected scale is
    formed with numpy binary32 and torch's BF16 rounding."""
    import torch
    q = random_codes(shape, seed=21)
    rng = np.random.default_rng(22)
    s = np.exp2(rng.uniform(-100.0, 100.0, size=tile_shape(q))).astype(np.float32)
    s *= np.where(rng.integers(0, 2, size=s.shape) == 1, np.float32(-1.0), np.float32(1.0))
    q2, s2 = O.fp8_block_requant(q, s)
    assert np.array_equal(q2 & 0x7F, q & 0x7F)
    # a negative scale flips every sign (the sign of zero included)
    flip = np.repeat(np.repeat(s < 0, 128, axis=1), 128, axis=2)[:, :q.shape[1], :q.shape[2]]
    assert np.array_equal(q2, np.where(flip, q ^ 0x80, q))
    top = np.float32(448.0) * np.abs(s)
    top_bf16 = torch.from_numpy(top).to(torch.bfloat16).to(torch.float32).numpy()
    assert np.array_equal(s2.view(np.uint32), (top_bf16 / np.float32(448.0)).astype(np.float32).view(np.uint32))


def test_mxfp8_power_of_two_scales_keep_codes_of_full_blocks():
    q = random_codes((1, 128, 256), seed=13, with_max=False)
    q[:, :, ::32] = 0x7E                                             # every 1x32 block holds 448
    s = np.array([[[2.0 ** -7, 2.0 ** 3]]], np.float32)
    q2, e = O.fp8_block_requant_mxfp8(q, s)
    assert np.array_equal(q2, q)
    assert (e[0, :, :4] == 127 - 7).all() and (e[0, :, 4:] == 127 + 3).all()


def _scaled(s, j):
    return (s.astype(np.float64) * 2.0 ** j).astype(np.float32)


@pytest.mark.parametrize("j", [-3, 1, 5])
def test_scale_equivariance_all_targets(j):
    x = W.bits(W.random_bf16((2, 130, 256), seed=14, std=0.02))
    q, s = O.fp8_block_quant(x)
    s = s * np.float32(1.75)                                         # scales not from this tensor
    q1, s1 = O.fp8_block_requant(q, s)
    q2, s2 = O.fp8_block_requant(q, _scaled(s, j))
    assert np.array_equal(q1, q2)
    assert np.array_equal(_scaled(s1, j).view(np.uint32), s2.view(np.uint32))
    m1, e1 = O.fp8_block_requant_mxfp8(q, s)
    m2, e2 = O.fp8_block_requant_mxfp8(q, _scaled(s, j))
    assert np.array_equal(m1, m2)
    assert np.array_equal(e1.astype(int) + j, e2.astype(int))
    A1, o1, g1 = O.fp8_block_requant_nvfp4([q], [s])
    A2, o2, g2 = O.fp8_block_requant_nvfp4([q], [_scaled(s, j)])
    assert np.array_equal(_scaled(A1, j), A2) and np.array_equal(_scaled(g1, j), g2)
    assert np.array_equal(o1[0][0], o2[0][0]) and np.array_equal(o1[0][1], o2[0][1])


def test_fp8_requant_is_idempotent():
    q = random_codes((2, 200, 300), seed=15, with_max=False)
    rng = np.random.default_rng(16)
    s = rng.uniform(1e-4, 1e-2, size=tile_shape(q)).astype(np.float32)
    q1, s1 = O.fp8_block_requant(q, s)
    q2, s2 = O.fp8_block_requant(q1, s1)
    assert np.array_equal(q1, q2) and np.array_equal(s1, s2)


def ex_fp8_dequant(q, s):
    """Exact-rational y = bf16(fl(dec(q) * s)), BF16 bits."""
    y = np.zeros(q.shape, np.uint16)
    for idx, c in np.ndenumerate(q):
        b, r, col = idx
        sc = X.f32_bits_to_exact(int(s[b, r // 128, col // 128].view(np.uint32)))
        dq = (bool(c & 0x80), X.e4m3_value(int(c) & 0x7F))
        y[idx] = X.exact_to_bf16_bits(X.rn(X.f32(X.mul(dq, sc)), X.BF16))
    return y


def test_requant_bruteforce_all_targets():
    q = random_codes((1, 130, 160), seed=17, with_max=False)
    q[0, 128:, 128:] = 0x80                                          # a tile of -0 only
    s = np.array([[[3.1e-3, 0.0], [1.7e-41, 6.0]]], np.float32)     # a zero and a subnormal scale
    y = ex_fp8_dequant(q, s)
    eq, es, _ = ex_fp8_block(y)
    oq, os_ = O.fp8_block_requant(q, s)
    assert np.array_equal(oq, eq)
    assert np.array_equal(os_.view(np.uint32), es)
    mq, me, _ = ex_mxfp8(y)
    oq, oe = O.fp8_block_requant_mxfp8(q, s)
    assert np.array_equal(oq, mq) and np.array_equal(oe, me)
    q2 = random_codes((1, 40, 96), seed=18, with_max=False)
    s2 = np.array([[[5e-4]]], np.float32)
    y2 = ex_fp8_dequant(q2, s2)
    gs, out = ex_nvfp4([y[0], y2[0]])
    A, o, g = O.fp8_block_requant_nvfp4([q, q2], [s, s2])
    assert int(g.view(np.uint32)[0]) == gs
    for (ep, esb, _), (op, osb) in zip(out, o):
        assert np.array_equal(op[0], ep) and np.array_equal(osb[0], esb)
