"""GPU parity on buffers at the smallest alignments the C ABI accepts.

Several kernels take 256-bit (32-byte) loads and stores when a tensor's base,
row stride and slab stride are multiples of 32 bytes, and narrower accesses
otherwise; the other tests mostly see freshly allocated (32-byte aligned)
tensors.  Here every operand starts 16 bytes (BF16) or 8 bytes (codes) into
a padded buffer, so the narrow paths run, and the results must still equal
the oracle's bit for bit.
"""
import numpy as np
import pytest
import torch

import guard
from oracle import oracle as O
import workloads as W

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module")
def P():
    import precision_weight_quantization_b200 as P
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return P


def u8(t):
    return t.detach().contiguous().cpu().view(torch.uint8).numpy()


def u16(t):
    return W.bits(t)


def rand_bits(shape, seed):
    rng = np.random.default_rng(seed)
    v = (rng.standard_normal(shape) * 0.02 * np.exp2(rng.integers(-3, 3, size=shape))).astype(np.float32)
    x = O.bf16_round(v)
    flat = x.reshape(-1)
    idx = rng.choice(flat.size, size=flat.size // 64, replace=False)
    flat[idx[0::3]] = 0x8000
    flat[idx[1::3]] = rng.integers(1, 0x80, size=idx[1::3].size)
    flat[idx[2::3]] = O.bf16_round((rng.standard_normal(idx[2::3].size)).astype(np.float32))
    return x


def bf16_at(xbits, lead_elems=8, pad_elems=16):
    """GPU BF16 copy of xbits whose base sits lead_elems * 2 bytes into its
    buffer and whose rows are lead + pad elements longer (base and row
    stride 16-byte but not 32-byte aligned)."""
    v = guard.empty(xbits.shape, torch.bfloat16, lead=lead_elems, pad=pad_elems)
    v.copy_(W.from_bits(xbits, DEV))
    assert v.data_ptr() % 32 == 16 and (v.stride(-2) * 2) % 32 == 16
    return v


def bf16_out(shape, lead_elems=8, pad_elems=16):
    v = guard.empty(shape, torch.bfloat16, lead=lead_elems, pad=pad_elems)
    assert v.data_ptr() % 32 == 16 and (v.stride(-2) * 2) % 32 == 16
    return v


def bytes_out(shape, lead=8, pad=8, dtype=torch.uint8):
    v = guard.empty(shape, dtype, lead=lead, pad=pad)
    assert v.data_ptr() % 16 == 8
    return v


@pytest.mark.parametrize("shape", [(3, 64), (2, 5, 256), (130, 512)], ids=str)
def test_mxfp8_narrow_alignment(P, shape):
    x = rand_bits(shape, seed=700 + sum(shape))
    q, e = P.mxfp8_quant(bf16_at(x), out=bytes_out(shape, dtype=torch.float8_e4m3fn))
    oq, oe = O.mxfp8_quant(x)
    assert np.array_equal(u8(q), oq) and np.array_equal(u8(e), oe)
    y = P.mxfp8_dequant(q, e, out=bf16_out(shape))
    assert np.array_equal(u16(y), O.mxfp8_dequant(oq, oe))


@pytest.mark.parametrize("shape", [(128, 256), (2, 130, 384)], ids=str)
def test_fp8_block_dequant_narrow_alignment(P, shape):
    # dense 16-byte aligned codes, BF16 output rows 16- but not 32-byte aligned
    x = rand_bits(shape, seed=720 + sum(shape))
    q, s = P.fp8_block_quant(W.from_bits(x, DEV))
    oq, os_ = O.fp8_block_quant(x)
    assert np.array_equal(u8(q), oq)
    y = P.fp8_block_dequant(q, s, out=bf16_out(shape))
    assert np.array_equal(u16(y), O.fp8_block_dequant(oq, os_))


def test_nvfp4_narrow_alignment(P):
    xs = [rand_bits((40, 256), seed=740), rand_bits((24, 256), seed=741)]
    xg = [bf16_at(x) for x in xs]
    A = O.nvfp4_group_amax(xs)
    ys = [bf16_out(x.shape) for x in xs]
    P.nvfp4_fake_quant(xg, out=ys)
    for x, y in zip(xs, ys):
        assert np.array_equal(u16(y), O.nvfp4_fake_quant(x, A))
    pk = [bytes_out((x.shape[0], x.shape[1] // 2)) for x in xs]
    packed, sb, gs = P.nvfp4_quant(xg, out=pk)
    for x, p, s in zip(xs, packed, sb):
        opk, osb, _ = O.nvfp4_quant(x, A)
        assert np.array_equal(u8(p), opk) and np.array_equal(u8(s), osb)
    torch.cuda.synchronize()
    assert P.device_error() == 0
