"""The threaded oracle driver gives exactly the single-threaded oracle's
results: pieces are whole FP8 tile-row bands, whole MXFP8 / NVFP4 rows, and
the group amax is the maximum of exact partial maxima (CPU)."""
import numpy as np
import pytest

from oracle import oracle as O
from oracle import parallel as PO


def rand_bits(shape, seed):
    rng = np.random.default_rng(seed)
    v = (rng.standard_normal(shape) * np.exp2(rng.integers(-6, 6, size=shape))).astype(np.float32)
    x = O.bf16_round(v)
    x.reshape(-1)[::97] = 0x8000
    return x


@pytest.mark.parametrize("threads", [1, 3, 7])
@pytest.mark.parametrize("shape", [(300, 260), (3, 257, 384), (1, 128, 64), (5, 16)], ids=str)
def test_fp8_block_parallel_equals_serial(shape, threads):
    x = rand_bits(shape, sum(shape))
    q, s = PO.fp8_block_quant(x, threads)
    oq, os_ = O.fp8_block_quant(x)
    assert np.array_equal(q, oq) and np.array_equal(s.view(np.uint32), os_.view(np.uint32))
    assert np.array_equal(PO.fp8_block_dequant(q, s, threads), O.fp8_block_dequant(oq, os_))


@pytest.mark.parametrize("threads", [1, 4, 9])
@pytest.mark.parametrize("shape", [(77, 256), (3, 41, 512), (1, 32)], ids=str)
def test_rowwise_parallel_equals_serial(shape, threads):
    x = rand_bits(shape, 7 + sum(shape))
    q, e = PO.mxfp8_quant(x, threads)
    oq, oe = O.mxfp8_quant(x)
    assert np.array_equal(q, oq) and np.array_equal(e, oe)
    assert np.array_equal(PO.mxfp8_dequant(q, e, threads), O.mxfp8_dequant(oq, oe))
    members = [x, rand_bits((13, shape[-1]), 99)]
    A = PO.nvfp4_group_amax(members, threads)
    assert A == O.nvfp4_group_amax(members)
    pk, sb, gs = PO.nvfp4_quant(x, A, threads)
    opk, osb, ogs = O.nvfp4_quant(x, A)
    assert np.array_equal(pk, opk) and np.array_equal(sb, osb) and gs == ogs
    assert np.array_equal(PO.nvfp4_dequant(pk, sb, gs, shape[-1], threads),
                          O.nvfp4_dequant(opk, osb, ogs, shape[-1]))
    assert np.array_equal(PO.nvfp4_fake_quant(x, A, threads), O.nvfp4_fake_quant(x, A))


def test_amax_of_empty_and_host_threads():
    assert PO.amax_bf16(np.zeros(0, np.uint16), 4) == 0.0
    assert PO.host_threads() >= 1
