"""GPU parity of the tensor-core block-scale layout (bit for bit against the
oracle's index map of the oracle's dense scales): the two converters, and
MXFP8 / NVFP4 quantisation writing the layout directly (codes and global
scales identical to the dense calls)."""
import numpy as np
import pytest
import torch

import guard
from oracle import oracle as O
import workloads as W

from test_gpu_parity import DEV, f32bits, gpu, rand_bits, u8

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def P():
    import precision_weight_quantization_b200 as P
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return P


@pytest.mark.parametrize("shape", [(1, 128, 4), (3, 200, 10), (2, 256, 64), (1, 7, 1), (5, 130, 448)], ids=str)
def test_converters_match_the_oracle(P, shape):
    rng = np.random.default_rng(sum(shape))
    dense = rng.integers(1, 256, size=shape, dtype=np.uint8)
    dg = torch.from_numpy(dense).to(DEV)
    m = P.scales_to_mma(dg, out=guard.empty((O.mma_scale_bytes(*shape),), torch.uint8))
    assert np.array_equal(u8(m), O.mma_scale_layout(dense))
    back = P.scales_from_mma(m, shape, out=guard.empty(shape, torch.uint8))
    assert np.array_equal(u8(back), dense)


MX_LIST = [(130, 96), (2, 256, 2048), (3, 64, 4096), (1, 32)]


def test_mxfp8_grouped_writes_the_tile_layout(P):
    xs = [rand_bits(s, seed=600 + i) for i, s in enumerate(MX_LIST)]
    xg = [gpu(x) for x in xs]
    q, sc = P.mxfp8_quant_grouped_mma(xg)
    qd, ed = P.mxfp8_quant_grouped(xg)
    for i, x in enumerate(xs):
        oq, oe = O.mxfp8_quant(x)
        assert np.array_equal(u8(q[i]), oq) and np.array_equal(u8(q[i]), u8(qd[i])), i
        assert np.array_equal(u8(sc[i]), O.mma_scale_layout(oe)), i
        assert torch.equal(P.scales_to_mma(ed[i]), sc[i]), i


NV_GROUPS = [[(130, 48)], [(256, 512), (64, 512)], [(3, 100, 256), (3, 40, 256)], [(2, 2048, 7168)]]


def test_nvfp4_grouped_writes_the_tile_layout(P):
    groups = [[rand_bits(s, seed=650 + 10 * g + i) for i, s in enumerate(grp)] for g, grp in enumerate(NV_GROUPS)]
    gg = [[gpu(x) for x in grp] for grp in groups]
    pk, sb, gs = P.nvfp4_quant_grouped_mma(gg)
    pkd, sbd, gsd = P.nvfp4_quant_grouped(gg)
    for g, grp in enumerate(groups):
        assert torch.equal(gs[g], gsd[g]), g
        m3 = [x if x.ndim == 3 else x[None] for x in grp]
        B = m3[0].shape[0]
        for i, x in enumerate(m3):
            assert torch.equal(pk[g][i], pkd[g][i]), (g, i)
            dense = np.stack([O.nvfp4_quant(x[b], O.nvfp4_group_amax([m[b] for m in m3]))[1] for b in range(B)])
            assert np.array_equal(u8(sb[g][i]), O.mma_scale_layout(dense)), (g, i)
            assert torch.equal(P.scales_to_mma(sbd[g][i].contiguous()), sb[g][i]), (g, i)
    torch.cuda.synchronize()
    assert P.device_error() == 0
