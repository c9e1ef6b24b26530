"""GPU parity of the grouped calls (a list of tensors per launch) and of the
single-pass NVFP4 path, against the CPU oracle, bit for bit.

Lists mix ragged, batched and strided tensors; lists longer than one launch
(16 tensors) and NVFP4 calls with more than 512 group instances (one launch's
worth) exercise the host-side splitting; members larger than one work item
(16384 elements) exercise the item queue.
"""
import numpy as np
import pytest
import torch

import guard
from oracle import oracle as O
import workloads as W

from test_gpu_parity import DEV, f32bits, gpu, rand_bits, strided, u8, u16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def P():
    import precision_weight_quantization_b200 as P
    assert torch.cuda.is_available()
    return P


FP8_LIST = [(130, 260), (1, 16), (3, 129, 136), (256, 512), (64, 1000)]


def test_fp8_block_grouped_matches_oracle(P):
    xs = [rand_bits(s, seed=300 + i) for i, s in enumerate(FP8_LIST)]
    xg = []
    outs = []
    for x in xs:
        N = x.shape[-1]
        pad = (-N) % 8
        xg.append(strided(x, pad) if pad else gpu(x))
        outs.append(guard.empty(x.shape, torch.uint8, pad=(-N) % 8))
    q, s = P.fp8_block_quant_grouped(xg, out=outs)
    ys = [guard.empty(x.shape, torch.bfloat16, pad=(-x.shape[-1]) % 8) for x in xs]
    y = P.fp8_block_dequant_grouped(q, s, out=ys)
    for i, x in enumerate(xs):
        oq, os_ = O.fp8_block_quant(x)
        assert np.array_equal(u8(q[i]), oq), i
        assert np.array_equal(f32bits(s[i]), os_.view(np.uint32)), i
        assert np.array_equal(u16(y[i]), O.fp8_block_dequant(oq, os_)), i


def test_mxfp8_and_nvfp4_dequant_grouped_long_list(P):
    # 20 tensors: more than one launch's worth
    shapes = [(1 + i % 5, 32 * (1 + i % 3)) for i in range(17)] + [(2, 9, 64), (130, 4096), (3, 5, 128)]
    xs = [rand_bits(s, seed=400 + i) for i, s in enumerate(shapes)]
    xg = [gpu(x) for x in xs]
    q, e = P.mxfp8_quant_grouped(xg)
    y = P.mxfp8_dequant_grouped(q, e)
    for i, x in enumerate(xs):
        oq, oe = O.mxfp8_quant(x)
        assert np.array_equal(u8(q[i]), oq) and np.array_equal(u8(e[i]), oe), i
        assert np.array_equal(u16(y[i]), O.mxfp8_dequant(oq, oe)), i
    # NVFP4 dequant of per-tensor quantisations, grouped
    pk, sb, gs = zip(*[P.nvfp4_quant(x) for x in xg])
    yd = P.nvfp4_dequant_grouped(pk, sb, gs)
    for i, t in enumerate(yd):
        assert torch.equal(t.view(torch.int16), P.nvfp4_dequant(pk[i], sb[i], gs[i]).view(torch.int16)), i


def _check_group(P, members_bits, packed, sbs, gs, fq=None):
    """members_bits: uint16 arrays [B][M][N] (or [M][N]) of one group."""
    B = members_bits[0].shape[0] if members_bits[0].ndim == 3 else 1
    m3 = [m if m.ndim == 3 else m[None] for m in members_bits]
    for b in range(B):
        A = O.nvfp4_group_amax([m[b] for m in m3])
        if gs is not None:
            assert f32bits(gs)[b] == np.float32(O.nvfp4_global_scale(A)).view(np.uint32), b
        for i, m in enumerate(m3):
            if packed is not None:
                opk, osb, _ = O.nvfp4_quant(m[b], A)
                assert np.array_equal(u8(packed[i]).reshape(B, -1, opk.shape[-1])[b], opk), (b, i)
                assert np.array_equal(u8(sbs[i]).reshape(B, -1, osb.shape[-1])[b], osb), (b, i)
            if fq is not None:
                assert np.array_equal(u16(fq[i]).reshape(B, m.shape[1], -1)[b], O.nvfp4_fake_quant(m[b], A)), (b, i)


LAYER_GROUPS = [[(96, 256), (32, 256), (32, 256)], [(64, 384)], [(160, 512), (160, 512)], [(128, 640)],
                [(3, 40, 256), (3, 24, 256)]]


def test_nvfp4_grouped_layer_single_pass(P):
    groups = [[rand_bits(s, seed=500 + 10 * g + i) for i, s in enumerate(grp)]
              for g, grp in enumerate(LAYER_GROUPS)]
    gg = [[gpu(x) for x in grp] for grp in groups]
    packed, sb, gs = P.nvfp4_quant_grouped(gg)
    amax = [guard.empty((grp[0].shape[0] if grp[0].dim() == 3 else 1,), torch.float32)
            for grp in gg]
    fq = P.nvfp4_fake_quant_grouped(gg, amax_out=amax)
    for g, grp in enumerate(groups):
        _check_group(P, grp, packed[g], sb[g], gs[g], fq[g])
        B = amax[g].numel()
        for b in range(B):
            A = O.nvfp4_group_amax([(x if x.ndim == 3 else x[None])[b] for x in grp])
            assert np.float32(amax[g][b].item()) == np.float32(A)
    # the grouped launch equals the per-group calls
    for g, grp in enumerate(gg):
        p1, s1, g1 = P.nvfp4_quant(grp)
        for i in range(len(grp)):
            assert torch.equal(p1[i], packed[g][i])
        assert torch.equal(g1, gs[g])


def test_nvfp4_single_pass_many_items_and_inplace(P):
    # one member spans 64 work items; a second, strided member; in place
    x0 = rand_bits((1024, 1024), seed=601)
    x1 = rand_bits((96, 512), seed=602)
    g0 = gpu(x0)
    g1 = strided(x1, 64)
    ref = P.nvfp4_fake_quant([g0.clone(), g1.clone()])
    P.nvfp4_fake_quant([g0, g1], inplace=True)
    A = O.nvfp4_group_amax([x0, x1])
    assert np.array_equal(u16(g0), O.nvfp4_fake_quant(x0, A))
    assert np.array_equal(u16(g1), O.nvfp4_fake_quant(x1, A))
    assert torch.equal(ref[0].view(torch.int16), g0.view(torch.int16))


def test_nvfp4_single_pass_more_than_2048_instances(P):
    # 2100 batched groups of a sibling pair: two launch pieces
    xa = W.random_bf16((2100, 4, 64), seed=700, std=0.5, device=DEV)
    xb = W.random_bf16((2100, 2, 64), seed=701, std=0.5, device=DEV)
    xa[7] *= 1000.0
    xb[2099] *= 1e-6
    packed, sb, gs = P.nvfp4_quant([xa, xb])
    fq = P.nvfp4_fake_quant([xa, xb])
    ba, bb = u16(xa), u16(xb)
    for b in [0, 7, 1000, 2047, 2048, 2099]:
        A = O.nvfp4_group_amax([ba[b], bb[b]])
        assert f32bits(gs)[b] == np.float32(O.nvfp4_global_scale(A)).view(np.uint32), b
        for i, m in enumerate((ba[b], bb[b])):
            opk, osb, _ = O.nvfp4_quant(m, A)
            assert np.array_equal(u8(packed[i][b]), opk) and np.array_equal(u8(sb[i][b]), osb), (b, i)
            assert np.array_equal(u16(fq[i][b]), O.nvfp4_fake_quant(m, A)), (b, i)
    torch.cuda.synchronize()
    assert P.device_error() == 0


def test_tile_scale_exhaustive(P):
    counts = guard.empty((4,), torch.int64)
    P.check(P.lib.pwq_selftest_division(3, counts.data_ptr(), None), "pwq_selftest_division")
    torch.cuda.synchronize()
    n, bad, _, slow = counts.tolist()
    print("tile-scale self-test values", n, "mismatches", bad, "IEEE path", slow)
    assert n == 0x7F80 and bad == 0
