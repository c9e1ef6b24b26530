"""The sharded NVFP4 path on one GPU: two ranks' row shards of a sibling group
are reduced separately with nvfp4_group_amax, the all-reduce (MAX) is
emulated on the device, and each shard quantised with the global amax must
give exactly the rows of the unsharded quantisation and of the oracle."""
import numpy as np
import pytest
import torch

from oracle import oracle as O
import workloads as W

from test_gpu_parity import DEV, f32bits, gpu, u8, u16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def P():
    import precision_weight_quantization_b200 as P
    assert torch.cuda.is_available()
    return P


def test_row_sharded_group_matches_unsharded(P):
    from precision_weight_quantization_b200.dist import nvfp4_fake_quant_sharded, row_shard
    shapes = [(1000, 512), (200, 512), (200, 512)]        # a q/k/v-like sibling group
    full = [W.random_bf16(s, seed=950 + i, std=0.02, device=DEV) for i, s in enumerate(shapes)]
    full[2][199, 5] = 3.0                                   # the amax sits in rank 1's rows
    world = 2
    shards = [[row_shard(x, r, world) for x in full] for r in range(world)]
    part = [P.nvfp4_group_amax(s) for s in shards]
    glob = torch.maximum(part[0], part[1])                  # the all-reduce (MAX)
    A = O.nvfp4_group_amax([W.bits(x) for x in full])
    assert f32bits(glob)[0] == np.float32(A).view(np.uint32)
    assert torch.equal(glob, P.nvfp4_group_amax(full))
    pk_full, sb_full, gs_full = P.nvfp4_quant(full)
    fq_full = P.nvfp4_fake_quant(full)
    for r in range(world):
        pk, sb, gs = P.nvfp4_quant(shards[r], amax=glob)
        assert torch.equal(gs, gs_full)
        for i, x in enumerate(full):
            rows = row_shard(torch.arange(x.shape[0], device=DEV)[:, None], r, world)[:, 0]
            assert torch.equal(pk[i], pk_full[i][rows]), (r, i)
            assert torch.equal(sb[i].view(torch.uint8), sb_full[i].view(torch.uint8)[rows]), (r, i)
            opk, osb, _ = O.nvfp4_quant(W.bits(shards[r][i]), A)
            assert np.array_equal(u8(pk[i]), opk) and np.array_equal(u8(sb[i]), osb), (r, i)
        fq = P.nvfp4_fake_quant(shards[r], amax=glob)
        for i, x in enumerate(full):
            rows = row_shard(torch.arange(x.shape[0], device=DEV)[:, None], r, world)[:, 0]
            assert torch.equal(fq[i].view(torch.int16), fq_full[i][rows].view(torch.int16)), (r, i)
    # without a process group the helper reduces the local shards only:
    # with every shard local it is the unsharded call
    out = nvfp4_fake_quant_sharded([full])
    for i in range(len(full)):
        assert torch.equal(out[0][i].view(torch.int16), fq_full[i].view(torch.int16))
