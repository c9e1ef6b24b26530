"""GPU parity of the NVFP4 "4over6" variant (vime pull request #503, NVFP4
QDQ config thread): codes, block scales, global scales and fake-quantised
values of nvfp4_4over6_quant / nvfp4_4over6_fake_quant, through the C ABI,
bit for bit against the oracle's restatement (readings R19-R21 of
pwq_oracle.c), for E4M3 maxima 256 and 448.  Also the division self-test
over the divisor families the variant adds.
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


def f32bits(t):
    return t.detach().contiguous().cpu().numpy().view(np.uint32)


def gpu(xbits):
    return W.from_bits(xbits, DEV)


def rand_bits(shape, seed, std=0.02):
    """Seeded BF16 bits: normals over several binades, zeros of both signs,
    subnormals and outliers."""
    rng = np.random.default_rng(seed)
    v = (rng.standard_normal(shape) * std * np.exp2(rng.integers(-3, 3, size=shape))).astype(np.float32)
    x = O.bf16_round(v)
    if x.size >= 64:
        flat = x.reshape(-1)
        idx = rng.choice(flat.size, size=flat.size // 64, replace=False)
        flat[idx[0::4]] = 0
        flat[idx[1::4]] = 0x8000
        flat[idx[2::4]] = rng.integers(1, 0x80, size=idx[2::4].size)
        flat[idx[3::4]] = O.bf16_round((rng.standard_normal(idx[3::4].size) * 50 * std).astype(np.float32))
    return x


def _oracle(xs, E):
    """Per batch index: (A, gs bits, [(packed, sb, y) per member])."""
    xs3 = [x if x.ndim == 3 else x[None] for x in xs]
    out = []
    for b in range(xs3[0].shape[0]):
        members = [x[b] for x in xs3]
        A = O.nvfp4_group_amax(members)
        res = []
        for m in members:
            pk, sb, gs = O.nvfp4_4over6_quant(m, A, E)
            res.append((pk, sb, O.nvfp4_4over6_fake_quant(m, A, E)))
        out.append((A, np.float32(O.nvfp4_4over6_global_scale(A, E)).view(np.uint32), res))
    return out


CASES = [[(1, 16)], [(2, 48)], [(33, 272)], [(3, 64, 512)], [(64, 512), (16, 512), (16, 512)],
         [(2, 40, 256), (2, 24, 256)], [(130, 1040)]]


@pytest.mark.parametrize("E", [256, 448])
@pytest.mark.parametrize("shapes", CASES, ids=lambda c: "+".join("x".join(map(str, s)) for s in c))
def test_4over6_group_exact(P, shapes, E):
    xs = [rand_bits(s, seed=300 + 5 * i + sum(s) + E) for i, s in enumerate(shapes)]
    xg = [gpu(x) for x in xs]
    packed, sb, gs = P.nvfp4_4over6_quant(xg, e4m3_max=E)
    amax_out = guard.empty((xs[0].shape[0] if xs[0].ndim == 3 else 1,), torch.float32)
    fq = P.nvfp4_4over6_fake_quant(xg, e4m3_max=E, amax_out=amax_out)
    ref = _oracle(xs, E)
    B = len(ref)
    for b, (A, gsb, outs) in enumerate(ref):
        assert f32bits(gs)[b] == gsb
        assert np.float32(amax_out[b].item()) == np.float32(A)
        for i, (opk, osb, oy) in enumerate(outs):
            assert np.array_equal(u8(sb[i]).reshape(B, -1, osb.shape[-1])[b], osb), (b, i)
            assert np.array_equal(u8(packed[i]).reshape(B, -1, opk.shape[-1])[b], opk), (b, i)
            assert np.array_equal(u16(fq[i]).reshape(B, -1, oy.shape[-1])[b], oy), (b, i)
            y = u16(P.nvfp4_dequant(packed[i], sb[i], gs)).reshape(B, -1, oy.shape[-1])[b]
            assert np.array_equal(y, oy), (b, i)


@pytest.mark.parametrize("E", [256, 448])
def test_4over6_degenerate_strided_inplace_amax_in(P, E):
    x = np.zeros((4, 32), np.uint16)
    x[0, :16] = 0x8000                                   # zero block in a live group
    x[0, 16:] = np.arange(1, 17)                         # BF16 subnormals
    x[1] = 0x3B40                                        # 1.5 * 2^-9, constant row
    x[2, ::2] = 0x4C00                                   # 2^25, the group amax
    x[3, :] = 0x0001
    A = O.nvfp4_group_amax([x])
    pk, sb, gs = P.nvfp4_4over6_quant(gpu(x), e4m3_max=E)
    opk, osb, ogs = O.nvfp4_4over6_quant(x, A, E)
    assert np.array_equal(u8(pk), opk) and np.array_equal(u8(sb), osb)
    assert np.float32(gs.item()) == np.float32(ogs)
    # all-zero group
    z = np.zeros((2, 16), np.uint16)
    z[1, 5] = 0x8000
    pz, sz, gz = P.nvfp4_4over6_quant(gpu(z), e4m3_max=E)
    assert gz.item() == 0.0 and not u8(sz).any()
    assert np.array_equal(u8(pz), O.nvfp4_4over6_quant(z, 0.0, E)[0])
    # padded rows (guarded gaps), then in place
    xs = [rand_bits((40, 256), seed=90 + E), rand_bits((24, 256), seed=91 + E)]
    xg = []
    for xb, pad in zip(xs, (32, 16)):
        v = guard.empty(xb.shape, torch.bfloat16, pad=pad)
        v.copy_(gpu(xb))
        xg.append(v)
    ref = _oracle(xs, E)[0][2]
    fq = P.nvfp4_4over6_fake_quant(xg, e4m3_max=E)
    for i in range(2):
        assert np.array_equal(u16(fq[i]), ref[i][2])
    P.nvfp4_4over6_fake_quant(xg, e4m3_max=E, inplace=True)
    for i in range(2):
        assert np.array_equal(u16(xg[i]), ref[i][2])
    # a given amax (cached / all-reduced) replaces the reduction
    xr = rand_bits((64, 512), seed=5 + E)
    Ar = O.nvfp4_group_amax([xr]) * 1.5
    amax = torch.tensor([Ar], dtype=torch.float32, device=DEV)
    p2, s2, g2 = P.nvfp4_4over6_quant(gpu(xr), e4m3_max=E, amax=amax)
    op2, os2, og2 = O.nvfp4_4over6_quant(xr, Ar, E)
    assert np.array_equal(u8(p2), op2) and np.array_equal(u8(s2), os2)
    assert np.float32(g2.item()) == np.float32(og2)
    assert np.array_equal(u16(P.nvfp4_4over6_fake_quant(gpu(xr), e4m3_max=E, amax=amax)),
                          O.nvfp4_4over6_fake_quant(xr, Ar, E))


def test_4over6_both_candidates_and_plain_nvfp4_blocks(P):
    """On a Gaussian weight both candidates occur; with E = 448 the blocks
    that keep 6 carry exactly the plain NVFP4 scale bytes."""
    x = gpu(rand_bits((256, 1024), seed=77, std=0.02))
    pk4, sb4, gs4 = P.nvfp4_4over6_quant(x, e4m3_max=448)
    pk0, sb0, gs0 = P.nvfp4_quant(x)
    assert gs4.item() == gs0.item()
    a, b = u8(sb4), u8(sb0)
    same = a == b
    assert same.any() and (~same).any()
    frac4 = 1.0 - same.mean()
    assert 0.05 < frac4 < 0.95, frac4


def test_4over6_qwen3_4b_attention_group_full_size(P):
    """q/k/v of a Qwen3-4B layer as one sibling group (E = 256): the group
    amax and global scale exactly, 24 sampled rows of every member against
    the oracle, and dequant(quant) == fake-quant on every element."""
    layer = W.qwen3_4b_layer(0, device=DEV)
    names = ["q_proj", "k_proj", "v_proj"]
    xg = [layer[n] for n in names]
    packed, sb, gs = P.nvfp4_4over6_quant(xg, e4m3_max=256)
    amax_out = torch.empty(1, dtype=torch.float32, device=DEV)
    fq = P.nvfp4_4over6_fake_quant(xg, e4m3_max=256, amax_out=amax_out)
    A = max(O.amax_bf16(u16(x)) for x in xg)
    assert np.float32(amax_out.item()) == np.float32(A)
    assert f32bits(gs)[0] == np.float32(O.nvfp4_4over6_global_scale(A, 256)).view(np.uint32)
    rng = np.random.default_rng(11)
    for i, x in enumerate(xg):
        M = x.shape[0]
        rows = sorted({0, M - 1} | set(int(r) for r in rng.integers(0, M, size=22)))
        xb = u16(x[rows])
        opk, osb, _ = O.nvfp4_4over6_quant(xb, A, 256)
        assert np.array_equal(u8(packed[i])[rows], opk), names[i]
        assert np.array_equal(u8(sb[i])[rows], osb), names[i]
        assert np.array_equal(u16(fq[i][rows]), O.nvfp4_4over6_fake_quant(xb, A, 256)), names[i]
        assert torch.equal(P.nvfp4_dequant(packed[i], sb[i], gs).view(torch.int16), fq[i].view(torch.int16))


@pytest.mark.parametrize("which", [6, 7, 8, 9])
def test_4over6_division_exhaustive(P, which):
    """The reciprocal path against IEEE division for every divisor the
    variant can form (global scale fl(a / 1536); block-scale multiplier 4)
    and every BF16 numerator it can be paired with."""
    counts = guard.empty((4,), torch.int64)
    P.check(P.lib.pwq_selftest_division(which, counts.data_ptr(), None), "pwq_selftest_division")
    torch.cuda.synchronize()
    n, code_bad, quot_bad, slow = counts.tolist()
    assert n > 10 ** 9 and code_bad == 0 and quot_bad == 0, (which, n, code_bad, quot_bad, slow)


@pytest.mark.parametrize("E", [256, 448])
def test_4over6_grouped_call_exact(P, E):
    """Several sibling groups in one grouped call: batched and plain groups,
    ragged rows, members with no rows, more than 16 members (two launches of
    each kind)."""
    shapes = [[(3, 40, 256), (3, 24, 256)], [(33, 272)], [(2, 64, 512), (2, 16, 512), (2, 16, 512)],
              [(130, 1040)], [(7, 64), (5, 64), (9, 64), (1, 64), (2, 64), (3, 64), (4, 64), (6, 64)],
              [(4, 48, 128), (4, 8, 128)], [(5, 64), (0, 64), (3, 64)], [(6, 32), (0, 32)]]
    groups = [[rand_bits(s, seed=900 + 11 * g + 3 * i + E) for i, s in enumerate(grp)] for g, grp in enumerate(shapes)]
    gg = [[gpu(x) for x in grp] for grp in groups]
    packed, sb, gs = P.nvfp4_4over6_quant_grouped(gg, E)
    amax_out = [guard.empty((grp[0].shape[0] if grp[0].ndim == 3 else 1,), torch.float32) for grp in groups]
    fq = P.nvfp4_4over6_fake_quant_grouped(gg, E, amax_out=amax_out)
    for g, grp in enumerate(groups):
        ref = _oracle(grp, E)
        B = len(ref)
        for b, (A, gsb, outs) in enumerate(ref):
            assert f32bits(gs[g])[b] == gsb, (g, b)
            assert np.float32(amax_out[g][b].item()) == np.float32(A), (g, b)
            for i, (opk, osb, oy) in enumerate(outs):
                assert np.array_equal(u8(sb[g][i]).reshape(B, -1, osb.shape[-1])[b], osb), (g, b, i)
                assert np.array_equal(u8(packed[g][i]).reshape(B, -1, opk.shape[-1])[b], opk), (g, b, i)
                assert np.array_equal(u16(fq[g][i]).reshape(B, -1, oy.shape[-1])[b], oy), (g, b, i)


def test_4over6_dsv3_experts_full_size(P):
    """The DeepSeek-V3 expert layer (256 experts; gate/up one sibling group
    per expert, down alone) through one grouped call: every expert's group
    amax and global scale exactly, and sampled rows of 6 experts (first,
    last, four random) against the oracle."""
    xs = [t for t in W.dsv3_experts(device=DEV).values()]
    packed, sb, gs = P.nvfp4_4over6_quant_grouped([xs[:2], xs[2:]], 256)
    fq = P.nvfp4_4over6_fake_quant_grouped([xs[:2], xs[2:]], 256)
    E = xs[0].shape[0]
    rng = np.random.default_rng(17)
    experts = sorted({0, E - 1} | set(int(e) for e in rng.integers(0, E, size=4)))
    for g, members in enumerate((xs[:2], xs[2:])):
        for e in experts:
            mb = [u16(m[e]) for m in members]
            A = max(O.amax_bf16(x) for x in mb)
            assert f32bits(gs[g])[e] == np.float32(O.nvfp4_4over6_global_scale(A, 256)).view(np.uint32), (g, e)
            for i, x in enumerate(mb):
                M = x.shape[0]
                rows = sorted({0, M - 1} | set(int(r) for r in rng.integers(0, M, size=6)))
                opk, osb, _ = O.nvfp4_4over6_quant(x[rows], A, 256)
                assert np.array_equal(u8(packed[g][i][e])[rows], opk), (g, e, i)
                assert np.array_equal(u8(sb[g][i][e])[rows], osb), (g, e, i)
                assert np.array_equal(u16(fq[g][i][e][rows]), O.nvfp4_4over6_fake_quant(x[rows], A, 256)), (g, e, i)


def test_4over6_w4_worked_example_on_gpu(P):
    from test_oracle_4over6 import read_w4, _bf16_bits
    w = read_w4()
    E = int(w["e4m3_max"][0])
    x = np.array([_bf16_bits(v) for v in w["x"]], np.uint16)[None]
    packed, sb, gs = P.nvfp4_4over6_quant(gpu(x), e4m3_max=E)
    assert f32bits(gs)[0] == int(w["global_scale"][0], 16)
    assert [int(v) for v in u8(sb)[0]] == [int(v, 16) for v in w["sb"]]
    assert list(u8(packed)[0]) == [int(v, 16) for v in w["packed"]]
    assert list(u16(P.nvfp4_4over6_fake_quant(gpu(x), e4m3_max=E))[0]) == [_bf16_bits(v) for v in w["y"]]
