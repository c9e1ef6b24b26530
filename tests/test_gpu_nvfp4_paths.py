"""GPU parity of the two NVFP4 quantise / fake-quantise paths on either side
of the size that selects them: calls whose every instance (batch index of
a sibling group) has at most 131072 elements run one thread-block cluster
per instance; larger ones run the single-pass queue.  Each side is checked
bit for bit against the oracle on plain, sibling, batched, ragged, strided,
in-place and amax_in inputs, with guard bytes around every output."""
import numpy as np
import pytest
import torch

import guard
from oracle import oracle as O
import workloads as W

pytestmark = pytest.mark.gpu

DEV = "cuda"
LIMIT = 131072          # elements per instance on the cluster path


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


def rand_bits(shape, seed, std=0.02):
    rng = np.random.default_rng(seed)
    v = (rng.standard_normal(shape) * std * np.exp2(rng.integers(-3, 3, size=shape))).astype(np.float32)
    x = O.bf16_round(v)
    flat = x.reshape(-1)
    if flat.size >= 64:
        idx = rng.choice(flat.size, size=flat.size // 64, replace=False)
        flat[idx[0::4]] = 0
        flat[idx[1::4]] = 0x8000
        flat[idx[2::4]] = rng.integers(1, 0x80, size=idx[2::4].size)
        flat[idx[3::4]] = O.bf16_round((rng.standard_normal(idx[3::4].size) * 50 * std).astype(np.float32))
    return x


def padded(xbits, pad):
    v = guard.empty(xbits.shape, torch.bfloat16, pad=pad)
    v.copy_(W.from_bits(xbits, DEV))
    return v


def check_group(P, xs_bits, xg):
    """nvfp4_quant / fake-quant / dequant of one sibling group (members
    [B][M][N] or [M][N]) against the oracle, per batch index."""
    packed, sb, gs = P.nvfp4_quant(xg)
    amax_out = guard.empty((xs_bits[0].shape[0] if xs_bits[0].ndim == 3 else 1,), torch.float32)
    fq = P.nvfp4_fake_quant(xg, amax_out=amax_out)
    xs3 = [x if x.ndim == 3 else x[None] for x in xs_bits]
    B = xs3[0].shape[0]
    for b in range(B):
        members = [x[b] for x in xs3]
        A = O.nvfp4_group_amax(members)
        assert np.float32(amax_out[b].item()) == np.float32(A), b
        for i, m in enumerate(members):
            opk, osb, ogs = O.nvfp4_quant(m, A)
            assert f32bits(gs)[b] == np.float32(ogs).view(np.uint32), (b, i)
            assert np.array_equal(u8(sb[i]).reshape(B, *osb.shape)[b], osb), (b, i)
            assert np.array_equal(u8(packed[i]).reshape(B, *opk.shape)[b], opk), (b, i)
            assert np.array_equal(u16(fq[i]).reshape(B, *m.shape)[b], O.nvfp4_fake_quant(m, A)), (b, i)
            y = u16(P.nvfp4_dequant(packed[i], sb[i], gs)).reshape(B, *m.shape)[b]
            assert np.array_equal(y, O.nvfp4_dequant(opk, osb, ogs, m.shape[-1])), (b, i)


# shapes per side: (members' shapes) whose instances sit at, just below or
# just above the limit
CLUSTER = [[(128, 1024)], [(64, 1024), (32, 1024), (32, 1024)], [(1, 16)], [(33, 272)], [(64, 256, 512)],
           [(3, 100, 640), (3, 60, 640)]]
FLOW = [[(129, 1024)], [(65, 1024), (32, 1024), (32, 1024)], [(520, 272)], [(2, 130, 1040)]]


@pytest.mark.parametrize("shapes", CLUSTER + FLOW, ids=lambda c: "+".join("x".join(map(str, s)) for s in c))
def test_nvfp4_paths_exact(P, shapes):
    per_instance = sum(int(np.prod(s[-2:])) for s in shapes)
    assert (per_instance <= LIMIT) == (shapes in CLUSTER)
    xs = [rand_bits(s, seed=4000 + 13 * i + sum(s)) for i, s in enumerate(shapes)]
    check_group(P, xs, [W.from_bits(x, DEV) for x in xs])


@pytest.mark.parametrize("shapes", [[(40, 256), (24, 256)], [(520, 272), (260, 272)]], ids=["cluster", "flow"])
def test_nvfp4_paths_strided_inplace_amax_in(P, shapes):
    xs = [rand_bits(s, seed=4100 + i) for i, s in enumerate(shapes)]
    A = O.nvfp4_group_amax(xs)
    want = [O.nvfp4_fake_quant(x, A) for x in xs]
    # padded rows (guarded gaps), then in place
    xg = [padded(x, 16 * (i + 1)) for i, x in enumerate(xs)]
    check_group(P, xs, xg)
    P.nvfp4_fake_quant(xg, inplace=True)
    for i in range(len(xs)):
        assert np.array_equal(u16(xg[i]), want[i])
    # a given amax (cached / all-reduced) replaces the reduction
    amax = torch.tensor([A * 2.0], dtype=torch.float32, device=DEV)
    xg = [W.from_bits(x, DEV) for x in xs]
    packed, sb, gs = P.nvfp4_quant(xg, amax=amax)
    fq = P.nvfp4_fake_quant(xg, amax=amax)
    for i, x in enumerate(xs):
        opk, osb, ogs = O.nvfp4_quant(x, A * 2.0)
        assert np.array_equal(u8(packed[i]), opk) and np.array_equal(u8(sb[i]), osb)
        assert np.float32(gs.item()) == np.float32(ogs)
        assert np.array_equal(u16(fq[i]), O.nvfp4_fake_quant(x, A * 2.0))


def test_nvfp4_cluster_grouped_mixed_with_flow(P):
    """A grouped call whose groups are all small runs the cluster path; one
    large group sends the whole call to the single pass.  Both must agree
    with the oracle group by group."""
    small = [[rand_bits((64, 512), seed=4200)], [rand_bits((16, 512), seed=4201), rand_bits((16, 512), seed=4202)]]
    large = small + [[rand_bits((300, 512), seed=4203)]]
    for groups in (small, large):
        gg = [[W.from_bits(x, DEV) for x in g] for g in groups]
        packed, sb, gs = P.nvfp4_quant_grouped(gg)
        fq = P.nvfp4_fake_quant_grouped(gg)
        for g, grp in enumerate(groups):
            A = O.nvfp4_group_amax(grp)
            for i, x in enumerate(grp):
                opk, osb, ogs = O.nvfp4_quant(x, A)
                assert np.array_equal(u8(packed[g][i]), opk) and np.array_equal(u8(sb[g][i]), osb), (g, i)
                assert f32bits(gs[g])[0] == np.float32(ogs).view(np.uint32), g
                assert np.array_equal(u16(fq[g][i]), O.nvfp4_fake_quant(x, A)), (g, i)


def test_nvfp4_amax_given_empty_and_strided_members(P):
    """Quantise / fake-quantise with a given amax over groups whose every
    instance exceeds the cluster path's limit (the streaming encode over
    member segments): empty members between and after non-empty ones, a
    member with padded rows, two batch indices."""
    shapes = [(2, 200, 512), (2, 0, 512), (2, 130, 512), (2, 0, 512)]
    xs = [rand_bits(s, seed=4300 + i) for i, s in enumerate(shapes)]
    A = [np.float32(2.0) * np.float32(O.nvfp4_group_amax([x[b] for x in xs if x.size])) for b in range(2)]
    amax = torch.tensor(A, dtype=torch.float32, device=DEV)
    xg = [W.from_bits(x, DEV) if x.size else torch.empty(x.shape, dtype=torch.bfloat16, device=DEV) for x in xs]
    xg[2] = padded(xs[2], 24)
    packed, sb, gs = P.nvfp4_quant(xg, amax=amax)
    fq = P.nvfp4_fake_quant(xg, amax=amax)
    for b in range(2):
        for i, x in enumerate(xs):
            if not x.size:
                assert packed[i].numel() == 0 and fq[i].numel() == 0
                continue
            opk, osb, ogs = O.nvfp4_quant(x[b], A[b])
            assert f32bits(gs)[b] == np.float32(ogs).view(np.uint32), b
            assert np.array_equal(u8(packed[i][b]), opk), (b, i)
            assert np.array_equal(u8(sb[i][b]), osb), (b, i)
            assert np.array_equal(u16(fq[i][b]), O.nvfp4_fake_quant(x[b], A[b])), (b, i)
