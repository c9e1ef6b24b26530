"""GPU parity: every code, scale byte, global scale and dequantised BF16 value
written by the CUDA library (through its C ABI) must equal the CPU oracle's,
bit for bit (tolerance 0: integer outputs and BF16 outputs alike).

Small and ragged cases are compared element by element; full-size workloads
are compared on sampled tiles / rows / experts, which the oracle computes
independently (tiles and rows are self-contained; NVFP4 rows get the group
amax, itself compared exactly), plus properties checked on every element.
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


def rand_bits(shape, seed, std=0.02, outliers=True):
    """Seeded BF16 bits with normals, zeros, -0, subnormals and outliers."""
    rng = np.random.default_rng(seed)
    v = (rng.standard_normal(shape) * std * np.exp2(rng.integers(-3, 3, size=shape))).astype(np.float32)
    x = O.bf16_round(v)
    if outliers and x.size >= 64:
        flat = x.reshape(-1)
        idx = rng.choice(flat.size, size=flat.size // 64, replace=False)
        flat[idx[0::4]] = 0
        flat[idx[1::4]] = 0x8000
        flat[idx[2::4]] = rng.integers(1, 0x80, size=idx[2::4].size)
        flat[idx[3::4]] = O.bf16_round((rng.standard_normal(idx[3::4].size) * 50 * std).astype(np.float32))
    return x


def strided(xbits, pad_cols, dtype_bytes=2):
    """A GPU BF16 view of xbits whose rows are padded by pad_cols elements
    (guarded: the padding must stay untouched, in place calls included)."""
    v = guard.empty(xbits.shape, torch.bfloat16, pad=pad_cols)
    v.copy_(gpu(xbits))
    return v


# ------------------------------------------------------------------ FP8 block-wise

FP8_SHAPES = [(1, 16), (2, 48), (1, 1), (7, 3), (128, 128), (130, 260), (257, 300), (3, 129, 131),
              (2, 256, 512), (1000, 8), (64, 1000), (2, 256, 640)]


@pytest.mark.parametrize("shape", FP8_SHAPES, ids=str)
def test_fp8_block_quant_dequant_exact(P, shape):
    x = rand_bits(shape, seed=sum(shape))
    N = shape[-1]
    pad = (-N) % 8                       # BF16 rows must be 16-byte aligned
    xg = strided(x, pad) if pad else gpu(x)
    if pad:
        q, s = P.fp8_block_quant(xg, out=guard.empty(shape, torch.uint8, pad=(-N) % 16))
    else:
        q, s = P.fp8_block_quant(xg)
    oq, os_ = O.fp8_block_quant(x)
    assert np.array_equal(f32bits(s), os_.view(np.uint32))
    assert np.array_equal(u8(q), oq)
    y = P.fp8_block_dequant(q, s, out=guard.empty(shape, torch.bfloat16, pad=pad))
    assert np.array_equal(u16(y), O.fp8_block_dequant(oq, os_))


def test_fp8_block_small_workload_and_degenerate_tiles(P):
    x = u16(W.small_matrix())
    q, s = P.fp8_block_quant(gpu(x))
    oq, os_ = O.fp8_block_quant(x)
    assert np.array_equal(u8(q), oq) and np.array_equal(f32bits(s), os_.view(np.uint32))
    d = np.zeros((256, 256), np.uint16)
    d[:128, :128] = 0x8000
    d[:128, 128:] = np.array([1, 0x8003, 0x7F, 0x0002], np.uint16)[np.arange(128 * 128) % 4].reshape(128, 128)
    d[128:, :128] = 0x7F7F
    d[128:, 128:] = (np.arange(128 * 128) % 0x7F00).astype(np.uint16).reshape(128, 128)
    q, s = P.fp8_block_quant(gpu(d))
    oq, os_ = O.fp8_block_quant(d)
    assert np.array_equal(u8(q), oq) and np.array_equal(f32bits(s), os_.view(np.uint32))
    assert np.array_equal(u16(P.fp8_block_dequant(q, s)), O.fp8_block_dequant(oq, os_))


# ------------------------------------------------------------------ MXFP8

MX_SHAPES = [(1, 32), (7, 96), (3, 5, 128), (130, 4096), (2, 64, 2048)]


@pytest.mark.parametrize("shape", MX_SHAPES, ids=str)
def test_mxfp8_quant_dequant_exact(P, shape):
    x = rand_bits(shape, seed=3 + sum(shape))
    q, e = P.mxfp8_quant(gpu(x))
    oq, oe = O.mxfp8_quant(x)
    assert np.array_equal(u8(e), oe)
    assert np.array_equal(u8(q), oq)
    assert np.array_equal(u16(P.mxfp8_dequant(q, e)), O.mxfp8_dequant(oq, oe))


def test_mxfp8_strided_and_extreme(P):
    x = rand_bits((3, 40, 256), seed=77)
    x[0, 0, :32] = 0x7F7F
    x[0, 1, :32] = np.arange(1, 33)
    x[1, 2, :] = 0x8000
    xg = strided(x, 64)
    q, e = P.mxfp8_quant(xg, out=guard.empty((3, 40, 256), torch.uint8, pad=48))
    oq, oe = O.mxfp8_quant(x)
    assert np.array_equal(u8(q), oq) and np.array_equal(u8(e), oe)
    y = P.mxfp8_dequant(q, e, out=guard.empty((3, 40, 256), torch.bfloat16, pad=8))
    assert np.array_equal(u16(y), O.mxfp8_dequant(oq, oe))


# ------------------------------------------------------------------ NVFP4

NV_GROUPS = [[(1, 16)], [(2, 48)], [(256, 512)], [(64, 256), (16, 256), (16, 256)],
             [(96, 2048), (96, 2048)], [(3, 8, 64), (3, 4, 64)], [(5, 33, 4096)]]


def _oracle_group(xs):
    """Per batch index b: oracle group amax over siblings' slice b, then each
    member's codes / scales / dequant / fake-quant."""
    B = xs[0].shape[0] if xs[0].ndim == 3 else 1
    xs3 = [x if x.ndim == 3 else x[None] for x in xs]
    res = []
    for b in range(B):
        members = [x[b] for x in xs3]
        A = O.nvfp4_group_amax(members)
        outs = []
        for m in members:
            packed, sb, gs = O.nvfp4_quant(m, A)
            outs.append((packed, sb, O.nvfp4_dequant(packed, sb, gs, m.shape[-1]),
                         O.nvfp4_fake_quant(m, A)))
        res.append((A, np.float32(O.nvfp4_global_scale(A)).view(np.uint32), outs))
    return res


@pytest.mark.parametrize("shapes", NV_GROUPS, ids=lambda c: "+".join("x".join(map(str, s)) for s in c))
def test_nvfp4_group_exact(P, shapes):
    xs = [rand_bits(s, seed=11 + i + sum(s)) for i, s in enumerate(shapes)]
    xg = [gpu(x) for x in xs]
    amax = P.nvfp4_group_amax(xg)
    packed, sb, gs = P.nvfp4_quant(xg)
    fq = P.nvfp4_fake_quant(xg)
    ref = _oracle_group(xs)
    B = len(ref)
    for b, (A, gsb, outs) in enumerate(ref):
        assert np.float32(amax[b].item()) == np.float32(A)
        assert f32bits(gs)[b] == gsb
        for i, (opk, osb, oy, ofq) in enumerate(outs):
            pk = u8(packed[i]).reshape(B, -1, opk.shape[-1])[b]
            sbi = u8(sb[i]).reshape(B, -1, osb.shape[-1])[b]
            assert np.array_equal(sbi, osb), (b, i)
            assert np.array_equal(pk, opk), (b, i)
            y = u16(P.nvfp4_dequant(packed[i], sb[i], gs)).reshape(B, -1, oy.shape[-1])[b]
            assert np.array_equal(y, oy), (b, i)
            assert np.array_equal(u16(fq[i]).reshape(B, -1, ofq.shape[-1])[b], ofq), (b, i)


def test_nvfp4_w3_worked_example_on_gpu(P):
    # the sibling pair of tests/golden/w3_nvfp4.txt (all values exact in BF16)
    q = O.bf16_round(np.array([2688, -2688, 2240, 1792, 1568, 1120, 784, 560, 336, 112, 120, -140,
                               0.0, -0.0, 448, 896], np.float32))[None]
    k = O.bf16_round(np.array([672, -336, 100, 3, 7, 14, 21, 28, 35, 42, 49, 56, 63, 70, 84, 0],
                              np.float32))[None]
    packed, sb, gs = P.nvfp4_quant([gpu(q), gpu(k)])
    assert f32bits(gs)[0] == 0x3F800000
    assert list(u8(packed[0])[0]) == [0xF7, 0x66, 0x46, 0x24, 0x02, 0x91, 0x80, 0x42]
    assert list(u8(packed[1])[0]) == [0xD7, 0x02, 0x00, 0x00, 0x11, 0x11, 0x11, 0x02]
    assert u8(sb[0])[0, 0] == 0x7E and u8(sb[1])[0, 0] == 0x6E


def test_nvfp4_degenerate_and_amax_in(P):
    x = np.zeros((4, 32), np.uint16)
    x[0, :16] = 0x8000
    x[0, 16:] = np.arange(1, 17)
    x[1] = 0x3B40                                    # 2^-9 * 1.5
    x[2, ::2] = 0x4C00
    x[3, :] = 0x0001
    packed, sb, gs = P.nvfp4_quant(gpu(x))
    A = O.nvfp4_group_amax([x])
    opk, osb, ogs = O.nvfp4_quant(x, A)
    assert np.array_equal(u8(packed), opk) and np.array_equal(u8(sb), osb)
    # all-zero group: gs = 0, codes keep the sign
    z = np.zeros((2, 16), np.uint16)
    z[1, 5] = 0x8000
    pz, sz, gz = P.nvfp4_quant(gpu(z))
    assert gz.item() == 0.0 and not u8(sz).any()
    assert np.array_equal(u8(pz), O.nvfp4_quant(z, 0.0)[0])
    assert np.array_equal(u16(P.nvfp4_fake_quant(gpu(z))), O.nvfp4_fake_quant(z, 0.0))
    # precomputed amax (a cached or all-reduced value) replaces the reduction
    xr = rand_bits((64, 512), seed=5)
    Ar = O.nvfp4_group_amax([xr]) * 2.0
    amax = torch.tensor([Ar], dtype=torch.float32, device=DEV)
    p2, s2, g2 = P.nvfp4_quant(gpu(xr), amax=amax)
    op2, os2, og2 = O.nvfp4_quant(xr, Ar)
    assert np.array_equal(u8(p2), op2) and np.array_equal(u8(s2), os2)
    assert np.float32(g2.item()) == np.float32(og2)
    assert np.array_equal(u16(P.nvfp4_fake_quant(gpu(xr), amax=amax)), O.nvfp4_fake_quant(xr, Ar))


def test_nvfp4_strided_inplace_and_ste(P):
    xs = [rand_bits((40, 256), seed=90), rand_bits((24, 256), seed=91)]
    xg = [strided(xs[0], 32), strided(xs[1], 16)]
    ref = _oracle_group(xs)[0]
    fq = P.nvfp4_fake_quant(xg)
    for i in range(2):
        assert np.array_equal(u16(fq[i]), ref[2][i][3])
    # in place
    xin = [gpu(x) for x in xs]
    P.nvfp4_fake_quant(xin, inplace=True)
    for i in range(2):
        assert np.array_equal(u16(xin[i]), ref[2][i][3])
    # straight-through backward: the gradient passes unchanged
    w = gpu(xs[0]).requires_grad_(True)
    y = P.NVFP4FakeQuantSTE.apply(w, None)
    g = W.normal_bf16(y.shape, 1e-3, seed=4100, device=DEV)
    y.backward(g)
    assert np.array_equal(u16(w.grad), u16(g))
    assert np.array_equal(u16(y), ref[2][0][3])
    ws = [gpu(x).requires_grad_(True) for x in xs]
    ys = P.nvfp4_fake_quant_ste(ws)
    sum((yy.float() * (k + 1)).sum() for k, yy in enumerate(ys)).backward()
    assert (ws[0].grad == 1).all() and (ws[1].grad == 2).all()


# ------------------------------------------------------------------ full-size workloads, sampled

def _sample_tiles(rng, M, N, k):
    TM, TN = -(-M // 128), -(-N // 128)
    picks = {(0, 0), (TM - 1, TN - 1)}
    while len(picks) < min(k, TM * TN):
        picks.add((int(rng.integers(TM)), int(rng.integers(TN))))
    return sorted(picks)


def test_qwen3_4b_layer_fp8_block_full_size(P):
    """Qwen3-4B decoder layer (7 weight tensors, 100.9 M elements), FP8
    block-wise: 24 sampled tiles per tensor against the oracle, dequant too."""
    layer = W.qwen3_4b_layer(0, device=DEV)
    rng = np.random.default_rng(2)
    for name, x in layer.items():
        q, s = P.fp8_block_quant(x)
        y = P.fp8_block_dequant(q, s)
        M, N = x.shape
        for tm, tn in _sample_tiles(rng, M, N, 24):
            sl = (slice(tm * 128, (tm + 1) * 128), slice(tn * 128, (tn + 1) * 128))
            xt = u16(x[sl])
            oq, os_ = O.fp8_block_quant(xt)
            assert np.float32(s[tm, tn].item()).view(np.uint32) == os_.view(np.uint32)[0, 0], (name, tm, tn)
            assert np.array_equal(u8(q[sl]), oq), (name, tm, tn)
            assert np.array_equal(u16(y[sl]), O.fp8_block_dequant(oq, os_)), (name, tm, tn)
        # every scale equals fl(tile amax / 448): tile amax from torch, the
        # IEEE binary32 division on the host
        amax = x.float().abs().reshape(M // 128, 128, N // 128, 128).amax(dim=(1, 3)).cpu().numpy()
        assert np.array_equal(f32bits(s), (amax / np.float32(448.0)).astype(np.float32).view(np.uint32)), name


def test_qwen3_30b_moe_layer_mxfp8_full_size(P):
    """128 batched experts (gate/up [128][768][2048], down [128][2048][768]),
    one call per tensor kind; sampled rows of experts {0, 127, 6 random}."""
    layer = W.qwen3_30b_moe_layer(0, device=DEV)
    rng = np.random.default_rng(3)
    experts = sorted({0, 127} | set(int(e) for e in rng.choice(128, 6, replace=False)))
    for name, x in layer.items():
        q, e = P.mxfp8_quant(x)
        y = P.mxfp8_dequant(q, e)
        rows = rng.choice(x.shape[1], 16, replace=False)
        for ex in experts:
            xr = u16(x[ex, rows])
            oq, oe = O.mxfp8_quant(xr)
            assert np.array_equal(u8(q[ex, rows]), oq) and np.array_equal(u8(e[ex, rows]), oe), (name, ex)
            assert np.array_equal(u16(y[ex, rows]), O.mxfp8_dequant(oq, oe)), (name, ex)


def test_block2048_nvfp4_qat_full_size(P):
    """2048-hidden block: q/k/v and gate/up sibling groups plus down, NVFP4
    fake-quant (W4A16) with the straight-through backward; group amax exact,
    sampled rows exact, fake-quant == dequant(quant) on every element."""
    blk = W.block2048(device=DEV)
    rng = np.random.default_rng(4)
    for group in W.BLOCK2048_GROUPS:
        xs = [blk[n] for n in group]
        A = O.nvfp4_group_amax([u16(x) for x in xs])
        amax_out = guard.empty((1,), torch.float32)
        fq = P.nvfp4_fake_quant(xs, amax_out=amax_out)
        assert np.float32(amax_out.item()) == np.float32(A)
        packed, sb, gs = P.nvfp4_quant(xs)
        for x, f, pk, s in zip(xs, fq, packed, sb):
            rows = rng.choice(x.shape[0], 24, replace=False)
            xr = u16(x[rows])
            opk, osb, _ = O.nvfp4_quant(xr, A)
            assert np.array_equal(u8(pk[rows]), opk) and np.array_equal(u8(s[rows]), osb)
            assert np.array_equal(u16(f[rows]), O.nvfp4_fake_quant(xr, A))
            assert torch.equal(P.nvfp4_dequant(pk, s, gs).view(torch.int16), f.view(torch.int16))
    # STE on the config's gradient shape
    w = blk["down_proj"].clone().requires_grad_(True)
    P.NVFP4FakeQuantSTE.apply(w, None).backward(W.block2048_grad("down_proj", device=DEV))
    assert torch.equal(w.grad.view(torch.int16), W.block2048_grad("down_proj", device=DEV).view(torch.int16))


def test_dsv3_experts_and_activation_full_size(P):
    """DeepSeek-V3-shaped experts (256 x gate/up 2048x7168 + down 7168x2048):
    FP8 block-wise and NVFP4 with per-expert gate/up siblings; W4A4
    activation 16384x7168 fake-quant.  Sampled experts / tiles / rows."""
    ex = W.dsv3_experts(device=DEV)
    rng = np.random.default_rng(5)
    pick = sorted({0, 255} | set(int(e) for e in rng.choice(256, 4, replace=False)))
    # FP8 block-wise of the batched gate tensor
    q, s = P.fp8_block_quant(ex["gate"])
    for e in pick:
        for tm, tn in _sample_tiles(rng, 2048, 7168, 4):
            sl = (e, slice(tm * 128, (tm + 1) * 128), slice(tn * 128, (tn + 1) * 128))
            oq, os_ = O.fp8_block_quant(u16(ex["gate"][sl]))
            assert np.array_equal(u8(q[sl]), oq)
            assert np.float32(s[e, tm, tn].item()).view(np.uint32) == os_.view(np.uint32)[0, 0]
    del q, s
    # NVFP4: gate/up siblings share one amax per expert; down alone
    packed, sb, gs = P.nvfp4_quant([ex["gate"], ex["up"]])
    for e in pick:
        A = O.nvfp4_group_amax([u16(ex["gate"][e]), u16(ex["up"][e])])
        assert f32bits(gs)[e] == np.float32(O.nvfp4_global_scale(A)).view(np.uint32)
        rows = rng.choice(2048, 8, replace=False)
        for i, n in enumerate(("gate", "up")):
            opk, osb, _ = O.nvfp4_quant(u16(ex[n][e, rows]), A)
            assert np.array_equal(u8(packed[i][e, rows]), opk) and np.array_equal(u8(sb[i][e, rows]), osb)
    del packed, sb, gs
    pd, sd, gd = P.nvfp4_quant(ex["down"])
    for e in pick[:3]:
        A = O.nvfp4_group_amax([u16(ex["down"][e])])
        rows = rng.choice(7168, 8, replace=False)
        opk, osb, _ = O.nvfp4_quant(u16(ex["down"][e, rows]), A)
        assert np.array_equal(u8(pd[e, rows]), opk) and np.array_equal(u8(sd[e, rows]), osb)
    del pd, sd, gd, ex
    torch.cuda.empty_cache()
    act = W.dsv3_activation(device=DEV)
    A = O.nvfp4_group_amax([u16(act)])
    fq = P.nvfp4_fake_quant(act)
    rows = rng.choice(act.shape[0], 16, replace=False)
    assert np.array_equal(u16(fq[rows]), O.nvfp4_fake_quant(u16(act[rows]), A))


# ------------------------------------------------------------------ device arithmetic self-tests

@pytest.mark.parametrize("which", [0, 1, 2], ids=["fp8_divisors", "nvfp4_divisors", "nvfp4_scale_divisors"])
def test_division_exhaustive(P, which):
    counts = guard.empty((4,), torch.int64)
    P.check(P.lib.pwq_selftest_division(which, counts.data_ptr(), None), "pwq_selftest_division")
    torch.cuda.synchronize()
    n, code_bad, quot_bad, fallback = counts.tolist()
    print("division self-test", ["fp8", "nvfp4", "nvfp4_sb"][which], "pairs", n, "code mismatches", code_bad,
          "quotient mismatches", quot_bad, "fallback pairs", fallback)
    if which in (0, 2):
        # every divisor's amax a (positive finite BF16) with every |x| <= a
        assert n == sum(2 * (a + 1) for a in range(1, 0x7F80))
    else:
        assert n > 65280 * 0x7F7F
    assert code_bad == 0
    assert quot_bad == 0


def test_absmax_rewrite_exhaustive(P):
    """The bf16x2 abs-max form of the block / tile amax equals the integer
    max of the BF16 magnitude bits for every ordered pair of finite BF16
    values (both halves of the word)."""
    counts = guard.empty((4,), torch.int64)
    P.check(P.lib.pwq_selftest_division(4, counts.data_ptr(), None), "pwq_selftest_division")
    torch.cuda.synchronize()
    n, bad = counts.tolist()[:2]
    finite = 0x10000 - 2 * 0x80    # BF16 patterns with exponent 0xff excluded
    assert n == finite * finite and bad == 0


def test_fp4_dequant_rewrite_exhaustive(P):
    """NVFP4 dequantisation through an exact binary16 product equals the
    binary32 form for every E2M1 code pair, every block scale code and every
    global scale fl(a / 2688) a BF16 group amax can give."""
    counts = guard.empty((4,), torch.int64)
    P.check(P.lib.pwq_selftest_division(5, counts.data_ptr(), None), "pwq_selftest_division")
    torch.cuda.synchronize()
    n, bad = counts.tolist()[:2]
    assert n == 0x7F80 * 127 * 256 and bad == 0


def test_device_codecs_match_oracle(P):
    """Hardware E4M3 / E2M1 / BF16 conversions against the oracle on every
    FP32 input of the active binades (both signs) and a strided sweep of the
    rest of the FP32 range."""
    def run(first, count):
        e4 = guard.empty((count,), torch.uint8)
        e2 = guard.empty((count,), torch.uint8)
        bf = guard.empty((count,), torch.int16)
        P.check(P.lib.pwq_selftest_codecs(first, count, e4.data_ptr(), e2.data_ptr(), bf.data_ptr(), None),
                "pwq_selftest_codecs")
        return e4.cpu().numpy(), e2.cpu().numpy(), bf.cpu().numpy().view(np.uint16)

    for sign in (0, 0x80000000):
        # every pattern of the E4M3 binades [2^-11, 2^10) and E2M1 binades [2^-3, 8)
        for e in range(116, 137):
            first, count = sign | (e << 23), 1 << 23
            e4, e2, bf = run(first, count)
            v = (np.arange(count, dtype=np.uint32) + np.uint32(first)).view(np.float32)
            assert np.array_equal(e4, O.e4m3_encode(v)), hex(first)
            if 124 <= e < 130:
                assert np.array_equal(e2, O.e2m1_encode(v)), hex(first)
            sel = slice(0, None, 97)
            assert np.array_equal(bf[sel], O.bf16_round(v[sel])), hex(first)
    # the rest of the FP32 range: 4096 runs of 4096 consecutive patterns,
    # one run every 2^20 patterns, every codec
    for k in range(0, 4096, 256):
        firsts = [(k + j) << 20 for j in range(256)]
        outs = [run(f, 4096) for f in firsts]
        u = np.concatenate([np.arange(f, f + 4096, dtype=np.uint64) for f in firsts]).astype(np.uint32)
        e4 = np.concatenate([o[0] for o in outs])
        e2 = np.concatenate([o[1] for o in outs])
        bf = np.concatenate([o[2] for o in outs])
        fin = (u & 0x7F800000) != 0x7F800000
        v = u[fin].view(np.float32)
        assert np.array_equal(e4[fin], O.e4m3_encode(v))
        assert np.array_equal(e2[fin], O.e2m1_encode(v))
        assert np.array_equal(bf[fin], O.bf16_round(v))


def test_no_device_errors_recorded(P):
    torch.cuda.synchronize()
    assert P.device_error() == 0


def test_empty_tensors_are_noops(P):
    x = torch.empty((0, 512), dtype=torch.bfloat16, device=DEV)
    q, s = P.fp8_block_quant(x)
    assert q.numel() == 0
    q, e = P.mxfp8_quant(x)
    assert q.numel() == 0
    assert P.nvfp4_fake_quant(x).numel() == 0


# ------------------------------------------------------------------ strided rows through the streaming dequantisers

def padded_codes(codes, pad):
    """GPU uint8 view of code bytes [.., M, N] whose rows are padded by pad bytes."""
    v = guard.empty(codes.shape, torch.uint8, pad=pad)
    v.copy_(torch.from_numpy(np.ascontiguousarray(codes)).to(DEV))
    return v


def padded_bf16_out(shape, pad):
    return guard.empty(shape, torch.bfloat16, pad=pad)


@pytest.mark.parametrize("shape,pad_q,pad_y", [((3, 130, 256), 16, 8), ((2, 256, 384), 32, 16),
                                               ((1, 96, 128), 16, 0)], ids=str)
def test_dequantisers_on_padded_rows(P, shape, pad_q, pad_y):
    """The row-streaming dequantisers on batched slabs whose code rows are
    16-byte aligned but not dense, writing BF16 rows that are 16-byte (pad
    of 8 elements) or 32-byte aligned: bit for bit the oracle's values."""
    x = rand_bits(shape, seed=sum(shape) + pad_q)
    oq, os_ = O.fp8_block_quant(x)
    y = padded_bf16_out(shape, pad_y)
    P.fp8_block_dequant(padded_codes(oq, pad_q), torch.from_numpy(os_).to(DEV), out=y)
    assert np.array_equal(u16(y), O.fp8_block_dequant(oq, os_))
    mq, me = O.mxfp8_quant(x)
    y = padded_bf16_out(shape, pad_y)
    P.mxfp8_dequant(padded_codes(mq, pad_q), torch.from_numpy(np.ascontiguousarray(me)).to(DEV), out=y)
    assert np.array_equal(u16(y), O.mxfp8_dequant(mq, me))
    per = [O.nvfp4_quant(x[b], O.nvfp4_group_amax([x[b]])) for b in range(shape[0])]
    pk = np.stack([p[0] for p in per])
    sb = np.stack([p[1] for p in per])
    gs = torch.tensor([p[2] for p in per], dtype=torch.float32, device=DEV)
    y = padded_bf16_out(shape, pad_y)
    P.nvfp4_dequant(padded_codes(pk, pad_q // 2), torch.from_numpy(sb).to(DEV), gs, out=y)
    expect = np.stack([O.nvfp4_dequant(per[b][0], per[b][1], per[b][2], shape[-1]) for b in range(shape[0])])
    assert np.array_equal(u16(y), expect)
