"""GPU parity of the FP8 block-wise -> {FP8 block-wise, MXFP8, NVFP4}
re-quantisation against the oracle's dequantise-then-quantise, bit for bit.

Inputs are FP8 block-wise codes and tile scales: the library's own
quantisation of seeded BF16 tensors with the scales perturbed (so new scales
differ from the old), and raw random codes with scales that include zero,
BF16-subnormal and power-of-two values.  Ragged, batched, strided, in-place
and sibling cases; a full Qwen3-4B gate_proj compared on sampled row blocks.
"""
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
    assert torch.cuda.is_available()
    return P


def codes_and_scales(shape, seed, raw=False, max_mag=0x7E):
    """(codes uint8 numpy, scales float32 numpy) of an FP8 block-wise tensor;
    raw codes have magnitudes 0..max_mag."""
    rng = np.random.default_rng(seed)
    B, M, N = (1,) + tuple(shape) if len(shape) == 2 else tuple(shape)
    TM, TN = -(-M // 128), -(-N // 128)
    if raw:
        q = rng.integers(0, max_mag + 1, size=(B, M, N), dtype=np.uint8) | (rng.integers(0, 2, size=(B, M, N),
                                                                                   dtype=np.uint8) << 7)
        s = rng.uniform(1e-5, 1e-1, size=(B, TM, TN)).astype(np.float32)
        flat = s.reshape(-1)
        flat[0] = 0.0
        if flat.size > 1:
            flat[1] = np.float32(3e-40)          # subnormal binary32 scale
        if flat.size > 2:
            flat[2] = np.float32(2.0 ** -9)
    else:
        q, s = O.fp8_block_quant(rand_bits((B, M, N), seed))
        s = (s * rng.uniform(0.5, 2.0, size=s.shape)).astype(np.float32)
    if len(shape) == 2:
        q, s = q[0], s[0]
    return q, s


def to_gpu_codes(q, pad=0):
    if pad == 0:
        return torch.from_numpy(np.ascontiguousarray(q)).to(DEV)
    v = guard.empty(q.shape, torch.uint8, pad=pad)
    v.copy_(torch.from_numpy(np.ascontiguousarray(q)).to(DEV))
    return v


FP8_SHAPES = [((130, 200), False, 0), ((3, 129, 136), True, 8), ((1, 8), True, 0), ((256, 512), False, 0),
              ((2, 300, 1000), True, 24), ((128, 128), True, 0)]


@pytest.mark.parametrize("shape,raw,pad", FP8_SHAPES)
def test_fp8_to_fp8(P, shape, raw, pad):
    q, s = codes_and_scales(shape, seed=hash(shape) % 1000, raw=raw)
    oq, os_ = O.fp8_block_requant(q, s)
    gq, gs = P.fp8_block_requant(to_gpu_codes(q, pad), torch.from_numpy(s).to(DEV))
    assert np.array_equal(u8(gq), oq)
    assert np.array_equal(f32bits(gs), os_.view(np.uint32))


def test_fp8_to_fp8_in_place(P):
    q, s = codes_and_scales((2, 260, 384), seed=5)
    tq, ts = to_gpu_codes(q), torch.from_numpy(s).to(DEV)
    P.fp8_block_requant(tq, ts, inplace=True)
    oq, os_ = O.fp8_block_requant(q, s)
    assert np.array_equal(u8(tq), oq) and np.array_equal(f32bits(ts), os_.view(np.uint32))


@pytest.mark.parametrize("max_mag", [0x7D, 0x70, 0x38, 0x06])
def test_fp8_to_fp8_tiles_below_448(P, max_mag):
    """Tiles whose largest code is below 448 change their codes (the per-tile
    code map is not the identity: normal, subnormal-only and mixed tiles),
    side by side in one launch with tiles that hold 448 (whose codes come
    back unchanged)."""
    q, s = codes_and_scales((3, 256, 384), seed=40 + max_mag, raw=True, max_mag=max_mag)
    qf, sf = codes_and_scales((3, 256, 384), seed=41, raw=False)
    q[:, :128, :] = qf[:, :128, :]
    s[:, 0, :] = sf[:, 0, :]
    s[1] = -s[1]                                   # negative scales flip signs
    oq, os_ = O.fp8_block_requant(q, s)
    assert not np.array_equal(oq[:, 128:, :], q[:, 128:, :])
    gq, gs = P.fp8_block_requant(to_gpu_codes(q), torch.from_numpy(s).to(DEV))
    assert np.array_equal(u8(gq), oq)
    assert np.array_equal(f32bits(gs), os_.view(np.uint32))


MX_SHAPES = [((130, 256), False, 0), ((3, 129, 160), True, 16), ((1, 32), True, 0), ((2, 300, 1024), False, 32)]


@pytest.mark.parametrize("shape,raw,pad", MX_SHAPES)
def test_fp8_to_mxfp8(P, shape, raw, pad):
    q, s = codes_and_scales(shape, seed=7 + len(shape), raw=raw)
    oq, oe = O.fp8_block_requant_mxfp8(q, s)
    gq, ge = P.fp8_block_requant_mxfp8(to_gpu_codes(q, pad), torch.from_numpy(s).to(DEV))
    assert np.array_equal(u8(gq), oq) and np.array_equal(u8(ge), oe)
    # in place over the codes
    tq = to_gpu_codes(q, pad)
    P.fp8_block_requant_mxfp8(tq, torch.from_numpy(s).to(DEV), inplace=True)
    assert np.array_equal(u8(tq), oq)


@pytest.mark.parametrize("shapes,raw", [([(96, 256), (32, 256), (32, 256)], False),
                                        ([(3, 40, 160), (3, 24, 160)], True),
                                        ([(130, 64)], True)])
def test_fp8_to_nvfp4_siblings(P, shapes, raw):
    members = [codes_and_scales(sh, seed=20 + i, raw=raw) for i, sh in enumerate(shapes)]
    A, out, gs = O.fp8_block_requant_nvfp4([m[0] for m in members], [m[1] for m in members])
    qs = [to_gpu_codes(m[0]) for m in members]
    ss = [torch.from_numpy(m[1]).to(DEV) for m in members]
    pk, sb, g = P.fp8_block_requant_nvfp4(qs, ss)
    assert np.array_equal(f32bits(g), gs.view(np.uint32))
    for i in range(len(shapes)):
        assert np.array_equal(u8(pk[i]), out[i][0]), i
        assert np.array_equal(u8(sb[i]), out[i][1]), i
    # the same with the amax given (e.g. after an all-reduce)
    pk2, sb2, g2 = P.fp8_block_requant_nvfp4(qs, ss, amax=torch.from_numpy(A).to(DEV))
    assert torch.equal(g2, g)
    for i in range(len(shapes)):
        assert torch.equal(pk2[i], pk[i]) and torch.equal(sb2[i].view(torch.uint8), sb[i].view(torch.uint8))


@pytest.mark.parametrize("pad", [8, 16])   # code rows 8- and 16-byte aligned
def test_fp8_to_nvfp4_strided_codes_amax_given(P, pad):
    """Padded (strided) code rows, batched, a sibling pair, with the group
    amax given: the streaming encode addresses each block through its row
    and column; codes, block scales and global scales against the oracle."""
    members = [codes_and_scales(sh, seed=60 + i, raw=True) for i, sh in enumerate([(2, 130, 272), (2, 70, 272)])]
    A, out, gs = O.fp8_block_requant_nvfp4([m[0] for m in members], [m[1] for m in members])
    qs = [to_gpu_codes(m[0], pad) for m in members]
    ss = [torch.from_numpy(m[1]).to(DEV) for m in members]
    pk, sb, g = P.fp8_block_requant_nvfp4(qs, ss, amax=torch.from_numpy(A).to(DEV))
    assert np.array_equal(f32bits(g), gs.view(np.uint32))
    for i in range(2):
        assert np.array_equal(u8(pk[i]), out[i][0]), i
        assert np.array_equal(u8(sb[i]), out[i][1]), i


def test_fp8_to_nvfp4_codes_only_8_byte_aligned(P):
    """E4M3 code tensors need only 8-byte alignment: dense code rows whose
    base, or whose batch stride, is 8 bytes off a 16-byte boundary are read
    with 8-byte loads instead of the stage copy, with the same results."""
    M, N = 256, 512
    q, s = codes_and_scales((2, M, N), seed=41)
    want = [O.fp8_block_requant_nvfp4([q[b]], [s[b]]) for b in range(2)]
    # one matrix at base + 8
    buf = torch.zeros(M * N + 8, dtype=torch.uint8, device=DEV)
    q0 = buf[8:8 + M * N].view(M, N)
    q0.copy_(torch.from_numpy(q[0]).to(DEV))
    assert q0.data_ptr() % 16 == 8
    pk, sb, g = P.fp8_block_requant_nvfp4(q0, torch.from_numpy(s[0]).to(DEV))
    A, out, gs = want[0]
    assert np.array_equal(f32bits(g), gs.view(np.uint32))
    assert np.array_equal(u8(pk), out[0][0]) and np.array_equal(u8(sb), out[0][1])
    # the same with the amax given (the streaming encode reads 8-byte code pairs)
    pk, sb, g = P.fp8_block_requant_nvfp4(q0, torch.from_numpy(s[0]).to(DEV), amax=torch.from_numpy(A).to(DEV))
    assert np.array_equal(f32bits(g), gs.view(np.uint32))
    assert np.array_equal(u8(pk), out[0][0]) and np.array_equal(u8(sb), out[0][1])
    # a batch of two with a batch stride of M * N + 8 bytes
    bs = M * N + 8
    buf2 = torch.zeros(2 * bs, dtype=torch.uint8, device=DEV)
    q2 = buf2.as_strided((2, M, N), (bs, N, 1))
    for b in range(2):
        q2[b].copy_(torch.from_numpy(q[b]).to(DEV))
    pk2, sb2, g2 = P.fp8_block_requant_nvfp4(q2, torch.from_numpy(s).to(DEV))
    for b in range(2):
        A, out, gs = want[b]
        assert f32bits(g2)[b] == gs.view(np.uint32)[0], b
        assert np.array_equal(u8(pk2[b]), out[0][0]) and np.array_equal(u8(sb2[b]), out[0][1]), b


def test_fp8_to_nvfp4_equals_quant_of_dequant_on_gpu(P):
    q, s = codes_and_scales((4, 200, 512), seed=31)
    tq, ts = to_gpu_codes(q), torch.from_numpy(s).to(DEV)
    y = P.fp8_block_dequant(tq, ts)
    pk_ref, sb_ref, gs_ref = P.nvfp4_quant(y)
    pk, sb, gs = P.fp8_block_requant_nvfp4(tq, ts)
    assert torch.equal(gs, gs_ref) and torch.equal(pk, pk_ref)
    assert torch.equal(sb.view(torch.uint8), sb_ref.view(torch.uint8))


def test_full_size_gate_proj_sampled(P):
    # Qwen3-4B gate_proj (9728 x 2560) quantised to FP8 block-wise on the GPU,
    # then re-quantised; the oracle recomputes sampled 128-row blocks
    x = W.qwen3_4b_layer(0, device=DEV)["gate_proj"]
    q, s = P.fp8_block_quant(x)
    s = s * 1.5
    rq, rs = P.fp8_block_requant(q, s)
    mq, me = P.fp8_block_requant_mxfp8(q, s)
    pk, sb, gs = P.fp8_block_requant_nvfp4(q, s)
    qn, sn = u8(q), s.cpu().numpy()
    y = O.fp8_block_dequant(qn, sn)
    A = np.float32(O.nvfp4_group_amax([y]))
    assert f32bits(gs)[0] == np.float32(O.nvfp4_global_scale(A)).view(np.uint32)
    rqn, rsn, mqn, men, pkn, sbn = u8(rq), f32bits(rs), u8(mq), u8(me), u8(pk), u8(sb)
    for tm in [0, 1, 37, 75]:
        r0, r1 = tm * 128, (tm + 1) * 128
        oq, os_ = O.fp8_block_requant(qn[r0:r1], sn[tm:tm + 1])
        assert np.array_equal(rqn[r0:r1], oq) and np.array_equal(rsn[tm:tm + 1], os_.view(np.uint32))
        oq, oe = O.fp8_block_requant_mxfp8(qn[r0:r1], sn[tm:tm + 1])
        assert np.array_equal(mqn[r0:r1], oq) and np.array_equal(men[r0:r1], oe)
        opk, osb, _ = O.nvfp4_quant(y[r0:r1], A)
        assert np.array_equal(pkn[r0:r1], opk) and np.array_equal(sbn[r0:r1], osb)


def test_fp8_to_nvfp4_grouped_single_pass(P):
    # a layer-like list of sibling groups in one launch: ragged rows, a batched
    # group, a strided member (read without the bulk copy) and a member larger
    # than one 16384-element work item
    specs = [[((96, 256), 0), ((32, 256), 16), ((32, 256), 0)], [((1024, 512), 0)],
             [((3, 40, 160), 0), ((3, 24, 160), 8)], [((130, 64), 0)]]
    groups, scales, oracle = [], [], []
    for g, grp in enumerate(specs):
        ms = [codes_and_scales(sh, seed=40 + 5 * g + i, raw=(g % 2 == 1)) for i, (sh, _) in enumerate(grp)]
        groups.append([to_gpu_codes(m[0], pad) for m, (_, pad) in zip(ms, grp)])
        scales.append([torch.from_numpy(m[1]).to(DEV) for m in ms])
        oracle.append(O.fp8_block_requant_nvfp4([m[0] for m in ms], [m[1] for m in ms]))
    pk, sb, gs = P.fp8_block_requant_nvfp4_grouped(groups, scales)
    for g, (A, out, ogs) in enumerate(oracle):
        assert np.array_equal(f32bits(gs[g]), ogs.view(np.uint32)), g
        for i in range(len(out)):
            assert np.array_equal(u8(pk[g][i]), out[i][0]), (g, i)
            assert np.array_equal(u8(sb[g][i]), out[i][1]), (g, i)
    torch.cuda.synchronize()
    assert P.device_error() == 0


def test_fp8_to_fp8_and_mxfp8_grouped(P):
    # 20 tensors (two launches of 16), ragged and batched; the MXFP8 list is
    # run twice: 16-byte aligned rows (grouped 16-code kernel) and with one
    # member on 8-byte row strides (per-tensor fallback)
    shapes = [(1 + 37 * i, 32 * (1 + i % 5)) for i in range(18)] + [(2, 130, 256), (129, 160)]
    ms = [codes_and_scales(sh, seed=60 + i, raw=(i % 3 == 0)) for i, sh in enumerate(shapes)]
    qs = [to_gpu_codes(m[0]) for m in ms]
    ss = [torch.from_numpy(m[1]).to(DEV) for m in ms]
    rq, rs = P.fp8_block_requant_grouped(qs, ss)
    mq, me = P.fp8_block_requant_mxfp8_grouped(qs, ss)
    for i, (q, s) in enumerate(ms):
        oq, os_ = O.fp8_block_requant(q, s)
        assert np.array_equal(u8(rq[i]), oq) and np.array_equal(f32bits(rs[i]), os_.view(np.uint32)), i
        oq, oe = O.fp8_block_requant_mxfp8(q, s)
        assert np.array_equal(u8(mq[i]), oq) and np.array_equal(u8(me[i]), oe), i
    qs8 = list(qs)
    qs8[5] = to_gpu_codes(ms[5][0], pad=8)
    mq8, me8 = P.fp8_block_requant_mxfp8_grouped(qs8, ss)
    for i in range(len(ms)):
        assert torch.equal(mq8[i].view(torch.uint8), mq[i].view(torch.uint8)) and torch.equal(me8[i], me[i]), i
    # in place, grouped
    qi = [q.clone() for q in qs]
    si = [s.clone() for s in ss]
    P.fp8_block_requant_grouped(qi, si, inplace=True)
    for i in range(len(ms)):
        assert torch.equal(qi[i].view(torch.uint8), rq[i].view(torch.uint8)) and torch.equal(si[i], rs[i]), i
