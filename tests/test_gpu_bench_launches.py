"""GPU parity of the very launches bench.py times, built by bench.py's own
workload builders (so the launch shape -- tensors per launch, sibling
groups, batch slabs, instances per single-pass launch -- is the timed one):

  - the headline: DeepSeek-V3 expert layer (256 experts x gate/up/down, one
    grouped launch per op; NVFP4 with 512 instances in one single-pass
    launch) and the W4A4 activation, at full size, sampled;
  - the Qwen3-4B sweep's grouped calls over two layers (14 tensors, 8
    sibling groups in one launch), sampled, group amax exact, and the
    next-row launches on them (FP8 block-wise -> NVFP4, NVFP4 4over6);
  - the Qwen3-30B-A3B expert layer's MXFP8 call on layers 0, 47 and 8
    random layers, sampled;
  - the 2048-hidden QAT block's single launch over three sibling groups,
    every element;
  - the 256 x 512 matrix alone and as a batch of 64, every element.

Every output buffer of the builders is a guarded buffer (the test hands
them the guard module's torch stand-in): bytes around each output must be
unchanged.  The oracle's threaded driver computes the group amax over whole
groups and the sampled rows / tiles.  Tolerance 0 throughout.
"""
import numpy as np
import pytest
import torch

import bench
import guard
from oracle import oracle as O
from oracle import parallel as PO
import workloads as W

pytestmark = pytest.mark.gpu

DEV = "cuda"
T = guard._TorchProxy()      # torch whose CUDA empty / empty_like give guarded buffers


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


def tiles(rng, M, N, k):
    TM, TN = -(-M // 128), -(-N // 128)
    picks = {(0, 0), (TM - 1, TN - 1), (0, TN - 1), (TM - 1, 0)}
    while len(picks) < min(k, TM * TN):
        picks.add((int(rng.integers(TM)), int(rng.integers(TN))))
    return sorted(picks)


def check_fp8(x, q, s, y, rng, k=8, lead=()):
    """Sampled 128x128 tiles (corners included) of one matrix x[lead]."""
    M, N = x.shape[-2:]
    for tm, tn in tiles(rng, M, N, k):
        sl = lead + (slice(tm * 128, (tm + 1) * 128), slice(tn * 128, (tn + 1) * 128))
        oq, os_ = O.fp8_block_quant(u16(x[sl]))
        assert np.array_equal(u8(q[sl]), oq), (lead, tm, tn)
        assert f32bits(s[lead + (tm, tn)].reshape(1))[0] == os_.view(np.uint32)[0, 0], (lead, tm, tn)
        assert np.array_equal(u16(y[sl]), O.fp8_block_dequant(oq, os_)), (lead, tm, tn)


def sample_rows(rng, M, k):
    return np.unique(np.concatenate([[0, M - 1], rng.choice(M, min(k, M), replace=False)]))


def check_mx(x, q, e, y, rng, k=16, lead=()):
    rows = sample_rows(rng, x.shape[-2], k)
    sl = lead + (rows,)
    oq, oe = O.mxfp8_quant(u16(x[sl]))
    assert np.array_equal(u8(q[sl]), oq) and np.array_equal(u8(e[sl]), oe), lead
    assert np.array_equal(u16(y[sl]), O.mxfp8_dequant(oq, oe)), lead


def check_nv_rows(x, A, pk, sb, rng, k=16, lead=()):
    rows = sample_rows(rng, x.shape[-2], k)
    sl = lead + (rows,)
    opk, osb, ogs = O.nvfp4_quant(u16(x[sl]), A)
    assert np.array_equal(u8(pk[sl]), opk) and np.array_equal(u8(sb[sl]), osb), lead
    return rows, opk, osb, ogs


# ------------------------------------------------------------------ the headline launch shapes

def test_headline_dsv3_experts_and_activation_launches(P):
    w = bench.dsv3_workload(P, T, DEV, rank=0, experts=256)
    t = w.tensors
    ops = {op.name: op for op in w.ops}
    xs, names = t["xs"], t["names"]
    rng = np.random.default_rng(55)
    experts = sorted({0, 255} | set(int(e) for e in rng.choice(256, 3, replace=False)))
    # FP8 block-wise: quantise all three tensors in one launch, dequantise
    ops["fp8_block_quant"].run()
    ops["fp8_block_dequant"].run()
    for i, x in enumerate(xs):
        for e in experts:
            check_fp8(x, t["q"][i], t["s"][i], t["y"][i], rng, k=6, lead=(e,))
    # MXFP8
    ops["mxfp8_quant"].run()
    ops["mxfp8_dequant"].run()
    for i, x in enumerate(xs):
        for e in experts:
            check_mx(x, t["mq"][i], t["me"][i], t["y"][i], rng, lead=(e,))
    # NVFP4: {gate, up} of each expert one group, down its own; 512 instances in one launch
    ops["nvfp4_quant"].run()
    ops["nvfp4_dequant"].run()
    for e in experts:
        for gi, members in enumerate(([0, 1], [2])):
            A = PO.nvfp4_group_amax([u16(xs[i][e]) for i in members])
            assert f32bits(t["gs"][gi])[e] == np.float32(O.nvfp4_global_scale(A)).view(np.uint32), (e, gi)
            for i in members:
                rows, opk, osb, ogs = check_nv_rows(xs[i], A, t["pk"][i], t["sb"][i], rng, lead=(e,))
                oy = O.nvfp4_dequant(opk, osb, ogs, xs[i].shape[-1])
                assert np.array_equal(u16(t["y"][i][e, rows]), oy), (e, i)
    # W4A4 activation: its own dynamic amax, one single-pass launch
    ops["nvfp4_fake_quant"].run()
    act = t["act"]
    A = PO.nvfp4_group_amax([u16(act)])
    assert np.float32(t["act_amax"].item()) == np.float32(A)
    rows = sample_rows(rng, act.shape[0], 24)
    assert np.array_equal(u16(t["yact"][rows]), O.nvfp4_fake_quant(u16(act[rows]), A))
    torch.cuda.synchronize()
    assert P.device_error() == 0


# ------------------------------------------------------------------ per-config launch shapes

def test_qwen3_4b_two_layer_grouped_launches(P):
    """bench.py's grouped calls over two Qwen3-4B layers: 14 tensors per
    launch, 8 NVFP4 sibling groups (q/k/v, o, gate/up, down per layer) in
    one single-pass launch."""
    w = bench.qwen3_4b_workload(P, T, DEV, rank=0, layers=2, per_call=2)
    layers, buf = w.tensors["layers"], w.tensors["buf"]
    ops = {op.name: op for op in w.ops}
    assert all(len(op.calls) == 1 for op in w.ops)
    rng = np.random.default_rng(42)
    ops["fp8_block_quant"].run()
    ops["fp8_block_dequant"].run()
    for i, lay in enumerate(layers):
        for n, x in lay.items():
            q, s = buf.fp8[i][n]
            check_fp8(x, q, s, buf.y[i][n], rng, k=12)
    ops["mxfp8_quant"].run()
    ops["mxfp8_dequant"].run()
    for i, lay in enumerate(layers):
        for n, x in lay.items():
            q, e = buf.mx[i][n]
            check_mx(x, q, e, buf.y[i][n], rng)
    ops["nvfp4_quant"].run()
    ops["nvfp4_dequant"].run()
    amax = {}
    for i, lay in enumerate(layers):
        for g in W.QWEN3_4B_GROUPS:
            pk, sb, gs = buf.nv[i][g]
            A = PO.nvfp4_group_amax([u16(lay[n]) for n in g])
            amax[i, g] = A
            assert f32bits(gs)[0] == np.float32(O.nvfp4_global_scale(A)).view(np.uint32), (i, g)
            for j, n in enumerate(g):
                rows, opk, osb, ogs = check_nv_rows(lay[n], A, pk[j], sb[j], rng)
                assert np.array_equal(u16(buf.y[i][n][rows]), O.nvfp4_dequant(opk, osb, ogs, lay[n].shape[-1]))
    ops["nvfp4_fake_quant"].run()
    for i, lay in enumerate(layers):
        for g in W.QWEN3_4B_GROUPS:
            for n in g:
                rows = sample_rows(rng, lay[n].shape[0], 16)
                assert np.array_equal(u16(buf.y[i][n][rows]), O.nvfp4_fake_quant(u16(lay[n][rows]), amax[i, g])), \
                    (i, n)
    torch.cuda.synchronize()
    assert P.device_error() == 0


def test_qwen3_4b_next_rows_launches(P):
    """bench.py's next-row launches over two Qwen3-4B layers: the FP8
    block-wise -> NVFP4 single pass over the sweep's FP8 outputs (14 members,
    8 sibling groups in one launch) and the NVFP4 4over6 grouped calls;
    group amax and global scales exact, sampled rows against the oracle."""
    w = bench.qwen3_4b_workload(P, T, DEV, rank=0, layers=2, per_call=2)
    layers, buf = w.tensors["layers"], w.tensors["buf"]
    ops = {op.name: op for op in w.ops}
    ops["fp8_block_quant"].run()          # the FP8 codes and tile scales the rows read
    rng = np.random.default_rng(77)
    calls, out = bench.next_calls("fp8_block_requant_nvfp4", layers, buf, P, T, 2)
    assert len(calls) == 1
    calls[0]()
    for i, lay in enumerate(layers):
        for j, g in enumerate(W.QWEN3_4B_GROUPS):
            # the dequantised members, from the oracle's threaded driver
            ys = [PO.fp8_block_dequant(u8(buf.fp8[i][n][0]), buf.fp8[i][n][1].cpu().numpy()) for n in g]
            A = PO.nvfp4_group_amax(ys)
            assert f32bits(out["gs"][i][j])[0] == np.float32(O.nvfp4_global_scale(A)).view(np.uint32), (i, g)
            for n, y in zip(g, ys):
                rows = sample_rows(rng, y.shape[0], 12)
                opk, osb, _ = O.nvfp4_quant(y[rows], A)
                assert np.array_equal(u8(out["pk"][i][n][rows]), opk), (i, n)
                assert np.array_equal(u8(out["sb"][i][n])[rows], osb), (i, n)
    for op in ("nvfp4_4over6_quant", "nvfp4_4over6_fake_quant"):
        calls, outs = bench.four_six_calls(op, layers, P, T, 2)
        assert len(calls) == 1
        calls[0]()
        groups = outs[0][0]
        assert len(groups) == 8 and sum(len(g) for g in groups) == 14
        for gi, grp in enumerate(groups):
            xb = [u16(x) for x in grp]
            A = PO.nvfp4_group_amax(xb)
            if op == "nvfp4_4over6_quant":
                _, pk, sb, gs = outs[0]
                assert f32bits(gs[gi])[0] == np.float32(O.nvfp4_4over6_global_scale(A, 256)).view(np.uint32), gi
            for mi, x in enumerate(xb):
                rows = sample_rows(rng, x.shape[0], 12)
                if op == "nvfp4_4over6_quant":
                    opk, osb, _ = O.nvfp4_4over6_quant(x[rows], A, 256)
                    assert np.array_equal(u8(pk[gi][mi])[rows], opk), (gi, mi)
                    assert np.array_equal(u8(sb[gi][mi])[rows], osb), (gi, mi)
                else:
                    ys = outs[0][1]
                    assert np.array_equal(u16(ys[gi][mi][rows]), O.nvfp4_4over6_fake_quant(x[rows], A, 256)), (gi, mi)
    torch.cuda.synchronize()
    assert P.device_error() == 0


def test_qwen3_30b_moe_mxfp8_first_last_and_random_layers(P):
    """The Qwen3-30B-A3B expert layer's grouped MXFP8 call (three batched
    tensors of 128 experts, one launch) on layers 0, 47 and 8 random ones."""
    rng = np.random.default_rng(30)
    picks = sorted({0, 47} | set(int(v) for v in rng.choice(np.arange(1, 47), 8, replace=False)))
    assert len(picks) == 10
    for L in picks:
        w = bench.qwen3_30b_workload(P, T, DEV, layers=1, layer_index=L)
        t = w.tensors
        for op in w.ops:
            op.run()
        for i, x in enumerate(t["xs"]):
            for e in sorted({0, 127} | set(int(v) for v in rng.choice(128, 2, replace=False))):
                check_mx(x, t["q"][i], t["e"][i], t["y"][i], rng, k=8, lead=(e,))
        del w, t
    torch.cuda.synchronize()
    assert P.device_error() == 0


def test_block2048_qat_launch_every_element(P):
    """The QAT block's one launch over its three sibling groups: group amax
    exact and every element of every member, against the oracle."""
    w = bench.block2048_workload(P, T, DEV)
    t = w.tensors
    w.ops[0].run()
    for gi, g in enumerate(t["groups"]):
        bits = [u16(x) for x in g]
        A = PO.nvfp4_group_amax(bits)
        assert np.float32(t["amax"][gi].item()) == np.float32(A), gi
        for j, b in enumerate(bits):
            assert np.array_equal(u16(t["ys"][gi][j]), PO.nvfp4_fake_quant(b, A)), (gi, j)


@pytest.mark.parametrize("batch", [1, 64])
def test_small_matrix_launches_every_element(P, batch):
    w = bench.small_workload(P, T, DEV, batch)
    t = w.tensors
    ops = {op.name: op for op in w.ops}
    xb = u16(t["x"])
    ops["fp8_block_quant"].run()
    ops["fp8_block_dequant"].run()
    oq, os_ = O.fp8_block_quant(xb)
    assert np.array_equal(u8(t["q"]), oq) and np.array_equal(f32bits(t["s"]).reshape(-1), os_.view(np.uint32).reshape(-1))
    assert np.array_equal(u16(t["y"]), O.fp8_block_dequant(oq, os_))
    ops["mxfp8_quant"].run()
    ops["mxfp8_dequant"].run()
    oq, oe = O.mxfp8_quant(xb)
    assert np.array_equal(u8(t["mq"]), oq) and np.array_equal(u8(t["me"]), oe)
    assert np.array_equal(u16(t["y"]), O.mxfp8_dequant(oq, oe))
    ops["nvfp4_quant"].run()
    ops["nvfp4_dequant"].run()
    x3 = xb.reshape(batch, 256, 512)
    y3 = u16(t["y"]).reshape(batch, 256, 512)
    for b in range(batch):
        A = O.nvfp4_group_amax([x3[b]])
        opk, osb, ogs = O.nvfp4_quant(x3[b], A)
        assert np.array_equal(u8(t["pk"]).reshape(batch, 256, -1)[b], opk), b
        assert np.array_equal(u8(t["sb"]).reshape(batch, 256, -1)[b], osb), b
        assert f32bits(t["gs"])[b] == np.float32(ogs).view(np.uint32), b
        assert np.array_equal(y3[b], O.nvfp4_dequant(opk, osb, ogs, 512)), b
    ops["nvfp4_fake_quant"].run()
    y3 = u16(t["y"]).reshape(batch, 256, 512)
    for b in range(batch):
        assert np.array_equal(y3[b], O.nvfp4_fake_quant(x3[b], O.nvfp4_group_amax([x3[b]]))), b
