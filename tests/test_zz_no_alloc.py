"""GPU test of nvfp4_fake_quant_noalloc, the entry point for callers that
cannot allocate device memory (for example code inside a framework or plugin
host that owns all device memory, or a step where cudaMalloc's implicit
synchronisation is not acceptable).  It must give exactly what the
workspace-taking nvfp4_fake_quant gives.

Two calls in a row: the second group's amax is far smaller than the first's,
so a scratch array that still held the first call's maxima would change the
second call's output.  The file is named so that pytest collects it last.
"""
import ctypes

import numpy as np
import pytest
import torch

import guard
from oracle import oracle as O
import workloads as W

pytestmark = pytest.mark.gpu


# (rows of the two siblings): small groups run one cluster each and leave the
# static scratch alone; larger ones (more than 131072 elements) use it
SHAPES = {"cluster": (64, 32), "scratch": (300, 100)}


@pytest.mark.parametrize("path", list(SHAPES))
def test_noalloc_entry_point_matches_workspace_entry_point_twice(path):
    import precision_weight_quantization_b200 as P
    from precision_weight_quantization_b200._lib import PwqTensor, lib

    f = lib.nvfp4_fake_quant_noalloc
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.POINTER(PwqTensor), ctypes.POINTER(PwqTensor), ctypes.c_int,
                  ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
    dev = torch.device("cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)
    for call, (seed, std) in enumerate(((11, 40.0), (12, 0.003))):
        # a batched sibling pair: 3 groups, each {x0[b], x1[b]}
        m0, m1 = SHAPES[path]
        xs = [W.random_bf16((3, m0, 512), seed=seed, std=std, device=dev),
              W.random_bf16((3, m1, 512), seed=seed + 100, std=std, device=dev)]
        ys = [guard.empty(x.shape, torch.bfloat16) for x in xs]
        amax_out = guard.empty((3,), torch.float32)
        ax = (PwqTensor * 2)(*[P._desc(x, "x") for x in xs])
        ay = (PwqTensor * 2)(*[P._desc(y, "y") for y in ys])
        st = f(ax, ay, 2, None, amax_out.data_ptr(), stream)
        assert st == 0, (call, P.status_string(st), lib.pwq_last_error_detail().decode())

        ref_amax = torch.empty(3, dtype=torch.float32, device=dev)
        ref = P.nvfp4_fake_quant(xs, amax_out=ref_amax)
        torch.cuda.synchronize()
        # tolerance 0: bit-identical BF16 outputs and amax
        for y, r in zip(ys, ref):
            assert torch.equal(y.view(torch.int16), r.view(torch.int16)), call
        assert torch.equal(amax_out, ref_amax), call
        expect = torch.stack([torch.maximum(xs[0][b].float().abs().max(), xs[1][b].float().abs().max())
                              for b in range(3)])
        assert torch.equal(amax_out, expect), call
        # and the oracle, group by group
        for b in range(3):
            bits = [W.bits(x[b]) for x in xs]
            A = O.nvfp4_group_amax(bits)
            for x_b, y in zip(bits, ys):
                assert np.array_equal(W.bits(y[b]), O.nvfp4_fake_quant(x_b, A)), (call, b)


def test_noalloc_with_amax_in_beyond_the_scratch_limit():
    """With amax_in the static scratch is unused, so more than 4096 groups
    are accepted; the result equals nvfp4_fake_quant's with the same amax."""
    import precision_weight_quantization_b200 as P
    from precision_weight_quantization_b200._lib import PwqTensor, lib

    dev = torch.device("cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)
    B = 4097
    x = W.random_bf16((B, 4, 32), seed=21, std=1.0, device=dev)
    amax = x.float().abs().amax(dim=(1, 2)).contiguous()
    amax[::7] *= 2.0                      # cached / all-reduced amax may exceed the slab's own
    y = guard.empty(x.shape, torch.bfloat16)
    ax, ay = P._desc(x, "x"), P._desc(y, "y")
    st = lib.nvfp4_fake_quant_noalloc(ctypes.byref(ax), ctypes.byref(ay), 1, amax.data_ptr(), None, stream)
    assert st == 0, (P.status_string(st), lib.pwq_last_error_detail().decode())
    ref = P.nvfp4_fake_quant(x, amax=amax)
    torch.cuda.synchronize()
    assert torch.equal(y.view(torch.int16), ref.view(torch.int16))
    xb, yb, ab = W.bits(x), W.bits(y), amax.cpu().numpy()
    for b in (0, 7, 2048, B - 1):
        assert np.array_equal(yb[b], O.nvfp4_fake_quant(xb[b], ab[b])), b
