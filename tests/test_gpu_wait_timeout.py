"""The bounded wait of the NVFP4 single-pass kernel gives up, reports, and
leaves the device usable (GPU).

pwq_selftest_flow_timeout runs the single-pass fake-quantisation with the
wait of every encode item (for its group's amax) pointed at a completion
count that nothing adds to, and with a 1 ms limit: every such wait runs out.
Nothing faults or hangs -- the kernel returns, the error word records bit
1, reading it clears it, and the next ordinary call is exact.
"""
import ctypes
import time

import numpy as np
import pytest
import torch

import guard
from oracle import oracle as O
import workloads as W

pytestmark = pytest.mark.gpu

DEV = "cuda"
FLOW_TIMEOUT_BIT = 2


@pytest.fixture(scope="module")
def P():
    import precision_weight_quantization_b200 as P
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return P


@pytest.mark.parametrize("shape", [(3, 64, 512), (1, 512, 4096)], ids=str)
def test_flow_wait_runs_out_reports_and_recovers(P, shape):
    from precision_weight_quantization_b200._lib import lib
    torch.cuda.synchronize()
    assert P.device_error() == 0
    x = W.random_bf16(shape, seed=77, std=0.5, device=DEV)
    y = guard.empty(shape, torch.bfloat16)
    dx, dy = P._desc(x, "x"), P._desc(y, "y")
    n = lib.pwq_selftest_flow_timeout_workspace_size(ctypes.byref(dx))
    assert n > 0
    ws = guard.empty((n,), torch.uint8)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    t0 = time.perf_counter()
    st = lib.pwq_selftest_flow_timeout(ctypes.byref(dx), ctypes.byref(dy), 1_000_000, ws.data_ptr(), n, stream)
    assert st == 0, (P.status_string(st), lib.pwq_last_error_detail().decode())
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    assert elapsed < 1.0, elapsed          # about 1 ms per waiting CTA, far below the normal 2 s limit
    code = P.device_error()
    assert code & FLOW_TIMEOUT_BIT, code
    assert P.device_error() == 0            # read and cleared
    # the next ordinary call runs clean and exact
    fq = P.nvfp4_fake_quant(x)
    torch.cuda.synchronize()
    assert P.device_error() == 0
    xb = W.bits(x).reshape((-1,) + shape[-2:])
    fb = W.bits(fq).reshape((-1,) + shape[-2:])
    for b in range(xb.shape[0]):
        assert np.array_equal(fb[b], O.nvfp4_fake_quant(xb[b], O.nvfp4_group_amax([xb[b]]))), b
