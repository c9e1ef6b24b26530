"""GPU parity of the W4A4 activation observers and of the W4A4 activation
fake-quant they drive, against the oracle, bit for bit, over sequences of
activations (ragged, batched, strided, with signed zeros and outliers)."""
import numpy as np
import pytest
import torch

from oracle import oracle as O
import workloads as W

from test_gpu_parity import DEV, f32bits, gpu, rand_bits, strided

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def P():
    import precision_weight_quantization_b200 as P
    assert torch.cuda.is_available()
    return P


SEQ = [((64, 256), 0), ((3, 40, 160), 0), ((130, 512), 32), ((1, 16), 0)]


@pytest.mark.parametrize("kind,c", [("memoryless_minmax", 0.01), ("static_minmax", 0.01), ("minmax", 0.01),
                                    ("minmax", 0.5), ("minmax", 1.0)])
def test_observer_sequence_matches_oracle(P, kind, c):
    obs = P.NVFP4ActivationObserver(kind, averaging_constant=c, device=DEV)
    state = np.array([np.inf, -np.inf], np.float32)
    for i, (shape, pad) in enumerate(SEQ):
        xb = rand_bits(shape, seed=800 + i, std=0.5 * (i + 1))
        xg = strided(xb, pad) if pad else gpu(xb)
        y = obs.fake_quant(xg)
        state, A, g = O.observe(state, xb, O.OBSERVERS_BY_NAME[kind], np.float32(c))
        assert np.array_equal(f32bits(obs.state), state.view(np.uint32)), (kind, i)
        assert f32bits(obs.amax)[0] == np.float32(A).view(np.uint32), (kind, i)
        assert f32bits(obs.input_global_scale)[0] == np.float32(g).view(np.uint32), (kind, i)
        assert np.array_equal(W.bits(y), O.nvfp4_fake_quant(xb, A)), (kind, i)


def test_observer_signed_zero_extremes(P):
    obs = P.NVFP4ActivationObserver("memoryless_minmax", device=DEV)
    xb = np.zeros((4, 16), np.uint16)
    xb[1, 3] = 0x8000
    obs.observe(gpu(xb))
    st = obs.state.cpu().numpy()
    assert st[0] == 0 and np.signbit(st[0]) and st[1] == 0 and not np.signbit(st[1])
    assert obs.amax.item() == 0.0 and obs.input_global_scale.item() == 0.0


def test_w4a4_ste_passes_the_gradient(P):
    obs = P.NVFP4ActivationObserver("static_minmax", device=DEV)
    x = W.random_bf16((32, 64), seed=850, std=1.0, device=DEV).requires_grad_(True)
    y = P.nvfp4_w4a4_fake_quant_ste(x, obs)
    g = W.random_bf16((32, 64), seed=851, std=1e-3, device=DEV)
    y.backward(g)
    assert torch.equal(x.grad.view(torch.int16), g.view(torch.int16))
