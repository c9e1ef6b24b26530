"""The guard-byte checker itself (CPU): writes inside a view pass, a write
into the head, the tail or a row gap is reported."""
import pytest
import torch

import guard


def test_writes_inside_the_view_pass():
    with guard.session() as gs:
        v = guard.empty((3, 5, 40), torch.bfloat16, device="cpu", lead=8, pad=16)
        v.fill_(1.0)
        w = guard.empty((7,), torch.float32, device="cpu")
        w.fill_(2.0)
    assert len(gs) == 2 and v.shape == (3, 5, 40) and v.stride(-2) == 64
    assert v.data_ptr() - gs[0].raw.data_ptr() == guard.HEAD + 16


@pytest.mark.parametrize("where", ["head", "tail", "lead", "pad"])
def test_each_guard_region_catches_a_write(where):
    with pytest.raises(AssertionError) as e:
        with guard.session() as gs:
            v = guard.empty((4, 24), torch.uint8, device="cpu", lead=8, pad=8)
            g = gs[0]
            if where == "head":
                g.raw[guard.HEAD - 1] = 0
            elif where == "tail":
                g.raw[guard.HEAD + g.nbytes + 100] = 0
            elif where == "lead":
                g.raw[guard.HEAD + 40 + 3] = 0           # row 1, inside its lead gap
            else:
                g.raw[guard.HEAD + 2 * 40 + 8 + 24] = 0  # row 2, first pad byte
            v.fill_(3)
    assert {"head": "head", "tail": "tail", "lead": "row lead gap", "pad": "row pad gap"}[where] in str(e.value)


def test_dense_scale_array_overrun_is_caught():
    with pytest.raises(AssertionError):
        with guard.session():
            s = guard.empty((2, 3), torch.float32, device="cpu")
            s.view(-1).fill_(0.5)
            # one float past the end, as a scale write one element too far would land
            torch.as_strided(s.view(-1), (7,), (1,)).fill_(0.5)
