"""Pins for the oracle's W4A4 activation observers (CPU).

The observer readings (verl NVFP4 QAT article 2.2 / 3.1 name static_minmax,
memoryless_minmax and minmax) are checked against facts computed another
way: the extremes against numpy's min / max of the decoded values, the
static observer against the extremes of the concatenated history, the
moving average against its closed forms at c = 1, c = 0 and, with values
for which every step is exact, c = 1/2, and at general constants (0.01,
0.3) on random extremes against an exact-rational restatement of the update
with one binary32 rounding per operation in the stated order; the global
scale against the weight path's fl(A / 2688).
"""
import numpy as np
import pytest

import exact as X
from oracle import oracle as O
import workloads as W

EMPTY = np.array([np.inf, -np.inf], np.float32)


def vals(bits):
    return O.bf16_to_f32(np.asarray(bits, np.uint16)).astype(np.float64)


def acts(n, seed, shape=(64, 256)):
    return [W.bits(W.random_bf16(shape, seed=seed + i, std=1.0 + i)) for i in range(n)]


def test_extremes_are_min_and_max_of_the_values():
    for x in acts(3, 10):
        lo, hi = O.activation_minmax(x)
        v = vals(x)
        assert lo == v.min() and hi == v.max()
    # signed zeros: -0 orders below +0
    lo, hi = O.activation_minmax(np.array([0x0000, 0x8000], np.uint16))
    assert lo == 0 and np.signbit(lo) and hi == 0 and not np.signbit(hi)
    lo, hi = O.activation_minmax(np.array([0x8000, 0x8000], np.uint16))
    assert np.signbit(lo) and np.signbit(hi)


def test_memoryless_forgets_and_static_keeps_the_extremes():
    xs = acts(4, 20)
    st_m, st_s = EMPTY.copy(), EMPTY.copy()
    seen = []
    for x in xs:
        st_m, A_m, g_m = O.observe(st_m, x, O.MEMORYLESS_MINMAX)
        st_s, A_s, g_s = O.observe(st_s, x, O.STATIC_MINMAX)
        seen.append(vals(x))
        v = vals(x)
        assert st_m[0] == v.min() and st_m[1] == v.max()
        allv = np.concatenate([s.ravel() for s in seen])
        assert st_s[0] == allv.min() and st_s[1] == allv.max()
        assert A_s == np.abs(allv).max() and A_m == np.abs(v).max()
        assert g_s == np.float32(O.nvfp4_global_scale(A_s))
        assert g_m == np.float32(np.float32(A_m) / np.float32(2688))


def test_moving_average_closed_forms():
    xs = acts(3, 30)
    # c = 1: the last tensor's extremes; c = 0: the first tensor's
    st1, st0 = EMPTY.copy(), EMPTY.copy()
    for x in xs:
        st1, _, _ = O.observe(st1, x, O.MINMAX, c=1.0)
        st0, _, _ = O.observe(st0, x, O.MINMAX, c=0.0)
    assert np.array_equal(st1, np.array(O.activation_minmax(xs[-1]), np.float32))
    assert np.array_equal(st0, np.array(O.activation_minmax(xs[0]), np.float32))
    # c = 1/2 with power-of-two extremes: every step exact, lo_k = (lo_{k-1} + m_k) / 2
    ext = [(-8.0, 4.0), (-2.0, 16.0), (-0.5, 1.0)]
    st = EMPTY.copy()
    ref = None
    for lo, hi in ext:
        x = O.bf16_round(np.array([lo, 0.25, hi], np.float32))
        st, A, g = O.observe(st, x, O.MINMAX, c=0.5)
        ref = (lo, hi) if ref is None else ((ref[0] + lo) / 2, (ref[1] + hi) / 2)
        assert st[0] == ref[0] and st[1] == ref[1]
        assert A == max(abs(ref[0]), abs(ref[1]))


def test_observed_amax_drives_the_fake_quant():
    # with the memoryless observer the W4A4 fake quant equals the plain one
    x = acts(1, 40)[0]
    _, A, _ = O.observe(EMPTY, x, O.MEMORYLESS_MINMAX)
    assert A == np.float32(O.nvfp4_group_amax([x]))
    assert np.array_equal(O.nvfp4_fake_quant(x, A), O.nvfp4_fake_quant(x, O.nvfp4_group_amax([x])))


def ema_step_exact(lo, m, c):
    """The moving-average update as the reading states it, in exact
    rationals with one RN-to-binary32 per operation, in this order:
    w = fl(1 - c), lo' = fl(fl(w * lo) + fl(c * m))."""
    cx = X.f32_value_to_exact(c)
    w = X.f32(X.add((False, X.Fraction(1)), X.neg(cx)))
    a = X.f32(X.mul(w, X.f32_value_to_exact(lo)))
    b = X.f32(X.mul(cx, X.f32_value_to_exact(m)))
    return np.uint32(X.exact_to_f32_bits(X.f32(X.add(a, b))))


def ema_variants(lo, m, c):
    """Plausible departures from the stated order, each one rounding fewer
    times or in another order (for the check that the pin tells them apart)."""
    c32, lo32, m32 = np.float32(c), np.float32(lo), np.float32(m)
    w = np.float32(np.float32(1) - c32)
    cx, wx = X.f32_value_to_exact(c32), X.f32_value_to_exact(w)
    # fused multiply-add: fl(w * lo + fl(c * m)), one rounding for the product and the sum
    fma = X.f32(X.add(X.mul(wx, X.f32_value_to_exact(lo32)), X.f32(X.mul(cx, X.f32_value_to_exact(m32)))))
    return {
        "fma": np.uint32(X.exact_to_f32_bits(fma)),
        "lo + c (m - lo)": np.float32(lo32 + np.float32(c32 * np.float32(m32 - lo32))).view(np.uint32),
        "binary64": np.float32((1.0 - float(c32)) * float(lo32) + float(c32) * float(m32)).view(np.uint32),
    }


@pytest.mark.parametrize("c", [0.01, 0.3])
def test_moving_average_general_constant_exact(c):
    """Random activations of varying spread: every step's state equals the
    exact-rational restatement bit for bit, and each plausible departure from
    the stated rounding order gives another state somewhere in the sequence."""
    rng = np.random.default_rng(int(c * 1000))
    st = EMPTY.copy()
    differs = {}
    steps = 0
    for k in range(40):
        std = float(np.exp(rng.uniform(-3, 3)))
        x = W.bits(W.random_bf16((8, 64), seed=5000 + k + int(c * 100), std=std))
        mn, mx = O.activation_minmax(x)
        prev = st.copy()
        st, A, g = O.observe(st, x, O.MINMAX, c=np.float32(c))
        if k == 0:
            assert st[0] == mn and st[1] == mx       # an empty state takes the extremes
            continue
        for j, m in ((0, mn), (1, mx)):
            want = ema_step_exact(prev[j], m, np.float32(c))
            assert st.view(np.uint32)[j] == want, (k, j)
            for name, v in ema_variants(prev[j], m, np.float32(c)).items():
                differs[name] = differs.get(name, False) or v != want
            steps += 1
        assert A == np.float32(max(abs(st[0]), abs(st[1])))
        assert g.view(np.uint32) == X.exact_to_f32_bits(X.f32(X.div(X.f32_value_to_exact(A),
                                                                      (False, X.Fraction(2688)))))
    assert steps == 78
    assert all(differs.values()), differs
