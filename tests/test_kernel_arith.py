"""Host checks of two arithmetic shortcuts in the kernels.

The quantiser kernel replaces the per-element IEEE division x / s by a
multiply with fl(1/s) wherever the product lies at least 2^-13 away from a
half-integer, and divides otherwise.  This checks, in IEEE float32 on the
host, that the shortcut always yields the code rint(fl(x / s)) that the
definition (and the oracle) use: every fp16 value x against many block
maxima, including subnormal and extreme ones.
"""
import numpy as np
import pytest

MARGIN = np.float32(0.5) - np.float32(2.0 ** -13)


def _all_fp16():
    x = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16).view(np.float16)
    return x[np.isfinite(x)].astype(np.float32)


def _shortcut(x, s):
    r = np.float32(1.0) / s
    y = (x * r).astype(np.float32)
    t = np.rint(y)
    fast = np.abs(y - t) < MARGIN
    exact = np.rint((x / s).astype(np.float32))
    q = np.where(fast, t, exact)
    return np.clip(q, -127, 127), fast


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_shortcut_equals_division_for_every_fp16(seed):
    xs = _all_fp16()
    rng = np.random.default_rng(seed)
    pos = xs[xs > 0]
    amaxes = list(rng.choice(pos, 60, replace=False)) + [
        np.float32(65504.0), np.float32(2.0 ** -24), np.float32(1.0),
        np.float32(127.0), np.float32(254.0), np.float32(0.5),
        np.float32(6.103515625e-05), np.float32(3.0)]
    slow_share = []
    for a in amaxes:
        a = np.float32(a)
        s = np.float32(a / np.float32(127.0))
        x = xs[np.abs(xs) <= a]
        q, fast = _shortcut(x, s)
        ref = np.clip(np.rint((x / s).astype(np.float32)), -127, 127)
        assert np.array_equal(q, ref), float(a)
        slow_share.append(1.0 - fast.mean())
    # the division path stays rare
    assert max(slow_share) < 0.01


# ---------------------------------------------------------------------------
# exp2 on the FMA pipe (the attention kernel's exp2_poly2), restated in IEEE
# float32: j = nearest integer by the 1.5 * 2^23 bias, a Remez cubic for
# 2^f on [-1/2, 1/2], 2^j added to the exponent bits.
# ---------------------------------------------------------------------------

def _exp2_poly(x):
    x = np.maximum(np.asarray(x, np.float32), np.float32(-125.0))
    bias = np.float32(12582912.0)
    t = (x + bias).astype(np.float32)
    j = (t - bias).astype(np.float32)
    f = (x - j).astype(np.float32)
    c = [np.float32(v) for v in (0.99992806, 0.69326097, 0.24261113,
                                 0.055171669)]
    q = ((c[3] * f + c[2]) * f + c[1]) * f + c[0]
    bits = q.astype(np.float32).view(np.uint32) + (t.view(np.uint32) << 23)
    return bits.astype(np.uint32).view(np.float32)


def test_exp2_poly_error_bound():
    x = np.linspace(-124.0, 9.0, 2_000_001, dtype=np.float32)
    got = _exp2_poly(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    assert np.abs(got / ref - 1.0).max() < 8e-5
    # very negative and masked (-inf) inputs give a positive normal number
    # far below fp16's smallest subnormal
    tiny = _exp2_poly(np.array([-200.0, -np.inf, -125.0], np.float32))
    assert (tiny > 0).all() and (tiny < 2.0 ** -120).all()
    assert (tiny.astype(np.float16) == 0).all()
