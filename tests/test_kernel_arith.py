"""Host check of an arithmetic shortcut in the quantiser kernel.

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
