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


MAGIC = np.float32(12582912.0)  # 1.5 * 2^23
MID = 0x4B400000


def _code_bits(x, s):
    """The quantiser's integer-free form: the bit pattern of
    u = fl(x * fl(1/s) + 1.5 * 2^23) (a fused multiply-add: the product is
    exact in float64 and so is the sum at these magnitudes up to one final
    rounding to float32, modelled here by rounding the float64 sum; any
    rounding still leaves t = u - 1.5 * 2^23 an integer), kept when the
    residual x r - t lies within 0.5 - 2^-13, else the pattern of
    fl(fl(x / s) + 1.5 * 2^23); its low byte is the code.  No clamp: the test
    checks that none is needed."""
    r = np.float32(1.0) / s if s != 0 else np.float32(0.0)
    prod = x.astype(np.float64) * np.float64(r)          # exact
    u = (prod + np.float64(MAGIC)).astype(np.float32)
    t = (u - MAGIC).astype(np.float32)
    fast = np.abs((prod - t.astype(np.float64)).astype(np.float32)) < MARGIN
    with np.errstate(divide="ignore", invalid="ignore"):
        z = (x / s).astype(np.float32) if s != 0 else np.zeros_like(x)
    slow = (z + MAGIC).astype(np.float32)
    return np.where(fast, u, slow).view(np.int32).astype(np.int64)


@pytest.mark.parametrize("seed", [0, 1])
def test_bit_pattern_code_equals_division_for_every_fp16(seed):
    xs = _all_fp16()
    rng = np.random.default_rng(100 + seed)
    pos = xs[xs > 0]
    amaxes = list(rng.choice(pos, 40, replace=False)) + [
        np.float32(65504.0), np.float32(2.0 ** -24), np.float32(1.0),
        np.float32(127.0), np.float32(0.5), np.float32(3.0)]
    for a in amaxes:
        a = np.float32(a)
        s = np.float32(a / np.float32(127.0))
        x = xs[np.abs(xs) <= a]
        bits = _code_bits(x, s)
        ref = np.clip(np.rint((x / s).astype(np.float32)), -127, 127)
        # the pattern is MID + code, and its low byte is the int8 code
        assert np.array_equal(bits - MID, ref.astype(np.int64)), float(a)
        low = (bits & 0xFF).astype(np.uint8).view(np.int8)
        assert np.array_equal(low.astype(np.int64), ref.astype(np.int64))
    # a zero block: s = 0 and r = 0 give code 0 for every finite x
    assert (_code_bits(xs, np.float32(0.0)) == MID).all()
