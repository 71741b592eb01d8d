"""Host check of the quantizer's division-free rounding (csrc/quantize.cu,
rint_quotient): with inv within 1 ulp of 1 / sc and r = fl(v * inv), the code
clamp(rint(r) + z) equals clamp(rint(fl(v / sc)) + z), the
code the quantization step defines (rounded IEEE fp32 quotient, then rint);
the exact quotient is used when r lies within 2^-15 of a half-integer (whatever
|r| is, so the fast value is kept for |r| >= 64 only when it is not near one).

numpy float32 arithmetic is IEEE round-to-nearest, so fl(v / sc) and fl(v * inv)
below are the exact fp32 operations the kernel performs.  The reciprocal is
taken as the correctly rounded value and both of its neighbours, the worst
cases a 1-ulp approximation can return."""
import numpy as np
import pytest

MARGIN = np.float32(2.0 ** -15)


def fast_rint(v, sc, inv):
    r = (v * inv).astype(np.float32)
    t = np.rint(r).astype(np.float32)
    d = np.abs((r - t).astype(np.float32))
    near = d >= (np.float32(0.5) - MARGIN)
    exact = np.rint((v / sc).astype(np.float32)).astype(np.float32)
    return np.where(near, exact, t), near


def code(t, z):
    return np.clip((t + z).astype(np.float32), 0, 15)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_fast_rounding_matches_ieee_quotient(seed):
    rng = np.random.default_rng(seed)
    n = 400_000
    # fp16 scales over their whole range (normal and subnormal), as the quantizer stores them
    sc = rng.uniform(-24, 15.9, n)
    sc = np.exp2(sc).astype(np.float16).astype(np.float32)
    sc[sc == 0] = 1.0
    # quotients spread over [-80, 80] and beyond, plus values within a few ulp of half-integers
    q = rng.uniform(-80, 80, n).astype(np.float32)
    k = rng.integers(-70, 70, n).astype(np.float32) + np.float32(0.5)
    ulps = rng.integers(-40, 41, n).astype(np.float32)
    q_adv = (k + ulps * np.spacing(np.abs(k)).astype(np.float32)).astype(np.float32)
    q = np.where(rng.random(n) < 0.5, q, q_adv)
    v = (q * sc).astype(np.float32)
    v[: n // 50] = (rng.standard_normal(n // 50) * 1e4).astype(np.float32)  # far outside the code range
    exact = np.rint((v / sc).astype(np.float32)).astype(np.float32)
    inv0 = (np.float32(1.0) / sc).astype(np.float32)
    z = rng.integers(0, 16, n).astype(np.float32)
    slow_total = 0
    for inv in (inv0, np.nextafter(inv0, np.float32(np.inf)), np.nextafter(inv0, np.float32(0))):
        t, near = fast_rint(v, sc, inv.astype(np.float32))
        slow_total += int(near.sum())
        np.testing.assert_array_equal(code(t, z), code(exact, z))
        # the symmetric variant clamps rint(q) to [-7, 7]
        np.testing.assert_array_equal(np.clip(t, -7, 7), np.clip(exact, -7, 7))
    # the adversarial half are the only ones that should need the exact quotient
    assert slow_total < 3 * n // 2


@pytest.mark.parametrize("den", [7, 15])
def test_scale_division_by_double_product_is_exact(den):
    """The scale fl32(d / 7) or fl32(d / 15) is formed as RN32(RN64(d * RN64(1 / c)))
    (csrc/quantize.cu, div_by_const).  Every fp32 d of three slices checked here:
    the subnormal binades, [1, 2) and the top binade; the full ranges of the
    subnormal/low, [1, 4) and top binades were checked the same way offline."""
    c = np.float64(1.0) / np.float64(den)
    f2b = lambda x: int(np.float32(x).view(np.uint32))
    for lo, hi in ((1, f2b(2.0 ** -126)), (f2b(1.0), f2b(2.0)), (f2b(2.0 ** 127), f2b(np.finfo(np.float32).max) + 1)):
        b = np.arange(lo, hi, dtype=np.uint32)
        d = b.view(np.float32)
        ref = d / np.float32(den)
        fast = (d.astype(np.float64) * c).astype(np.float32)
        np.testing.assert_array_equal(fast.view(np.uint32), ref.view(np.uint32))
