"""The quantize kernels code a value with one fp32 multiply by fl(1/scale) and fall back
to the division only when the product lies within 2^-12 of a half-integer.  This pins the
error argument behind that rule in IEEE float32 (numpy rounds every operation to nearest,
as the device's _rn operations do): outside the band, the multiply's nearest integer equals
that of the rounded quotient fl(fl(x - min) / scale), for groups of every scale range.
The device path itself is compared bit for bit with the oracle by the GPU tests."""
import numpy as np
import pytest

BAND = np.float32(2.0 ** -12)


def _groups(rng, n, bits):
    qmax = np.float32(2 ** bits - 1)
    span = np.float32(10.0) ** rng.uniform(-30, 4, n).astype(np.float32)
    lo = rng.standard_normal(n).astype(np.float32) * span
    x = lo[:, None] + rng.uniform(0, 1, (n, 32)).astype(np.float32) * span[:, None]
    x = x.astype(np.float32)
    mn, mx = x.min(axis=1), x.max(axis=1)
    scale = ((mx - mn) / qmax).astype(np.float32)
    keep = scale > 0
    return x[keep], mn[keep], scale[keep], qmax


@pytest.mark.parametrize("bits", [2, 4])
def test_multiply_agrees_with_rounded_quotient_outside_the_band(bits):
    rng = np.random.default_rng(bits)
    with np.errstate(over="ignore", invalid="ignore", divide="ignore"):
        x, mn, scale, qmax = _groups(rng, 20000, bits)
        d = (x - mn[:, None]).astype(np.float32)
        q_div = (d / scale[:, None]).astype(np.float32)
        inv = (np.float32(1) / scale).astype(np.float32)
        usable = inv >= np.float32(2.0 ** -126)
        t = (d * inv[:, None]).astype(np.float32)
        frac = t - np.floor(t)
        fast = (np.abs(frac - np.float32(0.5)) > BAND) & usable[:, None]
    c_div = np.clip(np.rint(q_div), 0, qmax)
    c_mul = np.clip(np.rint(t), 0, qmax)
    assert fast.mean() > 0.99  # the division is the rare case
    np.testing.assert_array_equal(c_mul[fast], c_div[fast])


def test_ties_and_near_ties_fall_in_the_band():
    """Exact half-integer quotients (0.5 -> 0, 1.5 -> 2 under half-to-even) and their
    float32 neighbours take the division."""
    scale = np.float32(1.0)
    for h in (0.5, 1.5, 2.5):
        for d in (np.float32(h), np.nextafter(np.float32(h), np.float32(0)),
                  np.nextafter(np.float32(h), np.float32(4))):
            t = np.float32(d * np.float32(1) / scale)
            assert not abs(t - np.floor(t) - np.float32(0.5)) > BAND
