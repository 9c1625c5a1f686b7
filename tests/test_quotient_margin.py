"""The residual quantiser's quotient shortcut, checked in float32 IEEE arithmetic on the host.

The GPU coder forms code = clip(rint(fl((x - zero) / scale))) as rint(fl(a * fl(1 / scale))) and
does the division only when that product lies within 2^-12 of a half-integer (|q| <= 512); the
two correctly rounded operations keep it within 1.5 * 2^-23 |q| of the exact quotient, so the
codes must equal those of the plain division. Planted near-ties exercise the fallback.
"""
import numpy as np


def shortcut_codes(a, s, levels):
    f32 = np.float32
    r = (f32(1) / s).astype(np.float32)
    q = (a * r).astype(np.float32)
    c = np.rint(q)
    near = (np.abs(q) <= 512) & (np.abs(q - c) >= f32(0.5) - f32(2.0 ** -12))
    c = np.where(near, np.rint((a / s).astype(np.float32)), c)
    return np.clip(c, 0, f32(levels))


def plain_codes(a, s, levels):
    return np.clip(np.rint((a / s).astype(np.float32)), 0, np.float32(levels))


def test_quotient_shortcut_matches_division():
    rng = np.random.default_rng(11)
    n = 400_000
    for levels in (3, 15, 255):
        s = rng.uniform(1e-4, 4.0, n).astype(np.float16).astype(np.float32)
        s = s[s > 0]
        m = s.size
        # ordinary values over the code range
        a = (rng.uniform(-0.2, levels + 0.7, m).astype(np.float32) * s).astype(np.float32)
        assert np.array_equal(shortcut_codes(a, s, levels), plain_codes(a, s, levels))
        # values one ulp either side of (k + 1/2) * scale
        k = rng.integers(-2, levels + 2, m).astype(np.float32)
        t = ((k + np.float32(0.5)) * s).astype(np.float32)
        for d in (-1, 1):
            a = np.nextafter(t, (t + np.float32(d)).astype(np.float32))
            assert np.array_equal(shortcut_codes(a, s, levels), plain_codes(a, s, levels))
