"""The column loops round with the 1.5 * 2^23 shift instead of rint (two fp32 adds).

The claim the kernels rely on, checked in IEEE float32 arithmetic (numpy): for |x| < 2^22 the
shifted sum rounds to the same integer as rint, ties to even; for larger magnitudes the result keeps
its sign and a magnitude of at least 2^22 - 1, so clamping to any b-bit grid gives the same code.
"""
import numpy as np

SHIFT = np.float32(12582912.0)  # 1.5 * 2^23


def shifted(x):
    x = np.asarray(x, dtype=np.float32)
    return (x + SHIFT) - SHIFT  # each operation rounds to float32


def test_equals_rint_on_ties_and_random_values():
    ties = np.arange(-4096, 4096, dtype=np.float32) + np.float32(0.5)
    np.testing.assert_array_equal(shifted(ties), np.rint(ties))
    rng = np.random.default_rng(0)
    x = (rng.standard_normal(200_000) * rng.choice([1, 16, 4096, 2 ** 21], 200_000)).astype(np.float32)
    x = x[np.abs(x) < 2 ** 22]
    np.testing.assert_array_equal(shifted(x), np.rint(x))
    near = np.nextafter(np.float32(2 ** 22), np.float32(0)) - np.arange(64, dtype=np.float32)
    np.testing.assert_array_equal(shifted(near), np.rint(near))
    np.testing.assert_array_equal(shifted(-near), np.rint(-near))


def test_large_magnitudes_clamp_to_the_same_code():
    rng = np.random.default_rng(1)
    big = (np.float32(2 ** 22) * (1 + rng.random(10_000) * 1e6)).astype(np.float32)
    for sign in (1, -1):
        x = np.float32(sign) * big
        got = shifted(x)
        assert np.all(np.sign(got) == sign)
        assert np.all(np.abs(got) >= 2 ** 22 - 1)
        for maxq, zero in ((3, 1), (7, 4), (15, 8), (15, 0)):
            lo, hi = np.float32(-zero), np.float32(maxq - zero)
            np.testing.assert_array_equal(np.clip(got, lo, hi), np.clip(np.rint(x), lo, hi))
