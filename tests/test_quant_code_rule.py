"""CPU: the rule the int8 quantisers use to skip the IEEE division.

The kernels code x as clamp(rint(fl(x / s)), -127, 127) with s = fl(max / 127)
(LASER results, W8A8 setting: per-token symmetric quantisation).  They form
t = fl(x * fl(1 / s)) and keep rint(t) whenever t lies farther than 1/8192
from every half-integer; only the remaining near-ties take the quotient.
That is exact if |t - fl(x / s)| stays below 1/8192 for |x| <= 127 s.  numpy's
float32 arithmetic is IEEE (correctly rounded), so the bound and the rule are
checked here by brute force on random and deliberately near-tie inputs,
independently of the GPU.
"""
import numpy as np
import pytest

F = np.float32
THRESH = F(1.0 / 8192.0)


def _scales(rng, n):
    # maxima over many magnitudes, the quantiser's scale s = fl(max / 127)
    amax = (rng.uniform(0.5, 2.0, n) * 10.0 ** rng.uniform(-6, 6, n)).astype(F)
    return amax, (amax / F(127.0)).astype(F)


def _check(x, s):
    inv = (F(1.0) / s).astype(F)
    t = (x * inv).astype(F)
    q = (x / s).astype(F)                      # the IEEE quotient
    err = np.abs(t.astype(np.float64) - q.astype(np.float64))
    assert err.max() < 2.3e-5
    r = np.rint(t)
    decided = (F(0.5) - np.abs(t - r)) > THRESH
    assert np.array_equal(r[decided], np.rint(q)[decided])
    return decided


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_rule_on_random_values(seed):
    rng = np.random.default_rng(seed)
    n = 400_000
    amax, s = _scales(rng, n)
    x = (rng.uniform(-1.0, 1.0, n) * amax).astype(F)
    x[:1000] = amax[:1000]                     # the row maximum itself codes to 127
    x[1000:2000] = -amax[1000:2000]
    decided = _check(x, s)
    assert decided.mean() > 0.999              # the division is the rare case


def test_rule_on_near_ties():
    # values whose quotient is within a few ulp of k + 1/2: the rule must hand
    # these to the division (or decide them the same way)
    rng = np.random.default_rng(7)
    n = 400_000
    amax, s = _scales(rng, n)
    k = rng.integers(-127, 127, n).astype(np.float64)
    target = (k + 0.5) * s.astype(np.float64)
    x = target.astype(F)
    # move each value by -4 .. 4 float32 steps from the rounded tie
    d = rng.integers(-4, 5, n)
    for _ in range(4):
        toward = np.where(d > 0, np.inf, -np.inf).astype(F)
        x = np.where(d != 0, np.nextafter(x, toward), x).astype(F)
        d = d - np.sign(d)
    x = np.clip(x, -amax, amax).astype(F)
    decided = _check(x, s)
    assert (~decided).sum() > 100000           # most of these go to the division


def test_exact_ties_go_to_the_division():
    # s a power of two: x / s is exact, so x = (k + 1/2) s is a tie rounded to even
    s = np.full(255, 0.5, dtype=F)
    x = ((np.arange(-127, 128) + 0.5) * 0.5).astype(F)
    inv = (F(1.0) / s).astype(F)
    t = (x * inv).astype(F)
    r = np.rint(t)
    assert not ((F(0.5) - np.abs(t - r)) > THRESH).any()
    assert np.array_equal(np.rint((x / s).astype(F)), np.rint(np.arange(-127, 128) + 0.5))
