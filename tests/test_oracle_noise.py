"""Pins for the oracle's counter-based Gumbel noise and the Gumbel-argmax draw.

The draw replaces softmax + multinomial; the diffusers issue "MiniMax Music 3
modular pipeline: 2.9x consumer-GPU speedup" (finding 3) states the two give
the same distribution and reports a unit test at L1 ~= 0.015 over 200k draws.
"""
import math
import os

import numpy as np
import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
GOLDEN = 0x9E3779B97F4A7C15


def _golden_splitmix():
    vals = []
    with open(os.path.join(HERE, "golden", "splitmix64.txt")) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                vals.append(int(line, 16))
    return vals


def test_splitmix64_published_stream(ora):
    L = ora.lib()
    want = _golden_splitmix()
    got = [L.ora_mix64((k * GOLDEN) % (1 << 64)) for k in range(len(want))]
    assert got == want


def test_uniform_open_interval_ends(ora):
    L = ora.lib()
    assert L.ora_uniform(0) == 2.0 ** -25
    assert L.ora_uniform((1 << 64) - 1) == 1.0 - 2.0 ** -25
    # every value is an odd multiple of 2^-25
    for b in [1 << 40, 12345 << 40, (1 << 63)]:
        u = L.ora_uniform(b)
        k = u * 2 ** 25
        assert k == int(k) and int(k) % 2 == 1


def _ulp(x):
    return math.ulp(x)


def test_ln_against_libm(ora):
    L = ora.lib()
    rng = np.random.default_rng(0)
    xs = np.concatenate([
        rng.uniform(2.0 ** -26, 1.0, 4000),
        np.exp(rng.uniform(-700, 700, 4000)),
        rng.uniform(0.7, 1.42, 4000),
        [1.0, 2.0, 0.5, 1.4142135623730951, 1.4142135623730950, 0.7071067811865476],
    ])
    worst = 0.0
    for x in xs:
        got = L.ora_ln(float(x))
        ref = math.log(float(x))
        err = abs(got - ref) / max(_ulp(ref), 5e-324)
        worst = max(worst, err)
    assert worst <= 2.0, worst


def test_ln_powers_of_two(ora):
    L = ora.lib()
    for e in range(-1000, 1000, 7):
        x = math.ldexp(1.0, e)
        assert abs(L.ora_ln(x) - math.log(x)) <= _ulp(math.log(x)) if e != 0 else L.ora_ln(x) == 0.0


def test_gumbel_marginal_is_standard_gumbel(ora):
    # Kolmogorov-Smirnov distance of 100k noise values against the CDF exp(-exp(-g)).
    L = ora.lib()
    n = 100_000
    g = np.sort(np.array([L.ora_gumbel(7, 3, 1, i) for i in range(n)], np.float64))
    cdf = np.exp(-np.exp(-g))
    emp_hi = np.arange(1, n + 1) / n
    emp_lo = np.arange(0, n) / n
    d = max(np.max(emp_hi - cdf), np.max(cdf - emp_lo))
    assert d < 1.63 / math.sqrt(n)  # 1% critical value
    # mean = Euler-Mascheroni constant, variance = pi^2 / 6
    assert abs(g.mean() - 0.5772156649) < 4 * math.sqrt(math.pi ** 2 / 6 / n)


def test_noise_depends_on_every_key(ora):
    L = ora.lib()
    base = L.ora_noise_bits(1, 2, 3, 4)
    assert len({base, L.ora_noise_bits(0, 2, 3, 4), L.ora_noise_bits(1, 0, 3, 4),
                L.ora_noise_bits(1, 2, 0, 4), L.ora_noise_bits(1, 2, 3, 0)}) == 5


@pytest.mark.parametrize("logits,T", [
    ([0.3, -1.0, 2.0, 0.0, 1.5, -0.5, 0.7, 1.1], 1.0),
    ([2.0, 1.0, 0.0, -1.0, -2.0, 3.0, 0.5, 0.25, -0.25, 1.75, 0.0, 0.1, -3.0, 2.5, 1.25, 0.6], 1.0),
    ([0.3, -1.0, 2.0, 0.0, 1.5, -0.5, 0.7, 1.1], 0.7),
])
def test_gumbel_argmax_matches_softmax(ora, logits, T):
    # The pages' test: L1 between the empirical draw frequencies and the
    # categorical softmax distribution, <= 0.015 over 200k draws (vocab <= 16).
    n = 200_000
    lg = np.array(logits, np.float32)
    draws = ora.gumbel_argmax_draws(lg, T, seed=11, frame0=0, ndraws=n)
    freq = np.bincount(draws, minlength=lg.size) / n
    z = lg.astype(np.float64) / T
    p = np.exp(z - z.max())
    p /= p.sum()
    l1 = np.abs(freq - p).sum()
    assert l1 <= 0.015, l1


def test_gumbel_argmax_degenerate(ora):
    lg = np.array([-np.inf, 5.0, -np.inf, -np.inf], np.float32)
    draws = ora.gumbel_argmax_draws(lg, 1.0, seed=3, frame0=0, ndraws=2000)
    assert (draws == 1).all()
    # a gap far larger than any Gumbel value (|G| < 40 for 24-bit uniforms) is deterministic
    lg = np.array([0.0, 100.0, 0.0], np.float32)
    assert (ora.gumbel_argmax_draws(lg, 1.0, seed=3, frame0=0, ndraws=2000) == 1).all()


def test_gumbel_range_bound(ora):
    # u in [2^-25, 1-2^-25] bounds G to [-ln(-ln 2^-25), -ln(-ln(1-2^-25))]
    lo = -math.log(-math.log(2.0 ** -25))
    hi = -math.log(-math.log1p(-2.0 ** -25))
    L = ora.lib()
    for i in range(20000):
        g = L.ora_gumbel(5, 5, 5, i)
        assert lo - 1e-5 <= g <= hi + 1e-5


def test_gumbel_fill_is_the_generator(ora):
    """The bulk fill returns the generator's values, including the depth
    decoder's indices (j << 32) | i and the end token's vocab row."""
    for seed, frame, row, base in [(0, 0, 0, 0), (7, 123, 3, 151675), (1, 2, 1, 5 << 32),
                                   (9, 9, 0, 151670)]:
        got = ora.gumbel_fill(seed, frame, row, base, 64)
        ref = np.array([ora.gumbel(seed, frame, row, base + i) for i in range(64)], np.float32)
        assert np.array_equal(got.view(np.uint32), ref.view(np.uint32))
