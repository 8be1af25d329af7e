"""The division-free bin quotient against the IEEE divide, in float64 on the CPU (no GPU).

The bin-id kernels take floor(RN(a / delta)), a = RN(pos + u), as floor(RN(a * RN(1/delta)))
whenever that product lies more than 2^-50 of its size away from every integer, and fall back to
the divide otherwise: the product is within 3 * 2^-53 of the quotient's size, so outside that
margin both floors agree. These tests run the same float64 steps in numpy (round to nearest, as
the kernels' explicit __dadd_rn / __dmul_rn / __drcp_rn / __ddiv_rn) on random and on
adversarial near-boundary inputs, and require the result to equal floor(RN(a / delta)).
"""
import numpy as np


def _floor_quotient(a, delta):
    rcp = 1.0 / delta
    xa = a * rcp
    fl = np.floor(xa)
    tol = xa * 2.0 ** -50
    safe = (xa - fl > tol) & ((fl + 1.0) - xa > tol)
    return np.where(safe, fl, np.floor(a / delta)), safe


def test_random_pitches_and_positions():
    r = np.random.default_rng(0)
    m = 2_000_000
    delta = np.exp(r.uniform(np.log(1e-3), np.log(2e4), m))
    u = r.uniform(0.0, 1.0, m) * delta
    pos = r.integers(0, 1 << 20, m).astype(np.float64)
    a = pos + u
    got, safe = _floor_quotient(a, delta)
    assert np.array_equal(got, np.floor(a / delta))
    assert safe.mean() > 0.999          # the divide is the rare path


def test_positions_on_and_next_to_bin_boundaries():
    # a within a few ulps of k * delta, where the product and the quotient are most likely to straddle
    r = np.random.default_rng(1)
    m = 400_000
    delta = np.exp(r.uniform(np.log(0.3), np.log(5e3), m))
    k = r.integers(1, 1 << 16, m).astype(np.float64)
    base = k * delta
    got_all, want_all = [], []
    for steps in (-3, -2, -1, 0, 1, 2, 3):
        a = base.copy()
        for _ in range(abs(steps)):
            a = np.nextafter(a, np.inf if steps > 0 else -np.inf)
        got, _ = _floor_quotient(a, delta)
        got_all.append(got)
        want_all.append(np.floor(a / delta))
    assert np.array_equal(np.concatenate(got_all), np.concatenate(want_all))


def test_integer_pitches_and_shifts():
    # small integer and half-integer pitches make exact quotients common
    for delta in (1.0, 2.0, 3.0, 7.0, 0.5, 1.5, 10.0, 1024.0):
        for u_frac in (0.0, 0.25, 0.5, 0.999):
            pos = np.arange(0, 100_000, dtype=np.float64)
            a = pos + u_frac * delta
            got, _ = _floor_quotient(a, np.full_like(a, delta))
            assert np.array_equal(got, np.floor(a / delta)), (delta, u_frac)
