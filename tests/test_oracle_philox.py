"""Pins for the oracle's random numbers (Philox4x64-10 and Box-Muller).

The generator is pinned against numpy's Philox bit generator, a separate
implementation of the same published definition (Salmon et al., SC'11);
numpy advances its counter by one before each block, so its output for
counter c is ours for counter c + 1.
"""
import math

import numpy as np
import pytest
from scipy import stats

from oracle import philox


@pytest.mark.parametrize("key", [(0, 0), (1, 0), (5, 7), (2**64 - 1, 2**63 + 11)])
@pytest.mark.parametrize("ctr", [(0, 0, 0, 0), (41, 0, 3, 0), (2**40 + 5, 9, 2**63, 17)])
def test_philox_matches_numpy_bit_generator(key, ctr):
    bg = np.random.Philox(counter=list(ctr), key=list(key))
    want = bg.random_raw(4)
    c0 = (ctr[0] + 1) % 2**64
    got = philox.philox4x64_10(np.uint64(c0), np.uint64(ctr[1]), np.uint64(ctr[2]),
                               np.uint64(ctr[3]), np.uint64(key[0]), np.uint64(key[1]))
    assert [int(x) for x in got] == [int(x) for x in want]


def test_philox_vectorised_equals_scalar():
    j = np.arange(37, dtype=np.uint64)
    zero = np.zeros_like(j)
    vec = philox.philox4x64_10(j, zero + 1, zero, zero, np.uint64(99), np.uint64(0))
    for i in (0, 5, 36):
        one = philox.philox4x64_10(np.uint64(i), np.uint64(1), np.uint64(0), np.uint64(0),
                                   np.uint64(99), np.uint64(0))
        assert [int(v[i]) for v in vec] == [int(x) for x in one]


def test_uniform52_open_interval():
    u = philox.uniform52(np.array([0, 2**64 - 1], dtype=np.uint64))
    assert u[0] == 2.0 ** -53
    assert u[1] == 1.0 - 2.0 ** -53
    assert 0.0 < u[0] < u[1] < 1.0


def test_box_muller_closed_form():
    # u0 = 1/2, u1 = 1/4: radius sqrt(2 ln 2), angle pi/2.
    z0, z1 = philox.box_muller(np.array([0.5]), np.array([0.25]))
    assert abs(z0[0]) < 1e-15
    assert z1[0] == pytest.approx(math.sqrt(2.0 * math.log(2.0)), rel=1e-15)


def test_normals_are_standard_normal():
    z = philox.normals(seed=123, tag=0, count=200_000)
    n = z.size
    assert abs(z.mean()) < 4.0 / math.sqrt(n)
    assert abs(z.var() - 1.0) < 4.0 * math.sqrt(2.0 / n)
    assert stats.kstest(z, "norm").pvalue > 1e-3
    # pairs from one Box-Muller call are uncorrelated
    assert abs(np.corrcoef(z[0::2], z[1::2])[0, 1]) < 4.0 / math.sqrt(n / 2)


def test_streams_are_distinct_and_prefix_stable():
    a = philox.normals(7, 0, 1001)
    b = philox.normals(7, 1, 1001)
    c = philox.normals(8, 0, 1001)
    assert not np.allclose(a, b) and not np.allclose(a, c)
    np.testing.assert_array_equal(philox.normals(7, 0, 10), a[:10])
