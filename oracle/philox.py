"""Counter-based random numbers for the oracle's random-feature matrix.

TEST INFRASTRUCTURE.  Everything under ``oracle/`` exists only to check the
CUDA path: it may be imported by ``tests/``, by ``__graft_entry__.smoke()`` and
by the ``cpu_baseline`` / ``--impl reference`` legs of ``bench.py``, and by
nothing else.  It shares no code with the library under
``linear_approximate_softmax_b200/``.

The method draws its random features once, from a seed ("Rethinking Attention
with Performers", Abstract: FAVOR+ samples positive orthogonal random
features).  Because the seed is the only input, the C library and this oracle
each implement the same published counter-based generator, independently:

* Philox4x64-10 (Salmon, Moraes, Dror, Shaw, "Parallel Random Numbers: As Easy
  as 1, 2, 3", SC'11).  One call maps a 4x64-bit counter and a 2x64-bit key to
  four 64-bit words through ten rounds of two 64x64->128-bit multiplies, with
  the key advanced by two Weyl constants between rounds.
* Box-Muller (Box and Muller, "A Note on the Generation of Random Normal
  Deviates", Ann. Math. Stat. 1958): two uniforms give two independent
  standard normals.

Stream convention (the same on both sides; it is a convention, not part of the
method): the n-th standard normal of stream ``tag`` under ``seed`` comes from
the Philox call with counter ``(n // 4, tag, 0, 0)`` and key ``(seed, 0)``.
Words (x0, x1) give normals n % 4 = 0, 1 and words (x2, x3) give 2, 3, each
pair through Box-Muller with u = ((x >> 12) + 1/2) * 2**-52, so u lies in
[2**-53, 1 - 2**-53] (both ends exact in fp64) and the logarithm is finite.

Pinned in ``tests/test_oracle_philox.py`` against numpy's own Philox4x64
bit generator, a separate implementation of the same definition.
"""
import numpy as np

_M32 = np.uint64(0xFFFFFFFF)
_S32 = np.uint64(32)

# Philox4x64 round multipliers and Weyl key increments (Salmon et al. 2011).
PHILOX_M0 = np.uint64(0xD2E7470EE14C6C93)
PHILOX_M1 = np.uint64(0xCA5A826395121157)
PHILOX_W0 = np.uint64(0x9E3779B97F4A7C15)
PHILOX_W1 = np.uint64(0xBB67AE8584CAA73B)


def _mulhilo64(a, b):
    """Full 64x64 -> 128-bit product of uint64 arrays, as (hi, lo)."""
    a = np.asarray(a, dtype=np.uint64)
    b = np.asarray(b, dtype=np.uint64)
    a_lo, a_hi = a & _M32, a >> _S32
    b_lo, b_hi = b & _M32, b >> _S32
    with np.errstate(over="ignore"):
        p0 = a_lo * b_lo
        p1 = a_lo * b_hi
        p2 = a_hi * b_lo
        p3 = a_hi * b_hi
        mid = (p0 >> _S32) + (p1 & _M32) + (p2 & _M32)
        hi = p3 + (p1 >> _S32) + (p2 >> _S32) + (mid >> _S32)
        lo = (mid << _S32) | (p0 & _M32)
    return hi, lo


def philox4x64_10(c0, c1, c2, c3, k0, k1):
    """Ten Philox4x64 rounds on counters (c0..c3) with key (k0, k1).

    All arguments broadcast as uint64 arrays; returns four uint64 arrays.
    """
    c = [np.asarray(x, dtype=np.uint64) for x in (c0, c1, c2, c3)]
    k0 = np.asarray(k0, dtype=np.uint64)
    k1 = np.asarray(k1, dtype=np.uint64)
    for r in range(10):
        if r > 0:
            with np.errstate(over="ignore"):
                k0 = k0 + PHILOX_W0
                k1 = k1 + PHILOX_W1
        hi0, lo0 = _mulhilo64(PHILOX_M0, c[0])
        hi1, lo1 = _mulhilo64(PHILOX_M1, c[2])
        c = [hi1 ^ c[1] ^ k0, lo1, hi0 ^ c[3] ^ k1, lo0]
    return c


def uniform52(x):
    """Map uint64 words to doubles strictly inside (0, 1) (top 52 bits + 1/2)."""
    x = np.asarray(x, dtype=np.uint64)
    return ((x >> np.uint64(12)).astype(np.float64) + 0.5) * 2.0 ** -52


def box_muller(u0, u1):
    """Two independent standard normals from two uniforms in (0, 1)."""
    r = np.sqrt(-2.0 * np.log(u0))
    t = 2.0 * np.pi * u1
    return r * np.cos(t), r * np.sin(t)


def normals(seed, tag, count):
    """Normals 0 .. count-1 of stream ``tag`` under ``seed`` (float64)."""
    ncalls = (count + 3) // 4
    j = np.arange(ncalls, dtype=np.uint64)
    zero = np.zeros_like(j)
    x = philox4x64_10(j, np.full_like(j, tag), zero, zero,
                      np.uint64(seed), np.uint64(0))
    z0, z1 = box_muller(uniform52(x[0]), uniform52(x[1]))
    z2, z3 = box_muller(uniform52(x[2]), uniform52(x[3]))
    out = np.stack([z0, z1, z2, z3], axis=1).reshape(-1)
    return out[:count]
