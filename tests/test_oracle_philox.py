"""Pins of the oracle's Philox4x32-10 and of the uniform map.

Philox4x32-10 follows Salmon, Moraes, Dror, Shaw, "Parallel Random Numbers:
As Easy as 1, 2, 3" (SC'11); it is pinned by the Random123 known-answer
vectors stored in ``tests/golden/philox4x32_10_kat.txt``.
"""
import os

import numpy as np
import scipy.stats

from oracle.philox import philox4x32_10, seed_key, to_uniform, uniforms

GOLDEN = os.path.join(os.path.dirname(__file__), "golden",
                      "philox4x32_10_kat.txt")


def _kat_rows():
    rows = []
    for line in open(GOLDEN):
        line = line.split("#")[0].split()
        if line:
            w = [int(x, 16) for x in line]
            rows.append((w[0:4], w[4:6], w[6:10]))
    return rows


def test_known_answer_vectors():
    rows = _kat_rows()
    assert len(rows) == 3
    for ctr, key, want in rows:
        got = [int(x) for x in philox4x32_10(ctr, key)]
        assert got == want, (ctr, key, [hex(x) for x in got])


def test_vectorised_matches_scalar():
    rng = np.random.default_rng(0)
    c = rng.integers(0, 2**32, size=(4, 64), dtype=np.uint64)
    k = rng.integers(0, 2**32, size=2, dtype=np.uint64)
    vec = philox4x32_10(tuple(c), tuple(k))
    for i in range(64):
        sc = philox4x32_10(tuple(int(c[j, i]) for j in range(4)),
                           (int(k[0]), int(k[1])))
        assert [int(vec[j][i]) for j in range(4)] == [int(x) for x in sc]


def test_uniform_map_exact_grid():
    x = np.array([0, 1, 511, 512, 2**31, 2**32 - 1], dtype=np.uint64)
    u = to_uniform(x)
    assert u[0] == 2.0**-24 and u[1] == 2.0**-24 and u[2] == 2.0**-24
    assert u[3] == 3 * 2.0**-24
    assert u[-1] == 1.0 - 2.0**-24
    # every value is an odd multiple of 2^-24 and exact in fp32
    k = u * 2**24
    assert np.all(k == np.round(k)) and np.all(np.round(k) % 2 == 1)
    assert np.all(u.astype(np.float32).astype(np.float64) == u)
    assert np.all((u > 0) & (u < 1))


def test_seed_key_split():
    assert seed_key(0x1122334455667788) == (0x55667788, 0x11223344)
    assert seed_key(5) == (5, 0)


def test_uniformity_of_accept_and_sample_lanes():
    n = 1 << 18
    pos = np.arange(n, dtype=np.uint64)
    u0, u1 = uniforms(12345, 7, 3, pos, 1)
    for u in (u0, u1):
        assert scipy.stats.kstest(u, "uniform").pvalue > 1e-4
        hist = np.bincount((u * 256).astype(np.int64), minlength=256)
        assert scipy.stats.chisquare(hist).pvalue > 1e-4
    # the two lanes are not the same stream
    assert abs(np.corrcoef(u0, u1)[0, 1]) < 0.02


def test_counter_fields_give_distinct_streams():
    base = uniforms(1, 2, 3, 4, 1)
    for args in [(1, 2, 3, 4, 2), (1, 2, 3, 5, 1), (1, 2, 4, 4, 1),
                 (1, 3, 3, 4, 1), (2, 2, 3, 4, 1), (1 << 32, 2, 3, 4, 1)]:
        assert uniforms(*args) != base
