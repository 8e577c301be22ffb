"""Pins of the oracle's Philox4x32-10 and uniform mapping (CPU only)."""

import os

import numpy as np

from oracle.philox import bits_to_uniform, philox4x32_10, uniform, KIND_DRAFT, KIND_FIRST

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "philox4x32_10_kat.txt")


def _kat_rows():
    rows = []
    with open(GOLDEN) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            w = [int(x, 16) for x in line.split()]
            rows.append((w[0:4], w[4:6], w[6:10]))
    return rows


def test_known_answer_vectors():
    rows = _kat_rows()
    assert len(rows) == 3
    for ctr, key, want in rows:
        got = [int(x) for x in philox4x32_10(ctr, key)]
        assert got == want, (ctr, key, [hex(x) for x in got])


def test_vectorised_matches_scalar():
    ctr0 = np.arange(37, dtype=np.uint64) * 1000003
    out = philox4x32_10((ctr0, 5, 7, 0), (123, 456))
    for i in range(37):
        one = philox4x32_10((int(ctr0[i]), 5, 7, 0), (123, 456))
        assert [int(w[i]) for w in out] == [int(x) for x in one]


def test_uniform_closed_forms():
    assert bits_to_uniform(0) == 2.0 ** -24
    assert bits_to_uniform(0xFFFFFFFF) == 1.0 - 2.0 ** -24
    assert bits_to_uniform(1 << 9) == 3.0 * 2.0 ** -24
    # exact in float32
    x = np.random.default_rng(0).integers(0, 2 ** 32, 10000, dtype=np.uint64)
    u = bits_to_uniform(x)
    assert np.all(u > 0) and np.all(u < 1)
    assert np.array_equal(u.astype(np.float32).astype(np.float64), u)


def test_uniform_keying_and_distribution():
    # different kinds / positions / streams give different draws
    a = uniform(1, 0, 10, KIND_FIRST)
    b = uniform(1, 0, 10, KIND_DRAFT)
    c = uniform(1, 0, 11, KIND_FIRST)
    d = uniform(1, 1, 10, KIND_FIRST)
    e = uniform(2, 0, 10, KIND_FIRST)
    assert len({float(a), float(b), float(c), float(d), float(e)}) == 5
    # mean / variance of 2^20 draws within 6 sigma of U(0,1)
    pos = np.arange(1 << 20, dtype=np.uint64)
    u = uniform(7, 3, pos, KIND_DRAFT)
    n = u.size
    assert abs(u.mean() - 0.5) < 6 * np.sqrt(1 / 12 / n)
    assert abs(u.var() - 1 / 12) < 6 * np.sqrt(1 / 180 / n)
    # the 64-bit seed uses both key words
    assert float(uniform(1 << 32, 0, 0, 0)) != float(uniform(0, 0, 0, 0))
