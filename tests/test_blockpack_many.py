"""The vectorised block encoders of tests/blockpack.py place every field
exactly where the one-block encoders do (CPU; no GPU).  The full-value-range
GPU parity tests pack their matrices with them."""
from __future__ import annotations

import numpy as np

from blockpack import pack_q4_k, pack_q4_k_many, pack_q6_k, pack_q6_k_many, pack_q8_0, pack_q8_0_many


def test_vectorised_encoders_match_one_block_encoders():
    g = np.random.default_rng(123)
    n = 40
    d = g.integers(0, 1 << 16, n)
    dm = g.integers(0, 1 << 16, n)
    q8 = g.integers(-128, 128, (n, 32))
    q8[0, :] = -128
    q8[1, :] = 127
    a = pack_q8_0_many(d, q8).reshape(n, 34)
    for i in range(n):
        assert np.array_equal(a[i], pack_q8_0(int(d[i]), q8[i]))
    sc, m = g.integers(0, 64, (n, 8)), g.integers(0, 64, (n, 8))
    sc[0, :], m[0, :], sc[1, :], m[1, :] = 0, 63, 63, 0
    q4 = g.integers(0, 16, (n, 256))
    b = pack_q4_k_many(d, dm, sc, m, q4).reshape(n, 144)
    for i in range(n):
        assert np.array_equal(b[i], pack_q4_k(int(d[i]), int(dm[i]), sc[i], m[i], q4[i]))
    s6, q6 = g.integers(-128, 128, (n, 16)), g.integers(0, 64, (n, 256))
    s6[0, :], s6[1, :] = -128, 127
    c = pack_q6_k_many(d, s6, q6).reshape(n, 210)
    for i in range(n):
        assert np.array_equal(c[i], pack_q6_k(int(d[i]), s6[i], q6[i]))
