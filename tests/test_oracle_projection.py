"""Pins for the oracle's Q/K/V projection (CPU only): a pure-Python triple
loop on tiny sizes, and the closed form of identity-block weights."""
import numpy as np

from oracle.projection import qkv_projection


def test_projection_matches_triple_loop():
    rng = np.random.default_rng(3)
    C, H, Hq, Hkv, d = 3, 5, 2, 1, 2
    x = rng.standard_normal((C, H))
    w = rng.standard_normal(((Hq + 2 * Hkv) * d, H))
    q, k, v = qkv_projection(x, w, Hq, Hkv, d)
    for t in range(C):
        for n in range((Hq + 2 * Hkv) * d):
            acc = 0.0
            for j in range(H):
                acc += x[t, j] * w[n, j]
            if n < Hq * d:
                got = q[t, n // d, n % d]
            elif n < (Hq + Hkv) * d:
                got = k[t, (n - Hq * d) // d, (n - Hq * d) % d]
            else:
                got = v[t, (n - (Hq + Hkv) * d) // d, (n - (Hq + Hkv) * d) % d]
            assert abs(got - acc) <= 1e-12 * max(1.0, abs(acc))


def test_identity_blocks_select_input_columns():
    """With W rows = unit vectors, Q/K/V are columns of X in the stacked order."""
    rng = np.random.default_rng(4)
    C, Hq, Hkv, d = 4, 2, 1, 3
    n_out = (Hq + 2 * Hkv) * d
    x = rng.standard_normal((C, n_out + 2))
    perm = rng.permutation(n_out + 2)[:n_out]
    w = np.eye(n_out + 2)[perm]
    q, k, v = qkv_projection(x, w, Hq, Hkv, d)
    y = x[:, perm]
    np.testing.assert_array_equal(q.reshape(C, -1), y[:, :Hq * d])
    np.testing.assert_array_equal(k.reshape(C, -1), y[:, Hq * d:(Hq + Hkv) * d])
    np.testing.assert_array_equal(v.reshape(C, -1), y[:, (Hq + Hkv) * d:])
