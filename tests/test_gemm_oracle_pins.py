"""Pins for the oracle's matrix product (``oracle.gemm``): a brute-force sum
written out on tiny inputs, identities, a rank-one closed form, the
transpose identity (a swapped operand fails it), and numpy's matmul."""
import numpy as np

import oracle


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def test_brute_force_tiny():
    a, b = _rand((3, 4), 1), _rand((4, 5), 2)
    c = oracle.gemm(a, b)
    for i in range(3):
        for j in range(5):
            s = 0.0
            for k in range(4):
                s += a[i, k] * b[k, j]
            assert abs(c[i, j] - s) <= 1e-14


def test_identities():
    a = _rand((7, 9), 3)
    np.testing.assert_array_equal(oracle.gemm(a, np.eye(9)), a)
    np.testing.assert_array_equal(oracle.gemm(np.eye(7), a), a)


def test_rank_one_closed_form():
    u, v, w, x = _rand(6, 4), _rand(5, 5), _rand(5, 6), _rand(8, 7)
    c = oracle.gemm(np.outer(u, v), np.outer(w, x))
    np.testing.assert_allclose(c, float(v @ w) * np.outer(u, x), rtol=1e-13, atol=1e-13)


def test_transpose_identity():
    a, b = _rand((11, 13), 8), _rand((13, 6), 9)
    np.testing.assert_allclose(oracle.gemm(a, b).T, oracle.gemm(b.T.copy(), a.T.copy()),
                               rtol=0, atol=1e-13)


def test_against_numpy():
    a, b = _rand((70, 50), 10), _rand((50, 61), 11)
    np.testing.assert_allclose(oracle.gemm(a, b), a @ b, rtol=0, atol=1e-12)
