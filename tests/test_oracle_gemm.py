"""Pins of the oracle's D = A B + C (fp64): a worked example, identities and
relations that a transposed operand, a dropped C or a wrong index would break.
CPU only."""
import os

import numpy as np

import oracle

HERE = os.path.dirname(os.path.abspath(__file__))


def fixture():
    vals = {}
    for line in open(os.path.join(HERE, "golden", "gemm_add_2x3x2.txt")):
        t = line.split("#")[0].split()
        if t:
            vals[t[0]] = np.array([float(x) for x in t[1:]])
    return vals


def test_worked_example():
    g = fixture()
    d = oracle.gemm_add(g["A"].reshape(2, 3), g["B"].reshape(3, 2), g["C"].reshape(2, 2))
    assert np.array_equal(d.ravel(), g["D"])


def test_identities():
    rng = np.random.default_rng(1)
    b = rng.standard_normal((6, 5))
    c = rng.standard_normal((6, 5))
    assert np.array_equal(oracle.gemm_add(np.eye(6), b, c), b + c)          # I B + C
    a = rng.standard_normal((7, 6))
    assert np.array_equal(oracle.gemm_add(a, b), oracle.gemm_add(a, b, np.zeros((7, 5))))  # no C = zero C
    assert np.array_equal(oracle.gemm_add(np.zeros((7, 0)), np.zeros((0, 5)), c[:1].repeat(7, 0)),
                          c[:1].repeat(7, 0))                               # K = 0: D = C


def test_relations():
    rng = np.random.default_rng(2)
    a, b = rng.standard_normal((9, 13)), rng.standard_normal((13, 11))
    c1, c2 = rng.standard_normal((9, 11)), rng.standard_normal((9, 11))
    d = oracle.gemm_add(a, b)
    # linear in C
    assert np.max(np.abs(oracle.gemm_add(a, b, c1 + c2) - (oracle.gemm_add(a, b, c1) + c2))) <= 1e-12
    # (A B)^T = B^T A^T: a transposed operand or swapped index fails this
    assert np.max(np.abs(oracle.gemm_add(b.T, a.T) - d.T)) <= 1e-12
    # associativity through a vector: (A B) x = A (B x)
    x = rng.standard_normal((11, 1))
    assert np.max(np.abs(oracle.gemm_add(d, x) - oracle.gemm_add(a, oracle.gemm_add(b, x)))) <= 1e-11
    # a single nonzero entry of A picks one row of B
    e = np.zeros((9, 13))
    e[4, 7] = 2.0
    row = oracle.gemm_add(e, b)
    assert np.array_equal(row[4], 2.0 * b[7]) and not row[np.arange(9) != 4].any()
