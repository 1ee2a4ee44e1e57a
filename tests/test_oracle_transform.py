"""Pins for the oracle's query/key transform (Dual-QK §3.1, Eq. 1).

* the fixed-order fma chain is reproduced bit for bit by an exact-rational
  brute force (fma(a, b, c) = round(a*b + c), one rounding);
* the result agrees with numpy's matmul to rounding;
* scores are invariant: (q A^{-T}) (K A)^T = q K^T to 1e-10 relative;
* the generator's closed-form A^{-T} really is the inverse transpose.
"""
from fractions import Fraction

import numpy as np

from long_context_decode_dual_b200 import workloads as wl
from oracle import oracle as orc


def _fma_exact(a: float, b: float, c: float) -> float:
    return float(Fraction(a) * Fraction(b) + Fraction(c))   # correctly rounded


def _chain(x, M):
    d = M.shape[0]
    y = np.zeros(d)
    for j in range(d):
        acc = 0.0
        for c in range(d):
            acc = _fma_exact(float(x[c]), float(M[c, j]), acc)
        y[j] = acc
    return y


def test_fma_chain_bit_exact_small():
    rng = np.random.default_rng(3)
    for d in (4, 8, 16):
        X = rng.standard_normal((3, d)) * 10.0 ** rng.integers(-3, 3, (3, d))
        M = rng.standard_normal((d, d))
        Y = orc.transform(X, M)
        for t in range(3):
            assert np.array_equal(Y[t], _chain(X[t], M)), d


def test_transform_matches_matmul():
    rng = np.random.default_rng(4)
    X = rng.standard_normal((64, 128))
    A, _ = wl.make_transform(9, 0)
    np.testing.assert_allclose(orc.transform(X, A), X @ A, rtol=1e-12, atol=1e-12)


def test_generator_inverse_transpose():
    for head in range(3):
        A, Ai = wl.make_transform(17, head)
        np.testing.assert_allclose(A @ Ai.T, np.eye(128), atol=1e-13)
        # non-orthogonal: singular values exp(N(0, 0.3))
        sv = np.linalg.svd(A, compute_uv=False)
        assert sv.max() / sv.min() > 1.5


def test_score_invariance():
    rng = np.random.default_rng(5)
    A, Ai = wl.make_transform(21, 0)
    q = rng.standard_normal((4, 128))
    K = rng.standard_normal((500, 128))
    K[:, [3, 40, 77]] *= 6.0
    qp = orc.transform(q, Ai)
    Kp = orc.transform(K, A)
    ref = q @ K.T
    got = qp @ Kp.T
    rel = np.abs(got - ref).max() / np.abs(ref).max()
    assert rel < 1e-10
    # and the transform really reshapes the data (not an identity)
    assert np.abs(Kp - K).max() > 0.1
