"""Pins for the oracle's attention (Dual-QK §3.2 normalisation, §3.4 one
global softmax).

* plain attention equals numpy/scipy softmax(q K^T / sqrt(d)) V;
* s = 0 on unquantized transformed keys equals plain attention on the
  original q, K (score invariance, Eq. 1);
* pruned attention equals the library computation restricted to the kept
  channels, still divided by sqrt(128);
* one token gives o = v exactly; equal scores give the mean of V; no tokens
  give zeros;
* the quantized decode step equals the library computation on the
  dequantized cache.
"""
import numpy as np
import pytest
from scipy.special import softmax

from long_context_decode_dual_b200 import workloads as wl
from oracle import oracle as orc


def _lib_attn(q, K, V, idx=None, d=128):
    if idx is None:
        idx = np.arange(q.shape[1])
    s = q[:, idx] @ K[:, idx].T / np.sqrt(d)
    return softmax(s, axis=1) @ V


def test_plain_attention_matches_library():
    rng = np.random.default_rng(0)
    q = rng.standard_normal((4, 128))
    K = rng.standard_normal((777, 128)) * 2
    V = rng.standard_normal((777, 128))
    np.testing.assert_allclose(orc.attention(q, K, V), _lib_attn(q, K, V), rtol=1e-12, atol=1e-13)


def test_unpruned_unquantized_is_invariant():
    rng = np.random.default_rng(1)
    A, Ai = wl.make_transform(33, 1)
    q = rng.standard_normal((4, 128))
    K = rng.standard_normal((600, 128))
    V = rng.standard_normal((600, 128))
    qp, Kp = orc.transform(q, Ai), orc.transform(K, A)
    idx, _ = orc.select(qp, orc.num_selected(0.0))
    got = orc.decode_dense(Kp, V, qp, idx)
    np.testing.assert_allclose(got, _lib_attn(q, K, V), rtol=1e-10, atol=1e-12)


def test_pruned_uses_full_dim_normalisation():
    rng = np.random.default_rng(2)
    qp = rng.standard_normal((4, 128)) * 2
    K = rng.standard_normal((333, 128))
    V = rng.standard_normal((333, 128))
    idx, _ = orc.select(qp, 77)
    got = orc.decode_dense(K, V, qp, idx)
    np.testing.assert_allclose(got, _lib_attn(qp, K, V, idx, d=128), rtol=1e-12, atol=1e-13)
    wrong = _lib_attn(qp, K, V, idx, d=77)
    assert np.abs(got - wrong).max() > 1e-3


def test_degenerate_cases():
    rng = np.random.default_rng(3)
    q = rng.standard_normal((2, 128))
    K = rng.standard_normal((1, 128))
    V = rng.standard_normal((1, 128))
    assert np.array_equal(orc.attention(q, K, V), np.repeat(V, 2, axis=0))
    K = rng.standard_normal((50, 128))
    V = rng.standard_normal((50, 128))
    np.testing.assert_allclose(orc.attention(np.zeros((1, 128)), K, V)[0], V.mean(axis=0),
                               rtol=1e-12, atol=1e-14)
    assert not orc.attention(q, K[:0], V[:0]).any()


@pytest.mark.parametrize("bits", [2, 4])
def test_quantized_decode_step(bits):
    rng = np.random.default_rng(4)
    A, Ai = wl.make_transform(44, 0)
    n = 300                                      # two pages and a ragged tail
    K = rng.standard_normal((n, 128))
    V = rng.standard_normal((n, 128))
    q = rng.standard_normal((4, 128))
    unit = orc.new_unit(384, bits)
    orc.append_unit(unit, bits, 0, orc.transform(K, A), V)
    qp = orc.transform(q, Ai)
    out, idx = orc.decode_unit(unit, bits, n, qp, 0.4)
    assert idx.size == 77 and idx[0] == 0
    Kh, Vh = orc.dequant_unit(unit, bits, n)
    np.testing.assert_allclose(out, _lib_attn(qp, Kh, Vh, idx), rtol=1e-12, atol=1e-13)
