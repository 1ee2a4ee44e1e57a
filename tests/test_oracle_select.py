"""Pins for the oracle's channel selection (Dual-QK §3.2, Eq. 4).

* k = ceil((1 - s) d) for the pages' sparsities;
* brute force with Python's sort on small d, with forced ties;
* s = 0 keeps every channel; g = 1 orders by |q'|;
* channel 0 is kept even when its energy is the smallest;
* the kept set minimises the variance of the dropped part of the score
  (Dual-QK App. C.2: Var_k[sum_{j not in M} q_j k_j] = sigma^2 sum q_j^2).
"""
import numpy as np
import pytest

from oracle import oracle as orc


@pytest.mark.parametrize("s,k", [(0.0, 128), (0.2, 103), (0.4, 77), (0.6, 52), (0.25, 96),
                                 (0.5, 64), (0.99, 2)])
def test_k(s, k):
    assert orc.num_selected(s) == k


def _brute(qp, k):
    e2 = (qp.astype(object) ** 2).sum(axis=0)          # exact for integer inputs
    d = qp.shape[1]
    rest = sorted(range(1, d), key=lambda j: (-e2[j], j))[:k - 1]
    return sorted([0] + rest)


def test_bruteforce_with_ties():
    rng = np.random.default_rng(0)
    for _ in range(400):
        d = int(rng.choice([8, 16]))
        g = int(rng.choice([1, 2, 4]))
        qp = rng.integers(-2, 3, size=(g, d)).astype(np.float64)   # many ties
        k = int(rng.integers(1, d + 1))
        idx, e2 = orc.select(qp, k)
        assert list(idx) == _brute(qp, k)
        assert np.array_equal(e2, (qp ** 2).sum(axis=0))


def test_all_and_single_head():
    rng = np.random.default_rng(1)
    qp = rng.standard_normal((4, 128))
    idx, _ = orc.select(qp, 128)
    assert list(idx) == list(range(128))
    q1 = rng.standard_normal((1, 128))
    idx, _ = orc.select(q1, 40)
    order = [0] + sorted(range(1, 128), key=lambda j: (-abs(q1[0, j]), j))[:39]
    assert list(idx) == sorted(order)


def test_channel0_always_kept():
    qp = np.ones((4, 16))
    qp[:, 0] = 0.0
    idx, _ = orc.select(qp, 3)
    assert list(idx) == [0, 1, 2]


def test_selection_minimises_dropped_variance():
    rng = np.random.default_rng(2)
    q = rng.standard_normal((1, 128)) * np.exp(rng.standard_normal(128))[None]
    k = 77
    idx, _ = orc.select(q, k)
    dropped = np.setdiff1d(np.arange(128), idx)
    keys = rng.standard_normal((200000, 128))
    var_emp = np.var(keys[:, dropped] @ q[0, dropped])
    var_formula = np.sum(q[0, dropped] ** 2)
    assert var_emp == pytest.approx(var_formula, rel=0.02)
    for _ in range(50):
        other = rng.choice(np.arange(1, 128), size=128 - k, replace=False)
        assert np.sum(q[0, other] ** 2) >= var_formula - 1e-12


def _by_ranks(e2, k):
    """The choice as rank counts (channel 0 always; channel j of 1..d-1 when
    fewer than k - 1 channels of 1..d-1 come before it by (energy descending,
    index ascending)), with energies compared as their float64 bit patterns,
    each rank summed from eight partial counts over 16-channel ranges."""
    d = e2.shape[0]
    key = e2.view(np.uint64)
    kept = [0]
    for j in range(1, d):
        parts = []
        for p in range(8):
            lo, hi = p * d // 8, (p + 1) * d // 8
            parts.append(sum(1 for i in range(lo, hi)
                             if i != 0 and (key[i] > key[j] or (key[i] == key[j] and i < j))))
        if sum(parts) < k - 1:
            kept.append(j)
    return kept


def test_rank_counts_equal_the_sort():
    """Reading of the channel choice used by the tensor-core path: counting
    each channel's rank gives the oracle's sorted choice, ties and zero
    energies included (energies are >= 0, so bit patterns order like values)."""
    rng = np.random.default_rng(3)
    for trial in range(60):
        g = int(rng.choice([1, 4, 8]))
        if trial % 3 == 0:
            qp = rng.integers(-2, 3, size=(g, 128)).astype(np.float64)     # many exact ties and zeros
        else:
            qp = rng.standard_normal((g, 128))
        k = int(rng.choice([1, 2, 52, 77, 103, 128]))
        idx, e2 = orc.select(qp, k)
        assert (e2 >= 0).all()
        assert list(idx) == _by_ranks(np.ascontiguousarray(e2, dtype=np.float64), k)
