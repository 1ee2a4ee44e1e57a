"""Pins for the oracle's bucket-relative RoPE (Dual-QK §3.4, App. C.4).

Keys are stored in the frame of their bucket's anchor, z_n = k_n T_b B; the
query of bucket b is q T_b A; each bucket chooses its own channels from its
base queries; one softmax covers every bucket.  T_b removes the rotary
rotation of the anchor a_b (rotate-half channel pairs (i, i + 64)).

* rope_unanchor against hand values (angles 0 and pi/2) and against RoPE
  applied directly at the relative position n - a_b (numpy), which fixes the
  pairing and the direction of the rotation;
* scores are unchanged by the bucket frames and transforms (unquantized);
* one bucket covering the context is the plain decode, bit for bit;
* the bucketed decode equals plain attention when nothing is quantized or
  pruned (scipy), and the numpy gather of each token's bucket otherwise;
* per-bucket channel lists are the brute-force choices of each bucket's
  queries, and they differ between buckets.
"""
import numpy as np
import pytest
from scipy.special import softmax

from long_context_decode_dual_b200 import workloads as wl
from oracle import oracle as orc

D = 128
H = D // 2


def _rope(x: np.ndarray, pos, base=500000.0) -> np.ndarray:
    """Rotate-half RoPE of rows x at positions pos (numpy, for the pins)."""
    x = np.atleast_2d(x)
    pos = np.broadcast_to(np.asarray(pos, dtype=np.float64), (x.shape[0],))
    theta = base ** (-2.0 * np.arange(H) / D)
    ang = pos[:, None] * theta[None, :]
    c, s = np.cos(ang), np.sin(ang)
    a, b = x[:, :H], x[:, H:]
    return np.concatenate([a * c - b * s, b * c + a * s], axis=1)


def test_unanchor_hand_values():
    x = np.arange(1, D + 1, dtype=np.float64)[None, :]
    ident = np.tile([1.0, 0.0], (H, 1))
    assert np.array_equal(orc.rope_unanchor(x, ident), x)
    quarter = np.tile([0.0, 1.0], (H, 1))                # a quarter turn back
    y = orc.rope_unanchor(x, quarter)
    assert np.array_equal(y[0, :H], x[0, H:]) and np.array_equal(y[0, H:], -x[0, :H])
    # one pair by hand: x = (3, 4) at angle with cos 0.6, sin 0.8
    cs = np.tile([1.0, 0.0], (H, 1))
    cs[5] = (0.6, 0.8)
    v = np.zeros((1, D))
    v[0, 5], v[0, 5 + H] = 3.0, 4.0
    y = orc.rope_unanchor(v, cs)
    assert y[0, 5] == 3.0 * 0.6 + 4.0 * 0.8 and y[0, 5 + H] == 4.0 * 0.6 - 3.0 * 0.8


@pytest.mark.parametrize("w", [128, 2048])
def test_unanchor_gives_relative_position(w):
    rng = np.random.default_rng(3)
    table = wl.rope_table(70, w)
    for n in (0, 5, w - 1, w, 3 * w + 17, 64 * w + 100):
        b = n // w
        k0 = rng.standard_normal(D)
        got = orc.rope_unanchor(_rope(k0, n), table[b])
        want = _rope(k0, n - b * w)
        assert np.abs(got - want).max() < 1e-9 * np.abs(want).max()


def test_scores_unchanged_by_bucket_frames():
    rng = np.random.default_rng(4)
    A, Ai = wl.make_transform(4, 0)
    table = wl.rope_table(9, 2048)
    q = rng.standard_normal((4, D))
    K = rng.standard_normal((50, D)) * 3
    want = q @ K.T
    for b in (0, 1, 8):
        got = orc.transform(orc.rope_unanchor(q, table[b]), Ai) @ orc.transform(orc.rope_unanchor(K, table[b]), A).T
        assert np.abs(got - want).max() < 1e-10 * np.abs(want).max()


def test_one_bucket_is_the_plain_decode():
    rng = np.random.default_rng(5)
    n, w = 600, 2048
    A, Ai = wl.make_transform(5, 0)
    table = wl.rope_table(1, w)
    assert np.array_equal(table[0], np.tile([1.0, 0.0], (H, 1)))
    K, V = rng.standard_normal((n, D)), rng.standard_normal((n, D))
    Kb = orc.bucket_keys(K, A, table, w)
    assert np.array_equal(Kb, orc.transform(K, A))
    unit = orc.new_unit(640, 2)
    orc.append_unit(unit, 2, 0, Kb, V)
    q = rng.standard_normal((4, D))
    qpb = orc.bucket_queries(q, Ai, table, 1)
    out_b, idx_b = orc.decode_unit_buckets(unit, 2, n, qpb, 0.4, w)
    out, idx = orc.decode_unit(unit, 2, n, orc.transform(q, Ai), 0.4)
    assert np.array_equal(out_b, out) and np.array_equal(idx_b[0], idx)


def test_unquantized_buckets_are_plain_attention():
    rng = np.random.default_rng(6)
    n, w = 700, 128
    A, Ai = wl.make_transform(6, 1)
    table = wl.rope_table(6, w)
    K, V = rng.standard_normal((n, D)) * 2, rng.standard_normal((n, D))
    q = rng.standard_normal((4, D))
    Kb = orc.bucket_keys(K, A, table, w)
    qpb = orc.bucket_queries(q, Ai, table, 6)
    all_ch = np.tile(np.arange(D, dtype=np.int32), (6, 1))
    got = orc.decode_buckets(Kb, V, qpb, all_ch, w)
    want = softmax(q @ K.T / np.sqrt(D), axis=1) @ V
    assert np.abs(got - want).max() < 1e-10 * np.abs(want).max()
    # a bucket frame used for the wrong tokens breaks it
    wrong = orc.decode_buckets(Kb, V, qpb[::-1].copy(), all_ch, w)
    assert np.abs(wrong - want).max() > 1e-3


@pytest.mark.parametrize("group", [32, 128])
def test_bucketed_decode_matches_numpy_gather(group):
    rng = np.random.default_rng(7)
    n, w, g = 900, 256, 4
    A, Ai = wl.make_transform(7, 2)
    table = wl.rope_table(4, w)
    K, V = rng.standard_normal((n, D)), rng.standard_normal((n, D))
    q = rng.standard_normal((g, D))
    unit = orc.new_unit(1024, 2, group)
    orc.append_unit(unit, 2, 0, orc.bucket_keys(K, A, table, w), V, group)
    qpb = orc.bucket_queries(q, Ai, table, 4)
    out, idxb = orc.decode_unit_buckets(unit, 2, n, qpb, 0.4, w, group)
    k = orc.num_selected(0.4)
    for b in range(4):
        e2 = (qpb[b] ** 2).sum(axis=0)
        order = sorted(range(1, D), key=lambda j: (-e2[j], j))
        assert np.array_equal(idxb[b], np.array(sorted([0] + order[:k - 1])))
    assert len({tuple(x) for x in idxb}) > 1           # the masks differ across buckets
    Kh, Vh = orc.dequant_unit(unit, 2, n, group)
    sc = np.empty((g, n))
    for t in range(n):
        b = t // w
        sc[:, t] = qpb[b][:, idxb[b]] @ Kh[t, idxb[b]]
    want = softmax(sc / np.sqrt(D), axis=1) @ Vh
    assert np.abs(out - want).max() < 1e-12 * np.abs(want).max()


def test_buckets_with_tier_rotation_and_refinement():
    rng = np.random.default_rng(8)
    n, w, g = 1000, 256, 4
    A0, Ai0 = wl.make_transform(8, 0)
    delta = wl.make_refinement(8, 0)
    A, Ai = A0 / delta[None, :], Ai0 * delta[None, :]
    R = wl.make_value_rotation(8, 0)
    table = wl.rope_table(4, w)
    K, V = rng.standard_normal((n, D)), rng.standard_normal((n, D))
    Kb, Vr = orc.bucket_keys(K, A, table, w), orc.value_rotate(V, R)
    unit = orc.new_unit(1024, 2, 128)
    slots = orc.new_slots(64, 256)
    orc.append_unit(unit, 2, 0, Kb, Vr, 128, vclip=0.92)
    orc.protect_store(slots, 64, 256, 0, Kb, Vr, n)
    q = rng.standard_normal((g, D))
    qpb = orc.bucket_queries(q, Ai, table, 4)
    out, idxb = orc.decode_unit_buckets(unit, 2, n, qpb, 0.4, w, 128, delta=delta, Rv=R, slots=slots,
                                        n_sink=64, n_recent=256)
    for b in range(4):
        # each bucket's mask: its base queries q T_b A0 (the unrefined transform)
        base = orc.transform(orc.rope_unanchor(q, table[b]), Ai0)
        assert np.array_equal(idxb[b], orc.select(base, orc.num_selected(0.4))[0])
    Kh, Vh = orc.dequant_unit(unit, 2, n, 128)
    for p in list(range(64)) + list(range(n - 256, n)):
        s_ = orc.protected_slot(p, 64, 256)
        Kh[p] = [orc.bf16_value(x) for x in slots[s_, :D]]
        Vh[p] = [orc.bf16_value(x) for x in slots[s_, D:]]
    sc = np.empty((g, n))
    for t in range(n):
        b = t // w
        sc[:, t] = qpb[b][:, idxb[b]] @ Kh[t, idxb[b]]
    want = softmax(sc / np.sqrt(D), axis=1) @ Vh @ R.T
    assert np.abs(out - want).max() < 1e-12 * np.abs(want).max()
