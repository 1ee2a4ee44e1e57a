"""Pins for the oracle's value rotation, value clipping and refined selection.

Dual-QK §3.3 and App. B.2: values are multiplied by an orthogonal rotation,
quantized per token with asymmetric INT2 and a clipping ratio of 0.92 (keys
are not clipped), and the aggregated output is rotated back.  §3.3 and
App. C.2: a positive diagonal refinement D (delta_0 = 1) is folded into the
transforms; selection uses the base queries q A0 = (q A0 D) D^{-1}, scores
the final ones.

* the clipped grid against hand-computed fp16 bits and codes, and against a
  nearest-level search with numpy's float16 rounding;
* clipping touches the value grids only;
* rotate -> attend -> rotate back equals plain attention (scipy) when nothing
  is quantized or pruned (this fixes the orientation of both rotations);
* the quantized, rotated decode equals the same computation written with
  numpy on the dequantized cache;
* refined selection equals a brute-force sort of the base queries' pooled
  energies computed with numpy from the unrefined transform, and scores are
  unchanged by the refinement.
"""
import numpy as np
import pytest
from scipy.special import softmax

from long_context_decode_dual_b200 import workloads as wl
from oracle import oracle as orc

D = 128


def _f16(x: float) -> float:
    return float(np.float16(x))


def test_clip_hand_computed():
    # range [-1, 2], clip 0.92: grid [-0.92, 1.84], step 2.76 / 3 = 0.92;
    # fp16(0.92) = 1884 / 2048 = 0.919921875 (bits 0x3B5C = 15196)
    s, z, c = orc.quantize_group([-1.0, 0.0, 0.5, 2.0], 2, 0.92)
    assert s == 15196 and z == 15196 | 0x8000
    # (x - z) / s = -0.087, 1, 1.54, 3.17 -> 0, 1, 2, 3 (both ends clamp)
    assert list(c) == [0, 1, 2, 3]
    # all positive: the clipped grid starts below the minimum
    s, z, c = orc.quantize_group([1.0, 2.0, 3.0, 4.0], 2, 0.92)
    assert s == 15196 and z == 15196                    # grid [0.92, 3.68]
    assert list(c) == [0, 1, 2, 3]                      # 0.087, 1.17, 2.26, 3.35
    # clip 1 is the plain min/max grid: [-1, 2], step 1 (0x3C00), zero -1
    # (0xBC00); 0.5 -> 1.5 rounds to the even code 2
    s, z, c = orc.quantize_group([-1.0, 0.0, 0.5, 2.0], 2, 1.0)
    assert (s, z, list(c)) == (0x3C00, 0xBC00, [0, 1, 2, 3])


@pytest.mark.parametrize("clip", [0.92, 0.5, 0.999])
@pytest.mark.parametrize("bits", [2, 4])
def test_clip_nearest_level(clip, bits):
    rng = np.random.default_rng(7)
    L = (1 << bits) - 1
    for trial in range(200):
        x = rng.standard_normal(32) * rng.uniform(0.1, 10)
        if trial % 3 == 0:
            x = np.abs(x) + 0.5                        # one-signed groups
        s_bits, z_bits, codes = orc.quantize_group(x, bits, clip)
        lo, hi = clip * x.min(), clip * x.max()
        z = _f16(lo)
        s = _f16((hi - lo) / L)
        assert np.float16(z).view(np.uint16) == z_bits
        assert np.float16(s).view(np.uint16) == s_bits
        levels = z + s * np.arange(L + 1)
        want = np.argmin(np.abs(x[:, None] - levels[None, :]), axis=1)
        assert np.array_equal(codes, want)


def test_clip_only_on_values():
    rng = np.random.default_rng(3)
    n = 300
    Kp = rng.standard_normal((n, D)) * 2
    V = rng.standard_normal((n, D))
    for group in (32, 128):
        u1 = orc.new_unit(384, 2, group)
        u2 = orc.new_unit(384, 2, group)
        orc.append_unit(u1, 2, 0, Kp, V, group)
        orc.append_unit(u2, 2, 0, Kp, V, group, vclip=0.92)
        K1, V1 = orc.dequant_unit(u1, 2, n, group)
        K2, V2 = orc.dequant_unit(u2, 2, n, group)
        assert np.array_equal(K1, K2)
        assert not np.array_equal(V1, V2)
        # each value group dequantizes to its clipped grid's levels
        for t in (0, 77, 299):
            for g0 in range(0, D, group):
                s, z, c = orc.quantize_group(V[t, g0:g0 + group], 2, 0.92)
                want = orc.f16_value(s) * c + orc.f16_value(z)
                assert np.array_equal(V2[t, g0:g0 + group], want)


def test_hadamard_and_rotation_inputs():
    H = wl.sylvester_hadamard(D)
    assert set(np.unique(H)) == {-1.0, 1.0}
    assert np.array_equal(H @ H.T, D * np.eye(D))
    R = wl.make_value_rotation(3000, 2)
    assert np.abs(R @ R.T - np.eye(D)).max() < 1e-13
    assert np.abs(R - R.T).max() > 0.1                  # not symmetric: orientation matters


def test_rotation_round_trip_and_plain_attention():
    rng = np.random.default_rng(11)
    R = wl.make_value_rotation(5, 0)
    V = rng.standard_normal((50, D))
    assert np.abs(orc.value_unrotate(orc.value_rotate(V, R), R) - V).max() < 1e-13
    # unquantized, unpruned: attention on rotated values, rotated back, is
    # plain attention on the original values
    A, Ai = wl.make_transform(9, 0)
    q = rng.standard_normal((4, D))
    K = rng.standard_normal((200, D)) * 2
    V = rng.standard_normal((200, D))
    out_rot = orc.decode_dense(orc.transform(K, A), orc.value_rotate(V, R), orc.transform(q, Ai), np.arange(D))
    got = orc.value_unrotate(out_rot, R)
    want = softmax(q @ K.T / np.sqrt(D), axis=1) @ V
    assert np.abs(got - want).max() < 1e-10 * np.abs(want).max()
    # rotating back with R instead of R^T is visibly wrong
    assert np.abs(orc.transform(out_rot, R) - want).max() > 1e-3


@pytest.mark.parametrize("group", [32, 128])
def test_rotated_clipped_decode_matches_numpy(group):
    rng = np.random.default_rng(21)
    n, g = 700, 4
    R = wl.make_value_rotation(21, 1)
    A, Ai = wl.make_transform(21, 1)
    K = rng.standard_normal((n, D))
    V = rng.standard_normal((n, D))
    q = rng.standard_normal((g, D))
    Kp = orc.transform(K, A)
    unit = orc.new_unit(768, 2, group)
    orc.append_unit(unit, 2, 0, Kp, orc.value_rotate(V, R), group, vclip=0.92)
    qp = orc.transform(q, Ai)
    out, idx = orc.decode_unit(unit, 2, n, qp, 0.4, group, Rv=R)
    Kh, Vh = orc.dequant_unit(unit, 2, n, group)
    sc = qp[:, idx] @ Kh[:, idx].T / np.sqrt(D)
    want = softmax(sc, axis=1) @ Vh @ R.T
    assert np.abs(out - want).max() < 1e-12 * np.abs(want).max()
    # the rotation and the clip reduce the value error on heavy-tailed values
    # (the reason the pages use them); a sanity check of the inputs, not a pin
    Vt = rng.standard_t(4, size=(n, D))
    u_plain = orc.new_unit(768, 2, group)
    u_rot = orc.new_unit(768, 2, group)
    orc.append_unit(u_plain, 2, 0, Kp, Vt, group)
    orc.append_unit(u_rot, 2, 0, Kp, orc.value_rotate(Vt, R), group, vclip=0.92)
    e_plain = np.mean((orc.dequant_unit(u_plain, 2, n, group)[1] - Vt) ** 2)
    e_rot = np.mean((orc.transform(orc.dequant_unit(u_rot, 2, n, group)[1], np.ascontiguousarray(R.T)) - Vt) ** 2)
    assert e_rot < e_plain


def test_protected_tier_holds_rotated_values():
    # every token protected: the decode is pruned attention on the BF16 keys
    # and BF16 rotated values, rotated back
    rng = np.random.default_rng(5)
    n, g = 150, 4
    R = wl.make_value_rotation(5, 3)
    Kp = rng.standard_normal((n, D)).astype(np.float32).astype(np.float64)
    Vr = orc.value_rotate(rng.standard_normal((n, D)), R)
    unit = orc.new_unit(256, 2)
    slots = orc.new_slots(64, 256)
    orc.append_unit(unit, 2, 0, Kp, Vr, vclip=0.92)
    orc.protect_store(slots, 64, 256, 0, Kp, Vr, n)
    qp = rng.standard_normal((g, D))
    out, idx = orc.decode_unit_protected(unit, slots, 2, n, qp, 0.4, 64, 256, Rv=R)
    kb = np.array([[orc.bf16_value(b) for b in orc.bf16_rne(row)] for row in Kp])
    vb = np.array([[orc.bf16_value(b) for b in orc.bf16_rne(row)] for row in Vr])
    want = softmax(qp[:, idx] @ kb[:, idx].T / np.sqrt(D), axis=1) @ vb @ R.T
    assert np.abs(out - want).max() < 1e-12 * np.abs(want).max()


def _base_selection(e2_base: np.ndarray, k: int) -> np.ndarray:
    order = sorted(range(1, D), key=lambda j: (-e2_base[j], j))
    return np.array(sorted([0] + order[:k - 1]), dtype=np.int32)


@pytest.mark.parametrize("g", [1, 4, 8])
@pytest.mark.parametrize("sparsity", [0.2, 0.4, 0.6])
def test_refined_selection_uses_base_queries(g, sparsity):
    k = orc.num_selected(sparsity)
    checked = 0
    for seed in range(12):
        A0, Ai0 = wl.make_transform(100 + seed, 0)
        delta = wl.make_refinement(100 + seed, 0)
        Ai = Ai0 * delta[None, :]                       # folded query transform A0 D
        q = np.random.default_rng(seed).standard_normal((g, D))
        base = q @ Ai0                                  # numpy, not the oracle's chain
        e2_base = (base ** 2).sum(axis=0)
        srt = np.sort(e2_base[1:])[::-1]
        if k - 1 < D - 1 and (srt[k - 2] - srt[k - 1]) < 1e-9 * srt[0]:
            continue                                    # a near tie at the cut: rounding may decide
        qp = orc.transform(q, Ai)
        idx, _ = orc.select(qp, k, delta)
        assert np.array_equal(idx, _base_selection(e2_base, k))
        # the same as selecting on the unrefined transform
        idx0, _ = orc.select(orc.transform(q, Ai0), k)
        assert np.array_equal(idx, idx0)
        checked += 1
    assert checked >= 8


def test_refined_selection_differs_from_final_energies():
    # the refinement does move the final queries' energies: selecting on them
    # (no delta) would give another mask for some seed
    k = orc.num_selected(0.4)
    differs = False
    for seed in range(8):
        _, Ai0 = wl.make_transform(200 + seed, 0)
        delta = wl.make_refinement(200 + seed, 0)
        qp = orc.transform(np.random.default_rng(seed).standard_normal((4, D)), Ai0 * delta[None, :])
        differs |= not np.array_equal(orc.select(qp, k, delta)[0], orc.select(qp, k)[0])
    assert differs


def test_refinement_unit_delta_and_score_invariance():
    rng = np.random.default_rng(1)
    qp = rng.standard_normal((4, D))
    for k in (52, 77, 103, 128):
        a, e_a = orc.select(qp, k)
        b, e_b = orc.select(qp, k, np.ones(D))
        assert np.array_equal(a, b) and np.array_equal(e_a, e_b)
    # folded transforms keep every score: (q A0 D)(K B0 D^{-1})^T = q K^T
    w = wl.workload("llama8b_b8_32k", refine=True)
    A, Ai = wl.make_transforms(w)
    A0, Ai0 = wl.make_transform(w.seed, 3)
    delta = wl.make_deltas(w)[3]
    assert delta[0] == 1.0 and np.all(delta > 0)
    assert abs(np.exp(np.log(delta[1:]).mean()) - 1.0) < 1e-12
    assert np.abs(A[3] - A0 / delta[None, :]).max() == 0.0
    q = rng.standard_normal((4, D))
    K = rng.standard_normal((64, D))
    want = q @ K.T
    got = orc.transform(q, Ai[3]) @ orc.transform(K, A[3]).T
    assert np.abs(got - want).max() < 1e-10 * np.abs(want).max()
