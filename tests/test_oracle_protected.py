"""Pins for the oracle's protected BF16 tier (Dual-QK §3.3: the first 64 and
the most recent 256 tokens stay in BF16 for keys and values and use the same
query-channel mask; §3.4: all tiers share one softmax).

* slot numbers and the protected set are checked against hand-computed values;
* storing tokens one at a time (the ring overwriting old slots) leaves the same
  slots as storing them at once, and a slot holds the RNE bfloat16 of its
  token, computed here independently from float32 bit patterns;
* when every token is protected the decode equals plain pruned attention on
  the BF16 keys and values (scipy softmax);
* protected tokens never read their INT2 codes, unprotected ones always do;
* with no protected tokens the decode is the plain INT2 decode.
"""
import numpy as np
import pytest
from scipy.special import softmax

from long_context_decode_dual_b200 import workloads as wl
from oracle import oracle as orc

NS, NR = 64, 256


def _bf16_of_f32(x: np.ndarray) -> np.ndarray:
    """RNE float32 -> bfloat16, written from the bit layout (for float32 inputs
    one rounding of the exact value)."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return r.astype(np.uint16)


def _bf16_value(b: np.ndarray) -> np.ndarray:
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def test_slot_numbers_and_protected_set():
    assert [orc.protected_slot(p, NS, NR) for p in (0, 10, 63, 64, 300, 319, 320, 575, 576)] == \
        [0, 10, 63, 128, 108, 127, 128, 127, 128]
    assert orc.protected_slot(70, 64, 0) == -1
    assert orc.protected_slot(5, 0, 256) == 5
    # length 1000: protected are 0..63 and 744..999
    prot = [p for p in range(1000) if orc.is_protected(p, 1000, NS, NR)]
    assert prot == list(range(64)) + list(range(744, 1000))
    # length 200 < 64 + 256: all protected; length 0: none
    assert all(orc.is_protected(p, 200, NS, NR) for p in range(200))
    assert not orc.is_protected(0, 0, NS, NR)
    # no tier
    assert not any(orc.is_protected(p, 500, 0, 0) for p in range(500))


def _tokens(n, seed):
    rng = np.random.default_rng(seed)
    # float32-representable values, so fp64 -> bf16 equals f32 -> bf16
    Kp = rng.standard_normal((n, 128)).astype(np.float32).astype(np.float64) * 3
    V = rng.standard_normal((n, 128)).astype(np.float32).astype(np.float64)
    return Kp, V


def test_one_at_a_time_equals_at_once_and_slots_hold_bf16():
    n = 1000
    Kp, V = _tokens(n, 1)
    a, b = orc.new_slots(NS, NR), orc.new_slots(NS, NR)
    for p in range(n):
        orc.protect_store(a, NS, NR, p, Kp[p:p + 1], V[p:p + 1], p + 1)
    orc.protect_store(b, NS, NR, 0, Kp, V, n)
    assert np.array_equal(a, b)
    for p in list(range(64)) + list(range(744, 1000)):
        s = orc.protected_slot(p, NS, NR)
        assert np.array_equal(a[s, :128], _bf16_of_f32(Kp[p])), p
        assert np.array_equal(a[s, 128:], _bf16_of_f32(V[p])), p
    # chunks that straddle the window edge store the same
    c = orc.new_slots(NS, NR)
    pos = 0
    for step in (100, 500, 150, 250):
        orc.protect_store(c, NS, NR, pos, Kp[pos:pos + step], V[pos:pos + step], pos + step)
        pos += step
    assert np.array_equal(c, b)


def _unit_with_tier(n, seed, n_sink=NS, n_recent=NR, bits=2, capacity=None):
    Kp, V = _tokens(n, seed)
    cap = capacity or ((n + 127) // 128) * 128
    unit = orc.new_unit(cap, bits)
    orc.append_unit(unit, bits, 0, Kp, V)
    slots = orc.new_slots(n_sink, n_recent)
    orc.protect_store(slots, n_sink, n_recent, 0, Kp, V, n)
    return unit, slots, Kp, V


@pytest.mark.parametrize("n", [1, 57, 200, 320])
def test_all_protected_is_pruned_attention_on_bf16(n):
    unit, slots, Kp, V = _unit_with_tier(n, 2)
    rng = np.random.default_rng(3)
    qp = rng.standard_normal((4, 128))
    out, idx = orc.decode_unit_protected(unit, slots, 2, n, qp, 0.4, NS, NR)
    Kb = _bf16_value(_bf16_of_f32(Kp))
    Vb = _bf16_value(_bf16_of_f32(V))
    s = qp[:, idx] @ Kb[:, idx].T / np.sqrt(128)
    np.testing.assert_allclose(out, softmax(s, axis=1) @ Vb, rtol=1e-11, atol=1e-12)


def test_protected_tokens_ignore_codes_and_middle_tokens_use_them():
    n = 900
    unit, slots, Kp, V = _unit_with_tier(n, 4)
    qp = np.random.default_rng(5).standard_normal((4, 128))
    ref, _ = orc.decode_unit_protected(unit, slots, 2, n, qp, 0.4, NS, NR)
    # wipe the codes and metadata of two protected tokens (5 and 880): no change
    bad = unit.copy()
    for p in (5, 880):
        K2, V2 = _tokens(1, 99)
        orc.append_unit(bad, 2, p, K2 * 7, V2 * 7)
    out, _ = orc.decode_unit_protected(bad, slots, 2, n, qp, 0.4, NS, NR)
    assert np.array_equal(out, ref)
    # change a middle (unprotected) token's codes: the output moves
    K2, V2 = _tokens(1, 98)
    orc.append_unit(bad, 2, 300, K2 * 7, V2 * 7)
    out, _ = orc.decode_unit_protected(bad, slots, 2, n, qp, 0.4, NS, NR)
    assert not np.allclose(out, ref)
    # change a protected token's slot: the output moves
    s2 = slots.copy()
    s2[orc.protected_slot(880, NS, NR), 128:] = _bf16_of_f32(np.full(128, 5.0))
    out, _ = orc.decode_unit_protected(unit, s2, 2, n, qp, 0.4, NS, NR)
    assert not np.allclose(out, ref)


@pytest.mark.parametrize("n_sink,n_recent", [(0, 0), (64, 0), (0, 256), (16, 40)])
def test_other_tiers(n_sink, n_recent):
    n = 700
    unit, slots, Kp, V = _unit_with_tier(n, 6, n_sink, n_recent)
    qp = np.random.default_rng(7).standard_normal((2, 128))
    out, idx = orc.decode_unit_protected(unit, slots, 2, n, qp, 0.2, n_sink, n_recent)
    Kh, Vh = orc.dequant_unit(unit, 2, n)
    Kb = _bf16_value(_bf16_of_f32(Kp))
    Vb = _bf16_value(_bf16_of_f32(V))
    for p in range(n):
        if p < n_sink or p >= n - n_recent:
            Kh[p], Vh[p] = Kb[p], Vb[p]
    s = qp[:, idx] @ Kh[:, idx].T / np.sqrt(128)
    np.testing.assert_allclose(out, softmax(s, axis=1) @ Vh, rtol=1e-11, atol=1e-12)
    if n_sink == n_recent == 0:
        plain, _ = orc.decode_unit(unit, 2, n, qp, 0.2)
        assert np.array_equal(out, plain)
