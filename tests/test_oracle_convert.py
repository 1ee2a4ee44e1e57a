"""Pins for the oracle's binary64 -> binary16 / bfloat16 rounding.

The definition: the nearest representable value, ties to the one with an even
last mantissa bit, overflow to infinity past the largest finite value's
rounding threshold (IEEE-754 §4.3.1, roundTiesToEven).  Checked against
numpy's float16 conversion, torch's bfloat16 decoding and a brute-force
nearest-value search with exact rational distances.
"""
import bisect
from fractions import Fraction

import numpy as np
import pytest
import torch

from oracle import oracle as orc


def _all_f16_values():
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    vals = bits.view(np.float16).astype(np.float64)
    return bits, vals


def test_f16_decode_matches_numpy():
    bits, vals = _all_f16_values()
    for b in list(range(0, 65536, 97)) + [0x0001, 0x03FF, 0x0400, 0x7BFF, 0x7C00, 0xFC00, 0x8001]:
        got = orc.f16_value(b)
        assert got == vals[b] or (np.isnan(got) and np.isnan(vals[b])), hex(b)


def test_bf16_decode_matches_torch():
    bits = torch.arange(0, 1 << 16, 31, dtype=torch.int32).to(torch.int16)
    ref = bits.view(torch.bfloat16).double().numpy()
    for b, r in zip(bits.numpy().astype(np.uint16), ref):
        got = orc.bf16_value(int(b))
        assert got == r or (np.isnan(got) and np.isnan(r)), hex(int(b))


def test_f16_roundtrip_all_finite():
    bits, vals = _all_f16_values()
    finite = np.isfinite(vals)
    out = orc.f16_rne(vals[finite])
    assert np.array_equal(out, bits[finite])


def test_f16_matches_numpy_random_and_midpoints():
    rng = np.random.default_rng(7)
    x = np.concatenate([
        rng.standard_normal(20000) * 10.0 ** rng.integers(-9, 6, 20000),
        rng.uniform(65000, 66000, 2000), -rng.uniform(65000, 66000, 2000),
        rng.uniform(0, 2 ** -13, 2000),
    ])
    _, vals = _all_f16_values()
    pos = np.unique(vals[np.isfinite(vals) & (vals >= 0)])
    mids = (pos[:-1] + pos[1:]) / 2.0                  # exact in binary64
    near = np.concatenate([mids, np.nextafter(mids, np.inf), np.nextafter(mids, -np.inf)])
    x = np.concatenate([x, near, -near, [65504.0, 65519.99, 65520.0, 1e300, -1e300, 2 ** -25,
                                         2 ** -25 * 1.0000001, 2 ** -24 * 1.5, 0.0, -0.0]])
    with np.errstate(over="ignore"):                  # values past the fp16 range round to inf on purpose
        ref = x.astype(np.float16).view(np.uint16)
    got = orc.f16_rne(x)
    bad = np.nonzero(got != ref)[0]
    assert bad.size == 0, [(x[i], hex(got[i]), hex(ref[i])) for i in bad[:5]]


def _bf16_grid():
    bits = torch.arange(0, 1 << 16, dtype=torch.int32).to(torch.int16)
    vals = bits.view(torch.bfloat16).double().numpy()
    b = bits.numpy().astype(np.uint16)
    ok = np.isfinite(vals) & (vals >= 0) & ~((vals == 0) & (b != 0))
    order = np.argsort(vals[ok], kind="stable")
    return vals[ok][order], b[ok][order]


def _bf16_bruteforce(x: float, grid_vals, grid_bits) -> int:
    """Nearest bf16 by exact distance; ties to even mantissa; beyond the
    largest finite value's rounding threshold -> infinity."""
    sign = 0x8000 if np.signbit(x) else 0
    a = abs(x)
    vmax = grid_vals[-1]
    ulp_top = Fraction(2) ** (127 - 7)
    if Fraction(a) >= Fraction(vmax) + ulp_top / 2:
        return sign | 0x7F80
    i = bisect.bisect_left(grid_vals, a)
    cands = [j for j in (i - 1, i) if 0 <= j < len(grid_vals)]
    best = None
    for j in cands:
        dist = abs(Fraction(a) - Fraction(grid_vals[j]))
        key = (dist, int(grid_bits[j]) & 1)
        if best is None or key < best[0]:
            best = (key, int(grid_bits[j]))
    return sign | best[1]


def test_bf16_matches_bruteforce():
    gv, gb = _bf16_grid()
    rng = np.random.default_rng(11)
    xs = list(rng.standard_normal(3000) * 10.0 ** rng.integers(-40, 38, 3000))
    # midpoints between neighbours and values a hair off them (these are the
    # cases that go wrong when a value is rounded through float32 first)
    for j in rng.integers(0, len(gv) - 1, 600):
        m = (gv[j] + gv[j + 1]) / 2.0
        xs += [m, np.nextafter(m, np.inf), np.nextafter(m, -np.inf),
               m + m * 2.0 ** -30, m - m * 2.0 ** -30]
    xs += [3.3895313892515355e38, 3.40e38, 3.3961e38, 1e-45, 9.2e-41, 2.0 ** -133,
           2.0 ** -134, 2.0 ** -134 * 1.0000001, 5e-324, -0.0]
    xs = np.array(xs, dtype=np.float64)
    got = orc.bf16_rne(xs)
    for x, g in zip(xs, got):
        assert int(g) == _bf16_bruteforce(float(x), gv, gb), (x, hex(int(g)))


def test_double_rounding_trap_bf16():
    # 1 + 2^-8 is the midpoint between bf16 1.0 and 1.0078125; a value just
    # above it must round up even though float32 would first round it back
    # down onto the midpoint.
    x = 1.0 + 2.0 ** -8 + 2.0 ** -40
    assert orc.bf16_rne(np.array([x]))[0] == 0x3F81
    assert orc.bf16_rne(np.array([1.0 + 2.0 ** -8]))[0] == 0x3F80      # tie -> even
    assert orc.bf16_rne(np.array([1.0 + 3 * 2.0 ** -8]))[0] == 0x3F82  # tie -> even


@pytest.mark.parametrize("x,bits", [(float("nan"), 0x7E00), (float("inf"), 0x7C00),
                                    (-float("inf"), 0xFC00)])
def test_f16_specials(x, bits):
    assert orc.f16_rne(np.array([x]))[0] == bits
