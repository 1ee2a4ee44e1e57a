"""Pins for the oracle's quantizer and page layout (Dual-QK §3.3).

* hand-computed groups (including round-half-even ties and a zero range);
* brute force: every code is the nearest grid level (after clamping);
* exact round trip: re-quantizing dequantized values reproduces the codes,
  scale and zero bit patterns;
* error bound |x - x_hat| <= s/2 + |z - min|;
* page layout: bytes of a hand-built token at a hand-computed offset.
"""
import numpy as np
import pytest

from oracle import oracle as orc

F16_ONE = 0x3C00


def test_hand_groups():
    s, z, c = orc.quantize_group([0.0, 1.0, 2.0, 3.0])
    assert (s, z) == (F16_ONE, 0) and list(c) == [0, 1, 2, 3]
    # ties go to even: 0.5 -> 0, 1.5 -> 2, 2.5 -> 2
    s, z, c = orc.quantize_group([0.0, 0.5, 1.5, 2.5, 3.0])
    assert (s, z) == (F16_ONE, 0) and list(c) == [0, 0, 2, 2, 3]
    s, z, c = orc.quantize_group([-1.0, 0.5, 2.0])
    assert orc.f16_value(z) == -1.0 and orc.f16_value(s) == 1.0 and list(c) == [0, 2, 3]
    # zero range: scale 0, all codes 0, zero-point carries the value
    s, z, c = orc.quantize_group([0.3] * 8)
    assert s == 0 and list(c) == [0] * 8 and z == orc.f16_rne(np.array([0.3]))[0]
    # INT4: 16 levels
    s, z, c = orc.quantize_group(np.arange(16.0), bits=4)
    assert (s, z) == (F16_ONE, 0) and list(c) == list(range(16))


@pytest.mark.parametrize("bits", [2, 4])
def test_nearest_level_and_bound(bits):
    rng = np.random.default_rng(1)
    L = (1 << bits) - 1
    for _ in range(300):
        n = int(rng.integers(2, 33))
        x = rng.standard_normal(n) * rng.uniform(0.01, 50)
        s16, z16, c = orc.quantize_group(x, bits)
        s, z = orc.f16_value(s16), orc.f16_value(z16)
        levels = z + s * np.arange(L + 1)
        err = np.abs(x[:, None] - levels[None, :])
        chosen = err[np.arange(n), c]
        assert np.all(chosen <= err.min(axis=1) + 1e-12 * s)
        assert np.all(np.abs(x - (z + s * c)) <= s / 2 + abs(z - x.min()) + 1e-12)
        assert s == pytest.approx((x.max() - x.min()) / L, rel=2 ** -10)


@pytest.mark.parametrize("bits", [2, 4])
def test_exact_roundtrip(bits):
    rng = np.random.default_rng(2)
    for _ in range(300):
        x = rng.standard_normal(32) * rng.uniform(0.1, 20)
        s16, z16, c = orc.quantize_group(x, bits)
        xh = orc.f16_value(z16) + orc.f16_value(s16) * c.astype(np.float64)
        s2, z2, c2 = orc.quantize_group(xh, bits)
        assert (s2, z2) == (s16, z16)
        assert np.array_equal(c2, c)


def _u16(buf, off):
    return int(buf[off]) | (int(buf[off + 1]) << 8)


def _token(c_mod):
    k = np.array([1.5] + [float(c % 4) for c in range(1, 128)])
    v = np.array([float(3 - (c % 4)) for c in range(128)])
    return k, v


@pytest.mark.parametrize("bits", [2, 4])
def test_page_layout_hand_computed(bits):
    R = 128 * bits // 8
    pb = orc.page_bytes(bits)
    assert pb == 256 * R + 256 + 4096
    unit = orc.new_unit(256, bits)
    k, v = _token(0)
    pos = 130                                  # page 1, token 2
    orc.append_unit(unit, bits, pos, k[None], v[None])
    pg = unit[1]
    t = 2
    per = 8 // bits
    step = 1 if bits == 2 else 5               # values 0..3 on a 4- or 16-level grid
    for c in range(1, 128):
        byte = pg[c * R + t // per]
        assert (byte >> ((t % per) * bits)) & ((1 << bits) - 1) == step * (c % 4), c
    for c in range(128):
        byte = pg[128 * R + c * R + t // per]
        assert (byte >> ((t % per) * bits)) & ((1 << bits) - 1) == step * (3 - c % 4), c
    # channel 0 in bf16 (1.5 = 0x3FC0), little-endian
    assert pg[256 * R + 2 * t] == 0xC0 and pg[256 * R + 2 * t + 1] == 0x3F
    kmeta = 256 * R + 256
    vmeta = kmeta + 2048
    levels = (1 << bits) - 1
    s_exp = orc.f16_rne(np.array([3.0 / levels]))[0]
    for g in range(4):
        # token 2 is in chunk 0 of block 0: permuted chunk 0 ^ (0 ^ 4 (g % 2))
        chunk = 0 ^ (4 if g % 2 else 0)
        off = 4 * (128 * g + 4 * chunk + t % 4)
        assert _u16(pg, kmeta + off) == s_exp
        assert _u16(pg, kmeta + off + 2) == 0
        assert _u16(pg, vmeta + off) == s_exp
    # a token in block 3 of the chunks (t = 101: chunk 25, 25 ^ (3 ^ 4) = 30 in odd groups)
    unit2 = orc.new_unit(128, bits)
    orc.append_unit(unit2, bits, 101, k[None], v[None])
    assert _u16(unit2[0], kmeta + 4 * (128 * 1 + 4 * 30 + 1)) == s_exp
    assert _u16(unit2[0], kmeta + 4 * (128 * 2 + 4 * (25 ^ 3) + 1)) == s_exp
    # everything else stays zero; the other page untouched
    assert not unit[0].any()
    # row 0 of the key codes is never written
    assert not pg[:R].any()


@pytest.mark.parametrize("bits", [2, 4])
def test_append_dequant_consistent(bits):
    """Tokens stored one by one or all at once give the same pages, and the
    dequantized values are the per-group s*code + z of the quantizer."""
    rng = np.random.default_rng(8)
    n = 300
    K = rng.standard_normal((n, 128))
    V = rng.standard_normal((n, 128))
    u1 = orc.new_unit(384, bits)
    orc.append_unit(u1, bits, 0, K, V)
    u2 = orc.new_unit(384, bits)
    for i in range(0, n, 7):
        orc.append_unit(u2, bits, i, K[i:i + 7], V[i:i + 7])
    assert np.array_equal(u1, u2)
    Kh, Vh = orc.dequant_unit(u1, bits, n)
    for t in (0, 1, 127, 128, 299):
        s, z, c = orc.quantize_group(K[t, 1:32], bits)
        np.testing.assert_array_equal(Kh[t, 1:32], orc.f16_value(s) * c + orc.f16_value(z))
        s, z, c = orc.quantize_group(V[t, 96:128], bits)
        np.testing.assert_array_equal(Vh[t, 96:128], orc.f16_value(s) * c + orc.f16_value(z))
        assert Kh[t, 0] == orc.bf16_value(orc.bf16_rne(np.array([K[t, 0]]))[0])


@pytest.mark.parametrize("bits", [2, 4])
def test_one_grid_per_token_layout_hand_computed(bits):
    """The pages' own format (§3.3: one asymmetric grid per token and KV head
    over key channels 1..127; values over channels 0..127): one metadata word
    per token, at the permuted chunk of group 0."""
    R = 128 * bits // 8
    pb = orc.page_bytes(bits, 128)
    assert pb == 256 * R + 256 + 1024
    unit = orc.new_unit(256, bits, 128)
    # keys: channel c (1..127) holds c % 4 -> range [0, 3] over the whole row
    k, v = _token(0)
    k[127] = 6.0                               # one outlier widens the single grid
    pos = 128 + 77                             # page 1, token 77 (chunk 19 -> 19 ^ 2 = 17)
    orc.append_unit(unit, bits, pos, k[None], v[None], group=128)
    pg = unit[1]
    t = 77
    per = 8 // bits
    levels = (1 << bits) - 1
    kmeta = 256 * R + 256
    vmeta = kmeta + 512
    off = 4 * (4 * 17 + t % 4)
    s_k = orc.f16_rne(np.array([6.0 / levels]))[0]
    assert _u16(pg, kmeta + off) == s_k and _u16(pg, kmeta + off + 2) == 0
    s_v = orc.f16_rne(np.array([3.0 / levels]))[0]
    assert _u16(pg, vmeta + off) == s_v and _u16(pg, vmeta + off + 2) == 0
    # key codes on the 6/levels grid: value x -> rint(x * levels / 6)
    sk = orc.f16_value(s_k)
    for c in range(1, 128):
        byte = pg[c * R + t // per]
        code = (byte >> ((t % per) * bits)) & levels
        assert code == min(levels, int(np.rint(k[c] / sk))), c
    for c in range(128):
        byte = pg[128 * R + c * R + t // per]
        assert (byte >> ((t % per) * bits)) & levels == (1 if bits == 2 else 5) * (3 - c % 4), c
    assert pg[256 * R + 2 * t] == 0xC0 and pg[256 * R + 2 * t + 1] == 0x3F
    assert not unit[0].any() and not pg[:R].any()


@pytest.mark.parametrize("bits", [2, 4])
def test_one_grid_per_token_dequant(bits):
    rng = np.random.default_rng(9)
    n = 260
    K = rng.standard_normal((n, 128))
    V = rng.standard_normal((n, 128))
    u = orc.new_unit(384, bits, 128)
    orc.append_unit(u, bits, 0, K, V, group=128)
    u2 = orc.new_unit(384, bits, 128)
    for i in range(0, n, 9):
        orc.append_unit(u2, bits, i, K[i:i + 9], V[i:i + 9], group=128)
    assert np.array_equal(u, u2)
    Kh, Vh = orc.dequant_unit(u, bits, n, group=128)
    for t in (0, 5, 128, 259):
        s, z, c = orc.quantize_group(K[t, 1:], bits)
        np.testing.assert_array_equal(Kh[t, 1:], orc.f16_value(s) * c + orc.f16_value(z))
        s, z, c = orc.quantize_group(V[t], bits)
        np.testing.assert_array_equal(Vh[t], orc.f16_value(s) * c + orc.f16_value(z))
    np.testing.assert_array_equal(Kh[:, 0], [orc.bf16_value(int(b)) for b in orc.bf16_rne(K[:, 0])])
