"""The seeded input generator (workloads.py): the recipe the design states,
checked on the CPU.

* per-(sequence, head) streams: a unit regenerated alone equals its slice of
  the batch draw, and draws are reproducible;
* the outlier channels and scale, the bf16 rounding (nearest, ties to even,
  against a slow reference), the transform pair A (A^{-T})^T = I;
* the diagonal refinement (delta_0 = 1, unit geometric mean), the value
  rotation (orthogonal) and the rotary table (cos / sin of b w theta_i).
"""
import math

import numpy as np
import pytest

from long_context_decode_dual_b200 import workloads as W


def test_units_are_their_own_streams():
    wl = W.workload("llama8b_b8_32k", batch=2, n_ctx=300)
    K, V = W.make_kv(wl)
    for b, h in ((0, 0), (1, 5)):
        k, v = W.make_kv_unit(wl, b, h, 300)
        assert np.array_equal(k, K[b, h]) and np.array_equal(v, V[b, h])
    K2, V2 = W.make_kv(wl)
    assert np.array_equal(K, K2) and np.array_equal(V, V2)
    assert not np.array_equal(W.make_q(wl, 0), W.make_q(wl, 1))
    kn, vn = W.make_step_kv(wl, 3)
    assert kn.shape == (2, 8, 1, 128) and vn.shape == (2, 8, 1, 128)


def test_outlier_channels():
    wl = W.workload("llama8b_b8_32k")
    ch = W.outlier_channels(wl, 3)
    assert len(ch) == math.ceil(0.02 * 128 - 1e-9) == 3 and np.all(np.diff(ch) > 0)
    assert list(W.outlier_channels(W.workload("single_head_4k"), 0)) == [0, 1, 2, 3]
    # the scaled channels carry the factor in the original space
    wl = W.workload("single_head_4k", n_ctx=4000)
    K, _ = W.make_kv(wl)
    k = K[0, 0].astype(np.float64)
    ratio = np.sqrt((k[:, :4] ** 2).mean()) / np.sqrt((k[:, 4:] ** 2).mean())
    assert 7.0 < ratio < 9.0


def _bf16_slow(x32: float) -> int:
    """Nearest bfloat16 (ties to even) of a float32 value, by search."""
    u = int(np.float32(x32).view(np.uint32))
    lo = u >> 16
    cands = [lo, lo + 1]
    def val(b):
        return float(np.uint32(b << 16).view(np.float32))
    x = float(np.float32(x32))
    best = min(cands, key=lambda b: (abs(val(b) - x), b & 1))
    return best


def test_bf16_rounding_is_nearest_even():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(3000).astype(np.float32),
                        np.float32([1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -1.0 - 2 ** -8, 3.0e38, 1e-40])])
    got = W.bf16_bits_from_f32(x)
    for xi, g in zip(x, got):
        assert int(g) == _bf16_slow(xi), (xi, hex(int(g)))
    # ties go to the even neighbour
    assert W.bf16_bits_from_f32(np.float32([1.0 + 2 ** -8]))[0] == 0x3F80
    assert W.bf16_bits_from_f32(np.float32([1.0 + 3 * 2 ** -8]))[0] == 0x3F82


def test_transform_pair():
    A, Ai = W.make_transform(123, 4)
    assert np.abs(A @ Ai.T - np.eye(128)).max() < 1e-12
    s = np.linalg.svd(A, compute_uv=False)
    assert s.max() / s.min() < 10.0                    # well conditioned (exp(N(0, 0.3^2)) spectrum)
    wl = W.workload("llama8b_b8_32k", refine=True)
    As, Ais = W.make_transforms(wl)
    d = W.make_deltas(wl)
    for h in (0, 7):
        assert np.abs(As[h] @ Ais[h].T - np.eye(128)).max() < 1e-12
        assert d[h][0] == 1.0 and abs(np.exp(np.log(d[h][1:]).mean()) - 1.0) < 1e-12


def test_value_rotation_and_rope_table():
    R = W.make_value_rotations(W.workload("llama8b_b8_32k", rotate_values=True))
    assert R.shape == (8, 128, 128)
    for h in range(8):
        assert np.abs(R[h] @ R[h].T - np.eye(128)).max() < 1e-13
    assert W.make_value_rotations(W.workload("llama8b_b8_32k")) is None
    t = W.rope_table(5, 2048, base=500000.0)
    assert t.shape == (5, 64, 2)
    for b, i in ((0, 0), (1, 0), (3, 17), (4, 63)):
        ang = b * 2048 * 500000.0 ** (-2.0 * i / 128)
        assert t[b, i, 0] == pytest.approx(math.cos(ang), abs=1e-15)
        assert t[b, i, 1] == pytest.approx(math.sin(ang), abs=1e-15)
    wl = W.workload("longctx_b1_128k", bucket=2048)
    assert W.n_buckets(wl) == -(-wl.capacity // 2048) and W.make_rope(wl).shape == (W.n_buckets(wl), 64, 2)
