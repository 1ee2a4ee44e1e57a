"""numpy front end of the fp64 CPU oracle (``kvq_oracle.c``).

TEST INFRASTRUCTURE ONLY: imported by the test suite, the package smoke check
and the CPU-baseline leg of the benchmark; never by the product path.  It
shares no code with the CUDA library.

Each function states the passage of "Dual-QK: Sharp Queries and Flat Keys for
Prunable 2-bit KV Caches" it follows; the C file's header has the full list.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "kvq_oracle.c")
LIB = os.path.join(HERE, "libkvq_oracle.so")
D = 128
T = 128
GROUP = 32

_lock = threading.Lock()
_lib = None

CFLAGS = ["-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared"]


def build(force: bool = False) -> str:
    """Compile the oracle into a shared library next to its source."""
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(SRC):
        tmp = LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *CFLAGS, SRC, "-o", tmp, "-lm"])
        os.replace(tmp, LIB)
    return LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(LIB)
            P = ctypes.c_void_p
            L = ctypes.c_long
            I = ctypes.c_int
            lib.orc_f16_rne.restype = ctypes.c_uint16
            lib.orc_f16_rne.argtypes = [ctypes.c_double]
            lib.orc_bf16_rne.restype = ctypes.c_uint16
            lib.orc_bf16_rne.argtypes = [ctypes.c_double]
            lib.orc_f16_to_f64.restype = ctypes.c_double
            lib.orc_f16_to_f64.argtypes = [ctypes.c_uint16]
            lib.orc_bf16_to_f64.restype = ctypes.c_double
            lib.orc_bf16_to_f64.argtypes = [ctypes.c_uint16]
            lib.orc_f16_rne_array.argtypes = [P, L, P]
            lib.orc_bf16_rne_array.argtypes = [P, L, P]
            lib.orc_transform.argtypes = [P, P, L, I, P]
            lib.orc_quantize_group.argtypes = [P, I, I, P, P, P]
            lib.orc_quantize_group_clip.argtypes = [P, I, I, ctypes.c_double, P, P, P]
            lib.orc_page_bytes.restype = L
            lib.orc_page_bytes.argtypes = [I]
            lib.orc_append_unit.argtypes = [P, I, L, L, P, P]
            lib.orc_dequant_unit.argtypes = [P, I, L, P, P]
            lib.orc_page_bytes_g.restype = L
            lib.orc_page_bytes_g.argtypes = [I, I]
            lib.orc_append_unit_g.argtypes = [P, I, I, L, L, P, P]
            lib.orc_append_unit_c.argtypes = [P, I, I, ctypes.c_double, L, L, P, P]
            lib.orc_dequant_unit_g.argtypes = [P, I, I, L, P, P]
            lib.orc_num_selected.restype = I
            lib.orc_num_selected.argtypes = [ctypes.c_float, I]
            lib.orc_select.argtypes = [P, I, I, I, P, P]
            lib.orc_select_scaled.argtypes = [P, I, I, I, P, P, P]
            lib.orc_decode_dense.argtypes = [P, P, L, P, I, I, P, I, P]
            lib.orc_attention.argtypes = [P, P, P, L, I, I, P]
            lib.orc_protected_slot.restype = L
            lib.orc_protected_slot.argtypes = [L, I, I]
            lib.orc_is_protected.restype = I
            lib.orc_is_protected.argtypes = [L, L, I, I]
            lib.orc_protect_store.argtypes = [P, I, I, L, L, L, P, P]
            lib.orc_protect_dequant.argtypes = [P, I, I, L, P, P]
            lib.orc_rope_unanchor.argtypes = [P, L, I, P, P]
            lib.orc_decode_buckets.argtypes = [P, P, L, P, I, I, P, I, L, P]
            _lib = lib
    return _lib


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float64)


# ------------------------------------------------------------- conversions
def f16_rne(x) -> np.ndarray:
    """binary64 -> binary16 bits, one rounding to nearest even."""
    x = _f64(x)
    out = np.empty(x.shape, dtype=np.uint16)
    _load().orc_f16_rne_array(_p(x), x.size, _p(out))
    return out


def bf16_rne(x) -> np.ndarray:
    """binary64 -> bfloat16 bits, one rounding to nearest even."""
    x = _f64(x)
    out = np.empty(x.shape, dtype=np.uint16)
    _load().orc_bf16_rne_array(_p(x), x.size, _p(out))
    return out


def f16_value(bits: int) -> float:
    return _load().orc_f16_to_f64(int(bits))


def bf16_value(bits: int) -> float:
    return _load().orc_bf16_to_f64(int(bits))


# --------------------------------------------------------------- transform
def transform(X, M) -> np.ndarray:
    """Rows of X times M (Dual-QK §3.1): fixed-order fma chain over channels."""
    X = _f64(X)
    M = _f64(M)
    d = M.shape[0]
    assert M.shape == (d, d) and X.shape[-1] == d
    Y = np.empty_like(X)
    _load().orc_transform(_p(X), _p(M), X.size // d, d, _p(Y))
    return Y


# --------------------------------------------------------------- quantizer
def quantize_group(x, bits: int = 2, clip: float = 1.0):
    """One (token, group) of the asymmetric min/max quantizer (Dual-QK §3.3);
    with clip < 1 the grid spans [clip*min, clip*max] (App. B.2: values use a
    clipping ratio of 0.92).

    Returns (scale fp16 bits, zero fp16 bits, codes uint8[len]).
    """
    x = _f64(x)
    s = np.zeros(1, np.uint16)
    z = np.zeros(1, np.uint16)
    c = np.zeros(x.size, np.uint8)
    _load().orc_quantize_group_clip(_p(x), x.size, (1 << bits) - 1, float(clip), _p(s), _p(z), _p(c))
    return int(s[0]), int(z[0]), c


def page_bytes(bits: int, group: int = GROUP) -> int:
    return int(_load().orc_page_bytes_g(bits, group))


def new_unit(capacity: int, bits: int, group: int = GROUP) -> np.ndarray:
    """Zeroed pages of one (batch, KV head): uint8 [capacity/128][page bytes]."""
    assert capacity % T == 0
    return np.zeros((capacity // T, page_bytes(bits, group)), dtype=np.uint8)


def append_unit(unit: np.ndarray, bits: int, pos0: int, Kp, V, group: int = GROUP, vclip: float = 1.0) -> None:
    """Quantize and store tokens pos0.. of one unit (K' already transformed, V
    already rotated where the values are rotated); groups of `group` channels
    (32, or 128: one grid per token); value grids clipped by vclip."""
    Kp = _f64(Kp).reshape(-1, D)
    V = _f64(V).reshape(-1, D)
    assert Kp.shape == V.shape
    assert unit.flags.c_contiguous and unit.dtype == np.uint8
    assert (pos0 + Kp.shape[0]) <= unit.shape[0] * T
    assert unit.shape[1] == page_bytes(bits, group)
    _load().orc_append_unit_c(_p(unit), bits, group, float(vclip), pos0, Kp.shape[0], _p(Kp), _p(V))


def dequant_unit(unit: np.ndarray, bits: int, n: int, group: int = GROUP):
    """Dequantized K' and V of tokens 0..n-1: float64 [n][128] each."""
    Kh = np.zeros((max(n, 0), D))
    Vh = np.zeros((max(n, 0), D))
    _load().orc_dequant_unit_g(_p(np.ascontiguousarray(unit)), bits, group, n, _p(Kh), _p(Vh))
    return Kh, Vh


# --------------------------------------------------------------- selection
def num_selected(sparsity: float, d: int = D) -> int:
    return int(_load().orc_num_selected(float(sparsity), d))


def select(qp, k: int, delta=None):
    """Channel 0 plus the top k-1 channels by pooled energy (Dual-QK Eq. 4).

    qp: [g][d] transformed queries of one GQA group.  delta: the diagonal
    refinement D folded into the query transform (§3.3), or None; selection
    then uses the base queries qp / delta (App. C.2).  Returns (idx int32[k]
    ascending, e2 float64[d]).
    """
    qp = _f64(qp)
    g, d = qp.shape
    assert 1 <= k <= d
    e2 = np.zeros(d)
    idx = np.zeros(k, np.int32)
    if delta is None:
        _load().orc_select(_p(qp), g, d, k, _p(e2), _p(idx))
    else:
        delta = _f64(delta)
        assert delta.shape == (d,) and np.all(delta > 0)
        _load().orc_select_scaled(_p(qp), g, d, k, _p(delta), _p(e2), _p(idx))
    return idx, e2


# --------------------------------------------------------------- attention
def decode_dense(Khat, Vhat, qp, idx) -> np.ndarray:
    """Softmax attention over retained channels idx, 1/sqrt(d) scaling."""
    Khat = _f64(Khat)
    Vhat = _f64(Vhat)
    qp = _f64(qp)
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    g, d = qp.shape
    n = Khat.shape[0]
    out = np.zeros((g, d))
    _load().orc_decode_dense(_p(Khat), _p(Vhat), n, _p(qp), g, d, _p(idx), idx.size, _p(out))
    return out


def attention(q, K, V) -> np.ndarray:
    """Plain softmax(q K^T / sqrt(d)) V."""
    q = _f64(q)
    K = _f64(K)
    V = _f64(V)
    g, d = q.shape
    out = np.zeros((g, d))
    _load().orc_attention(_p(q), _p(K), _p(V), K.shape[0], g, d, _p(out))
    return out


# ----------------------------------------------------------- value rotation
def value_rotate(V, Rv) -> np.ndarray:
    """Values in the rotated basis, V Rv (Dual-QK §3.3, App. B.2: the value
    rotation precedes quantization); the fma chain of ``transform``."""
    return transform(V, Rv)


def value_unrotate(o, Rv) -> np.ndarray:
    """Aggregated output back in the original basis, o Rv^T (§3.3: the value
    rotation is reversed after aggregation; Rv is orthogonal)."""
    return transform(o, np.ascontiguousarray(_f64(Rv).T))


# ------------------------------------------------------ whole decode step
def decode_unit(unit: np.ndarray, bits: int, n: int, qp, sparsity: float, group: int = GROUP,
                delta=None, Rv=None):
    """Select channels for one GQA group and attend over n cached tokens;
    with delta, selection on the base queries; with Rv, the output is rotated
    back (the cache then holds rotated values).

    Returns (out [g][d] float64, idx int32[k]).
    """
    k = num_selected(sparsity)
    idx, _ = select(qp, k, delta)
    Kh, Vh = dequant_unit(unit, bits, n, group)
    out = decode_dense(Kh, Vh, qp, idx)
    return (out if Rv is None else value_unrotate(out, Rv)), idx


# ------------------------------------------------------ protected BF16 tier
def protected_slot(pos: int, n_sink: int, n_recent: int) -> int:
    """Slot of a position in the protected tier (Dual-QK §3.3), -1 if none."""
    return int(_load().orc_protected_slot(pos, n_sink, n_recent))


def is_protected(pos: int, length: int, n_sink: int, n_recent: int) -> bool:
    return bool(_load().orc_is_protected(pos, length, n_sink, n_recent))


def new_slots(n_sink: int, n_recent: int) -> np.ndarray:
    """Zeroed protected slots of one unit: uint16 [n_sink + n_recent][256]
    (128 BF16 key values, then 128 BF16 value values)."""
    return np.zeros((n_sink + n_recent, 2 * D), dtype=np.uint16)


def protect_store(slots: np.ndarray, n_sink: int, n_recent: int, pos0: int, Kp, V, len_after: int) -> None:
    """Store the BF16 copies of tokens pos0.. that belong to the protected
    tier of a sequence of length len_after."""
    Kp = _f64(Kp).reshape(-1, D)
    V = _f64(V).reshape(-1, D)
    assert slots.flags.c_contiguous and slots.dtype == np.uint16
    assert slots.shape == (n_sink + n_recent, 2 * D)
    _load().orc_protect_store(_p(slots), n_sink, n_recent, pos0, Kp.shape[0], len_after, _p(Kp), _p(V))


def decode_unit_protected(unit: np.ndarray, slots: np.ndarray, bits: int, n: int, qp, sparsity: float,
                          n_sink: int, n_recent: int, group: int = GROUP, delta=None, Rv=None):
    """decode_unit with the protected tier: the first n_sink and the last
    n_recent tokens are read from their BF16 slots, the rest from the INT2
    codes; one softmax over all of them, then (with Rv) the inverse value
    rotation (Dual-QK §3.3, §3.4)."""
    k = num_selected(sparsity)
    idx, _ = select(qp, k, delta)
    Kh, Vh = dequant_unit(unit, bits, n, group)
    _load().orc_protect_dequant(_p(np.ascontiguousarray(slots)), n_sink, n_recent, n, _p(Kh), _p(Vh))
    out = decode_dense(Kh, Vh, qp, idx)
    return (out if Rv is None else value_unrotate(out, Rv)), idx


# ------------------------------------------------------ bucket-relative RoPE
def rope_unanchor(X, cs) -> np.ndarray:
    """Rows of post-RoPE vectors moved into the frame of a bucket anchor
    (Dual-QK §3.4, App. C.4): channel pairs (i, i + 64) rotated by -a*theta_i,
    cs [64][2] = (cos, sin) of a*theta_i."""
    X = _f64(X)
    cs = _f64(cs)
    d = X.shape[-1]
    assert cs.shape == (d // 2, 2)
    Y = np.empty_like(X)
    _load().orc_rope_unanchor(_p(X), X.size // d, d, _p(cs), _p(Y))
    return Y


def bucket_queries(q, Ai, rope, n_buckets: int) -> np.ndarray:
    """q'_b = (q T_b) A^{-T} for buckets 0..n_buckets-1: [nb][g][d]."""
    return np.stack([transform(rope_unanchor(q, rope[b]), Ai) for b in range(n_buckets)])


def bucket_keys(K, A, rope, w: int, pos0: int = 0) -> np.ndarray:
    """K' of tokens pos0.. in their buckets' frames, z_n = (k_n T_b) A with
    b = n // w (§3.4)."""
    K = _f64(K).reshape(-1, D)
    out = np.empty_like(K)
    i = 0
    while i < K.shape[0]:                       # the tokens of one bucket at a time
        b = (pos0 + i) // w
        j = min(K.shape[0], (b + 1) * w - pos0)
        out[i:j] = transform(rope_unanchor(K[i:j], rope[b]), A)
        i = j
    return out


def decode_buckets(Khat, Vhat, qpb, idxb, w: int) -> np.ndarray:
    """One softmax over all tokens; token t scored with bucket t // w's
    queries qpb [nb][g][d] over its channel list idxb [nb][k]."""
    Khat = _f64(Khat)
    Vhat = _f64(Vhat)
    qpb = _f64(qpb)
    idxb = np.ascontiguousarray(idxb, dtype=np.int32)
    nb, g, d = qpb.shape
    n = Khat.shape[0]
    assert (n + w - 1) // w <= nb and idxb.shape[0] == nb
    out = np.zeros((g, d))
    _load().orc_decode_buckets(_p(Khat), _p(Vhat), n, _p(qpb), g, d, _p(idxb), idxb.shape[1], w, _p(out))
    return out


def decode_unit_buckets(unit: np.ndarray, bits: int, n: int, qpb, sparsity: float, w: int, group: int = GROUP,
                        delta=None, Rv=None, slots=None, n_sink: int = 0, n_recent: int = 0):
    """Decode with bucket-relative RoPE (§3.4): per bucket b < ceil(n / w),
    the channel choice on that bucket's queries qpb[b] (base queries with
    delta), then one softmax over every token with its bucket's queries and
    channels, the protected tier's BF16 rows in place of their codes, and
    (with Rv) the inverse value rotation.  Returns (out [g][d], idx [nb][k])
    for the buckets in use."""
    k = num_selected(sparsity)
    nb = max(1, (n + w - 1) // w)
    qpb = _f64(qpb)[:nb]
    idxb = np.stack([select(qpb[b], k, delta)[0] for b in range(nb)])
    Kh, Vh = dequant_unit(unit, bits, n, group)
    if slots is not None and n_sink + n_recent > 0:
        _load().orc_protect_dequant(_p(np.ascontiguousarray(slots)), n_sink, n_recent, n, _p(Kh), _p(Vh))
    out = decode_buckets(Kh, Vh, qpb, idxb, w)
    return (out if Rv is None else value_unrotate(out, Rv)), idxb
