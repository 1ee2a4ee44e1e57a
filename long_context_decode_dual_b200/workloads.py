"""Seeded synthetic inputs for the prunable 2-bit KV decode path.

This module only draws random numbers and shapes them. It holds none of the
method's arithmetic (no transform, quantizer, selection or attention), so both
the CUDA path and the CPU oracle can take their inputs from it.

Workloads follow the shapes of the Dual-QK pages ("Dual-QK: Sharp Queries and
Flat Keys for Prunable 2-bit KV Caches", §3 and §4.4): head dim 128, GQA groups
of 4 query heads per KV head, contexts up to 128K, 40% query-channel sparsity.
The pages evaluate on model activations; none exist here, so keys and values
are i.i.d. draws with a few scaled outlier channels, as listed below.

Recipe (every array comes from its own numpy PCG64 stream keyed by
``(seed, stream_id)``):

* ``A = U diag(exp(g)) W^T`` with ``U, W`` the Q factors of seeded 128x128
  Gaussian matrices (R's diagonal made positive), ``g ~ N(0, 0.3^2)``
  (0.3 read as the standard deviation).  ``A^{-T} = U diag(exp(-g)) W^T`` in
  closed form, so no side ever inverts a matrix.
* keys / values: N(0,1) (or Student-t with 4 degrees of freedom, drawn as
  z / sqrt(chi2_4 / 4)); selected key channels are multiplied by an outlier
  factor in the original (untransformed) space.
* queries: N(0,1).
* bf16 inputs are the round-to-nearest-even bf16 of float32 draws.
* diagonal refinement (optional): ``delta_0 = 1``, ``delta_j = exp(N(0, 0.3^2))``
  for j >= 1, the free scales divided by their geometric mean (the pages fit
  D offline, keep its channel-0 entry at one and normalise the free scales to
  unit geometric mean).  It is folded into the transforms as the pages do:
  key transform ``A D^{-1}``, query transform ``A^{-T} D``.
* value rotation (optional): ``Rv = Q H / sqrt(128)``, ``Q`` a seeded Haar
  orthogonal matrix standing in for the calibrated rotation and ``H`` the
  Sylvester Hadamard matrix of order 128; ``Rv`` is orthogonal.
* bucket-relative RoPE (optional): buckets of ``bucket`` tokens with anchors
  ``a_b = b * bucket``; the rotary table holds ``cos`` and ``sin`` of
  ``a_b * theta_i``, ``theta_i = base^(-2i/128)`` (base 500000, a
  Llama-3-like model's).  Keys and queries are taken as already rotated by
  the model's RoPE (the draws above).
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional, Sequence

import numpy as np

HEAD_DIM = 128
BLOCK_TOKENS = 128

# stream ids, one per drawn tensor kind
_S_A_U, _S_A_W, _S_A_G, _S_OUTLIER, _S_K, _S_V, _S_Q, _S_KNEW, _S_VNEW, _S_DELTA, _S_RV = range(11)


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic decode workload.

    ``n_ctx`` is the number of tokens already in the cache when decoding
    starts; ``n_steps`` decode steps each append one token and decode.
    """
    name: str
    batch: int
    n_q_heads: int
    n_kv_heads: int
    n_ctx: int
    dtype: str             # "f32" or "bf16" for q, K, V
    dist: str              # "normal" or "t4"
    outlier_mode: str      # "first4" (channels 0-3) or "frac" (a seeded fraction)
    outlier_frac: float
    outlier_scale: float
    sparsity: float
    bits: int = 2
    quant_group: int = 32   # channels per quantization group: 32, or 128 (one grid per token)
    per_head_transform: bool = True
    n_steps: int = 0
    seed: int = 0
    refine: bool = False    # diagonal refinement D folded into the transforms
    rotate_values: bool = False
    v_clip: float = 1.0     # value clipping ratio (the pages use 0.92 with rotated values)
    bucket: int = 0         # tokens per RoPE bucket (the pages use 2048); 0: no buckets
    rope_base: float = 500000.0

    @property
    def group_size(self) -> int:
        return self.n_q_heads // self.n_kv_heads

    @property
    def capacity(self) -> int:
        """Cache capacity in tokens: context plus decode steps, whole blocks."""
        need = self.n_ctx + max(self.n_steps, 1)
        return ((need + BLOCK_TOKENS - 1) // BLOCK_TOKENS) * BLOCK_TOKENS

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


def _wl(name, **kw) -> Workload:
    base = dict(batch=1, n_q_heads=32, n_kv_heads=8, n_ctx=131072, dtype="bf16",
                dist="normal", outlier_mode="frac", outlier_frac=0.02,
                outlier_scale=6.0, sparsity=0.4, bits=2,
                per_head_transform=True, n_steps=0, seed=0)
    base.update(kw)
    return Workload(name=name, **base)


# The five workloads.  Seeds follow 1000 * index.
WORKLOADS = {
    # single head, 4K context, fp32, channels 0-3 of K scaled x8, one transform
    "single_head_4k": _wl("single_head_4k", batch=1, n_q_heads=1, n_kv_heads=1,
                          n_ctx=4096, dtype="f32", outlier_mode="first4",
                          outlier_scale=8.0, per_head_transform=False, seed=1000),
    # Llama-3-8B-like layer: batch 8, 32/8 heads, 32K context
    "llama8b_b8_32k": _wl("llama8b_b8_32k", batch=8, n_ctx=32768, seed=2000),
    # headline long context: batch 1, 32/8 heads, 128K context
    "longctx_b1_128k": _wl("longctx_b1_128k", batch=1, n_ctx=131072, seed=3000),
    # sparsity / batch sweep: batch 32, 16K context (sparsity varies per run)
    "sweep_b32_16k": _wl("sweep_b32_16k", batch=32, n_ctx=16384, seed=4000),
    # append + decode pipeline: 128K prefill then 256 one-token decode steps,
    # heavy-tailed Student-t(4) keys and values
    "pipeline_128k_t4": _wl("pipeline_128k_t4", batch=1, n_ctx=131072, dist="t4",
                            outlier_frac=0.0, outlier_scale=1.0, n_steps=256,
                            seed=5000),
}

SWEEP_SPARSITIES = (0.0, 0.2, 0.4, 0.6)


def _rng(seed: int, stream: int, sub: int = 0) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64([seed, stream, sub]))


# ---------------------------------------------------------------- bf16 bits
def bf16_bits_from_f32(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (nearest, ties to even); returns uint16 bits.

    Input preparation only: the draws are defined as these rounded values.
    """
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    nan = (u & 0x7FFFFFFF) > 0x7F800000
    lsb = (u >> 16) & 1
    r = ((u + 0x7FFF + lsb) >> 16).astype(np.uint16)
    r[nan] = 0x7FC0
    return r


def f32_from_bf16_bits(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def as_float(x: np.ndarray, dtype: str) -> np.ndarray:
    """Exact float64 values of an input array stored as f32 or bf16 bits."""
    if dtype == "f32":
        return np.asarray(x, dtype=np.float32).astype(np.float64)
    return f32_from_bf16_bits(x).astype(np.float64)


def _store(x32: np.ndarray, dtype: str) -> np.ndarray:
    if dtype == "f32":
        return np.ascontiguousarray(x32, dtype=np.float32)
    if dtype == "bf16":
        return bf16_bits_from_f32(x32)
    raise ValueError(dtype)


# ------------------------------------------------------------ the transform
def _haar_q(rng: np.random.Generator, d: int) -> np.ndarray:
    g = rng.standard_normal((d, d))
    q, r = np.linalg.qr(g)
    return q * np.sign(np.diag(r))[None, :]


def make_transform(seed: int, head: int, d: int = HEAD_DIM, sigma: float = 0.3):
    """Seeded key transform ``A`` and its inverse transpose, both float64 [d][d]."""
    U = _haar_q(_rng(seed, _S_A_U, head), d)
    W = _haar_q(_rng(seed, _S_A_W, head), d)
    g = _rng(seed, _S_A_G, head).normal(0.0, sigma, size=d)
    A = (U * np.exp(g)[None, :]) @ W.T
    Ainvt = (U * np.exp(-g)[None, :]) @ W.T
    return np.ascontiguousarray(A), np.ascontiguousarray(Ainvt)


def make_refinement(seed: int, head: int, d: int = HEAD_DIM, sigma: float = 0.3) -> np.ndarray:
    """Positive diagonal scales delta [d], delta[0] = 1, free scales with unit
    geometric mean."""
    g = _rng(seed, _S_DELTA, head).normal(0.0, sigma, size=d - 1)
    g -= g.mean()
    return np.concatenate([[1.0], np.exp(g)])


def sylvester_hadamard(n: int) -> np.ndarray:
    """Hadamard matrix of order n (a power of two), entries +-1."""
    H = np.ones((1, 1))
    while H.shape[0] < n:
        H = np.block([[H, H], [H, -H]])
    assert H.shape[0] == n
    return H


def make_value_rotation(seed: int, head: int, d: int = HEAD_DIM) -> np.ndarray:
    """Orthogonal value rotation Q H / sqrt(d), float64 [d][d]."""
    Q = _haar_q(_rng(seed, _S_RV, head), d)
    return np.ascontiguousarray(Q @ (sylvester_hadamard(d) / math.sqrt(d)))


def make_transforms(wl: Workload):
    """A and A^{-T} for every KV head: float64 [Hkv][d][d] each (with the
    workload's diagonal refinement folded in, when it has one)."""
    As, Ais = [], []
    for h in range(wl.n_kv_heads):
        hh = h if wl.per_head_transform else 0
        A, Ai = make_transform(wl.seed, hh)
        if wl.refine:
            delta = make_refinement(wl.seed, hh)
            A = A / delta[None, :]
            Ai = Ai * delta[None, :]
        As.append(A)
        Ais.append(Ai)
    return np.ascontiguousarray(np.stack(As)), np.ascontiguousarray(np.stack(Ais))


def rope_table(n_buckets: int, w: int, base: float = 500000.0, d: int = HEAD_DIM) -> np.ndarray:
    """cos and sin of a_b * theta_i for anchors a_b = b * w: float64 [n_buckets][d/2][2]."""
    theta = base ** (-2.0 * np.arange(d // 2) / d)
    ang = (np.arange(n_buckets, dtype=np.float64) * w)[:, None] * theta[None, :]
    return np.ascontiguousarray(np.stack([np.cos(ang), np.sin(ang)], axis=-1))


def n_buckets(wl: Workload) -> int:
    """Buckets that cover the workload's cache capacity (0 without buckets)."""
    return 0 if not wl.bucket else (wl.capacity + wl.bucket - 1) // wl.bucket


def make_rope(wl: Workload) -> Optional[np.ndarray]:
    """The rotary anchor table of the workload's buckets, or None."""
    return None if not wl.bucket else rope_table(n_buckets(wl), wl.bucket, wl.rope_base)


def make_deltas(wl: Workload) -> Optional[np.ndarray]:
    """The diagonal refinement of every KV head, float64 [Hkv][d], or None."""
    if not wl.refine:
        return None
    return np.ascontiguousarray(np.stack([make_refinement(wl.seed, h if wl.per_head_transform else 0)
                                          for h in range(wl.n_kv_heads)]))


def make_value_rotations(wl: Workload) -> Optional[np.ndarray]:
    """The value rotation of every KV head, float64 [Hkv][d][d], or None."""
    if not wl.rotate_values:
        return None
    return np.ascontiguousarray(np.stack([make_value_rotation(wl.seed, h if wl.per_head_transform else 0)
                                          for h in range(wl.n_kv_heads)]))


# ---------------------------------------------------------- keys and values
def outlier_channels(wl: Workload, head: int) -> np.ndarray:
    if wl.outlier_mode == "first4":
        return np.arange(4)
    n = int(math.ceil(wl.outlier_frac * HEAD_DIM - 1e-9))
    if n == 0:
        return np.zeros(0, dtype=np.int64)
    rng = _rng(wl.seed, _S_OUTLIER, head)
    return np.sort(rng.choice(HEAD_DIM, size=n, replace=False))


def _draw(rng: np.random.Generator, shape, dist: str) -> np.ndarray:
    if dist == "normal":
        return rng.standard_normal(shape, dtype=np.float32)
    if dist == "t4":
        z = rng.standard_normal(shape, dtype=np.float32)
        c = rng.chisquare(4.0, size=shape).astype(np.float32)
        return (z / np.sqrt(c / 4.0)).astype(np.float32)
    raise ValueError(dist)


def make_kv(wl: Workload, n_tokens: Optional[int] = None, stream_k: int = _S_K,
            stream_v: int = _S_V, sub: int = 0):
    """Keys and values [B][Hkv][n][d] in the workload's input dtype.

    Each (batch, head) slice is its own stream so that any subset can be
    regenerated alone.
    """
    n = wl.n_ctx if n_tokens is None else n_tokens
    B, H, d = wl.batch, wl.n_kv_heads, HEAD_DIM
    K = np.empty((B, H, n, d), dtype=np.float32)
    V = np.empty((B, H, n, d), dtype=np.float32)
    for b in range(B):
        for h in range(H):
            k = _draw(_rng(wl.seed, stream_k, (sub << 20) | (b << 8) | h), (n, d), wl.dist)
            k[:, outlier_channels(wl, h)] *= np.float32(wl.outlier_scale)
            K[b, h] = k
            V[b, h] = _draw(_rng(wl.seed, stream_v, (sub << 20) | (b << 8) | h), (n, d), wl.dist)
    return _store(K, wl.dtype), _store(V, wl.dtype)


def make_kv_unit(wl: Workload, b: int, h: int, n_tokens: Optional[int] = None):
    """Keys and values [n][d] of one (batch, KV head): the same draws as make_kv."""
    n = wl.n_ctx if n_tokens is None else n_tokens
    k = _draw(_rng(wl.seed, _S_K, (b << 8) | h), (n, HEAD_DIM), wl.dist)
    k[:, outlier_channels(wl, h)] *= np.float32(wl.outlier_scale)
    v = _draw(_rng(wl.seed, _S_V, (b << 8) | h), (n, HEAD_DIM), wl.dist)
    return _store(k, wl.dtype), _store(v, wl.dtype)


def make_q(wl: Workload, step: int = 0):
    """Decode query [B][Hq][d] for one step, in the workload's input dtype."""
    q = _rng(wl.seed, _S_Q, step).standard_normal(
        (wl.batch, wl.n_q_heads, HEAD_DIM), dtype=np.float32)
    return _store(q, wl.dtype)


def make_step_kv(wl: Workload, step: int):
    """The one new key/value token per (batch, KV head) appended at a decode step."""
    return make_kv(wl, n_tokens=1, stream_k=_S_KNEW, stream_v=_S_VNEW, sub=step + 1)


def workload(name: str, **overrides) -> Workload:
    wl = WORKLOADS[name]
    return wl.with_(**overrides) if overrides else wl


def names() -> Sequence[str]:
    return tuple(WORKLOADS)
