"""Shared helpers for the GPU parity tests: seeded inputs from the workload
generator, the oracle's cache/selection/decode for the same inputs, and the
CUDA path through the Python binding of the C ABI."""
from __future__ import annotations

import numpy as np
import torch

from long_context_decode_dual_b200 import kvq
from long_context_decode_dual_b200 import workloads as W
from oracle import oracle as orc


def to_dev(x: np.ndarray, dtype: str) -> torch.Tensor:
    if dtype == "f32":
        return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).cuda()
    return torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).cuda().view(torch.bfloat16)


def dev64(x: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float64)).cuda()


class Case:
    """Inputs of one workload (possibly shortened) plus both implementations."""

    def __init__(self, wl: W.Workload, n_ctx: int | None = None, capacity: int | None = None):
        self.wl = wl if n_ctx is None else wl.with_(n_ctx=n_ctx)
        self.capacity = capacity or self.wl.capacity
        self.A, self.Ai = W.make_transforms(self.wl)      # refinement folded in when the workload has one
        self.delta = W.make_deltas(self.wl)                # [Hkv][128] or None
        self.Rv = W.make_value_rotations(self.wl)          # [Hkv][128][128] or None
        w = self.wl.bucket                                 # RoPE anchors of the cache's buckets, or None
        self.rope = W.rope_table(-(-self.capacity // w), w, self.wl.rope_base) if w else None
        self.K, self.V = W.make_kv(self.wl)
        self._oracle_units = {}

    def cache_kw(self) -> dict:
        """new_cache keywords of the workload's format (group, value rotation, clip)."""
        return dict(group=self.wl.quant_group, v_rot=None if self.Rv is None else dev64(self.Rv),
                    v_clip=self.wl.v_clip, bucket=self.wl.bucket,
                    rope=None if self.rope is None else dev64(self.rope))

    def dev_delta(self):
        return None if self.delta is None else dev64(self.delta)

    def delta_of(self, h: int):
        return None if self.delta is None else self.delta[h]

    def rv_of(self, h: int):
        return None if self.Rv is None else self.Rv[h]

    def oracle_values(self, Vf: np.ndarray, h: int) -> np.ndarray:
        """Values as the cache stores them: rotated when the workload rotates them."""
        return Vf if self.Rv is None else orc.value_rotate(Vf, self.Rv[h])

    def oracle_keys(self, Kf: np.ndarray, h: int, pos0: int = 0) -> np.ndarray:
        """K' as the cache stores it: in the frame of each token's RoPE bucket
        when the workload has buckets."""
        if self.rope is None:
            return orc.transform(Kf, self.A[h])
        return orc.bucket_keys(Kf, self.A[h], self.rope, self.wl.bucket, pos0)

    def n_buckets(self, n: int) -> int:
        return max(1, -(-n // self.wl.bucket)) if self.wl.bucket else 1

    def oracle_decode_any(self, q, b, h, sparsity, n, slots=None, n_sink=0, n_recent=0):
        """The oracle's decode of one unit over n tokens in the workload's
        format (buckets, tier, rotation, refinement).  Returns (out, idx) with
        idx [n_buckets][k] when the workload has buckets, else [k]."""
        wl = self.wl
        unit = self.oracle_unit(b, h, n)
        g = wl.group_size
        qf = W.as_float(q[b, h * g:(h + 1) * g], wl.dtype)
        if self.rope is not None:
            qpb = orc.bucket_queries(qf, self.Ai[h], self.rope, self.n_buckets(n))
            return orc.decode_unit_buckets(unit, wl.bits, n, qpb, sparsity, wl.bucket, wl.quant_group,
                                           delta=self.delta_of(h), Rv=self.rv_of(h), slots=slots, n_sink=n_sink,
                                           n_recent=n_recent)
        qp = orc.transform(qf, self.Ai[h])
        if slots is not None and n_sink + n_recent > 0:
            return orc.decode_unit_protected(unit, slots, wl.bits, n, qp, sparsity, n_sink, n_recent,
                                             wl.quant_group, delta=self.delta_of(h), Rv=self.rv_of(h))
        return orc.decode_unit(unit, wl.bits, n, qp, sparsity, wl.quant_group, delta=self.delta_of(h),
                               Rv=self.rv_of(h))

    # ---------------------------------------------------------------- GPU
    def gpu_cache(self, chunks=None) -> kvq.KVCache:
        wl = self.wl
        cache = kvq.new_cache(wl.batch, wl.n_kv_heads, self.capacity, wl.bits, **self.cache_kw())
        A = dev64(self.A)
        n = self.K.shape[2]
        chunks = chunks or [n]
        pos = 0
        for c in chunks:
            kvq.append(cache, to_dev(self.K[:, :, pos:pos + c], wl.dtype),
                       to_dev(self.V[:, :, pos:pos + c], wl.dtype), A)
            pos += c
        assert pos == n
        return cache

    def q(self, step: int = 0) -> np.ndarray:
        return W.make_q(self.wl, step)

    # ------------------------------------------------------------- oracle
    def oracle_unit(self, b: int, h: int, n: int | None = None) -> np.ndarray:
        key = (b, h, n)
        if key not in self._oracle_units:
            wl = self.wl
            n = self.K.shape[2] if n is None else n
            Kf = W.as_float(self.K[b, h, :n], wl.dtype)
            Vf = W.as_float(self.V[b, h, :n], wl.dtype)
            u = orc.new_unit(self.capacity, wl.bits, wl.quant_group)
            orc.append_unit(u, wl.bits, 0, self.oracle_keys(Kf, h), self.oracle_values(Vf, h),
                            group=wl.quant_group, vclip=wl.v_clip)
            self._oracle_units[key] = u
        return self._oracle_units[key]

    def oracle_qp(self, q: np.ndarray, b: int, h: int) -> np.ndarray:
        g = self.wl.group_size
        qf = W.as_float(q[b, h * g:(h + 1) * g], self.wl.dtype)
        return orc.transform(qf, self.Ai[h])

    def oracle_decode(self, q: np.ndarray, b: int, h: int, sparsity: float, n: int | None = None):
        n = self.K.shape[2] if n is None else n
        qp = self.oracle_qp(q, b, h)
        out, idx = self.oracle_decode_any(q, b, h, sparsity, n)
        return out, idx, qp


def expected_qsel_qgsum(qp: np.ndarray, idx: np.ndarray, group: int = 32):
    """fp32 rounding of q'[h][idx] and of the float64 ascending sum per key
    group of the kept channels other than channel 0 (the documented
    definition of kvq_select_channels' outputs; with one grid per token the
    single sum is entry 0 and the other entries are 0)."""
    qsel = qp[:, idx].astype(np.float32)
    g = qp.shape[0]
    qgsum = np.zeros((g, 4), dtype=np.float32)
    for hl in range(g):
        for gr in range(128 // group):
            s = 0.0
            for c in idx:
                if c != 0 and c // group == gr:
                    s += float(qp[hl, c])
            qgsum[hl, gr] = np.float32(s)
    return qsel, qgsum


def rel_errors(out: np.ndarray, ref: np.ndarray):
    """The tolerance reading of the output check, per (sequence, head) output
    vector (the last axis): e_i = |out_i - ref_i| / ||ref||_inf of that
    vector.  Returns (largest e_i over every vector, largest per-vector mean
    of e_i), the two numbers held to 2e-3 and 1e-3."""
    ref = np.asarray(ref, dtype=np.float64)
    out = np.asarray(out, dtype=np.float64)
    scale = np.abs(ref).max(axis=-1, keepdims=True)
    scale = np.where(scale == 0, 1.0, scale)
    e = np.abs(out - ref) / scale
    return e.max(), e.mean(axis=-1).max()


def check_pages(case: Case, cache: kvq.KVCache, units=None, n=None):
    """The cache's pages of the given units equal the oracle's, byte for byte."""
    pages = cache.all_pages().cpu().numpy()
    wl = case.wl
    units = units or [(b, h) for b in range(wl.batch) for h in range(wl.n_kv_heads)]
    for b, h in units:
        ref = case.oracle_unit(b, h, n)
        got = pages[b, h]
        if not np.array_equal(got, ref):
            bad = np.argwhere(got != ref)
            raise AssertionError(f"unit {(b, h)}: {len(bad)} bytes differ, first (page, byte) {bad[:4].tolist()}")
