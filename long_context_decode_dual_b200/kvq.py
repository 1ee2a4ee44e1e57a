"""Python binding of the kvq C ABI (include/kvq.h).

Argument marshalling only: every step of the decode path runs in the CUDA
kernels of ``libkvq.so``.  PyTorch supplies device memory and streams.  There
is no fallback: if the library is missing, importing it raises.

Names follow the C entry points:
  kvq_append           -> append(cache, K, V, A)
  kvq_select_channels  -> select_channels(cache, q, Ainvt, sparsity, delta=None)
  kvq_decode_attn      -> decode_attn(cache, sel)
  kvq_decode_step      -> decode_step(cache, q, k_new, v_new, A, Ainvt, sparsity, delta=None)
  kvq_bf16_decode_attn -> bf16_decode_attn(q, K, V)
"""
from __future__ import annotations

import ctypes
import dataclasses
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libkvq.so")

KVQ_OK = 0
KVQ_DTYPE_F32 = 0
KVQ_DTYPE_BF16 = 1
KVQ_DEV_CAPACITY = 1
KVQ_DEV_TIMEOUT = 2
KVQ_DEV_INDEX = 4
HEAD_DIM = 128
GROUP = 32
BLOCK_TOKENS = 128


class KvqError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn}: {status_string(status)} ({status})")
        self.status = status


class CacheDesc(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int32), ("n_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
        ("group", ctypes.c_int32), ("bits", ctypes.c_int32), ("capacity", ctypes.c_int32),
        ("pages", ctypes.c_void_p), ("seq_len", ctypes.c_void_p), ("status", ctypes.c_void_p),
        ("n_sink", ctypes.c_int32), ("n_recent", ctypes.c_int32),
        ("v_rot", ctypes.c_void_p), ("v_clip", ctypes.c_double),
        ("bucket", ctypes.c_int32), ("rope", ctypes.c_void_p),
    ]


_lib = None

EXPORTS = (
    "kvq_status_words", "kvq_page_bytes", "kvq_cache_bytes", "kvq_cache_init", "kvq_append", "kvq_num_selected",
    "kvq_select_channels", "kvq_decode_workspace", "kvq_decode_attn",
    "kvq_bf16_decode_workspace", "kvq_bf16_decode_attn", "kvq_read_status",
    "kvq_status_string", "kvq_version", "kvq_decode_static_scratch_bytes",
    "kvq_decode_attn_static", "kvq_decode_step", "kvq_num_buckets", "kvq_copy_async",
    "kvq_decode_attn_wait_bound",
)


def lib() -> ctypes.CDLL:
    """The loaded C library (raises if it was not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"kvq CUDA library not built: {LIB_PATH} is missing "
                               "(run python -m long_context_decode_dual_b200.build)")
        L = ctypes.CDLL(LIB_PATH)
        P, I, S = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
        C = ctypes.POINTER(CacheDesc)
        sig = {
            "kvq_status_words": (S, [I, I]),
            "kvq_page_bytes": (S, [I, I]),
            "kvq_cache_bytes": (S, [C]),
            "kvq_cache_init": (I, [C, P]),
            "kvq_append": (I, [C, P, P, I, I, P, P]),
            "kvq_num_selected": (I, [ctypes.c_float, I]),
            "kvq_select_channels": (I, [C, P, I, I, P, P, ctypes.c_float, P, P, P, ctypes.POINTER(I), P]),
            "kvq_decode_workspace": (S, [C, I, I]),
            "kvq_decode_attn": (I, [C, I, P, P, P, I, P, P, S, P]),
            "kvq_bf16_decode_workspace": (S, [I, I, I, I]),
            "kvq_bf16_decode_attn": (I, [P, P, P, I, I, I, I, P, P, S, P]),
            "kvq_read_status": (I, [C, ctypes.POINTER(ctypes.c_uint32), P]),
            "kvq_status_string": (ctypes.c_char_p, [I]),
            "kvq_version": (I, []),
            "kvq_decode_static_scratch_bytes": (S, []),
            "kvq_decode_attn_static": (I, [C, I, P, P, P, I, P, P]),
            "kvq_decode_step": (I, [C, P, P, P, I, I, I, P, P, P, ctypes.c_float, P, P, P, P, P, S, P]),
            "kvq_num_buckets": (I, [C]),
            "kvq_copy_async": (I, [P, P, S, P]),
            "kvq_decode_attn_wait_bound": (I, [C, I, P, P, P, I, P, P, S, ctypes.c_uint32, P]),
        }
        for name, (res, args) in sig.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().kvq_status_string(int(status)).decode()


def _check(fn: str, status: int) -> None:
    if status != KVQ_OK:
        raise KvqError(fn, status)


def _stream(stream: Optional[torch.cuda.Stream]):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t: Optional[torch.Tensor]):
    return ctypes.c_void_p(0 if t is None else t.data_ptr())


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return KVQ_DTYPE_F32
    if t.dtype in (torch.bfloat16, torch.int16, torch.uint16):
        return KVQ_DTYPE_BF16
    raise TypeError(f"unsupported input dtype {t.dtype} (float32 or bfloat16)")


def num_selected(sparsity: float, head_dim: int = HEAD_DIM) -> int:
    return int(lib().kvq_num_selected(float(sparsity), head_dim))


@dataclasses.dataclass
class KVCache:
    """A prunable INT2/INT4 KV cache in device memory (kvq_cache)."""
    batch: int
    n_kv_heads: int
    capacity: int
    bits: int
    pages: torch.Tensor
    seq_len: torch.Tensor
    status: torch.Tensor
    n_sink: int = 0           # protected BF16 tier: first tokens kept
    n_recent: int = 0         # and most recent tokens kept
    group: int = GROUP        # channels per quantization group: 32, or 128 (one grid per token)
    v_rot: Optional[torch.Tensor] = None   # value rotation [Hkv][128][128] f64 (orthogonal), or None
    v_clip: float = 1.0       # clipping ratio of the value grids
    bucket: int = 0           # tokens per RoPE bucket (0: none)
    rope: Optional[torch.Tensor] = None    # anchors' rotary table [n_buckets][64][2] f64

    @property
    def desc(self) -> CacheDesc:
        return CacheDesc(self.batch, self.n_kv_heads, HEAD_DIM, self.group, self.bits, self.capacity,
                         self.pages.data_ptr(), self.seq_len.data_ptr(), self.status.data_ptr(),
                         self.n_sink, self.n_recent, 0 if self.v_rot is None else self.v_rot.data_ptr(),
                         float(self.v_clip), self.bucket, 0 if self.rope is None else self.rope.data_ptr())

    @property
    def n_buckets(self) -> int:
        """Entries per selection array: RoPE buckets of the capacity, 1 without."""
        return (self.capacity + self.bucket - 1) // self.bucket if self.bucket else 1

    @property
    def n_blocks(self) -> int:
        return self.capacity // BLOCK_TOKENS

    @property
    def page_array_bytes(self) -> int:
        return self.batch * self.n_kv_heads * self.n_blocks * page_bytes(self.bits, self.group)

    def all_pages(self) -> torch.Tensor:
        """The page array without the protected slots: uint8 [B][Hkv][blocks][page bytes]."""
        return self.pages[:self.page_array_bytes].view(self.batch, self.n_kv_heads, self.n_blocks,
                                                       page_bytes(self.bits, self.group))

    def unit_pages(self, b: int, h: int) -> torch.Tensor:
        """Pages of one (sequence, KV head): uint8 [capacity/128][page bytes]."""
        return self.all_pages()[b, h]

    def slots(self) -> torch.Tensor:
        """Protected BF16 slots: int16 bit patterns [B][Hkv][n_sink + n_recent][256]
        (128 of the transformed key, then 128 of the value)."""
        n = self.n_sink + self.n_recent
        return self.pages[self.page_array_bytes:].view(torch.int16).view(self.batch, self.n_kv_heads, n, 256)


def page_bytes(bits: int, group: int = GROUP) -> int:
    return int(lib().kvq_page_bytes(bits, group))


def new_cache(batch: int, n_kv_heads: int, capacity: int, bits: int = 2,
              device="cuda", stream=None, n_sink: int = 0, n_recent: int = 0, group: int = GROUP,
              v_rot: Optional[torch.Tensor] = None, v_clip: float = 1.0, bucket: int = 0,
              rope: Optional[torch.Tensor] = None) -> KVCache:
    """A zeroed cache.  ``v_rot`` (device f64 [Hkv][128][128], orthogonal) makes
    appends store rotated values and decodes rotate their output back;
    ``v_clip`` clips the value grids (Dual-QK App. B.2 uses 0.92); ``bucket``
    tokens per RoPE bucket with the anchors' rotary table ``rope`` (device f64
    [n_buckets][64][2] of cos, sin) store keys in their bucket's frame and
    choose channels per bucket (Dual-QK §3.4)."""
    if v_rot is not None:
        assert v_rot.dtype == torch.float64 and v_rot.is_contiguous()
        assert tuple(v_rot.shape) == (n_kv_heads, HEAD_DIM, HEAD_DIM)
    if bucket:
        assert rope is not None and rope.dtype == torch.float64 and rope.is_contiguous()
        assert tuple(rope.shape) == ((capacity + bucket - 1) // bucket, HEAD_DIM // 2, 2)
    desc = CacheDesc(batch, n_kv_heads, HEAD_DIM, group, bits, capacity, 0, 0, 0, n_sink, n_recent,
                     None, float(v_clip), bucket, None)
    nbytes = int(lib().kvq_cache_bytes(ctypes.byref(desc)))
    if nbytes == 0:
        raise KvqError("kvq_cache_bytes", -2)
    pages = torch.empty(nbytes, dtype=torch.uint8, device=device)
    seq_len = torch.empty(batch, dtype=torch.int32, device=device)
    status = torch.empty(int(lib().kvq_status_words(batch, n_kv_heads)), dtype=torch.int32,
                         device=device)
    c = KVCache(batch, n_kv_heads, capacity, bits, pages, seq_len, status, n_sink, n_recent, group, v_rot,
                float(v_clip), bucket, rope)
    _check("kvq_cache_init", lib().kvq_cache_init(ctypes.byref(c.desc), _stream(stream)))
    return c


def append(cache: KVCache, K: torch.Tensor, V: torch.Tensor, A: torch.Tensor, stream=None) -> None:
    """kvq_append: K, V [B][Hkv][n_new][128] (f32 or bf16), A [Hkv][128][128] f64."""
    assert K.is_contiguous() and V.is_contiguous() and A.is_contiguous()
    assert K.shape == V.shape and K.dim() == 4 and A.dtype == torch.float64
    _check("kvq_append", lib().kvq_append(ctypes.byref(cache.desc), _ptr(K), _ptr(V), _dtype_code(K),
                                          int(K.shape[2]), _ptr(A), _stream(stream)))


@dataclasses.dataclass
class Selection:
    idx: torch.Tensor     # [B][Hkv][k] int32
    qsel: torch.Tensor    # [B][Hq][k] f32
    qgsum: torch.Tensor   # [B][Hq][4] f32
    k: int


def alloc_selection(cache: KVCache, n_q_heads: int, k: int, device="cuda") -> Selection:
    """Selection arrays: idx [B][Hkv][k], qsel [B][Hq][k], qgsum [B][Hq][4];
    with RoPE buckets one entry per bucket, [B][H][n_buckets][...]."""
    nb = (cache.n_buckets,) if cache.bucket else ()
    return Selection(
        torch.empty(cache.batch, cache.n_kv_heads, *nb, k, dtype=torch.int32, device=device),
        torch.empty(cache.batch, n_q_heads, *nb, k, dtype=torch.float32, device=device),
        torch.empty(cache.batch, n_q_heads, *nb, 4, dtype=torch.float32, device=device), k)


def select_channels(cache: KVCache, q: torch.Tensor, Ainvt: torch.Tensor, sparsity: float,
                    out: Optional[Selection] = None, stream=None, delta: Optional[torch.Tensor] = None) -> Selection:
    """kvq_select_channels: q [B][Hq][128] (f32 or bf16), Ainvt [Hkv][128][128] f64,
    delta (diagonal refinement folded into Ainvt) [Hkv][128] f64 or None."""
    assert q.is_contiguous() and Ainvt.is_contiguous() and Ainvt.dtype == torch.float64
    _check_delta(delta)
    Hq = int(q.shape[1])
    k = num_selected(sparsity)
    if k < 0:
        raise KvqError("kvq_num_selected", -1)
    sel = out if out is not None else alloc_selection(cache, Hq, k, q.device)
    assert sel.k == k
    kout = ctypes.c_int(0)
    _check("kvq_select_channels", lib().kvq_select_channels(
        ctypes.byref(cache.desc), _ptr(q), _dtype_code(q), Hq, _ptr(Ainvt), _ptr(delta), float(sparsity),
        _ptr(sel.idx), _ptr(sel.qsel), _ptr(sel.qgsum), ctypes.byref(kout), _stream(stream)))
    assert kout.value == k
    return sel


def _check_delta(delta: Optional[torch.Tensor]) -> None:
    if delta is not None:
        assert delta.dtype == torch.float64 and delta.is_contiguous() and delta.shape[-1] == HEAD_DIM


def decode_workspace_bytes(cache: KVCache, n_q_heads: int, k: int) -> int:
    return int(lib().kvq_decode_workspace(ctypes.byref(cache.desc), n_q_heads, k))


def alloc_workspace(nbytes: int, device="cuda") -> torch.Tensor:
    return torch.empty(max(nbytes, 16), dtype=torch.uint8, device=device)


def decode_attn(cache: KVCache, sel: Selection, out: Optional[torch.Tensor] = None,
                ws: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """kvq_decode_attn: returns out [B][Hq][128] f32."""
    B, Hq, k = cache.batch, int(sel.qsel.shape[1]), sel.k
    if out is None:
        out = torch.empty(B, Hq, HEAD_DIM, dtype=torch.float32, device=sel.qsel.device)
    if ws is None:
        ws = alloc_workspace(decode_workspace_bytes(cache, Hq, k), sel.qsel.device)
    _check("kvq_decode_attn", lib().kvq_decode_attn(
        ctypes.byref(cache.desc), Hq, _ptr(sel.idx), _ptr(sel.qsel), _ptr(sel.qgsum), k, _ptr(out),
        _ptr(ws), ws.numel(), _stream(stream)))
    return out


def decode_attn_wait_bound(cache: KVCache, sel: Selection, wait_polls: int, out: Optional[torch.Tensor] = None,
                           ws: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """kvq_decode_attn_wait_bound: kvq_decode_attn with an explicit bound on
    each wait for a staged page (a fault-handling test hook; 0 gives up at
    once unless the page has landed, which sets KVQ_DEV_TIMEOUT)."""
    B, Hq, k = cache.batch, int(sel.qsel.shape[1]), sel.k
    if out is None:
        out = torch.empty(B, Hq, HEAD_DIM, dtype=torch.float32, device=sel.qsel.device)
    if ws is None:
        ws = alloc_workspace(decode_workspace_bytes(cache, Hq, k), sel.qsel.device)
    _check("kvq_decode_attn_wait_bound", lib().kvq_decode_attn_wait_bound(
        ctypes.byref(cache.desc), Hq, _ptr(sel.idx), _ptr(sel.qsel), _ptr(sel.qgsum), k, _ptr(out),
        _ptr(ws), ws.numel(), int(wait_polls), _stream(stream)))
    return out


def decode_step(cache: KVCache, q: torch.Tensor, k_new: Optional[torch.Tensor], v_new: Optional[torch.Tensor],
                A: torch.Tensor, Ainvt: torch.Tensor, sparsity: float, sel: Optional[Selection] = None,
                out: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None,
                stream=None, delta: Optional[torch.Tensor] = None) -> tuple[torch.Tensor, Selection]:
    """kvq_decode_step: append k_new / v_new [B][Hkv][n_new][128], select the
    channels of q [B][Hq][128], decode; returns (out [B][Hq][128] f32, sel)."""
    assert q.is_contiguous() and A.is_contiguous() and Ainvt.is_contiguous()
    assert A.dtype == torch.float64 and Ainvt.dtype == torch.float64
    _check_delta(delta)
    B, Hq = cache.batch, int(q.shape[1])
    n_new = 0 if k_new is None else int(k_new.shape[2])
    if n_new:
        assert k_new.is_contiguous() and v_new.is_contiguous() and k_new.dtype == q.dtype == v_new.dtype
    k = num_selected(sparsity)
    if k < 0:
        raise KvqError("kvq_num_selected", -1)
    if sel is None:
        sel = alloc_selection(cache, Hq, k, q.device)
    assert sel.k == k
    if out is None:
        out = torch.empty(B, Hq, HEAD_DIM, dtype=torch.float32, device=q.device)
    if ws is None:
        ws = alloc_workspace(decode_workspace_bytes(cache, Hq, k), q.device)
    _check("kvq_decode_step", lib().kvq_decode_step(
        ctypes.byref(cache.desc), _ptr(q), _ptr(k_new if n_new else None), _ptr(v_new if n_new else None),
        _dtype_code(q), Hq, n_new, _ptr(A), _ptr(Ainvt), _ptr(delta), float(sparsity), _ptr(sel.idx), _ptr(sel.qsel),
        _ptr(sel.qgsum), _ptr(out), _ptr(ws), ws.numel(), _stream(stream)))
    return out, sel


def decode_attn_static(cache: KVCache, sel: Selection, out: Optional[torch.Tensor] = None,
                       stream=None) -> torch.Tensor:
    """kvq_decode_attn_static: decode without a caller workspace.

    For callers that cannot allocate device memory when they decode; the
    split partials use the library's one static device array, shared by all
    calls (serialise calls that could overlap on the GPU).
    """
    B, Hq, k = cache.batch, int(sel.qsel.shape[1]), sel.k
    if out is None:
        out = torch.empty(B, Hq, HEAD_DIM, dtype=torch.float32, device=sel.qsel.device)
    _check("kvq_decode_attn_static", lib().kvq_decode_attn_static(
        ctypes.byref(cache.desc), Hq, _ptr(sel.idx), _ptr(sel.qsel), _ptr(sel.qgsum), k, _ptr(out),
        _stream(stream)))
    return out


def decode_static_scratch_bytes() -> int:
    return int(lib().kvq_decode_static_scratch_bytes())


def bf16_workspace_bytes(B: int, Hq: int, Hkv: int, N: int) -> int:
    return int(lib().kvq_bf16_decode_workspace(B, Hq, Hkv, N))


def bf16_decode_attn(q: torch.Tensor, K: torch.Tensor, V: torch.Tensor,
                     out: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None,
                     stream=None) -> torch.Tensor:
    """kvq_bf16_decode_attn: q [B][Hq][128], K, V [B][Hkv][N][128], all bf16."""
    B, Hq = int(q.shape[0]), int(q.shape[1])
    Hkv, N = int(K.shape[1]), int(K.shape[2])
    for t in (q, K, V):
        assert t.is_contiguous() and _dtype_code(t) == KVQ_DTYPE_BF16
    if out is None:
        out = torch.empty(B, Hq, HEAD_DIM, dtype=torch.float32, device=q.device)
    if ws is None:
        ws = alloc_workspace(bf16_workspace_bytes(B, Hq, Hkv, N), q.device)
    _check("kvq_bf16_decode_attn", lib().kvq_bf16_decode_attn(
        _ptr(q), _ptr(K), _ptr(V), B, Hq, Hkv, N, _ptr(out), _ptr(ws), ws.numel(), _stream(stream)))
    return out


def read_status(cache: KVCache, stream=None) -> int:
    flags = ctypes.c_uint32(0)
    _check("kvq_read_status", lib().kvq_read_status(ctypes.byref(cache.desc), ctypes.byref(flags),
                                                    _stream(stream)))
    return int(flags.value)


def copy_async(dst: torch.Tensor, src: torch.Tensor, stream=None) -> None:
    """kvq_copy_async: stream-ordered copy of src's bytes into dst (device or
    pinned host tensors, same byte size); capturable into a CUDA graph."""
    nbytes = src.numel() * src.element_size()
    assert dst.numel() * dst.element_size() == nbytes and dst.is_contiguous() and src.is_contiguous()
    _check("kvq_copy_async", lib().kvq_copy_async(_ptr(dst), _ptr(src), nbytes, _stream(stream)))


def _packed(n_elems, dtype: torch.dtype, device, pin: bool = False):
    """One byte buffer holding tensors of the given element counts, each at a
    256-byte aligned offset; returns (buffer, views)."""
    esize = torch.tensor([], dtype=dtype).element_size()
    offs, total = [], 0
    for n in n_elems:
        offs.append(total)
        total += (n * esize + 255) // 256 * 256
    buf = torch.zeros(total, dtype=torch.uint8, device=device)
    if pin:
        buf = buf.pin_memory()
    views = [buf[o:o + n * esize].view(dtype) for o, n in zip(offs, n_elems)]
    return buf, views


class DecodeStep:
    """One decode step of the path -- append the new token, select channels,
    decode -- on static device buffers, replayable as a CUDA graph.

    Fill ``q`` [B][Hq][128] and ``k_new`` / ``v_new`` [B][Hkv][1][128] (f32 or
    bf16, the dtype given), call :meth:`run`; the result is in ``out``
    [B][Hq][128] f32.  ``fused`` (default) makes the step one kvq_decode_step
    call; otherwise it is kvq_append, kvq_select_channels and kvq_decode_attn.
    :meth:`capture` records the step once (after at least one eager
    :meth:`run`, so every kernel is loaded); later runs replay the graph.

    The three inputs are views of one device buffer, and ``q_host``,
    ``k_host``, ``v_host`` / ``out_host`` of pinned host buffers with the same
    layout: :meth:`run_host` moves the inputs in with one copy, runs the step
    and moves the result out with one copy -- all three in one graph replay
    once :meth:`capture` has run.
    """

    def __init__(self, cache: KVCache, A: torch.Tensor, Ainvt: torch.Tensor, sparsity: float,
                 n_q_heads: int, dtype: torch.dtype = torch.bfloat16, fused: bool = True,
                 delta: Optional[torch.Tensor] = None):
        dev = cache.pages.device
        B, Hkv = cache.batch, cache.n_kv_heads
        self.cache, self.A, self.Ainvt, self.sparsity = cache, A, Ainvt, float(sparsity)
        self.delta = delta
        self.fused = fused
        shapes = [(B, n_q_heads, HEAD_DIM), (B, Hkv, 1, HEAD_DIM), (B, Hkv, 1, HEAD_DIM)]
        counts = [B * n_q_heads * HEAD_DIM, B * Hkv * HEAD_DIM, B * Hkv * HEAD_DIM]
        self._in_dev, views = _packed(counts, dtype, dev)
        self.q, self.k_new, self.v_new = (v.view(*sh) for v, sh in zip(views, shapes))
        self._in_host, hviews = _packed(counts, dtype, "cpu", pin=True)
        self.q_host, self.k_host, self.v_host = (v.view(*sh) for v, sh in zip(hviews, shapes))
        self.k = num_selected(sparsity)
        self.sel = alloc_selection(cache, n_q_heads, self.k, dev)
        self.out = torch.empty(B, n_q_heads, HEAD_DIM, dtype=torch.float32, device=dev)
        self.out_host = torch.empty(B, n_q_heads, HEAD_DIM, dtype=torch.float32).pin_memory()
        self.ws = alloc_workspace(decode_workspace_bytes(cache, n_q_heads, self.k), dev)
        self.graph = None
        self.host_graph = None         # inputs in, the step, result out
        self.decode_events = None      # optional (start, end) events around the decode call

    @property
    def h2d_bytes(self) -> int:
        return self._in_host.numel()

    @property
    def d2h_bytes(self) -> int:
        return self.out_host.numel() * 4

    def _pre(self):
        if not self.fused:
            append(self.cache, self.k_new, self.v_new, self.A)
            select_channels(self.cache, self.q, self.Ainvt, self.sparsity, out=self.sel, delta=self.delta)

    def _decode(self):
        if self.fused:
            decode_step(self.cache, self.q, self.k_new, self.v_new, self.A, self.Ainvt, self.sparsity,
                        sel=self.sel, out=self.out, ws=self.ws, delta=self.delta)
        else:
            decode_attn(self.cache, self.sel, out=self.out, ws=self.ws)

    def _host_step(self):
        copy_async(self._in_dev, self._in_host)
        self._pre()
        self._decode()
        copy_async(self.out_host, self.out)

    def time_decode(self) -> None:
        """Record timing events around the decode call (the whole fused step)
        of every later run."""
        self.decode_events = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))

    def capture(self) -> None:
        """Record the step as CUDA graphs: append + select (unfused only) and
        the decode call, the decode timing events, if any, recorded between
        the replays; and the whole host step (inputs in, the step, result
        out) as one more graph."""
        pre = None
        if not self.fused:
            pre = torch.cuda.CUDAGraph()
            with torch.cuda.graph(pre):
                self._pre()
        dec = torch.cuda.CUDAGraph()
        with torch.cuda.graph(dec):
            self._decode()
        self.graph = (pre, dec)
        hg = torch.cuda.CUDAGraph()
        with torch.cuda.graph(hg):
            self._host_step()
        self.host_graph = hg

    def run(self) -> torch.Tensor:
        ev = self.decode_events
        if self.graph is not None:
            if self.graph[0] is not None:
                self.graph[0].replay()
        else:
            self._pre()
        if ev is not None:
            ev[0].record()
        if self.graph is not None:
            self.graph[1].replay()
        else:
            self._decode()
        if ev is not None:
            ev[1].record()
        return self.out

    def run_host(self, q_host: Optional[torch.Tensor] = None, k_host: Optional[torch.Tensor] = None,
                 v_host: Optional[torch.Tensor] = None) -> torch.Tensor:
        """One step from host inputs to a host result: the inputs (given as
        host tensors, or already written into ``q_host`` / ``k_host`` /
        ``v_host``) go in with one copy and the result comes back into
        ``out_host`` (returned) with one copy, stream-ordered on the current
        stream; synchronise before reading it."""
        for src, dst in ((q_host, self.q_host), (k_host, self.k_host), (v_host, self.v_host)):
            if src is not None and src.data_ptr() != dst.data_ptr():
                dst.copy_(src)
        if self.host_graph is not None:
            self.host_graph.replay()
        else:
            self._host_step()
        return self.out_host
