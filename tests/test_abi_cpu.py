"""The C ABI library loads on a machine without a GPU and exports every entry
point declared in include/kvq.h; host-side validation answers without
touching the device."""
import ctypes
import os
import re

import pytest

from long_context_decode_dual_b200 import kvq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "kvq.h")


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(kvq_[a-z0-9_]+)\s*\(", src)))


def test_every_declared_symbol_is_exported():
    names = _declared()
    assert len(names) >= 12
    L = kvq.lib()
    missing = [n for n in names if not hasattr(L, n)]
    assert not missing, missing
    assert set(names) == set(kvq.EXPORTS)


def test_host_side_queries():
    L = kvq.lib()
    assert L.kvq_version() == 102
    assert L.kvq_page_bytes(2, 32) == 12544 and L.kvq_page_bytes(4, 32) == 20736 and L.kvq_page_bytes(3, 32) == 0
    assert L.kvq_page_bytes(2, 128) == 9472 and L.kvq_page_bytes(4, 128) == 17664 and L.kvq_page_bytes(2, 64) == 0
    for s, k in ((0.0, 128), (0.2, 103), (0.4, 77), (0.6, 52), (0.25, 96)):
        assert kvq.num_selected(s) == k
    assert kvq.num_selected(1.0) == -1 and kvq.num_selected(-0.1) == -1
    d = kvq.CacheDesc(2, 8, 128, 32, 2, 256, 0, 0, 0)
    assert L.kvq_cache_bytes(ctypes.byref(d)) == 2 * 8 * 2 * 12544
    bad = kvq.CacheDesc(2, 8, 64, 32, 2, 256, 0, 0, 0)
    assert L.kvq_cache_bytes(ctypes.byref(bad)) == 0
    one = kvq.CacheDesc(2, 8, 128, 128, 2, 256, 0, 0, 0)            # one grid per token
    assert L.kvq_cache_bytes(ctypes.byref(one)) == 2 * 8 * 2 * 9472
    tier = kvq.CacheDesc(2, 8, 128, 128, 2, 256, 0, 0, 0, 64, 256)  # plus the BF16 slots
    assert L.kvq_cache_bytes(ctypes.byref(tier)) == 2 * 8 * (2 * 9472 + 320 * 512)
    assert L.kvq_cache_bytes(ctypes.byref(kvq.CacheDesc(2, 8, 128, 64, 2, 256, 0, 0, 0))) == 0
    assert L.kvq_cache_bytes(ctypes.byref(kvq.CacheDesc(2, 8, 128, 32, 2, 256, 0, 0, 0, 1000, 25))) == 0
    assert kvq.status_string(-3) == "capacity exceeded"
    assert L.kvq_copy_async(None, None, 0, None) == 0                 # nothing to copy
    assert L.kvq_copy_async(None, 8, 16, None) == -1


def test_validation_rejects_before_launch():
    L = kvq.lib()
    nullc = kvq.CacheDesc(1, 1, 128, 32, 2, 128, 0, 0, 0)
    assert L.kvq_cache_init(ctypes.byref(nullc), None) == -1
    assert L.kvq_append(None, None, None, 0, 1, None, None) == -1
    fake = kvq.CacheDesc(1, 1, 128, 32, 3, 128, 256, 256, 256)     # bits 3
    assert L.kvq_append(ctypes.byref(fake), 8, 8, 0, 1, 8, None) == -2
    mis = kvq.CacheDesc(1, 1, 128, 32, 2, 128, 0x1010, 256, 256)  # pages not 256-aligned
    assert L.kvq_append(ctypes.byref(mis), 8, 8, 0, 1, 8, None) == -6
    ok = kvq.CacheDesc(1, 1, 128, 32, 2, 128, 0x1000, 256, 256)
    assert L.kvq_append(ctypes.byref(ok), 8, 8, 0, -1, 16, None) == -1
    assert L.kvq_append(ctypes.byref(ok), 8, 8, 7, 1, 16, None) == -1            # dtype
    assert L.kvq_append(ctypes.byref(ok), 8, 8, 0, 1, 8, None) == -6             # A not 16-aligned
    assert L.kvq_append(ctypes.byref(ok), 8, 8, 0, 129, 16, None) == -3         # > capacity
    assert L.kvq_append(ctypes.byref(ok), 8, 8, 0, 0, 16, None) == 0            # no-op
    two = kvq.CacheDesc(1, 2, 128, 32, 2, 128, 0x1000, 256, 256)
    assert L.kvq_select_channels(ctypes.byref(two), 8, 0, 3, 8, None, ctypes.c_float(0.4), 8, 8, 8,
                                 None, None) == -2                              # 3 % 2 heads
    assert L.kvq_select_channels(ctypes.byref(two), 8, 0, 4, 8, None, ctypes.c_float(1.5), 8, 8, 8,
                                 None, None) == -1                              # sparsity
    assert L.kvq_select_channels(ctypes.byref(two), 8, 0, 4, 8, None, ctypes.c_float(0.4), 8, 8, 8,
                                 None, None) == -6                              # Ainvt not 16-aligned
    assert L.kvq_select_channels(ctypes.byref(two), 8, 0, 4, 16, 12, ctypes.c_float(0.4), 8, 8, 8,
                                 None, None) == -6                              # delta not 8-aligned
    # value rotation / clip fields of the descriptor
    rot_mis = kvq.CacheDesc(1, 1, 128, 32, 2, 128, 0x1000, 256, 256, 0, 0, 0x1008, 0.92)
    assert L.kvq_append(ctypes.byref(rot_mis), 8, 8, 0, 1, 16, None) == -6      # v_rot not 16-aligned
    for clip in (-0.5, 1.5, float("nan")):
        bad_clip = kvq.CacheDesc(1, 1, 128, 32, 2, 128, 0x1000, 256, 256, 0, 0, 0x1000, clip)
        assert L.kvq_append(ctypes.byref(bad_clip), 8, 8, 0, 1, 16, None) == -1
    ok_rot = kvq.CacheDesc(1, 1, 128, 32, 2, 128, 0x1000, 256, 256, 0, 0, 0x1000, 0.92)
    assert L.kvq_append(ctypes.byref(ok_rot), 8, 8, 0, 0, 16, None) == 0        # valid, no-op
    # RoPE buckets: a multiple of 128 tokens, with the anchors' table
    def bk(w, rope):
        return kvq.CacheDesc(1, 1, 128, 32, 2, 1000 * 128, 0x1000, 256, 256, 0, 0, 0, 0.0, w, rope)
    assert L.kvq_append(ctypes.byref(bk(200, 0x2000)), 8, 8, 0, 0, 16, None) == -2
    assert L.kvq_append(ctypes.byref(bk(-128, 0x2000)), 8, 8, 0, 0, 16, None) == -2
    assert L.kvq_append(ctypes.byref(bk(2048, 0)), 8, 8, 0, 0, 16, None) == -1
    assert L.kvq_append(ctypes.byref(bk(2048, 0x2008)), 8, 8, 0, 0, 16, None) == -6
    assert L.kvq_append(ctypes.byref(bk(2048, 0x2000)), 8, 8, 0, 0, 16, None) == 0
    assert L.kvq_num_buckets(ctypes.byref(bk(2048, 0x2000))) == 63          # ceil(128000 / 2048)
    assert L.kvq_num_buckets(ctypes.byref(bk(128, 0x2000))) == 1000
    assert L.kvq_num_buckets(ctypes.byref(bk(0, 0))) == 1
    assert L.kvq_num_buckets(ctypes.byref(bk(200, 0x2000))) == 0
    assert L.kvq_decode_attn(ctypes.byref(two), 6, 8, 8, 8, 77, 8, 8, 1 << 20, None) == -2  # g = 3
    assert L.kvq_decode_attn(ctypes.byref(two), 4, 8, 8, 8, 0, 8, 8, 1 << 20, None) == -1   # k = 0
    assert L.kvq_bf16_decode_attn(8, 8, 8, 1, 3, 2, 10, 8, 8, 1 << 20, None) == -2
