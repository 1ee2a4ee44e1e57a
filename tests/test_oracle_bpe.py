"""Pins for the byte-accounting model against the pages' printed BPE values
(Dual-QK Table 1 and abstract; fixture tests/golden/bpe_table1.txt)."""
import os

import pytest

from oracle import bpe

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "bpe_table1.txt")
N_CTX = 131072


def _golden():
    rows = {}
    for line in open(GOLDEN):
        line = line.split("#")[0].split()
        if line:
            rows[line[0]] = [float(v) for v in line[1:]]
    return rows


def test_pages_formats_reproduce_table1():
    g = _golden()
    for name, fmt in (("dual_qk", bpe.DUAL_QK_PAGES), ("oscar", bpe.OSCAR_PAGES)):
        cap = bpe.capacity_bpe(fmt, N_CTX)
        bw = bpe.bandwidth_bpe(fmt, N_CTX, 0.4)
        assert round(cap, 2) == g[name][0], (name, cap)
        assert round(bw, 2) == g[name][1], (name, bw)


def test_pages_ratios():
    g = _golden()
    cap = bpe.capacity_bpe(bpe.DUAL_QK_PAGES, N_CTX)
    bw = bpe.bandwidth_bpe(bpe.DUAL_QK_PAGES, N_CTX, 0.4)
    assert round(16 / cap, 1) == g["dual_qk_compression"][0]
    assert round(16 / bw, 1) == g["dual_qk_read_reduction"][0]


@pytest.mark.parametrize("s,bytes_per_token", [(0.0, 97.75), (0.2, 91.5), (0.4, 85.0), (0.6, 78.75)])
def test_group32_read_bytes(s, bytes_per_token):
    assert bpe.read_bits_per_token(bpe.GROUP32_INT2, s) / 8 == bytes_per_token
    assert bpe.stored_bits_per_token(bpe.GROUP32_INT2) / 8 == 97.75
    assert bpe.read_bits_per_token(bpe.GROUP32_INT4, 0.4) / 8 == 136.0
