"""GPU parity of the pages' own cache format (Dual-QK §3.3: one asymmetric
INT2 grid per token and KV head over key channels 1..127 and over the value
channels; cache group = 128), alone and with the protected BF16 tier -- the
complete format behind the pages' Table 1 byte counts.

Same bars as the groups-of-32 format: pages, slots, indices and the
documented qsel / qgsum roundings byte-exact against the oracle; attention
outputs within 2e-3 max / 1e-3 mean of the oracle's.
"""
import numpy as np
import pytest
import torch

from long_context_decode_dual_b200 import kvq
from long_context_decode_dual_b200 import workloads as W
from oracle import oracle as orc

from helpers import Case, check_pages, dev64, expected_qsel_qgsum, rel_errors, to_dev
import test_gpu_protected as tp

pytestmark = pytest.mark.gpu

TOL_MAX = 2e-3
TOL_MEAN = 1e-3


@pytest.mark.parametrize("name,n_ctx", [("single_head_4k", 700), ("llama8b_b8_32k", 300),
                                        ("pipeline_128k_t4", 1000)])
@pytest.mark.parametrize("bits", [2, 4])
def test_append_bit_exact(name, n_ctx, bits):
    wl = W.workload(name, bits=bits, quant_group=128, batch=min(2, W.workload(name).batch))
    case = Case(wl, n_ctx=n_ctx)
    cache = case.gpu_cache(chunks=[n_ctx - 5, 1, 4])          # a prefill, then decode-sized appends
    check_pages(case, cache)


@pytest.mark.parametrize("sparsity", W.SWEEP_SPARSITIES)
def test_select_bit_exact(sparsity):
    wl = W.workload("llama8b_b8_32k", batch=2, quant_group=128)
    case = Case(wl, n_ctx=128)
    cache = case.gpu_cache()
    q = case.q(0)
    sel = kvq.select_channels(cache, to_dev(q, "bf16"), dev64(case.Ai), sparsity)
    k = orc.num_selected(sparsity)
    for b in range(2):
        for h in range(wl.n_kv_heads):
            qp = case.oracle_qp(q, b, h)
            ref_idx, _ = orc.select(qp, k)
            assert np.array_equal(sel.idx[b, h].cpu().numpy(), ref_idx)
            rq, rg = expected_qsel_qgsum(qp, ref_idx, group=128)
            assert np.array_equal(sel.qsel[b, h * 4:(h + 1) * 4].cpu().numpy(), rq)
            assert np.array_equal(sel.qgsum[b, h * 4:(h + 1) * 4].cpu().numpy(), rg)


def _steps(case: Case, n0: int, n_new: int, n_steps: int, fused: bool, sparsity: float = 0.4, units=None):
    wl = case.wl
    g = wl.group_size
    A, Ai = dev64(case.A), dev64(case.Ai)
    cache = kvq.new_cache(wl.batch, wl.n_kv_heads, case.capacity, wl.bits, group=128)
    kvq.append(cache, to_dev(case.K[:, :, :n0], wl.dtype), to_dev(case.V[:, :, :n0], wl.dtype), A)
    pos = n0
    us = units or [(b, h) for b in range(wl.batch) for h in range(wl.n_kv_heads)]
    for i in range(n_steps):
        q = case.q(i)
        qd = to_dev(q, wl.dtype)
        kn = to_dev(case.K[:, :, pos:pos + n_new], wl.dtype)
        vn = to_dev(case.V[:, :, pos:pos + n_new], wl.dtype)
        if fused:
            out, sel = kvq.decode_step(cache, qd, kn, vn, A, Ai, sparsity)
        else:
            kvq.append(cache, kn, vn, A)
            sel = kvq.select_channels(cache, qd, Ai, sparsity)
            out = kvq.decode_attn(cache, sel)
        torch.cuda.synchronize()
        pos += n_new
        out = out.cpu().numpy()
        for b, h in us:
            want, ref_idx, _ = case.oracle_decode(q, b, h, sparsity, pos)
            assert np.array_equal(sel.idx[b, h].cpu().numpy(), ref_idx)
            emax, emean = rel_errors(out[b, h * g:(h + 1) * g], want)
            assert emax <= TOL_MAX and emean <= TOL_MEAN, (i, b, h, emax, emean)
    assert kvq.read_status(cache) == 0 and not cache.status[1:].any()
    check_pages(case, cache, units, pos)


@pytest.mark.parametrize("fused", [True, False])
@pytest.mark.parametrize("n0,n_new", [(300, 1), (127, 1), (126, 4), (1000, 2)])
def test_decode_int2_gqa4(n0, n_new, fused):
    wl = W.workload("llama8b_b8_32k", batch=2, quant_group=128)
    case = Case(wl, n_ctx=n0 + 2 * n_new)
    _steps(case, n0, n_new, 2, fused)


@pytest.mark.parametrize("sparsity", W.SWEEP_SPARSITIES)
def test_decode_sparsities(sparsity):
    wl = W.workload("llama8b_b8_32k", batch=1, quant_group=128)
    case = Case(wl, n_ctx=900 + 1)
    _steps(case, 900, 1, 1, True, sparsity)


@pytest.mark.parametrize("bits,g", [(4, 4), (2, 2), (2, 1), (4, 8)])
def test_decode_other_shapes(bits, g):
    wl = W.workload("llama8b_b8_32k", batch=2, bits=bits, n_q_heads=8 * g, quant_group=128)
    case = Case(wl, n_ctx=600 + 1)
    _steps(case, 600, 1, 1, True)


@pytest.mark.parametrize("fused", [True, False])
def test_pages_format_with_protected_tier(fused):
    """The pages' complete format: one grid per token plus the BF16 sink and
    recent tokens."""
    wl = W.workload("llama8b_b8_32k", batch=2, quant_group=128)
    case = Case(wl, n_ctx=1000 + 2)
    tp._run(case, 1000, 1, 2, 64, 256, fused)


def test_pages_format_long_context_sampled_units():
    wl = W.workload("longctx_b1_128k", quant_group=128)
    case = Case(wl, n_ctx=6000 + 2)
    tp._run(case, 6000, 1, 2, 64, 256, True, units=[(0, 1), (0, 6)])
