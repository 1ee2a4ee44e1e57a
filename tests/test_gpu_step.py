"""GPU parity of kvq_decode_step, the whole decode step in one call.

The step must equal kvq_append + kvq_select_channels + kvq_decode_attn made
in that order: the same stored bytes and the same selection outputs; the
attention output agrees to float32 accumulation order (the one-launch kernel
runs the same page code but may split the context differently, which only
reorders float32 sums: within 1e-5 of the largest entry).  After the steps,
the pages equal the oracle's over every token appended so far and the outputs
are within the decode tolerance of the oracle's attention.
"""
import numpy as np
import pytest
import torch

from long_context_decode_dual_b200 import kvq
from long_context_decode_dual_b200 import workloads as W

from helpers import Case, check_pages, dev64, rel_errors, to_dev

pytestmark = pytest.mark.gpu

TOL_MAX = 2e-3
TOL_MEAN = 1e-3


def _prefill(case: Case, n0: int) -> kvq.KVCache:
    wl = case.wl
    cache = kvq.new_cache(wl.batch, wl.n_kv_heads, case.capacity, wl.bits)
    if n0:
        kvq.append(cache, to_dev(case.K[:, :, :n0], wl.dtype), to_dev(case.V[:, :, :n0], wl.dtype),
                   dev64(case.A))
    return cache


def _run_steps(case: Case, n0: int, n_new: int, n_steps: int, sparsity: float, units=None):
    wl = case.wl
    g = wl.group_size
    A, Ai = dev64(case.A), dev64(case.Ai)
    fused, ref = _prefill(case, n0), _prefill(case, n0)
    pos = n0
    for i in range(n_steps):
        q = case.q(i)
        qd = to_dev(q, wl.dtype)
        kn = to_dev(case.K[:, :, pos:pos + n_new], wl.dtype)
        vn = to_dev(case.V[:, :, pos:pos + n_new], wl.dtype)
        out_f, sel_f = kvq.decode_step(fused, qd, kn, vn, A, Ai, sparsity)
        kvq.append(ref, kn, vn, A)
        sel_r = kvq.select_channels(ref, qd, Ai, sparsity)
        out_r = kvq.decode_attn(ref, sel_r)
        torch.cuda.synchronize()
        pos += n_new
        assert fused.seq_len.tolist() == [pos] * wl.batch
        assert torch.equal(sel_f.idx, sel_r.idx)
        assert torch.equal(sel_f.qsel, sel_r.qsel)
        assert torch.equal(sel_f.qgsum, sel_r.qgsum)
        assert torch.equal(fused.pages, ref.pages), f"step {i}: pages differ from the three calls"
        emax, _ = rel_errors(out_f.cpu().numpy(), out_r.cpu().numpy())
        assert emax <= TOL_MAX, f"step {i}: outputs differ from the three calls by {emax}"
        us = units or [(b, h) for b in range(wl.batch) for h in range(wl.n_kv_heads)]
        out = out_f.cpu().numpy()
        for b, h in us:
            want, ref_idx, _ = case.oracle_decode(q, b, h, sparsity, pos)
            assert np.array_equal(sel_f.idx[b, h].cpu().numpy(), ref_idx)
            emax, emean = rel_errors(out[b, h * g:(h + 1) * g], want)
            assert emax <= TOL_MAX and emean <= TOL_MEAN, (i, b, h, emax, emean)
    assert kvq.read_status(fused) == 0
    assert not fused.status[1:].any()
    check_pages(case, fused, units, pos)
    return fused


@pytest.mark.parametrize("n0,n_new", [(300, 1), (127, 1), (128, 1), (255, 1), (126, 4), (381, 3), (0, 2)])
def test_step_fused_shape(n0, n_new):
    """INT2, 4 query heads per KV head: one launch per step, including new
    tokens that fill a page, open one, straddle two, or start an empty cache."""
    n_steps = 3
    wl = W.workload("llama8b_b8_32k", batch=2)
    case = Case(wl, n_ctx=n0 + n_steps * n_new)
    _run_steps(case, n0, n_new, n_steps, 0.4)


@pytest.mark.parametrize("sparsity", W.SWEEP_SPARSITIES)
def test_step_fused_sparsities(sparsity):
    wl = W.workload("llama8b_b8_32k", batch=1)
    case = Case(wl, n_ctx=700 + 2)
    _run_steps(case, 700, 1, 2, sparsity)


def test_step_fused_long_context_sampled_units():
    wl = W.workload("longctx_b1_128k")
    case = Case(wl, n_ctx=6000 + 2)
    _run_steps(case, 6000, 1, 2, 0.4, units=[(0, 0), (0, 5)])


@pytest.mark.parametrize("bits,g,n_new", [(4, 4, 1), (2, 2, 1), (2, 8, 1), (2, 4, 9)])
def test_step_other_shapes_compose_the_three_calls(bits, g, n_new):
    wl = W.workload("llama8b_b8_32k", batch=2, bits=bits, n_q_heads=8 * g)
    case = Case(wl, n_ctx=250 + 2 * n_new)
    _run_steps(case, 250, n_new, 2, 0.4)


def test_step_capacity_overflow_appends_nothing():
    """A step whose tokens do not fit raises KVQ_DEV_CAPACITY, leaves pages
    and lengths alone and attends over the stored tokens, as the three calls
    do."""
    wl = W.workload("llama8b_b8_32k", batch=2)
    case = Case(wl, n_ctx=258, capacity=256)
    A, Ai = dev64(case.A), dev64(case.Ai)
    fused, ref = _prefill(case, 255), _prefill(case, 255)
    before = fused.pages.clone()
    q = to_dev(case.q(0), "bf16")
    kn = to_dev(case.K[:, :, 255:257], "bf16")
    vn = to_dev(case.V[:, :, 255:257], "bf16")
    out_f, sel_f = kvq.decode_step(fused, q, kn, vn, A, Ai, 0.4)
    sel_r = kvq.select_channels(ref, q, Ai, 0.4)
    out_r = kvq.decode_attn(ref, sel_r)
    torch.cuda.synchronize()
    assert kvq.read_status(fused) & kvq.KVQ_DEV_CAPACITY
    assert fused.seq_len.tolist() == [255, 255]
    assert torch.equal(before, fused.pages)
    emax, _ = rel_errors(out_f.cpu().numpy(), out_r.cpu().numpy())
    assert emax <= TOL_MAX
    assert not fused.status[1:].any()
